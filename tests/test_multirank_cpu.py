"""The multi-process path of bench.py on CPU: world size 2 over gloo (replicas only, so the
only collectives are the barrier and the MAX reduction of the timed region), and the
reference arm under torchrun-style environments."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    dist.barrier()
    slowest = bench.max_over_ranks(10.0 * (rank + 1), dist, "cpu")
    value = bench.job_throughput(world, 1000, 10, slowest)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, slowest, value))


def test_max_over_ranks_and_weak_scaling_value_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slower rank's 20 ms; 2 replicas x 1000 tokens x 10 steps in 20 ms
    assert [r[1] for r in res] == [20.0, 20.0]
    assert all(abs(r[2] - 2 * 1000 * 10 / 0.02) < 1e-6 for r in res)


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.job_throughput(1, 196608, 100, 250.0) == pytest.approx(196608 * 100 / 0.25)


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                           "tiny_mlp2_n196_fp32", "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_other_ranks_exit_without_work():
    r = _run_reference(1, 2)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_json_line():
    r = _run_reference(0, 2)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
