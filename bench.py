#!/usr/bin/env python
"""Throughput of the TTT-layer forward pass (weight update + apply) on B200.

One step = one ttt_forward call over one batch of the workload: every chunk's
update (inner forward on the keys, loss gradient, weight gradients, optimizer,
row norm) and the apply on the queries.  Inputs are seeded synthetic tensors of
the workload's shapes, resident in HBM before the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With N > 1 the script runs under torchrun, one process per GPU; each rank runs
its own copy of the workload (the heads of a layer are independent problems, so
the path shards with no data-path collective: weak scaling).  Rank 0 prints one
JSON line.  `--impl reference` times the fp64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from synth_inputs import WORKLOADS, gen_inputs, matrix_shapes, param_count, workload  # noqa: E402

DEFAULT_WORKLOAD = "lact_scene_n1m_c131k"
METRIC = "TTT-layer tokens/s (update+apply) and % of B200 bf16 dense tensor peak, 1 GPU"
L2_BYTES = 126 * 1024 * 1024
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# tokens per reference-arm step (bounded CPU sample) and per CPU-baseline sample
CPU_SAMPLE_TOKENS = {
    "tiny_mlp2_n196_fp32": 196, "vit3s_1248_mlp2_n6084": 6084, "lact_lm_causal_n32k_c2048": 16384,
    "lact_nvs_n196k_d512": 65536, "lact_scene_n1m_c131k": 32768, "vit3s_1248_dwconv_n6084": 8 * 6084,
    "vit3s_1248_glu_n6084": 6084,
}


# ---------------------------------------------------------------------------- work accounting
def algorithmic_flops(cfg) -> dict:
    """Algorithmic FLOPs of one forward pass per stage (2 per multiply-add; all heads)."""
    B, H, N, Nq, d, h = cfg["B"], cfg["H"], cfg["N"], cfg["Nq"], cfg["d"], cfg["h"]
    BH = B * H
    kind, loss = cfg["inner"], cfg["loss"]
    ep = max(1, int(cfg.get("epochs", 1)))  # full-batch steps per chunk
    if kind == "dwconv":  # k*k taps per (token, channel): gradient (and the MSE forward), apply
        kk = cfg["ksize"] ** 2
        return {"token_phase": 0.0, "newton_schulz": 0.0,
                "weight_grad": float(BH) * N * 2 * kk * d * (2 if loss in ("mse", "rmse") else 1) * ep,
                "apply": float(BH) * Nq * 2 * kk * d}
    if kind == "swiglu":  # token phase: Z1, Z3, V W2; weight grads: G2, G1, G3
        tok, grad, app = 6 * d * h, 6 * d * h, 6 * d * h
    elif kind == "glu":  # token phase: [Zb | Za] = X [Wb; Wa]^T; grads: [Gb; Ga] = dZ^T X; apply: Q [Wb; Wa]^T
        tok, grad, app = 4 * d * d, 4 * d * d, 4 * d * d
    elif kind == "mlp2_gelu":  # token phase: Z, [V_hat], dH; grads: G2, G1
        tok = (6 if loss in ("mse", "rmse") else 4) * d * h
        grad, app = 4 * d * h, 4 * d * h
    else:  # linear: [V_hat]; grad G
        tok, grad, app = (2 * d * d if loss in ("mse", "rmse") else 0), 2 * d * d, 2 * d * d
    chunk = cfg["chunk"] if 0 < cfg["chunk"] < N else N
    nchunks = math.ceil(N / chunk)
    ns = 0
    if cfg["opt"] in ("muon", "momentum_muon"):
        for _, r, c in matrix_shapes(cfg):
            m, n = min(r, c), max(r, c)
            ns += cfg["ns_iters"] * (4 * m * m * n + 2 * m ** 3)
    return {
        "token_phase": float(BH) * N * tok * ep,
        "weight_grad": float(BH) * N * grad * ep,
        "newton_schulz": float(BH) * nchunks * ns * ep,
        "apply": float(BH) * Nq * app,
    }


def algorithmic_bytes(cfg) -> dict:
    """HBM bytes per stage of a bandwidth-bound path (DWConv): every input read once and
    every output written once.  Tap gradients: K and V (and eta); apply: Q in, O out."""
    es = 4 if cfg["dtype"] == "f32" else 2
    BH, N, Nq, d = cfg["B"] * cfg["H"], cfg["N"], cfg["Nq"], cfg["d"]
    ep = max(1, int(cfg.get("epochs", 1)))
    eta = 4 * N if cfg["eta_mode"] == "per_token" else 0
    return {"weight_grad": float(BH) * (2 * N * d * es + eta) * ep, "apply": float(BH) * 2 * Nq * d * es}


def io_bytes(cfg) -> tuple[int, int]:
    es = 4 if cfg["dtype"] == "f32" else 2
    B, H, N, Nq, d = cfg["B"], cfg["H"], cfg["N"], cfg["Nq"], cfg["d"]
    P = param_count(cfg)
    h2d = B * H * (Nq + 2 * N) * d * es + H * P * 4 + (B * H * N * 4 if cfg["eta_mode"] == "per_token" else 0)
    d2h = B * H * Nq * d * es + B * H * P * 4
    return h2d, d2h


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources that define each timed kernel (its launch function included): a DRAM
# traffic figure recorded for a stage stays valid only while these files are unchanged.
STAGE_SOURCES = {
    "token_phase": ["token_pair.cuh", "token_phase.cuh", "epilogues.cuh", "tc_gemm.cuh", "ptx.cuh"],
    "weight_grad": ["wgrad_pair.cuh", "wgrad.cuh", "epilogues.cuh", "tc_gemm.cuh", "ptx.cuh"],
    "newton_schulz": ["ns_fused.cuh", "epilogues.cuh", "tc_gemm.cuh", "ptx.cuh"],
}


def source_digest(stage: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_sequence_mixing_b200", "csrc")
    names = STAGE_SOURCES.get(stage)
    files = ([os.path.join(csrc, n) for n in names] if names else
             sorted(glob.glob(os.path.join(csrc, "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))))
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:12]


def measured_traffic(workload_name: str, stage: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(stage)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 4 and not line.startswith("#") and parts[0] == workload_name and parts[1] == stage:
                return float(parts[3]) if parts[2] == digest else None
    return None


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        # the raw samples (the JSON line carries their summary); TTT_BENCH_OUT picks the folder
        out = os.environ.get("TTT_BENCH_OUT", os.path.join(ROOT, "bench_out"))
        self.path = os.path.join(out, f"clocks_rank{device_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx.append(float(p[2]))
                except ValueError:
                    continue
                for name, v in zip(names, p[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- CPU oracle timing
def cpu_sample_config(cfg, tokens):
    """The workload cut to its first `tokens` key/value tokens (one update), Nq scaled alike;
    a DWConv layer keeps whole grids and is cut to its first tokens // N batch entries."""
    import copy
    s = copy.deepcopy(cfg)
    if cfg["inner"] == "dwconv":
        s["B"] = max(1, min(cfg["B"], tokens // cfg["N"]))
        return s
    S = min(tokens, cfg["N"])
    s["N"] = S
    s["Nq"] = S if cfg["causal"] else max(1, round(cfg["Nq"] * S / cfg["N"]))
    if 0 < cfg["chunk"] < cfg["N"]:
        s["chunk"] = min(cfg["chunk"], S)
    return s


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("internal_api") in ("openblas", "mkl")]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(cfg, tokens, reps=1):
    import oracle
    s = cpu_sample_config(cfg, tokens)
    x = gen_inputs(s)
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        oracle.forward(s, x["Q"], x["K"], x["V"], x["eta"], x["W0"])
        times.append(time.perf_counter() - t0)
    return s, times, sample_text(cfg, s)


def sample_text(cfg, s) -> str:
    if cfg["inner"] == "dwconv":
        return (f"{s['B']} of {cfg['B']} batch entries (whole {cfg['grid_h']}x{cfg['grid_w']} grids), "
                f"fp64 numpy oracle")
    return (f"first {s['N']} of {cfg['N']} tokens of all {cfg['B'] * cfg['H']} heads, Nq {s['Nq']}, "
            f"chunk {s['chunk'] or s['N']}, fp64 numpy oracle")


# ---------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload with N cut to this many key/value tokens (profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = workload(args.workload)
    if args.tokens:
        cfg = cpu_sample_config(cfg, args.tokens)

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, cfg, world)
        return

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        from datetime import timedelta
        dist_mod.init_process_group("nccl", timeout=timedelta(seconds=120))
        dist = dist_mod

    from weight_sequence_mixing_b200 import binding

    # a dedicated stream: ttt_forward replays a cached CUDA graph of its launches on
    # any stream but the legacy default one
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    x = gen_inputs(cfg)
    dev = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    layer = binding.TTTLayer(cfg)
    O = torch.empty((cfg["B"], cfg["H"], cfg["Nq"], cfg["d"]), dtype=layer.io_dtype, device="cuda")
    W = torch.empty((cfg["B"], cfg["H"], layer.P), dtype=torch.float32, device="cuda")

    h2d, d2h = io_bytes(cfg)
    in_bytes = h2d
    flush = in_bytes < 2 * L2_BYTES
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda") if flush else None

    def step():
        layer.forward(dev["Q"], dev["K"], dev["V"], dev["eta"], dev["W0"], O=O, W_out=W, check=False)

    # The per-stage event pairs are extra graph nodes between launches (several us each),
    # so the step time is taken in a pass without them and the stage times in a second
    # pass of the same steps with them.
    layer.profile(False)
    for _ in range(args.warmup):
        step()
    layer.check_status()
    torch.cuda.synchronize()

    # ---- timed region: per-step CUDA events on the launching stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = layer.launch_count()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            if flush:
                scratch.fill_(i & 0xFF)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    launches = layer.launch_count() - launches0
    layer.check_status()

    # ---- stage pass: the same steps with an event pair around every launch inside the library
    layer.profile(True)
    for _ in range(2):  # a profiled graph keeps two instances: capture both
        step()
    torch.cuda.synchronize()
    layer.profile(True)  # clears the warm-up's stage times
    if dist:
        dist.barrier()
    for i in range(args.steps):
        if flush:
            scratch.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    stages = layer.profile_collect()
    layer.profile(False)
    layer.check_status()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), dist, "cuda")
    tokens_per_step = cfg["B"] * cfg["N"]
    value = job_throughput(world, tokens_per_step, args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    # ---- end to end through the host-buffer entry point (pinned host memory)
    e2e = run_e2e(args, cfg, layer, x, h2d, d2h, stream, dist, world)

    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return

    flops = algorithmic_flops(cfg)
    total_flops = sum(flops.values())
    # a stage with work but no launches of its own ran inside the token-phase kernel (the
    # fused MSE path of the d = 64 GELU MLP reduces its weight gradients there)
    if flops.get("weight_grad", 0) > 0 and stages.get("weight_grad", (0.0, 0))[1] == 0 and "token_phase" in stages:
        flops["token_phase"] += flops["weight_grad"]
        flops["weight_grad"] = 0.0
    peaks, peak_src = load_peaks()
    tflops = total_flops / (ms_per_step / 1e3) / 1e12
    stage_out = {}
    for name, (ms, cnt) in stages.items():
        f = flops.get(name, 0.0) * args.steps
        stage_out[name] = {"ms_per_step": ms / args.steps, "launches_per_step": cnt / args.steps,
                           "tflops": (f / (ms / 1e3) / 1e12) if (f and ms > 0) else None}
    dom = max((n for n in stages if n in flops and flops[n] > 0), key=lambda n: stages[n][0], default=None)
    clocks = clk.summary()
    # the burst peak when the SM clock stayed at its maximum through the timed region,
    # the sustained (power-capped) one when it dropped
    burst = bool(clocks) and clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"]
    peak_key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    roof = None
    if cfg["inner"] == "dwconv":  # SIMT and bandwidth-bound: the roofline is HBM, not the tensor pipe
        nbytes = algorithmic_bytes(cfg)
        dom = max((n for n in stages if nbytes.get(n, 0) > 0), key=lambda n: stages[n][0], default=None)
        if dom:
            ms, cnt = stages[dom]
            per_launch = nbytes[dom] * args.steps / cnt
            achieved = per_launch / (ms / cnt / 1e3) / 1e9
            peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
            roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": measured_traffic(args.workload, dom),
                    "bytes_per_launch": per_launch, "launches": cnt, "peak_source": f"{peak_src} HBM copy bandwidth"}
        dom = None
    if dom:
        ms, cnt = stages[dom]
        per_launch = flops[dom] * args.steps / cnt
        achieved = per_launch / (ms / cnt / 1e3) / 1e12
        peak = float(peaks.get(peak_key, peaks.get("bf16_tflops")))
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": measured_traffic(args.workload, dom),
                "flops_per_launch": per_launch, "launches": cnt,
                "peak_source": (f"{peak_src} bf16 dense " + ("burst (SM clock at its maximum in the timed region)"
                                                            if burst else "sustained (SM clock below its maximum)"))}

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        s, times, sample = time_oracle(cfg, min(cfg["N"], CPU_SAMPLE_TOKENS[args.workload]))
        cpu = {"value": s["B"] * s["N"] / times[0], "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
               "sample": sample, "seconds": times[0]}

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if cfg["dtype"] == "f32" else "bf16",
        "data": "synthetic (seeded Gaussians of the workload's shapes)",
        "config": {"workload": args.workload + (f" cut to {cfg['N']} tokens" if args.tokens else ""),
                   **{k: cfg[k] for k in ("B", "H", "N", "Nq", "d", "h", "chunk", "causal", "inner", "loss", "opt")},
                   "weight_l2norm": cfg["weight_l2norm"], "key_instnorm": cfg["key_instnorm"],
                   "l2": (f"L2 flushed between steps (256 MiB write); inputs {in_bytes / 2**20:.0f} MiB" if flush
                          else f"inputs {in_bytes / 2**20:.0f} MiB > 2x L2, no flush")},
        "tflops": tflops,
        "pct_of_bf16_peak": {"measured_sustained": 100 * tflops / float(peaks.get("bf16_tflops_sustained", 1)),
                             "measured_burst": 100 * tflops / float(peaks.get("bf16_tflops", 1)),
                             "datasheet": 100 * tflops / DATASHEET_BF16_TFLOPS, "source": peak_src},
        "roofline": roof,
        "stages": stage_out,
        "stage_timing": "CUDA event pair around every launch, in a second pass of the same steps (the step time "
                        "comes from a pass without these events)",
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "plan": dict(binding.plan_info(cfg), token_pair_capacity=binding.token_pair_capacity(cfg["inner"] == "swiglu")),
        "clocks": clocks,
        "step_ms_min_median_max": [min(step_ms), statistics.median(step_ms), max(step_ms)],
    }
    print(json.dumps(line))
    if dist:
        dist.destroy_process_group()


def max_over_ranks(ms: float, dist, device: str) -> float:
    """The slowest rank's device time: every rank takes part (MAX all-reduce)."""
    if not dist:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank runs its own replica of the workload (weak scaling),
    timed by the slowest rank."""
    return world * tokens_per_step * steps / (total_ms / 1e3)


def run_e2e(args, cfg, layer, x, h2d, d2h, stream, dist, world):
    pin = {k: (v.pin_memory() if v is not None else None) for k, v in x.items()}
    O_h = torch.empty((cfg["B"], cfg["H"], cfg["Nq"], cfg["d"]), dtype=layer.io_dtype).pin_memory()
    W_h = torch.empty((cfg["B"], cfg["H"], layer.P), dtype=torch.float32).pin_memory()
    staging = layer.staging()

    def call():
        layer.forward_host(pin["Q"], pin["K"], pin["V"], pin["eta"], pin["W0"], O_h, W_h, staging, stream=stream)

    call()
    torch.cuda.synchronize()
    layer.check_status()
    n = max(1, args.e2e_steps)
    s = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    e = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(n):
        s[i].record(stream)
        call()
        e[i].record(stream)
    torch.cuda.synchronize()
    total = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(s, e)), dist, "cuda")
    del staging
    return {"value": job_throughput(world, cfg["B"] * cfg["N"], n, total), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": total / n,
            "api": "ttt_forward_host (pinned host buffers; copies inside the timed region)"}


def run_reference(args, cfg, world):
    """The fp64 CPU oracle, as it stands, on a bounded sample per step (rank 0 only)."""
    import oracle
    # about ten full samples of CPU work in all (10-30 s each): a run of many steps times a
    # proportionally smaller sample per step, so that any --steps K --warmup W ends in minutes
    full = CPU_SAMPLE_TOKENS[args.workload]
    scale = min(1.0, 10.0 / max(1, args.steps + args.warmup))
    tokens = full if scale >= 1.0 else max(min(full, 256), int(full * scale) // 128 * 128)
    s = cpu_sample_config(cfg, tokens)
    x = gen_inputs(s)
    for _ in range(args.warmup):
        oracle.forward(s, x["Q"], x["K"], x["V"], x["eta"], x["W0"])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward(s, x["Q"], x["K"], x["V"], x["eta"], x["W0"])
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = s["B"] * s["N"] * args.steps / total
    sample = sample_text(cfg, s)
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded Gaussians of the workload's shapes)",
        "config": {"workload": args.workload, **{k: cfg[k] for k in ("B", "H", "N", "Nq", "d", "h", "chunk",
                                                                    "causal", "inner", "loss", "opt")}},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
