"""Host-side planning (ttt_create, no GPU): the chunking and the weight-gradient
decomposition chosen for each workload, and the invariants of the split heuristic."""
import itertools

import pytest

from synth_inputs import make_config, workload

binding = pytest.importorskip("weight_sequence_mixing_b200.binding")

EXPECTED = {
    # fp32 SIMT path: one chunk of 196 tokens
    "tiny_mlp2_n196_fp32": dict(path=0, chunk=196, nchunks=1),
    # d = 64: 256-row single-CTA tiles of 64 columns, 3 splits of 2048 tokens
    "vit3s_1248_mlp2_n6084": dict(path=1, chunk=6084, nchunks=1, splits=3, tile_rows=256, grad_bn=64, direct=0),
    # 2048-token chunks are not split: gradients go straight into U and the momentum;
    # 128-column tiles give the 96 CTAs the 256-column tiles would halve
    "lact_lm_causal_n32k_c2048": dict(path=1, chunk=2048, nchunks=16, splits=1, tile_rows=128, grad_bn=128,
                                      direct=1),
    # one 196608-token chunk: 512-row pair tiles (24 of them), 6 splits (144 pair tiles)
    "lact_nvs_n196k_d512": dict(path=1, chunk=196608, nchunks=1, splits=6, tile_rows=512, grad_bn=256, direct=0),
    # 8 chunks of 131072 (the last one 111616): 12 pair tiles x 12 splits
    "lact_scene_n1m_c131k": dict(path=1, chunk=131072, nchunks=8, splits=12, tile_rows=512, grad_bn=256, direct=0),
}


@pytest.mark.parametrize("name", list(EXPECTED))
def test_workload_plans(name):
    got = binding.plan_info(workload(name))
    for k, v in EXPECTED[name].items():
        assert got[k] == v, f"{name}: {k} = {got[k]}, expected {v}"


def test_single_cta_flag_keeps_gradient_tiles_on_single_ctas():
    got = binding.plan_info(workload("lact_nvs_n196k_d512", single_cta=True))
    assert got["tile_rows"] == 256 and got["splits"] == 6


CASES = list(itertools.product([128, 256, 512], [128, 256, 1024], [1024, 4096, 8192, 65536], ["gd", "momentum", "muon"]))


@pytest.mark.parametrize("d,h,n,opt", CASES, ids=lambda v: str(v))
def test_split_heuristic_invariants(d, h, n, opt):
    cfg = make_config(B=1, H=2, N=n, d=d, h=h, inner="swiglu", loss="neg_dot", opt=opt, dtype="bf16")
    got = binding.plan_info(cfg)
    kblocks = (got["chunk"] + 127) // 128 * 128 // 64
    assert 1 <= got["splits"] <= 64
    if got["chunk"] <= 4096:
        assert got["splits"] == 1  # short chunks are never split
    if got["splits"] > 1:
        per = -(-kblocks // got["splits"])
        assert per >= 16  # at least 1024 tokens per split
        assert (got["splits"] - 1) * per < kblocks  # every split owns k-blocks
    assert got["tile_rows"] in (128, 256, 512)
    assert d % got["grad_bn"] == 0
    if got["tile_rows"] == 512:
        assert h % 512 == 0 and got["grad_bn"] in (128, 256)
    # with Muon the row norms are summed over at most two column tiles of a row
    if opt == "muon" and got["direct"]:
        assert got["grad_bn"] == d
    assert got["direct"] == (1 if got["splits"] == 1 and not (opt == "muon" and got["grad_bn"] != d) else 0)


def _sizes(cfg):
    import ctypes
    c = binding.make_config(cfg)
    h = ctypes.c_void_p()
    assert binding.LIB.ttt_create(ctypes.byref(c), ctypes.byref(h)) == 0
    try:
        return int(binding.LIB.ttt_workspace_size(h)), int(binding.LIB.ttt_host_staging_size(h)), \
            int(binding.LIB.ttt_param_count(h))
    finally:
        binding.LIB.ttt_destroy(h)


def _up(x, a=256):
    return (x + a - 1) // a * a


@pytest.mark.parametrize("per_batch", [False, True])
def test_host_staging_holds_every_input_and_output(per_batch):
    cfg = make_config(B=2, H=3, N=300, Nq=200, d=64, h=128, inner="swiglu", loss="neg_dot", dtype="bf16",
                      eta_mode="per_token", w0_per_batch=per_batch)
    _, staging, P = _sizes(cfg)
    BH = 2 * 3
    expect = (_up(BH * 200 * 64 * 2) + 2 * _up(BH * 300 * 64 * 2) + _up(BH * 300 * 4)
              + _up((BH if per_batch else 3) * P * 4) + _up(BH * 200 * 64 * 2) + _up(BH * P * 4))
    assert staging == expect


def test_workspace_grows_with_the_chunk_and_fits_the_static_scratch_when_small():
    small_ws, _, _ = _sizes(workload("tiny_mlp2_n196_fp32"))
    big_ws, _, _ = _sizes(workload("lact_nvs_n196k_d512"))
    assert small_ws <= 32 * 1024 * 1024 < big_ws  # the no-allocation entry takes the first only
    a, _, _ = _sizes(make_config(B=1, H=2, N=4096, d=128, h=256, inner="swiglu", loss="neg_dot", dtype="bf16"))
    b, _, _ = _sizes(make_config(B=1, H=2, N=8192, d=128, h=256, inner="swiglu", loss="neg_dot", dtype="bf16"))
    assert b > a
