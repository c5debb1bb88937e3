"""Host-side planning (ttt_create, no GPU): the chunking and the weight-gradient
decomposition chosen for each workload, and the invariants of the split heuristic."""
import itertools

import pytest

from synth_inputs import make_config, workload

binding = pytest.importorskip("weight_sequence_mixing_b200.binding")

EXPECTED = {
    # fp32 SIMT path: one chunk of 196 tokens
    "tiny_mlp2_n196_fp32": dict(path=0, chunk=196, nchunks=1),
    # d = 64 GELU MLP with the MSE loss: token phase and gradients in one kernel, one CTA
    # per (head, third of the 48 token tiles): 144 CTAs, 3 split partials per head
    "vit3s_1248_mlp2_n6084": dict(path=1, chunk=6084, nchunks=1, splits=3, tile_rows=128, grad_bn=64, direct=0),
    # 2048-token chunks are not split: gradients go straight into U and the momentum;
    # 128-column tiles give the 96 CTAs the 256-column tiles would halve
    "lact_lm_causal_n32k_c2048": dict(path=1, chunk=2048, nchunks=16, splits=1, tile_rows=128, grad_bn=128,
                                      direct=1),
    # one 196608-token chunk: 512-row pair tiles (24 of them), 3 splits (72 pair tiles: one
    # wave of the 74 pairs)
    "lact_nvs_n196k_d512": dict(path=1, chunk=196608, nchunks=1, splits=3, tile_rows=512, grad_bn=256, direct=0),
    # 8 chunks of 131072 (the last one 111616): 12 pair tiles x 6 splits, one wave
    "lact_scene_n1m_c131k": dict(path=1, chunk=131072, nchunks=8, splits=6, tile_rows=512, grad_bn=256, direct=0),
}


@pytest.mark.parametrize("name", list(EXPECTED))
def test_workload_plans(name):
    got = binding.plan_info(workload(name))
    for k, v in EXPECTED[name].items():
        assert got[k] == v, f"{name}: {k} = {got[k]}, expected {v}"


def test_single_cta_flag_keeps_gradient_tiles_on_single_ctas():
    got = binding.plan_info(workload("lact_nvs_n196k_d512", single_cta=True))
    assert got["tile_rows"] == 256 and got["splits"] == 6
    # pair tiles split only as far as one wave of the 74 CTA pairs holds
    for name in ("lact_nvs_n196k_d512", "lact_scene_n1m_c131k"):
        cfg = workload(name)
        info = binding.plan_info(cfg)
        tiles = 3 * cfg["h"] // 512 * (cfg["d"] // info["grad_bn"]) * cfg["B"] * cfg["H"]
        assert info["tile_rows"] == 512 and tiles * info["splits"] <= 74 < tiles * (info["splits"] + 1)


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


# ---------------------------------------------------------------- random configurations
# Any configuration, valid or not, gets a defined status from ttt_create (host only), and
# an accepted one has sizes that agree with their definitions.
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

_INNER = ["linear", "mlp2_gelu", "swiglu", "dwconv"]


@st.composite
def _configs(draw):
    inner = draw(st.sampled_from(_INNER))
    dtype = draw(st.sampled_from(["f32", "bf16"]))
    d = draw(st.sampled_from([1, 8, 24, 64, 96, 128, 256, 512]))
    h = draw(st.sampled_from([1, 40, 128, 256, 384, 1024]))
    N = draw(st.one_of(st.integers(1, 1 << 20), st.integers((1 << 30) - 300, (1 << 31) - 1)))
    kw = dict(B=draw(st.integers(1, 8)), H=draw(st.integers(1, 8)), N=N, d=d, h=h, inner=inner, dtype=dtype,
              loss=draw(st.sampled_from(["mse", "neg_dot", "rmse"])),
              opt=draw(st.sampled_from(["gd", "momentum", "muon", "momentum_muon"])),
              chunk=draw(st.sampled_from([0, 1, 64, 100, 2048, N, N + 5])),
              causal=draw(st.sampled_from([0, 1])),
              weight_l2norm=draw(st.booleans()), key_instnorm=draw(st.booleans()),
              w0_per_batch=draw(st.booleans()), epochs=draw(st.integers(0, 3)))
    kw["Nq"] = N if kw["causal"] or inner == "dwconv" else draw(st.integers(1, 5000))
    if inner == "dwconv":
        gh = draw(st.integers(1, 64))
        kw.update(N=gh * draw(st.integers(1, 64)), grid_h=gh, ksize=draw(st.sampled_from([1, 2, 3, 5, 7, 9])))
        kw["grid_w"] = kw["N"] // gh
        kw["Nq"] = kw["N"]
        kw["chunk"] = draw(st.sampled_from([0, kw["N"], 7]))
    return make_config(**kw)


@settings(max_examples=300, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(_configs())
def test_random_configurations_get_a_status_and_consistent_sizes(cfg):
    import ctypes

    c = binding.make_config(cfg)
    h = ctypes.c_void_p()
    st_ = binding.LIB.ttt_create(ctypes.byref(c), ctypes.byref(h))
    assert st_ in (binding.TTT_OK, binding.TTT_ERR_INVALID_ARG, binding.TTT_ERR_UNSUPPORTED)
    if max(cfg["N"], cfg["Nq"]) > (1 << 30):
        assert st_ != binding.TTT_OK
    if st_ != binding.TTT_OK:
        assert not h.value
        return
    try:
        d, hh, k = cfg["d"], cfg["h"], cfg["ksize"]
        P = {"linear": d * d, "mlp2_gelu": 2 * d * hh, "swiglu": 3 * d * hh, "dwconv": d * k * k}[cfg["inner"]]
        assert binding.LIB.ttt_param_count(h) == P
        Z = cfg["B"] * cfg["H"]
        mom = cfg["opt"] in ("momentum", "momentum_muon")
        state = binding.LIB.ttt_state_size(h)
        assert (state > 0) == mom and state % 4 == 0 and (state == 0 or state >= Z * P * 4)
        es = 4 if cfg["dtype"] == "f32" else 2
        io = (2 * Z * cfg["Nq"] * d * es + 2 * Z * cfg["N"] * d * es + Z * cfg["N"] * 4
              + (Z if cfg["w0_per_batch"] else cfg["H"]) * P * 4 + Z * P * 4)
        assert binding.LIB.ttt_host_staging_size(h) >= io
        assert binding.LIB.ttt_workspace_size(h) >= 256 + Z * P * 4
        buf = (ctypes.c_int * len(binding.PLAN_FIELDS))()
        binding.LIB.ttt_plan_info(h, buf, len(binding.PLAN_FIELDS))
        info = dict(zip(binding.PLAN_FIELDS, buf))
        N, chunk = cfg["N"], cfg["chunk"]
        assert info["chunk"] == (N if chunk <= 0 or chunk >= N else chunk)
        assert info["nchunks"] == -(-N // info["chunk"])
        assert info["path"] == (2 if cfg["inner"] == "dwconv" else 0 if cfg["dtype"] == "f32" else 1)
        if info["path"] == 1:
            assert info["splits"] >= 1 and info["tile_rows"] in (128, 256, 512) and info["grad_bn"] in (32, 64, 128, 256)
    finally:
        binding.LIB.ttt_destroy(h)


@pytest.mark.parametrize("kw,status", [
    (dict(dtype="bf16"), 0),
    (dict(dtype="bf16", loss="mse", opt="momentum", chunk=256, causal=1), 0),
    (dict(dtype="f32"), -2),                   # the fp32 path runs the GLU in its SwiGLU form
    (dict(dtype="bf16", opt="muon"), -2),
    (dict(dtype="bf16", opt="momentum_muon"), -2),
    (dict(dtype="bf16", loss="rmse"), -2),
    (dict(dtype="bf16", d=96), -2),            # channels in whole 64-channel blocks
])
def test_glu_combinations(kw, status):
    import ctypes
    base = dict(B=1, H=2, N=1024, d=128, h=7, inner="glu", loss="neg_dot", opt="gd")
    base.update(kw)
    cfg = make_config(**base)
    c = binding.make_config(cfg)
    h = ctypes.c_void_p()
    st = binding.LIB.ttt_create(ctypes.byref(c), ctypes.byref(h))
    assert st == status, binding.status_string(st)
    if st == 0:
        # two d x d matrices (h is ignored), 64-channel blocks of gate and linear rows
        assert binding.LIB.ttt_param_count(h) == 2 * cfg["d"] ** 2
        binding.LIB.ttt_destroy(h)


@pytest.mark.parametrize("B,H,N,chunk,h", [(8, 6, 6084, 0, 256), (1, 1, 300, 0, 128), (2, 2, 700, 512, 256),
                                           (1, 200, 1000, 0, 256), (4, 1, 65536, 0, 128)])
def test_fused_mse_plan(B, H, N, chunk, h):
    # one CTA per (head, token-tile range): at most one wave of 148 CTAs, every range at
    # least one tile of a full chunk, split partials always reduced (never direct)
    cfg = make_config(B=B, H=H, N=N, chunk=chunk, d=64, h=h, inner="mlp2_gelu", loss="mse", opt="gd",
                      dtype="bf16")
    got = binding.plan_info(cfg)
    tiles = -(-got["chunk"] // 128)
    assert got["direct"] == 0 and got["tile_rows"] == 128
    assert got["splits"] == max(1, min(tiles, 148 // (B * H)))


@pytest.mark.parametrize("B,H,N,chunk,loss", [(8, 5, 6084, 0, "neg_dot"), (2, 2, 700, 512, "mse"), (1, 1, 300, 0, "neg_dot")])
def test_fused_glu_plan(B, H, N, chunk, loss):
    # d = 64 GLU: token GEMM, gating gradient and gradient reduction in one kernel, one CTA
    # per (head, token-tile range), split partials summed by the row finish
    cfg = make_config(B=B, H=H, N=N, chunk=chunk, d=64, h=64, inner="glu", loss=loss, opt="gd", dtype="bf16")
    got = binding.plan_info(cfg)
    tiles = -(-got["chunk"] // 128)
    assert got["direct"] == 0 and got["splits"] == max(1, min(tiles, 148 // (B * H)))
