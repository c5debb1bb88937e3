"""bf16 tensor-core CUDA path against the fp64 oracle.

Gate: relative Frobenius error <= 2e-2 per output and per final weight matrix
(the bf16-input / fp32-accumulate bound of the layer's target).  The change
of the weights, W* - W0, is also compared (a looser diagnostic bound), since a
small update hides inside W* when ||W* - W0|| << ||W0||.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import gen_inputs, make_config, matrix_shapes, workload
from weight_sequence_mixing_b200 import binding
from tests.parity_util import compare, rel_fro, run_gpu

pytestmark = pytest.mark.gpu
TOL = 2e-2
DW_TOL = 5e-2


def _check(errs, tol=TOL):
    for k, v in errs.items():
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


def _delta_w_check(cfg, x, heads=None):
    Og, Wg = run_gpu(cfg, x)
    Or, Wr = orc.forward(cfg, x["Q"], x["K"], x["V"], x["eta"], x["W0"], heads=heads)
    sel = heads or [(b, h) for b in range(cfg["B"]) for h in range(cfg["H"])]
    W0 = x["W0"].double().numpy()
    out = {"O": max(rel_fro(Og[b, h], Or[b, h]) for b, h in sel)}
    off = 0
    for name, r, c in matrix_shapes(cfg):
        sl = slice(off, off + r * c)
        out[name] = max(rel_fro(Wg[b, h, sl], Wr[b, h, sl]) for b, h in sel)
        if not cfg["weight_l2norm"]:
            out["d" + name] = max(rel_fro(Wg[b, h, sl] - W0[h, sl], Wr[b, h, sl] - W0[h, sl]) for b, h in sel)
        off += r * c
    return out


SMALL = [
    dict(inner="swiglu", loss="neg_dot", opt="gd", d=128, h=256, N=300),
    dict(inner="swiglu", loss="neg_dot", opt="momentum", d=128, h=128, N=450, chunk=128, causal=1, weight_l2norm=True),
    dict(inner="swiglu", loss="neg_dot", opt="muon", d=128, h=256, N=384, weight_l2norm=True),
    dict(inner="swiglu", loss="neg_dot", opt="momentum_muon", d=128, h=256, N=700, chunk=256, Nq=200,
         weight_l2norm=True),
    dict(inner="swiglu", loss="neg_dot", opt="gd", d=256, h=512, N=520, Nq=130, eta_mode="scalar",
         eta_scalar=0.002),
    dict(inner="mlp2_gelu", loss="mse", opt="gd", d=64, h=256, N=700, key_instnorm=True, data="vit",
         eta_mode="scalar", eta_scalar=1.0),
    dict(inner="mlp2_gelu", loss="mse", opt="momentum", d=64, h=128, N=333, chunk=128, key_instnorm=True,
         data="vit", eta_mode="scalar"),
    # fused MSE kernel: 4 tile ranges per head, the last chunk's 2 tiles leave two ranges empty
    dict(inner="mlp2_gelu", loss="mse", opt="momentum", d=64, h=256, N=700, chunk=512, key_instnorm=True,
         data="vit"),
    dict(inner="mlp2_gelu", loss="neg_dot", opt="momentum", d=128, h=256, N=400, chunk=256, weight_l2norm=True),
    dict(inner="linear", loss="neg_dot", opt="gd", d=128, h=128, N=260),
    dict(inner="linear", loss="mse", opt="momentum_muon", d=128, h=128, N=390, chunk=128, weight_l2norm=True),
    # inner epochs: repeated full-batch steps per chunk, momentum carried through them
    dict(inner="swiglu", loss="neg_dot", opt="momentum_muon", d=128, h=256, N=700, chunk=256, Nq=200,
         weight_l2norm=True, epochs=2),
    dict(inner="mlp2_gelu", loss="mse", opt="gd", d=64, h=256, N=700, key_instnorm=True, data="vit",
         eta_mode="scalar", eta_scalar=1.0, epochs=3),
    # split-K partials with momentum: reduced by their own pass (models with W2), or summed by
    # the row finish (linear, GLU)
    dict(inner="swiglu", loss="neg_dot", opt="momentum", d=128, h=256, N=6000, weight_l2norm=True),
    dict(inner="mlp2_gelu", loss="neg_dot", opt="momentum", d=128, h=256, N=6000, chunk=4608, epochs=2),
    dict(inner="linear", loss="neg_dot", opt="momentum", d=128, h=128, N=6000, weight_l2norm=True),
    dict(inner="glu", loss="mse", opt="momentum", d=64, h=64, N=6000, chunk=4608, data="vit", eta_mode="scalar",
         eta_scalar=1.0, epochs=2),
]


@pytest.mark.parametrize("kw", SMALL, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_small_bf16_variants(kw):
    base = dict(B=2, H=2, dtype="bf16", data="lact", eta_mode="per_token", seed=91)
    base.update(kw)
    cfg = make_config(**base)
    errs = _delta_w_check(cfg, gen_inputs(cfg))
    for k, v in errs.items():
        tol = DW_TOL if k.startswith("d") else TOL
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


# Token phase and weight gradients on single CTAs instead of CTA pairs: both
# against the oracle, and against each other.  Token counts leave a ragged last
# pair tile (N = 300: 384 padded rows, the second pair tile's upper half lies past
# the activation buffers) and several pair tiles per CTA pair.
TOKEN_KERNEL_CASES = [
    dict(inner="swiglu", d=128, h=256, N=300),
    dict(inner="swiglu", d=256, h=512, N=1200, chunk=640, opt="momentum", weight_l2norm=True),
    dict(inner="swiglu", d=512, h=256, N=520, opt="muon", weight_l2norm=True),
    dict(inner="mlp2_gelu", d=128, h=384, N=700, chunk=384),
    # enough k-blocks for split weight gradients on 512-row pair tiles (rows 3h = 1536)
    dict(inner="swiglu", d=256, h=512, N=8192, opt="momentum_muon", weight_l2norm=True),
    # enough token tiles per pair for resident weight blocks: the pairs' token-tile ranges
    # cross from one head into the next (a weight reload) and end on a ragged tile
    dict(inner="swiglu", d=256, h=512, N=5000, opt="momentum", weight_l2norm=True),
    dict(inner="mlp2_gelu", d=128, h=256, N=9800),
]


def test_token_pair_kernel_is_resident():
    # the pair kernel must fit an SM pair (registers x threads, shared memory), or the
    # token phase silently runs on single CTAs
    from weight_sequence_mixing_b200 import binding

    assert binding.token_pair_capacity(True) >= 64
    assert binding.token_pair_capacity(False) >= 64


@pytest.mark.parametrize("kw", TOKEN_KERNEL_CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_token_kernels_pair_and_single_cta(kw):
    base = dict(B=2, H=2, dtype="bf16", data="lact", eta_mode="per_token", loss="neg_dot", opt="gd", seed=17)
    base.update(kw)
    x = gen_inputs(make_config(**base))
    for single in (False, True):
        cfg = make_config(single_cta=single, **base)
        errs = _delta_w_check(cfg, x)
        for k, v in errs.items():
            tol = DW_TOL if k.startswith("d") else TOL
            assert v <= tol, f"single={single} {k}: relative Frobenius error {v:.3e} > {tol}"
    Op, Wp = run_gpu(make_config(**base), x)
    Os, Ws = run_gpu(make_config(single_cta=True, **base), x)
    # With the same split-K count the two kernels round the same fp32 accumulators to
    # bf16: near-identical results.  With different counts the gradient sums run in another
    # order, and Muon's Newton-Schulz map (slope about 3.4 per step near a zero singular
    # value) magnifies that rounding noise in the weak directions: a looser bound.
    same = binding.plan_info(make_config(**base))["splits"] == \
        binding.plan_info(make_config(single_cta=True, **base))["splits"]
    muon = base["opt"] in ("muon", "momentum_muon")
    near = 1e-3 if same or not muon else 1e-2
    assert rel_fro(Op, Os) < near and rel_fro(Wp, Ws) < near


def test_causal_chunk_n_equals_single_chunk_weights_on_gpu():
    # apply-before-update with one chunk: W* equals the non-causal single chunk's,
    # and O reads the initial weights (the non-causal eta = 0 output).
    kw = dict(B=1, H=2, N=256, d=128, h=128, inner="swiglu", loss="neg_dot", opt="momentum", dtype="bf16",
              weight_l2norm=False, data="lact", eta_mode="per_token", seed=5)
    x = gen_inputs(make_config(**kw))
    Oc, Wc = run_gpu(make_config(chunk=256, causal=1, **kw), x)
    On, Wn = run_gpu(make_config(chunk=0, causal=0, **kw), x)
    assert rel_fro(Wc, Wn) < 1e-6
    x0 = dict(x)
    x0["eta"] = torch.zeros_like(x["eta"])
    O0, _ = run_gpu(make_config(chunk=0, causal=0, **kw), x0)
    assert rel_fro(Oc, O0) < 1e-6


# ---------------------------------------------------------------- full-size workloads
# every (batch, head) of every workload; the million-token scene layer's four heads
# take the oracle about a minute each
FULL = ["vit3s_1248_mlp2_n6084", "lact_lm_causal_n32k_c2048", "lact_nvs_n196k_d512", "lact_scene_n1m_c131k"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    cfg = workload(name)
    errs = compare(cfg)
    # the whole layer and, with the _worst_head keys, its worst single (batch, head)
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})
    _check(errs)


def test_vit3s_full_size_weight_change():
    # In the ViT-S layer one step moves W* by about 3% of W0, so the W* gate alone
    # would pass a badly wrong update: compare the change W* - W0 itself (every head).
    cfg = workload("vit3s_1248_mlp2_n6084")
    assert not cfg["weight_l2norm"]
    errs = _delta_w_check(cfg, gen_inputs(cfg))
    print({k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        tol = DW_TOL if k.startswith("d") else TOL
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


@pytest.mark.parametrize("profiled,causal", [(False, 0), (True, 0), (False, 1), (True, 1)])
def test_graph_replay_matches_direct_launch(profiled, causal):
    # on a non-default stream ttt_forward captures its launches into a CUDA graph on the
    # first call and replays it afterwards (two alternating instances when profiling);
    # every replay must give the bits the direct launches give.  Causal: each chunk's apply
    # runs on the handle's second stream, forked and joined inside the graph too.
    from weight_sequence_mixing_b200 import binding
    kw = dict(B=1, H=2, N=640, chunk=256, Nq=640 if causal else 300, causal=causal, d=128, h=256,
              inner="swiglu", loss="neg_dot", opt="momentum_muon", weight_l2norm=True, dtype="bf16", data="lact",
              eta_mode="per_token", seed=8)
    x = gen_inputs(make_config(**kw))
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    direct = binding.TTTLayer(make_config(direct_launch=True, **kw))
    O0, W0 = direct.forward(d["Q"], d["K"], d["V"], d["eta"], d["W0"])
    side = torch.cuda.Stream()
    layer = binding.TTTLayer(make_config(**kw))
    if profiled:
        layer.profile(True)
    O = torch.empty_like(O0)
    W = torch.empty_like(W0)
    with torch.cuda.stream(side):
        for _ in range(4):
            O.fill_(float("nan"))
            layer.forward(d["Q"], d["K"], d["V"], d["eta"], d["W0"], O=O, W_out=W, stream=side)
            assert torch.equal(O, O0) and torch.equal(W, W0)
    side.synchronize()
    if profiled:
        stages = layer.profile_collect()
        assert stages["token_phase"][1] == 4 * 3 and stages["newton_schulz"][1] > 0
        assert all(ms > 0 for ms, _ in stages.values())
