"""First-layer-only updates and the simplified GLU inner model on the GPU, against the
fp64 oracle.

* First-layer-only (the SD3.5-T5 TTT layer of "Test-Time Training vs Sleep", Side
  one): only the matrices that read the input take the step; W2 must come back
  bit for bit equal to W0's.
* The simplified GLU FC(x) * SiLU(FC(x)) of the ViT3 digest (section 03, inner-model
  table) runs as a SwiGLU with h = d, W1 = the gate's matrix Wb, W3 = the linear
  branch's Wa, W2 = I and the first-layer-only flag; it is checked against the
  oracle's own GLU model, with the ViT3 recipe (dot loss, one full-batch step,
  learning rate 1) and with momentum + Muon over several chunks.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import gen_inputs, make_config, matrix_shapes
from tests.parity_util import compare, rel_fro, run_gpu

pytestmark = pytest.mark.gpu
TOL = {"bf16": 2e-2, "f32": 1e-4}


def _check(errs, tol):
    for k, v in errs.items():
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


def _w2_slice(cfg):
    off = 0
    for name, r, c in matrix_shapes(cfg):
        if name == "W2":
            return slice(off, off + r * c)
        off += r * c
    return None


FIRST_LAYER_CASES = [
    dict(dtype="bf16", inner="mlp2_gelu", loss="mse", opt="gd", d=64, h=256, N=700, key_instnorm=True, data="vit",
         eta_mode="scalar"),
    dict(dtype="bf16", inner="mlp2_gelu", loss="neg_dot", opt="momentum", d=128, h=256, N=400, chunk=256, causal=1,
         weight_l2norm=True),
    dict(dtype="bf16", inner="swiglu", loss="neg_dot", opt="momentum_muon", d=128, h=256, N=700, chunk=256, Nq=200,
         weight_l2norm=True),
    dict(dtype="f32", inner="mlp2_gelu", loss="mse", opt="gd", d=24, h=40, N=96, key_instnorm=True, data="vit",
         eta_mode="scalar"),
    dict(dtype="f32", inner="swiglu", loss="neg_dot", opt="momentum_muon", d=24, h=40, N=96, chunk=32,
         weight_l2norm=True),
]


@pytest.mark.parametrize("kw", FIRST_LAYER_CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_first_layer_only_against_the_oracle(kw):
    base = dict(B=2, H=2, data="lact", eta_mode="per_token", seed=71, first_layer_only=True)
    base.update(kw)
    cfg = make_config(**base)
    x = gen_inputs(cfg)
    _check(compare(cfg, x), TOL[cfg["dtype"]])
    _, W = run_gpu(cfg, x)
    sl = _w2_slice(cfg)
    W0 = x["W0"].double().numpy()
    for b in range(cfg["B"]):
        assert np.array_equal(W[b, :, sl], W0[:, sl])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_first_layer_only_changes_nothing_for_the_linear_model(dtype):
    d = 128 if dtype == "bf16" else 24
    base = dict(B=2, H=2, N=300, d=d, h=d, inner="linear", loss="neg_dot", opt="momentum", chunk=128,
                weight_l2norm=True, dtype=dtype, data="lact", eta_mode="per_token", seed=73)
    x = gen_inputs(make_config(**base))
    Oa, Wa = run_gpu(make_config(**base), x)
    Ob, Wb = run_gpu(make_config(first_layer_only=True, **base), x)
    assert np.array_equal(Oa, Ob) and np.array_equal(Wa, Wb)


GLU_CASES = [
    # the ViT3 recipe: dot loss, one full-batch step, learning rate 1
    dict(dtype="bf16", d=128, N=600, opt="gd", eta_mode="scalar", eta_scalar=1.0),
    dict(dtype="bf16", d=128, N=600, opt="gd", eta_mode="scalar", eta_scalar=1.0, data="vit"),
    dict(dtype="bf16", d=256, N=1000, opt="momentum", chunk=384, weight_l2norm=True, eta_mode="per_token"),
    dict(dtype="bf16", d=128, N=700, Nq=200, opt="momentum_muon", chunk=256, weight_l2norm=True,
         eta_mode="per_token"),
    dict(dtype="bf16", d=128, N=450, opt="momentum", chunk=128, causal=1, weight_l2norm=True,
         eta_mode="per_token"),
    dict(dtype="f32", d=24, N=96, opt="gd", eta_mode="scalar", eta_scalar=1.0),
    dict(dtype="f32", d=24, N=96, opt="momentum_muon", chunk=40, weight_l2norm=True, eta_mode="per_token"),
]


@pytest.mark.parametrize("kw", GLU_CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_glu_as_swiglu_against_the_oracle_glu(kw):
    base = dict(B=2, H=2, inner="swiglu", loss="neg_dot", data="lact", seed=79, first_layer_only=True)
    base.update(kw)
    base["h"] = base["d"]
    cfg = make_config(**base)
    d, P = cfg["d"], cfg["d"] * cfg["d"]
    x = gen_inputs(cfg)
    # W0 = [W1 = Wb | W3 = Wa | W2 = I]; the oracle's GLU takes [Wa | Wb]
    W0 = x["W0"].clone()
    W0[:, 2 * P:] = torch.eye(d).reshape(-1)
    x["W0"] = W0.contiguous()
    W0_glu = torch.cat([W0[:, P:2 * P], W0[:, :P]], dim=1)
    cfg_glu = dict(cfg, inner="glu", first_layer_only=False)
    Or, Wr = orc.forward(cfg_glu, x["Q"], x["K"], x["V"], x["eta"], W0_glu)
    Og, Wg = run_gpu(cfg, x)
    tol = TOL[cfg["dtype"]]
    errs = {"O": rel_fro(Og, Or), "Wb (W1)": rel_fro(Wg[..., :P], Wr[..., P:]),
            "Wa (W3)": rel_fro(Wg[..., P:2 * P], Wr[..., :P])}
    _check(errs, tol)
    assert np.isfinite(Og).all()
    assert np.array_equal(Wg[..., 2 * P:], np.broadcast_to(np.eye(d).reshape(-1), Wg[..., 2 * P:].shape))
