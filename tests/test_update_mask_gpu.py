"""First-layer-only updates (the SD3.5-T5 TTT layer of "Test-Time Training vs Sleep",
Side one) on the GPU against the fp64 oracle: only the matrices that read the input
take the step; W2 must come back bit for bit equal to W0's."""
import numpy as np
import pytest

from synth_inputs import gen_inputs, make_config, matrix_shapes
from tests.parity_util import compare, run_gpu

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
