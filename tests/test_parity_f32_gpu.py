"""fp32 CUDA path against the fp64 oracle: relative Frobenius error <= 1e-4 per
output and per final weight matrix (the fp32 bound of the layer's target)."""
import pytest

from synth_inputs import make_config, workload
from tests.parity_util import compare

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _check(errs):
    for k, v in errs.items():
        assert v <= TOL, f"{k}: relative Frobenius error {v:.3e} > {TOL}"


def test_tiny_mlp2_n196_fp32_workload():
    _check(compare(workload("tiny_mlp2_n196_fp32")))


SMALL = [
    dict(inner="linear", loss="neg_dot", opt="gd"),
    dict(inner="linear", loss="mse", opt="momentum", chunk=37),
    dict(inner="mlp2_gelu", loss="mse", opt="gd", key_instnorm=True),
    dict(inner="mlp2_gelu", loss="neg_dot", opt="momentum_muon", chunk=64, weight_l2norm=True),
    dict(inner="swiglu", loss="neg_dot", opt="momentum", chunk=50, causal=1, weight_l2norm=True),
    dict(inner="swiglu", loss="mse", opt="muon", weight_l2norm=True, key_instnorm=True),
    dict(inner="swiglu", loss="neg_dot", opt="momentum_muon", chunk=70, weight_l2norm=True, Nq=33),
    # inner epochs: repeated full-batch steps per chunk, momentum carried through them
    dict(inner="mlp2_gelu", loss="mse", opt="momentum", chunk=64, key_instnorm=True, epochs=3),
    dict(inner="swiglu", loss="neg_dot", opt="momentum", chunk=50, causal=1, weight_l2norm=True, epochs=2),
]


@pytest.mark.parametrize("kw", SMALL, ids=lambda kw: "-".join(str(v) for v in kw.values()))
def test_small_fp32_variants(kw):
    base = dict(B=2, H=3, N=161, d=24, h=40, dtype="f32", data="lact", eta_mode="per_token", seed=77)
    base.update(kw)
    _check(compare(make_config(**base)))


def test_eta_scalar_and_single_head_edge():
    _check(compare(make_config(B=1, H=1, N=1, d=8, h=8, dtype="f32", inner="mlp2_gelu", loss="mse",
                               eta_mode="scalar", eta_scalar=0.7)))

