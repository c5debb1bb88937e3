"""DWConv inner model (the F2 module of the ViT3 design) on the GPU against the fp64
oracle: a 'same' depthwise k x k cross-correlation over the token grid whose kernels
take the layer's gradient step.  fp32 inputs within 1e-4, bf16 inputs within 2e-2
(relative Frobenius error per output and per weight tensor)."""
import pytest
import torch

from synth_inputs import gen_inputs, make_config
from tests.parity_util import compare, rel_fro, run_gpu

pytestmark = pytest.mark.gpu
TOL = {"bf16": 2e-2, "f32": 1e-4}


def _check(errs, tol):
    for k, v in errs.items():
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


CASES = [
    # the ViT3 recipe at 384^2 / patch 16: dot loss, one full-batch step, rate 1
    dict(dtype="bf16", gh=24, gw=24, d=64, loss="neg_dot", opt="gd", data="vit", eta_mode="scalar"),
    dict(dtype="f32", gh=24, gw=24, d=64, loss="neg_dot", opt="gd", data="vit", eta_mode="scalar"),
    # ragged grids, channel counts off the 128-channel groups, other kernel sizes
    dict(dtype="bf16", gh=7, gw=9, d=96, loss="mse", opt="gd", data="vit", eta_mode="scalar"),
    dict(dtype="f32", gh=7, gw=9, d=200, loss="mse", opt="momentum", epochs=3, weight_l2norm=True),
    dict(dtype="bf16", gh=1, gw=50, d=64, loss="neg_dot", opt="gd", ksize=5),
    dict(dtype="f32", gh=5, gw=6, d=32, loss="neg_dot", opt="momentum", epochs=2, ksize=7),
    dict(dtype="bf16", gh=16, gw=16, d=128, loss="mse", opt="gd", ksize=1),
    dict(dtype="f32", gh=12, gw=10, d=64, loss="neg_dot", opt="gd", no_update=True),
]


@pytest.mark.parametrize("kw", CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_dwconv_against_the_oracle(kw):
    kw = dict(kw)
    gh, gw = kw.pop("gh"), kw.pop("gw")
    base = dict(B=2, H=2, N=gh * gw, grid_h=gh, grid_w=gw, inner="dwconv", data="lact", eta_mode="per_token",
                seed=97)
    base.update(kw)
    cfg = make_config(**base)
    _check(compare(cfg), TOL[cfg["dtype"]])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dwconv_state_handed_on_equals_more_epochs(dtype):
    # two calls of one step each, (W, M) handed on, equal one call of two steps
    from weight_sequence_mixing_b200 import binding

    base = dict(B=2, H=2, N=80, grid_h=8, grid_w=10, d=64, inner="dwconv", loss="neg_dot", opt="momentum",
                weight_l2norm=True, dtype=dtype, data="lact", eta_mode="per_token", seed=101)
    x = gen_inputs(make_config(**base))
    O2, W2 = run_gpu(make_config(epochs=2, **base), x)
    dev = lambda t: t.contiguous().cuda()
    first = binding.TTTLayer(make_config(**base))
    second = binding.TTTLayer(make_config(w0_per_batch=True, **base))
    state = first.new_state()
    _, Wa = first.forward_state(dev(x["Q"]), dev(x["K"]), dev(x["V"]), dev(x["eta"]), dev(x["W0"]),
                                state_out=state)
    Ob, Wb = second.forward_state(dev(x["Q"]), dev(x["K"]), dev(x["V"]), dev(x["eta"]), Wa, state_in=state,
                                  state_out=state)
    torch.cuda.synchronize()
    assert rel_fro(Wb.double().cpu().numpy(), W2) < 1e-6
    assert rel_fro(Ob.double().cpu().numpy(), O2) < 1e-5
    first.close()
    second.close()
