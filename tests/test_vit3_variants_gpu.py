"""Inner models and losses of the ViT3 ablations on the GPU against the fp64 oracle
(ViT3 digest, section 03: the inner-loss and inner-model tables and the F1 / F2
modules of the ViT3 design).  fp32 inputs within 1e-4, bf16 inputs within 2e-2
(relative Frobenius error per output and per weight tensor).

* The simplified GLU FC(x) * SiLU(FC(x)) (F1): as its own inner model on the tensor
  cores (bf16, any multiple of 64 channels, ViT3's 64 included), and in its SwiGLU form
  (h = d, W1 = the gate's matrix Wb, W3 = the linear branch's Wa, W2 = I and the
  first-layer-only flag) on both dtypes; both against the oracle's own GLU model, with
  the ViT3 recipe (dot loss, one full-batch step, learning rate 1) and with momentum
  (+ Muon in the SwiGLU form) over several chunks.
* DWConv (F2): a 'same' depthwise k x k cross-correlation over the token grid whose
  kernels take the layer's gradient step.
* The RMSE inner loss: the chunk's RMSE is reduced on the device, then scales the MSE
  gradient.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth_inputs import gen_inputs, make_config
from tests.parity_util import compare, rel_fro, run_gpu

pytestmark = pytest.mark.gpu
TOL = {"bf16": 2e-2, "f32": 1e-4}


def _check(errs, tol):
    for k, v in errs.items():
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


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


# The GLU as its own inner model on the tensor cores (TTT_INNER_GLU, bf16): 64-channel
# blocks [Wb rows | Wa rows] per GEMM tile, so ViT3's own 64-channel heads run there, and
# no W2 = I products.  Against the oracle's GLU.
GLU_NATIVE_CASES = [
    # the ViT3 recipe at ViT3's head width
    dict(d=64, N=600, opt="gd", eta_mode="scalar", eta_scalar=1.0, data="vit"),
    dict(d=64, N=333, Nq=150, opt="gd", eta_mode="scalar", eta_scalar=1.0, data="vit", key_instnorm=True),
    dict(d=128, N=700, opt="momentum", chunk=256, weight_l2norm=True, eta_mode="per_token"),
    dict(d=64, N=450, opt="momentum", chunk=128, causal=1, weight_l2norm=True, eta_mode="per_token"),
    dict(d=192, N=520, opt="gd", loss="mse", eta_mode="scalar", eta_scalar=1.0, data="vit"),
    dict(d=64, N=300, opt="momentum", loss="mse", chunk=128, eta_mode="per_token", epochs=2),
]


@pytest.mark.parametrize("kw", GLU_NATIVE_CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_glu_inner_model_against_the_oracle(kw):
    base = dict(B=2, H=2, inner="glu", loss="neg_dot", dtype="bf16", data="lact", seed=81)
    base.update(kw)
    base["h"] = base["d"]
    cfg = make_config(**base)
    _check(compare(cfg), TOL["bf16"])


def test_glu_matches_its_swiglu_form_on_the_gpu():
    # the native GLU and its SwiGLU form (W1 = Wb, W3 = Wa, W2 = I, first layer only) run
    # different kernels on the same bf16 inputs: their results agree to bf16 rounding
    kw = dict(B=1, H=2, N=500, d=128, h=128, loss="neg_dot", opt="gd", dtype="bf16", data="vit",
              eta_mode="scalar", eta_scalar=1.0, seed=83)
    cfg_glu = make_config(inner="glu", **kw)
    x = gen_inputs(cfg_glu)
    d, P = 128, 128 * 128
    Og, Wg = run_gpu(cfg_glu, x)
    xs = dict(x)
    xs["W0"] = torch.cat([x["W0"][:, P:], x["W0"][:, :P], torch.eye(d).reshape(1, -1).expand(2, -1)], dim=1).contiguous()
    Os, Ws = run_gpu(make_config(inner="swiglu", first_layer_only=True, **kw), xs)
    assert rel_fro(Og, Os) < 1e-2
    assert rel_fro(Wg[..., :P], Ws[..., P:2 * P]) < 1e-2 and rel_fro(Wg[..., P:], Ws[..., :P]) < 1e-2


def test_glu_bench_workload_at_full_size():
    # the GLU heads of the ViT3-S-like 1248^2 layer (B8 H5 N6084 d64): every head
    from synth_inputs import workload
    errs = compare(workload("vit3s_1248_glu_n6084"))
    print({k: f"{v:.2e}" for k, v in errs.items()})
    _check(errs, TOL["bf16"])


# ---------------------------------------------------------------- RMSE loss
RMSE_CASES = [
    dict(dtype="f32", inner="linear", opt="gd", d=24, h=24, N=161),
    dict(dtype="f32", inner="mlp2_gelu", opt="gd", key_instnorm=True, data="vit", eta_mode="scalar", d=24, h=40,
         N=161),
    dict(dtype="f32", inner="swiglu", opt="momentum_muon", chunk=70, weight_l2norm=True, Nq=33, d=24, h=40, N=161),
    dict(dtype="f32", inner="mlp2_gelu", opt="momentum", chunk=50, causal=1, d=24, h=40, N=161),
    # bf16: the RMSE is recovered from the bf16 MSE gradient, then rescales it
    dict(dtype="bf16", inner="mlp2_gelu", opt="gd", d=64, h=256, N=700, key_instnorm=True, data="vit",
         eta_mode="scalar"),
    dict(dtype="bf16", inner="mlp2_gelu", opt="momentum", d=64, h=128, N=333, chunk=128, key_instnorm=True,
         data="vit", eta_mode="scalar"),
    dict(dtype="bf16", inner="linear", opt="momentum_muon", d=128, h=128, N=390, chunk=128, weight_l2norm=True),
]


@pytest.mark.parametrize("kw", RMSE_CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_rmse_loss_against_the_oracle(kw):
    base = dict(B=2, H=2, loss="rmse", data="lact", eta_mode="per_token", seed=83)
    base.update(kw)
    cfg = make_config(**base)
    _check(compare(cfg), TOL[cfg["dtype"]])


# ---------------------------------------------------------------- DWConv


DW_CASES = [
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


@pytest.mark.parametrize("kw", DW_CASES, ids=lambda kw: "-".join(f"{v}" for v in kw.values()))
def test_dwconv_against_the_oracle(kw):
    kw = dict(kw)
    gh, gw = kw.pop("gh"), kw.pop("gw")
    base = dict(B=2, H=2, N=gh * gw, grid_h=gh, grid_w=gw, inner="dwconv", data="lact", eta_mode="per_token",
                seed=97)
    base.update(kw)
    cfg = make_config(**base)
    _check(compare(cfg), TOL[cfg["dtype"]])


def test_dwconv_bench_workload_at_full_size():
    # the workload bench.py times (B8, a 78 x 78 grid, d64), in its launch configuration
    from synth_inputs import workload

    _check(compare(workload("vit3s_1248_dwconv_n6084")), TOL["bf16"])


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
