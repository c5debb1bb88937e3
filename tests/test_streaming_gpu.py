"""Streaming use of the layer on the GPU: one fast-weight state per batch entry (W0
[B, H, P], e.g. the W_out of the previous call on the same sequences) and read-only calls,
against the fp64 oracle, and two calls over the halves of a sequence against one call."""
import pytest
import torch

from synth_inputs import gen_inputs, make_config
from tests.parity_util import compare, rel_fro, run_gpu

pytestmark = pytest.mark.gpu

BASE = {
    "bf16": dict(B=2, H=2, N=512, d=128, h=256, inner="swiglu", loss="neg_dot", dtype="bf16"),
    "f32": dict(B=2, H=2, N=96, d=24, h=40, inner="swiglu", loss="neg_dot", dtype="f32"),
}
TOL = {"bf16": 2e-2, "f32": 1e-4}


def _check(errs, tol):
    for k, v in errs.items():
        assert v <= tol, f"{k}: relative Frobenius error {v:.3e} > {tol}"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("no_update", [False, True])
def test_per_batch_initial_state(dtype, no_update):
    cfg = make_config(opt="momentum", weight_l2norm=True, data="lact", eta_mode="per_token", seed=41, chunk=0,
                      w0_per_batch=True, no_update=no_update, **BASE[dtype])
    x = gen_inputs(cfg)
    # a different state per batch entry
    g = torch.Generator().manual_seed(3)
    W0 = x["W0"].unsqueeze(0).repeat(cfg["B"], 1, 1)
    W0[1] += 0.05 * torch.randn(W0[1].shape, generator=g)
    x["W0"] = W0.contiguous()
    _check(compare(cfg, x), TOL[dtype])
    if no_update:
        _, W = run_gpu(cfg, x)
        assert rel_fro(W, x["W0"].double().numpy()) == 0.0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [0, 1])
def test_two_streamed_calls_equal_one_chunked_call(dtype, causal):
    base = dict(opt="gd", weight_l2norm=True, data="lact", eta_mode="per_token", seed=43, causal=causal,
                **BASE[dtype])
    N = base["N"]
    half = N // 2
    full = make_config(chunk=half, **base)
    x = gen_inputs(full)
    O1, W1 = run_gpu(full, x)

    def part(a, b, w0, per_batch):
        kw = dict(base, N=half, Nq=half if causal else N)  # non-causal: the whole query set
        cfg = make_config(chunk=0, w0_per_batch=per_batch, **kw)
        q = x["Q"][:, :, a:b] if causal else x["Q"]
        xi = dict(Q=q.contiguous(), K=x["K"][:, :, a:b].contiguous(), V=x["V"][:, :, a:b].contiguous(),
                  eta=x["eta"][:, :, a:b].contiguous(), W0=w0)
        return run_gpu(cfg, xi)

    Oa, Wa = part(0, half, x["W0"], False)
    Ob, Wb = part(half, N, torch.from_numpy(Wa).float().contiguous(), True)
    assert rel_fro(Wb, W1) < 1e-5
    O2 = torch.cat([torch.from_numpy(Oa), torch.from_numpy(Ob)], dim=2).numpy() if causal else Ob
    assert rel_fro(O2, O1) < 1e-5


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("opt", ["momentum", "momentum_muon"])
def test_two_streamed_calls_with_momentum_state_equal_one_chunked_call(dtype, causal, opt):
    # (W, M) handed on: W_out -> W0 and the opaque momentum blob state_out -> state_in
    from weight_sequence_mixing_b200 import binding
    import oracle as orc

    base = dict(opt=opt, weight_l2norm=True, data="lact", eta_mode="per_token", seed=47, causal=causal,
                **BASE[dtype])
    N = base["N"]
    half = N // 2
    full = make_config(chunk=half, **base)
    x = gen_inputs(full)
    O1, W1 = run_gpu(full, x)

    def part(a, b, w0, per_batch, state_in, state_out):
        kw = dict(base, N=half, Nq=half if causal else N)
        layer = binding.TTTLayer(make_config(chunk=0, w0_per_batch=per_batch, **kw))
        q = x["Q"][:, :, a:b] if causal else x["Q"]
        dev = lambda t: t.contiguous().cuda()
        O, W = layer.forward_state(dev(q), dev(x["K"][:, :, a:b]), dev(x["V"][:, :, a:b]),
                                   dev(x["eta"][:, :, a:b]), dev(w0), state_in=state_in, state_out=state_out)
        torch.cuda.synchronize()
        out = O.double().cpu(), W
        layer.close()
        return out

    probe = binding.TTTLayer(make_config(chunk=0, **dict(base, N=half, Nq=half if causal else N)))
    assert probe.state_size > 0
    state = probe.new_state()
    probe.close()
    Oa, Wa = part(0, half, x["W0"], False, None, state)
    Ob, Wb = part(half, N, Wa, True, state, state)
    Wb = Wb.double().cpu().numpy()
    assert rel_fro(Wb, W1) < 1e-5
    O2 = torch.cat([Oa, Ob], dim=2).numpy() if causal else Ob.numpy()
    assert rel_fro(O2, O1) < 1e-5
    # and against the oracle's one chunked call
    Or, Wr = orc.forward(full, x["Q"], x["K"], x["V"], x["eta"], x["W0"])
    assert rel_fro(O2, Or) <= TOL[dtype] and rel_fro(Wb, Wr) <= TOL[dtype]
