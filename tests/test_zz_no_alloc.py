"""ttt_forward_noalloc: the forward pass for callers that cannot allocate device
memory (the library's static device scratch replaces the caller's workspace).

Collected last on purpose, so that a run stopping at the first failure has run
every other test first.  It must pass alone in a fresh process and after the
rest of the suite.
"""
import ctypes

import pytest
import torch

from synth_inputs import gen_inputs, make_config
from tests.parity_util import rel_fro

pytestmark = pytest.mark.gpu
TOL = {"bf16": 2e-2, "f32": 1e-4}

CASES = [
    make_config(B=1, H=2, N=700, chunk=256, Nq=200, d=128, h=256, inner="swiglu", loss="neg_dot",
                opt="momentum_muon", weight_l2norm=True, dtype="bf16", data="lact", eta_mode="per_token", seed=21),
    make_config(B=1, H=1, N=196, d=64, h=64, inner="mlp2_gelu", loss="mse", opt="gd", key_instnorm=True,
                dtype="f32", data="vit", seed=22),
]


@pytest.mark.parametrize("cfg", CASES, ids=["swiglu_bf16", "mlp2_fp32"])
def test_noalloc_matches_workspace_entry_point_twice(cfg):
    from weight_sequence_mixing_b200 import binding

    lib = binding.LIB
    x = gen_inputs(cfg)
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    layer = binding.TTTLayer(cfg)
    assert lib.ttt_workspace_size(layer._handle) <= 32 * 1024 * 1024
    O_ref, W_ref = layer.forward(d["Q"], d["K"], d["V"], d["eta"], d["W0"])  # existing entry point
    torch.cuda.synchronize()
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    for _ in range(2):  # two calls in a row share the scratch; the second must not see the first's state
        O = torch.full_like(O_ref, float("nan"))
        W = torch.full_like(W_ref, float("nan"))
        st = lib.ttt_forward_noalloc(layer._handle, ctypes.c_void_p(d["Q"].data_ptr()),
                                     ctypes.c_void_p(d["K"].data_ptr()), ctypes.c_void_p(d["V"].data_ptr()),
                                     None if d["eta"] is None else ctypes.c_void_p(d["eta"].data_ptr()),
                                     ctypes.c_void_p(d["W0"].data_ptr()), ctypes.c_void_p(O.data_ptr()),
                                     ctypes.c_void_p(W.data_ptr()), ctypes.c_void_p(status.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, binding.status_string(st)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        tol = TOL[cfg["dtype"]]
        assert rel_fro(O.double().cpu().numpy(), O_ref.double().cpu().numpy()) <= tol
        assert rel_fro(W.double().cpu().numpy(), W_ref.double().cpu().numpy()) <= tol
    layer.close()


def test_noalloc_rejects_layers_larger_than_the_scratch():
    from weight_sequence_mixing_b200 import binding

    cfg = make_config(B=1, H=2, N=65536, d=256, h=512, inner="swiglu", loss="neg_dot", opt="gd", dtype="bf16",
                      data="lact", eta_mode="per_token")
    layer = binding.TTTLayer(cfg)
    assert binding.LIB.ttt_workspace_size(layer._handle) > 32 * 1024 * 1024
    fake = ctypes.c_void_p(1 << 20)
    st = binding.LIB.ttt_forward_noalloc(layer._handle, fake, fake, fake, None, fake, fake, None, None, None)
    assert st == binding.TTT_ERR_WORKSPACE
    layer.close()
