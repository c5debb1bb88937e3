"""Failure detection on the GPU, without a fault: a bounded wait that runs out, and a
non-finite value in the inputs, each reported through the device status word while the
CUDA context stays usable."""
import math

import pytest
import torch

from synth_inputs import gen_inputs, make_config
from tests.parity_util import compare

pytestmark = pytest.mark.gpu


def _binding():
    from weight_sequence_mixing_b200 import binding

    return binding


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    b = _binding()
    word = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert b.selftest_timeout(word) == b.TTT_ERR_TIMEOUT
    torch.cuda.synchronize()
    # the context still runs the layer correctly afterwards
    cfg = make_config(B=1, H=2, N=300, d=128, h=256, inner="swiglu", loss="neg_dot", opt="gd", dtype="bf16",
                      data="lact", eta_mode="per_token", seed=23)
    errs = compare(cfg)
    assert errs["O"] <= 2e-2 and errs["W1"] <= 2e-2


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_nonfinite_learning_rate_is_reported(dtype):
    b = _binding()
    cfg = make_config(B=1, H=2, N=256, d=128, h=128, inner="swiglu" if dtype == "bf16" else "mlp2_gelu",
                      loss="neg_dot", opt="momentum", dtype=dtype, data="lact", eta_mode="per_token", seed=29)
    x = gen_inputs(cfg)
    x["eta"][0, 1, 17] = math.nan
    layer = b.TTTLayer(cfg)
    dev = lambda t: None if t is None else t.contiguous().cuda()
    with pytest.raises(b.TTTError) as info:
        layer.forward(dev(x["Q"]), dev(x["K"]), dev(x["V"]), dev(x["eta"]), dev(x["W0"]))
    assert info.value.status == b.TTT_ERR_NONFINITE
    # the status word was cleared by the query: a clean call on the same handle succeeds
    x["eta"][0, 1, 17] = 0.01
    layer.forward(dev(x["Q"]), dev(x["K"]), dev(x["V"]), dev(x["eta"]), dev(x["W0"]))
    layer.close()
