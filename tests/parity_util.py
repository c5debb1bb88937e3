"""Helpers shared by the GPU parity tests: run the CUDA layer and the oracle on the
same seeded inputs and compare them per output and per final weight matrix."""
import numpy as np
import torch

import oracle as orc
from synth_inputs import gen_inputs, matrix_shapes


def rel_fro(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def run_gpu(cfg, x):
    from weight_sequence_mixing_b200 import binding

    layer = binding.TTTLayer(cfg)
    dev = lambda t: None if t is None else t.contiguous().cuda()
    O, W = layer.forward(dev(x["Q"]), dev(x["K"]), dev(x["V"]), dev(x["eta"]), dev(x["W0"]))
    torch.cuda.synchronize()
    out = O.double().cpu().numpy(), W.double().cpu().numpy()
    layer.close()
    return out


def compare(cfg, x=None, heads=None):
    """Returns dict of relative Frobenius errors: O and each matrix of W* (worst over heads too)."""
    if x is None:
        x = gen_inputs(cfg)
    Og, Wg = run_gpu(cfg, x)
    Or, Wr = orc.forward(cfg, x["Q"], x["K"], x["V"], x["eta"], x["W0"], heads=heads)
    sel = heads if heads is not None else [(b, h) for b in range(cfg["B"]) for h in range(cfg["H"])]
    bi = [b for b, _ in sel]
    hi = [h for _, h in sel]
    errs = {"O": rel_fro(Og[bi, hi], Or[bi, hi])}
    off = 0
    for name, r, c in matrix_shapes(cfg):
        sl = slice(off, off + r * c)
        errs[name] = rel_fro(Wg[bi, hi, sl], Wr[bi, hi, sl])
        errs[name + "_worst_head"] = max(rel_fro(Wg[b, h, sl], Wr[b, h, sl]) for b, h in sel)
        off += r * c
    errs["O_worst_head"] = max(rel_fro(Og[b, h], Or[b, h]) for b, h in sel)
    assert np.isfinite(Og).all() and np.isfinite(Wg).all()
    return errs
