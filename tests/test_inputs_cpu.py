"""The seeded input recipes (synth_inputs.py): shapes, value distributions and
structure of the stand-ins for the pages' workloads, and determinism."""
import math

import pytest
import torch

from synth_inputs import WORKLOADS, gen_head, gen_inputs, gen_w0, make_config, matrix_shapes, param_count, workload


def small(name, **kw):
    cfg = workload(name)
    cfg.update(B=min(cfg["B"], 2), H=min(cfg["H"], 2), N=min(cfg["N"], 1024), Nq=min(cfg["Nq"], 256), **kw)
    if cfg["causal"]:
        cfg["Nq"] = cfg["N"]
    return cfg


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_shapes_and_dtypes(name):
    cfg = small(name)
    x = gen_inputs(cfg)
    dt = torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16
    assert x["Q"].shape == (cfg["B"], cfg["H"], cfg["Nq"], cfg["d"]) and x["Q"].dtype == dt
    assert x["K"].shape == x["V"].shape == (cfg["B"], cfg["H"], cfg["N"], cfg["d"])
    assert x["W0"].shape == (cfg["H"], param_count(cfg)) and x["W0"].dtype == torch.float32
    if cfg["eta_mode"] == "per_token":
        assert x["eta"].shape == (cfg["B"], cfg["H"], cfg["N"])
    else:
        assert x["eta"] is None


def test_generation_is_deterministic_and_per_slice():
    cfg = small("lact_nvs_n196k_d512")
    a, b = gen_inputs(cfg), gen_inputs(cfg)
    for k in ("Q", "K", "V", "eta", "W0"):
        assert torch.equal(a[k], b[k])
    # every (batch, head) slice regenerates on its own
    h = gen_head(cfg, 0, 1)
    assert torch.equal(h["K"], a["K"][0, 1]) and torch.equal(h["eta"], a["eta"][0, 1])
    # another seed gives other values
    c = gen_inputs(dict(cfg, seed=cfg["seed"] + 1))
    assert not torch.equal(a["K"], c["K"])


def test_lact_recipe_unit_rows_and_learning_rates():
    cfg = small("lact_lm_causal_n32k_c2048")
    x = gen_inputs(cfg)
    for t in ("Q", "K"):
        norms = x[t].double().norm(dim=-1)
        assert torch.allclose(norms, torch.ones_like(norms), atol=1e-2)  # unit rows, bf16-rounded
    eta = x["eta"]
    assert (eta > 0).all() and (eta < 0.01).all()  # 0.01 * sigmoid(z)
    assert abs(eta.mean().item() - 0.005) < 5e-4
    # V ~ N(0, 1)
    v = x["V"].double()
    assert abs(v.mean().item()) < 0.02 and abs(v.std().item() - 1.0) < 0.02


def test_vit_recipe_key_shift_and_w0_scale():
    cfg = small("vit3s_1248_mlp2_n6084")
    x = gen_inputs(cfg)
    k = x["K"].double()
    assert abs(k.mean().item() - 0.5) < 0.02  # +0.5 on every key element
    assert abs(k.std().item() - 1.0) < 0.02
    w0 = x["W0"].double()
    assert abs(w0.std().item() - 1 / math.sqrt(cfg["d"])) < 0.01  # N(0, 1/d) for every matrix


def test_lact_w0_fan_in_scale():
    cfg = make_config(B=1, H=2, N=16, d=64, h=256, inner="swiglu", loss="neg_dot", data="lact", seed=5)
    w0 = gen_w0(cfg)[0].double()
    off = 0
    for _, r, c in matrix_shapes(cfg):
        m = w0[off:off + r * c]
        assert abs(m.std().item() - 1 / math.sqrt(c)) < 0.15 / math.sqrt(c)  # N(0, 1/fan_in)
        off += r * c


def test_scene_workload_has_a_partial_last_chunk():
    cfg = workload("lact_scene_n1m_c131k")
    assert cfg["N"] == 7 * 131072 + 111616 and cfg["chunk"] == 131072


@pytest.mark.parametrize("kind,k", [("glu", 3), ("dwconv", 1), ("dwconv", 3), ("dwconv", 7)])
def test_packing_of_the_ablation_inner_models(kind, k):
    # GLU: [Wa (d x d) | Wb (d x d)]; DWConv: [Wc (d x k*k)]; W0 has one row of P per head
    cfg = make_config(B=1, H=3, N=20, d=8, h=8, inner=kind, ksize=k, grid_h=4, grid_w=5)
    P = 2 * 8 * 8 if kind == "glu" else 8 * k * k
    assert param_count(cfg) == P
    W0 = gen_w0(cfg)
    assert W0.shape == (3, P) and torch.isfinite(W0).all()
    assert not torch.equal(W0[0], W0[1])  # each head draws its own weights
