"""bench.py's work accounting (host only): the algorithmic FLOPs of each workload against
the closed forms of the flop count (2 per multiply-add; the update of a SwiGLU with the
dot loss is 12 N d h, of a GELU MLP with MSE 10 N d h; the apply 6 or 4 Nq d h; Newton-Schulz
4 m^2 n + 2 m^3 per iteration and matrix), the bytes of the bandwidth-bound DWConv head,
and the CPU samples of the reference arm."""
import pytest

import bench
from synth_inputs import workload

# total algorithmic GFLOP per forward pass, from the closed forms above
CLOSED_FORM_GFLOP = {
    # B1 H1 N196 d64 h64, MLP2 + MSE: 10 N d h + apply 4 Nq d h
    "tiny_mlp2_n196_fp32": (10 * 196 * 64 * 64 + 4 * 196 * 64 * 64) / 1e9,
    # B8 H6 N6084 d64 h256, MLP2 + MSE
    "vit3s_1248_mlp2_n6084": 48 * (10 * 6084 * 64 * 256 + 4 * 6084 * 64 * 256) / 1e9,
    # B2 H4 N32768 d = h = 256, SwiGLU + dot, causal: apply on every token
    "lact_lm_causal_n32k_c2048": 8 * (12 * 32768 * 256 * 256 + 6 * 32768 * 256 * 256) / 1e9,
    # B1 H2 N196608 Nq4096 d512 h1024, SwiGLU + dot, Muon: 3 matrices of 512 x 1024, 5 iterations
    "lact_nvs_n196k_d512": 2 * (12 * 196608 * 512 * 1024 + 6 * 4096 * 512 * 1024
                                + 3 * 5 * (4 * 512 ** 2 * 1024 + 2 * 512 ** 3)) / 1e9,
    # B1 H4 N1029120 (8 chunks) Nq8040 d256 h512, SwiGLU + dot, momentum + Muon on 256 x 512
    "lact_scene_n1m_c131k": 4 * (12 * 1029120 * 256 * 512 + 6 * 8040 * 256 * 512
                                 + 8 * 3 * 5 * (4 * 256 ** 2 * 512 + 2 * 256 ** 3)) / 1e9,
    # B8 H5 N6084 d64, GLU + dot: two d x d products on the keys (4 N d^2), their gradients
    # (4 N d^2) and two on the queries (4 Nq d^2)
    "vit3s_1248_glu_n6084": 40 * (8 * 6084 * 64 * 64 + 4 * 6084 * 64 * 64) / 1e9,
    # B8 H1 N6084 d64, 3 x 3 DWConv + dot: tap gradients 2 k^2 N d, apply 2 k^2 Nq d
    "vit3s_1248_dwconv_n6084": 8 * (2 * 9 * 6084 * 64 * 2) / 1e9,
}


@pytest.mark.parametrize("name", sorted(CLOSED_FORM_GFLOP))
def test_algorithmic_flops_match_the_closed_forms(name):
    got = sum(bench.algorithmic_flops(workload(name)).values()) / 1e9
    assert abs(got - CLOSED_FORM_GFLOP[name]) <= 1e-9 * CLOSED_FORM_GFLOP[name]


def test_headline_workload_is_about_2540_gflop():
    # the novel-view layer: 2474 (update) + 25.8 (apply) + 40.3 (Newton-Schulz) GFLOP
    f = bench.algorithmic_flops(workload("lact_nvs_n196k_d512"))
    assert round((f["token_phase"] + f["weight_grad"]) / 1e9) == 2474
    assert round(f["apply"] / 1e8) == 258 and round(f["newton_schulz"] / 1e8) == 403


def test_epochs_multiply_the_update_only():
    cfg = workload("lact_nvs_n196k_d512")
    one, three = bench.algorithmic_flops(cfg), bench.algorithmic_flops(dict(cfg, epochs=3))
    for k in ("token_phase", "weight_grad", "newton_schulz"):
        assert three[k] == 3 * one[k]
    assert three["apply"] == one["apply"]


def test_dwconv_bytes_and_cpu_sample_keep_whole_grids():
    cfg = workload("vit3s_1248_dwconv_n6084")
    b = bench.algorithmic_bytes(cfg)
    # bf16: K and V read by the tap-gradient pass, Q read and O written by the apply; eta is a scalar
    assert b["weight_grad"] == 8 * 2 * 6084 * 64 * 2 and b["apply"] == 8 * 2 * 6084 * 64 * 2
    s = bench.cpu_sample_config(cfg, 2 * 6084 + 5)
    assert (s["B"], s["N"], s["grid_h"], s["grid_w"]) == (2, 6084, 78, 78)
    assert bench.cpu_sample_config(cfg, 10)["B"] == 1
    assert "whole 78x78 grids" in bench.sample_text(cfg, s)
