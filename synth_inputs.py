"""Seeded synthetic inputs for the TTT layer (test-time-training layer) forward pass.

This module is shared by the CPU oracle, the tests and the benchmark.  It holds
the workload definitions (sizes and options) and the seeded generators of the
layer's inputs Q, K, V, the per-token learning rates eta and the initial fast
weights W0.  It holds none of the layer's arithmetic.

Tensor layouts (row-major, contiguous):
  Q [B, H, Nq, d], K [B, H, N, d], V [B, H, N, d]   in the path dtype (bf16 or fp32)
  eta [B, H, N] fp32 (or None: the scalar ``eta_scalar`` is used for every token)
  W0 [H, P] fp32, shared by every batch entry.  Per head the matrices are stored
  PyTorch-Linear style ([out, in], row-major) and packed one after the other:
    linear    [W  (d x d)]
    mlp2_gelu [W1 (h x d) | W2 (d x h)]
    swiglu    [W1 (h x d) | W3 (h x d) | W2 (d x h)]
    glu       [Wa (d x d) | Wb (d x d)]   (bf16: TTT_INNER_GLU; the fp32 path runs it as a
              SwiGLU with h = d, W1 = Wb, W3 = Wa, W2 = I and the first-layer-only flag)
    dwconv    [Wc (d x k*k)]              (oracle only: one k x k kernel per channel)

Data recipes (the pages' workloads use image / text / multi-view data that is
not available here; seeded Gaussians of the same shapes stand in for them):
  "vit"  : Q, V ~ N(0, 1); K ~ N(0, 1) + 0.5 on every element (the constant
           per-channel key shift that motivates key instance-norm, "Test-Time
           Training vs Sleep", Side one); W0 ~ N(0, 1/d) for every matrix; eta scalar.
  "lact" : Q, K ~ N(0, 1) then L2-normalised per token; V ~ N(0, 1);
           eta_i = 0.01 * sigmoid(z_i), z ~ N(0, 1); W0 ~ N(0, 1/fan_in).

Every (tensor, batch, head) slice is drawn from its own torch CPU generator,
seeded from (workload seed, tensor id, b, h), so any head can be regenerated on
its own and CPU and GPU sides read bit-identical values.
"""
from __future__ import annotations

import copy
import math

import torch

# tensor ids inside a workload's seed space
_TID = {"Q": 1, "K": 2, "V": 3, "eta": 4, "W0": 5}

_DEFAULTS = dict(
    B=1, H=1, N=128, Nq=None, d=64, h=64, chunk=0, causal=0,
    inner="mlp2_gelu", loss="mse", opt="gd", dtype="bf16",
    key_instnorm=False, weight_l2norm=False, direct_launch=False, single_cta=False,
    w0_per_batch=False, no_update=False, first_layer_only=False,
    grid_h=0, grid_w=0, ksize=3,  # DWConv: token grid and kernel size
    eta_mode="scalar",           # "scalar" | "per_token"
    eta_scalar=1.0, lr=1.0, momentum=0.9,
    ns_iters=5, ns_coeff=(3.4445, -4.7750, 2.0315), in_eps=1e-5, epochs=1,
    data="vit", seed=7,
)

# The five workloads of the layer, named by what they are.
WORKLOADS = {
    # tiny non-causal layer, fp32: B1 H1 N196 d64, MLP 64->64->64 GELU, MSE, one step, eta=1, key instance-norm
    "tiny_mlp2_n196_fp32": dict(B=1, H=1, N=196, d=64, h=64, inner="mlp2_gelu", loss="mse", opt="gd",
                                dtype="f32", key_instnorm=True, eta_mode="scalar", eta_scalar=1.0,
                                data="vit", seed=1000),
    # ViT^3-S-like 1248^2 layer: B8 H6 N6084 d64, MLP 64->256->64 GELU, MSE, eta=1, key instance-norm
    "vit3s_1248_mlp2_n6084": dict(B=8, H=6, N=6084, d=64, h=256, inner="mlp2_gelu", loss="mse", opt="gd",
                                  dtype="bf16", key_instnorm=True, eta_mode="scalar", eta_scalar=1.0,
                                  data="vit", seed=2000),
    # LaCT-style causal language layer: B2 H4 N32768 chunk 2048 d256, SwiGLU 256->256->256,
    # negative dot product, per-token eta, momentum 0.9, weight row L2-norm, apply-then-update
    "lact_lm_causal_n32k_c2048": dict(B=2, H=4, N=32768, chunk=2048, causal=1, d=256, h=256,
                                      inner="swiglu", loss="neg_dot", opt="momentum", momentum=0.9,
                                      dtype="bf16", weight_l2norm=True, eta_mode="per_token",
                                      data="lact", seed=3000),
    # LaCT-style novel-view layer: B1 H2 N196608 Nq4096 d512, SwiGLU 512->1024->512,
    # negative dot product, per-token eta, Muon (5 Newton-Schulz iterations), weight row L2-norm
    "lact_nvs_n196k_d512": dict(B=1, H=2, N=196608, Nq=4096, d=512, h=1024, inner="swiglu",
                                loss="neg_dot", opt="muon", dtype="bf16", weight_l2norm=True,
                                eta_mode="per_token", data="lact", seed=4000),
    # LaCT-style million-token scene layer: B1 H4 N1029120 chunk 131072 Nq8040 d256,
    # SwiGLU 256->512->256, negative dot product, momentum 0.9 + Muon, weight row L2-norm
    "lact_scene_n1m_c131k": dict(B=1, H=4, N=1029120, chunk=131072, Nq=8040, d=256, h=512,
                                 inner="swiglu", loss="neg_dot", opt="momentum_muon", momentum=0.9,
                                 dtype="bf16", weight_l2norm=True, eta_mode="per_token",
                                 data="lact", seed=5000),
    # the GLU heads of a ViT^3-S-like 1248^2 layer: B8, 5 heads (the sixth is the DWConv head),
    # N6084, d64, F(x) = (x Wa^T) * SiLU(x Wb^T), the ViT^3 recipe (dot loss, one full-batch step,
    # eta = 1)
    "vit3s_1248_glu_n6084": dict(B=8, H=5, N=6084, d=64, h=64, inner="glu", loss="neg_dot", opt="gd",
                                 dtype="bf16", eta_mode="scalar", eta_scalar=1.0, data="vit", seed=7000),
    # the DWConv head of a ViT^3-S-like 1248^2 layer: B8, one head, the 78 x 78 token grid,
    # d64, 3 x 3 depthwise kernels, the ViT^3 recipe (dot loss, one full-batch step, eta = 1)
    "vit3s_1248_dwconv_n6084": dict(B=8, H=1, N=6084, grid_h=78, grid_w=78, ksize=3, d=64, h=64,
                                    inner="dwconv", loss="neg_dot", opt="gd", dtype="bf16",
                                    eta_mode="scalar", eta_scalar=1.0, data="vit", seed=6000),
}


def make_config(**kw) -> dict:
    """A full workload dict: defaults overridden by ``kw``; Nq defaults to N."""
    cfg = copy.deepcopy(_DEFAULTS)
    unknown = set(kw) - set(cfg)
    if unknown:
        raise KeyError(f"unknown workload keys: {sorted(unknown)}")
    cfg.update(kw)
    if cfg["Nq"] is None:
        cfg["Nq"] = cfg["N"]
    cfg["ns_coeff"] = tuple(float(c) for c in cfg["ns_coeff"])
    return cfg


def workload(name: str, **overrides) -> dict:
    base = dict(WORKLOADS[name])
    base.update(overrides)
    cfg = make_config(**base)
    cfg["name"] = name
    return cfg


def matrix_shapes(cfg) -> list[tuple[str, int, int]]:
    """(name, rows, cols) of each fast-weight matrix in packing order ([out, in] layout)."""
    d, h = cfg["d"], cfg["h"]
    kind = cfg["inner"]
    if kind == "linear":
        return [("W", d, d)]
    if kind == "mlp2_gelu":
        return [("W1", h, d), ("W2", d, h)]
    if kind == "swiglu":
        return [("W1", h, d), ("W3", h, d), ("W2", d, h)]
    if kind == "glu":
        return [("Wa", d, d), ("Wb", d, d)]
    if kind == "dwconv":
        return [("Wc", d, cfg["ksize"] * cfg["ksize"])]
    raise ValueError(kind)


def param_count(cfg) -> int:
    return sum(r * c for _, r, c in matrix_shapes(cfg))


def torch_dtype(cfg):
    return torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16


def _gen(cfg, tid: int, b: int, h: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    s = (int(cfg["seed"]) * 1_000_003 + tid * 100_003 + b * 1_009 + h * 17 + 1) % (2**63 - 1)
    g.manual_seed(s)
    return g


def _normal(shape, g) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32)


def _rows_unit(x: torch.Tensor) -> torch.Tensor:
    x64 = x.double()
    return (x64 / x64.norm(dim=-1, keepdim=True).clamp_min(1e-30)).float()


def gen_head(cfg, b: int, h: int) -> dict:
    """Inputs of one (batch, head) slice: Q [Nq,d], K [N,d], V [N,d], eta [N] or None."""
    N, Nq, d = cfg["N"], cfg["Nq"], cfg["d"]
    dt = torch_dtype(cfg)
    q = _normal((Nq, d), _gen(cfg, _TID["Q"], b, h))
    k = _normal((N, d), _gen(cfg, _TID["K"], b, h))
    v = _normal((N, d), _gen(cfg, _TID["V"], b, h))
    if cfg["data"] == "vit":
        k = k + 0.5
    elif cfg["data"] == "lact":
        q = _rows_unit(q)
        k = _rows_unit(k)
    elif cfg["data"] != "plain":
        raise ValueError(cfg["data"])
    eta = None
    if cfg["eta_mode"] == "per_token":
        z = _normal((N,), _gen(cfg, _TID["eta"], b, h))
        eta = (0.01 * torch.sigmoid(z.double())).float()
    return dict(Q=q.to(dt), K=k.to(dt), V=v.to(dt), eta=eta)


def gen_w0(cfg) -> torch.Tensor:
    """W0 [H, P] fp32 (shared by every batch entry)."""
    H = cfg["H"]
    out = torch.empty((H, param_count(cfg)), dtype=torch.float32)
    for hh in range(H):
        g = _gen(cfg, _TID["W0"], 0, hh)
        off = 0
        for _, r, c in matrix_shapes(cfg):
            fan_in = cfg["d"] if cfg["data"] == "vit" else c
            std = 1.0 / math.sqrt(fan_in)
            out[hh, off:off + r * c] = _normal((r * c,), g) * std
            off += r * c
    return out


def gen_inputs(cfg) -> dict:
    """All inputs as torch CPU tensors: Q, K, V [B,H,*,d] (path dtype), eta [B,H,N] fp32 or None, W0 [H,P] fp32."""
    B, H, N, Nq, d = cfg["B"], cfg["H"], cfg["N"], cfg["Nq"], cfg["d"]
    dt = torch_dtype(cfg)
    Q = torch.empty((B, H, Nq, d), dtype=dt)
    K = torch.empty((B, H, N, d), dtype=dt)
    V = torch.empty((B, H, N, d), dtype=dt)
    eta = torch.empty((B, H, N), dtype=torch.float32) if cfg["eta_mode"] == "per_token" else None
    for b in range(B):
        for hh in range(H):
            x = gen_head(cfg, b, hh)
            Q[b, hh] = x["Q"]
            K[b, hh] = x["K"]
            V[b, hh] = x["V"]
            if eta is not None:
                eta[b, hh] = x["eta"]
    return dict(Q=Q, K=K, V=V, eta=eta, W0=gen_w0(cfg))
