"""Plain fp64 CPU oracle of the TTT-layer forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline / reference arm may import this module.  The CUDA path never calls
it, and it shares no code with the CUDA path: the only thing both sides share is
the seeded input generator in ``synth_inputs``.

What is computed (sources: the pages' text, cited per function):

* The TTT layer treats the keys and values of a chunk as a small training set.
  The inner model F_W predicts V_hat = F_W(K); one gradient step on a
  reconstruction loss updates W; the queries then read the updated weights,
  O = F_{W*}(Q).  [ViT3 digest, section 02 "method essence", update equation;
  section 02 note (i) forward on keys, (ii) loss backward, (iii) forward on queries]
* Inner models, PyTorch-Linear layout ([out, in], applied to row vectors as x W^T):
  linear F(x) = x W^T [ViT3 digest, section 01: linear attention is a d x d layer];
  two-layer GELU MLP F(x) = GELU(x W1^T) W2^T [ViT3 digest, inner-model table;
  TTT vs Sleep, "Side one"]; SwiGLU F(x) = (SiLU(x W1^T) * x W3^T) W2^T with three
  matrices [LaCT analysis, "Nonlinear memory complements local attention"];
  simplified GLU F(x) = (x Wa^T) * SiLU(x Wb^T) with two d x d matrices and no
  output projection [ViT3 digest, section 03, inner-model table and the F1 module
  of the ViT3 design]; depthwise convolution DWConv(x) over the token grid, one k x k
  kernel per channel [ViT3 digest, section 03, guideline 6 and the inner-model table;
  the F2 module of the ViT3 design].
* Losses: MSE, RMSE = sqrt(MSE), and the negative dot product -<F(k_i), v_i> [ViT3
  digest, inner-loss table; LaCT analysis, "Nonlinear memory"], summed with each
  token's learning rate eta_i [LaCT analysis, "Nonlinear memory"].
* One full-batch step per chunk [ViT3 digest, guideline 2]; large chunks and
  apply-then-update order for causal data, update-then-apply otherwise
  [LaCT analysis, "Fast weights" and "Order of operations"].
* Optimizers: plain gradient step, momentum, Muon (Newton-Schulz orthogonalisation of
  each matrix gradient), then L2 normalisation of the weights [LaCT analysis,
  "Nonlinear memory"].
* Key instance normalisation over tokens [TTT vs Sleep, "Side one": keys carry a
  constant shift that must be removed].

Readings taken where the pages are silent (numbered R1-R24 wherever they are cited):
  R1 every fast-weight matrix is updated; R2 MSE is the mean over the chunk's
  (token, channel) elements, weighted per token by eta_i; R3 the dot loss is a sum
  over tokens with no 1/n; R4 exact erf GELU; R5 SwiGLU W1 = SiLU gate, W3 = linear
  branch, W2 = down projection; R6 no biases; R7 instance norm per channel over the
  chunk's tokens, biased variance, eps, no affine, keys only, the target V stays raw;
  R8 each [out,in] row scaled to unit L2 norm after every update; R9 heavy-ball
  momentum M <- beta M + G, M0 = 0 (or the momentum a previous call on the same
  sequence ended with), carried across chunks;
  R10 Muon = Newton-Schulz quintic (a, b, c) on G / (||G||_F + 1e-7), transposed so
  rows <= cols, applied to the momentum buffer when momentum is on; R11 lr scales the
  update; R12 order G -> momentum -> NS -> W <- W - lr U -> row norm; R21 with
  ``first_layer_only`` only the matrices that read the input (W1, and W3 for SwiGLU;
  the single matrix of the linear model) take the step, W2 keeps its initial value
  and is not row-normalised [TTT vs Sleep, "Side one": the first layer is adjusted];
  R22 the simplified GLU has no biases, Wa is the linear branch, Wb the SiLU gate;
  R23 RMSE is the square root of the R2 MSE of the chunk (eta inside the root); its
  gradient is the MSE gradient over 2 sqrt(MSE), and zero where the MSE is zero;
  R24 DWConv: tokens in raster order on a grid_h x grid_w grid, a 'same' depthwise
  cross-correlation with zero padding, odd k (3 by default, the size of the pages'
  convolution row), no bias, weights [d][k*k] (PyTorch's [d, 1, k, k]); the whole grid
  is one chunk (non-causal) and the queries lie on the same grid.

Parity: every part here is pinned by tests in tests/test_oracle_pins.py (closed forms,
finite differences, SVD, invariances).  The full-size GELU-MLP / SwiGLU / Muon results
have no published worked values; they are pinned only through those parts.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf as _erf

F64 = np.float64
_SQRT2 = np.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / np.sqrt(2.0 * np.pi)


# ---------------------------------------------------------------------------
# activations (reading R4: exact GELU; SiLU = x * sigmoid(x))
# ---------------------------------------------------------------------------
def gelu(x):
    return 0.5 * x * (1.0 + _erf(x / _SQRT2))


def gelu_prime(x):
    cdf = 0.5 * (1.0 + _erf(x / _SQRT2))
    pdf = _INV_SQRT_2PI * np.exp(-0.5 * x * x)
    return cdf + x * pdf


def sigmoid(x):
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def silu(x):
    return x * sigmoid(x)


def silu_prime(x):
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


# ---------------------------------------------------------------------------
# fast-weight packing ([out, in] matrices, concatenated per head)
# ---------------------------------------------------------------------------
def matrix_shapes(kind: str, d: int, h: int, ksize: int = 3):
    if kind == "linear":
        return [("W", d, d)]
    if kind == "mlp2_gelu":
        return [("W1", h, d), ("W2", d, h)]
    if kind == "swiglu":
        return [("W1", h, d), ("W3", h, d), ("W2", d, h)]
    if kind == "glu":
        return [("Wa", d, d), ("Wb", d, d)]
    if kind == "dwconv":
        return [("Wc", d, ksize * ksize)]
    raise ValueError(kind)


def unpack(kind, d, h, flat, ksize=3):
    flat = np.asarray(flat, dtype=F64)
    out, off = {}, 0
    for name, r, c in matrix_shapes(kind, d, h, ksize):
        out[name] = flat[off:off + r * c].reshape(r, c).copy()
        off += r * c
    assert off == flat.size
    return out


def pack(kind, d, h, W, ksize=3):
    return np.concatenate([W[name].reshape(-1) for name, _, _ in matrix_shapes(kind, d, h, ksize)])


# ---------------------------------------------------------------------------
# depthwise convolution over the token grid (reading R24)
# ---------------------------------------------------------------------------
def _pad_grid(X, grid, r):
    gh, gw = grid
    Xp = np.zeros((gh + 2 * r, gw + 2 * r, X.shape[1]), dtype=F64)
    Xp[r:r + gh, r:r + gw] = X.reshape(gh, gw, X.shape[1])
    return Xp


def dwconv_apply(Wc, X, grid):
    """Y[(y, x), c] = sum_{a, b < k} Wc[c, a k + b] X[(y + a - r, x + b - r), c], r = k // 2,
    zero outside the grid.  X [gh * gw, d] in raster order."""
    gh, gw = grid
    k = int(round(np.sqrt(Wc.shape[1])))
    Xp = _pad_grid(X, grid, k // 2)
    Y = np.zeros((gh, gw, X.shape[1]), dtype=F64)
    for a in range(k):
        for b in range(k):
            Y += Wc[:, a * k + b] * Xp[a:a + gh, b:b + gw]
    return Y.reshape(gh * gw, X.shape[1])


def dwconv_weight_grad(X, dY, grid, k):
    """Gradient of sum(dY * dwconv_apply(Wc, X)) in Wc: for each channel and tap, the sum
    over the grid of dY times the input shifted by that tap."""
    gh, gw = grid
    Xp = _pad_grid(X, grid, k // 2)
    dYg = dY.reshape(gh, gw, dY.shape[1])
    G = np.zeros((dY.shape[1], k * k), dtype=F64)
    for a in range(k):
        for b in range(k):
            G[:, a * k + b] = np.sum(dYg * Xp[a:a + gh, b:b + gw], axis=(0, 1))
    return G


# ---------------------------------------------------------------------------
# inner model: forward and hand-derived backward
# [ViT3 digest section 02; LaCT analysis "Nonlinear memory"]
# ---------------------------------------------------------------------------
def inner_forward(kind, W, X, grid=None):
    """Returns (F_W(X), cache).  X is [n, d] (rows are tokens; for DWConv the n = gh * gw
    tokens of the grid ``grid`` = (gh, gw) in raster order)."""
    if kind == "linear":
        return X @ W["W"].T, dict(X=X)
    if kind == "mlp2_gelu":
        Z = X @ W["W1"].T
        Hh = gelu(Z)
        return Hh @ W["W2"].T, dict(X=X, Z=Z, H=Hh)
    if kind == "swiglu":
        Z1 = X @ W["W1"].T
        Z3 = X @ W["W3"].T
        A = silu(Z1)
        Hh = A * Z3
        return Hh @ W["W2"].T, dict(X=X, Z1=Z1, Z3=Z3, A=A, H=Hh)
    if kind == "glu":
        Za = X @ W["Wa"].T
        Zb = X @ W["Wb"].T
        S = silu(Zb)
        return Za * S, dict(X=X, Za=Za, Zb=Zb, S=S)
    if kind == "dwconv":
        return dwconv_apply(W["Wc"], X, grid), dict(X=X, grid=grid)
    raise ValueError(kind)


def inner_backward(kind, W, cache, dY):
    """Gradients of sum(dY * F_W(X)) with respect to every matrix of W."""
    X = cache["X"]
    if kind == "linear":
        return dict(W=dY.T @ X)
    if kind == "mlp2_gelu":
        G2 = dY.T @ cache["H"]
        dH = dY @ W["W2"]
        dZ = dH * gelu_prime(cache["Z"])
        return dict(W1=dZ.T @ X, W2=G2)
    if kind == "swiglu":
        G2 = dY.T @ cache["H"]
        dH = dY @ W["W2"]
        dZ3 = dH * cache["A"]
        dZ1 = dH * cache["Z3"] * silu_prime(cache["Z1"])
        return dict(W1=dZ1.T @ X, W3=dZ3.T @ X, W2=G2)
    if kind == "glu":
        dZa = dY * cache["S"]
        dZb = dY * cache["Za"] * silu_prime(cache["Zb"])
        return dict(Wa=dZa.T @ X, Wb=dZb.T @ X)
    if kind == "dwconv":
        k = int(round(np.sqrt(W["Wc"].shape[1])))
        return dict(Wc=dwconv_weight_grad(X, dY, cache["grid"], k))
    raise ValueError(kind)


# ---------------------------------------------------------------------------
# reconstruction losses, weighted per token by eta_i
# [ViT3 digest, inner-loss table; LaCT analysis "Nonlinear memory"; readings R2, R3]
# ---------------------------------------------------------------------------
def loss_value(loss, Vhat, V, eta):
    n, d = V.shape
    if loss == "mse":
        return float(np.sum(eta[:, None] * (Vhat - V) ** 2) / (n * d))
    if loss == "rmse":
        return float(np.sqrt(np.sum(eta[:, None] * (Vhat - V) ** 2) / (n * d)))
    if loss == "neg_dot":
        return float(-np.sum(eta[:, None] * Vhat * V))
    raise ValueError(loss)


def loss_grad(loss, Vhat, V, eta):
    """dL/dV_hat for the chunk (eta already folded in)."""
    n, d = V.shape
    if loss == "mse":
        return 2.0 * eta[:, None] * (Vhat - V) / (n * d)
    if loss == "rmse":
        mse = np.sum(eta[:, None] * (Vhat - V) ** 2) / (n * d)
        if mse == 0.0:
            return np.zeros_like(V)
        return eta[:, None] * (Vhat - V) / (n * d * np.sqrt(mse))
    if loss == "neg_dot":
        return -eta[:, None] * V
    raise ValueError(loss)


# ---------------------------------------------------------------------------
# optimizer pieces [LaCT analysis "Nonlinear memory"; readings R8-R12]
# ---------------------------------------------------------------------------
def newton_schulz(G, iters, coeff):
    """Muon orthogonalisation: X0 = G/(||G||_F + 1e-7), rows <= cols, then
    `iters` times  A = X X^T;  X <- a X + (b A + c A^2) X."""
    a, b, c = coeff
    X = np.array(G, dtype=F64)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    X = X / (np.sqrt(np.sum(X * X)) + 1e-7)
    for _ in range(iters):
        A = X @ X.T
        Bm = b * A + c * (A @ A)
        X = a * X + Bm @ X
    return X.T if transposed else X


def row_l2_normalize(W):
    """Each [out, in] row scaled to unit L2 norm (reading R8)."""
    norms = np.sqrt(np.sum(W * W, axis=1, keepdims=True))
    return W / np.maximum(norms, 1e-12)


def instance_norm(K, eps):
    """Per channel over the chunk's tokens, biased variance, no affine (reading R7)."""
    mu = K.mean(axis=0, keepdims=True)
    var = ((K - mu) ** 2).mean(axis=0, keepdims=True)
    return (K - mu) / np.sqrt(var + eps)


def chunk_bounds(N, chunk):
    """Token ranges of the chunks; the last one may be partial (reading R15)."""
    if chunk is None or chunk <= 0 or chunk >= N:
        return [(0, N)]
    return [(s, min(s + chunk, N)) for s in range(0, N, chunk)]


def update_chunk(cfg, W, M, Kc, Vc, etac):
    """One full-batch gradient step on one chunk (W, M updated in place)."""
    kind = cfg["inner"]
    X = instance_norm(Kc, cfg["in_eps"]) if cfg["key_instnorm"] else Kc
    Vhat, cache = inner_forward(kind, W, X, _grid(cfg))
    dY = loss_grad(cfg["loss"], Vhat, Vc, etac)
    G = inner_backward(kind, W, cache, dY)
    opt = cfg["opt"]
    # reading R21: the second layer keeps its initial value (no step, no row norm)
    frozen = {"W2"} if cfg.get("first_layer_only", False) else set()
    for name in W:
        if name in frozen:
            continue
        g = G[name]
        if opt in ("momentum", "momentum_muon"):
            M[name] = cfg["momentum"] * M[name] + g
            u = M[name]
        else:
            u = g
        if opt in ("muon", "momentum_muon"):
            u = newton_schulz(u, cfg["ns_iters"], cfg["ns_coeff"])
        W[name] = W[name] - cfg["lr"] * u
        if cfg["weight_l2norm"]:
            W[name] = row_l2_normalize(W[name])


def _grid(cfg):
    return (int(cfg["grid_h"]), int(cfg["grid_w"])) if cfg["inner"] == "dwconv" else None


def forward_head(cfg, Q, K, V, eta, w0, m0=None, return_m=False):
    """One (batch, head): returns (O [Nq, d], W* packed [P]) in fp64, and with
    ``return_m`` also the momentum buffer after the last step (packed [P]).

    Non-causal: update over every chunk in order, then O = F_{W*}(Q).
    Causal (Nq == N): for each chunk, first O_c = F_W(Q_c), then update with chunk c.
    ``m0`` (packed [P]) is the momentum a previous call on the same sequence ended
    with (streamed state, LaCT "Video and distributed"); None means zero (R9).
    """
    kind, d, h = cfg["inner"], cfg["d"], cfg["h"]
    ks = int(cfg.get("ksize", 3))
    grid = _grid(cfg)
    Q = np.asarray(Q, dtype=F64)
    K = np.asarray(K, dtype=F64)
    V = np.asarray(V, dtype=F64)
    N = K.shape[0]
    if eta is None:
        eta = np.full((N,), float(cfg["eta_scalar"]), dtype=F64)
    else:
        eta = np.asarray(eta, dtype=F64)
    W = unpack(kind, d, h, w0, ks)
    M = unpack(kind, d, h, m0, ks) if m0 is not None else {name: np.zeros_like(m) for name, m in W.items()}
    bounds = chunk_bounds(N, cfg["chunk"])
    if grid is not None:  # reading R24: the whole grid is one non-causal chunk, queries on it too
        if grid[0] * grid[1] != N or Q.shape[0] != N or len(bounds) != 1 or cfg["causal"] or ks % 2 == 0:
            raise ValueError("DWConv needs one non-causal chunk over a grid_h x grid_w grid, Nq == N, odd k")
    # inner epochs: that many full-batch steps on each chunk before the next one
    # (ViT3 digest, inner-training ablation); momentum carries through them.  A
    # read-only call takes none (LaCT "Video and distributed": chunks that only read).
    epochs = 0 if cfg.get("no_update", False) else max(1, int(cfg.get("epochs", 1)))
    if cfg["causal"]:
        if Q.shape[0] != N:
            raise ValueError("causal order needs Nq == N")
        O = np.empty((N, d), dtype=F64)
        for s, e in bounds:
            O[s:e] = inner_forward(kind, W, Q[s:e], grid)[0]
            for _ in range(epochs):
                update_chunk(cfg, W, M, K[s:e], V[s:e], eta[s:e])
    else:
        for s, e in bounds:
            for _ in range(epochs):
                update_chunk(cfg, W, M, K[s:e], V[s:e], eta[s:e])
        O = inner_forward(kind, W, Q, grid)[0]
    if return_m:
        return O, pack(kind, d, h, W, ks), pack(kind, d, h, M, ks)
    return O, pack(kind, d, h, W, ks)


def _np(t):
    if t is None:
        return None
    if hasattr(t, "detach"):  # a torch tensor (bf16 widens exactly to fp64)
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=F64)


def forward(cfg, Q, K, V, eta, W0, heads=None, M0=None, return_m=False):
    """All (batch, head) pairs, or the listed ``heads`` [(b, h), ...].

    Returns O [B, H, Nq, d] and W* [B, H, P] in fp64 (entries of unlisted heads are NaN);
    with ``return_m`` also the final momentum buffers [B, H, P].  ``M0`` [B, H, P]
    is the momentum carried in from a previous call (None: zero).
    """
    B, H = cfg["B"], cfg["H"]
    Nq, d = cfg["Nq"], cfg["d"]
    P = sum(r * c for _, r, c in matrix_shapes(cfg["inner"], d, cfg["h"], int(cfg.get("ksize", 3))))
    O = np.full((B, H, Nq, d), np.nan)
    Ws = np.full((B, H, P), np.nan)
    Ms = np.full((B, H, P), np.nan)
    M0n = _np(M0)
    todo = heads if heads is not None else [(b, hh) for b in range(B) for hh in range(H)]
    W0n = _np(W0)
    per_batch = bool(cfg.get("w0_per_batch", False))  # W0 [B, H, P]: one state per entry
    for b, hh in todo:
        e = None if eta is None else _np(eta[b, hh])
        w0 = W0n[b, hh] if per_batch else W0n[hh]
        m0 = None if M0n is None else M0n[b, hh]
        O[b, hh], Ws[b, hh], Ms[b, hh] = forward_head(cfg, _np(Q[b, hh]), _np(K[b, hh]), _np(V[b, hh]), e, w0,
                                                      m0=m0, return_m=True)
    if return_m:
        return O, Ws, Ms
    return O, Ws
