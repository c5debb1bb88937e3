"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a closed form
(linear attention), a hand-worked example, brute-force scalar loops, central
finite differences, an SVD, or an invariance the method must have.  None of
these needs a GPU.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as orc
from synth_inputs import make_config

RNG = np.random.default_rng(12345)
KINDS = ["linear", "mlp2_gelu", "swiglu", "glu"]
LOSSES = ["mse", "neg_dot", "rmse"]


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def cfg_for(kind, loss, **kw):
    base = dict(inner=kind, loss=loss, opt="gd", dtype="f32", d=4, h=6, N=8, key_instnorm=False,
                weight_l2norm=False, eta_mode="per_token")
    base.update(kw)
    return make_config(**base)


def rand_w(kind, d, h, scale=0.5):
    return {name: rand(r, c, scale=scale) for name, r, c in orc.matrix_shapes(kind, d, h)}


# ---------------------------------------------------------------- activations
def test_gelu_textbook_values():
    # GELU(x) = x * Phi(x); Phi(1) = 0.8413447460685429 (standard normal CDF)
    x = np.array([0.0, 1.0, -1.0, 8.0, -8.0])
    g = orc.gelu(x)
    assert g[0] == 0.0
    assert abs(g[1] - 0.8413447460685429) < 1e-15
    assert abs(g[2] + 0.15865525393145707) < 1e-15
    assert abs(g[3] - 8.0) < 1e-12 and abs(g[4]) < 1e-12


def test_silu_textbook_values():
    x = np.array([0.0, 1.0, -1.0])
    s = orc.silu(x)
    assert s[0] == 0.0
    assert abs(s[1] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    assert abs(s[2] + 1.0 / (1.0 + math.exp(1.0))) < 1e-15


@pytest.mark.parametrize("fn,dfn", [(orc.gelu, orc.gelu_prime), (orc.silu, orc.silu_prime)])
def test_activation_derivatives_by_finite_difference(fn, dfn):
    x = np.linspace(-6, 6, 97)
    eps = 1e-6
    fd = (fn(x + eps) - fn(x - eps)) / (2 * eps)
    assert np.max(np.abs(fd - dfn(x))) < 1e-8


# ---------------------------------------------------------------- brute-force forward
def _brute_forward(kind, W, x):
    """Scalar loops with math.erf / math.exp on one token (no numpy linear algebra)."""
    def gelu(z):
        return 0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0)))

    def silu(z):
        return z / (1.0 + math.exp(-z))

    def matvec(M, v):
        return [sum(M[i][j] * v[j] for j in range(len(v))) for i in range(len(M))]

    if kind == "linear":
        return matvec(W["W"].tolist(), x)
    if kind == "mlp2_gelu":
        hid = [gelu(z) for z in matvec(W["W1"].tolist(), x)]
        return matvec(W["W2"].tolist(), hid)
    if kind == "glu":  # FC(x) * SiLU(FC(x))
        za = matvec(W["Wa"].tolist(), x)
        zb = matvec(W["Wb"].tolist(), x)
        return [a * silu(b) for a, b in zip(za, zb)]
    z1 = matvec(W["W1"].tolist(), x)
    z3 = matvec(W["W3"].tolist(), x)
    hid = [silu(a) * b for a, b in zip(z1, z3)]
    return matvec(W["W2"].tolist(), hid)


@pytest.mark.parametrize("kind", KINDS)
def test_inner_forward_matches_scalar_loops(kind):
    d, h = 5, 7
    W = rand_w(kind, d, h)
    X = rand(6, d)
    Y = orc.inner_forward(kind, W, X)[0]
    for i in range(X.shape[0]):
        ref = _brute_forward(kind, W, X[i].tolist())
        assert np.allclose(Y[i], ref, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- gradients
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("loss", LOSSES)
def test_gradients_by_central_finite_differences(kind, loss):
    d, h, n = 4, 6, 8
    W = rand_w(kind, d, h)
    X, V = rand(n, d), rand(n, d)
    eta = np.abs(rand(n)) + 0.1

    def L(Wd):
        return orc.loss_value(loss, orc.inner_forward(kind, Wd, X)[0], V, eta)

    Vhat, cache = orc.inner_forward(kind, W, X)
    G = orc.inner_backward(kind, W, cache, orc.loss_grad(loss, Vhat, V, eta))
    eps = 1e-6
    for name, M in W.items():
        fd = np.zeros_like(M)
        for idx in np.ndindex(M.shape):
            Wp = {k: v.copy() for k, v in W.items()}
            Wm = {k: v.copy() for k, v in W.items()}
            Wp[name][idx] += eps
            Wm[name][idx] -= eps
            fd[idx] = (L(Wp) - L(Wm)) / (2 * eps)
        rel = np.linalg.norm(fd - G[name]) / np.linalg.norm(G[name])
        assert rel < 1e-7, (name, rel)


# ---------------------------------------------------------------- closed forms
def _linear_attention_state(W0, K, V, eta):
    """W0 + sum_i eta_i v_i k_i^T, accumulated token by token with outer products."""
    W = W0.copy()
    for i in range(K.shape[0]):
        W += eta[i] * np.outer(V[i], K[i])
    return W


@pytest.mark.parametrize("chunk", [0, 3, 5, 16])
def test_linear_dot_is_linear_attention(chunk):
    # linear inner model + negative dot loss + plain step: W* = W0 + V^T diag(eta) K and O = Q W*^T,
    # whatever the chunking, because the gradient does not depend on W.
    d, n = 5, 16
    cfg = cfg_for("linear", "neg_dot", d=d, h=d, N=n, chunk=chunk)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n))
    W0 = rand(d, d)
    O, Ws = orc.forward_head(cfg, Q, K, V, eta, W0.reshape(-1))
    Wref = _linear_attention_state(W0, K, V, eta)
    assert np.allclose(Ws.reshape(d, d), Wref, rtol=1e-12, atol=1e-12)
    Oref = np.array([[sum(Wref[r, c] * Q[i, c] for c in range(d)) for r in range(d)] for i in range(n)])
    assert np.allclose(O, Oref, rtol=1e-12, atol=1e-12)


def test_linear_dot_causal_is_chunkwise_causal_linear_attention():
    d, n, C = 4, 10, 3
    cfg = cfg_for("linear", "neg_dot", d=d, h=d, N=n, chunk=C, causal=1)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n))
    W0 = rand(d, d)
    O, Ws = orc.forward_head(cfg, Q, K, V, eta, W0.reshape(-1))
    for s in range(0, n, C):
        Wc = _linear_attention_state(W0, K[:s], V[:s], eta[:s])  # only earlier chunks
        for i in range(s, min(s + C, n)):
            assert np.allclose(O[i], Wc @ Q[i], rtol=1e-12, atol=1e-12)
    assert np.allclose(Ws.reshape(d, d), _linear_attention_state(W0, K, V, eta), rtol=1e-12, atol=1e-12)


def test_linear_mse_closed_form():
    # V_hat = K W0^T; dL/dV_hat = 2 eta (V_hat - V)/(n d); W* = W0 - sum_i 2 eta_i/(n d) (W0 k_i - v_i) k_i^T
    d, n = 4, 9
    cfg = cfg_for("linear", "mse", d=d, h=d, N=n)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n))
    W0 = rand(d, d)
    _, Ws = orc.forward_head(cfg, Q, K, V, eta, W0.reshape(-1))
    G = np.zeros((d, d))
    for i in range(n):
        G += 2.0 * eta[i] / (n * d) * np.outer(W0 @ K[i] - V[i], K[i])
    assert np.allclose(Ws.reshape(d, d), W0 - G, rtol=1e-12, atol=1e-12)


def test_linear_mse_eta_is_a_rescaling_of_k_and_v():
    # ViT3 digest, guideline 3: for a linear inner model with MSE, eta is equivalent to scaling K and V.
    # With W0 = 0:  O(eta * a * b; K, V) == O(eta; a K, b V).
    d, n, a, b, eta0 = 4, 7, 1.7, -0.6, 0.8
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    W0 = np.zeros(d * d)
    c1 = cfg_for("linear", "mse", d=d, h=d, N=n, eta_mode="scalar", eta_scalar=eta0 * a * b)
    c2 = cfg_for("linear", "mse", d=d, h=d, N=n, eta_mode="scalar", eta_scalar=eta0)
    O1, _ = orc.forward_head(c1, Q, K, V, None, W0)
    O2, _ = orc.forward_head(c2, Q, a * K, b * V, None, W0)
    assert np.allclose(O1, O2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["neg_dot", "mse", "rmse"])
def test_hand_worked_linear_example(repo_root, name):
    g = json.load(open(os.path.join(repo_root, "tests", "golden", "linear_two_tokens.json")))
    d = g["d"]
    K, V, eta = np.array(g["K"], float), np.array(g["V"], float), np.array(g["eta"], float)
    W0 = np.array(g["W0"], float)
    q = np.array(g["q"], float)[None, :]
    cfg = cfg_for("linear", name, d=d, h=d, N=2, Nq=1)
    O, Ws = orc.forward_head(cfg, q, K, V, eta, W0.reshape(-1))
    case = g["cases"][name]
    assert np.allclose(Ws.reshape(d, d), np.array(case["W_star"]), rtol=0, atol=1e-14)
    assert np.allclose(O[0], np.array(case["O"]), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- special cases
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("loss", LOSSES)
@pytest.mark.parametrize("rownorm", [False, True])
def test_eta_zero_reduces_to_initial_weights(kind, loss, rownorm):
    d, h, n = 4, 6, 9
    cfg = cfg_for(kind, loss, d=d, h=h, N=n, eta_mode="scalar", eta_scalar=0.0, weight_l2norm=rownorm,
                  key_instnorm=True)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    W = rand_w(kind, d, h)
    w0 = orc.pack(kind, d, h, W)
    O, Ws = orc.forward_head(cfg, Q, K, V, None, w0)
    Wexp = {k: (orc.row_l2_normalize(v) if rownorm else v) for k, v in W.items()}
    assert np.allclose(Ws, orc.pack(kind, d, h, Wexp), rtol=1e-14, atol=1e-14)
    for i in range(n):
        assert np.allclose(O[i], _brute_forward(kind, Wexp, Q[i].tolist()), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("opt", ["gd", "momentum", "muon", "momentum_muon"])
def test_causal_with_chunk_n_equals_single_chunk(kind, opt):
    # apply-before-update: W* is that of the non-causal single chunk; O reads W0 (reading R16).
    d, h, n = 4, 6, 10
    kw = dict(d=d, h=h, N=n, opt=opt, weight_l2norm=True)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n)) * 0.1
    W = rand_w(kind, d, h)
    w0 = orc.pack(kind, d, h, W)
    Oc, Wc = orc.forward_head(cfg_for(kind, "neg_dot", chunk=n, causal=1, **kw), Q, K, V, eta, w0)
    On, Wn = orc.forward_head(cfg_for(kind, "neg_dot", chunk=0, causal=0, **kw), Q, K, V, eta, w0)
    assert np.allclose(Wc, Wn, rtol=1e-13, atol=1e-13)
    for i in range(n):
        assert np.allclose(Oc[i], _brute_forward(kind, W, Q[i].tolist()), rtol=1e-12, atol=1e-12)


def test_causal_prefix_consistency():
    # the causal output of chunk c is F applied with the weights a non-causal chunked run
    # reaches on the first c chunks (no future leakage, LaCT analysis "Order of operations").
    kind, d, h, n, C = "swiglu", 4, 6, 12, 4
    kw = dict(d=d, h=h, opt="momentum", weight_l2norm=True)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n)) * 0.1
    w0 = orc.pack(kind, d, h, rand_w(kind, d, h))
    Oc, _ = orc.forward_head(cfg_for(kind, "neg_dot", N=n, chunk=C, causal=1, **kw), Q, K, V, eta, w0)
    for c in range(1, n // C):
        s = c * C
        cfgp = cfg_for(kind, "neg_dot", N=s, Nq=C, chunk=C, causal=0, **kw)
        Op, _ = orc.forward_head(cfgp, Q[s:s + C], K[:s], V[:s], eta[:s], w0)
        assert np.allclose(Oc[s:s + C], Op, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- optimizer pieces
def _quintic_on_singular_values(G, iters, coeff):
    a, b, c = coeff
    U, S, Vt = np.linalg.svd(G, full_matrices=False)
    s = S / (np.linalg.norm(G) + 1e-7)
    for _ in range(iters):
        s = a * s + b * s ** 3 + c * s ** 5
    return (U * s) @ Vt


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (7, 7)])
@pytest.mark.parametrize("iters", [0, 1, 5])
def test_newton_schulz_is_a_polynomial_of_the_singular_values(shape, iters):
    coeff = (3.4445, -4.7750, 2.0315)
    G = rand(*shape)
    X = orc.newton_schulz(G, iters, coeff)
    assert np.allclose(X, _quintic_on_singular_values(G, iters, coeff), rtol=1e-10, atol=1e-12)


def test_newton_schulz_orientation_and_zero_iterations():
    coeff = (3.4445, -4.7750, 2.0315)
    G = rand(5, 9)
    assert np.allclose(orc.newton_schulz(G.T, 5, coeff), orc.newton_schulz(G, 5, coeff).T, rtol=1e-12, atol=1e-14)
    assert np.allclose(orc.newton_schulz(G, 0, coeff), G / (np.linalg.norm(G) + 1e-7), rtol=1e-14, atol=0)


def test_newton_schulz_cubic_converges_to_polar_factor():
    # classical cubic (1.5, -0.5, 0) on a well-conditioned matrix converges to U V^T
    U, _ = np.linalg.qr(rand(6, 6))
    Vt = np.linalg.qr(rand(9, 9))[0][:6]
    G = (U * np.linspace(0.3, 1.0, 6)) @ Vt
    X = orc.newton_schulz(G, 40, (1.5, -0.5, 0.0))
    assert np.allclose(X @ X.T, np.eye(6), atol=1e-10)
    assert np.allclose(X, U @ Vt, atol=1e-10)


def test_momentum_two_chunk_closed_form():
    # linear + dot: the chunk gradient G_c = -sum eta_i v_i k_i^T does not depend on W, so
    # W1 = W0 - G0 and W2 = W1 - (beta G0 + G1).
    d, n, C, beta = 3, 8, 4, 0.9
    cfg = cfg_for("linear", "neg_dot", d=d, h=d, N=n, chunk=C, opt="momentum", momentum=beta)
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n))
    W0 = rand(d, d)
    _, Ws = orc.forward_head(cfg, Q, K, V, eta, W0.reshape(-1))
    G0 = -sum(eta[i] * np.outer(V[i], K[i]) for i in range(C))
    G1 = -sum(eta[i] * np.outer(V[i], K[i]) for i in range(C, n))
    W2 = (W0 - G0) - (beta * G0 + G1)
    assert np.allclose(Ws.reshape(d, d), W2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_momentum_zero_is_plain_step(kind):
    d, h, n = 4, 6, 12
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n)) * 0.3
    w0 = orc.pack(kind, d, h, rand_w(kind, d, h))
    a = orc.forward_head(cfg_for(kind, "neg_dot", N=n, chunk=4, opt="momentum", momentum=0.0), Q, K, V, eta, w0)
    b = orc.forward_head(cfg_for(kind, "neg_dot", N=n, chunk=4, opt="gd"), Q, K, V, eta, w0)
    assert np.allclose(a[0], b[0], rtol=1e-13, atol=1e-13) and np.allclose(a[1], b[1], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("kind", KINDS)
def test_row_norm_gives_unit_rows_and_is_idempotent(kind):
    d, h, n = 4, 6, 9
    cfg = cfg_for(kind, "neg_dot", d=d, h=h, N=n, weight_l2norm=True, opt="muon")
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    _, Ws = orc.forward_head(cfg, Q, K, V, np.abs(rand(n)), orc.pack(kind, d, h, rand_w(kind, d, h)))
    W = orc.unpack(kind, d, h, Ws)
    for name, M in W.items():
        assert np.allclose(np.sqrt((M * M).sum(axis=1)), 1.0, atol=1e-13), name
        assert np.allclose(orc.row_l2_normalize(M), M, atol=1e-15)


# ---------------------------------------------------------------- instance norm
def test_instance_norm_moments():
    K = rand(50, 6) * 3 + 2
    Kt = orc.instance_norm(K, 0.0)
    assert np.allclose(Kt.mean(axis=0), 0.0, atol=1e-13)
    assert np.allclose((Kt ** 2).mean(axis=0), 1.0, atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
def test_key_instance_norm_removes_per_channel_shift_and_scale(kind):
    # TTT vs Sleep, "Side one": a constant per-channel key shift must not change the layer.
    d, h, n = 5, 6, 11
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    w0 = orc.pack(kind, d, h, rand_w(kind, d, h))
    cfg = cfg_for(kind, "mse", d=d, h=h, N=n, key_instnorm=True, in_eps=0.0, eta_mode="scalar")
    O1, W1 = orc.forward_head(cfg, Q, K, V, None, w0)
    shift = rand(1, d) * 5
    O2, W2 = orc.forward_head(cfg, Q, K + shift, V, None, w0)
    scale = np.abs(rand(1, d)) + 0.5
    O3, W3 = orc.forward_head(cfg, Q, K * scale, V, None, w0)
    for O, Wx in ((O2, W2), (O3, W3)):
        assert np.allclose(O, O1, rtol=1e-10, atol=1e-10)
        assert np.allclose(Wx, W1, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- token-set semantics
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("loss", LOSSES)
def test_single_chunk_is_invariant_to_token_permutation(kind, loss):
    # LaCT analysis, "Nonlinear memory": a large-chunk update treats the tokens as a set.
    d, h, n = 4, 6, 13
    Q, K, V = rand(n, d), rand(n, d), rand(n, d)
    eta = np.abs(rand(n))
    w0 = orc.pack(kind, d, h, rand_w(kind, d, h))
    cfg = cfg_for(kind, loss, d=d, h=h, N=n, key_instnorm=True, weight_l2norm=True, opt="muon")
    O1, W1 = orc.forward_head(cfg, Q, K, V, eta, w0)
    p = RNG.permutation(n)
    O2, W2 = orc.forward_head(cfg, Q, K[p], V[p], eta[p], w0)
    assert np.allclose(O1, O2, rtol=1e-11, atol=1e-11) and np.allclose(W1, W2, rtol=1e-11, atol=1e-11)


def test_chunk_bounds_cover_tokens_once():
    assert orc.chunk_bounds(10, 0) == [(0, 10)]
    assert orc.chunk_bounds(10, 10) == [(0, 10)]
    assert orc.chunk_bounds(10, 4) == [(0, 4), (4, 8), (8, 10)]
    b = orc.chunk_bounds(1029120, 131072)
    assert len(b) == 8 and b[-1] == (917504, 1029120) and b[-1][1] - b[-1][0] == 111616


def test_forward_all_heads_matches_per_head():
    cfg = make_config(B=2, H=2, N=9, d=4, h=6, inner="swiglu", loss="neg_dot", opt="momentum",
                      chunk=4, eta_mode="per_token", dtype="f32", data="lact")
    from synth_inputs import gen_inputs
    x = gen_inputs(cfg)
    O, W = orc.forward(cfg, x["Q"], x["K"], x["V"], x["eta"], x["W0"])
    for b in range(2):
        for hh in range(2):
            o, w = orc.forward_head(cfg, x["Q"][b, hh].double().numpy(), x["K"][b, hh].double().numpy(),
                                    x["V"][b, hh].double().numpy(), x["eta"][b, hh].double().numpy(),
                                    x["W0"][hh].double().numpy())
            assert np.array_equal(O[b, hh], o) and np.array_equal(W[b, hh], w)


# ---------------------------------------------------------------- inner epochs
@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("rownorm", [False, True])
def test_epochs_are_repeated_full_batch_steps(kind, rownorm):
    # plain GD (no state carried between calls): E epochs over one chunk equal E calls
    # that each take one step, the next starting from the previous call's W*
    d, h, N = 4, 6, 9
    cfg1 = cfg_for(kind, "mse", d=d, h=h, N=N, weight_l2norm=rownorm)
    cfg3 = cfg_for(kind, "mse", d=d, h=h, N=N, weight_l2norm=rownorm, epochs=3)
    Q, K, V, eta = rand(1, 1, N, d), rand(1, 1, N, d), rand(1, 1, N, d), np.abs(rand(1, 1, N, scale=0.3))
    W = orc.pack(kind, d, h, rand_w(kind, d, h))[None]
    O3, W3 = orc.forward(cfg3, Q, K, V, eta, W)
    Wi = W
    for _ in range(3):
        Oi, Wstep = orc.forward(cfg1, Q, K, V, eta, Wi)
        Wi = Wstep[:, 0]
    assert np.allclose(W3[:, 0], Wi, rtol=1e-12, atol=1e-12)
    assert np.allclose(O3, Oi, rtol=1e-12, atol=1e-12)
    # and one epoch is the default
    O1, W1 = orc.forward(cfg1, Q, K, V, eta, W)
    O1b, W1b = orc.forward(cfg_for(kind, "mse", d=d, h=h, N=N, weight_l2norm=rownorm, epochs=1), Q, K, V, eta, W)
    assert np.array_equal(W1, W1b) and np.array_equal(O1, O1b)


# ---------------------------------------------------------------- streaming state
def _data(B, H, N, d, scale=0.3):
    return (rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d), np.abs(rand(B, H, N, scale=scale)))


@pytest.mark.parametrize("kind", KINDS)
def test_w0_per_batch_with_equal_states_matches_shared_w0(kind):
    d, h, N, B, H = 4, 6, 7, 2, 2
    Q, K, V, eta = _data(B, H, N, d)
    W0 = np.stack([orc.pack(kind, d, h, rand_w(kind, d, h)) for _ in range(H)])
    cfg = dict(B=B, H=H, d=d, h=h, N=N, opt="momentum", weight_l2norm=True)
    Os, Ws = orc.forward(cfg_for(kind, "neg_dot", **cfg), Q, K, V, eta, W0)
    Ob, Wb = orc.forward(cfg_for(kind, "neg_dot", w0_per_batch=True, **cfg), Q, K, V, eta,
                         np.broadcast_to(W0, (B, H, W0.shape[1])))
    assert np.array_equal(Os, Ob) and np.array_equal(Ws, Wb)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("causal", [0, 1])
def test_no_update_reads_the_initial_weights(kind, causal):
    d, h, N = 4, 6, 9
    Q, K, V, eta = _data(1, 1, N, d)
    w = rand_w(kind, d, h)
    W0 = orc.pack(kind, d, h, w)[None]
    cfg = cfg_for(kind, "mse", d=d, h=h, N=N, chunk=4, causal=causal, no_update=True, weight_l2norm=True,
                  opt="momentum")
    O, W = orc.forward(cfg, Q, K, V, eta, W0)
    assert np.array_equal(W[0, 0], W0[0])
    assert np.allclose(O[0, 0], orc.inner_forward(kind, w, Q[0, 0])[0], rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("causal", [0, 1])
def test_streaming_two_calls_equal_one_chunked_call(kind, causal):
    # plain GD: the state is the weights alone, so feeding W_out of a call on the first half
    # of the tokens back as W0 of a call on the second half gives the one-call result
    d, h, N, B, H = 4, 6, 12, 2, 1
    Q, K, V, eta = _data(B, H, N, d)
    W0 = orc.pack(kind, d, h, rand_w(kind, d, h))[None]
    half = N // 2
    base = dict(B=B, H=H, d=d, h=h, weight_l2norm=True, causal=causal)
    O1, W1 = orc.forward(cfg_for(kind, "neg_dot", N=N, chunk=half, **base), Q, K, V, eta, W0)
    sl = lambda t, a, b: t[:, :, a:b]
    qa = sl(Q, 0, half) if causal else Q
    qb = sl(Q, half, N) if causal else Q
    Oa, Wa = orc.forward(cfg_for(kind, "neg_dot", N=half, Nq=qa.shape[2], **base), qa, sl(K, 0, half),
                         sl(V, 0, half), sl(eta, 0, half), W0)
    Ob, Wb = orc.forward(cfg_for(kind, "neg_dot", N=half, Nq=qb.shape[2], w0_per_batch=True, **base), qb,
                         sl(K, half, N), sl(V, half, N), sl(eta, half, N), Wa)
    assert np.allclose(Wb, W1, rtol=1e-12, atol=1e-12)
    if causal:
        assert np.allclose(np.concatenate([Oa, Ob], axis=2), O1, rtol=1e-12, atol=1e-12)
    else:
        assert np.allclose(Ob, O1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("opt", ["momentum", "momentum_muon"])
def test_streaming_with_momentum_state_equals_one_chunked_call(kind, causal, opt):
    # with momentum the state is (W, M): handing both to the call on the second half
    # gives the one-call result, as momentum is carried across chunks (reading R9)
    d, h, N, B, H = 4, 6, 12, 2, 1
    Q, K, V, eta = _data(B, H, N, d)
    W0 = orc.pack(kind, d, h, rand_w(kind, d, h))[None]
    half = N // 2
    base = dict(B=B, H=H, d=d, h=h, weight_l2norm=True, causal=causal, opt=opt, ns_iters=3)
    O1, W1, M1 = orc.forward(cfg_for(kind, "neg_dot", N=N, chunk=half, **base), Q, K, V, eta, W0, return_m=True)
    sl = lambda t, a, b: t[:, :, a:b]
    qa = sl(Q, 0, half) if causal else Q
    qb = sl(Q, half, N) if causal else Q
    Oa, Wa, Ma = orc.forward(cfg_for(kind, "neg_dot", N=half, Nq=qa.shape[2], **base), qa, sl(K, 0, half),
                             sl(V, 0, half), sl(eta, 0, half), W0, return_m=True)
    Ob, Wb, Mb = orc.forward(cfg_for(kind, "neg_dot", N=half, Nq=qb.shape[2], w0_per_batch=True, **base), qb,
                             sl(K, half, N), sl(V, half, N), sl(eta, half, N), Wa, M0=Ma, return_m=True)
    assert np.allclose(Wb, W1, rtol=1e-12, atol=1e-12) and np.allclose(Mb, M1, rtol=1e-12, atol=1e-12)
    O2 = np.concatenate([Oa, Ob], axis=2) if causal else Ob
    assert np.allclose(O2, O1, rtol=1e-12, atol=1e-12)
    # without the momentum handed over the second call restarts it at zero: a different result
    _, Wc = orc.forward(cfg_for(kind, "neg_dot", N=half, Nq=qb.shape[2], w0_per_batch=True, **base), qb,
                        sl(K, half, N), sl(V, half, N), sl(eta, half, N), Wa)
    assert not np.allclose(Wc, W1, rtol=1e-6, atol=1e-9)


def test_momentum_state_of_the_linear_dot_layer_in_closed_form():
    # linear + dot: every chunk's gradient is -sum_i eta_i v_i k_i^T whatever W is, so
    # M after chunks 1 and 2 is beta (-V1^T E1 K1) + (-V2^T E2 K2), token by token
    d, N, C, beta = 3, 10, 4, 0.7
    Q, K, V, eta = rand(2, d), rand(N, d), rand(N, d), np.abs(rand(N)) + 0.1
    M0 = rand(d * d)
    cfg = cfg_for("linear", "neg_dot", opt="momentum", momentum=beta, d=d, N=N, chunk=C)
    _, _, m = orc.forward_head(cfg, Q, K, V, eta, rand(d * d), m0=M0, return_m=True)
    M = M0.reshape(d, d).copy()
    for s in range(0, N, C):
        G = np.zeros((d, d))
        for i in range(s, min(s + C, N)):
            for r in range(d):
                for c in range(d):
                    G[r, c] -= eta[i] * V[i, r] * K[i, c]
        M = beta * M + G
    assert np.allclose(m, M.reshape(-1), rtol=1e-13, atol=1e-13)
    _, _, mg = orc.forward_head(dict(cfg, opt="gd"), Q, K, V, eta, rand(d * d), return_m=True)
    assert np.array_equal(mg, np.zeros(d * d))


# ---------------------------------------------------------------- first layer only (SD3.5-T5 layer)
def _run(cfg, Q, K, V, eta, w0):
    return orc.forward_head(cfg, Q, K, V, eta, w0)


@pytest.mark.parametrize("kind", ["mlp2_gelu", "swiglu"])
@pytest.mark.parametrize("opt", ["gd", "momentum", "muon", "momentum_muon"])
@pytest.mark.parametrize("rownorm", [False, True])
def test_first_layer_only_keeps_w2_and_takes_the_same_first_layer_step(kind, opt, rownorm):
    # one chunk: every matrix's gradient is taken at W0, so freezing W2 leaves the
    # first layer's step unchanged; W2 must come back bit for bit
    d, h, n = 4, 6, 9
    cfg = cfg_for(kind, "neg_dot", opt=opt, weight_l2norm=rownorm, d=d, h=h, N=n, ns_iters=3)
    W0 = rand_w(kind, d, h)
    w0 = orc.pack(kind, d, h, W0)
    Q, K, V, eta = rand(5, d), rand(n, d), rand(n, d), np.abs(rand(n)) + 0.1
    _, wf = _run(cfg, Q, K, V, eta, w0)
    O1, w1 = _run(dict(cfg, first_layer_only=True), Q, K, V, eta, w0)
    Wf, W1 = orc.unpack(kind, d, h, wf), orc.unpack(kind, d, h, w1)
    assert np.array_equal(W1["W2"], W0["W2"])
    for name in W0:
        if name != "W2":
            assert np.allclose(W1[name], Wf[name], rtol=1e-13, atol=1e-13), name
    assert np.allclose(O1, orc.inner_forward(kind, W1, Q)[0], rtol=1e-13, atol=1e-13)


def test_first_layer_only_changes_nothing_for_the_linear_model():
    d, n = 5, 7
    cfg = cfg_for("linear", "mse", opt="momentum_muon", weight_l2norm=True, d=d, N=n, chunk=3, ns_iters=2)
    w0 = rand(d * d)
    Q, K, V, eta = rand(n, d), rand(n, d), rand(n, d), np.abs(rand(n)) + 0.1
    O0, w_a = _run(cfg, Q, K, V, eta, w0)
    O1, w_b = _run(dict(cfg, first_layer_only=True), Q, K, V, eta, w0)
    assert np.array_equal(O0, O1) and np.array_equal(w_a, w_b)


@pytest.mark.parametrize("kind", ["mlp2_gelu", "swiglu"])
@pytest.mark.parametrize("loss", LOSSES)
def test_first_layer_only_chunks_step_on_finite_difference_gradients(kind, loss):
    # two chunks of plain gradient steps, checked against central finite differences
    # of each chunk's loss in the first-layer matrices, with W2 held at W0
    d, h, n, C = 3, 4, 8, 4
    cfg = cfg_for(kind, loss, d=d, h=h, N=n, chunk=C)
    W = rand_w(kind, d, h)
    w0 = orc.pack(kind, d, h, W)
    Q, K, V, eta = rand(3, d), rand(n, d), rand(n, d), np.abs(rand(n)) + 0.1
    _, w_or = _run(dict(cfg, first_layer_only=True), Q, K, V, eta, w0)
    eps = 1e-6
    for s in range(0, n, C):
        Kc, Vc, ec = K[s:s + C], V[s:s + C], eta[s:s + C]

        def L(Wd):
            return orc.loss_value(loss, orc.inner_forward(kind, Wd, Kc)[0], Vc, ec)

        step = {}
        for name, M in W.items():
            if name == "W2":
                continue
            g = np.zeros_like(M)
            for idx in np.ndindex(M.shape):
                Wp = {k: v.copy() for k, v in W.items()}
                Wm = {k: v.copy() for k, v in W.items()}
                Wp[name][idx] += eps
                Wm[name][idx] -= eps
                g[idx] = (L(Wp) - L(Wm)) / (2 * eps)
            step[name] = M - g
        W.update(step)
    assert np.allclose(w_or, orc.pack(kind, d, h, W), rtol=1e-7, atol=1e-8)


# ---------------------------------------------------------------- simplified GLU (ViT3's F1)
def _glu_as_swiglu(Wg, d):
    """The GLU's matrices as a SwiGLU with h = d: W1 = Wb (gate), W3 = Wa, W2 = I."""
    return {"W1": Wg["Wb"], "W3": Wg["Wa"], "W2": np.eye(d)}


@pytest.mark.parametrize("opt", ["gd", "momentum", "muon", "momentum_muon"])
@pytest.mark.parametrize("causal,chunk,rownorm", [(0, 0, False), (0, 4, True), (1, 3, True), (1, 0, False)])
def test_glu_is_a_swiglu_with_identity_w2_and_first_layer_only(opt, causal, chunk, rownorm):
    d, n = 4, 10
    cfg = cfg_for("glu", "neg_dot", opt=opt, weight_l2norm=rownorm, d=d, h=d, N=n, chunk=chunk, causal=causal,
                  ns_iters=3)
    Wg = rand_w("glu", d, d)
    Q, K, V, eta = rand(n, d), rand(n, d), rand(n, d), np.abs(rand(n)) + 0.1
    Og, wg = _run(cfg, Q, K, V, eta, orc.pack("glu", d, d, Wg))
    Ws0 = _glu_as_swiglu(Wg, d)
    Os, ws = _run(dict(cfg, inner="swiglu", first_layer_only=True), Q, K, V, eta, orc.pack("swiglu", d, d, Ws0))
    Wgs, Wss = orc.unpack("glu", d, d, wg), orc.unpack("swiglu", d, d, ws)
    assert np.allclose(Og, Os, rtol=1e-12, atol=1e-12)
    assert np.allclose(Wss["W1"], Wgs["Wb"], rtol=1e-12, atol=1e-12)
    assert np.allclose(Wss["W3"], Wgs["Wa"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(Wss["W2"], np.eye(d))


def test_glu_dot_step_in_closed_form():
    # one GD step of the dot loss written out per token:
    #   Wa += sum_i eta_i (v_i * SiLU(zb_i)) k_i^T
    #   Wb += sum_i eta_i (v_i * za_i * SiLU'(zb_i)) k_i^T
    # with SiLU'(z) from the quotient rule on z / (1 + e^-z), evaluated by math.exp
    d, n = 3, 6
    Wg = rand_w("glu", d, d)
    K, V, eta = rand(n, d), rand(n, d), np.abs(rand(n)) + 0.1
    Wa, Wb = Wg["Wa"].copy(), Wg["Wb"].copy()
    for i in range(n):
        za, zb = Wg["Wa"] @ K[i], Wg["Wb"] @ K[i]
        s = np.array([z / (1 + math.exp(-z)) for z in zb])
        ds = np.array([(1 + math.exp(-z) + z * math.exp(-z)) / (1 + math.exp(-z)) ** 2 for z in zb])
        Wa += eta[i] * np.outer(V[i] * s, K[i])
        Wb += eta[i] * np.outer(V[i] * za * ds, K[i])
    cfg = cfg_for("glu", "neg_dot", d=d, h=d, N=n)
    _, w = _run(cfg, rand(2, d), K, V, eta, orc.pack("glu", d, d, Wg))
    W = orc.unpack("glu", d, d, w)
    assert np.allclose(W["Wa"], Wa, rtol=1e-13, atol=1e-13)
    assert np.allclose(W["Wb"], Wb, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- RMSE loss (ViT3 inner-loss table)
def test_rmse_textbook_value():
    # errors 1, 2, 3, 4 over n = 2 tokens, d = 2 channels: sqrt((1 + 4 + 9 + 16) / 4)
    Vhat = np.array([[1.0, 2.0], [3.0, 4.0]])
    V = np.zeros((2, 2))
    assert orc.loss_value("rmse", Vhat, V, np.ones(2)) == math.sqrt(7.5)
    # eta weights each token's squared error inside the root
    assert abs(orc.loss_value("rmse", Vhat, V, np.array([2.0, 0.0])) - math.sqrt(2 * 5 / 4)) < 1e-15


def test_rmse_gradient_has_norm_one_over_sqrt_nd():
    # with eta = 1, dL/dV_hat = (V_hat - V) / (n d RMSE), whose Frobenius norm is
    # ||V_hat - V|| / (n d ||V_hat - V|| / sqrt(n d)) = 1 / sqrt(n d) for any data
    for n, d in ((3, 5), (17, 4)):
        g = orc.loss_grad("rmse", rand(n, d), rand(n, d), np.ones(n))
        assert abs(np.linalg.norm(g) - 1.0 / math.sqrt(n * d)) < 1e-14


@pytest.mark.parametrize("kind", KINDS)
def test_rmse_at_zero_error_takes_no_step(kind):
    # values the inner model already reproduces exactly: the MSE is 0 and the step is 0
    d, h, n = 4, 6, 7
    W = rand_w(kind, d, h)
    K = rand(n, d)
    V = orc.inner_forward(kind, W, K)[0]
    cfg = cfg_for(kind, "rmse", d=d, h=h, N=n)
    _, w = orc.forward_head(cfg, rand(2, d), K, V, np.abs(rand(n)) + 0.1, orc.pack(kind, d, h, W))
    assert np.array_equal(w, orc.pack(kind, d, h, W))


# ---------------------------------------------------------------- DWConv (ViT3's F2 module)
def _dw_cfg(loss, gh, gw, d, k=3, **kw):
    return cfg_for("dwconv", loss, d=d, h=d, N=gh * gw, grid_h=gh, grid_w=gw, ksize=k, **kw)


def _brute_dwconv(Wc, X, gh, gw, k):
    """Scalar loops: every output pixel and channel sums its k x k neighbours that lie on the grid."""
    r = k // 2
    out = []
    for y in range(gh):
        for x in range(gw):
            row = []
            for c in range(X.shape[1]):
                s = 0.0
                for a in range(k):
                    for b in range(k):
                        yy, xx = y + a - r, x + b - r
                        if 0 <= yy < gh and 0 <= xx < gw:
                            s += float(Wc[c, a * k + b]) * float(X[yy * gw + xx, c])
                row.append(s)
            out.append(row)
    return np.array(out)


@pytest.mark.parametrize("gh,gw,k", [(4, 5, 3), (1, 7, 3), (3, 3, 5), (2, 6, 1)])
def test_dwconv_forward_matches_scalar_loops(gh, gw, k):
    d = 3
    Wc, X = rand(d, k * k), rand(gh * gw, d)
    Y = orc.inner_forward("dwconv", {"Wc": Wc}, X, (gh, gw))[0]
    assert np.allclose(Y, _brute_dwconv(Wc, X, gh, gw, k), rtol=1e-13, atol=1e-13)


def test_dwconv_forward_and_weight_gradient_match_scipy_correlate2d():
    # per channel: the layer is a 'same' 2-D cross-correlation with zero fill, and the kernel
    # gradient is the 'valid' cross-correlation of the zero-padded input with dL/dY
    from scipy.signal import correlate2d

    gh, gw, d, k = 5, 6, 4, 3
    Wc, X, dY = rand(d, k * k), rand(gh * gw, d), rand(gh * gw, d)
    Y = orc.inner_forward("dwconv", {"Wc": Wc}, X, (gh, gw))[0]
    G = orc.inner_backward("dwconv", {"Wc": Wc}, {"X": X, "grid": (gh, gw)}, dY)["Wc"]
    for c in range(d):
        Xc = X[:, c].reshape(gh, gw)
        ref = correlate2d(Xc, Wc[c].reshape(k, k), mode="same", boundary="fill", fillvalue=0.0)
        assert np.allclose(Y[:, c].reshape(gh, gw), ref, rtol=1e-13, atol=1e-13)
        Xpad = np.pad(Xc, 1)
        gref = correlate2d(Xpad, dY[:, c].reshape(gh, gw), mode="valid")
        assert np.allclose(G[c].reshape(k, k), gref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("loss", LOSSES)
def test_dwconv_gradients_by_central_finite_differences(loss):
    gh, gw, d, k = 3, 4, 2, 3
    W = {"Wc": rand(d, k * k)}
    X, V = rand(gh * gw, d), rand(gh * gw, d)
    eta = np.abs(rand(gh * gw)) + 0.1
    grid = (gh, gw)

    def L(Wd):
        return orc.loss_value(loss, orc.inner_forward("dwconv", Wd, X, grid)[0], V, eta)

    Vhat, cache = orc.inner_forward("dwconv", W, X, grid)
    G = orc.inner_backward("dwconv", W, cache, orc.loss_grad(loss, Vhat, V, eta))["Wc"]
    fd = np.zeros_like(G)
    eps = 1e-6
    for idx in np.ndindex(G.shape):
        Wp, Wm = {"Wc": W["Wc"].copy()}, {"Wc": W["Wc"].copy()}
        Wp["Wc"][idx] += eps
        Wm["Wc"][idx] -= eps
        fd[idx] = (L(Wp) - L(Wm)) / (2 * eps)
    assert np.linalg.norm(fd - G) / np.linalg.norm(G) < 1e-7


@pytest.mark.parametrize("loss", LOSSES)
def test_dwconv_with_one_tap_is_the_diagonal_of_the_linear_model(loss):
    # k = 1: each channel is scaled by its own weight, i.e. the linear model with a diagonal W;
    # one gradient step moves the diagonal of the linear model's W by the same amount
    gh, gw, d = 3, 5, 4
    w0 = rand(d)
    Q, K, V, eta = rand(gh * gw, d), rand(gh * gw, d), rand(gh * gw, d), np.abs(rand(gh * gw)) + 0.1
    Od, wd = orc.forward_head(_dw_cfg(loss, gh, gw, d, k=1), Q, K, V, eta, w0)
    _, wl = orc.forward_head(cfg_for("linear", loss, d=d, N=gh * gw), Q, K, V, eta, np.diag(w0).reshape(-1))
    assert np.allclose(wd, np.diag(wl.reshape(d, d)), rtol=1e-13, atol=1e-13)
    assert np.allclose(Od, Q * wd, rtol=1e-13, atol=1e-13)


def test_dwconv_layer_reads_the_grid_once_as_one_chunk():
    gh, gw, d = 3, 4, 2
    Q, K, V, eta = rand(gh * gw, d), rand(gh * gw, d), rand(gh * gw, d), np.abs(rand(gh * gw)) + 0.1
    w0 = rand(d * 9)
    with pytest.raises(ValueError):
        orc.forward_head(_dw_cfg("neg_dot", gh, gw, d, chunk=4), Q, K, V, eta, w0)
    with pytest.raises(ValueError):
        orc.forward_head(_dw_cfg("neg_dot", gh, gw, d, causal=1), Q, K, V, eta, w0)
    with pytest.raises(ValueError):
        orc.forward_head(_dw_cfg("neg_dot", gh, gw + 1, d), Q, K, V, eta, w0)
    # the ViT3 recipe: dot loss, one full-batch step, rate 1 -> W* = W0 + sum_p eta_p v_p (x) shifted k_p
    O, w = orc.forward_head(_dw_cfg("neg_dot", gh, gw, d, eta_mode="scalar"), Q, K, V, None, w0)
    G = orc.dwconv_weight_grad(K, -V, (gh, gw), 3)
    assert np.allclose(w, w0 - G.reshape(-1), rtol=1e-13, atol=1e-13)
    assert np.allclose(O, _brute_dwconv(w.reshape(d, 9), Q, gh, gw, 3), rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- the same identities on drawn shapes
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None, derandomize=True)
@given(d=st.integers(1, 7), n=st.integers(1, 30), chunk=st.integers(0, 35), causal=st.booleans(),
       seed=st.integers(0, 2**31 - 1))
def test_linear_dot_is_chunkwise_linear_attention_on_drawn_shapes(d, n, chunk, causal, seed):
    # W_c = W0 + sum of eta_i v_i k_i^T over the tokens of the chunks before c (causal reads),
    # or over all tokens (non-causal), accumulated one outer product at a time
    rng = np.random.default_rng(seed)
    Q, K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    eta, W0 = np.abs(rng.standard_normal(n)), rng.standard_normal((d, d))
    cfg = cfg_for("linear", "neg_dot", d=d, h=d, N=n, chunk=chunk, causal=int(causal))
    O, Ws = orc.forward_head(cfg, Q, K, V, eta, W0.reshape(-1))
    C = n if chunk <= 0 or chunk >= n else chunk
    W = W0.copy()
    Oref = np.zeros((n, d))
    for s in range(0, n, C):
        if causal:
            Oref[s:s + C] = Q[s:s + C] @ W.T
        for i in range(s, min(s + C, n)):
            W += eta[i] * np.outer(V[i], K[i])
    if not causal:
        Oref = Q @ W.T
    assert np.allclose(Ws.reshape(d, d), W, rtol=1e-11, atol=1e-11)
    assert np.allclose(O, Oref, rtol=1e-11, atol=1e-11)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(d=st.integers(1, 5), n=st.integers(1, 12), opt=st.sampled_from(["gd", "momentum", "muon", "momentum_muon"]),
       chunk=st.integers(0, 14), causal=st.booleans(), rownorm=st.booleans(), seed=st.integers(0, 2**31 - 1))
def test_glu_is_a_swiglu_with_identity_w2_on_drawn_shapes(d, n, opt, chunk, causal, rownorm, seed):
    rng = np.random.default_rng(seed)
    Wg = {"Wa": rng.standard_normal((d, d)) * 0.5, "Wb": rng.standard_normal((d, d)) * 0.5}
    Q, K, V = rng.standard_normal((n, d)), rng.standard_normal((n, d)), rng.standard_normal((n, d))
    eta = np.abs(rng.standard_normal(n)) + 0.1
    cfg = cfg_for("glu", "neg_dot", opt=opt, weight_l2norm=rownorm, d=d, h=d, N=n, chunk=chunk, causal=int(causal),
                  ns_iters=2)
    Og, wg = orc.forward_head(cfg, Q, K, V, eta, orc.pack("glu", d, d, Wg))
    Ws0 = {"W1": Wg["Wb"], "W3": Wg["Wa"], "W2": np.eye(d)}
    Os, ws = orc.forward_head(dict(cfg, inner="swiglu", first_layer_only=True), Q, K, V, eta,
                              orc.pack("swiglu", d, d, Ws0))
    Wgs, Wss = orc.unpack("glu", d, d, wg), orc.unpack("swiglu", d, d, ws)
    assert np.allclose(Og, Os, rtol=1e-10, atol=1e-10)
    assert np.allclose(Wss["W1"], Wgs["Wb"], rtol=1e-10, atol=1e-10)
    assert np.allclose(Wss["W3"], Wgs["Wa"], rtol=1e-10, atol=1e-10)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(gh=st.integers(1, 9), gw=st.integers(1, 9), d=st.integers(1, 4), k=st.sampled_from([1, 3, 5, 7]),
       seed=st.integers(0, 2**31 - 1))
def test_dwconv_matches_scipy_correlate2d_on_drawn_shapes(gh, gw, d, k, seed):
    from scipy.signal import correlate2d

    rng = np.random.default_rng(seed)
    Wc, X, dY = rng.standard_normal((d, k * k)), rng.standard_normal((gh * gw, d)), rng.standard_normal((gh * gw, d))
    Y = orc.dwconv_apply(Wc, X, (gh, gw))
    G = orc.dwconv_weight_grad(X, dY, (gh, gw), k)
    for c in range(d):
        Xc = X[:, c].reshape(gh, gw)
        ref = correlate2d(Xc, Wc[c].reshape(k, k), mode="same", boundary="fill", fillvalue=0.0)
        assert np.allclose(Y[:, c].reshape(gh, gw), ref, rtol=1e-12, atol=1e-12)
        gref = correlate2d(np.pad(Xc, k // 2), dY[:, c].reshape(gh, gw), mode="valid")
        assert np.allclose(G[c].reshape(k, k), gref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["neg_dot", "mse"])
def test_hand_worked_dwconv_example(repo_root, name):
    g = json.load(open(os.path.join(repo_root, "tests", "golden", "dwconv_row_of_three.json")))
    gh, gw = g["grid"]
    col = lambda key: np.array(g[key], float)[:, None]  # one channel
    cfg = cfg_for("dwconv", name, d=1, h=1, N=gh * gw, grid_h=gh, grid_w=gw, ksize=g["ksize"])
    O, Ws = orc.forward_head(cfg, col("Q"), col("K"), col("V"), np.array(g["eta"], float), np.array(g["W0"], float))
    case = g["cases"][name]
    assert np.allclose(Ws, np.array(case["W_star"]), rtol=0, atol=1e-14)
    assert np.allclose(O[:, 0], np.array(case["O"]), rtol=0, atol=1e-14)


def test_hand_worked_glu_example(repo_root):
    g = json.load(open(os.path.join(repo_root, "tests", "golden", "glu_two_tokens.json")))
    col = lambda key: np.array(g[key], float)[:, None]
    cfg = cfg_for("glu", "neg_dot", d=1, h=1, N=2, Nq=1)
    O, Ws = orc.forward_head(cfg, col("q"), col("K"), col("V"), np.array(g["eta"], float),
                             np.array([g["Wa0"], g["Wb0"]], float))
    assert np.allclose(Ws, [g["Wa_star"], g["Wb_star"]], rtol=0, atol=1e-14)
    assert abs(O[0, 0] - 14.0 / (1.0 + math.exp(-7.0))) < 1e-13 and abs(O[0, 0] - g["O"]) < 1e-13
