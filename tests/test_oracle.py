"""Pins of the fp64 oracle against what the paper and the mathematics fix.

Paper: "Rethinking Expressivity and Efficiency in Test-Time Training" (E2-TTT).
  * abstract / atlas "Approach": the closed form reproduces EXACTLY the chunk-end
    states of the per-token recurrence with chunk-start gradients   -> P1
  * plain chunk-summed update when momentum is off and decay is 1    -> P2
  * geometric-series closed forms for constant gates                 -> P3
  * chunk size 1 is token-wise TTT (atlas "Limitations")            -> P4
  * hand-derived C=2 example (tests/golden)                          -> P5
  * finite differences of the per-token recurrence pin the backward  -> P6
  * gradients / VJPs of the fast MLP against finite differences      -> P7
"""
import json
import os

import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_case(kind, B=1, H=2, T=10, C=4, d_k=4, d_v=3, d_h=5, seed=0, m0=0.3,
               mom=(0.8, 0.99), decay=(0.9, 1.0), lr=(0.05, 0.5)):
    w = gen.Workload("t", kind, gen.F32, B, H, d_k, d_v, d_h if kind != O.LINEAR else 0, T, C,
                     "uniform", decay[0], seed=seed, lr_lo=lr[0], lr_hi=lr[1], mom_lo=mom[0],
                     mom_hi=mom[1], decay_hi=decay[1])
    x = gen.generate(w, m0_scale=m0)
    return w, x


def fwd_args(w, x):
    return (w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"], x["M0"], w.C)


# ------------------------------------------------------------------ P1: closed == per-token
@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
@pytest.mark.parametrize("T,C", [(12, 4), (11, 4), (9, 9), (7, 3)])
def test_closed_equals_sequential(kind, loss, T, C):
    w, x = small_case(kind, T=T, C=C, seed=T * 7 + C)
    o1, W1, M1 = O.seq_fwd(*fwd_args(w, x), d_h=w.d_h, loss=loss)
    o2, W2, M2 = O.closed_fwd(*fwd_args(w, x), d_h=w.d_h, loss=loss)
    assert O.rel_fro(o2, o1) < 1e-12
    assert O.rel_fro(W2, W1) < 1e-12
    assert O.rel_fro(M2, M1) < 1e-12


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
@pytest.mark.parametrize("edge", ["mu0", "lam1", "lam0", "mixed0"])
def test_closed_equals_sequential_gate_edges(kind, edge):
    w, x = small_case(kind, T=12, C=5, seed=3)
    if edge == "mu0":
        x["mom"][:] = 0.0
    elif edge == "lam1":
        x["decay"][:] = 1.0
    elif edge == "lam0":
        x["decay"][..., ::3] = 0.0
    else:
        x["mom"][..., 1::4] = 0.0
        x["decay"][..., 2::5] = 0.0
    o1, W1, M1 = O.seq_fwd(*fwd_args(w, x), d_h=w.d_h)
    o2, W2, M2 = O.closed_fwd(*fwd_args(w, x), d_h=w.d_h)
    assert np.all(np.isfinite(W2)) and np.all(np.isfinite(M2))
    assert O.rel_fro(W2, W1) < 1e-12
    assert O.rel_fro(M2, M1) < 1e-12
    assert O.rel_fro(o2, o1) < 1e-12


# ------------------------------------------------------------------ P2: plain chunk update
@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
def test_no_momentum_unit_decay_is_plain_chunk_update(kind):
    w, x = small_case(kind, T=6, C=6, H=1, seed=5)
    x["mom"][:] = 0.0
    x["decay"][:] = 1.0
    eta = x["lr"][0, 0].astype(np.float64)
    a, b, PU, PL, c = O.chunk_kernels(eta, x["mom"][0, 0], x["decay"][0, 0])
    np.testing.assert_array_equal(b, eta)
    np.testing.assert_array_equal(a[:-1], 0.0)
    assert a[-1] == eta[-1] and PU == 0.0 and PL == 1.0 and c == 0.0
    # W_end = W0 - sum_t eta_t g_t(W0) and M_end = -eta_C g_C(W0)
    _, W_end, M_end = O.seq_fwd(*fwd_args(w, x), d_h=w.d_h)
    P = O.unpack(kind, x["W0"][0, 0].astype(np.float64), w.d_k, w.d_v, w.d_h)
    gs = [O.pack(kind, O.loss_grad(kind, O.LOSS_MSE, P, x["k"][0, 0, t].astype(np.float64),
                                   x["v"][0, 0, t].astype(np.float64))) for t in range(6)]
    W_ref = x["W0"][0, 0] + x["M0"][0, 0] * 0.0 - sum(eta[t] * gs[t] for t in range(6))
    np.testing.assert_allclose(W_end[0, 0], W_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(M_end[0, 0], -eta[5] * gs[5], rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ P3: geometric closed forms
@pytest.mark.parametrize("mu,lam", [(0.9, 0.97), (0.5, 0.8), (0.95, 0.95), (0.0, 0.9), (0.7, 1.0)])
def test_constant_gates_geometric(mu, lam):
    C = 9
    eta = 0.3
    a, b, PU, PL, c = O.chunk_kernels(np.full(C, eta), np.full(C, mu), np.full(C, lam))
    t = np.arange(1, C + 1)
    np.testing.assert_allclose(a, eta * mu ** (C - t), rtol=1e-14, atol=1e-300)
    if mu != lam:
        R = (lam ** (C - t + 1) - mu ** (C - t + 1)) / (lam - mu)
    else:
        R = (C - t + 1) * lam ** (C - t)
    np.testing.assert_allclose(b, eta * R, rtol=1e-13)
    assert abs(PU - mu ** C) <= 1e-15 and abs(PL - lam ** C) <= 1e-15
    # c = mu * R_1  (the weight kernel's sum started one step earlier)
    np.testing.assert_allclose(c, mu * R[0], rtol=1e-13, atol=1e-300)


# ------------------------------------------------------------------ P4: chunk size 1
@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
def test_chunk_size_one_is_tokenwise(kind):
    w, x = small_case(kind, T=9, C=1, seed=11)
    o1, W1, M1 = O.seq_fwd(*fwd_args(w, x), d_h=w.d_h)
    o2, W2, M2 = O.tokenwise_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                                 x["W0"], x["M0"], d_h=w.d_h)
    assert O.rel_fro(o1, o2) < 1e-14 and O.rel_fro(W1, W2) < 1e-14 and O.rel_fro(M1, M2) < 1e-14
    # and with C > 1 the chunk-start approximation really differs from token-wise TTT
    o3, W3, _ = O.seq_fwd(*fwd_args(w.replace(C=3), x), d_h=w.d_h)
    assert O.rel_fro(W3, W2) > 1e-6


# ------------------------------------------------------------------ P5: hand-derived example
def test_golden_c2_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "c2_worked_example.json")))
    a, b, PU, PL, c = O.chunk_kernels(g["gates"]["eta"], g["gates"]["mu"], g["gates"]["lam"])
    K = g["kernels"]
    assert list(a) == K["a"] and list(b) == K["b"]
    assert PU == K["P_U"] and PL == K["P_L"] and c == K["c"]
    s = g["scalar_linear_case"]
    sh = (1, 1, 2, 1)
    args = (O.LINEAR, np.reshape(s["q"], sh), np.reshape(s["k"], sh), np.reshape(s["v"], sh),
            np.reshape(g["gates"]["eta"], (1, 1, 2)), np.reshape(g["gates"]["mu"], (1, 1, 2)),
            np.reshape(g["gates"]["lam"], (1, 1, 2)), np.full((1, 1, 1), s["W0"]),
            np.full((1, 1, 1), s["M0"]), 2)
    for fn in (O.seq_fwd, O.closed_fwd):
        out, W_end, M_end = fn(*args)
        assert list(out.reshape(-1)) == s["out"]
        assert W_end.item() == s["W_end"] and M_end.item() == s["M_end"]


# ------------------------------------------------------------------ P7: derivatives by FD
def _fd(f, x, d, eps=1e-6):
    return (f(x + eps * d) - f(x - eps * d)) / (2 * eps)


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_loss_grad_matches_fd(kind, loss):
    rng = np.random.default_rng(1)
    d_k, d_v, d_h = 5, 4, 6
    S = O.state_elems(kind, d_k, d_v, d_h)
    s = rng.standard_normal(S)
    k = rng.standard_normal(d_k)
    v = rng.standard_normal(d_v)
    g = O.pack(kind, O.loss_grad(kind, loss, O.unpack(kind, s, d_k, d_v, d_h), k, v))
    for _ in range(3):
        d = rng.standard_normal(S)
        fd = _fd(lambda z: O.loss_value(kind, loss, O.unpack(kind, z, d_k, d_v, d_h), k, v), s, d)
        assert abs(fd - g @ d) <= 1e-8 * max(1.0, abs(fd))


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_loss_grad_vjp_matches_fd(kind, loss):
    rng = np.random.default_rng(2)
    d_k, d_v, d_h = 5, 4, 6
    S = O.state_elems(kind, d_k, d_v, d_h)
    s = rng.standard_normal(S)
    k = rng.standard_normal(d_k)
    v = rng.standard_normal(d_v)
    gb = rng.standard_normal(S)

    def phi(s_, k_, v_):
        return O.pack(kind, O.loss_grad(kind, loss, O.unpack(kind, s_, d_k, d_v, d_h), k_, v_)) @ gb

    Pb, kb, vb = O.loss_grad_vjp(kind, loss, O.unpack(kind, s, d_k, d_v, d_h), k, v,
                                 O.unpack(kind, gb, d_k, d_v, d_h))
    Pb = O.pack(kind, Pb)
    ds, dk, dv = rng.standard_normal(S), rng.standard_normal(d_k), rng.standard_normal(d_v)
    assert abs(_fd(lambda z: phi(z, k, v), s, ds) - Pb @ ds) < 1e-7
    assert abs(_fd(lambda z: phi(s, z, v), k, dk) - kb @ dk) < 1e-7
    assert abs(_fd(lambda z: phi(s, k, z), v, dv) - vb @ dv) < 1e-7


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
def test_fast_apply_and_vjp(kind):
    rng = np.random.default_rng(3)
    d_k, d_v, d_h = 5, 4, 6
    S = O.state_elems(kind, d_k, d_v, d_h)
    s = rng.standard_normal(S)
    x = rng.standard_normal(d_k)
    yb = rng.standard_normal(d_v)
    P = O.unpack(kind, s, d_k, d_v, d_h)
    if kind == O.LINEAR:  # the linear fast weight is a plain matrix-vector product
        np.testing.assert_allclose(O.fast_apply(kind, P, x), np.dot(P["W"], x), rtol=1e-15)
    elif kind == O.SWIGLU:
        h1 = P["W1"] @ x
        np.testing.assert_allclose(O.silu(h1), h1 / (1 + np.exp(-h1)), rtol=1e-14)
    Pb, xb = O.fast_apply_vjp(kind, P, x, yb)
    ds, dx = rng.standard_normal(S), rng.standard_normal(d_k)
    f = lambda s_, x_: O.fast_apply(kind, O.unpack(kind, s_, d_k, d_v, d_h), x_) @ yb
    assert abs(_fd(lambda z: f(z, x), s, ds) - O.pack(kind, Pb) @ ds) < 1e-8
    assert abs(_fd(lambda z: f(s, z), x, dx) - xb @ dx) < 1e-8


def test_gelu_is_the_library_gelu_and_its_derivatives_fd():
    """The GELU MLP's activation is the exact GELU (torch's default, the erf form),
    and its first and second derivatives match finite differences."""
    import torch
    z = np.linspace(-7, 7, 57)
    ref = torch.nn.functional.gelu(torch.from_numpy(z)).numpy()
    np.testing.assert_allclose(O.gelu(z), ref, rtol=1e-13, atol=1e-15)
    assert abs(O.gelu(np.array(1.0)) - 0.8413447460685429) < 1e-15   # Phi(1)
    # atol: central-difference roundoff (eps = 1e-6) where gelu' crosses zero
    np.testing.assert_allclose(O.dgelu(z), _fd(O.gelu, z, np.ones_like(z)), rtol=1e-8, atol=1e-9)
    np.testing.assert_allclose(O.d2gelu(z), _fd(O.dgelu, z, np.ones_like(z)), rtol=1e-7, atol=1e-9)


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_seq_bwd_fd_tiny_gelu(loss):
    """Finite differences of the per-token recurrence with the GELU MLP fast weight
    (second-order terms through gelu'' included), ragged last chunk."""
    w, x = small_case(O.GELU, B=1, H=1, T=7, C=3, d_k=4, d_v=4, d_h=8, seed=61)
    _check_bwd_fd(w, x, loss=loss, seed=3)


def test_silu_derivatives_fd():
    z = np.linspace(-6, 6, 25)
    np.testing.assert_allclose(O.dsilu(z), _fd(O.silu, z, np.ones_like(z)), rtol=1e-8, atol=1e-10)
    np.testing.assert_allclose(O.d2silu(z), _fd(O.dsilu, z, np.ones_like(z)), rtol=1e-7, atol=1e-9)


# ------------------------------------------------------------------ P6: backward by FD
def _objective(w, x, dW, dM, loss=O.LOSS_MSE):
    out, W_end, M_end = O.seq_fwd(*fwd_args(w, x), d_h=w.d_h, loss=loss)
    return float(np.sum(out * x["dout"]) + np.sum(W_end * dW) + np.sum(M_end * dM))


NAMES = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("lr", "dlr"), ("mom", "dmom"),
         ("decay", "ddecay"), ("W0", "dW0"), ("M0", "dM0")]


def _check_bwd_fd(w, x, loss=O.LOSS_MSE, seed=0, tol=2e-7):
    x = {n: np.asarray(a, np.float64) for n, a in x.items()}
    rng = np.random.default_rng(seed)
    S = w.state_elems
    dW = rng.standard_normal((w.B, w.H, S))
    dM = rng.standard_normal((w.B, w.H, S))
    g = O.seq_bwd(*fwd_args(w, x), x["dout"], dW, dM, d_h=w.d_h, loss=loss)
    for name, gname in NAMES:
        d = rng.standard_normal(x[name].shape)
        eps = 1e-6

        def L(delta):
            y = dict(x)
            y[name] = x[name] + delta
            return _objective(w, y, dW, dM, loss)

        fd = (L(eps * d) - L(-eps * d)) / (2 * eps)
        an = float(np.sum(g[gname] * d))
        assert abs(fd - an) <= tol * max(1.0, abs(fd)), (name, fd, an)
    return g, dW, dM


def test_seq_bwd_fd_config0():
    """The tiny linear fp32 workload at its full size, all eight input groups."""
    w = gen.WORKLOADS[0]
    x = gen.generate(w, m0_scale=0.5)
    _check_bwd_fd(w, x, seed=0, tol=1e-6)


@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
@pytest.mark.parametrize("T,C", [(8, 4), (7, 3)])
def test_seq_bwd_fd_tiny_swiglu(loss, T, C):
    w, x = small_case(O.SWIGLU, B=1, H=1, T=T, C=C, d_k=4, d_v=4, d_h=8, seed=T + C)
    _check_bwd_fd(w, x, loss=loss, seed=T)


def test_seq_bwd_fd_linear_ragged():
    w, x = small_case(O.LINEAR, B=1, H=2, T=7, C=3, seed=9)
    _check_bwd_fd(w, x, seed=9)


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
@pytest.mark.parametrize("loss", [O.LOSS_MSE, O.LOSS_NEG_DOT])
def test_closed_bwd_equals_seq_bwd(kind, loss):
    w, x = small_case(kind, B=1, H=2, T=11, C=4, seed=21)
    rng = np.random.default_rng(5)
    dW = rng.standard_normal((w.B, w.H, w.state_elems))
    dM = rng.standard_normal((w.B, w.H, w.state_elems))
    g1 = O.seq_bwd(*fwd_args(w, x), x["dout"], dW, dM, d_h=w.d_h, loss=loss)
    g2 = O.closed_bwd(*fwd_args(w, x), x["dout"], dW, dM, d_h=w.d_h, loss=loss)
    for _, gname in NAMES:
        assert O.rel_fro(g2[gname], g1[gname]) < 1e-11, gname


def test_linear_adjoint_formulas():
    """Linear MSE, one chunk: the written-out closed-form adjoint
    dW0 = P_L D_W + sum dout q^T - sum (G k) k^T, dM0 = P_U D_M + c D_W,
    dq = W0^T dout, dv = G k, dk = -G^T e - W0^T G k,
    abar = -e^T D_M k, bbar = -e^T D_W k, with G_t = a_t D_M + b_t D_W."""
    w, x = small_case(O.LINEAR, B=1, H=1, T=6, C=6, d_k=4, d_v=3, seed=4)
    rng = np.random.default_rng(6)
    DW = rng.standard_normal((1, 1, 12))
    DM = rng.standard_normal((1, 1, 12))
    g = O.seq_bwd(*fwd_args(w, x), x["dout"], DW, DM)
    X = {n: np.asarray(a, np.float64)[0, 0] for n, a in x.items()}
    W0 = X["W0"].reshape(3, 4)
    M0 = X["M0"].reshape(3, 4)
    Dw, Dm = DW[0, 0].reshape(3, 4), DM[0, 0].reshape(3, 4)
    a, b, PU, PL, c = O.chunk_kernels(X["lr"], X["mom"], X["decay"])
    dW0 = PL * Dw
    dk = np.zeros((6, 4))
    dv = np.zeros((6, 3))
    abar = np.zeros(6)
    bbar = np.zeros(6)
    for t in range(6):
        k, v, q, do = X["k"][t], X["v"][t], X["q"][t], X["dout"][t]
        e = W0 @ k - v
        G = a[t] * Dm + b[t] * Dw
        dW0 = dW0 + np.outer(do, q) - np.outer(G @ k, k)
        dv[t] = G @ k
        dk[t] = -G.T @ e - W0.T @ (G @ k)
        abar[t] = -e @ Dm @ k
        bbar[t] = -e @ Dw @ k
    np.testing.assert_allclose(g["dW0"][0, 0], dW0.reshape(-1), rtol=1e-11)
    np.testing.assert_allclose(g["dM0"][0, 0], (PU * Dm + c * Dw).reshape(-1), rtol=1e-11)
    np.testing.assert_allclose(g["dq"][0, 0], X["dout"] @ W0, rtol=1e-11)
    np.testing.assert_allclose(g["dv"][0, 0], dv, rtol=1e-11)
    np.testing.assert_allclose(g["dk"][0, 0], dk, rtol=1e-10)
    deta, dmu, dlam = O.chunk_kernels_vjp(X["lr"], X["mom"], X["decay"], abar, bbar,
                                          np.sum(Dm * M0), np.sum(Dw * W0), np.sum(Dw * M0))
    np.testing.assert_allclose(g["dlr"][0, 0], deta, rtol=1e-10)
    np.testing.assert_allclose(g["dmom"][0, 0], dmu, rtol=1e-10)
    np.testing.assert_allclose(g["ddecay"][0, 0], dlam, rtol=1e-10)


def test_chunk_kernels_vjp_fd():
    rng = np.random.default_rng(8)
    C = 7
    eta = rng.uniform(0.1, 0.5, C)
    mu = rng.uniform(0.5, 0.99, C)
    lam = rng.uniform(0.8, 1.0, C)
    ab, bb = rng.standard_normal(C), rng.standard_normal(C)
    PUb, PLb, cb = rng.standard_normal(3)

    def L(e, m, l):
        a, b, PU, PL, c = O.chunk_kernels(e, m, l)
        return a @ ab + b @ bb + PU * PUb + PL * PLb + c * cb

    deta, dmu, dlam = O.chunk_kernels_vjp(eta, mu, lam, ab, bb, PUb, PLb, cb)
    for i in range(C):
        e = np.zeros(C)
        e[i] = 1.0
        assert abs(_fd(lambda z: L(z, mu, lam), eta, e) - deta[i]) < 1e-8
        assert abs(_fd(lambda z: L(eta, z, lam), mu, e) - dmu[i]) < 1e-8
        assert abs(_fd(lambda z: L(eta, mu, z), lam, e) - dlam[i]) < 1e-8


# ------------------------------------------------------------------ planted mistakes
@pytest.mark.parametrize("mutation", ["drop_decay_term", "wrong_sign_momentum", "shift_index",
                                      "swap_silu_deriv", "scale_w2_grad"])
def test_pins_catch_planted_mistakes(mutation, monkeypatch):
    """Each plausible slip, planted in the oracle on the CPU, trips a pin."""
    import oracle.e2ttt_oracle as M
    if mutation == "drop_decay_term":
        real = M.chunk_kernels

        def bad(eta, mu, lam):
            a, b, PU, PL, c = real(eta, mu, lam)
            return a, np.asarray(eta, np.float64) * 1.0, PU, PL, c     # b_t = eta_t: no ratio sum
        monkeypatch.setattr(M, "chunk_kernels", bad)
        with pytest.raises(AssertionError):
            test_closed_equals_sequential(O.LINEAR, O.LOSS_MSE, 12, 4)
    elif mutation == "wrong_sign_momentum":
        real = M.chunk_kernels

        def bad(eta, mu, lam):
            a, b, PU, PL, c = real(eta, mu, lam)
            return -a, b, PU, PL, c
        monkeypatch.setattr(M, "chunk_kernels", bad)
        with pytest.raises(AssertionError):
            test_golden_c2_worked_example()
    elif mutation == "shift_index":
        real = M.chunk_kernels

        def bad(eta, mu, lam):
            a, b, PU, PL, c = real(np.roll(np.asarray(eta), 1), mu, lam)
            return a, b, PU, PL, c
        monkeypatch.setattr(M, "chunk_kernels", bad)
        with pytest.raises(AssertionError):
            test_closed_equals_sequential(O.SWIGLU, O.LOSS_MSE, 12, 4)
    elif mutation == "swap_silu_deriv":
        monkeypatch.setattr(M, "d2silu", lambda z: np.zeros_like(z))
        with pytest.raises(AssertionError):
            test_loss_grad_vjp_matches_fd(O.SWIGLU, O.LOSS_MSE)
    elif mutation == "scale_w2_grad":
        real = M.loss_grad

        def bad(kind, loss, P, k, v):
            g = real(kind, loss, P, k, v)
            if "W2" in g:
                g["W2"] = g["W2"] * 1.0001
            return g
        monkeypatch.setattr(M, "loss_grad", bad)
        monkeypatch.setattr(O, "loss_grad", bad)
        with pytest.raises(AssertionError):
            test_loss_grad_matches_fd(O.SWIGLU, O.LOSS_MSE)


# ------------------------------------------------------------------ input generator
def test_generator_is_seeded_and_shaped():
    w = gen.WORKLOADS[1].replace(B=1, H=2, T=64, C=32)
    x1 = gen.generate(w)
    x2 = gen.generate(w)
    for n in x1:
        np.testing.assert_array_equal(x1[n], x2[n])
    assert x1["q"].shape == (1, 2, 64, 128) and x1["W0"].shape == (1, 2, w.state_elems)
    np.testing.assert_allclose(np.linalg.norm(gen.generate(w, dtype_round=False)["k"], axis=-1), 1.0,
                               rtol=1e-6)
    # bf16 rounding leaves exactly representable values (low 16 bits zero)
    assert np.all((x1["q"].view(np.uint32) & 0xFFFF) == 0)
    assert np.all(x1["M0"] == 0)


def test_bf16_rounding_ties_to_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], np.float32)
    r = gen.round_to_bf16(x)
    np.testing.assert_array_equal(r, np.array([1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5], np.float32))


def test_bf16_rounding_matches_torch_conversion():
    """The input module's bf16 rounding against torch's own float -> bf16
    conversion (round to nearest, ties to even) on a million values spread over
    the exponent range, both signs, exact ties, subnormals, the largest finite
    values (which round to infinity) and non-finite inputs."""
    import torch
    rng = np.random.default_rng(7)
    mant = rng.integers(0, 1 << 23, size=1 << 20, dtype=np.uint32)
    expo = rng.integers(1, 255, size=1 << 20, dtype=np.uint32)
    sign = rng.integers(0, 2, size=1 << 20, dtype=np.uint32)
    x = ((sign << 31) | (expo << 23) | mant).view(np.float32)
    ties = (((sign[:4096] << 31) | (expo[:4096] << 23) | (mant[:4096] & ~np.uint32(0xFFFF))
             | np.uint32(0x8000))).view(np.float32)
    special = np.array([0.0, -0.0, 1e-45, -3e-39, 3.3e38, -3.4028235e38, np.inf, -np.inf], np.float32)
    x = np.concatenate([x, ties, special])
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(gen.round_to_bf16(x), ref)
    nan = gen.round_to_bf16(np.array([np.nan], np.float32))
    assert np.isnan(nan[0])


# ------------------------------------------------------------------ chunk-averaged variant
# atlas.scime.ai summary, "Surprising findings": the per-token factors collapsed to
# chunk scalars (read as the chunk means of a_t and b_t; P_U, P_L, c unchanged).
@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
def test_chunk_mean_chunk_size_one_is_tokenwise(kind):
    """With one token per chunk the mean is the token's own factor: the variant is
    token-wise TTT (the independent third loop)."""
    w, x = small_case(kind, T=9, C=1, seed=21)
    o1, W1, M1 = O.closed_fwd(*fwd_args(w, x), d_h=w.d_h, coef=O.COEF_CHUNK_MEAN)
    o2, W2, M2 = O.tokenwise_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                                 x["W0"], x["M0"], d_h=w.d_h)
    assert O.rel_fro(o1, o2) < 1e-13 and O.rel_fro(W1, W2) < 1e-13 and O.rel_fro(M1, M2) < 1e-13


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
def test_chunk_mean_no_momentum_unit_decay(kind):
    """mu = 0, lam = 1: a_t = eta_t [t = C] and b_t = eta_t, so the variant is the
    plain chunk update with the chunk's mean learning rate,
        W <- W - mean(eta) sum_t g_t(W),   M <- -(eta_C / C) sum_t g_t(W),
    written here as its own loop over chunks."""
    w, x = small_case(kind, T=12, C=4, H=1, seed=23)
    x["mom"][:] = 0.0
    x["decay"][:] = 1.0
    _, W_end, M_end = O.closed_fwd(*fwd_args(w, x), d_h=w.d_h, coef=O.COEF_CHUNK_MEAN)
    W = x["W0"][0, 0].astype(np.float64)
    M = x["M0"][0, 0].astype(np.float64)
    for t0 in range(0, 12, 4):
        P = O.unpack(kind, W, w.d_k, w.d_v, w.d_h)
        gsum = sum(O.pack(kind, O.loss_grad(kind, O.LOSS_MSE, P, x["k"][0, 0, t].astype(np.float64),
                                            x["v"][0, 0, t].astype(np.float64)))
                   for t in range(t0, t0 + 4))
        eta = x["lr"][0, 0, t0:t0 + 4].astype(np.float64)
        W = W - eta.mean() * gsum
        M = -(eta[-1] / 4) * gsum
    np.testing.assert_allclose(W_end[0, 0], W, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(M_end[0, 0], M, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("mu,lam", [(0.9, 0.97), (0.5, 0.8), (0.95, 0.95), (0.0, 0.9)])
def test_chunk_mean_constant_gates_geometric(mu, lam):
    """Constant gates: mean_t eta mu^(C-t) = eta (1 - mu^C) / (C (1 - mu)) and
    mean_t eta R_t = eta / C * sum_{j=1..C} (lam^j - mu^j) / (lam - mu) (or
    eta / C * sum_j j lam^(j-1) when mu = lam)."""
    C, eta = 9, 0.3
    a, b, PU, PL, c = O.chunk_mean_kernels(np.full(C, eta), np.full(C, mu), np.full(C, lam))
    abar = eta * (1 - mu ** C) / (C * (1 - mu))
    j = np.arange(1, C + 1)
    if mu != lam:
        bbar = eta / C * np.sum((lam ** j - mu ** j) / (lam - mu))
    else:
        bbar = eta / C * np.sum(j * lam ** (j - 1))
    np.testing.assert_allclose(a, abar, rtol=1e-13)
    np.testing.assert_allclose(b, bbar, rtol=1e-13)
    assert abs(PU - mu ** C) <= 1e-15 and abs(PL - lam ** C) <= 1e-15


@pytest.mark.parametrize("kind", [O.LINEAR, O.SWIGLU, O.GELU])
def test_chunk_mean_bwd_matches_fd(kind):
    """closed_bwd of the variant against central finite differences of closed_fwd
    of the variant, every input group, ragged last chunk."""
    w, x = small_case(kind, B=1, H=1, T=7, C=3, d_k=4, d_v=4, d_h=6, seed=27)
    x = {n: np.asarray(a, np.float64) for n, a in x.items()}
    rng = np.random.default_rng(4)
    S = w.state_elems
    dW = rng.standard_normal((1, 1, S))
    dM = rng.standard_normal((1, 1, S))
    args = lambda y: (w.kind, y["q"], y["k"], y["v"], y["lr"], y["mom"], y["decay"], y["W0"],
                      y["M0"], w.C)
    g = O.closed_bwd(*args(x), x["dout"], dW, dM, d_h=w.d_h, coef=O.COEF_CHUNK_MEAN)

    def L(y):
        out, W_end, M_end = O.closed_fwd(*args(y), d_h=w.d_h, coef=O.COEF_CHUNK_MEAN)
        return float(np.sum(out * x["dout"]) + np.sum(W_end * dW) + np.sum(M_end * dM))

    for name, gname in NAMES:
        d = rng.standard_normal(x[name].shape)
        eps = 1e-6
        yp, ym = dict(x), dict(x)
        yp[name] = x[name] + eps * d
        ym[name] = x[name] - eps * d
        fd = (L(yp) - L(ym)) / (2 * eps)
        an = float(np.sum(g[gname] * d))
        assert abs(fd - an) <= 2e-7 * max(1.0, abs(fd)), (name, fd, an)
    # and the variant really differs from the per-token kernels
    g0 = O.closed_bwd(*args(x), x["dout"], dW, dM, d_h=w.d_h)
    assert O.rel_fro(g["dlr"], g0["dlr"]) > 1e-3


def test_closed_bwd_given_starts_equals_recomputed():
    """closed_bwd with starts= the states closed_fwd computes equals closed_bwd that
    recomputes them (the option only replaces the chunk-start states)."""
    w, x = small_case(O.GELU, B=1, H=1, T=7, C=3, d_k=4, d_v=4, d_h=6, seed=71)
    args = (w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"], x["M0"], w.C)
    _, _, _, st = O.closed_fwd(*args, d_h=w.d_h, return_starts=True)
    g1 = O.closed_bwd(*args, x["dout"], d_h=w.d_h)
    g2 = O.closed_bwd(*args, x["dout"], d_h=w.d_h, starts=st)
    for n in g1:
        np.testing.assert_array_equal(g1[n], g2[n])


def _grads_moved_by_bf16_weights(kind, m0_scale):
    """How far the oracle's exact gradients move when only the fast-weight part
    of every chunk-start state is rounded to bf16 (what the tensor-core GEMMs
    consume), for the d = 128 bf16 workload used by the GPU backward tests:
    relative Frobenius change per gradient."""
    w = gen.Workload("cond", kind, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=49, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=m0_scale)
    dW, dM = gen.upstream_state_grads(w, seed=8, scale=0.1)
    args = (w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"], x["M0"], w.C)
    _, _, _, starts = O.closed_fwd(*args, d_h=w.d_h, return_starts=True)
    ref = O.closed_bwd(*args, x["dout"], dW, dM, d_h=w.d_h, starts=starts)
    rounded = starts.copy()
    rounded[:, :, :, 0] = gen.round_to_bf16(starts[:, :, :, 0].astype(np.float32))
    got = O.closed_bwd(*args, x["dout"], dW, dM, d_h=w.d_h, starts=rounded)
    return {n: O.rel_fro(got[n], ref[n]) for n in ref}


@pytest.mark.slow
def test_gelu_backward_conditioning_under_bf16_weights():
    """Conditioning of the exact backward, oracle only. The GELU MLP with a
    non-zero momentum state M0 and upstream state gradients is ill-conditioned in
    its weights: rounding the chunk-start weights to bf16 (a relative change of
    at most 2^-9 per element) moves the exact gradients w.r.t. k, v, the gates and
    the initial states by 3-15 %, more than the 2e-2 bar of the bf16 paths. No
    implementation whose GEMMs take bf16 weight operands can meet 2e-2 against
    the fp64 gradients there, so its GPU test compares with the oracle at the
    bf16-rounded chunk-start states it computes from. With M0 = 0 the same
    rounding moves them by under 5e-3, and the SwiGLU fast weight stays under
    1e-2 either way: those cases are compared with the fp64 oracle directly."""
    ill = _grads_moved_by_bf16_weights(O.GELU, 0.5)
    for n in ("dk", "dv", "dlr", "dmom", "ddecay", "dW0", "dM0"):
        assert 3e-2 < ill[n] < 0.15, (n, ill[n])
    assert ill["dq"] < 2e-3   # the output path does not go through the ill-conditioned terms
    well = _grads_moved_by_bf16_weights(O.GELU, 0.0)
    assert max(well.values()) < 5e-3, well
    sw = _grads_moved_by_bf16_weights(O.SWIGLU, 0.5)
    assert max(sw.values()) < 1e-2, sw
