"""Plain fp64 CPU oracle of E2-TTT's chunk-parallel closed-form fast-weight update.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
baseline may import this module. The product path (the CUDA library and its
binding) never imports or calls it, and it shares no code with that path.

Source: "Rethinking Expressivity and Efficiency in Test-Time Training"
(E2-TTT, arXiv 2608.21308), read from five web summaries that carry no
equations. What they fix:
  * abstract: under gradients taken at the chunk-start weights, a closed-form
    state transition reproduces exactly the chunk-end fast-weight and momentum
    states of the per-token recurrence;
  * atlas.scime.ai summary, "Approach": two scalar kernels (momentum kernel and
    weight kernel) come from unrolling the token-wise momentum-plus-decay
    recurrence, and the chunk-end states are two weighted gradient
    aggregations built from chunk-start gradients;
  * arxivlens summary, "Limitations" and atlas "Surprising findings": the chunk
    output is taken at the chunk-start weights (fixed within a chunk).
Readings the pages leave open (all written out here):
  * recurrence  M_t = mu_t M_{t-1} - eta_t g_t ,  W_t = lam_t W_{t-1} + M_t ;
  * loss  l(W; k, v) = 1/2 |f_W(k) - v|^2  (or -<f_W(k), v> for the dot loss);
  * fast weight  f(x) = W x  (linear),  W2 (silu(W1 x) * (W3 x))  (SwiGLU), or
    W2 gelu(W1 x)  (the MLP variant: atlas "Key results" names E2-TTT_MLP and
    the codewithpapers JSON a gelu_derivative function; read as the exact GELU
    z Phi(z) of the standard normal CDF, no biases);
  * out_t = f_{W_chunk_start}(q_t); gates are values (not logits); chunk i holds
    tokens [iC, (i+1)C), the last chunk may be short.

Functions, and what each follows:
  seq_fwd        the per-token recurrence with gradients frozen at the chunk
                 start, token by token (the abstract's "per-token recurrence");
  tokenwise_fwd  fully sequential TTT, gradient at W_{t-1} (the exact method the
                 chunk-start approximation departs from; atlas "Limitations");
  chunk_kernels  the momentum kernel a_t, weight kernel b_t and chunk scalars
                 by direct products (atlas "Approach": unrolled recurrence);
  closed_fwd     chunk-end states as decayed M0/W0 plus two weighted gradient
                 aggregations (abstract; atlas "Approach");
  seq_bwd        the reverse of seq_fwd's loop, token by token, with the second
                 order terms through g_t(W_chunk_start, k_t, v_t);
  closed_bwd     the adjoint of closed_fwd (a second route; pinned to seq_bwd);
  chunk_mean_kernels  the chunk-averaged variant (atlas "Surprising findings":
                 per-token factors collapsed to chunk scalars), read as the
                 chunk means of a_t and b_t; closed_fwd / closed_bwd take it
                 with coef=COEF_CHUNK_MEAN.
State layout per (b, h): linear W [d_v, d_k]; SwiGLU [W1 (d_h x d_k) | W3
(d_h x d_k) | W2 (d_v x d_h)]; GELU MLP [W1 (d_h x d_k) | W2 (d_v x d_h)]; each
row-major, concatenated.
"""
from __future__ import annotations

import math
import numpy as np
from scipy.special import erf

LINEAR = 0
SWIGLU = 1
GELU = 2               # the two-matrix GELU MLP fast weight (E2-TTT_MLP)
LOSS_MSE = 0
LOSS_NEG_DOT = 1
COEF_PER_TOKEN = 0     # per-token momentum / weight kernels (the method)
COEF_CHUNK_MEAN = 1    # the chunk-averaged variant


# --------------------------------------------------------------------------- layout
def state_elems(kind, d_k, d_v, d_h):
    if kind == LINEAR:
        return d_v * d_k
    if kind == GELU:
        return d_h * d_k + d_v * d_h
    return 2 * d_h * d_k + d_v * d_h


def unpack(kind, s, d_k, d_v, d_h):
    """Views of the matrices inside a flat state vector."""
    if kind == LINEAR:
        return {"W": s.reshape(d_v, d_k)}
    n1 = d_h * d_k
    if kind == GELU:
        return {"W1": s[:n1].reshape(d_h, d_k), "W2": s[n1:].reshape(d_v, d_h)}
    return {"W1": s[:n1].reshape(d_h, d_k),
            "W3": s[n1:2 * n1].reshape(d_h, d_k),
            "W2": s[2 * n1:].reshape(d_v, d_h)}


def pack(kind, P):
    if kind == LINEAR:
        return P["W"].reshape(-1).copy()
    if kind == GELU:
        return np.concatenate([P["W1"].reshape(-1), P["W2"].reshape(-1)])
    return np.concatenate([P["W1"].reshape(-1), P["W3"].reshape(-1), P["W2"].reshape(-1)])


# --------------------------------------------------------------------------- activations
def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * sigmoid(z)


def dsilu(z):
    """d/dz [z sigma(z)] = sigma(z) (1 + z (1 - sigma(z)))."""
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def d2silu(z):
    """d^2/dz^2 [z sigma(z)] = sigma(z) (1 - sigma(z)) (2 + z (1 - 2 sigma(z)))."""
    s = sigmoid(z)
    return s * (1.0 - s) * (2.0 + z * (1.0 - 2.0 * s))


def Phi(z):
    """Standard normal CDF."""
    return 0.5 * (1.0 + erf(z / math.sqrt(2.0)))


def phi(z):
    """Standard normal density."""
    return np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def gelu(z):
    return z * Phi(z)


def dgelu(z):
    """d/dz [z Phi(z)] = Phi(z) + z phi(z)."""
    return Phi(z) + z * phi(z)


def d2gelu(z):
    """d^2/dz^2 [z Phi(z)] = 2 phi(z) + z phi'(z) = phi(z) (2 - z^2)."""
    return phi(z) * (2.0 - z * z)


# --------------------------------------------------------------------------- fast weight
def fast_apply(kind, P, x):
    """f_W(x) for one token x [d_k] -> [d_v]."""
    if kind == LINEAR:
        return P["W"] @ x
    if kind == GELU:
        return P["W2"] @ gelu(P["W1"] @ x)
    h1 = P["W1"] @ x
    h3 = P["W3"] @ x
    return P["W2"] @ (silu(h1) * h3)


def loss_value(kind, loss, P, k, v):
    y = fast_apply(kind, P, k)
    if loss == LOSS_MSE:
        return 0.5 * float(np.sum((y - v) ** 2))
    return -float(np.dot(y, v))


def loss_grad(kind, loss, P, k, v):
    """g = grad_W l(W; k, v) for one token, as a dict shaped like P."""
    if kind == LINEAR:
        y = P["W"] @ k
        e = (y - v) if loss == LOSS_MSE else -v
        return {"W": np.outer(e, k)}
    if kind == GELU:
        h = P["W1"] @ k
        u = gelu(h)
        y = P["W2"] @ u
        e = (y - v) if loss == LOSS_MSE else -v
        dh = (P["W2"].T @ e) * dgelu(h)
        return {"W1": np.outer(dh, k), "W2": np.outer(e, u)}
    h1 = P["W1"] @ k
    h3 = P["W3"] @ k
    s = silu(h1)
    u = s * h3
    y = P["W2"] @ u
    e = (y - v) if loss == LOSS_MSE else -v
    du = P["W2"].T @ e
    dh3 = du * s
    dh1 = du * h3 * dsilu(h1)
    return {"W1": np.outer(dh1, k), "W3": np.outer(dh3, k), "W2": np.outer(e, u)}


def loss_grad_vjp(kind, loss, P, k, v, gbar):
    """Reverse-mode pass through loss_grad: given the adjoint gbar of g(P, k, v),
    return (Pbar, kbar, vbar). Each step undoes one line of loss_grad."""
    if kind == LINEAR:
        W = P["W"]
        y = W @ k
        e = (y - v) if loss == LOSS_MSE else -v
        G = gbar["W"]
        ebar = G @ k                  # g = e k^T
        kbar = G.T @ e
        vbar = -ebar                  # e = y - v  (or -v)
        Wbar = np.zeros_like(W)
        if loss == LOSS_MSE:
            Wbar += np.outer(ebar, k)  # y = W k
            kbar = kbar + W.T @ ebar
        return {"W": Wbar}, kbar, vbar
    if kind == GELU:
        W1, W2 = P["W1"], P["W2"]
        h = W1 @ k
        u = gelu(h)
        gp = dgelu(h)
        y = W2 @ u
        e = (y - v) if loss == LOSS_MSE else -v
        du = W2.T @ e
        dh = du * gp
        G1, G2 = gbar["W1"], gbar["W2"]
        W2b = np.zeros_like(W2)
        # gW1 = dh k^T
        dhb = G1 @ k
        kbar = G1.T @ dh
        # dh = du * gelu'(h)
        dub = dhb * gp
        hb = dhb * du * d2gelu(h)
        # du = W2^T e
        W2b += np.outer(e, dub)
        eb = W2 @ dub
        # gW2 = e u^T
        eb = eb + G2 @ u
        ub = G2.T @ e
        # e = y - v   (dot loss: e = -v)
        vbar = -eb
        if loss == LOSS_MSE:
            W2b += np.outer(eb, u)       # y = W2 u
            ub = ub + W2.T @ eb
        # u = gelu(h) ; h = W1 k
        hb = hb + ub * gp
        kbar = kbar + W1.T @ hb
        return {"W1": np.outer(hb, k), "W2": W2b}, kbar, vbar
    W1, W3, W2 = P["W1"], P["W3"], P["W2"]
    h1 = W1 @ k
    h3 = W3 @ k
    s = silu(h1)
    ds = dsilu(h1)
    u = s * h3
    y = W2 @ u
    e = (y - v) if loss == LOSS_MSE else -v
    du = W2.T @ e
    dh3 = du * s
    dh1 = du * h3 * ds
    G1, G3, G2 = gbar["W1"], gbar["W3"], gbar["W2"]
    W1b = np.zeros_like(W1)
    W3b = np.zeros_like(W3)
    W2b = np.zeros_like(W2)
    # gW1 = dh1 k^T ; gW3 = dh3 k^T
    dh1b = G1 @ k
    dh3b = G3 @ k
    kbar = G1.T @ dh1 + G3.T @ dh3
    # dh1 = du * h3 * silu'(h1)
    dub = dh1b * h3 * ds
    h3b = dh1b * du * ds
    h1b = dh1b * du * h3 * d2silu(h1)
    # dh3 = du * s
    dub = dub + dh3b * s
    sb = dh3b * du
    # du = W2^T e
    W2b += np.outer(e, dub)
    eb = W2 @ dub
    # gW2 = e u^T
    eb = eb + G2 @ u
    ub = G2.T @ e
    # e = y - v   (dot loss: e = -v)
    vbar = -eb
    if loss == LOSS_MSE:
        W2b += np.outer(eb, u)       # y = W2 u
        ub = ub + W2.T @ eb
    # u = s * h3 ; s = silu(h1)
    sb = sb + ub * h3
    h3b = h3b + ub * s
    h1b = h1b + sb * ds
    # h1 = W1 k ; h3 = W3 k
    W1b += np.outer(h1b, k)
    W3b += np.outer(h3b, k)
    kbar = kbar + W1.T @ h1b + W3.T @ h3b
    return {"W1": W1b, "W3": W3b, "W2": W2b}, kbar, vbar


def fast_apply_vjp(kind, P, x, ybar):
    """Reverse-mode pass through fast_apply: (Pbar, xbar)."""
    if kind == LINEAR:
        return {"W": np.outer(ybar, x)}, P["W"].T @ ybar
    if kind == GELU:
        h = P["W1"] @ x
        hb = (P["W2"].T @ ybar) * dgelu(h)
        return {"W1": np.outer(hb, x), "W2": np.outer(ybar, gelu(h))}, P["W1"].T @ hb
    W1, W3, W2 = P["W1"], P["W3"], P["W2"]
    h1 = W1 @ x
    h3 = W3 @ x
    s = silu(h1)
    u = s * h3
    ub = W2.T @ ybar
    W2b = np.outer(ybar, u)
    h1b = ub * h3 * dsilu(h1)
    h3b = ub * s
    return ({"W1": np.outer(h1b, x), "W3": np.outer(h3b, x), "W2": W2b},
            W1.T @ h1b + W3.T @ h3b)


# --------------------------------------------------------------------------- helpers
def _chunks(T, C):
    return [(s, min(s + C, T)) for s in range(0, T, C)]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _dims(kind, q, v, W0, d_h):
    d_k = q.shape[-1]
    d_v = v.shape[-1]
    S = state_elems(kind, d_k, d_v, d_h)
    assert W0.shape[-1] == S, (W0.shape, S)
    return d_k, d_v, S


# --------------------------------------------------------------------------- forward: per token
def seq_fwd(kind, q, k, v, lr, mom, decay, W0, M0, C, d_h=0, loss=LOSS_MSE,
            return_starts=False):
    """The per-token momentum + decay recurrence with every gradient of a chunk
    taken at that chunk's start weights, run literally token by token.

    q, k [B,H,T,d_k]; v [B,H,T,d_v]; lr, mom, decay [B,H,T]; W0, M0 [B,H,S].
    Returns out [B,H,T,d_v], W_end, M_end [B,H,S] (and, if asked, the chunk-start
    states [n_chunks,B,H,2,S]).
    """
    q, k, v, lr, mom, decay, W0, M0 = map(_f64, (q, k, v, lr, mom, decay, W0, M0))
    B, H, T = lr.shape
    d_k, d_v, S = _dims(kind, q, v, W0, d_h)
    chunks = _chunks(T, C)
    out = np.zeros((B, H, T, d_v))
    W_end = np.zeros((B, H, S))
    M_end = np.zeros((B, H, S))
    starts = np.zeros((len(chunks), B, H, 2, S))
    for b in range(B):
        for h in range(H):
            W = W0[b, h].copy()
            M = M0[b, h].copy()
            for ci, (t0, t1) in enumerate(chunks):
                starts[ci, b, h, 0] = W
                starts[ci, b, h, 1] = M
                Wc = unpack(kind, W.copy(), d_k, d_v, d_h)   # frozen chunk-start weights
                for t in range(t0, t1):
                    out[b, h, t] = fast_apply(kind, Wc, q[b, h, t])
                for t in range(t0, t1):
                    g = pack(kind, loss_grad(kind, loss, Wc, k[b, h, t], v[b, h, t]))
                    M = mom[b, h, t] * M - lr[b, h, t] * g
                    W = decay[b, h, t] * W + M
            W_end[b, h] = W
            M_end[b, h] = M
    if return_starts:
        return out, W_end, M_end, starts
    return out, W_end, M_end


def tokenwise_fwd(kind, q, k, v, lr, mom, decay, W0, M0, d_h=0, loss=LOSS_MSE):
    """Fully sequential token-wise TTT: the gradient of token t is taken at the
    current weights W_{t-1}, and out_t = f_{W_{t-1}}(q_t)."""
    q, k, v, lr, mom, decay, W0, M0 = map(_f64, (q, k, v, lr, mom, decay, W0, M0))
    B, H, T = lr.shape
    d_k, d_v, S = _dims(kind, q, v, W0, d_h)
    out = np.zeros((B, H, T, d_v))
    W_end = np.zeros((B, H, S))
    M_end = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            W = W0[b, h].copy()
            M = M0[b, h].copy()
            for t in range(T):
                P = unpack(kind, W.copy(), d_k, d_v, d_h)
                out[b, h, t] = fast_apply(kind, P, q[b, h, t])
                g = pack(kind, loss_grad(kind, loss, P, k[b, h, t], v[b, h, t]))
                M = mom[b, h, t] * M - lr[b, h, t] * g
                W = decay[b, h, t] * W + M
            W_end[b, h] = W
            M_end[b, h] = M
    return out, W_end, M_end


# --------------------------------------------------------------------------- scalar kernels
def chunk_kernels(eta, mu, lam):
    """Momentum kernel a, weight kernel b and chunk scalars for ONE chunk, from
    the definitions obtained by unrolling the recurrence over the chunk's C
    tokens (1-based t; U(i,j) = prod_{s=i..j} mu_s, L(i,j) = prod_{s=i..j} lam_s,
    empty products = 1):
        M_C = U(1,C) M0 - sum_t a_t g_t,            a_t = eta_t U(t+1,C)
        W_C = L(1,C) W0 + c M0 - sum_t b_t g_t,     b_t = eta_t R_t
        R_t = sum_{j=t..C} L(j+1,C) U(t+1,j),       c = sum_{j=1..C} L(j+1,C) U(1,j)
    Computed with plain running products (no logarithms), O(C^2).
    Returns (a, b, P_U, P_L, c)."""
    eta, mu, lam = _f64(eta), _f64(mu), _f64(lam)
    n = eta.shape[0]
    # sufL[j] = L(j+1, C) for j = 0..C (0-based j means "after j tokens")
    sufL = np.ones(n + 1)
    for j in range(n - 1, -1, -1):
        sufL[j] = sufL[j + 1] * lam[j]
    a = np.zeros(n)
    b = np.zeros(n)
    for t in range(n):                       # 0-based token t  (1-based t+1)
        # U(t+2, C): product of mu over the tokens after t
        a[t] = eta[t] * np.prod(mu[t + 1:])
        # R: sum over j >= t of L(j+1,C) * U(t+1, j)  (1-based), i.e. running
        # products of mu over tokens t+1..j (0-based)
        # running products mu_{t+1} ... mu_j for j = t+1 .. C-1 (0-based)
        run = np.cumprod(mu[t + 1:])
        r = sufL[t + 1] + np.sum(sufL[t + 2:] * run)   # first term: j = t, empty product
        b[t] = eta[t] * r
    P_U = float(np.prod(mu))
    P_L = float(np.prod(lam))
    c = float(np.sum(sufL[1:] * np.cumprod(mu)))
    return a, b, P_U, P_L, c


def chunk_mean_kernels(eta, mu, lam):
    """The chunk-averaged variant (atlas.scime.ai summary, "Surprising findings":
    the per-token factors collapsed to chunk scalars): chunk_kernels' momentum
    and weight kernels replaced by their means over the chunk's tokens, so every
    token of the chunk carries a_bar = mean_t a_t and b_bar = mean_t b_t; the
    chunk scalars P_U, P_L, c are those of the recurrence. Reading: "collapsed to
    chunk scalars" = the arithmetic mean."""
    a, b, P_U, P_L, c = chunk_kernels(eta, mu, lam)
    return np.full_like(a, a.mean()), np.full_like(b, b.mean()), P_U, P_L, c


def _kernels(coef):
    return chunk_mean_kernels if coef == COEF_CHUNK_MEAN else chunk_kernels


def all_chunk_kernels(lr, mom, decay, C, coef=COEF_PER_TOKEN):
    """chunk_kernels (or chunk_mean_kernels) over [B,H,T] gates: a, b [B,H,T];
    P_U, P_L, c [B,H,n_chunks]."""
    lr, mom, decay = _f64(lr), _f64(mom), _f64(decay)
    B, H, T = lr.shape
    chunks = _chunks(T, C)
    a = np.zeros((B, H, T))
    b = np.zeros((B, H, T))
    sc = np.zeros((3, B, H, len(chunks)))
    for bb in range(B):
        for hh in range(H):
            for ci, (t0, t1) in enumerate(chunks):
                aa, bbv, pu, pl, cc = _kernels(coef)(lr[bb, hh, t0:t1], mom[bb, hh, t0:t1],
                                                     decay[bb, hh, t0:t1])
                a[bb, hh, t0:t1] = aa
                b[bb, hh, t0:t1] = bbv
                sc[:, bb, hh, ci] = (pu, pl, cc)
    return a, b, sc[0], sc[1], sc[2]


# --------------------------------------------------------------------------- forward: closed form
def chunk_grads(kind, loss, P, K, V):
    """All chunk-start gradients of one chunk as the factors of their outer
    products: g_t = sum over factor pairs (left_t right_t^T).
    Returns a dict name -> (Left [n, rows], Right [n, cols])."""
    if kind == LINEAR:
        Y = K @ P["W"].T
        E = (Y - V) if loss == LOSS_MSE else -V
        return {"W": (E, K)}
    if kind == GELU:
        Hg = K @ P["W1"].T
        U = gelu(Hg)
        E = (U @ P["W2"].T - V) if loss == LOSS_MSE else -V
        dH = (E @ P["W2"]) * dgelu(Hg)
        return {"W1": (dH, K), "W2": (E, U)}
    H1 = K @ P["W1"].T
    H3 = K @ P["W3"].T
    S = silu(H1)
    U = S * H3
    Y = U @ P["W2"].T
    E = (Y - V) if loss == LOSS_MSE else -V
    dU = E @ P["W2"]
    dH3 = dU * S
    dH1 = dU * H3 * dsilu(H1)
    return {"W1": (dH1, K), "W3": (dH3, K), "W2": (E, U)}


def weighted_sum(factors, w):
    """sum_t w_t left_t right_t^T  for every matrix (the weighted aggregations)."""
    return {name: L.T @ (w[:, None] * R) for name, (L, R) in factors.items()}


def closed_fwd(kind, q, k, v, lr, mom, decay, W0, M0, C, d_h=0, loss=LOSS_MSE,
               return_starts=False, heads=None, coef=COEF_PER_TOKEN):
    """Closed-form chunk transition: per chunk
        out_t = f_{W0}(q_t),
        M_end = P_U M0 - sum_t a_t g_t,
        W_end = P_L W0 + c M0 - sum_t b_t g_t,
    with g_t at the chunk-start weights W0 (a_t, b_t the chunk means for
    coef=COEF_CHUNK_MEAN). ``heads`` optionally restricts the computation to a
    list of (b, h) pairs (the others are left zero)."""
    q, k, v, lr, mom, decay, W0, M0 = map(_f64, (q, k, v, lr, mom, decay, W0, M0))
    B, H, T = lr.shape
    d_k, d_v, S = _dims(kind, q, v, W0, d_h)
    chunks = _chunks(T, C)
    out = np.zeros((B, H, T, d_v))
    W_end = np.zeros((B, H, S))
    M_end = np.zeros((B, H, S))
    starts = np.zeros((len(chunks), B, H, 2, S)) if return_starts else None
    hl = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in hl:
        W = W0[b, h].copy()
        M = M0[b, h].copy()
        for ci, (t0, t1) in enumerate(chunks):
            if return_starts:
                starts[ci, b, h, 0] = W
                starts[ci, b, h, 1] = M
            P = unpack(kind, W, d_k, d_v, d_h)
            Q = q[b, h, t0:t1]
            out[b, h, t0:t1] = _fast_apply_rows(kind, P, Q)
            a, bb, P_U, P_L, c = _kernels(coef)(lr[b, h, t0:t1], mom[b, h, t0:t1],
                                                decay[b, h, t0:t1])
            fac = chunk_grads(kind, loss, P, k[b, h, t0:t1], v[b, h, t0:t1])
            dM = pack(kind, weighted_sum(fac, a))
            dW = pack(kind, weighted_sum(fac, bb))
            M_new = P_U * M - dM
            W_new = P_L * W + c * M - dW
            W, M = W_new, M_new
        W_end[b, h] = W
        M_end[b, h] = M
    if return_starts:
        return out, W_end, M_end, starts
    return out, W_end, M_end


def _fast_apply_rows(kind, P, X):
    if kind == LINEAR:
        return X @ P["W"].T
    if kind == GELU:
        return gelu(X @ P["W1"].T) @ P["W2"].T
    return (silu(X @ P["W1"].T) * (X @ P["W3"].T)) @ P["W2"].T


# --------------------------------------------------------------------------- backward: per token
def seq_bwd(kind, q, k, v, lr, mom, decay, W0, M0, C, dout, dW_end=None, dM_end=None,
            d_h=0, loss=LOSS_MSE, heads=None):
    """Reverse of seq_fwd's token loop. For the scalar objective
        L = sum_t <dout_t, out_t> + <dW_end, W_end> + <dM_end, M_end>
    returns dict dq, dk, dv, dlr, dmom, ddecay, dW0, dM0.

    Per token (reverse order), undoing  W_t = lam_t W_{t-1} + M_t  and then
    M_t = mu_t M_{t-1} - eta_t g_t:
        Mbar += Wbar ; dlam_t = <Wbar, W_{t-1}> ; Wbar = lam_t Wbar
        dmu_t = <Mbar, M_{t-1}> ; deta_t = -<Mbar, g_t> ; gbar_t = -eta_t Mbar ;
        Mbar = mu_t Mbar
    and gbar_t flows through g_t(W_chunk_start, k_t, v_t) (second-order terms).
    After a chunk's tokens, the chunk-start weights collect the chain adjoint,
    the gradient-path adjoints and the output-path adjoints. The states
    W_{t-1}, M_{t-1} are recomputed per segment of about sqrt(C) tokens from
    checkpoints, so memory stays O(sqrt(C) S)."""
    q, k, v, lr, mom, decay, W0, M0, dout = map(_f64, (q, k, v, lr, mom, decay, W0, M0, dout))
    B, H, T = lr.shape
    d_k, d_v, S = _dims(kind, q, v, W0, d_h)
    chunks = _chunks(T, C)
    dW_end = np.zeros((B, H, S)) if dW_end is None else _f64(dW_end)
    dM_end = np.zeros((B, H, S)) if dM_end is None else _f64(dM_end)
    res = {n: np.zeros(x.shape) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("dlr", lr), ("dmom", mom), ("ddecay", decay),
            ("dW0", W0), ("dM0", M0))}
    hl = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in hl:
        # forward pass to get each chunk's start state
        W = W0[b, h].copy()
        M = M0[b, h].copy()
        starts = []
        for (t0, t1) in chunks:
            starts.append((W.copy(), M.copy()))
            Wc = unpack(kind, W.copy(), d_k, d_v, d_h)
            for t in range(t0, t1):
                g = pack(kind, loss_grad(kind, loss, Wc, k[b, h, t], v[b, h, t]))
                M = mom[b, h, t] * M - lr[b, h, t] * g
                W = decay[b, h, t] * W + M
        Wbar = dW_end[b, h].copy()
        Mbar = dM_end[b, h].copy()
        for ci in range(len(chunks) - 1, -1, -1):
            t0, t1 = chunks[ci]
            Ws, Ms = starts[ci]
            Pc = unpack(kind, Ws.copy(), d_k, d_v, d_h)
            Pbar = np.zeros(S)
            seg = max(1, int(math.isqrt(t1 - t0)))
            # checkpoints of (W, M) before each segment
            ckpt = []
            Wr, Mr = Ws.copy(), Ms.copy()
            for s0 in range(t0, t1, seg):
                ckpt.append((s0, Wr.copy(), Mr.copy()))
                for t in range(s0, min(s0 + seg, t1)):
                    g = pack(kind, loss_grad(kind, loss, Pc, k[b, h, t], v[b, h, t]))
                    Mr = mom[b, h, t] * Mr - lr[b, h, t] * g
                    Wr = decay[b, h, t] * Wr + Mr
            for (s0, Wc0, Mc0) in reversed(ckpt):
                s1 = min(s0 + seg, t1)
                prevW, prevM, grads = [], [], []
                Wr, Mr = Wc0.copy(), Mc0.copy()
                for t in range(s0, s1):
                    prevW.append(Wr.copy())
                    prevM.append(Mr.copy())
                    g = pack(kind, loss_grad(kind, loss, Pc, k[b, h, t], v[b, h, t]))
                    grads.append(g)
                    Mr = mom[b, h, t] * Mr - lr[b, h, t] * g
                    Wr = decay[b, h, t] * Wr + Mr
                for i in range(s1 - s0 - 1, -1, -1):
                    t = s0 + i
                    # undo W_t = lam_t W_{t-1} + M_t
                    Mbar = Mbar + Wbar
                    res["ddecay"][b, h, t] = np.dot(Wbar, prevW[i])
                    Wbar = decay[b, h, t] * Wbar
                    # undo M_t = mu_t M_{t-1} - eta_t g_t
                    res["dmom"][b, h, t] = np.dot(Mbar, prevM[i])
                    res["dlr"][b, h, t] = -np.dot(Mbar, grads[i])
                    gbar = unpack(kind, -lr[b, h, t] * Mbar, d_k, d_v, d_h)
                    Mbar = mom[b, h, t] * Mbar
                    Pb, kb, vb = loss_grad_vjp(kind, loss, Pc, k[b, h, t], v[b, h, t], gbar)
                    Pbar += pack(kind, Pb)
                    res["dk"][b, h, t] += kb
                    res["dv"][b, h, t] += vb
            for t in range(t0, t1):
                Pb, qb = fast_apply_vjp(kind, Pc, q[b, h, t], dout[b, h, t])
                Pbar += pack(kind, Pb)
                res["dq"][b, h, t] = qb
            Wbar = Wbar + Pbar
        res["dW0"][b, h] = Wbar
        res["dM0"][b, h] = Mbar
    return res


# --------------------------------------------------------------------------- backward: closed form
def chunk_kernels_vjp(eta, mu, lam, abar, bbar, PUbar, PLbar, cbar):
    """Adjoint of chunk_kernels for one chunk, without dividing by any gate.
    With X_1 = PUbar, X_{s+1} = mu_s X_s + abar_s eta_s  and
         Y_1 = cbar,  Y_{s+1} = mu_s Y_s + bbar_s eta_s,
         V_1 = PLbar, V_{s+1} = lam_s V_s + Y_{s+1}:
        deta_t = abar_t U(t+1,C) + bbar_t R_t
        dmu_s  = U(s+1,C) X_s + R_s Y_s
        dlam_s = L(s+1,C) V_s
    (each term is the derivative of a product definition with the factor s
    removed, summed with the running products above)."""
    eta, mu, lam = _f64(eta), _f64(mu), _f64(lam)
    abar, bbar = _f64(abar), _f64(bbar)
    n = eta.shape[0]
    sufU = np.ones(n + 1)
    sufL = np.ones(n + 1)
    for j in range(n - 1, -1, -1):
        sufU[j] = sufU[j + 1] * mu[j]
        sufL[j] = sufL[j + 1] * lam[j]
    # R_t (0-based t): R_{n-1} = 1 ; R_t = L(t+2..) + mu_{t+1} R_{t+1}
    R = np.zeros(n)
    R[n - 1] = 1.0
    for t in range(n - 2, -1, -1):
        R[t] = sufL[t + 1] + mu[t + 1] * R[t + 1]
    deta = abar * sufU[1:] + bbar * R
    dmu = np.zeros(n)
    dlam = np.zeros(n)
    X, Y, V = float(PUbar), float(cbar), float(PLbar)
    for s in range(n):
        dmu[s] = sufU[s + 1] * X + R[s] * Y
        dlam[s] = sufL[s + 1] * V
        X = mu[s] * X + abar[s] * eta[s]
        Y = mu[s] * Y + bbar[s] * eta[s]
        V = lam[s] * V + Y
    return deta, dmu, dlam


def closed_bwd(kind, q, k, v, lr, mom, decay, W0, M0, C, dout, dW_end=None, dM_end=None,
               d_h=0, loss=LOSS_MSE, heads=None, coef=COEF_PER_TOKEN, starts=None):
    """Adjoint of closed_fwd, chunk by chunk in reverse. With D_W, D_M the
    adjoints of the chunk-end states and G_t = a_t D_M + b_t D_W:
        dM0 = P_U D_M + c D_W
        dW0 = P_L D_W + grad_W0 sum_t <dout_t, f_W0(q_t)> - sum_t VJP_g(G_t)
        abar_t = -<D_M, g_t>,  bbar_t = -<D_W, g_t>
        PUbar = <D_M, M0>,  PLbar = <D_W, W0>,  cbar = <D_W, M0>
    then chunk_kernels_vjp gives the gate gradients. For the chunk-averaged
    variant every token's a_t is the mean of the per-token kernels, so each
    per-token kernel receives the mean of abar (and of bbar) before the VJP.
    ``starts`` [n_chunks,B,H,2,S] optionally gives the chunk-start states to
    differentiate at (the backward's saved-state input) instead of recomputing
    them from W0, M0."""
    q, k, v, lr, mom, decay, W0, M0, dout = map(_f64, (q, k, v, lr, mom, decay, W0, M0, dout))
    B, H, T = lr.shape
    d_k, d_v, S = _dims(kind, q, v, W0, d_h)
    chunks = _chunks(T, C)
    dW_end = np.zeros((B, H, S)) if dW_end is None else _f64(dW_end)
    dM_end = np.zeros((B, H, S)) if dM_end is None else _f64(dM_end)
    res = {n: np.zeros(x.shape) for n, x in
           (("dq", q), ("dk", k), ("dv", v), ("dlr", lr), ("dmom", mom), ("ddecay", decay),
            ("dW0", W0), ("dM0", M0))}
    if starts is None:
        _, _, _, starts = closed_fwd(kind, q, k, v, lr, mom, decay, W0, M0, C, d_h, loss,
                                     return_starts=True, heads=heads, coef=coef)
    else:
        starts = _f64(starts)
    hl = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in hl:
        DW = dW_end[b, h].copy()
        DM = dM_end[b, h].copy()
        for ci in range(len(chunks) - 1, -1, -1):
            t0, t1 = chunks[ci]
            Ws, Ms = starts[ci, b, h, 0], starts[ci, b, h, 1]
            P = unpack(kind, Ws, d_k, d_v, d_h)
            eta, mu, lam = lr[b, h, t0:t1], mom[b, h, t0:t1], decay[b, h, t0:t1]
            a, bb, P_U, P_L, c = _kernels(coef)(eta, mu, lam)
            abar = np.zeros(t1 - t0)
            bbar = np.zeros(t1 - t0)
            Pbar = P_L * DW
            for i, t in enumerate(range(t0, t1)):
                g = pack(kind, loss_grad(kind, loss, P, k[b, h, t], v[b, h, t]))
                abar[i] = -np.dot(DM, g)
                bbar[i] = -np.dot(DW, g)
                G = unpack(kind, -(a[i] * DM + bb[i] * DW), d_k, d_v, d_h)
                Pb, kb, vb = loss_grad_vjp(kind, loss, P, k[b, h, t], v[b, h, t], G)
                Pbar += pack(kind, Pb)
                res["dk"][b, h, t] += kb
                res["dv"][b, h, t] += vb
                Pb, qb = fast_apply_vjp(kind, P, q[b, h, t], dout[b, h, t])
                Pbar += pack(kind, Pb)
                res["dq"][b, h, t] = qb
            if coef == COEF_CHUNK_MEAN:
                abar = np.full_like(abar, abar.mean())
                bbar = np.full_like(bbar, bbar.mean())
            PUbar = np.dot(DM, Ms)
            PLbar = np.dot(DW, Ws)
            cbar = np.dot(DW, Ms)
            deta, dmu, dlam = chunk_kernels_vjp(eta, mu, lam, abar, bbar, PUbar, PLbar, cbar)
            res["dlr"][b, h, t0:t1] = deta
            res["dmom"][b, h, t0:t1] = dmu
            res["ddecay"][b, h, t0:t1] = dlam
            DM, DW = P_U * DM + c * DW, Pbar
        res["dW0"][b, h] = DW
        res["dM0"][b, h] = DM
    return res


def rel_fro(x, ref):
    """Relative Frobenius error |x - ref| / |ref| (|ref| = 0 -> absolute)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.linalg.norm(ref))
    num = float(np.linalg.norm(x - ref))
    return num / den if den > 0 else num
