"""Rounding model of the tensor-core forward, for diagnosing parity.

Not the oracle: this restates the closed-form chunk transition with every GEMM
operand rounded to bf16 at the points where the tcgen05 path rounds it (bf16
copies of the chunk-start weights, the activations A = silu(H1) H3, the
residual E and its a-/b-scaled copies, dH1 and dH3, the a-/b-scaled keys,
silu(H1_k) and H3_k silu'(H1_k)),
everything else in fp64, the fast-weight state rounded to fp32 once per chunk.
Comparing the GPU with this model separates kernel mistakes (GPU far from the
model) from the precision bf16 operands allow (model far from the oracle).
"""
import numpy as np

import e2ttt_inputs as gen
import oracle as O


def bf(x):
    return gen.round_to_bf16(np.asarray(x, np.float32)).astype(np.float64)


def f32(x):
    return np.asarray(x, np.float32).astype(np.float64)


def model_fwd(w, x, heads):
    d_k, d_v, d_h, C = w.d_k, w.d_v, w.d_h, w.C
    S = w.state_elems
    out = np.zeros((w.B, w.H, w.T, d_v))
    W_end = np.zeros((w.B, w.H, S))
    M_end = np.zeros((w.B, w.H, S))
    for (b, h) in heads:
        W = f32(x["W0"][b, h])
        M = f32(x["M0"][b, h])
        for t0 in range(0, w.T, C):
            t1 = t0 + C
            a, bb, PU, PL, c = O.chunk_kernels(x["lr"][b, h, t0:t1], x["mom"][b, h, t0:t1],
                                               x["decay"][b, h, t0:t1])
            Q = np.asarray(x["q"][b, h, t0:t1], np.float64)
            K = np.asarray(x["k"][b, h, t0:t1], np.float64)
            V = np.asarray(x["v"][b, h, t0:t1], np.float64)
            if w.kind == gen.LINEAR:
                Ws = bf(W.reshape(d_v, d_k))
                out[b, h, t0:t1] = bf(Q @ Ws.T)
                e = (K @ Ws.T - V) if w.loss == gen.LOSS_MSE else -V
                dM = (bf(a[:, None] * e).T @ K).reshape(-1)
                dW = (bf(bb[:, None] * e).T @ K).reshape(-1)
            else:
                n1 = d_h * d_k
                W1s = bf(W[:n1].reshape(d_h, d_k))
                W3s = bf(W[n1:2 * n1].reshape(d_h, d_k))
                W2s = bf(W[2 * n1:].reshape(d_v, d_h))
                H1q, H3q = f32(Q @ W1s.T), f32(Q @ W3s.T)
                H1k, H3k = f32(K @ W1s.T), f32(K @ W3s.T)
                Aq = bf(O.silu(H1q) * H3q)
                Ak = bf(O.silu(H1k) * H3k)
                s1 = bf(O.silu(H1k))
                s2 = bf(H3k * O.dsilu(H1k))
                out[b, h, t0:t1] = bf(Aq @ W2s.T)
                e = f32(Ak @ W2s.T) - V if w.loss == gen.LOSS_MSE else -V
                dA = f32(bf(e) @ W2s)
                dH1, dH3 = bf(dA * s2), bf(dA * s1)
                Ka, Kb = bf(a[:, None] * K), bf(bb[:, None] * K)
                Ea, Eb = bf(a[:, None] * e), bf(bb[:, None] * e)
                dM = np.concatenate([(dH1.T @ Ka).reshape(-1), (dH3.T @ Ka).reshape(-1),
                                     (Ea.T @ Ak).reshape(-1)])
                dW = np.concatenate([(dH1.T @ Kb).reshape(-1), (dH3.T @ Kb).reshape(-1),
                                     (Eb.T @ Ak).reshape(-1)])
            M_new = f32(PU * M - dM)
            W = f32(PL * W + c * M - dW)
            M = M_new
        W_end[b, h] = W
        M_end[b, h] = M
    return out, W_end, M_end
