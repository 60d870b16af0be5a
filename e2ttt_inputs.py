"""Seeded synthetic inputs for the E2-TTT chunk scan.

This module is shared by the tests, the benchmark and the oracle's pins. It holds
the workload table and the random draws only; none of the method's arithmetic
lives here.

Workloads (shapes and distributions of the layer sizes the paper trains and
evaluates: a tiny linear fast weight, a per-head SwiGLU fast MLP, the 1.3B
hybrid layer at the 2K training context, and the same layer at 8x that context
for the length-extrapolation setting of "Rethinking Expressivity and
Efficiency in Test-Time Training", abstract and "Key results"):

    name             kind    act   B  H  d_k=d_v d_h   T      C    lr                mom          decay
    tiny_linear      linear  f32   1  1  32      -     256    64   U(.01,.1)         U(.8,.99)    U(.95,1)
    swiglu_d128      swiglu  bf16  2  4  128     256   2048   256  U(.01,.1)         U(.8,.99)    U(.95,1)
    layer_1p3b_2k    swiglu  bf16  4  8  256     512   2048   512  softplus(N(-3,1)) U(.8,.99)    U(.95,1)
    layer_1p3b_16k   swiglu  bf16  1  8  256     512   16384  512  softplus(N(-3,1)) U(.8,.99)    U(.98,1)
    train_1p3b_2k    = layer_1p3b_2k, plus an upstream gradient dOut ~ N(0,1)

Draw order (one numpy PCG64 generator seeded with the workload index):
q, k, v, lr, mom, decay, W0 (W1, W3, W2 for SwiGLU; W1, W2 for the GELU MLP; W
for linear), M0, dout.
q and k are N(0,1) then scaled to unit L2 norm per token and head; v ~ N(0,1).
Fast-weight matrices are N(0, 1/fan_in). M0 is zero unless ``m0_scale`` > 0, in
which case it is N(0, m0_scale^2 / fan_in) (tests use this to exercise the M0
terms). Activations of bf16 workloads are rounded once to bf16 (round to
nearest even) on the host; gates and fast-weight state are fp32.
"""
from __future__ import annotations

import dataclasses
import numpy as np

LINEAR = 0
SWIGLU = 1
GELU = 2      # two-matrix GELU MLP fast weight W2 gelu(W1 x)
F32 = 0
BF16 = 1
LOSS_MSE = 0
LOSS_NEG_DOT = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: int
    act: int
    B: int
    H: int
    d_k: int
    d_v: int
    d_h: int
    T: int
    C: int
    lr_dist: str          # "uniform" -> U(lr_lo, lr_hi); "softplus" -> softplus(N(-3, 1))
    decay_lo: float
    seed: int
    lr_lo: float = 0.01
    lr_hi: float = 0.1
    mom_lo: float = 0.8
    mom_hi: float = 0.99
    decay_hi: float = 1.0
    loss: int = LOSS_MSE
    with_bwd: bool = False

    @property
    def n_chunks(self) -> int:
        return -(-self.T // self.C)

    @property
    def state_elems(self) -> int:
        if self.kind == LINEAR:
            return self.d_v * self.d_k
        if self.kind == GELU:
            return self.d_h * self.d_k + self.d_v * self.d_h
        return 2 * self.d_h * self.d_k + self.d_v * self.d_h

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = [
    Workload("tiny_linear", LINEAR, F32, 1, 1, 32, 32, 0, 256, 64, "uniform", 0.95, seed=0),
    Workload("swiglu_d128", SWIGLU, BF16, 2, 4, 128, 128, 256, 2048, 256, "uniform", 0.95, seed=1),
    Workload("layer_1p3b_2k", SWIGLU, BF16, 4, 8, 256, 256, 512, 2048, 512, "softplus", 0.95, seed=2),
    Workload("layer_1p3b_16k", SWIGLU, BF16, 1, 8, 256, 256, 512, 16384, 512, "softplus", 0.98, seed=3),
    Workload("train_1p3b_2k", SWIGLU, BF16, 4, 8, 256, 256, 512, 2048, 512, "softplus", 0.95, seed=4,
             with_bwd=True),
    Workload("layer_1p3b_2k_gelu", GELU, BF16, 4, 8, 256, 256, 512, 2048, 512, "softplus", 0.95,
             seed=5),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def state_preserving(w: Workload) -> Workload:
    """The same shapes with gates that keep the fast-weight state O(1) over many
    chunks: lr ~ U(0.002, 0.02), decay ~ U(0.999, 1) (momentum unchanged).

    With the stated distributions (decay ~ U(0.95, 1) over 256-512 token chunks)
    the per-chunk decay product is about e^-13, so the SwiGLU state collapses to
    the W = 0 fixed point within two or three chunks and later chunks carry
    little signal. Parity tests run both variants."""
    return w.replace(name=w.name + "_preserving", lr_dist="uniform", lr_lo=0.002, lr_hi=0.02,
                     decay_lo=max(w.decay_lo, 0.999))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding bf16 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(x)
    out[nan] = np.nan
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The upper 16 bits of fp32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


def _softplus(z: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, z)


def generate(w: Workload, m0_scale: float = 0.0, seed: int | None = None,
             dtype_round: bool = True) -> dict:
    """Draw the seeded inputs of workload ``w``.

    Returns a dict of fp32 numpy arrays: q, k [B,H,T,d_k]; v [B,H,T,d_v];
    lr, mom, decay [B,H,T]; W0, M0 [B,H,S]; dout [B,H,T,d_v] (always drawn, last,
    so the earlier draws do not depend on whether a backward is run).
    For bf16 workloads q, k, v and dout hold bf16-representable values.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    B, H, T = w.B, w.H, w.T
    q = _unit_rows(rng.standard_normal((B, H, T, w.d_k)))
    k = _unit_rows(rng.standard_normal((B, H, T, w.d_k)))
    v = rng.standard_normal((B, H, T, w.d_v)).astype(np.float32)
    if w.lr_dist == "uniform":
        lr = rng.uniform(w.lr_lo, w.lr_hi, (B, H, T))
    elif w.lr_dist == "softplus":
        lr = _softplus(rng.normal(-3.0, 1.0, (B, H, T)))
    else:
        raise ValueError(w.lr_dist)
    mom = rng.uniform(w.mom_lo, w.mom_hi, (B, H, T))
    decay = rng.uniform(w.decay_lo, w.decay_hi, (B, H, T))
    if w.kind == LINEAR:
        W = rng.standard_normal((B, H, w.d_v, w.d_k)) / np.sqrt(w.d_k)
        W0 = W.reshape(B, H, -1)
        fan = np.full(W0.shape[-1], float(w.d_k))
    elif w.kind == GELU:
        W1 = rng.standard_normal((B, H, w.d_h, w.d_k)) / np.sqrt(w.d_k)
        W2 = rng.standard_normal((B, H, w.d_v, w.d_h)) / np.sqrt(w.d_h)
        W0 = np.concatenate([W1.reshape(B, H, -1), W2.reshape(B, H, -1)], axis=-1)
        fan = np.concatenate([np.full(w.d_h * w.d_k, float(w.d_k)),
                              np.full(w.d_v * w.d_h, float(w.d_h))])
    else:
        W1 = rng.standard_normal((B, H, w.d_h, w.d_k)) / np.sqrt(w.d_k)
        W3 = rng.standard_normal((B, H, w.d_h, w.d_k)) / np.sqrt(w.d_k)
        W2 = rng.standard_normal((B, H, w.d_v, w.d_h)) / np.sqrt(w.d_h)
        W0 = np.concatenate([W1.reshape(B, H, -1), W3.reshape(B, H, -1), W2.reshape(B, H, -1)], axis=-1)
        fan = np.concatenate([np.full(2 * w.d_h * w.d_k, float(w.d_k)),
                              np.full(w.d_v * w.d_h, float(w.d_h))])
    if m0_scale > 0:
        M0 = rng.standard_normal(W0.shape) * m0_scale / np.sqrt(fan)
    else:
        M0 = np.zeros(W0.shape)
    dout = rng.standard_normal((B, H, T, w.d_v)).astype(np.float32)
    out = dict(q=q, k=k, v=v,
               lr=lr.astype(np.float32), mom=mom.astype(np.float32), decay=decay.astype(np.float32),
               W0=W0.astype(np.float32), M0=M0.astype(np.float32), dout=dout)
    if w.act == BF16 and dtype_round:
        for name in ("q", "k", "v", "dout"):
            out[name] = round_to_bf16(out[name])
    return out


def upstream_state_grads(w: Workload, seed: int, scale: float = 1.0) -> tuple[np.ndarray, np.ndarray]:
    """Seeded upstream gradients dW_end, dM_end [B,H,S] (N(0, scale^2))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    S = w.state_elems
    dW = (rng.standard_normal((w.B, w.H, S)) * scale).astype(np.float32)
    dM = (rng.standard_normal((w.B, w.H, S)) * scale).astype(np.float32)
    return dW, dM
