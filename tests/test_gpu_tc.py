"""GPU parity of the tcgen05 tensor-core forward (bf16 GEMM operands, fp32
accumulation and state) against the fp64 oracle, at the workloads' full sizes.

Each workload runs as stated and with state-preserving gates (the stated decay
range collapses the SwiGLU state within a few chunks). The GPU computes every
head; the oracle recomputes a sample of heads (heads are independent).
Tolerance: 2e-2 relative Frobenius error per output and per sampled head;
where the exact value lies below fp32 range (|ref| < 1e-30) the error is taken
relative to that floor.
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import device_inputs, host, run_fwd

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


def err(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    floor = 1e-30 * np.sqrt(ref.size)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), floor))


def shape_of(E, w):
    return E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss)


CASES = {
    "swiglu_d128": (gen.BY_NAME["swiglu_d128"], None),
    "swiglu_d128_preserving": (gen.state_preserving(gen.BY_NAME["swiglu_d128"]), None),
    "layer_1p3b_2k": (gen.BY_NAME["layer_1p3b_2k"], [(0, 0), (1, 3), (2, 5), (3, 7)]),
    "layer_1p3b_2k_preserving": (gen.state_preserving(gen.BY_NAME["layer_1p3b_2k"]), [(0, 1), (3, 6)]),
    "layer_1p3b_16k": (gen.BY_NAME["layer_1p3b_16k"], [(0, 0), (0, 5)]),
    "layer_1p3b_16k_preserving": (gen.state_preserving(gen.BY_NAME["layer_1p3b_16k"]), [(0, 2)]),
    "linear_bf16": (gen.Workload("lin", gen.LINEAR, gen.BF16, 2, 2, 128, 256, 0, 512, 128, "uniform",
                                 0.999, seed=21, lr_lo=0.002, lr_hi=0.02), None),
    "swiglu_dot": (gen.Workload("dot", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 256, "uniform",
                                0.999, seed=22, lr_lo=0.0005, lr_hi=0.005, mom_lo=0.5, mom_hi=0.9,
                                loss=gen.LOSS_NEG_DOT), None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_tc_fwd_matches_oracle(E, name):
    w, heads = CASES[name]
    assert E.e2ttt_fwd_uses_tensor_cores(shape_of(E, w)) == 1
    stated = name in ("swiglu_d128", "layer_1p3b_2k", "layer_1p3b_16k")
    x = gen.generate(w, m0_scale=0.0 if stated else 0.5)  # the stated workloads have M0 = 0
    d = device_inputs(w, x)
    ws = E.workspace(shape_of(E, w))
    out, W_end, M_end, saved = run_fwd(E, w, d, save=True, ws=ws)
    E.e2ttt_workspace_status(ws)
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    ro, rW, rM, starts = O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                                      x["W0"], x["M0"], w.C, d_h=w.d_h, loss=w.loss,
                                      return_starts=True, heads=heads)
    o, We, Me, sv = host(out), host(W_end), host(M_end), host(saved)
    for (b, h) in heads:
        errs = {"out": err(o[b, h], ro[b, h]), "W_end": err(We[b, h], rW[b, h]),
                "M_end": err(Me[b, h], rM[b, h])}
        for c in range(1, w.n_chunks):
            errs[f"W@{c}"] = err(sv[c, b, h, 0], starts[c, b, h, 0])
            errs[f"M@{c}"] = err(sv[c, b, h, 1], starts[c, b, h, 1])
        bad = {k: v for k, v in errs.items() if not v < TOL}
        assert not bad, (name, (b, h), bad)


def test_tc_and_cuda_core_paths_agree(E):
    """The same bf16 problem through both paths: a 2-byte offset view of q makes
    the pointers unaligned for TMA, which routes the call to the CUDA-core path."""
    import torch
    w = gen.Workload("agree", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=23, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    a = run_fwd(E, w, d)
    qbuf = torch.empty(d["q"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    qv = qbuf[1:].view_as(d["q"])
    qv.copy_(d["q"])
    d2 = dict(d)
    d2["q"] = qv
    b = run_fwd(E, w, d2)
    for i in range(3):
        assert err(host(a[i]), host(b[i])) < TOL
