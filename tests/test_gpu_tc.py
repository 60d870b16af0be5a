"""GPU parity of the tcgen05 tensor-core forward (bf16 GEMM operands, fp32
accumulation and state) against the fp64 oracle, at the workloads' full sizes.

Each workload runs as stated and with state-preserving gates (the stated decay
range collapses the SwiGLU state within a few chunks). The GPU computes every
head. Tolerance: 2e-2 relative Frobenius error of each output tensor (out,
W_end, M_end and the saved chunk-start states) over the heads the oracle
recomputes: all heads for the stated workloads, a sample for the
state-preserving variants (heads are independent), where every sampled head
must also pass on its own. Where the exact value lies below fp32 range
(|ref| < 1e-30) the error is taken relative to that floor.

On the stated 1.3B workloads the state collapses toward W = 0, where the
SwiGLU gradients are about quadratic in W, so a relative error in the state
roughly doubles every chunk; single heads whose state has collapsed then show
up to ~4e-2 while the tensor-level error stays near 1e-2 (the per-head maxima
are printed). test_tc_matches_rounding_model shows the GPU follows a model with
exactly the kernels' bf16 rounding points far more closely than that model
follows the oracle, i.e. this is the precision bf16 operands allow.
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from bf16_model import model_fwd
from gpu_util import device_inputs, host, run_fwd

pytestmark = pytest.mark.gpu
TOL = 2e-2
# Chunk-start states saved in the middle of a collapse (stated workloads only):
# while the state decays toward W = 0 a relative error roughly doubles per chunk
# before the state underflows; outputs and final states keep TOL.
TOL_COLLAPSE_MID = 5e-2


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


STATED = ("swiglu_d128", "layer_1p3b_2k", "layer_1p3b_16k")
# one head of every batch row and every head index, for the 32-head 1.3B layer
EIGHT_HEADS = [(0, 0), (0, 5), (1, 1), (1, 6), (2, 2), (2, 7), (3, 3), (3, 4)]
CASES = {
    "swiglu_d128": (gen.BY_NAME["swiglu_d128"], None),
    "swiglu_d128_preserving": (gen.state_preserving(gen.BY_NAME["swiglu_d128"]), None),
    "layer_1p3b_2k": (gen.BY_NAME["layer_1p3b_2k"], None),
    "layer_1p3b_2k_preserving": (gen.state_preserving(gen.BY_NAME["layer_1p3b_2k"]), EIGHT_HEADS),
    "layer_1p3b_16k": (gen.BY_NAME["layer_1p3b_16k"], None),
    "layer_1p3b_16k_preserving": (gen.state_preserving(gen.BY_NAME["layer_1p3b_16k"]), None),
    "linear_bf16": (gen.Workload("lin", gen.LINEAR, gen.BF16, 2, 2, 128, 256, 0, 512, 128, "uniform",
                                 0.999, seed=21, lr_lo=0.002, lr_hi=0.02), None),
    "swiglu_dot": (gen.Workload("dot", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 256, "uniform",
                                0.999, seed=22, lr_lo=0.0005, lr_hi=0.005, mom_lo=0.5, mom_hi=0.9,
                                loss=gen.LOSS_NEG_DOT), None),
    # the GELU MLP fast weight (state-preserving gates: W = 0 is a fixed point here too)
    "gelu_d128_preserving": (gen.Workload("gelu", gen.GELU, gen.BF16, 1, 2, 128, 128, 256, 512, 128,
                                          "uniform", 0.999, seed=24, lr_lo=0.002, lr_hi=0.02), None),
    "layer_1p3b_2k_gelu_preserving": (gen.state_preserving(gen.BY_NAME["layer_1p3b_2k_gelu"]),
                                      EIGHT_HEADS),
    # a shorter last chunk (T % C != 0), run padded to C tokens: 88 real tokens
    # in the last chunk (one part-filled 128-row tile, one all padding) ...
    "swiglu_tail_88": (gen.Workload("tail88", gen.SWIGLU, gen.BF16, 2, 2, 128, 128, 256, 600, 256,
                                    "uniform", 0.999, seed=26, lr_lo=0.002, lr_hi=0.02), None),
    # ... a single chunk shorter than C ...
    "swiglu_single_short": (gen.Workload("short", gen.SWIGLU, gen.BF16, 1, 3, 128, 128, 256, 200, 256,
                                         "uniform", 0.999, seed=27, lr_lo=0.002, lr_hi=0.02), None),
    # ... one whole 128-row tile real and the rest padding, linear fast weight ...
    "linear_tail_128": (gen.Workload("lintail", gen.LINEAR, gen.BF16, 2, 2, 128, 256, 0, 640, 512,
                                     "uniform", 0.999, seed=28, lr_lo=0.002, lr_hi=0.02), None),
    # ... and the GELU MLP with 44 real tokens in the last of three chunks
    "gelu_tail_44": (gen.Workload("geltail", gen.GELU, gen.BF16, 2, 2, 128, 128, 256, 300, 128,
                                  "uniform", 0.999, seed=29, lr_lo=0.002, lr_hi=0.02), None),
}


def _run(E, name):
    w, heads = CASES[name]
    assert E.e2ttt_fwd_uses_tensor_cores(shape_of(E, w)) == 1
    x = gen.generate(w, m0_scale=0.0 if name in STATED else 0.5)  # the stated workloads have M0 = 0
    d = device_inputs(w, x)
    ws = E.workspace(shape_of(E, w))
    out, W_end, M_end, saved = run_fwd(E, w, d, save=True, ws=ws)
    E.e2ttt_workspace_status(ws)
    return w, heads, x, (host(out), host(W_end), host(M_end), host(saved))


@pytest.mark.parametrize("name", list(CASES))
def test_tc_fwd_matches_oracle(E, name):
    w, heads, x, (o, We, Me, sv) = _run(E, name)
    per_head_check = heads is not None or name not in STATED
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    ro, rW, rM, starts = O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                                      x["W0"], x["M0"], w.C, d_h=w.d_h, loss=w.loss,
                                      return_starts=True, heads=heads)
    bi = tuple(np.array(heads).T)
    whole = {"out": err(o[bi], ro[bi]), "W_end": err(We[bi], rW[bi]), "M_end": err(Me[bi], rM[bi])}
    for c in range(1, w.n_chunks):
        whole[f"W@{c}"] = err(sv[c][bi][:, 0], starts[c][bi][:, 0])
        whole[f"M@{c}"] = err(sv[c][bi][:, 1], starts[c][bi][:, 1])
    per_head = {n: max(err(a[b, h], r[b, h]) for (b, h) in heads)
                for n, a, r in (("out", o, ro), ("W_end", We, rW), ("M_end", Me, rM))}
    print(f"\n{name}: tensor-level {dict((k, f'{v:.2e}') for k, v in list(whole.items())[:3])}"
          f" per-head max {dict((k, f'{v:.2e}') for k, v in per_head.items())}")
    tol = lambda k: TOL_COLLAPSE_MID if (name in STATED and "@" in k) else TOL
    print(f"  saved-state max {max([v for k, v in whole.items() if '@' in k] or [0]):.2e}")
    bad = {k: v for k, v in whole.items() if not v < tol(k)}
    assert not bad, (name, bad)
    if per_head_check:
        bad = {k: v for k, v in per_head.items() if not v < TOL}
        assert not bad, (name, "per head", bad)


@pytest.mark.parametrize("name", ["swiglu_d128", "layer_1p3b_2k", "linear_bf16"])
def test_tc_matches_rounding_model(E, name):
    """GPU vs a model with the kernels' bf16 rounding points: much closer than
    either is to the fp64 oracle on the stated workloads."""
    w, heads, x, (o, We, Me, _) = _run(E, name)
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    mo, mW, mM = model_fwd(w, x, heads)
    for (b, h) in heads:
        assert err(o[b, h], mo[b, h]) < 2e-3
        assert err(We[b, h], mW[b, h]) < 5e-3
        assert err(Me[b, h], mM[b, h]) < 1e-2


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


def test_gelu_tc_and_cuda_core_paths_agree(E):
    """The GELU MLP through both forward paths (an unaligned view of q routes the
    call to the CUDA-core path)."""
    import torch
    w = gen.Workload("agree_gelu", gen.GELU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform",
                     0.999, seed=25, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    o1, W1, M1, _ = run_fwd(E, w, d)
    buf = torch.empty(d["q"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    qu = buf[1:].view_as(d["q"])
    qu.copy_(d["q"])
    d2 = dict(d)
    d2["q"] = qu
    o2, W2, M2, _ = run_fwd(E, w, d2)
    errs = (err(host(o1), host(o2)), err(host(W1), host(W2)), err(host(M1), host(M2)))
    print(f"\ngelu tensor-core vs CUDA-core: {errs}")
    assert max(errs) < 2e-2, errs
