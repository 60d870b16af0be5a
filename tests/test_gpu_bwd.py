"""GPU parity of e2ttt_chunk_scan_bwd against the fp64 oracle's adjoint.

The oracle's closed-form adjoint is pinned on the CPU to the per-token reverse
loop and to finite differences (tests/test_oracle.py). Here the GPU forward
saves the chunk-start states, the GPU backward consumes them, and every
gradient (dq, dk, dv, dlr, dmom, ddecay, dW0, dM0) is compared with the oracle
at tensor level: 1e-4 relative Frobenius error for fp32 activations, 2e-2 for
bf16 activations (bf16 inputs and forward operands).
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import dev, device_inputs, host, run_fwd

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dlr", "dmom", "ddecay", "dW0", "dM0")


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


def err(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30 * np.sqrt(ref.size)))


def run_bwd(E, w, x, dW, dM, heads=None):
    import torch
    d = device_inputs(w, x)
    _, _, _, saved = run_fwd(E, w, d, save=True)
    g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], saved, d["dout"],
                         None if dW is None else dev(dW), None if dM is None else dev(dM),
                         C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss)
    torch.cuda.synchronize()
    gpu = {n: host(t) for n, t in g.items()}
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, dM, d_h=w.d_h, loss=w.loss, heads=heads)
    return gpu, ref


def check(gpu, ref, tol, heads=None, label=""):
    if heads is None:
        errs = {n: err(gpu[n], ref[n]) for n in NAMES}
    else:
        bi = tuple(np.array(heads).T)
        errs = {n: err(gpu[n][bi], ref[n][bi]) for n in NAMES}
    print(f"\n{label}: " + " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    bad = {n: e for n, e in errs.items() if not e < tol}
    assert not bad, (label, bad)


F32 = {
    "linear_mse": gen.Workload("bl", gen.LINEAR, gen.F32, 1, 2, 24, 16, 0, 70, 32, "uniform", 0.99,
                               seed=41),
    "linear_dot": gen.Workload("bld", gen.LINEAR, gen.F32, 2, 1, 16, 24, 0, 64, 16, "uniform", 0.99,
                               seed=42, loss=gen.LOSS_NEG_DOT),
    "swiglu_mse": gen.Workload("bs", gen.SWIGLU, gen.F32, 1, 2, 16, 12, 24, 50, 16, "uniform", 0.99,
                               seed=43, lr_lo=0.002, lr_hi=0.02, mom_lo=0.7, mom_hi=0.95),
    "swiglu_dot": gen.Workload("bsd", gen.SWIGLU, gen.F32, 2, 1, 12, 16, 20, 48, 16, "uniform", 0.99,
                               seed=44, loss=gen.LOSS_NEG_DOT, lr_lo=0.001, lr_hi=0.005,
                               mom_lo=0.5, mom_hi=0.9),
    "gelu_mse": gen.Workload("bg", gen.GELU, gen.F32, 1, 2, 16, 12, 24, 50, 16, "uniform", 0.99,
                             seed=47, lr_lo=0.002, lr_hi=0.02, mom_lo=0.7, mom_hi=0.95),
    "gelu_dot": gen.Workload("bgd", gen.GELU, gen.F32, 2, 1, 12, 16, 20, 48, 16, "uniform", 0.99,
                             seed=48, loss=gen.LOSS_NEG_DOT, lr_lo=0.001, lr_hi=0.005,
                             mom_lo=0.5, mom_hi=0.9),
    # full chunks of 128, 256 and 512 tokens, where the gate gradients come from
    # the block-per-chunk form of the K1 adjoint (1, 2 and 4 tokens per thread;
    # the chunks of 16 to 32 tokens above take its one-warp-per-chunk form)
    "linear_c128": gen.Workload("blc1", gen.LINEAR, gen.F32, 1, 2, 16, 12, 0, 384, 128, "uniform",
                                0.99, seed=61, lr_lo=0.002, lr_hi=0.02),
    "swiglu_c256": gen.Workload("bsc2", gen.SWIGLU, gen.F32, 1, 2, 12, 16, 20, 512, 256, "uniform",
                                0.99, seed=62, lr_lo=0.002, lr_hi=0.02, mom_lo=0.7, mom_hi=0.95),
    "linear_c512": gen.Workload("blc5", gen.LINEAR, gen.F32, 2, 1, 8, 8, 0, 1024, 512, "uniform",
                                0.99, seed=63, lr_lo=0.002, lr_hi=0.01),
}


@pytest.mark.parametrize("name", list(F32))
@pytest.mark.parametrize("upstream", [True, False])
def test_bwd_f32_matches_oracle(E, name, upstream):
    w = F32[name]
    x = gen.generate(w, m0_scale=0.5)
    dW, dM = gen.upstream_state_grads(w, seed=7, scale=0.3) if upstream else (None, None)
    gpu, ref = run_bwd(E, w, x, dW, dM)
    check(gpu, ref, 1e-4, label=f"{name} upstream={upstream}")


def test_bwd_tiny_linear_workload(E):
    """The tiny linear fp32 workload at its full size (256 tokens, 4 chunks)."""
    w = gen.BY_NAME["tiny_linear"]
    x = gen.generate(w)
    dW, dM = gen.upstream_state_grads(w, seed=0)
    gpu, ref = run_bwd(E, w, x, dW, dM)
    check(gpu, ref, 1e-4, label="tiny_linear")


def test_bwd_bf16_small(E):
    w = gen.Workload("bb", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=45, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    dW, dM = gen.upstream_state_grads(w, seed=8, scale=0.1)
    gpu, ref = run_bwd(E, w, x, dW, dM)
    check(gpu, ref, 2e-2, label="swiglu_bf16_small")


@pytest.mark.parametrize("variant", ["stated", "preserving", "preserving_upstream"])
def test_bwd_training_workload(E, variant):
    """fwd then bwd at the 1.3B layer's shapes (B=4, H=8, d=256, d_h=512, T=2048,
    C=512), upstream dOut ~ N(0,1); the oracle recomputes two heads. The last
    variant also feeds upstream gradients of the final states, dW_end and
    dM_end ~ N(0, 0.1^2) (a layer whose carried state is read by a later
    segment), on the state-preserving gates that keep them from decaying away."""
    w = gen.BY_NAME["train_1p3b_2k"]
    if variant != "stated":
        w = gen.state_preserving(w)
    x = gen.generate(w, m0_scale=0.0 if variant == "stated" else 0.5)
    dW, dM = (gen.upstream_state_grads(w, seed=11, scale=0.1) if variant == "preserving_upstream"
              else (None, None))
    heads = [(0, 0), (3, 7)]
    gpu, ref = run_bwd(E, w, x, dW, dM, heads=heads)
    check(gpu, ref, 2e-2, heads=heads, label=f"train_1p3b_2k {variant}")


def test_bwd_tensor_core_and_cuda_core_agree(E):
    """One bf16 problem through both backward paths: a 2-byte offset view of dout
    makes the pointers unaligned for TMA, which routes the call to the CUDA-core
    backward."""
    import torch
    w = gen.Workload("agreeb", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=46, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    _, _, _, saved = run_fwd(E, w, d, save=True)
    dW, dM = (dev(a) for a in gen.upstream_state_grads(w, seed=9, scale=0.1))
    args = (d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], saved)
    kw = dict(C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss)
    g_tc = E.chunk_scan_bwd(*args, d["dout"], dW, dM, **kw)
    buf = torch.empty(d["dout"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    dout_u = buf[1:].view_as(d["dout"])
    dout_u.copy_(d["dout"])
    g_cc = E.chunk_scan_bwd(*args, dout_u, dW, dM, **kw)
    torch.cuda.synchronize()
    errs = {n: err(host(g_tc[n]), host(g_cc[n])) for n in NAMES}
    print("\ntensor-core vs CUDA-core backward:", " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    assert all(e < 2e-2 for e in errs.values()), errs


@pytest.mark.parametrize("T,C,B,H", [(600, 256, 2, 2), (200, 256, 1, 3), (640, 512, 1, 2)])
def test_bwd_bf16_shorter_last_chunk(E, T, C, B, H):
    """SwiGLU, bf16, T % C != 0: the tensor-core forward and backward run the last
    chunk padded to C tokens (88 real tokens in two 128-row tiles; one chunk of
    200; one real 128-row tile of four)."""
    w = gen.Workload("btail", gen.SWIGLU, gen.BF16, B, H, 128, 128, 256, T, C, "uniform", 0.999,
                     seed=47 + T, lr_lo=0.002, lr_hi=0.02)
    assert E.e2ttt_fwd_uses_tensor_cores(
        E.make_shape(B, H, T, C, 128, 128, 256, E.SWIGLU, E.BF16)) == 1
    x = gen.generate(w, m0_scale=0.5)
    dW, dM = gen.upstream_state_grads(w, seed=10, scale=0.1)
    gpu, ref = run_bwd(E, w, x, dW, dM)
    check(gpu, ref, 2e-2, label=f"swiglu_bf16 T={T} C={C}")


def test_bwd_shorter_last_chunk_paths_agree(E):
    """T % C != 0 through both backward paths (the unaligned view of dout routes
    the call to the CUDA-core backward)."""
    import torch
    w = gen.Workload("agreet", gen.SWIGLU, gen.BF16, 2, 2, 128, 128, 256, 600, 256, "uniform", 0.999,
                     seed=48, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    _, _, _, saved = run_fwd(E, w, d, save=True)
    dW, dM = (dev(a) for a in gen.upstream_state_grads(w, seed=11, scale=0.1))
    args = (d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], saved)
    kw = dict(C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss)
    g_tc = E.chunk_scan_bwd(*args, d["dout"], dW, dM, **kw)
    buf = torch.empty(d["dout"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    dout_u = buf[1:].view_as(d["dout"])
    dout_u.copy_(d["dout"])
    g_cc = E.chunk_scan_bwd(*args, dout_u, dW, dM, **kw)
    torch.cuda.synchronize()
    errs = {n: err(host(g_tc[n]), host(g_cc[n])) for n in NAMES}
    print("\nshorter last chunk, tensor-core vs CUDA-core backward:",
          " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    assert all(e < 2e-2 for e in errs.values()), errs


def test_bwd_gelu_bf16_small(E):
    """The GELU MLP with bf16 activations end to end: GPU forward (saved states)
    and tensor-core backward against the fp64 oracle's adjoint computed from the
    inputs alone (no GPU value enters the reference). M0 = 0 as in the stated
    workloads, where the exact gradients move by under 5e-3 when the weights are
    rounded to bf16 (test_oracle.py: test_gelu_backward_conditioning_under_bf16_weights),
    so the 2e-2 bar applies as for SwiGLU."""
    w = gen.Workload("bgb", gen.GELU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=49, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.0)
    dW, dM = gen.upstream_state_grads(w, seed=8, scale=0.1)
    gpu, ref = run_bwd(E, w, x, dW, dM)
    check(gpu, ref, 2e-2, label="gelu_bf16_small end to end")


def test_bwd_gelu_ill_conditioned_fp32_gemms(E):
    """GELU MLP, bf16 activations, M0 != 0 and upstream state gradients: rounding
    the chunk-start weights to bf16 moves the exact gradients by 3-15 % (pinned
    on the CPU by test_gelu_backward_conditioning_under_bf16_weights), so no
    path with bf16 weight operands meets 2e-2 here. With gemm = GEMM_FP32 the
    forward and the backward run the fp32 CUDA-core kernels; compared end to end
    with the oracle from the inputs alone."""
    import torch
    w = gen.Workload("bgi", gen.GELU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=49, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    dW, dM = gen.upstream_state_grads(w, seed=8, scale=0.1)
    d = device_inputs(w, x)
    assert E.e2ttt_fwd_uses_tensor_cores(
        E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, gemm=E.GEMM_FP32)) == 0
    kw = dict(C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss, gemm=E.GEMM_FP32)
    _, _, _, saved = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], d["W0"],
                                      d["M0"], save_states=True, **kw)
    g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], saved, d["dout"],
                         dev(dW), dev(dM), **kw)
    torch.cuda.synchronize()
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, dM, d_h=w.d_h, loss=w.loss)
    # dq, dk, dv come back in the activations' bf16 (rounding 2^-9 per element):
    # 1e-2, a tenth of what bf16 weights move; the gate and state gradients are
    # fp32 throughout: 1e-3
    gpu = {n: host(t) for n, t in g.items()}
    check(gpu, ref, 1e-2, label="gelu ill-conditioned, fp32 GEMMs, end to end")
    for n in ("dlr", "dmom", "ddecay", "dW0", "dM0"):
        assert err(gpu[n], ref[n]) < 1e-3, (n, err(gpu[n], ref[n]))


@pytest.mark.parametrize("T,C,loss", [(300, 128, gen.LOSS_MSE), (512, 128, gen.LOSS_NEG_DOT)])
def test_bwd_gelu_bf16_tail_and_dot(E, T, C, loss):
    """GELU MLP, tensor-core forward and backward: a shorter last chunk (44 real
    tokens of 128) and the negative-dot loss, end to end (M0 = 0, where bf16
    weights move the exact gradients by under 5e-3)."""
    w = gen.Workload("bgt", gen.GELU, gen.BF16, 2, 2, 128, 128, 256, T, C, "uniform", 0.999,
                     seed=61 + T, lr_lo=0.002, lr_hi=0.02, loss=loss)
    x = gen.generate(w, m0_scale=0.0)
    dW, dM = gen.upstream_state_grads(w, seed=12, scale=0.1)
    gpu, ref = run_bwd(E, w, x, dW, dM)
    check(gpu, ref, 2e-2, label=f"gelu_bf16 T={T} C={C} loss={loss}")


def test_bwd_gelu_tensor_core_and_cuda_core_agree(E):
    """The GELU MLP backward through both paths on the same saved states (an
    unaligned view of dout routes the call to the CUDA-core backward), M0 = 0."""
    import torch
    w = gen.Workload("agreeg", gen.GELU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=63, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.0)
    d = device_inputs(w, x)
    _, _, _, saved = run_fwd(E, w, d, save=True)
    dW, dM = (dev(a) for a in gen.upstream_state_grads(w, seed=13, scale=0.1))
    args = (d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], saved)
    kw = dict(C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss)
    g_tc = E.chunk_scan_bwd(*args, d["dout"], dW, dM, **kw)
    buf = torch.empty(d["dout"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    dout_u = buf[1:].view_as(d["dout"])
    dout_u.copy_(d["dout"])
    g_cc = E.chunk_scan_bwd(*args, dout_u, dW, dM, **kw)
    torch.cuda.synchronize()
    errs = {n: err(host(g_tc[n]), host(g_cc[n])) for n in NAMES}
    print("\ngelu tensor-core vs CUDA-core backward:", " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    assert all(e < 2e-2 for e in errs.values()), errs


def test_bwd_gelu_training_shapes(E):
    """GELU MLP at the 1.3B layer's training shapes (B=4, H=8, d=256, d_h=512,
    T=2048, C=512; state-preserving gates, M0 = 0), tensor-core forward and
    backward end to end; the oracle recomputes two heads from the inputs."""
    w = gen.state_preserving(gen.BY_NAME["layer_1p3b_2k_gelu"])
    x = gen.generate(w, m0_scale=0.0)
    heads = [(0, 0), (3, 7)]
    gpu, ref = run_bwd(E, w, x, None, None, heads=heads)
    check(gpu, ref, 2e-2, heads=heads, label="layer_1p3b_2k_gelu preserving")
