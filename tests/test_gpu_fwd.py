"""GPU parity of the forward path against the fp64 oracle, through the C ABI.

Tolerances (relative Frobenius error): 1e-4 for fp32 activations, 2e-2 where
GEMM operands are rounded to bf16, 1e-5 for the scalar kernels (K1).
Bit-exact: carried-state composition, head permutation, NULL M0 == zero M0,
run-to-run determinism.
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import dev, device_inputs, host, rel, run_fwd

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2
TOL_COEF = 1e-5


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import test_weight_layers_chunk_b200 as E
    return E


def oracle_fwd(w, x, heads=None):
    return O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                        x["M0"], w.C, d_h=w.d_h, loss=w.loss, return_starts=True, heads=heads)


def _coeffs(E, w, x):
    import torch
    s = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss)
    nc = E.e2ttt_num_chunks(s)
    a = torch.empty((w.B, w.H, w.T), device="cuda")
    b = torch.empty_like(a)
    sc = torch.empty((3, w.B, w.H, nc), device="cuda")
    E.e2ttt_chunk_coeffs(s, dev(x["lr"]), dev(x["mom"]), dev(x["decay"]), a, b, sc)
    torch.cuda.synchronize()
    return host(a), host(b), host(sc)


# ------------------------------------------------------------------ K1
@pytest.mark.parametrize("wi", range(len(gen.WORKLOADS)))
def test_chunk_coeffs_match_oracle(E, wi):
    w = gen.WORKLOADS[wi]
    x = gen.generate(w)
    a, b, sc = _coeffs(E, w, x)
    # all heads and chunks of the small workloads; a sample of chunks otherwise
    rng = np.random.default_rng(wi)
    nc = w.n_chunks
    pairs = [(bh, c) for bh in range(w.B * w.H) for c in range(nc)]
    if len(pairs) > 24:
        pairs = [pairs[i] for i in rng.choice(len(pairs), 24, replace=False)]
    for bh, c in pairs:
        bb, hh = divmod(bh, w.H)
        t0, t1 = c * w.C, min(w.T, (c + 1) * w.C)
        ra, rb, pu, pl, cc = O.chunk_kernels(x["lr"][bb, hh, t0:t1], x["mom"][bb, hh, t0:t1],
                                             x["decay"][bb, hh, t0:t1])
        assert rel(a[bb, hh, t0:t1], ra) < TOL_COEF
        assert rel(b[bb, hh, t0:t1], rb) < TOL_COEF
        for i, ref in enumerate((pu, pl, cc)):
            assert abs(sc[i, bb, hh, c] - ref) <= TOL_COEF * abs(ref) + 1e-30, (i, ref, sc[i, bb, hh, c])


@pytest.mark.parametrize("C", [128, 256, 512, 1024])
@pytest.mark.parametrize("mode", ["per_token", "chunk_mean", "no_momentum"])
def test_chunk_coeffs_vector_path_matches_block_path(E, C, mode):
    """Full chunks of C = 128 x {1, 2, 4, 8} tokens with aligned buffers run the
    vectorised K1 kernel; the same gates in buffers shifted by one float (not
    vector-aligned) run the block kernel. Same arithmetic in the same order:
    the results must agree bit for bit, and match the oracle."""
    import torch
    T = 4 * C
    w = gen.Workload("k1v", gen.LINEAR, gen.F32, 2, 3, 8, 8, 0, T, C, "uniform", 0.9, seed=C)
    x = gen.generate(w)
    coef = E.COEF_CHUNK_MEAN if mode == "chunk_mean" else E.COEF_PER_TOKEN
    mom_mode = E.NO_MOMENTUM if mode == "no_momentum" else E.MOMENTUM
    s = E.make_shape(w.B, w.H, w.T, w.C, 8, 8, 0, E.LINEAR, E.F32, coef=coef, momentum=mom_mode)
    nc = E.e2ttt_num_chunks(s)

    def run(shift):
        bufs = []
        for name in ("lr", "mom", "decay"):
            if name == "mom" and mode == "no_momentum":
                bufs.append(None)
                continue
            t = torch.empty(w.B * w.H * T + shift, device="cuda")
            t[shift:] = dev(x[name]).reshape(-1)
            bufs.append(t[shift:].view(w.B, w.H, T))
        outs = [torch.empty(w.B * w.H * T + shift, device="cuda")[shift:].view(w.B, w.H, T)
                for _ in range(2)]
        sc = torch.empty((3, w.B, w.H, nc), device="cuda")
        E.e2ttt_chunk_coeffs(s, *bufs, outs[0], outs[1], sc)
        torch.cuda.synchronize()
        return outs[0], outs[1], sc

    va, vb, vs = run(0)
    ba, bb, bs = run(1)
    assert torch.equal(va, ba) and torch.equal(vb, bb) and torch.equal(vs, bs)
    mom = np.zeros_like(x["mom"]) if mode == "no_momentum" else x["mom"]
    kern = O.chunk_mean_kernels if mode == "chunk_mean" else O.chunk_kernels
    a, b = host(va), host(vb)
    for bh in range(w.B * w.H):
        bi, hi = divmod(bh, w.H)
        for c in range(nc):
            sl = slice(c * C, (c + 1) * C)
            ra, rb, pu, pl, cc = kern(x["lr"][bi, hi, sl], mom[bi, hi, sl], x["decay"][bi, hi, sl])
            assert rel(a[bi, hi, sl], ra) < TOL_COEF and rel(b[bi, hi, sl], rb) < TOL_COEF


@pytest.mark.parametrize("C", [128, 512, 1024])
@pytest.mark.parametrize("mode", ["per_token", "chunk_mean"])
def test_chunk_coeffs_vector_path_walks_several_chunks_per_block(E, C, mode):
    """More (head, chunk) pairs than one resident wave of the vectorised K1
    kernel holds (4096 pairs; at most 148 SMs x 16 blocks resident), so each
    block scans several pairs, loading the next pair's gates during the current
    scan. Bit-identical to the block kernel on every pair, and the oracle on a
    sample that includes the first and last pairs."""
    import torch
    B, H, nc = 16, 16, 16
    T = nc * C
    w = gen.Workload("k1w", gen.LINEAR, gen.F32, B, H, 1, 1, 0, T, C, "uniform", 0.9, seed=C + 1)
    x = gen.generate(w)
    coef = E.COEF_CHUNK_MEAN if mode == "chunk_mean" else E.COEF_PER_TOKEN
    s = E.make_shape(B, H, T, C, 1, 1, 0, E.LINEAR, E.F32, coef=coef)

    def run(shift):
        bufs = []
        for name in ("lr", "mom", "decay"):
            t = torch.empty(B * H * T + shift, device="cuda")
            t[shift:] = dev(x[name]).reshape(-1)
            bufs.append(t[shift:].view(B, H, T))
        outs = [torch.empty(B * H * T + shift, device="cuda")[shift:].view(B, H, T) for _ in range(2)]
        sc = torch.empty((3, B, H, nc), device="cuda")
        E.e2ttt_chunk_coeffs(s, *bufs, outs[0], outs[1], sc)
        torch.cuda.synchronize()
        return outs[0], outs[1], sc

    va, vb, vs = run(0)
    ba, bb, bs = run(1)
    assert torch.equal(va, ba) and torch.equal(vb, bb) and torch.equal(vs, bs)
    kern = O.chunk_mean_kernels if mode == "chunk_mean" else O.chunk_kernels
    a, b, sc = host(va), host(vb), host(vs)
    rng = np.random.default_rng(C)
    pairs = [0, B * H * nc - 1] + list(rng.choice(B * H * nc, 10, replace=False))
    for p in pairs:
        bh, c = divmod(int(p), nc)
        bi, hi = divmod(bh, H)
        sl = slice(c * C, (c + 1) * C)
        ra, rb, pu, pl, cc = kern(x["lr"][bi, hi, sl], x["mom"][bi, hi, sl], x["decay"][bi, hi, sl])
        assert rel(a[bi, hi, sl], ra) < TOL_COEF and rel(b[bi, hi, sl], rb) < TOL_COEF, (p,)
        for i, ref in enumerate((pu, pl, cc)):
            assert abs(sc[i, bi, hi, c] - ref) <= TOL_COEF * abs(ref) + 1e-30, (p, i)


@pytest.mark.parametrize("edge", ["mu0", "lam1", "lam0", "ragged", "C1", "C1024"])
def test_chunk_coeffs_edges(E, edge):
    T, C = 300, 64
    if edge == "C1":
        C = 1
    if edge == "C1024":
        T, C = 2500, 1024
    if edge == "ragged":
        T = 301
    w = gen.Workload("e", gen.LINEAR, gen.F32, 1, 3, 8, 8, 0, T, C, "uniform", 0.9, seed=7)
    x = gen.generate(w)
    if edge == "mu0":
        x["mom"][..., ::3] = 0.0
    if edge == "lam1":
        x["decay"][:] = 1.0
    if edge == "lam0":
        x["decay"][..., 5::7] = 0.0
    a, b, sc = _coeffs(E, w, x)
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b)) and np.all(np.isfinite(sc))
    ra, rb, pu, pl, cc = O.all_chunk_kernels(x["lr"], x["mom"], x["decay"], C)
    assert rel(a, ra) < TOL_COEF and rel(b, rb) < TOL_COEF
    assert rel(sc[0], pu) < TOL_COEF and rel(sc[1], pl) < TOL_COEF and rel(sc[2], cc) < TOL_COEF


# ------------------------------------------------------------------ fp32 CUDA-core path
F32_CASES = {
    "tiny_linear": gen.WORKLOADS[0],
    "tiny_linear_m0": gen.WORKLOADS[0],
    "linear_ragged": gen.Workload("lr", gen.LINEAR, gen.F32, 2, 3, 40, 24, 0, 203, 48, "uniform",
                                  0.99, seed=11),
    "gelu_f32": gen.Workload("gf", gen.GELU, gen.F32, 2, 2, 24, 20, 40, 100, 32, "uniform", 0.99,
                             seed=14, lr_lo=0.005, lr_hi=0.05),
    "swiglu_f32": gen.Workload("sf", gen.SWIGLU, gen.F32, 2, 2, 24, 20, 40, 100, 32, "uniform",
                               0.99, seed=12, lr_lo=0.002, lr_hi=0.02, mom_lo=0.7, mom_hi=0.95),
    "swiglu_f32_dot": gen.Workload("sd", gen.SWIGLU, gen.F32, 1, 2, 16, 16, 32, 96, 32, "uniform",
                                   0.99, seed=13, loss=gen.LOSS_NEG_DOT, lr_lo=0.0005, lr_hi=0.005,
                                   mom_lo=0.5, mom_hi=0.9),
}


@pytest.mark.parametrize("name", list(F32_CASES))
def test_fwd_f32_matches_oracle(E, name):
    w = F32_CASES[name]
    x = gen.generate(w, m0_scale=0.0 if name == "tiny_linear" else 0.5)
    d = device_inputs(w, x)
    out, W_end, M_end, saved = run_fwd(E, w, d, save=True)
    ro, rW, rM, starts = oracle_fwd(w, x)
    assert rel(host(out), ro) < TOL_F32
    assert rel(host(W_end), rW) < TOL_F32
    assert rel(host(M_end), rM) < TOL_F32
    s = host(saved)
    for c in range(w.n_chunks):
        assert rel(s[c, :, :, 0], starts[c, :, :, 0]) < TOL_F32
        assert rel(s[c, :, :, 1], starts[c, :, :, 1]) < TOL_F32 or np.linalg.norm(starts[c, :, :, 1]) == 0


def test_fwd_bf16_untiled_shape_matches_oracle(E):
    """bf16 activations on a shape the tensor-core path does not tile."""
    w = gen.Workload("bu", gen.SWIGLU, gen.BF16, 1, 3, 48, 40, 72, 150, 64, "uniform", 0.99, seed=14,
                     lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    out, W_end, M_end, _ = run_fwd(E, w, device_inputs(w, x))
    ro, rW, rM, _ = oracle_fwd(w, x)
    assert rel(host(out), ro) < TOL_BF16
    assert rel(host(W_end), rW) < TOL_BF16
    assert rel(host(M_end), rM) < TOL_BF16


# ------------------------------------------------------------------ bit-exact structure
STRUCT_CASES = {
    "f32": F32_CASES["swiglu_f32"],
    "bf16_tc": gen.Workload("bt", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform",
                            0.999, seed=15, lr_lo=0.002, lr_hi=0.02),
}


@pytest.mark.parametrize("name", list(STRUCT_CASES))
def test_resume_composes_bitexact(E, name):
    """fwd(T1) then fwd(T2) from its end state == fwd(T1 + T2) (T1 a multiple of C)."""
    import torch
    w = STRUCT_CASES[name]
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    out, W_end, M_end, _ = run_fwd(E, w, d)
    T1 = (w.T // w.C // 2) * w.C
    w1, w2 = w.replace(T=T1), w.replace(T=w.T - T1)
    d1 = {n: (t[:, :, :T1].contiguous() if t is not None and t.dim() >= 3 and t.shape[2] == w.T else t)
          for n, t in d.items()}
    d2 = {n: (t[:, :, T1:].contiguous() if t is not None and t.dim() >= 3 and t.shape[2] == w.T else t)
          for n, t in d.items()}
    o1, W1, M1, _ = run_fwd(E, w1, d1)
    d2["W0"], d2["M0"] = W1, M1
    o2, W2, M2, _ = run_fwd(E, w2, d2)
    assert torch.equal(torch.cat([o1, o2], dim=2), out)
    assert torch.equal(W2, W_end) and torch.equal(M2, M_end)


@pytest.mark.parametrize("name", list(STRUCT_CASES))
def test_head_permutation_bitexact(E, name):
    import torch
    w = STRUCT_CASES[name]
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    out, W_end, M_end, _ = run_fwd(E, w, d)
    perm = torch.arange(w.H - 1, -1, -1, device="cuda")
    dp = {n: (t[:, perm].contiguous() if t is not None else None) for n, t in d.items()}
    op, Wp, Mp, _ = run_fwd(E, w, dp)
    assert torch.equal(op, out[:, perm]) and torch.equal(Wp, W_end[:, perm]) and torch.equal(Mp, M_end[:, perm])


@pytest.mark.parametrize("name", list(STRUCT_CASES))
def test_null_m0_and_determinism(E, name):
    import torch
    w = STRUCT_CASES[name]
    x = gen.generate(w)  # M0 = 0
    d = device_inputs(w, x)
    a = run_fwd(E, w, d, save=True)
    b = run_fwd(E, w, device_inputs(w, x, zero_m0_as_none=True), save=True)
    c = run_fwd(E, w, d, save=True)
    for i in range(4):
        assert torch.equal(a[i], b[i]) and torch.equal(a[i], c[i])
