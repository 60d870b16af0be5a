"""GPU parity of the chunk-averaged variant (coef = E2TTT_COEF_CHUNK_MEAN) against
the fp64 oracle.

"Rethinking Expressivity and Efficiency in Test-Time Training", atlas.scime.ai
summary, "Surprising findings": a variant with the per-token factors collapsed to
chunk scalars. Every token of a chunk carries the chunk means of the momentum and
weight kernels; the oracle's variant is pinned on the CPU (tests/test_oracle.py).
Tolerances as for the method: 1e-4 relative Frobenius (fp32 activations), 2e-2
(bf16 activations); K1 coefficients 1e-5.
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import dev, device_inputs, host, rel

pytestmark = pytest.mark.gpu
MEAN = O.COEF_CHUNK_MEAN
NAMES = ("dq", "dk", "dv", "dlr", "dmom", "ddecay", "dW0", "dM0")


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


@pytest.mark.parametrize("T,C", [(300, 64), (301, 64), (2500, 1024), (40, 1)])
def test_chunk_mean_coeffs(E, T, C):
    """K1 with chunk means, ragged last chunk, C = 1 and the largest C."""
    import torch
    w = gen.Workload("cm", gen.LINEAR, gen.F32, 1, 2, 8, 8, 0, T, C, "uniform", 0.95, seed=31)
    x = gen.generate(w)
    s = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, 0, w.kind, w.act, w.loss, coef=MEAN)
    nc = E.e2ttt_num_chunks(s)
    a = torch.empty((w.B, w.H, w.T), device="cuda")
    b = torch.empty_like(a)
    sc = torch.empty((3, w.B, w.H, nc), device="cuda")
    E.e2ttt_chunk_coeffs(s, dev(x["lr"]), dev(x["mom"]), dev(x["decay"]), a, b, sc)
    torch.cuda.synchronize()
    ra, rb, pu, pl, cc = O.all_chunk_kernels(x["lr"], x["mom"], x["decay"], C, coef=MEAN)
    assert rel(host(a), ra) < 1e-5 and rel(host(b), rb) < 1e-5
    assert rel(host(sc)[0], pu) < 1e-5 and rel(host(sc)[1], pl) < 1e-5 and rel(host(sc)[2], cc) < 1e-5
    # constant within every chunk
    ha = host(a)
    for t0 in range(0, T, C):
        seg = ha[:, :, t0:t0 + C]
        assert np.all(seg == seg[:, :, :1])


CASES = {
    "linear_f32": gen.Workload("cml", gen.LINEAR, gen.F32, 1, 2, 24, 16, 0, 70, 32, "uniform", 0.99,
                               seed=41),
    "swiglu_f32": gen.Workload("cms", gen.SWIGLU, gen.F32, 1, 2, 16, 12, 24, 50, 16, "uniform", 0.99,
                               seed=43, lr_lo=0.002, lr_hi=0.02, mom_lo=0.7, mom_hi=0.95),
    # full chunks of 256 tokens: the block-per-chunk K1 adjoint with chunk means
    "linear_f32_c256": gen.Workload("cmlc", gen.LINEAR, gen.F32, 1, 2, 16, 12, 0, 512, 256,
                                    "uniform", 0.99, seed=65, lr_lo=0.002, lr_hi=0.02),
    "swiglu_bf16_tc": gen.Workload("cmb", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128,
                                   "uniform", 0.999, seed=45, lr_lo=0.002, lr_hi=0.02),
}


def _tol(w):
    return 2e-2 if w.act == gen.BF16 else 1e-4


@pytest.mark.parametrize("name", list(CASES))
def test_chunk_mean_forward(E, name):
    import torch
    w = CASES[name]
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    out, W_end, M_end, _ = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"],
                                            d["W0"], d["M0"], C=w.C, d_h=w.d_h, kind=w.kind,
                                            loss=w.loss, coef=MEAN)
    torch.cuda.synchronize()
    ro, rW, rM = O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                              x["W0"], x["M0"], w.C, d_h=w.d_h, loss=w.loss, coef=MEAN)
    errs = (rel(host(out), ro), rel(host(W_end), rW), rel(host(M_end), rM))
    print(f"\n{name}: out={errs[0]:.2e} W_end={errs[1]:.2e} M_end={errs[2]:.2e}")
    assert max(errs) < _tol(w), errs
    # the variant is not the method: the per-token result differs
    po, pW, _ = O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                             x["W0"], x["M0"], w.C, d_h=w.d_h, loss=w.loss)
    assert rel(pW, rW) > 10 * _tol(w) or rel(po, ro) > 10 * _tol(w) or w.act == gen.BF16


@pytest.mark.parametrize("name", list(CASES))
def test_chunk_mean_backward(E, name):
    import torch
    w = CASES[name]
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    _, _, _, saved = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"],
                                      d["W0"], d["M0"], C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss,
                                      coef=MEAN, save_states=True)
    dW, dM = gen.upstream_state_grads(w, seed=7, scale=0.1)
    g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], saved, d["dout"],
                         dev(dW), dev(dM), C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss, coef=MEAN)
    torch.cuda.synchronize()
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, dM, d_h=w.d_h, loss=w.loss, coef=MEAN)
    errs = {n: rel(host(g[n]), ref[n]) for n in NAMES}
    print(f"\n{name}: " + " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    assert all(e < _tol(w) for e in errs.values()), errs
