"""GPU parity of the no-momentum mode (momentum = E2TTT_NO_MOMENTUM) against the
fp64 oracle with mu = 0 and M0 = 0.

Without momentum the recurrence is W_t = lam_t W_{t-1} - eta_t g_t; the momentum
state never feeds W, so the library keeps none: mom, M0, M_end are NULL and the
tensor-core forward aggregates only the b-weighted gradients and moves only W.
The oracle runs its general closed form with mu = 0 (pinned on the CPU:
closed form = per-token loop with mu = 0; mu = 0, lam = 1 = plain chunk update).
Tolerances: 1e-4 relative Frobenius (fp32), 2e-2 (bf16).
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import dev, device_inputs, host, rel

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dlr", "ddecay", "dW0")


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


CASES = {
    "linear_f32": gen.Workload("nml", gen.LINEAR, gen.F32, 1, 2, 24, 16, 0, 70, 32, "uniform", 0.99,
                               seed=51),
    "swiglu_f32": gen.Workload("nms", gen.SWIGLU, gen.F32, 1, 2, 16, 12, 24, 50, 16, "uniform", 0.99,
                               seed=53, lr_lo=0.002, lr_hi=0.02),
    # full chunks of 128 tokens: the block-per-chunk K1 adjoint with no momentum
    "linear_f32_c128": gen.Workload("nmlc", gen.LINEAR, gen.F32, 1, 2, 16, 12, 0, 384, 128,
                                    "uniform", 0.99, seed=67, lr_lo=0.002, lr_hi=0.02),
    "linear_bf16_tc": gen.Workload("nmlb", gen.LINEAR, gen.BF16, 1, 2, 128, 128, 0, 512, 128,
                                   "uniform", 0.999, seed=55, lr_lo=0.002, lr_hi=0.02),
    "swiglu_bf16_tc": gen.Workload("nmsb", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128,
                                   "uniform", 0.999, seed=57, lr_lo=0.002, lr_hi=0.02),
    # a shorter last chunk (T % C != 0) on the tensor cores: 44 real tokens of 128
    "swiglu_bf16_tc_tail": gen.Workload("nmst", gen.SWIGLU, gen.BF16, 2, 2, 128, 128, 256, 300, 128,
                                        "uniform", 0.999, seed=59, lr_lo=0.002, lr_hi=0.02),
}


def _tol(w):
    return 2e-2 if w.act == gen.BF16 else 1e-4


def _inputs(w):
    x = gen.generate(w)
    x["mom"] = np.zeros_like(x["mom"])
    x["M0"] = np.zeros_like(x["M0"])
    return x


@pytest.mark.parametrize("name", list(CASES))
def test_no_momentum_forward(E, name):
    import torch
    w = CASES[name]
    x = _inputs(w)
    d = device_inputs(w, x)
    if w.act == gen.BF16:
        s = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss,
                         momentum=E.NO_MOMENTUM)
        assert E.e2ttt_fwd_uses_tensor_cores(s) == 1
    out, W_end, M_end, saved = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], None, d["decay"],
                                                d["W0"], None, C=w.C, d_h=w.d_h, kind=w.kind,
                                                loss=w.loss, momentum=E.NO_MOMENTUM,
                                                save_states=True)
    torch.cuda.synchronize()
    assert M_end is None
    ro, rW, _, starts = O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"],
                                     x["W0"], x["M0"], w.C, d_h=w.d_h, loss=w.loss,
                                     return_starts=True)
    errs = (rel(host(out), ro), rel(host(W_end), rW), rel(host(saved)[:, :, :, 0], starts[:, :, :, 0]))
    print(f"\n{name}: out={errs[0]:.2e} W_end={errs[1]:.2e} saved W={errs[2]:.2e}")
    assert max(errs) < _tol(w), errs
    if w.act == gen.BF16:   # the tensor-core path stores no momentum: saved M is zero
        assert np.all(host(saved)[:, :, :, 1] == 0.0)


@pytest.mark.parametrize("name", list(CASES))
def test_no_momentum_backward(E, name):
    import torch
    w = CASES[name]
    x = _inputs(w)
    d = device_inputs(w, x)
    _, _, _, saved = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], None, d["decay"], d["W0"],
                                      None, C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss,
                                      momentum=E.NO_MOMENTUM, save_states=True)
    dW, _ = gen.upstream_state_grads(w, seed=9, scale=0.1)
    g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], None, d["decay"], saved, d["dout"],
                         dev(dW), None, C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss,
                         momentum=E.NO_MOMENTUM)
    torch.cuda.synchronize()
    assert g["dmom"] is None and g["dM0"] is None
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, None, d_h=w.d_h, loss=w.loss)
    errs = {n: rel(host(g[n]), ref[n]) for n in NAMES}
    print(f"\n{name}: " + " ".join(f"{n}={e:.2e}" for n, e in errs.items()))
    assert all(e < _tol(w) for e in errs.values()), errs
