"""GPU parity of the variants in combination, on the tensor-core path (bf16):
fast weight (SwiGLU, GELU MLP, linear) x coefficients (per token, chunk means)
x momentum (with, without) x a shorter last chunk, forward and backward,
against the fp64 oracle (closed form; mu = 0 and M0 = 0 stand for no momentum).

Forward and backward are compared end to end with the oracle computed from the
inputs alone; inputs have M0 = 0, where the GELU MLP's gradients are
well-conditioned under the bf16 rounding of the GEMM operands. Tolerance 2e-2
relative Frobenius, as for every bf16 case.
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import dev, device_inputs, host, rel

pytestmark = pytest.mark.gpu
TOL = 2e-2
MEAN = O.COEF_CHUNK_MEAN


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


# name: (kind, d_h, T, C, coef, momentum)
CASES = {
    "gelu_no_momentum": (gen.GELU, 256, 512, 128, 0, False),
    "gelu_chunk_mean": (gen.GELU, 256, 512, 128, 1, True),
    "gelu_no_momentum_tail": (gen.GELU, 256, 300, 128, 0, False),
    "swiglu_chunk_mean_tail": (gen.SWIGLU, 256, 600, 256, 1, True),
    "swiglu_no_momentum_chunk_mean": (gen.SWIGLU, 256, 512, 128, 1, False),
    "linear_no_momentum_tail": (gen.LINEAR, 0, 640, 512, 0, False),
}


def _setup(E, name):
    kind, d_h, T, C, coef, mom = CASES[name]
    w = gen.Workload("combo", kind, gen.BF16, 2, 2, 128, 128, d_h, T, C, "uniform", 0.999,
                     seed=81 + T + 7 * coef, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.0)
    if not mom:
        x["mom"] = np.zeros_like(x["mom"])
    shape = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss, coef=coef,
                         momentum=E.MOMENTUM if mom else E.NO_MOMENTUM)
    assert E.e2ttt_fwd_uses_tensor_cores(shape) == 1
    return w, x, coef, mom


@pytest.mark.parametrize("name", list(CASES))
def test_combination_forward_and_backward(E, name):
    import torch
    w, x, coef, mom = _setup(E, name)
    d = device_inputs(w, x)
    momentum = E.MOMENTUM if mom else E.NO_MOMENTUM
    out, W_end, M_end, saved = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], d["mom"] if mom else None,
                                                d["decay"], d["W0"], None, C=w.C, d_h=w.d_h,
                                                kind=w.kind, loss=w.loss, coef=coef, momentum=momentum,
                                                save_states=True)
    dW, dM = gen.upstream_state_grads(w, seed=14, scale=0.1)
    g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], d["mom"] if mom else None, d["decay"], saved,
                         d["dout"], dev(dW), dev(dM) if mom else None, C=w.C, d_h=w.d_h, kind=w.kind,
                         loss=w.loss, coef=coef, momentum=momentum)
    torch.cuda.synchronize()
    ro, rW, rM = O.closed_fwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                              x["M0"], w.C, d_h=w.d_h, loss=w.loss, coef=coef)
    errs = {"out": rel(host(out), ro), "W_end": rel(host(W_end), rW)}
    if mom:
        errs["M_end"] = rel(host(M_end), rM)
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, dM if mom else None, d_h=w.d_h, loss=w.loss,
                       coef=coef)
    names = ("dq", "dk", "dv", "dlr", "ddecay", "dW0") + (("dmom", "dM0") if mom else ())
    errs.update({n: rel(host(g[n]), ref[n]) for n in names})
    print(f"\n{name}: " + " ".join(f"{k}={v:.2e}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if not v < TOL}
    assert not bad, (name, bad)
