"""Saved activations (shape.save_acts): the tensor-core forward keeps every
chunk's E (the key rows' residual) and dH (the inner loss's hidden gradient)
in saved_states, in place of its per-call scratch, and the backward reads them
instead of recomputing them (no R2, no R3).

The forward's arithmetic is the same in both modes (only the addresses of E and
dH change), so out, W_end, M_end and the chunk-start states must be equal bit
for bit. The backward then uses the forward's own E and dH, formed from the
bf16 SwiGLU / GELU factors the forward wrote, where the recomputing backward
forms dH from bf16 h1, h3 in fp32: the gradients of the two modes agree to
bf16 rounding, and both meet the oracle at the bf16 tolerance (2e-2, tensor
level, the oracle recomputing sampled heads from the inputs).
"""

import numpy as np
import pytest

import e2ttt_inputs as gen
import oracle as O
from gpu_util import dev, device_inputs, host

pytestmark = pytest.mark.gpu
NAMES = ("dq", "dk", "dv", "dlr", "dmom", "ddecay", "dW0", "dM0")
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
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30 * np.sqrt(ref.size)))


CASES = {
    # the 1.3B training layer with upstream state gradients and M0 != 0
    "train_1p3b_2k_upstream": (gen.state_preserving(gen.BY_NAME["train_1p3b_2k"]), 0.5, True,
                               [(0, 0), (3, 7)]),
    # the GELU MLP at the 1.3B shapes
    "gelu_1p3b_2k": (gen.state_preserving(gen.BY_NAME["layer_1p3b_2k_gelu"]), 0.0, False,
                     [(0, 0), (3, 7)]),
    # a shorter last chunk (88 of 256 tokens) and the -dot loss
    "swiglu_tail": (gen.Workload("sa_tail", gen.SWIGLU, gen.BF16, 2, 2, 128, 128, 256, 600, 256,
                                 "uniform", 0.999, seed=81, lr_lo=0.002, lr_hi=0.02), 0.5, True, None),
    "gelu_dot": (gen.Workload("sa_dot", gen.GELU, gen.BF16, 1, 3, 128, 128, 256, 512, 128,
                              "uniform", 0.999, seed=82, lr_lo=0.002, lr_hi=0.02,
                              loss=gen.LOSS_NEG_DOT), 0.5, False, None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_saved_activations(E, name):
    import torch
    w, m0, upstream, heads = CASES[name]
    x = gen.generate(w, m0_scale=m0)
    dW, dM = gen.upstream_state_grads(w, seed=9, scale=0.1) if upstream else (None, None)
    d = device_inputs(w, x)
    kw = dict(C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss)
    fwd_args = (d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], d["W0"], d["M0"])
    res = {}
    for mode in (E.RECOMPUTE_ACTS, E.SAVE_ACTS):
        f = E.chunk_scan_fwd(*fwd_args, save_states=True, save_acts=mode, **kw)
        g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"], f[3], d["dout"],
                             None if dW is None else dev(dW), None if dM is None else dev(dM),
                             save_acts=mode, **kw)
        torch.cuda.synchronize()
        res[mode] = (f, {n: host(t) for n, t in g.items()})
    (fr, gr), (fs, gs) = res[E.RECOMPUTE_ACTS], res[E.SAVE_ACTS]
    for a, b, n in zip(fr, fs, ("out", "W_end", "M_end", "saved")):
        assert torch.equal(a, b), (name, n)
    between = {n: err(gs[n], gr[n]) for n in NAMES}
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, dM, d_h=w.d_h, loss=w.loss, heads=heads)
    if heads is None:
        vs = {n: err(gs[n], ref[n]) for n in NAMES}
    else:
        bi = tuple(np.array(heads).T)
        vs = {n: err(gs[n][bi], ref[n][bi]) for n in NAMES}
    print(f"\n{name}: saved vs recomputed " + " ".join(f"{n}={e:.1e}" for n, e in between.items())
          + "\n  saved vs oracle " + " ".join(f"{n}={e:.1e}" for n, e in vs.items()))
    assert all(e < TOL for e in vs.values()), (name, vs)
    assert all(e < TOL for e in between.values()), (name, between)


def test_saved_activations_no_momentum(E):
    """No momentum (the W-only aggregation reads the saved dH too): forward
    outputs equal bit for bit across the two modes, gradients against the oracle
    at mu = 0 and against the recomputing backward."""
    import torch
    w = gen.Workload("sa_nm", gen.SWIGLU, gen.BF16, 2, 2, 128, 128, 256, 512, 128, "uniform", 0.999,
                     seed=83, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w)
    x["mom"] = np.zeros_like(x["mom"])
    x["M0"] = np.zeros_like(x["M0"])
    d = device_inputs(w, x)
    dW, _ = gen.upstream_state_grads(w, seed=10, scale=0.1)
    kw = dict(C=w.C, d_h=w.d_h, kind=w.kind, loss=w.loss, momentum=E.NO_MOMENTUM)
    res = {}
    for mode in (E.RECOMPUTE_ACTS, E.SAVE_ACTS):
        f = E.chunk_scan_fwd(d["q"], d["k"], d["v"], d["lr"], None, d["decay"], d["W0"], None,
                             save_states=True, save_acts=mode, **kw)
        g = E.chunk_scan_bwd(d["q"], d["k"], d["v"], d["lr"], None, d["decay"], f[3], d["dout"],
                             dev(dW), None, save_acts=mode, **kw)
        torch.cuda.synchronize()
        res[mode] = (f, {n: host(t) for n, t in g.items() if t is not None})
    (fr, gr), (fs, gs) = res[E.RECOMPUTE_ACTS], res[E.SAVE_ACTS]
    for a, b, n in zip((fr[0], fr[1], fr[3]), (fs[0], fs[1], fs[3]), ("out", "W_end", "saved")):
        assert torch.equal(a, b), n
    names = ("dq", "dk", "dv", "dlr", "ddecay", "dW0")
    ref = O.closed_bwd(w.kind, x["q"], x["k"], x["v"], x["lr"], x["mom"], x["decay"], x["W0"],
                       x["M0"], w.C, x["dout"], dW, None, d_h=w.d_h, loss=w.loss)
    vs = {n: err(gs[n], ref[n]) for n in names}
    between = {n: err(gs[n], gr[n]) for n in names}
    print("\nno momentum: saved vs oracle", vs, "saved vs recomputed", between)
    assert all(e < TOL for e in vs.values()), vs
    assert all(e < TOL for e in between.values()), between
