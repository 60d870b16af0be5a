"""The forward entry point for callers that cannot allocate device memory.

e2ttt_chunk_scan_fwd_noalloc takes its scratch from a 32 MiB array owned by
the library instead of a caller workspace; it is meant for callers that cannot
call cudaMalloc (device memory already claimed by their own pool allocator, C
hosts without a device allocator, loops that cannot afford cudaMalloc's
implicit synchronisation). Here it is called through the C ABI and compared
with e2ttt_chunk_scan_fwd on the same inputs, twice in a row (the static array
keeps the previous call's contents). Both run the same deterministic kernels
on the same inputs (no atomics in any reduction), so the outputs must be
identical bit for bit: a second call that read stale scratch from the first
would show up. The status word of the bounded waits, which lives in the static
array, is read back through e2ttt_noalloc_status after each call. This file is
named to be collected last.
"""
import numpy as np
import pytest

import e2ttt_inputs as gen
from gpu_util import device_inputs, host, rel, run_fwd

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_linear_f32": gen.BY_NAME["tiny_linear"],
    "swiglu_bf16_tensor_cores": gen.Workload("na", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512,
                                             128, "uniform", 0.999, seed=31, lr_lo=0.002,
                                             lr_hi=0.02),
}


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_forward_matches_workspace_forward(E, name):
    import torch
    w = CASES[name]
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    ref = run_fwd(E, w, d, save=True)
    shape = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss)
    for call in range(2):
        out = torch.full_like(ref[0], float("nan"))
        W_end = torch.full_like(ref[1], float("nan"))
        M_end = torch.full_like(ref[2], float("nan"))
        saved = torch.full_like(ref[3], float("nan"))
        E.e2ttt_chunk_scan_fwd_noalloc(shape, d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"],
                                       d["W0"], d["M0"], out, W_end, M_end, saved)
        assert E.e2ttt_noalloc_status(raw=True) == E.OK, E.e2ttt_last_error()
        torch.cuda.synchronize()
        for got, want in zip((out, W_end, M_end, saved), ref):
            assert np.all(np.isfinite(host(got))), (name, call)
            assert torch.equal(got, want), (name, call, rel(host(got), host(want)))


def test_noalloc_rejects_shapes_beyond_its_scratch(E):
    w = gen.BY_NAME["layer_1p3b_2k"]
    shape = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss)
    fake = 1 << 40  # never dereferenced: the size check runs first
    st = E.e2ttt_chunk_scan_fwd_noalloc(shape, *[fake + i * (1 << 32) for i in range(11)], None,
                                        raw=True, stream=None)
    assert st == E.ERR_INVALID_ARG
    assert "static scratch" in E.e2ttt_last_error()
