"""Failure detection on the GPU without a fault: a device-side bounded wait that
runs out.

Every mbarrier wait of the tensor-core kernels is bounded. The test hook
e2ttt_test_stall_next_forward makes one CTA of the next forward's first GEMM
launch wait on an mbarrier that nothing completes, with that launch's waits
limited to 1 ms: the wait gives up, the CTA drains its own copies in flight,
frees its tensor memory and exits, and the workspace status word reports
E2TTT_ERR_TIMEOUT. No memory access is changed and nothing traps. A normal call
on the same stream afterwards must succeed and give the same results bit for
bit as one made before the stalled call.
"""
import pytest

import e2ttt_inputs as gen
from gpu_util import device_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    import torch
    assert torch.cuda.is_available()
    import test_weight_layers_chunk_b200 as E
    return E


@pytest.mark.parametrize("driver", ["phases", "persistent", "pairs"])
def test_bounded_wait_runs_out_and_the_context_recovers(E, driver, monkeypatch):
    """Three forward drivers: the per-phase launches; the persistent kernel
    (E2TTT_PERSISTENT=1, one launch for all chunks), where the stalled CTA's
    tiles never complete and every CTA waiting on them gives up too; and the
    CTA-pair launches (E2TTT_PAIRS=1, at the 1.3B layer's shapes where they
    apply), where the even CTA of the first pair stalls before its MMAs, its
    partner's producer and both CTAs' epilogues give up, and the pair meets at
    its cluster barrier before freeing tensor memory."""
    import torch
    monkeypatch.setenv("E2TTT_PERSISTENT", "1" if driver == "persistent" else "0")
    monkeypatch.setenv("E2TTT_PAIRS", "1" if driver == "pairs" else "0")
    saved = False
    if driver == "pairs":
        w = gen.BY_NAME["layer_1p3b_2k"]
    else:
        w = gen.Workload("stall", gen.SWIGLU, gen.BF16, 1, 2, 128, 128, 256, 512, 128, "uniform",
                         0.999, seed=61, lr_lo=0.002, lr_hi=0.02)
    x = gen.generate(w, m0_scale=0.5)
    d = device_inputs(w, x)
    shape = E.make_shape(w.B, w.H, w.T, w.C, w.d_k, w.d_v, w.d_h, w.kind, w.act, w.loss)
    assert E.e2ttt_fwd_uses_tensor_cores(shape) == 1
    ws = E.workspace(shape)

    nc = E.e2ttt_num_chunks(shape)
    sv = torch.empty((nc, w.B, w.H, 2, w.state_elems), device="cuda") if saved else None

    def call():
        out = torch.empty_like(d["v"])
        We, Me = torch.empty_like(d["W0"]), torch.empty_like(d["W0"])
        E.e2ttt_chunk_scan_fwd(shape, d["q"], d["k"], d["v"], d["lr"], d["mom"], d["decay"],
                               d["W0"], d["M0"], out, We, Me, sv, ws)
        return out, We, Me

    before = call()
    assert E.e2ttt_workspace_status(ws, raw=True) == E.OK

    E.e2ttt_test_stall_next_forward(True)
    call()
    st = E.e2ttt_workspace_status(ws, raw=True)
    assert st == E.ERR_TIMEOUT, (st, E.e2ttt_last_error())
    assert "gave up" in E.e2ttt_last_error()

    after = call()   # the hook disarmed itself; the context is usable
    assert E.e2ttt_workspace_status(ws, raw=True) == E.OK
    torch.cuda.synchronize()
    for a, b in zip(before, after):
        assert torch.equal(a, b)
