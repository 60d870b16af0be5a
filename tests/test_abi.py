"""The C ABI without a GPU: the library loads, exports every function the header
declares, and rejects bad arguments on the host (no launch, nothing written)."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "test_weight_layers_chunk_b200", "libe2ttt.so")


@pytest.fixture(scope="module")
def E():
    if not os.path.exists(LIB):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "_e2ttt_build", os.path.join(ROOT, "test_weight_layers_chunk_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    import test_weight_layers_chunk_b200 as E
    return E


def test_exports_every_declared_symbol(E):
    names = E.header_functions()
    assert set(names) >= {"e2ttt_chunk_scan_fwd", "e2ttt_chunk_scan_bwd", "e2ttt_chunk_coeffs",
                          "e2ttt_workspace_bytes", "e2ttt_state_elems", "e2ttt_status_string",
                          "e2ttt_last_error", "e2ttt_num_chunks"}
    lib = ctypes.CDLL(LIB)
    for n in names:
        assert hasattr(lib, n), n


def test_sizes(E):
    s = E.make_shape(4, 8, 2048, 512, 256, 256, 512, E.SWIGLU, E.BF16)
    assert E.e2ttt_state_elems(s) == 2 * 512 * 256 + 256 * 512
    assert E.e2ttt_num_chunks(s) == 4
    assert E.e2ttt_workspace_bytes(s, 0) > 0
    lin = E.make_shape(1, 1, 256, 64, 32, 32, 0, E.LINEAR, E.F32)
    assert E.e2ttt_state_elems(lin) == 32 * 32
    assert E.e2ttt_num_chunks(E.make_shape(1, 1, 257, 64, 32, 32, 0, E.LINEAR, E.F32)) == 5
    for bad in (E.make_shape(0, 1, 8, 4, 4, 4, 4), E.make_shape(1, 1, 8, 2048, 4, 4, 4),
                E.make_shape(1, 1, 8, 4, 4, 4, 0, E.SWIGLU), E.make_shape(1, 1, 8, 4, 4, 4, 4, 7),
                E.make_shape(1, 1, 8, 4, 4, 4, 4, E.SWIGLU, coef=2)):
        assert E.e2ttt_state_elems(bad) == 0 and E.e2ttt_workspace_bytes(bad, 0) == 0


def test_status_strings(E):
    for s in range(5):
        assert E.e2ttt_status_string(s).startswith("E2TTT_")


FAKE = 1 << 40  # never dereferenced: every call below fails its host-side checks


def _fwd(E, shape, **over):
    S = max(E.e2ttt_state_elems(shape), 1)
    n = 1 << 30
    args = dict(q=FAKE, k=FAKE + n, v=FAKE + 2 * n, lr=FAKE + 3 * n, mom=FAKE + 4 * n,
                decay=FAKE + 5 * n, W0=FAKE + 6 * n, M0=FAKE + 7 * n, out=FAKE + 8 * n,
                W_end=FAKE + 9 * n, M_end=FAKE + 10 * n, saved_states=None, workspace=FAKE + 12 * n,
                workspace_bytes=E.e2ttt_workspace_bytes(shape, 0))
    args.update(over)
    return E.e2ttt_chunk_scan_fwd(shape, raw=True, stream=None, **args)


def test_fwd_rejects_bad_arguments(E):
    s = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32)
    for over in (dict(q=None), dict(W0=None), dict(out=None), dict(workspace=None),
                 dict(workspace_bytes=16), dict(workspace=FAKE + 12 * (1 << 30) + 8),
                 dict(out=FAKE + 7),                       # out overlaps q
                 dict(W_end=FAKE + 6 * (1 << 30)),         # W_end aliases W0
                 dict(M_end=FAKE + 9 * (1 << 30) + 4)):    # M_end overlaps W_end
        assert _fwd(E, s, **over) == E.ERR_INVALID_ARG, over
        assert E.e2ttt_last_error() != ""
    bad = E.make_shape(1, 2, 64, 0, 8, 8, 16, E.SWIGLU, E.F32)
    assert _fwd(E, bad) == E.ERR_INVALID_ARG
    assert "sizes" in E.e2ttt_last_error()


def test_bwd_rejects_bad_arguments(E):
    s = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32)
    n = 1 << 30
    args = dict(q=FAKE, k=FAKE + n, v=FAKE + 2 * n, lr=FAKE + 3 * n, mom=FAKE + 4 * n,
                decay=FAKE + 5 * n, saved_states=FAKE + 6 * n, dout=FAKE + 7 * n, dW_end=None,
                dM_end=None, dq=FAKE + 8 * n, dk=FAKE + 9 * n, dv=FAKE + 10 * n, dlr=FAKE + 11 * n,
                dmom=FAKE + 12 * n, ddecay=FAKE + 13 * n, dW0=FAKE + 14 * n, dM0=FAKE + 15 * n,
                workspace=FAKE + 16 * n, workspace_bytes=E.e2ttt_workspace_bytes(s, 1))
    for over in (dict(saved_states=None), dict(dq=None), dict(workspace_bytes=0),
                 dict(dk=FAKE + 8 * n + 2)):
        a = dict(args)
        a.update(over)
        assert E.e2ttt_chunk_scan_bwd(s, raw=True, stream=None, **a) == E.ERR_INVALID_ARG, over


def test_coeffs_rejects_bad_arguments(E):
    s = E.make_shape(1, 1, 64, 16, 8, 8, 0, E.LINEAR, E.F32)
    assert E.e2ttt_chunk_coeffs(s, None, FAKE, FAKE, FAKE, FAKE, FAKE, raw=True) == E.ERR_INVALID_ARG
    assert E.e2ttt_chunk_coeffs(s, FAKE, FAKE + 4096, FAKE + 8192, FAKE, FAKE + (1 << 20),
                                FAKE + (1 << 21), raw=True) == E.ERR_INVALID_ARG  # a aliases lr


def test_no_momentum_pointer_rules(E):
    """No-momentum mode (E2TTT_NO_MOMENTUM): mom, M0, M_end (forward) and mom, dM_end,
    dmom, dM0 (backward) must be NULL; with momentum, mom and M_end are required.
    All checks run on the host before any CUDA call."""
    nm = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32, momentum=E.NO_MOMENTUM)
    ws = E.e2ttt_workspace_bytes(nm, 0)
    assert ws > E.e2ttt_workspace_bytes(E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32), 0)
    for over in (dict(), dict(M0=None), dict(M0=None, M_end=None)):     # mom given
        assert _fwd(E, nm, workspace_bytes=ws, **over) == E.ERR_INVALID_ARG, over
        assert "no-momentum" in E.e2ttt_last_error()
    s = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32)
    assert _fwd(E, s, mom=None) == E.ERR_INVALID_ARG
    assert _fwd(E, s, M_end=None) == E.ERR_INVALID_ARG
    n = 1 << 30
    args = dict(q=FAKE, k=FAKE + n, v=FAKE + 2 * n, lr=FAKE + 3 * n, mom=None,
                decay=FAKE + 5 * n, saved_states=FAKE + 6 * n, dout=FAKE + 7 * n, dW_end=None,
                dM_end=None, dq=FAKE + 8 * n, dk=FAKE + 9 * n, dv=FAKE + 10 * n, dlr=FAKE + 11 * n,
                dmom=None, ddecay=FAKE + 13 * n, dW0=FAKE + 14 * n, dM0=None,
                workspace=FAKE + 16 * n, workspace_bytes=E.e2ttt_workspace_bytes(nm, 1))
    for over in (dict(mom=FAKE + 4 * n), dict(dmom=FAKE + 12 * n), dict(dM0=FAKE + 15 * n),
                 dict(dM_end=FAKE + 15 * n)):
        a = dict(args)
        a.update(over)
        assert E.e2ttt_chunk_scan_bwd(nm, raw=True, stream=None, **a) == E.ERR_INVALID_ARG, over
    assert E.e2ttt_chunk_coeffs(nm, FAKE, FAKE + n, FAKE + 2 * n, FAKE + 3 * n, FAKE + 4 * n,
                                FAKE + 5 * n, raw=True) == E.ERR_INVALID_ARG   # mom given
    bad = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32, momentum=3)
    assert E.e2ttt_state_elems(bad) == 0


def test_gelu_mlp_state_size(E):
    g = E.make_shape(1, 2, 64, 16, 8, 6, 16, E.GELU_MLP, E.F32)
    assert E.e2ttt_state_elems(g) == 16 * 8 + 6 * 16
    assert E.e2ttt_workspace_bytes(g, 0) > 0 and E.e2ttt_workspace_bytes(g, 1) > 0


def test_gemm_precision_field(E):
    """The shape's gemm field: GEMM_AUTO (zero) picks the tensor cores for a
    tensor-core shape, GEMM_FP32 always the fp32 CUDA-core kernels (with their
    smaller workspace), other values are rejected on the host."""
    import ctypes
    assert [n for n, _ in E.e2ttt_shape._fields_][-2:] == ["gemm", "save_acts"]
    assert ctypes.sizeof(E.e2ttt_shape) == 14 * ctypes.sizeof(ctypes.c_int)
    auto = E.make_shape(1, 2, 512, 128, 128, 128, 256, E.GELU_MLP, E.BF16)
    fp32 = E.make_shape(1, 2, 512, 128, 128, 128, 256, E.GELU_MLP, E.BF16, gemm=E.GEMM_FP32)
    assert auto.gemm == E.GEMM_AUTO == 0
    assert E.e2ttt_fwd_uses_tensor_cores(auto) in (0, 1)  # 1 where a GPU driver is present
    assert E.e2ttt_fwd_uses_tensor_cores(fp32) == 0
    for fb in (0, 1):
        assert 0 < E.e2ttt_workspace_bytes(fp32, fb)
    bad = E.make_shape(1, 2, 512, 128, 128, 128, 256, E.GELU_MLP, E.BF16, gemm=2)
    assert E.e2ttt_fwd_uses_tensor_cores(bad) == -1
    assert E.e2ttt_workspace_bytes(bad, 0) == 0


def test_noalloc_status_without_a_device(E):
    """The no-allocation status readout needs a current device: with none (this
    CPU-only host) it returns E2TTT_ERR_CUDA with a message, never crashes."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the readout is covered by the GPU test")
    st = E.e2ttt_noalloc_status(raw=True, stream=None)
    assert st == E.ERR_CUDA
    assert "e2ttt_noalloc_status" in E.e2ttt_last_error()


def test_save_acts_field(E):
    """save_acts: the saved-states size grows by the per-chunk bf16 E ([NC, B, H,
    C, d_v]) and dH ([NC, B, H, C, 2 d_h] for SwiGLU, d_h for the GELU MLP),
    each region 256-byte aligned; the linear fast weight saves no activations;
    other values are rejected; the forward refuses save_acts on the host where
    it cannot keep them (no saved_states, the linear fast weight, fp32
    activations)."""
    up = lambda x: (x + 255) // 256 * 256
    for kind, nf in ((E.SWIGLU, 2), (E.GELU_MLP, 1)):
        B, H, T, C, dk, dv, dh = 2, 3, 1000, 256, 128, 128, 256
        base = E.make_shape(B, H, T, C, dk, dv, dh, kind, E.BF16)
        acts = E.make_shape(B, H, T, C, dk, dv, dh, kind, E.BF16, save_acts=E.SAVE_ACTS)
        nc, S = E.e2ttt_num_chunks(base), E.e2ttt_state_elems(base)
        states = nc * B * H * 2 * S * 4
        assert E.e2ttt_saved_bytes(base) == states
        e_off = up(states)
        dh_off = up(e_off + nc * B * H * C * dv * 2)
        assert E.e2ttt_saved_bytes(acts) == dh_off + nc * B * H * C * nf * dh * 2
    lin = E.make_shape(1, 2, 64, 16, 8, 8, 0, E.LINEAR, E.F32, save_acts=E.SAVE_ACTS)
    assert E.e2ttt_saved_bytes(lin) == E.e2ttt_num_chunks(lin) * 2 * 2 * E.e2ttt_state_elems(lin) * 4
    bad = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32, save_acts=2)
    assert E.e2ttt_saved_bytes(bad) == 0
    f32 = E.make_shape(1, 2, 64, 16, 8, 8, 16, E.SWIGLU, E.F32, save_acts=E.SAVE_ACTS)
    assert _fwd(E, f32) == E.ERR_INVALID_ARG                  # no saved_states
    assert "saved_states" in E.e2ttt_last_error()
    assert _fwd(E, f32, saved_states=FAKE + 11 * (1 << 30)) == E.ERR_UNSUPPORTED  # fp32: CUDA cores
    assert "tensor-core" in E.e2ttt_last_error()
    assert _fwd(E, lin, saved_states=FAKE + 11 * (1 << 30)) == E.ERR_UNSUPPORTED
