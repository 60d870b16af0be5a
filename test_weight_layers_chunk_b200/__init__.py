"""Python binding of libe2ttt.so, the E2-TTT chunk-parallel closed-form
fast-weight update for NVIDIA B200 (sm_100a).

Method: "Rethinking Expressivity and Efficiency in Test-Time Training"
(E2-TTT): per chunk, gradients of the fast-weight loss at the chunk-start
weights, a momentum kernel and a weight kernel from the lr / momentum / decay
gates, chunk-end states as two weighted gradient aggregations plus decayed
start states, and the chunk output at the chunk-start weights.

The functions named e2ttt_* mirror the C entry points of include/e2ttt.h one to
one: they only marshal arguments (torch tensors or raw device pointers) and
raise E2TTTError on a non-zero status. All computation happens in the CUDA
library; there is no Python or CPU fallback, and importing this package fails
if the library has not been built (python test_weight_layers_chunk_b200/build.py).
chunk_scan_fwd / chunk_scan_bwd are conveniences that allocate the outputs and
the workspace with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libe2ttt.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "e2ttt.h")

LINEAR, SWIGLU, GELU_MLP = 0, 1, 2
F32, BF16 = 0, 1
LOSS_MSE, LOSS_NEG_DOT = 0, 1
COEF_PER_TOKEN, COEF_CHUNK_MEAN = 0, 1
MOMENTUM, NO_MOMENTUM = 0, 1
GEMM_AUTO, GEMM_FP32 = 0, 1
RECOMPUTE_ACTS, SAVE_ACTS = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4


class e2ttt_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("B", "H", "T", "C", "d_k", "d_v", "d_h", "kind", "act", "loss", "coef", "momentum",
                 "gemm", "save_acts")]


class E2TTTError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{e2ttt_status_string(status)}: {detail}")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      f"`python test_weight_layers_chunk_b200/build.py` (needs nvcc)")
_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_S = ctypes.POINTER(e2ttt_shape)
_SIGS = {
    "e2ttt_state_elems": (ctypes.c_size_t, [_S]),
    "e2ttt_workspace_bytes": (ctypes.c_size_t, [_S, ctypes.c_int]),
    "e2ttt_num_chunks": (ctypes.c_int, [_S]),
    "e2ttt_saved_bytes": (ctypes.c_size_t, [_S]),
    "e2ttt_fwd_uses_tensor_cores": (ctypes.c_int, [_S]),
    "e2ttt_chunk_coeffs": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P]),
    "e2ttt_chunk_scan_fwd": (ctypes.c_int, [_S] + [_P] * 13 + [ctypes.c_size_t, _P]),
    "e2ttt_chunk_scan_fwd_noalloc": (ctypes.c_int, [_S] + [_P] * 13),
    "e2ttt_chunk_scan_bwd": (ctypes.c_int, [_S] + [_P] * 19 + [ctypes.c_size_t, _P]),
    "e2ttt_workspace_status": (ctypes.c_int, [_P, _P]),
    "e2ttt_noalloc_status": (ctypes.c_int, [_P]),
    "e2ttt_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "e2ttt_last_error": (ctypes.c_char_p, []),
    "e2ttt_trace_enable": (None, [ctypes.c_int]),
    "e2ttt_test_stall_next_forward": (None, [ctypes.c_int]),
    "e2ttt_trace_summary": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def header_functions() -> list[str]:
    """Names of the functions include/e2ttt.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(e2ttt_[a-z_]+)\s*\(", src)))


def make_shape(B, H, T, C, d_k, d_v, d_h=0, kind=SWIGLU, act=BF16, loss=LOSS_MSE,
               coef=COEF_PER_TOKEN, momentum=MOMENTUM, gemm=GEMM_AUTO,
               save_acts=RECOMPUTE_ACTS) -> e2ttt_shape:
    return e2ttt_shape(B, H, T, C, d_k, d_v, d_h, kind, act, loss, coef, momentum, gemm, save_acts)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != OK:
        raise E2TTTError(status, _lib.e2ttt_last_error().decode())


def e2ttt_status_string(status: int) -> str:
    return _lib.e2ttt_status_string(status).decode()


def e2ttt_last_error() -> str:
    return _lib.e2ttt_last_error().decode()


def e2ttt_workspace_status(workspace, stream=None, raw=False):
    st = _lib.e2ttt_workspace_status(_ptr(workspace), _stream(stream) if not raw else stream)
    if raw:
        return st
    _check(st)


def e2ttt_test_stall_next_forward(on: bool = True) -> None:
    """Failure-detection test hook: the next tensor-core forward times out."""
    _lib.e2ttt_test_stall_next_forward(int(bool(on)))


def e2ttt_trace_enable(on: bool = True) -> None:
    _lib.e2ttt_trace_enable(int(bool(on)))


def e2ttt_trace_summary() -> dict:
    import json
    return json.loads(_lib.e2ttt_trace_summary().decode())


def e2ttt_state_elems(shape: e2ttt_shape) -> int:
    return _lib.e2ttt_state_elems(ctypes.byref(shape))


def e2ttt_workspace_bytes(shape: e2ttt_shape, for_bwd: int = 0) -> int:
    return _lib.e2ttt_workspace_bytes(ctypes.byref(shape), int(for_bwd))


def e2ttt_num_chunks(shape: e2ttt_shape) -> int:
    return _lib.e2ttt_num_chunks(ctypes.byref(shape))


def e2ttt_saved_bytes(shape: e2ttt_shape) -> int:
    return _lib.e2ttt_saved_bytes(ctypes.byref(shape))


def saved_states(shape, device="cuda"):
    """The saved-states buffer of `shape`: a float32 tensor viewed as
    [n_chunks, B, H, 2, S] (the chunk-start states) whose storage also holds the
    saved activations when shape.save_acts is set (e2ttt_saved_bytes in all)."""
    import torch
    nc, S = e2ttt_num_chunks(shape), e2ttt_state_elems(shape)
    n = (e2ttt_saved_bytes(shape) + 3) // 4
    flat = torch.empty(n, dtype=torch.float32, device=device)
    return flat[:nc * shape.B * shape.H * 2 * S].view(nc, shape.B, shape.H, 2, S)


def e2ttt_fwd_uses_tensor_cores(shape: e2ttt_shape) -> int:
    return _lib.e2ttt_fwd_uses_tensor_cores(ctypes.byref(shape))


def e2ttt_chunk_coeffs(shape, lr, mom, decay, a, b, chunk_scalars, stream=None, raw=False):
    st = _lib.e2ttt_chunk_coeffs(ctypes.byref(shape), _ptr(lr), _ptr(mom), _ptr(decay), _ptr(a),
                                 _ptr(b), _ptr(chunk_scalars), _stream(stream) if not raw else stream)
    if raw:
        return st
    _check(st)


def e2ttt_chunk_scan_fwd(shape, q, k, v, lr, mom, decay, W0, M0, out, W_end, M_end, saved_states,
                         workspace, workspace_bytes=None, stream=None, raw=False):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = _lib.e2ttt_chunk_scan_fwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(mom), _ptr(decay), _ptr(W0),
        _ptr(M0), _ptr(out), _ptr(W_end), _ptr(M_end), _ptr(saved_states), _ptr(workspace),
        workspace_bytes, _stream(stream) if not raw else stream)
    if raw:
        return st
    _check(st)


def e2ttt_chunk_scan_fwd_noalloc(shape, q, k, v, lr, mom, decay, W0, M0, out, W_end, M_end,
                                 saved_states, stream=None, raw=False):
    """The forward without a workspace (library-owned static scratch, at most
    32 MiB of it): for callers that cannot allocate device memory."""
    st = _lib.e2ttt_chunk_scan_fwd_noalloc(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(mom), _ptr(decay), _ptr(W0),
        _ptr(M0), _ptr(out), _ptr(W_end), _ptr(M_end), _ptr(saved_states),
        _stream(stream) if not raw else stream)
    if raw:
        return st
    _check(st)


def e2ttt_noalloc_status(stream=None, raw=False):
    """Status word of the last no-allocation forward on the current device."""
    st = _lib.e2ttt_noalloc_status(_stream(stream) if not raw else stream)
    if raw:
        return st
    _check(st)


def e2ttt_chunk_scan_bwd(shape, q, k, v, lr, mom, decay, saved_states, dout, dW_end, dM_end,
                         dq, dk, dv, dlr, dmom, ddecay, dW0, dM0, workspace, workspace_bytes=None,
                         stream=None, raw=False):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    st = _lib.e2ttt_chunk_scan_bwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(mom), _ptr(decay),
        _ptr(saved_states), _ptr(dout), _ptr(dW_end), _ptr(dM_end), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(dlr), _ptr(dmom), _ptr(ddecay), _ptr(dW0), _ptr(dM0), _ptr(workspace),
        workspace_bytes, _stream(stream) if not raw else stream)
    if raw:
        return st
    _check(st)


# ---------------------------------------------------------------- conveniences
def _shape_of(q, v, lr, C, d_h, kind, loss, coef=COEF_PER_TOKEN, momentum=MOMENTUM, gemm=GEMM_AUTO,
              save_acts=RECOMPUTE_ACTS):
    import torch
    B, H, T, d_k = q.shape
    act = BF16 if q.dtype == torch.bfloat16 else F32
    return make_shape(B, H, T, C, d_k, v.shape[-1], d_h, kind, act, loss, coef, momentum, gemm,
                      save_acts)


def workspace(shape, for_bwd=False, device="cuda"):
    """A torch uint8 buffer of the workspace size (torch's allocator returns
    256-byte aligned blocks)."""
    import torch
    n = e2ttt_workspace_bytes(shape, int(for_bwd))
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device)


def chunk_scan_fwd(q, k, v, lr, mom, decay, W0, M0=None, *, C, d_h=0, kind=SWIGLU,
                   loss=LOSS_MSE, coef=COEF_PER_TOKEN, momentum=MOMENTUM, save_states=False,
                   ws=None, stream=None, gemm=GEMM_AUTO, save_acts=RECOMPUTE_ACTS):
    """Allocate out / W_end / M_end (and saved_states) and run the forward.
    Returns (out, W_end, M_end, saved_states or None); M_end is None without
    momentum (momentum=NO_MOMENTUM: pass mom=None, M0=None). save_acts=SAVE_ACTS
    (with save_states) keeps the per-chunk E and dH for the backward; pass the
    same save_acts to chunk_scan_bwd."""
    import torch
    shape = _shape_of(q, v, lr, C, d_h, kind, loss, coef, momentum, gemm, save_acts)
    out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    W_end = torch.empty_like(W0)
    M_end = None if momentum == NO_MOMENTUM else torch.empty_like(W0)
    saved = saved_states(shape, q.device) if save_states else None
    if ws is None:
        ws = workspace(shape, False, q.device)
    e2ttt_chunk_scan_fwd(shape, q, k, v, lr, mom, decay, W0, M0, out, W_end, M_end, saved, ws,
                         stream=stream)
    return out, W_end, M_end, saved


def chunk_scan_bwd(q, k, v, lr, mom, decay, saved_states, dout, dW_end=None, dM_end=None, *, C,
                   d_h=0, kind=SWIGLU, loss=LOSS_MSE, coef=COEF_PER_TOKEN, momentum=MOMENTUM,
                   ws=None, stream=None, gemm=GEMM_AUTO, save_acts=RECOMPUTE_ACTS):
    """Allocate the gradients and run the backward. Returns a dict (dmom and dM0
    are None without momentum)."""
    import torch
    shape = _shape_of(q, v, lr, C, d_h, kind, loss, coef, momentum, gemm, save_acts)
    nomom = momentum == NO_MOMENTUM
    g = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
             dlr=torch.empty_like(lr), dmom=None if nomom else torch.empty_like(mom),
             ddecay=torch.empty_like(decay),
             dW0=torch.empty(saved_states.shape[1:3] + saved_states.shape[-1:], dtype=torch.float32,
                             device=q.device))
    g["dM0"] = None if nomom else torch.empty_like(g["dW0"])
    if ws is None:
        ws = workspace(shape, True, q.device)
    e2ttt_chunk_scan_bwd(shape, q, k, v, lr, mom, decay, saved_states, dout, dW_end, dM_end,
                         g["dq"], g["dk"], g["dv"], g["dlr"], g["dmom"], g["ddecay"], g["dW0"],
                         g["dM0"], ws, stream=stream)
    return g
