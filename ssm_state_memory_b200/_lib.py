"""ctypes binding of libdart.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks that tensors live on a CUDA device, passes
their data pointers, sizes and the current CUDA stream to the library, and
raises :class:`DartError` on a non-zero status. If ``libdart.so`` is missing
or cannot be loaded, importing this module raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdart.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python ssm_state_memory_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

DART_F32 = 0
DART_BF16 = 1
OP_CHUNK_STATES, OP_SSD_SCAN, OP_SMA_FWD, OP_LAYER_FWD, OP_SMA_BWD, OP_SMA_BWD_NORM, OP_SMA_FWD_NORM = range(7)

STATUS = {
    0: "DART_OK", 1: "DART_ERR_NULL", 2: "DART_ERR_DIMS", 3: "DART_ERR_DTYPE", 4: "DART_ERR_ALIGN",
    5: "DART_ERR_UNSUPPORTED", 6: "DART_ERR_WORKSPACE", 7: "DART_ERR_CUDA",
}


class dart_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seqlen", "nheads", "ngroups", "dstate", "headdim", "chunk")]


class DartError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        self.name = STATUS.get(status, str(status))
        msg = lib.dart_status_string(status).decode()
        if status == 7:
            msg += "; " + lib.dart_last_error().decode()
        super().__init__(f"{fn}: {self.name} ({msg})")


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_dims_p = ctypes.POINTER(dart_dims)

lib.dart_status_string.argtypes = [ctypes.c_int]
lib.dart_status_string.restype = ctypes.c_char_p
lib.dart_version.restype = ctypes.c_char_p
lib.dart_supported.argtypes = [_dims_p, ctypes.c_int]
lib.dart_supported.restype = ctypes.c_int
lib.dart_workspace_size.argtypes = [ctypes.c_int, _dims_p, ctypes.c_int]
lib.dart_workspace_size.restype = _sz
lib.dart_decode_workspace_size.argtypes = [_i64] * 5 + [ctypes.c_int]
lib.dart_decode_workspace_size.restype = _sz
lib.dart_chunk_states.argtypes = [_dims_p, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
lib.dart_ssd_scan.argtypes = [_dims_p, ctypes.c_int] + [_vp] * 8 + [_sz, _vp]
lib.dart_sma_fwd.argtypes = [_dims_p, ctypes.c_int] + [_vp] * 7
lib.dart_layer_fwd.argtypes = [_dims_p, ctypes.c_int] + [_vp] * 7 + [_i64] * 3 + [_vp] * 4 + [_sz, _vp]
lib.dart_sma_decode.argtypes = [_i64] * 7 + [ctypes.c_int] + [_vp] * 5 + [_i64] * 2 + [_vp] * 4 + [_sz, _vp]
lib.dart_sma_decode_noalloc.argtypes = [_i64] * 7 + [ctypes.c_int] + [_vp] * 5 + [_i64] * 2 + [_vp] * 3 + [_vp]
lib.dart_sma_fwd_norm.argtypes = [ctypes.POINTER(dart_dims), ctypes.c_int] + [_vp] * 6 + [ctypes.c_float, _vp]
lib.dart_sma_fwd_norm_ws.argtypes = [_dims_p, ctypes.c_int] + [_vp] * 6 + [ctypes.c_float, _vp, _sz, _vp]
lib.dart_decode_step_workspace_size.argtypes = [_i64] * 5 + [ctypes.c_int]
lib.dart_decode_step_workspace_size.restype = _sz
lib.dart_decode_step.argtypes = ([_i64] * 7 + [ctypes.c_int, ctypes.c_int] + [_vp] * 7 + [_i64] * 2 + [_vp] * 6
                                 + [_sz, _vp])
lib.dart_sma_bwd.argtypes = [_dims_p, ctypes.c_int] + [_vp] * 12 + [_sz, _vp]
lib.dart_sma_fwd_ge.argtypes = [_dims_p, ctypes.c_int, _i64] + [_vp] * 7
lib.dart_sma_bwd_ge.argtypes = [_dims_p, ctypes.c_int, _i64] + [_vp] * 12 + [_sz, _vp]
lib.dart_sma_bwd_norm.argtypes = [_dims_p, ctypes.c_int, ctypes.c_float] + [_vp] * 12 + [_sz, _vp]
lib.dart_layer_fwd_ge.argtypes = [_dims_p, ctypes.c_int, _i64] + [_vp] * 7 + [_i64] * 3 + [_vp] * 4 + [_sz, _vp]
lib.dart_sma_decode_ge.argtypes = [_i64] * 8 + [ctypes.c_int] + [_vp] * 5 + [_i64] * 2 + [_vp] * 4 + [_sz, _vp]
for _f in ("dart_chunk_states", "dart_ssd_scan", "dart_sma_fwd", "dart_layer_fwd", "dart_sma_decode",
           "dart_sma_decode_noalloc", "dart_decode_step", "dart_sma_fwd_norm", "dart_sma_bwd", "dart_sma_fwd_ge",
           "dart_layer_fwd_ge", "dart_sma_decode_ge", "dart_sma_bwd_norm", "dart_sma_fwd_norm_ws",
           "dart_sma_bwd_ge"):
    getattr(lib, _f).restype = ctypes.c_int
lib.dart_kernel_launches.restype = _i64
lib.dart_kernel_kinds.restype = ctypes.c_int
lib.dart_kernel_name.argtypes = [ctypes.c_int]
lib.dart_kernel_name.restype = ctypes.c_char_p
lib.dart_profile_enable.argtypes = [ctypes.c_int]
lib.dart_profile_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)]
lib.dart_profile_reset.argtypes = []
lib.dart_device_error.restype = ctypes.c_int
lib.dart_fp16_range_flags.restype = ctypes.c_int
lib.dart_set_wait_limit.argtypes = [ctypes.c_uint64]
lib.dart_set_wait_limit.restype = ctypes.c_int
lib.dart_last_error.restype = ctypes.c_char_p

# every symbol include/dart.h declares
EXPORTS = (
    "dart_status_string", "dart_version", "dart_supported", "dart_workspace_size", "dart_chunk_states",
    "dart_ssd_scan", "dart_sma_fwd", "dart_layer_fwd", "dart_decode_workspace_size", "dart_sma_decode",
    "dart_kernel_launches", "dart_kernel_kinds", "dart_kernel_name", "dart_profile_enable", "dart_profile_read",
    "dart_profile_reset", "dart_device_error", "dart_last_error", "dart_sma_decode_noalloc",
    "dart_decode_step_workspace_size", "dart_decode_step", "dart_sma_fwd_norm", "dart_sma_bwd",
    "dart_sma_fwd_ge", "dart_layer_fwd_ge", "dart_sma_decode_ge", "dart_sma_bwd_norm", "dart_sma_fwd_norm_ws",
    "dart_sma_bwd_ge", "dart_fp16_range_flags", "dart_set_wait_limit",
)


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise DartError(fn, status)


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return DART_BF16
    if t.dtype == torch.float32:
        return DART_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t, name: str, optional: bool = False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(t) -> int:
    import torch

    return torch.cuda.current_stream(t.device).cuda_stream


def dims_of(batch, seqlen, nheads, ngroups, dstate, headdim, chunk) -> dart_dims:
    return dart_dims(batch, seqlen, nheads, ngroups, dstate, headdim, chunk)


def dims_from(X, B, chunk: int) -> dart_dims:
    """dart_dims from X [b, L, H, P] and B [b, L, G, N]."""
    b, L, H, P = X.shape
    G, N = B.shape[2], B.shape[3]
    return dart_dims(b, L, H, G, N, P, chunk)


def dart_supported(d: dart_dims, dtype_code: int) -> int:
    return lib.dart_supported(ctypes.byref(d), dtype_code)


def dart_workspace_size(op: int, d: dart_dims, dtype_code: int) -> int:
    return int(lib.dart_workspace_size(op, ctypes.byref(d), dtype_code))


def dart_decode_workspace_size(batch, nheads, dstate, headdim, n_chunks, dtype_code) -> int:
    return int(lib.dart_decode_workspace_size(batch, nheads, dstate, headdim, n_chunks, dtype_code))


def _ws_args(ws):
    if ws is None:
        return None, 0
    return _ptr(ws, "ws"), ws.numel() * ws.element_size()


def dart_chunk_states(d: dart_dims, X, B, logA, dH, ws) -> None:
    w, wb = _ws_args(ws)
    _check("dart_chunk_states", lib.dart_chunk_states(ctypes.byref(d), _dtype_code(X), _ptr(X, "X"), _ptr(B, "B"),
                                                      _ptr(logA, "logA"), _ptr(dH, "dH"), w, wb, _stream(X)))


def dart_ssd_scan(d: dart_dims, X, B, C, logA, dH, Y, final_state, ws) -> None:
    w, wb = _ws_args(ws)
    _check("dart_ssd_scan", lib.dart_ssd_scan(ctypes.byref(d), _dtype_code(X), _ptr(X, "X"), _ptr(B, "B"),
                                              _ptr(C, "C"), _ptr(logA, "logA"), _ptr(dH, "dH"), _ptr(Y, "Y"),
                                              _ptr(final_state, "final_state", True), w, wb, _stream(X)))


def dart_sma_fwd(d: dart_dims, Q, C, E, dH, R, lse) -> None:
    _check("dart_sma_fwd", lib.dart_sma_fwd(ctypes.byref(d), _dtype_code(Q), _ptr(Q, "Q"), _ptr(C, "C"),
                                            _ptr(E, "E"), _ptr(dH, "dH"), _ptr(R, "R"), _ptr(lse, "lse", True),
                                            _stream(Q)))


def dart_sma_fwd_ge(d: dart_dims, e_groups: int, Q, C, E, dH, R, lse) -> None:
    _check("dart_sma_fwd_ge", lib.dart_sma_fwd_ge(ctypes.byref(d), _dtype_code(Q), int(e_groups), _ptr(Q, "Q"),
                                                  _ptr(C, "C"), _ptr(E, "E"), _ptr(dH, "dH"), _ptr(R, "R"),
                                                  _ptr(lse, "lse", True), _stream(Q)))


def dart_layer_fwd_ge(d: dart_dims, e_groups: int, X, B, C, Q, E, logA, g, g_strides: Sequence[int], out, dH_out,
                      lse_out, ws) -> None:
    w, wb = _ws_args(ws)
    sb, st, sh = g_strides
    _check("dart_layer_fwd_ge", lib.dart_layer_fwd_ge(ctypes.byref(d), _dtype_code(X), int(e_groups), _ptr(X, "X"),
                                                      _ptr(B, "B"), _ptr(C, "C"), _ptr(Q, "Q"), _ptr(E, "E"),
                                                      _ptr(logA, "logA"), _ptr(g, "g"), sb, st, sh,
                                                      _ptr(out, "out"), _ptr(dH_out, "dH_out"),
                                                      _ptr(lse_out, "lse_out", True), w, wb, _stream(X)))


def dart_sma_decode_ge(n_chunks: int, Q, C, E, Y, g, g_strides: Tuple[int, int], cache, out, lse, ws) -> None:
    """dart_sma_decode with E [b, e_groups, P] (e_groups read from E's shape)."""
    b, G, N = Q.shape
    H, P = Y.shape[1], Y.shape[2]
    EG = E.shape[1]
    cs = cache.shape[2]
    w, wb = _ws_args(ws)
    sb, sh = g_strides
    _check("dart_sma_decode_ge", lib.dart_sma_decode_ge(b, H, G, EG, N, P, n_chunks, cs, _dtype_code(Q),
                                                        _ptr(Q, "Q"), _ptr(C, "C"), _ptr(E, "E"), _ptr(Y, "Y"),
                                                        _ptr(g, "g"), sb, sh, _ptr(cache, "cache"), _ptr(out, "out"),
                                                        _ptr(lse, "lse", True), w, wb, _stream(Q)))


def dart_layer_fwd(d: dart_dims, X, B, C, Q, E, logA, g, g_strides: Sequence[int], out, dH_out, lse_out, ws) -> None:
    w, wb = _ws_args(ws)
    sb, st, sh = g_strides
    _check("dart_layer_fwd", lib.dart_layer_fwd(ctypes.byref(d), _dtype_code(X), _ptr(X, "X"), _ptr(B, "B"),
                                                _ptr(C, "C"), _ptr(Q, "Q"), _ptr(E, "E"), _ptr(logA, "logA"),
                                                _ptr(g, "g"), sb, st, sh, _ptr(out, "out"), _ptr(dH_out, "dH_out"),
                                                _ptr(lse_out, "lse_out", True), w, wb, _stream(X)))


def dart_sma_decode(n_chunks: int, Q, C, E, Y, g, g_strides: Tuple[int, int], cache, out, lse, ws) -> None:
    """Q, C [b, G, N]; E, Y, out [b, H, P]; cache [b, H, cs, N, P]; lse [b, H]."""
    b, G, N = Q.shape
    H, P = E.shape[1], E.shape[2]
    cs = cache.shape[2]
    w, wb = _ws_args(ws)
    sb, sh = g_strides
    _check("dart_sma_decode", lib.dart_sma_decode(b, H, G, N, P, n_chunks, cs, _dtype_code(Q), _ptr(Q, "Q"),
                                                  _ptr(C, "C"), _ptr(E, "E"), _ptr(Y, "Y"), _ptr(g, "g"), sb, sh,
                                                  _ptr(cache, "cache"), _ptr(out, "out"), _ptr(lse, "lse", True),
                                                  w, wb, _stream(Q)))


def dart_sma_fwd_norm(d: dart_dims, Q, C, E, dH, R, lse, eps: float) -> None:
    _check("dart_sma_fwd_norm", lib.dart_sma_fwd_norm(ctypes.byref(d), _dtype_code(Q), _ptr(Q, "Q"), _ptr(C, "C"),
                                                      _ptr(E, "E"), _ptr(dH, "dH"), _ptr(R, "R"),
                                                      _ptr(lse, "lse", True), float(eps), _stream(Q)))


def dart_sma_fwd_norm_ws(d: dart_dims, Q, C, E, dH, R, lse, eps: float, ws) -> None:
    w, wb = _ws_args(ws)
    _check("dart_sma_fwd_norm_ws", lib.dart_sma_fwd_norm_ws(ctypes.byref(d), _dtype_code(Q), _ptr(Q, "Q"),
                                                            _ptr(C, "C"), _ptr(E, "E"), _ptr(dH, "dH"), _ptr(R, "R"),
                                                            _ptr(lse, "lse", True), float(eps), w, wb, _stream(Q)))


def dart_sma_bwd(d: dart_dims, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws) -> None:
    w, wb = _ws_args(ws)
    _check("dart_sma_bwd", lib.dart_sma_bwd(ctypes.byref(d), _dtype_code(Q), _ptr(Q, "Q"), _ptr(C, "C"), _ptr(E, "E"),
                                            _ptr(dH, "dH"), _ptr(R, "R"), _ptr(lse, "lse"), _ptr(dR, "dR"),
                                            _ptr(dQ, "dQ"), _ptr(dC, "dC"), _ptr(dE, "dE"), _ptr(ddH, "ddH"), w, wb,
                                            _stream(Q)))


def dart_sma_bwd_ge(d: dart_dims, e_groups: int, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws) -> None:
    w, wb = _ws_args(ws)
    _check("dart_sma_bwd_ge", lib.dart_sma_bwd_ge(ctypes.byref(d), _dtype_code(Q), int(e_groups), _ptr(Q, "Q"),
                                                  _ptr(C, "C"), _ptr(E, "E"), _ptr(dH, "dH"), _ptr(R, "R"),
                                                  _ptr(lse, "lse"), _ptr(dR, "dR"), _ptr(dQ, "dQ"), _ptr(dC, "dC"),
                                                  _ptr(dE, "dE"), _ptr(ddH, "ddH"), w, wb, _stream(Q)))


def dart_sma_bwd_norm(d: dart_dims, eps: float, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws) -> None:
    w, wb = _ws_args(ws)
    _check("dart_sma_bwd_norm", lib.dart_sma_bwd_norm(ctypes.byref(d), _dtype_code(Q), float(eps), _ptr(Q, "Q"),
                                                      _ptr(C, "C"), _ptr(E, "E"), _ptr(dH, "dH"),
                                                      _ptr(R, "R", True), _ptr(lse, "lse", True), _ptr(dR, "dR"),
                                                      _ptr(dQ, "dQ"),
                                                      _ptr(dC, "dC"), _ptr(dE, "dE"), _ptr(ddH, "ddH"), w, wb,
                                                      _stream(Q)))


def dart_decode_step_workspace_size(b: int, H: int, N: int, P: int, n_chunks: int, dtype: int) -> int:
    return int(lib.dart_decode_step_workspace_size(b, H, N, P, n_chunks, dtype))


def dart_decode_step(n_chunks: int, close_chunk: bool, X, B, C, Q, E, logA, g, g_strides: Tuple[int, int], state,
                     chunk_acc, cache, out, lse, ws) -> None:
    """X, E, out [b, H, P]; B, C, Q [b, G, N]; logA [b, H]; state, chunk_acc [b, H, N, P] fp32;
    cache [b, H, cs, N, P]; lse [b, H]."""
    b, G, N = Q.shape
    H, P = E.shape[1], E.shape[2]
    cs = cache.shape[2]
    w, wb = _ws_args(ws)
    sb, sh = g_strides
    _check("dart_decode_step", lib.dart_decode_step(
        b, H, G, N, P, n_chunks, cs, 1 if close_chunk else 0, _dtype_code(Q), _ptr(X, "X"), _ptr(B, "B"),
        _ptr(C, "C"), _ptr(Q, "Q"), _ptr(E, "E"), _ptr(logA, "logA"), _ptr(g, "g"), sb, sh, _ptr(state, "state"),
        _ptr(chunk_acc, "chunk_acc"), _ptr(cache, "cache"), _ptr(out, "out"), _ptr(lse, "lse", True), w, wb,
        _stream(Q)))


def dart_last_error() -> str:
    return lib.dart_last_error().decode()


def dart_device_error() -> int:
    return int(lib.dart_device_error())


def dart_fp16_range_flags() -> int:
    return int(lib.dart_fp16_range_flags())


def dart_set_wait_limit(ns: int) -> None:
    _check("dart_set_wait_limit", lib.dart_set_wait_limit(int(ns)))


def dart_sma_decode_noalloc(n_chunks: int, Q, C, E, Y, g, g_strides: Tuple[int, int], cache, out, lse) -> None:
    """dart_sma_decode with the library's fixed device scratch instead of a workspace (allocates nothing)."""
    b, G, N = Q.shape
    H, P = E.shape[1], E.shape[2]
    cs = cache.shape[2]
    sb, sh = g_strides
    _check("dart_sma_decode_noalloc", lib.dart_sma_decode_noalloc(
        b, H, G, N, P, n_chunks, cs, _dtype_code(Q), _ptr(Q, "Q"), _ptr(C, "C"), _ptr(E, "E"), _ptr(Y, "Y"),
        _ptr(g, "g"), sb, sh, _ptr(cache, "cache"), _ptr(out, "out"), _ptr(lse, "lse", True), _stream(Q)))


def dart_kernel_launches() -> int:
    return int(lib.dart_kernel_launches())


def kernel_names():
    return [lib.dart_kernel_name(i).decode() for i in range(lib.dart_kernel_kinds())]


def dart_profile_enable(on: bool) -> None:
    _check("dart_profile_enable", lib.dart_profile_enable(1 if on else 0))


def dart_profile_reset() -> None:
    _check("dart_profile_reset", lib.dart_profile_reset())


def dart_profile_read(kind: int) -> Tuple[float, int]:
    ms = ctypes.c_double()
    n = _i64()
    _check("dart_profile_read", lib.dart_profile_read(kind, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


def profile_table():
    """{kernel name: (total ms, launches)} for every kernel kind."""
    return {name: dart_profile_read(i) for i, name in enumerate(kernel_names())}
