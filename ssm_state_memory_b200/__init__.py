"""DART forward hot path on B200 (sm_100a): Python binding of libdart.so.

The functions named ``dart_*`` mirror the C entry points of ``include/dart.h``
one to one. The helpers below them only allocate outputs and workspace with
PyTorch (device memory is plumbing) and then call those entry points; every
step of the computation runs in the library's CUDA kernels.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence, Tuple

from ._lib import (  # noqa: F401
    DART_BF16, DART_F32, EXPORTS, LIB_PATH, OP_CHUNK_STATES, OP_LAYER_FWD, OP_SMA_BWD, OP_SMA_BWD_NORM, OP_SMA_FWD,
    OP_SMA_FWD_NORM, OP_SSD_SCAN,
    DartError, dart_chunk_states, dart_decode_step, dart_decode_step_workspace_size, dart_decode_workspace_size,
    dart_layer_fwd_ge, dart_sma_bwd, dart_sma_bwd_ge, dart_sma_bwd_norm, dart_sma_decode_ge, dart_sma_fwd_ge, dart_sma_fwd_norm,
    dart_sma_fwd_norm_ws,
    dart_device_error, dart_dims, dart_fp16_range_flags, dart_kernel_launches, dart_set_wait_limit,
    dart_last_error, dart_layer_fwd,
    dart_profile_enable, dart_profile_read, dart_profile_reset, dart_sma_decode, dart_sma_decode_noalloc,
    dart_sma_fwd, dart_ssd_scan,
    dart_supported, dart_workspace_size, dims_from, dims_of, kernel_names, lib, profile_table,
)


def _empty(shape, dtype, device):
    import torch

    return torch.empty(shape, dtype=dtype, device=device)


def workspace(op: int, d: dart_dims, dtype, device):
    import torch

    code = DART_BF16 if dtype == torch.bfloat16 else DART_F32
    n = dart_workspace_size(op, d, code)
    return _empty((max(n, 256),), torch.uint8, device)


def layer_fwd(X, B, C, Q, E, logA, g, g_strides: Sequence[int], chunk: int, ws=None, want_lse: bool = True):
    """Whole mixer forward. Returns (out [b, L, H, P], dH [b, H, M, N, P], lse [b, H, L] or None)."""
    import torch

    d = dims_from(X, B, chunk)
    M = -(-d.seqlen // chunk)
    out = _empty(X.shape, torch.float32, X.device)
    dH = _empty((d.batch, d.nheads, M, d.dstate, d.headdim), X.dtype, X.device)
    lse = _empty((d.batch, d.nheads, d.seqlen), torch.float32, X.device) if want_lse else None
    if ws is None:
        ws = workspace(OP_LAYER_FWD, d, X.dtype, X.device)
    if E.shape[2] != d.nheads:  # grouped E [b, L, e_groups, P]
        dart_layer_fwd_ge(d, E.shape[2], X, B, C, Q, E, logA, g, g_strides, out, dH, lse, ws)
    else:
        dart_layer_fwd(d, X, B, C, Q, E, logA, g, g_strides, out, dH, lse, ws)
    return out, dH, lse


def chunk_states(X, B, logA, chunk: int, ws=None):
    d = dims_from(X, B, chunk)
    M = -(-d.seqlen // chunk)
    dH = _empty((d.batch, d.nheads, M, d.dstate, d.headdim), X.dtype, X.device)
    if ws is None:
        ws = workspace(OP_CHUNK_STATES, d, X.dtype, X.device)
    dart_chunk_states(d, X, B, logA, dH, ws)
    return dH


def ssd_scan(X, B, C, logA, dH, chunk: int, want_final: bool = True, ws=None):
    import torch

    d = dims_from(X, B, chunk)
    Y = _empty(X.shape, torch.float32, X.device)
    fin = _empty((d.batch, d.nheads, d.dstate, d.headdim), torch.float32, X.device) if want_final else None
    if ws is None:
        ws = workspace(OP_SSD_SCAN, d, X.dtype, X.device)
    dart_ssd_scan(d, X, B, C, logA, dH, Y, fin, ws)
    return Y, fin


def sma_fwd(Q, C, E, dH, chunk: int, norm_eps: Optional[float] = None, ws=None, prep_pass: bool = True):
    """SMA forward; with norm_eps, the normalised score branch (dart_sma_fwd_norm_ws, with the fp16 key rows
    and Q rows prepared once into ws unless prep_pass is False: then dart_sma_fwd_norm, whose kernel rescales
    them itself). E may be grouped, [b, L, e_groups, P] with fewer groups than dH has heads
    (dart_sma_fwd_ge)."""
    import torch

    b, L, EG, P = E.shape
    H = dH.shape[1]
    G, N = Q.shape[2], Q.shape[3]
    d = dims_of(b, L, H, G, N, P, chunk)
    R = _empty((b, L, H, P), torch.float32, E.device)
    lse = _empty((b, H, L), torch.float32, E.device)
    if norm_eps is not None:
        if EG != H:
            raise ValueError("the normalised score branch takes E per head")
        if prep_pass:
            if ws is None:
                ws = workspace(OP_SMA_FWD_NORM, d, Q.dtype, Q.device)
            dart_sma_fwd_norm_ws(d, Q, C, E, dH, R, lse, norm_eps, ws)
        else:
            dart_sma_fwd_norm(d, Q, C, E, dH, R, lse, norm_eps)
    elif EG != H:
        dart_sma_fwd_ge(d, EG, Q, C, E, dH, R, lse)
    else:
        dart_sma_fwd(d, Q, C, E, dH, R, lse)
    return R, lse


def sma_bwd(Q, C, E, dH, R, lse, dR, chunk: int, ws=None, norm_eps: Optional[float] = None):
    """SMA backward by recomputation (dart_sma_bwd; with norm_eps, the normalised branch's,
    dart_sma_bwd_norm, which recomputes the softmax statistics: R and lse may then be None). E may be
    grouped, [b, L, e_groups, P] (dart_sma_bwd_ge; dE then has E's shape). Returns (dQ, dC, dE, ddH),
    fp32."""
    import torch

    b, L, EG, P = E.shape
    H = dH.shape[1]
    G, N = Q.shape[2], Q.shape[3]
    d = dims_of(b, L, H, G, N, P, chunk)
    dQ = _empty(Q.shape, torch.float32, Q.device)
    dC = _empty(C.shape, torch.float32, Q.device)
    dE = _empty(E.shape, torch.float32, Q.device)
    ddH = _empty(dH.shape, torch.float32, Q.device)
    if ws is None:
        ws = workspace(OP_SMA_BWD if norm_eps is None else OP_SMA_BWD_NORM, d, Q.dtype, Q.device)
    if norm_eps is None:
        if EG != H:
            dart_sma_bwd_ge(d, EG, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws)
        else:
            dart_sma_bwd(d, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws)
    else:
        if EG != H:
            raise ValueError("the normalised score branch takes E per head")
        dart_sma_bwd_norm(d, norm_eps, Q, C, E, dH, R, lse, dR, dQ, dC, dE, ddH, ws)
    return dQ, dC, dE, ddH


def decode_step(X, B, C, Q, E, logA, g, g_strides: Tuple[int, int], state, chunk_acc, cache, n_chunks: int,
                close_chunk: bool, ws=None):
    """One decode step for one new token per batch row; state, chunk_acc and cache are updated in place
    (see dart_decode_step). Returns (out, lse)."""
    import torch

    b, G, N = Q.shape
    H, P = E.shape[1], E.shape[2]
    out = _empty((b, H, P), torch.float32, E.device)
    lse = _empty((b, H), torch.float32, E.device)
    if ws is None:
        code = DART_BF16 if Q.dtype == torch.bfloat16 else DART_F32
        ws = _empty((max(dart_decode_step_workspace_size(b, H, N, P, n_chunks, code), 256),), torch.uint8, E.device)
    dart_decode_step(n_chunks, close_chunk, X, B, C, Q, E, logA, g, g_strides, state, chunk_acc, cache, out, lse, ws)
    return out, lse


def sma_decode(Q, C, E, Y, g, g_strides: Tuple[int, int], cache, n_chunks: Optional[int] = None, ws=None):
    import torch

    b, G, N = Q.shape
    H, P = Y.shape[1], Y.shape[2]
    n = cache.shape[2] if n_chunks is None else n_chunks
    out = _empty(Y.shape, torch.float32, Y.device)
    lse = _empty((b, H), torch.float32, Y.device)
    if ws is None:
        code = DART_BF16 if Q.dtype == torch.bfloat16 else DART_F32
        ws = _empty((max(dart_decode_workspace_size(b, H, N, P, n, code), 256),), torch.uint8, Y.device)
    if E.shape[1] != H:  # grouped E [b, e_groups, P]
        dart_sma_decode_ge(n, Q, C, E, Y, g, g_strides, cache, out, lse, ws)
    else:
        dart_sma_decode(n, Q, C, E, Y, g, g_strides, cache, out, lse, ws)
    return out, lse
