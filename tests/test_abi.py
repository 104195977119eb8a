"""The C-ABI library loads, exports what include/dart.h declares, and rejects bad
arguments on the host before anything is enqueued (no GPU needed: no call below
reaches a kernel launch)."""
import ctypes
import os
import re
import subprocess

import pytest

import ssm_state_memory_b200 as dart
from ssm_state_memory_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "dart.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dart_[a-z_0-9]+)\s*\(", text)))


def test_header_and_exports_agree():
    declared = header_functions()
    assert declared == sorted(_lib.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", dart.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (dart_[a-z_0-9]+)$", out, flags=re.M))
    for name in declared:
        assert name in exported, name
        assert hasattr(dart.lib, name)


def test_library_has_no_driver_dependency():
    out = subprocess.run(["ldd", dart.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out


def test_status_strings_and_version():
    assert dart.lib.dart_status_string(0) == b"ok"
    for code in range(1, 8):
        assert dart.lib.dart_status_string(code) != b"unknown status"
    assert b"sm_100a" in dart.lib.dart_version()
    names = dart.kernel_names()
    assert "sma_fwd_tc" in names and "sma_decode" in names and "state_pass" in names


def dims(**kw):
    base = dict(batch=2, seqlen=512, nheads=4, ngroups=1, dstate=128, headdim=64, chunk=256)
    base.update(kw)
    return dart.dims_of(*[base[k] for k in ("batch", "seqlen", "nheads", "ngroups", "dstate", "headdim", "chunk")])


def test_supported_and_workspace_sizes():
    assert dart.dart_supported(dims(), dart.DART_BF16) == 0
    assert dart.dart_supported(dims(nheads=5, ngroups=2), dart.DART_BF16) == 2
    assert dart.dart_supported(dims(dstate=512), dart.DART_BF16) == 5
    assert dart.dart_supported(dims(chunk=0), dart.DART_F32) == 2
    assert dart.dart_supported(dims(), 7) == 3
    d = dims()
    M = 2
    need_cs = 2 * 4 * 512 * 4 + 2 * 4 * M * 4
    ws_layer = dart.dart_workspace_size(dart.OP_LAYER_FWD, d, dart.DART_BF16)
    assert ws_layer >= need_cs + 2 * 4 * M * 128 * 64 * 2 and ws_layer % 256 == 0
    assert dart.dart_workspace_size(dart.OP_SMA_FWD, d, dart.DART_BF16) == 0
    # normalised branch on the tensor-core path: the fp16 key rows [b, H, M, N, P], the fp16 Q rows
    # [b, L, G, N] and their factors [b, L, G] fp32, each part 256-byte aligned; none off it
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert dart.dart_workspace_size(dart.OP_SMA_FWD_NORM, d, dart.DART_BF16) == (
        up(2 * 4 * M * 128 * 64 * 2) + up(2 * 512 * 1 * 128 * 2) + up(2 * 512 * 1 * 4))
    assert dart.dart_workspace_size(dart.OP_SMA_FWD_NORM, d, dart.DART_F32) == 0
    assert dart.dart_workspace_size(dart.OP_SMA_FWD_NORM, dims(dstate=64), dart.DART_BF16) == 0
    assert dart.dart_workspace_size(dart.OP_CHUNK_STATES, d, dart.DART_BF16) < ws_layer
    assert dart.dart_workspace_size(dart.OP_LAYER_FWD, dims(dstate=1024), dart.DART_BF16) == 0
    assert dart.dart_decode_workspace_size(64, 32, 128, 64, 256, dart.DART_BF16) > 0
    assert dart.dart_decode_workspace_size(64, 32, 128, 60, 256, dart.DART_BF16) == 0  # 120-byte rows


FAKE = 1 << 20  # a 16-byte-aligned address that is never dereferenced: every call below fails validation first


def layer_call(d, **over):
    a = dict(X=FAKE, B=FAKE, C=FAKE, Q=FAKE, E=FAKE, logA=FAKE, g=FAKE, out=FAKE, dH=FAKE, lse=None, ws=None,
             ws_bytes=0)
    a.update(over)
    return dart.lib.dart_layer_fwd(ctypes.byref(d), dart.DART_BF16, a["X"], a["B"], a["C"], a["Q"], a["E"], a["logA"],
                                   a["g"], 0, 0, 0, a["out"], a["dH"], a["lse"], a["ws"], a["ws_bytes"], None)


def test_host_side_validation_statuses():
    before = dart.dart_kernel_launches()
    d = dims()
    need = dart.dart_workspace_size(dart.OP_LAYER_FWD, d, dart.DART_BF16)
    assert layer_call(d, X=None) == 1
    assert layer_call(d, out=None, ws=FAKE, ws_bytes=need) == 1
    assert layer_call(d, E=FAKE + 8) == 4
    assert layer_call(d) == 6  # no workspace
    assert layer_call(d, ws=FAKE, ws_bytes=need - 1) == 6
    assert layer_call(d, ws=FAKE + 16, ws_bytes=need) == 4  # workspace must be 256-byte aligned
    assert layer_call(dims(nheads=3, ngroups=2)) == 2
    assert layer_call(dims(headdim=300)) == 5
    dd = dims()
    assert dart.lib.dart_sma_fwd(ctypes.byref(dd), 9, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == 3
    assert dart.lib.dart_sma_fwd_norm(ctypes.byref(dd), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, None, -1.0,
                                      None) == 2  # eps must be >= 0
    assert dart.lib.dart_sma_fwd_norm(ctypes.byref(dd), dart.DART_BF16, FAKE, FAKE, None, FAKE, FAKE, None, 1e-6,
                                      None) == 1
    nws = dart.dart_workspace_size(dart.OP_SMA_FWD_NORM, dd, dart.DART_BF16)
    assert dart.lib.dart_sma_fwd_norm_ws(ctypes.byref(dd), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1e-6,
                                         FAKE, nws - 1, None) == 6  # scratch too small
    assert dart.lib.dart_sma_fwd_norm_ws(ctypes.byref(dd), dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1e-6,
                                         FAKE + 16, nws, None) == 4  # scratch must be 256-byte aligned
    assert dart.lib.dart_sma_fwd_norm_ws(ctypes.byref(dd), dart.DART_BF16, FAKE, FAKE, FAKE, None, FAKE, None, 1e-6,
                                         FAKE, nws, None) == 1
    assert dart.lib.dart_sma_decode(2, 4, 1, 128, 64, 5, 4, dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0,
                                    FAKE, FAKE, None, None, 0, None) == 2  # chunk_stride < n_chunks
    assert dart.lib.dart_sma_decode(2, 4, 1, 128, 64, 5, 8, dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 0,
                                    FAKE, FAKE, None, None, 0, None) == 6  # needs partials workspace
    assert dart.dart_kernel_launches() == before  # nothing was launched by any of the rejected calls


def step_call(n_chunks=3, chunk_stride=8, close=0, dtype=None, **over):
    a = dict(X=FAKE, B=FAKE, C=FAKE, Q=FAKE, E=FAKE, logA=FAKE, g=FAKE, state=FAKE, acc=FAKE, cache=FAKE, out=FAKE,
             lse=None, ws=None, ws_bytes=0)
    a.update(over)
    return dart.lib.dart_decode_step(2, 4, 1, 128, 64, n_chunks, chunk_stride, close,
                                     dart.DART_BF16 if dtype is None else dtype, a["X"], a["B"], a["C"], a["Q"],
                                     a["E"], a["logA"], a["g"], 0, 0, a["state"], a["acc"], a["cache"], a["out"],
                                     a["lse"], a["ws"], a["ws_bytes"], None)


def test_decode_step_validation_statuses():
    before = dart.dart_kernel_launches()
    need = dart.dart_decode_step_workspace_size(2, 4, 128, 64, 3, dart.DART_BF16)
    # the step's own fp32 Y [b, H, P] comes first in the workspace, then the readout partials
    assert need >= 2 * 4 * 64 * 4 + dart.dart_decode_workspace_size(2, 4, 128, 64, 3, dart.DART_BF16)
    assert need % 256 == 0
    assert dart.dart_decode_step_workspace_size(2, 4, 128, 60, 3, dart.DART_BF16) == 0
    ok = dict(ws=FAKE, ws_bytes=need)
    assert step_call(n_chunks=8, chunk_stride=8, close=1, **ok) == 2  # a closing chunk needs a free slot
    assert step_call(n_chunks=9, chunk_stride=8, **ok) == 2
    assert step_call(dtype=5, **ok) == 3
    assert step_call(X=None, **ok) == 1
    assert step_call(logA=None, **ok) == 1
    assert step_call(state=None, **ok) == 1
    assert step_call(acc=FAKE + 4, **ok) == 4
    assert step_call(logA=FAKE + 2, **ok) == 4
    assert step_call() == 6
    assert step_call(ws=FAKE, ws_bytes=need - 1) == 6
    assert dart.dart_kernel_launches() == before


def test_binding_refuses_host_tensors():
    import torch

    x = torch.zeros(2, 8, 1, 64, dtype=torch.bfloat16)
    b = torch.zeros(2, 8, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        dart.chunk_states(x, b, torch.zeros(2, 8, 1), 4, ws=torch.zeros(16, dtype=torch.uint8))


def bwd_call(d, **over):
    a = dict(Q=FAKE, C=FAKE, E=FAKE, dH=FAKE, R=FAKE, lse=FAKE, dR=FAKE, dQ=FAKE, dC=FAKE, dE=FAKE, ddH=FAKE,
             ws=None, ws_bytes=0, dtype=dart.DART_BF16)
    a.update(over)
    return dart.lib.dart_sma_bwd(ctypes.byref(d), a["dtype"], a["Q"], a["C"], a["E"], a["dH"], a["R"], a["lse"],
                                 a["dR"], a["dQ"], a["dC"], a["dE"], a["ddH"], a["ws"], a["ws_bytes"], None)


def test_sma_bwd_validation_statuses():
    before = dart.dart_kernel_launches()
    d = dims()
    need = dart.dart_workspace_size(dart.OP_SMA_BWD, d, dart.DART_BF16)
    assert need >= 2 * 4 * 512 * 4 and need % 256 == 0  # D_t = dR_t . R_t for every (b, h, t)
    assert bwd_call(d) == 6  # no workspace
    assert bwd_call(d, ws=FAKE, ws_bytes=need - 1) == 6
    for name in ("Q", "C", "E", "dH", "R", "lse", "dR", "dQ", "dC", "dE", "ddH"):
        assert bwd_call(d, ws=FAKE, ws_bytes=need, **{name: None}) == 1, name
    assert bwd_call(d, ws=FAKE, ws_bytes=need, dR=FAKE + 4) == 4
    assert bwd_call(d, ws=FAKE, ws_bytes=need, dtype=7) == 3
    assert bwd_call(dims(dstate=512), ws=FAKE, ws_bytes=need) == 5
    assert dart.dart_kernel_launches() == before


def bwd_norm_call(d, eps=1e-6, **over):
    a = dict(Q=FAKE, C=FAKE, E=FAKE, dH=FAKE, R=None, lse=None, dR=FAKE, dQ=FAKE, dC=FAKE, dE=FAKE, ddH=FAKE,
             ws=None, ws_bytes=0)
    a.update(over)
    return dart.lib.dart_sma_bwd_norm(ctypes.byref(d), dart.DART_BF16, eps, a["Q"], a["C"], a["E"], a["dH"], a["R"],
                                      a["lse"], a["dR"], a["dQ"], a["dC"], a["dE"], a["ddH"], a["ws"], a["ws_bytes"],
                                      None)


def test_sma_bwd_norm_validation_statuses():
    before = dart.dart_kernel_launches()
    d = dims()
    need = dart.dart_workspace_size(dart.OP_SMA_BWD_NORM, d, dart.DART_BF16)
    need_f32 = dart.dart_workspace_size(dart.OP_SMA_BWD_NORM, d, dart.DART_F32)
    assert need_f32 >= 2 * 2 * 4 * 512 * 4 and need_f32 % 256 == 0  # recomputed lse and D for every (b, h, t)
    # bf16 at these sizes runs on the tensor cores, which also keep the weights of every (token, chunk) pair
    # (three [b, H, M, L] arrays) and the key rows as bf16 hi + lo pairs
    M = -(-d.seqlen // d.chunk)
    assert need % 256 == 0 and need >= need_f32 + 3 * 4 * d.batch * d.nheads * M * d.seqlen
    assert bwd_norm_call(d) == 6  # no workspace
    assert bwd_norm_call(d, ws=FAKE, ws_bytes=need - 1) == 6
    assert bwd_norm_call(d, eps=-1.0, ws=FAKE, ws_bytes=need) == 2
    assert bwd_norm_call(d, eps=float("inf"), ws=FAKE, ws_bytes=need) == 2
    for name in ("Q", "C", "E", "dH", "dR", "dQ", "dC", "dE", "ddH"):
        assert bwd_norm_call(d, ws=FAKE, ws_bytes=need, **{name: None}) == 1, name
    assert bwd_norm_call(d, ws=FAKE, ws_bytes=need, R=FAKE + 4) == 4  # R and lse optional, aligned when given
    assert bwd_norm_call(d, ws=FAKE, ws_bytes=need, ddH=FAKE + 8) == 4
    assert dart.dart_kernel_launches() == before


def test_grouped_e_validation_statuses():
    before = dart.dart_kernel_launches()
    d = dims()  # 4 heads
    for eg in (0, 3, 5, -1):
        assert dart.lib.dart_sma_fwd_ge(ctypes.byref(d), dart.DART_BF16, eg, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                        None) == 2, eg
        assert dart.lib.dart_sma_decode_ge(2, 4, 1, eg, 128, 64, 5, 8, dart.DART_BF16, FAKE, FAKE, FAKE, FAKE, FAKE,
                                           0, 0, FAKE, FAKE, None, FAKE, 1 << 20, None) == 2, eg
    need = dart.dart_workspace_size(dart.OP_LAYER_FWD, d, dart.DART_BF16)
    assert dart.lib.dart_layer_fwd_ge(ctypes.byref(d), dart.DART_BF16, 3, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                      0, 0, 0, FAKE, FAKE, None, FAKE, need, None) == 2
    assert dart.lib.dart_sma_fwd_ge(ctypes.byref(d), dart.DART_BF16, 2, FAKE, FAKE, None, FAKE, FAKE, None,
                                    None) == 1
    nb = dart.dart_workspace_size(dart.OP_SMA_BWD, d, dart.DART_BF16)
    for eg in (0, 3, 5, -1):
        assert dart.lib.dart_sma_bwd_ge(ctypes.byref(d), dart.DART_BF16, eg, *([FAKE] * 11), FAKE, nb, None) == 2, eg
    assert dart.lib.dart_sma_bwd_ge(ctypes.byref(d), dart.DART_BF16, 2, *([FAKE] * 10), None, FAKE, nb,
                                    None) == 1  # ddH
    assert dart.lib.dart_sma_bwd_ge(ctypes.byref(d), dart.DART_BF16, 2, *([FAKE] * 11), None, 0, None) == 6
    assert dart.dart_kernel_launches() == before
