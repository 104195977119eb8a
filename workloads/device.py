"""Device-side input generation (the counter-based cache generator) for the workloads.

``fill_cache`` writes the decode workload's chunk-memory cache straight into a
device buffer with the same SplitMix64 / Irwin-Hall(4) values that
:func:`workloads.irwin_hall_bf16` produces on the host.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

from . import DecodeWorkload, IRWIN_HALL_STD

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csrc", "gen.cu")
_LIB = os.path.join(_HERE, "libdart_workloads.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc, "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
                           "-shared", "-cudart", "static", "-o", tmp, _SRC])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _get():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.dartw_fill_irwin_hall_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                                    ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p]
        _lib.dartw_fill_irwin_hall_bf16.restype = ctypes.c_int
    return _lib


def fill_irwin_hall_bf16(ptr: int, count: int, key: int, start: int, sigma: float, stream: int = 0) -> None:
    scale = float(np.float32(sigma / IRWIN_HALL_STD))
    rc = _get().dartw_fill_irwin_hall_bf16(ctypes.c_void_p(ptr), count, key, start, scale, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"device generator failed (code {rc})")


def fill_cache(tensor, w: DecodeWorkload, key: int) -> None:
    """Fill a contiguous torch bf16 CUDA tensor [b, H, cs, N, P] with the workload's cache values."""
    import torch

    assert tensor.is_cuda and tensor.dtype == torch.bfloat16 and tensor.is_contiguous()
    stream = torch.cuda.current_stream(tensor.device).cuda_stream
    fill_irwin_hall_bf16(tensor.data_ptr(), tensor.numel(), key, 0, w.cache_sigma, stream)
