"""dart_sma_decode_noalloc: the decode entry point for callers that cannot allocate.

Some callers only hold the input and output buffers a host framework gave them
and may not allocate device memory (e.g. a plug-in whose serving threads must not
call cudaMalloc). This entry point keeps its scratch in a fixed array inside the
library. These tests call it through the C ABI twice in a row and compare each
call with the float64 oracle and with dart_sma_decode, which takes a
caller-provided workspace. The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import workloads as W
from _util import assert_close, assert_lse, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _inputs(rng, Bt, H, G, N, P, cs, dt):
    Q = W.store(rng.standard_normal((Bt, G, N)) / np.sqrt(N) * 3, dt)
    C = W.store(rng.standard_normal((Bt, G, N)) / np.sqrt(N), dt)
    E = W.store(rng.standard_normal((Bt, H, P)) / np.sqrt(P) * 3, dt)
    Y = W.store(rng.standard_normal((Bt, H, P)) / np.sqrt(P), dt)
    cache = W.store(rng.standard_normal((Bt, H, cs, N, P)) * 0.03, dt)
    g = rng.uniform(size=(Bt, H)).astype(np.float32)
    host = [x.f64 for x in (Q, C, E, Y)] + [g.astype(np.float64), cache.f64]
    return [to_dev(x) for x in (Q, C, E, Y)], to_dev(g), to_dev(cache), host


@pytest.mark.parametrize("dt,Bt,H,G,N,P,n,cs", [
    ("bf16", 8, 32, 1, 128, 64, 256, 256),
    ("bf16", 3, 4, 2, 64, 32, 37, 40),
    ("f32", 2, 4, 1, 16, 8, 9, 9),
])
def test_noalloc_decode_matches_oracle_and_workspace_decode(orc, dt, Bt, H, G, N, P, n, cs):
    import torch

    import ssm_state_memory_b200 as dart

    rng = np.random.default_rng(11)
    (Q, C, E, Y), g, cache, host = _inputs(rng, Bt, H, G, N, P, cs, dt)
    orc_out, orc_lse = orc.decode(*host[:5], (H, 1), host[5], n_chunks=n)
    ws_out, ws_lse = dart.sma_decode(Q, C, E, Y, g, (H, 1), cache, n_chunks=n)
    for _ in range(2):  # the shared scratch keeps the previous call's contents
        out = torch.full((Bt, H, P), float("nan"), device="cuda")
        lse = torch.full((Bt, H), float("nan"), device="cuda")
        dart.dart_sma_decode_noalloc(n, Q, C, E, Y, g, (H, 1), cache, out, lse)
        torch.cuda.synchronize()
        assert_close(to_f64(out), orc_out, dt, "noalloc decode out vs oracle")
        assert_lse(to_f64(lse), orc_lse, dt, "noalloc decode lse vs oracle")
        assert_close(to_f64(out), to_f64(ws_out), dt, "noalloc decode out vs dart_sma_decode")
        assert_lse(to_f64(lse), to_f64(ws_lse), dt, "noalloc decode lse vs dart_sma_decode")


def test_noalloc_decode_rejects_sizes_beyond_its_scratch():
    import torch

    import ssm_state_memory_b200 as dart

    # 64 x 512 heads x splits x (2 + 64) x 4 bytes is far above the 4 MiB array
    Bt, H, N, P, n = 64, 512, 128, 64, 256
    need = dart.dart_decode_workspace_size(Bt, H, N, P, n, dart.DART_BF16)
    assert need > (4 << 20)
    before = dart.dart_kernel_launches()
    q = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    p = q.data_ptr()
    st = dart.lib.dart_sma_decode_noalloc(Bt, H, 1, N, P, n, n, dart.DART_BF16, p, p, p, p, p, 0, 0, p, p, None,
                                          None)
    assert st == 6  # DART_ERR_WORKSPACE, nothing launched
    assert dart.dart_kernel_launches() == before
