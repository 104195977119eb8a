"""GPU parity of dart_sma_decode (single new token over cached chunk memories)."""
import numpy as np
import pytest

import workloads as W
import workloads.device as WD
from _util import assert_close, assert_lse, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dart():
    import ssm_state_memory_b200 as d

    return d


def test_device_generator_matches_host():
    import torch

    w = W.DECODE_BF16.with_(batch=2, nheads=3, n_chunks=5)
    key = W.cache_key(99)
    cache = torch.empty((2, 3, 5, 128, 64), dtype=torch.bfloat16, device="cuda")
    WD.fill_cache(cache, w, key)
    host = W.decode_cache_slice(w, key, 1, 2).storage
    dev = cache[1, 2].view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(dev, host)


def test_decode_full_workload_sampled(dart, orc):
    import torch

    w = W.DECODE_BF16
    inp = W.make_decode_inputs(w)
    cache = torch.empty((w.batch, w.nheads, w.n_chunks, w.dstate, w.headdim), dtype=torch.bfloat16, device="cuda")
    WD.fill_cache(cache, w, inp["key"])
    dv = {k: to_dev(inp[k]) for k in ("Q", "C", "E", "Y")}
    g = to_dev(inp["g"])
    out, lse = dart.sma_decode(dv["Q"], dv["C"], dv["E"], dv["Y"], g, inp["g_strides"], cache)
    torch.cuda.synchronize()
    for b, h in [(0, 0), (17, 5), (63, 31), (40, 12)]:
        mem = W.decode_cache_slice(w, inp["key"], b, h).f64[None, None]
        ref_out, ref_lse = orc.decode(inp["Q"].f64[b:b + 1], inp["C"].f64[b:b + 1], inp["E"].f64[b:b + 1, h:h + 1],
                                      inp["Y"].f64[b:b + 1, h:h + 1], inp["g"], (0, 0), mem)
        assert_close(to_f64(out[b, h]), ref_out[0, 0], "bf16", f"decode out ({b},{h})")
        assert_lse(to_f64(lse[b, h:h + 1]), ref_lse[0], "bf16", f"decode lse ({b},{h})")
    del cache
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dt,N,P,n,cs,G", [
    ("bf16", 128, 64, 7, 9, 1),    # capacity larger than the filled part
    ("f32", 16, 8, 33, 33, 1),     # fp32 cache, 16-byte rows of 2 vectors
    ("bf16", 64, 32, 300, 300, 2), # many chunks, 2 groups
    ("f32", 128, 64, 1, 1, 1),     # a single chunk: softmax weight 1
])
def test_decode_small(dart, orc, dt, N, P, n, cs, G):
    import torch

    rng = np.random.default_rng(5)
    Bt, H = 3, 4
    Q = W.store(rng.standard_normal((Bt, G, N)) / np.sqrt(N) * 4, dt)
    C = W.store(rng.standard_normal((Bt, G, N)) / np.sqrt(N), dt)
    E = W.store(rng.standard_normal((Bt, H, P)) / np.sqrt(P) * 4, dt)
    Y = W.store(rng.standard_normal((Bt, H, P)) / np.sqrt(P), dt)
    cache = W.store(rng.standard_normal((Bt, H, cs, N, P)) * 0.3, dt)
    g = rng.uniform(size=(Bt, H)).astype(np.float32)
    out, lse = dart.sma_decode(to_dev(Q), to_dev(C), to_dev(E), to_dev(Y), to_dev(g), (H, 1), to_dev(cache),
                               n_chunks=n)
    ref_out, ref_lse = orc.decode(Q.f64, C.f64, E.f64, Y.f64, g, (H, 1), cache.f64, n_chunks=n)
    assert_close(to_f64(out), ref_out, dt, "decode out")
    assert_lse(to_f64(lse), ref_lse, dt, "decode lse")


def test_decode_without_history_returns_Y(dart):
    import torch

    Q = torch.randn(2, 1, 128, device="cuda").bfloat16()
    E = torch.randn(2, 4, 64, device="cuda").bfloat16()
    Y = torch.randn(2, 4, 64, device="cuda").bfloat16()
    cache = torch.randn(2, 4, 3, 128, 64, device="cuda").bfloat16()
    g = torch.ones(1, device="cuda")
    out, lse = dart.sma_decode(Q, Q, E, Y, g, (0, 0), cache, n_chunks=0)
    assert torch.equal(out, Y.float())
    assert torch.all(torch.isneginf(lse))
