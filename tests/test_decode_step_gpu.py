"""GPU parity of dart_decode_step: a sequence decoded token by token against the parallel forward.

The float64 oracle runs the whole sequence in parallel (recurrence, direct-sum chunk memories, SMA,
combine). The GPU decodes the same tokens one call per token, carrying the recurrent state, the open
chunk's memory and the chunk-memory cache between calls. Every token's out and lse, every chunk memory
the steps append, and the final state must match within the dtype's tolerance.
"""
import numpy as np
import pytest

import workloads as W
from _util import assert_close, assert_lse, assert_stored, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dart():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import ssm_state_memory_b200 as d

    return d


def token_slice(st: W.Stored, t: int) -> W.Stored:
    return W.Stored(np.ascontiguousarray(st.storage[:, t]), st.dtype)


def decode_sequence(dart, orc, w: W.LayerWorkload):
    import torch

    inp = W.make_layer_inputs(w)
    X, B, C, Q, E = (inp[k].f64 for k in "XBCQE")
    ref = orc.layer(X, B, C, Q, E, inp["logA"], inp["g"], inp["g_strides"], w.chunk)
    Bt, L, H, P, N, S = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.chunk
    M = w.nchunks
    gd = W.gate_dense(inp["g"], inp["g_strides"], Bt, L, H)  # [Bt, L, H]
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    state = torch.zeros(Bt, H, N, P, device="cuda")
    acc = torch.zeros_like(state)
    cache = torch.zeros(Bt, H, M, N, P, device="cuda", dtype=tdt)
    outs, lses = [], []
    for t in range(L):
        dv = {k: to_dev(token_slice(inp[k], t)) for k in "XBCQE"}
        logA_t = to_dev(np.ascontiguousarray(inp["logA"][:, t]))
        g_t = to_dev(np.ascontiguousarray(gd[:, t]))
        out, lse = dart.decode_step(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], logA_t, g_t, (H, 1), state, acc,
                                    cache, t // S, (t + 1) % S == 0)
        outs.append(out)
        lses.append(lse)
    torch.cuda.synchronize()
    dt = w.dtype
    assert_close(to_f64(torch.stack(outs, 1)), ref["out"], dt, "decode steps: out")
    assert_lse(to_f64(torch.stack(lses, 2)), ref["lse"], dt, "decode steps: lse")
    nfull = L // S
    if nfull:
        assert_stored(to_f64(cache[:, :, :nfull]), ref["dH"][:, :, :nfull], dt, "decode steps: appended chunk memories")
    assert_close(to_f64(state), ref["Hfinal"], dt, "decode steps: final state")
    if L % S:
        assert_close(to_f64(acc), ref["dH"][:, :, nfull], dt, "decode steps: open chunk memory")
    else:
        assert torch.count_nonzero(acc) == 0


@pytest.mark.parametrize("shape", [
    # (batch, L, H, G, N, P, S, dtype)
    (2, 3 * 64 + 17, 4, 1, 128, 64, 64, "bf16"),   # the tensor-core state shape, ragged last chunk
    (2, 70, 4, 2, 16, 8, 16, "f32"),               # small fp32 shape, two groups
    (1, 2 * 128, 2, 1, 64, 128, 128, "bf16"),      # P = 128, chunks close exactly at the end
])
def test_decode_steps_reproduce_the_parallel_forward(dart, orc, shape):
    Bt, L, H, G, N, P, S, dt = shape
    w = W.LayerWorkload("decode_steps", 11, Bt, H, G, L, S, N, P, dt, "mamba2", "per_head_uniform")
    decode_sequence(dart, orc, w)


def test_first_token_sees_no_history(dart):
    """n_chunks = 0: out = Y = C (B^T X) for a zero state, lse = -inf, and nothing is appended."""
    import torch

    torch.manual_seed(0)
    b, H, G, N, P = 2, 4, 1, 128, 64
    X = torch.randn(b, H, P, device="cuda").bfloat16()
    B = torch.randn(b, G, N, device="cuda").bfloat16()
    C = torch.randn(b, G, N, device="cuda").bfloat16()
    Q = torch.randn(b, G, N, device="cuda").bfloat16()
    E = torch.randn(b, H, P, device="cuda").bfloat16()
    logA = -torch.rand(b, H, device="cuda")
    g = torch.full((b, H), 0.5, device="cuda")
    state = torch.zeros(b, H, N, P, device="cuda")
    acc = torch.zeros_like(state)
    cache = torch.zeros(b, H, 2, N, P, device="cuda", dtype=torch.bfloat16)
    out, lse = dart.decode_step(X, B, C, Q, E, logA, g, (H, 1), state, acc, cache, 0, False)
    outer = B.float()[:, 0, None, :, None] * X.float()[:, :, None, :]  # [b, H, N, P]
    y = torch.einsum("bn,bhnp->bhp", C.float()[:, 0], outer)
    torch.testing.assert_close(out, y, rtol=1e-5, atol=1e-4)
    assert torch.all(torch.isneginf(lse))
    torch.testing.assert_close(state, outer, rtol=0, atol=0)
    torch.testing.assert_close(acc, outer, rtol=0, atol=0)
    assert torch.count_nonzero(cache) == 0
