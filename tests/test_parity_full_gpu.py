"""GPU parity at the full workload sizes, in the launch configuration bench.py times.

The GPU runs the whole workload; the float64 oracle recomputes sampled (batch,
head) pairs completely (recurrence, chunk memories) and SMA on sampled tokens.
"""
import numpy as np
import pytest

import workloads as W
from _util import assert_close, assert_lse, assert_stored, layer_inputs_dev, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dart():
    import ssm_state_memory_b200 as d

    return d


def sampled_tokens(w: W.LayerWorkload, rng, extra=()):
    S, L = w.chunk, w.seqlen
    M = w.nchunks
    tok = set(extra)
    for c in (0, 1, 2, M // 2, M - 1):
        tok.update(range(c * S, min(L, c * S + 16)))
    tok.update(rng.choice(L, size=min(L, 256), replace=False).tolist())
    tok.update(range(L - 8, L))
    return np.array(sorted(tok), dtype=np.int64)


def part(st: W.Stored, b, heads=None) -> np.ndarray:
    """float64 of one batch row (and a head subset) of a stored input, without converting the rest."""
    a = st.storage[b:b + 1]
    if heads is not None:
        a = a[:, :, list(heads)]
    return W.Stored(np.ascontiguousarray(a), st.dtype).f64


def check_sampled(dart, orc, w, pairs):
    import torch

    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    out, dH, lse = dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], dv["logA"], dv["g"],
                                  inp["g_strides"], w.chunk)
    torch.cuda.synchronize()
    rng = np.random.default_rng(w.index)
    extra = inp["plant"]["queries"].tolist() if "plant" in inp else ()
    tok = sampled_tokens(w, rng, extra)
    tok_t = torch.as_tensor(tok, device=out.device)
    assert w.ngroups == 1
    g_dense = W.gate_dense(inp["g"], inp["g_strides"], w.batch, w.seqlen, w.nheads)
    for b, hs in pairs:
        hs = list(hs)
        X = part(inp["X"], b, hs)
        B = part(inp["B"], b)
        C = part(inp["C"], b)
        Q = part(inp["Q"], b)
        E = part(inp["E"], b, hs)
        logA = inp["logA"][b:b + 1][:, :, hs]
        gsel = np.ascontiguousarray(g_dense[b:b + 1][:, :, hs])
        H = len(hs)
        ref = orc.layer(X, B, C, Q, E, logA, gsel, (w.seqlen * H, H, 1), w.chunk, sma_tokens=tok)
        assert_stored(to_f64(dH[b, hs]), ref["dH"][0], w.dtype, f"dH b={b}")
        assert_close(to_f64(dH[b, hs]), ref["dH"][0], w.dtype, f"dH b={b} (per-tensor bound)")
        assert_close(to_f64(out[b][tok_t][:, hs]), ref["out"][0], w.dtype, f"out b={b}")
        assert_lse(to_f64(lse[b][hs][:, tok_t]), ref["lse"][0], w.dtype, f"lse b={b}")


def test_m370m_bf16_workload_sampled(dart, orc):
    check_sampled(dart, orc, W.M370M_BF16, [(0, (0, 13)), (3, (7, 31))])


def test_long_bf16_workload_sampled(dart, orc):
    check_sampled(dart, orc, W.LONG_BF16, [(0, (0, 19))])


def test_m370m_bf16_normalised_branch_sampled(dart, orc):
    """dart_sma_fwd_norm (App. B.1) at the full 8192-token workload in its launch configuration.

    Both sides read the oracle's chunk memories rounded once to bf16; the oracle recomputes the
    normalised SMA on sampled tokens of sampled (batch, head) pairs."""
    import torch

    w = W.M370M_BF16
    eps = 1e-6
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    dH_in = W.store(orc.chunk_states(inp["X"].f64, inp["B"].f64, inp["logA"], w.chunk), w.dtype)
    dH_dev = to_dev(dH_in)
    R, lse = dart.sma_fwd(dv["Q"], dv["C"], dv["E"], dH_dev, w.chunk, norm_eps=eps)
    torch.cuda.synchronize()
    rng = np.random.default_rng(w.index + 7)
    tok = sampled_tokens(w, rng)
    tok_t = torch.as_tensor(tok, device=R.device)
    dH64 = dH_in.f64
    for b, hs in [(0, (0, 13)), (3, (7, 31))]:
        hs = list(hs)
        R_ref, lse_ref = orc.sma(part(inp["Q"], b), part(inp["C"], b), part(inp["E"], b, hs),
                                 np.ascontiguousarray(dH64[b:b + 1][:, hs]), w.chunk, tokens=tok, norm_eps=eps)
        assert_close(to_f64(R[b][tok_t][:, hs]), R_ref[0], w.dtype, f"normalised R b={b}")
        assert_lse(to_f64(lse[b][hs][:, tok_t]), lse_ref[0], w.dtype, f"normalised lse b={b}")


def test_m370m_bf16_backward_sampled(dart, orc):
    """dart_sma_bwd at the full 8192-token workload, in the launch configuration bench.py times.

    Both sides read the oracle's chunk memories rounded once to bf16 and a seeded dR; the GPU also takes
    R and lse from its own forward, as a caller would (the oracle recomputes its weights). The oracle
    recomputes the per-token gradients of sampled tokens (every head) and the gradients of a few chunk
    memories (every later token)."""
    import torch

    w = W.M370M_BF16
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    dH_in = W.store(orc.chunk_states(inp["X"].f64, inp["B"].f64, inp["logA"], w.chunk), w.dtype)
    dH_dev = to_dev(dH_in)
    dR = W.make_readout_grad(w)
    R, lse = dart.sma_fwd(dv["Q"], dv["C"], dv["E"], dH_dev, w.chunk)
    dQ, dC, dE, ddH = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, R, lse, torch.from_numpy(dR).cuda(), w.chunk)
    torch.cuda.synchronize()
    del R, lse
    rng = np.random.default_rng(w.index + 11)
    tok = np.unique(np.concatenate([rng.choice(w.seqlen, 96, replace=False), [0, 255, 256, 257, 4095, 8191]]))
    Qf, Cf, Ef = inp["Q"].f64, inp["C"].f64, inp["E"].f64
    dH64 = dH_in.f64
    for b in (0, 3):
        sl = slice(b, b + 1)
        ref = orc.sma_bwd_tokens(Qf[sl], Cf[sl], Ef[sl], dH64[sl], dR[sl].astype(np.float64), w.chunk, tok)
        tt = torch.as_tensor(tok, device=dQ.device)
        assert_close(to_f64(dQ[b][tt]), ref["dQ"][0], w.dtype, f"dQ b={b}")
        assert_close(to_f64(dC[b][tt]), ref["dC"][0], w.dtype, f"dC b={b}")
        assert_close(to_f64(dE[b][tt]), ref["dE"][0], w.dtype, f"dE b={b}")
    trip = [(0, 0, 0), (3, 31, 15), (1, 7, 30), (2, 12, 31)]
    ref = orc.sma_bwd_ddh(Qf, Cf, Ef, dH64, dR.astype(np.float64), w.chunk, trip)
    for i, (b, h, c) in enumerate(trip):
        got = to_f64(ddH[b, h, c])
        if c == w.nchunks - 1:  # the last chunk memory has no later token
            assert np.all(got == 0.0) and np.all(ref[i] == 0.0)
        else:
            assert_close(got, ref[i], w.dtype, f"ddH b={b} h={h} c={c}")


def test_m370m_bf16_normalised_backward_sampled(dart, orc):
    """dart_sma_bwd_norm (App. B.1) at the full 8192-token workload on the tensor cores, in the launch
    configuration bench.py times: sampled tokens of two batch rows (every head) and four chunk memories
    against the oracle's normalised backward at those places, on the oracle's chunk memories rounded once to
    bf16 and a seeded dR."""
    import torch

    w = W.M370M_BF16
    eps = 1e-6
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    dH_in = W.store(orc.chunk_states(inp["X"].f64, inp["B"].f64, inp["logA"], w.chunk), w.dtype)
    dH_dev = to_dev(dH_in)
    dR = W.make_readout_grad(w)
    dQ, dC, dE, ddH = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, None, None, torch.from_numpy(dR).cuda(),
                                   w.chunk, norm_eps=eps)
    torch.cuda.synchronize()
    rng = np.random.default_rng(w.index + 13)
    tok = np.unique(np.concatenate([rng.choice(w.seqlen, 48, replace=False), [0, 255, 256, 4095, 8191]]))
    Qf, Cf, Ef = inp["Q"].f64, inp["C"].f64, inp["E"].f64
    dH64 = dH_in.f64
    for b in (0, 3):
        sl = slice(b, b + 1)
        ref = orc.sma_bwd_tokens(Qf[sl], Cf[sl], Ef[sl], dH64[sl], dR[sl].astype(np.float64), w.chunk, tok,
                                 norm_eps=eps)
        tt = torch.as_tensor(tok, device=dQ.device)
        assert_close(to_f64(dQ[b][tt]), ref["dQ"][0], w.dtype, f"normalised dQ b={b}")
        assert_close(to_f64(dC[b][tt]), ref["dC"][0], w.dtype, f"normalised dC b={b}")
        assert_close(to_f64(dE[b][tt]), ref["dE"][0], w.dtype, f"normalised dE b={b}")
    trip = [(0, 0, 0), (3, 31, 15), (1, 7, 29), (2, 12, 31)]
    ref = orc.sma_bwd_ddh(Qf, Cf, Ef, dH64, dR.astype(np.float64), w.chunk, trip, norm_eps=eps)
    for i, (b, h, c) in enumerate(trip):
        got = to_f64(ddH[b, h, c])
        if c == w.nchunks - 1:  # the last chunk memory has no later token
            assert np.all(got == 0.0) and np.all(ref[i] == 0.0)
        else:
            assert_close(got, ref[i], w.dtype, f"normalised ddH b={b} h={h} c={c}")
