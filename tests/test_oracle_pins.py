"""Pins of the float64 oracle against what the DART paper and plain mathematics fix.

None of these compares the oracle with itself: each check is a closed form, an
identity between two different oracle code paths that the paper states, a
special case that reduces to a library routine (numpy matmul, scipy softmax /
logsumexp), or brute force over an explicit matrix on tiny inputs. The
mutation tests at the bottom plant a plausible mistake in a copy of the oracle
source and check that some pin catches it.
"""
import math
import os
import re
import shutil
import subprocess

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle

RTOL = 1e-11


def rand_case(seed, Bt=2, L=48, H=2, G=1, N=4, P=3, S=16, decay=0.3):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((Bt, L, H, P))
    B = rng.standard_normal((Bt, L, G, N))
    C = rng.standard_normal((Bt, L, G, N))
    Q = rng.standard_normal((Bt, L, G, N))
    E = rng.standard_normal((Bt, L, H, P))
    logA = -np.abs(rng.standard_normal((Bt, L, H))) * decay
    return dict(X=X, B=B, C=C, Q=Q, E=E, logA=logA, S=S)


def close(a, b, rtol=RTOL):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    np.testing.assert_allclose(a, b, rtol=0, atol=rtol * scale)


def grp(H, G, h):
    return h // (H // G)


# ---------------------------------------------------------------------------
# recurrence, eq (2)
# ---------------------------------------------------------------------------


def check_quadratic_form(orc, case):
    """Eq (4): Y = (L_SSD o C B^T) X with L_SSD[i, j] = prod_{k=j+1}^{i} a_k (i >= j), 0 above."""
    X, B, C, logA, S = case["X"], case["B"], case["C"], case["logA"], case["S"]
    Y, _, _ = orc.recurrence(X, B, C, logA, S)
    Bt, L, H, P = X.shape
    G = B.shape[2]
    for b in range(Bt):
        for h in range(H):
            g = grp(H, G, h)
            a = np.exp(logA[b, :, h])
            Lm = np.zeros((L, L))
            for i in range(L):
                for j in range(i + 1):
                    Lm[i, j] = np.prod(a[j + 1:i + 1])  # empty product = 1 on the diagonal
            Yq = (Lm * (C[b, :, g] @ B[b, :, g].T)) @ X[b, :, h]
            close(Y[b, :, h], Yq)


@pytest.mark.parametrize("seed,G,H", [(0, 1, 2), (1, 2, 4)])
def test_recurrence_equals_quadratic_ssd_form(orc, seed, G, H):
    check_quadratic_form(orc, rand_case(seed, G=G, H=H, L=40))


def test_recurrence_without_decay_is_causal_linear_attention(orc):
    c = rand_case(2, L=37)
    c["logA"][:] = 0.0
    Y, _, _ = orc.recurrence(c["X"], c["B"], c["C"], c["logA"], c["S"])
    for b in range(2):
        for h in range(2):
            ref = np.tril(c["C"][b, :, 0] @ c["B"][b, :, 0].T) @ c["X"][b, :, h]
            close(Y[b, :, h], ref)


def test_recurrence_with_full_forgetting_keeps_only_the_current_token(orc):
    c = rand_case(3, L=20)
    c["logA"][:] = -np.inf  # a_t = 0
    Y, _, _ = orc.recurrence(c["X"], c["B"], c["C"], c["logA"], c["S"])
    ref = np.einsum("bln,bln->bl", c["C"][:, :, 0], c["B"][:, :, 0])[:, :, None, None] * c["X"]
    close(Y, ref)


# ---------------------------------------------------------------------------
# chunk state memories, eq (5) / App. A eq (18)-(20)
# ---------------------------------------------------------------------------


def check_chunk_identity(orc, case):
    """App. A eq (18): H_[c] = A_{a_c:b_c} H_[c-1] + dH[c]; recurrence ends vs direct sums."""
    X, B, C, logA, S = case["X"], case["B"], case["C"], case["logA"], case["S"]
    _, Hend, _ = orc.recurrence(X, B, C, logA, S)
    dH = orc.chunk_states(X, B, logA, S)
    Bt, L, H, P = X.shape
    M = dH.shape[2]
    for b in range(Bt):
        for h in range(H):
            prev = np.zeros(dH.shape[3:])
            for c in range(M):
                decay = math.exp(float(np.sum(logA[b, c * S:min(L, (c + 1) * S), h])))
                close(Hend[b, h, c], decay * prev + dH[b, h, c])
                prev = Hend[b, h, c]


@pytest.mark.parametrize("L,S", [(48, 16), (53, 16), (16, 16), (7, 16)])
def test_chunk_identity(orc, L, S):
    check_chunk_identity(orc, rand_case(4, L=L, S=S))


def test_chunk_states_without_decay_are_plain_products(orc):
    c = rand_case(5, L=45, S=16)
    c["logA"][:] = 0.0
    dH = orc.chunk_states(c["X"], c["B"], c["logA"], 16)
    for b in range(2):
        for h in range(2):
            for ch in range(3):
                sl = slice(ch * 16, min(45, (ch + 1) * 16))
                close(dH[b, h, ch], c["B"][b, sl, 0].T @ c["X"][b, sl, h])


def test_single_token_chunks_are_outer_products(orc):
    c = rand_case(6, L=9, S=1)
    dH = orc.chunk_states(c["X"], c["B"], c["logA"], 1)
    ref = np.einsum("bln,blhp->bhlnp", c["B"][:, :, 0], c["X"])
    close(dH, ref)


def test_chunked_output_decomposition(orc):
    """App. A eq (19)-(22): Y_t = intra (zero initial state) + C_t A_{a_c:t} H_[c-1]."""
    c = rand_case(7, L=50, S=16, H=1)
    X, B, C, logA, S = c["X"], c["B"], c["C"], c["logA"], c["S"]
    Y, Hend, _ = orc.recurrence(X, B, C, logA, S)
    for b in range(2):
        for t in range(50):
            ch = t // S
            first = ch * S
            intra = np.zeros(3)
            for s in range(first, t + 1):
                w = math.exp(float(np.sum(logA[b, s + 1:t + 1, 0])))
                intra += (C[b, t, 0] @ B[b, s, 0]) * w * X[b, s, 0]
            inter = np.zeros(3)
            if ch > 0:
                w = math.exp(float(np.sum(logA[b, first:t + 1, 0])))
                inter = w * (C[b, t, 0] @ Hend[b, 0, ch - 1])
            close(Y[b, t, 0], intra + inter)


# ---------------------------------------------------------------------------
# state-memory attention, eq (8)-(10)
# ---------------------------------------------------------------------------


def sma_case(seed, L=64, S=16, N=4, P=3, H=2, G=1, Bt=2):
    c = rand_case(seed, Bt=Bt, L=L, H=H, G=G, N=N, P=P, S=S)
    rng = np.random.default_rng(seed + 100)
    M = -(-L // S)
    c["dH"] = rng.standard_normal((Bt, H, M, N, P))
    return c


def check_first_chunk(orc, c):
    R, lse = orc.sma(c["Q"], c["C"], c["E"], c["dH"], c["S"])
    S = c["S"]
    assert np.all(R[:, :S] == 0.0)
    assert np.all(np.isneginf(lse[:, :, :S]))
    assert np.all(np.isfinite(lse[:, :, S:]))


def test_first_chunk_has_zero_readout_and_minus_inf_lse(orc):
    check_first_chunk(orc, sma_case(10))


def check_single_history(orc, c):
    """Tokens of chunk 1 see one memory: softmax weight 1, R_t = C_t dH[0], lse = l_{t,0}."""
    Q, C, E, dH, S = c["Q"], c["C"], c["E"], c["dH"], c["S"]
    R, lse = orc.sma(Q, C, E, dH, S)
    Bt, L, H, P = E.shape
    G, N = Q.shape[2], Q.shape[3]
    for b in range(Bt):
        for h in range(H):
            g = grp(H, G, h)
            for t in range(S, 2 * S):
                close(R[b, t, h], C[b, t, g] @ dH[b, h, 0])
                close(lse[b, h, t], (Q[b, t, g] @ dH[b, h, 0] @ E[b, t, h]) / math.sqrt(N))


def test_single_historical_chunk(orc):
    check_single_history(orc, sma_case(11, N=5, P=3, G=2, H=4))


def test_zero_query_gives_uniform_weights(orc):
    c = sma_case(12)
    c["Q"][:] = 0.0
    R, lse = orc.sma(c["Q"], c["C"], c["E"], c["dH"], c["S"])
    S = c["S"]
    for b in range(2):
        for h in range(2):
            for t in range(S, 64):
                k = t // S
                close(R[b, t, h], c["C"][b, t, 0] @ c["dH"][b, h, :k].mean(axis=0))
                close(lse[b, h, t], math.log(k))


def check_brute_force(orc, c):
    """Explicit logits matrix [L, M] (einsum), masked, normalised with scipy softmax/logsumexp."""
    Q, C, E, dH, S = c["Q"], c["C"], c["E"], c["dH"], c["S"]
    R, lse = orc.sma(Q, C, E, dH, S)
    Bt, L, H, P = E.shape
    G, N = Q.shape[2], Q.shape[3]
    M = dH.shape[2]
    for b in range(Bt):
        for h in range(H):
            g = grp(H, G, h)
            logits = np.einsum("tn,cnp,tp->tc", Q[b, :, g], dH[b, h], E[b, :, h]) / math.sqrt(N)
            V = np.einsum("tn,cnp->tcp", C[b, :, g], dH[b, h])
            hist = (np.arange(M)[None, :] < (np.arange(L) // S)[:, None])
            for t in range(L):
                k = int(hist[t].sum())
                if k == 0:
                    continue
                w = softmax(logits[t, :k])
                close(R[b, t, h], w @ V[t, :k])
                close(lse[b, h, t], logsumexp(logits[t, :k]))


@pytest.mark.parametrize("L,S", [(64, 16), (61, 8)])
def test_sma_brute_force(orc, L, S):
    c = sma_case(13, L=L, S=S)
    c["Q"] *= 3.0  # spread the logits so the softmax is far from uniform
    check_brute_force(orc, c)


def test_sampled_tokens_match_dense_rows(orc):
    c = sma_case(14, L=70, S=8)
    R, lse = orc.sma(c["Q"], c["C"], c["E"], c["dH"], c["S"])
    tok = [0, 7, 8, 33, 69]
    Rs, ls = orc.sma(c["Q"], c["C"], c["E"], c["dH"], c["S"], tokens=tok)
    np.testing.assert_array_equal(Rs, R[:, tok])
    np.testing.assert_array_equal(ls, lse[:, :, tok])


# ---------------------------------------------------------------------------
# combine, eq (11), and decode
# ---------------------------------------------------------------------------


def check_combine(orc):
    rng = np.random.default_rng(20)
    Y = rng.standard_normal((2, 5, 3, 4))
    R = rng.standard_normal((2, 5, 3, 4))
    out0 = orc.combine(Y, R, np.zeros(1), (0, 0, 0))
    np.testing.assert_array_equal(out0, Y)  # W_G = 0 at init: pure Mamba-2 output
    gd = rng.uniform(size=(2, 5, 3))
    out = orc.combine(Y, R, gd, (15, 3, 1))
    close(out, Y + gd[..., None] * R)
    gh = rng.uniform(size=3)
    out = orc.combine(Y, R, gh, (0, 0, 1))
    close(out, Y + gh[None, None, :, None] * R)


def test_combine(orc):
    check_combine(orc)


def test_decode_matches_last_chunk_token_and_permutation(orc):
    rng = np.random.default_rng(21)
    Bt, H, G, N, P, cs = 2, 4, 2, 5, 3, 7
    Q = rng.standard_normal((Bt, G, N)) * 3
    C = rng.standard_normal((Bt, G, N))
    E = rng.standard_normal((Bt, H, P))
    Y = rng.standard_normal((Bt, H, P))
    g = rng.uniform(size=(Bt * H,))
    cache = rng.standard_normal((Bt, H, cs, N, P))
    n = 6
    out, lse = orc.decode(Q, C, E, Y, g, (H, 1), cache, n_chunks=n)
    # the same token placed in chunk n of an S=2 sequence sees exactly chunks 0..n-1
    S, L = 2, 2 * n + 1
    Qs = np.zeros((Bt, L, G, N)); Qs[:, -1] = Q
    Cs = np.zeros((Bt, L, G, N)); Cs[:, -1] = C
    Es = np.zeros((Bt, L, H, P)); Es[:, -1] = E
    R, lse2 = orc.sma(Qs, Cs, Es, cache[:, :, :n + 1], S, tokens=[L - 1])
    close(lse, lse2[:, :, 0])
    close(out, Y + g.reshape(Bt, H)[..., None] * R[:, 0])
    perm = rng.permutation(n)
    cache_p = cache.copy()
    cache_p[:, :, :n] = cache[:, :, perm]
    out_p, lse_p = orc.decode(Q, C, E, Y, g, (H, 1), cache_p, n_chunks=n)
    close(out_p, out)
    close(lse_p, lse)
    out_0, lse_0 = orc.decode(Q, C, E, Y, g, (H, 1), cache, n_chunks=0)
    np.testing.assert_array_equal(out_0, Y)
    assert np.all(np.isneginf(lse_0))


def test_cache_ratio_eq14():
    """Eq (14) with the paper's worked example, from the decode workload's real buffer sizes."""
    import workloads as W

    gold = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "cache_ratio_eq14.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()
                gold[k] = float(v)
    w = W.DECODE_BF16
    assert (w.chunk, w.dstate) == (gold["S"], gold["N"])
    itemsize = 2  # bf16 for both caches
    L = w.n_chunks * w.chunk
    dart_bytes = w.batch * w.nheads * w.n_chunks * w.dstate * w.headdim * itemsize
    kv_bytes = w.batch * w.nheads * L * 2 * w.headdim * itemsize
    assert dart_bytes == 8_589_934_592
    assert dart_bytes / kv_bytes == gold["ratio"] == w.dstate / (2 * w.chunk)
    assert 1.0 - dart_bytes / kv_bytes == gold["saving"]


def test_layer_composes_the_pieces(orc):
    c = rand_case(22, L=40, S=8)
    g = np.array([0.7]); gs = (0, 0, 0)
    res = orc.layer(c["X"], c["B"], c["C"], c["Q"], c["E"], c["logA"], g, gs, 8)
    Y, _, _ = orc.recurrence(c["X"], c["B"], c["C"], c["logA"], 8)
    dH = orc.chunk_states(c["X"], c["B"], c["logA"], 8)
    R, lse = orc.sma(c["Q"], c["C"], c["E"], dH, 8)
    close(res["out"], Y + 0.7 * R)
    sub = orc.layer(c["X"], c["B"], c["C"], c["Q"], c["E"], c["logA"], g, gs, 8, sma_tokens=[3, 17, 39])
    close(sub["out"], res["out"][:, [3, 17, 39]])


def check_decode_steps(orc, c, g=0.6):
    """Decoding a sequence token by token, with the recurrent state and the open chunk's memory carried
    across steps and each closed chunk appended to the cache, reproduces the parallel forward: every
    token's out and lse, every chunk memory (direct sums, eq 5) and the final state (eq 2)."""
    X, B, C, Q, E, logA, S = (c[k] for k in ("X", "B", "C", "Q", "E", "logA", "S"))
    Bt, L, H, P = X.shape
    G, N = B.shape[2], B.shape[3]
    ref = orc.layer(X, B, C, Q, E, logA, np.array([g]), (0, 0, 0), S)
    M = -(-L // S)
    state = np.zeros((Bt, H, N, P))
    acc = np.zeros_like(state)
    cache = np.zeros((Bt, H, M, N, P))
    outs, lses = [], []
    for t in range(L):
        out, lse = orc.decode_step(X[:, t], B[:, t], C[:, t], Q[:, t], E[:, t], logA[:, t], np.array([g]), (0, 0),
                                   state, acc, cache, t // S, (t + 1) % S == 0)
        outs.append(out)
        lses.append(lse)
    close(np.stack(outs, 1), ref["out"])
    lse_steps = np.stack(lses, 2)
    np.testing.assert_array_equal(np.isneginf(lse_steps), np.isneginf(ref["lse"]))
    fin = np.isfinite(ref["lse"])
    close(lse_steps[fin], ref["lse"][fin])
    nfull = L // S
    close(cache[:, :, :nfull], ref["dH"][:, :, :nfull])
    close(state, ref["Hfinal"])
    if L % S:  # the open chunk's memory is the partial chunk's direct sum
        close(acc, ref["dH"][:, :, nfull])
    else:
        np.testing.assert_array_equal(acc, 0.0)


@pytest.mark.parametrize("L,S,G,H", [(40, 8, 1, 2), (37, 8, 2, 4)])
def test_decode_steps_reproduce_the_parallel_forward(orc, L, S, G, H):
    c = rand_case(40 + L, L=L, S=S, G=G, H=H)
    c["Q"] *= 2.0
    check_decode_steps(orc, c)


# ---------------------------------------------------------------------------
# normalised score branch, App. B.1 eq (25)-(27)
# ---------------------------------------------------------------------------


def unit_rms(x, axis):
    return x / np.sqrt(np.mean(x ** 2, axis=axis, keepdims=True))


def check_norm_reduces_to_plain(orc, c):
    """With eps = 0 and Q_t, E_t and every memory row already of unit RMS, the normalised branch is the
    plain SMA of eq (8)-(10) (pinned separately above)."""
    Q, E, dH = unit_rms(c["Q"], 3), unit_rms(c["E"], 3), unit_rms(c["dH"], 4)
    R0, l0 = orc.sma(Q, c["C"], E, dH, c["S"])
    R1, l1 = orc.sma(Q, c["C"], E, dH, c["S"], norm_eps=0.0)
    close(R1, R0)
    np.testing.assert_array_equal(np.isneginf(l1), np.isneginf(l0))
    fin = np.isfinite(l0)
    close(l1[fin], l0[fin])


def check_norm_invariances(orc, c):
    """RMSNorm makes the logits blind to the scale of Q_t and E_t, and r_c to the scale of any memory
    row n (eq 26); the value side V = C_t dH[c] is not normalised."""
    Q, C, E, dH, S = c["Q"], c["C"].copy(), c["E"], c["dH"].copy(), c["S"]
    n0 = 1
    C[..., n0] = 0.0  # row n0 of a memory then reaches R only through the (normalised) key side
    R, lse = orc.sma(Q, C, E, dH, S, norm_eps=0.0)
    fin = np.isfinite(lse)
    for Q2, E2, D2 in ((Q * 7.0, E, dH), (Q, E * 0.3, dH)):
        R2, l2 = orc.sma(Q2, C, E2, D2, S, norm_eps=0.0)
        close(R2, R)
        close(l2[fin], lse[fin])
    D2 = dH.copy()
    D2[:, :, :, n0, :] *= 5.0
    R2, l2 = orc.sma(Q, C, E, D2, S, norm_eps=0.0)
    close(R2, R)
    close(l2[fin], lse[fin])
    # one historical chunk: the weight is 1 and R = C_t dH[0]; scaling dH[0] scales R, not the logit
    t = np.arange(S, 2 * S)
    Rs, ls = orc.sma(Q, C, E, dH * 3.0, S, tokens=t, norm_eps=0.0)
    Rb, lb = orc.sma(Q, C, E, dH, S, tokens=t, norm_eps=0.0)
    close(Rs, 3.0 * Rb)
    close(ls, lb)


def test_normalised_branch_reduces_to_plain_sma(orc):
    check_norm_reduces_to_plain(orc, sma_case(50, L=64, S=16, N=6, P=5, H=2, G=1))


def test_normalised_branch_invariances(orc):
    check_norm_invariances(orc, sma_case(51, L=64, S=16, N=6, P=5, H=2, G=1))


def test_normalised_branch_epsilon_enters_every_rms(orc):
    """eps shifts the three RMS values: a large eps (relative to the data) changes the logits."""
    c = sma_case(52, L=48, S=16, N=4, P=3)
    R0, l0 = orc.sma(c["Q"], c["C"], c["E"], c["dH"], c["S"], norm_eps=0.0)
    R1, l1 = orc.sma(c["Q"], c["C"], c["E"], c["dH"], c["S"], norm_eps=10.0)
    fin = np.isfinite(l0)
    assert np.max(np.abs(l1[fin] - l0[fin])) > 1e-3


def check_norm_eps_closed_form(orc, eps=0.3, seed=53):
    """Where eps sits in eq (25)-(26), fixed by a case worked by hand. Every Q_t is a constant vector q_t 1,
    every E_t a constant e_t 1 and every row n of the memory dH[0] the constant d_n, so RMSNorm gives
    Qb = q_t / sqrt(q_t^2 + eps) in every entry, Eb = e_t / sqrt(e_t^2 + eps), and the key factor
    r_n = (d_n^2 + eps)^(-1/2). A token of chunk 1 sees only dH[0] (softmax weight 1), so
    lse_t = l_{t,0} = Qb Eb P sum_n r_n d_n / sqrt(N) and R_t = C_t dH[0] (the value side is not
    normalised). The scalars are of order one, so 1/(sqrt(x) + eps), or eps left out of one RMS, moves
    the logit by more than 1e-2."""
    rng = np.random.default_rng(seed)
    Bt, H, G, N, P, S = 2, 3, 1, 5, 3, 8
    L = 2 * S
    q = rng.uniform(0.2, 2.0, (Bt, L)) * rng.choice([-1.0, 1.0], (Bt, L))
    e = rng.uniform(0.2, 2.0, (Bt, L, H)) * rng.choice([-1.0, 1.0], (Bt, L, H))
    d = rng.uniform(0.2, 2.0, (Bt, H, N)) * rng.choice([-1.0, 1.0], (Bt, H, N))
    Q = np.repeat(q[:, :, None, None], N, axis=3)
    E = np.repeat(e[:, :, :, None], P, axis=3)
    C = rng.standard_normal((Bt, L, G, N))
    dH = rng.standard_normal((Bt, H, 2, N, P))
    dH[:, :, 0] = np.repeat(d[:, :, :, None], P, axis=3)
    t = np.arange(S, L)
    R, lse = orc.sma(Q, C, E, dH, S, tokens=t, norm_eps=eps)
    for b in range(Bt):
        for h in range(H):
            row = sum(dn / math.sqrt(dn * dn + eps) for dn in d[b, h])
            for j, tt in enumerate(t):
                qb = q[b, tt] / math.sqrt(q[b, tt] ** 2 + eps)
                eb = e[b, tt, h] / math.sqrt(e[b, tt, h] ** 2 + eps)
                close(lse[b, h, j], qb * eb * P * row / math.sqrt(N))
                close(R[b, j, h], C[b, tt, 0] @ dH[b, h, 0])


def test_normalised_branch_epsilon_closed_form(orc):
    check_norm_eps_closed_form(orc)


# ---------------------------------------------------------------------------
# SMA backward (§4 "Efficient Training"; App. C eq (32)-(35))
# ---------------------------------------------------------------------------

BWD_INPUTS = (("dQ", "Q"), ("dC", "C"), ("dE", "E"), ("ddH", "dH"))


def check_bwd_finite_differences(orc, c, h=1e-6, tol=1e-7, norm_eps=None):
    """The gradient is the derivative: for loss = sum(R * dR), every element of dQ, dC, dE and ddH equals
    the central difference of the (separately pinned) forward SMA, to O(h^2) plus rounding. With norm_eps,
    the same for the normalised score branch (App. B.1)."""
    rng = np.random.default_rng(77)
    dR = rng.standard_normal(c["E"].shape)
    S = c["S"]
    grads = orc.sma_bwd(c["Q"], c["C"], c["E"], c["dH"], dR, S, norm_eps=norm_eps)

    def loss(**kw):
        args = {k: c[k] for k in ("Q", "C", "E", "dH")} | kw
        return float(np.sum(orc.sma(args["Q"], args["C"], args["E"], args["dH"], S, threads=1,
                                    norm_eps=norm_eps)[0] * dR))

    for gname, xname in BWD_INPUTS:
        x = c[xname]
        fd = np.empty(x.size)
        for i in range(x.size):
            xp = x.copy().reshape(-1)
            xp[i] += h
            xm = x.copy().reshape(-1)
            xm[i] -= h
            fd[i] = (loss(**{xname: xp.reshape(x.shape)}) - loss(**{xname: xm.reshape(x.shape)})) / (2 * h)
        close(grads[gname], fd.reshape(x.shape), rtol=tol)


def check_bwd_single_history(orc, c):
    """With one historical chunk every weight is 1, so the logits take no gradient: dQ = dE = 0, and
    R_t = C_t dH[0] gives dC_t = dH[0] dR_t and ddH[0] = sum_t C_t^T dR_t (tokens of chunk 1)."""
    S = c["S"]
    Q, C, E = (c[k][:, :2 * S] for k in "QCE")
    dH = c["dH"][:, :, :2]
    rng = np.random.default_rng(78)
    dR = rng.standard_normal(E.shape)
    g = orc.sma_bwd(Q, C, E, dH, dR, S)
    Bt, L, H, P = E.shape
    G = Q.shape[2]
    assert np.all(g["dQ"] == 0.0) and np.all(g["dE"] == 0.0)
    dC = np.zeros_like(C)
    for b in range(Bt):
        for hh in range(H):
            gg = grp(H, G, hh)
            dC[b, S:, gg] += dR[b, S:, hh] @ dH[b, hh, 0].T
            close(g["ddH"][b, hh, 0], C[b, S:, gg].T @ dR[b, S:, hh])
            assert np.all(g["ddH"][b, hh, 1] == 0.0)
    close(g["dC"], dC)


def check_bwd_first_chunk(orc, c):
    """R is 0 in the first chunk whatever the inputs: a dR there produces no gradient at all."""
    S = c["S"]
    dR = np.zeros(c["E"].shape)
    dR[:, :S] = np.random.default_rng(79).standard_normal(dR[:, :S].shape)
    g = orc.sma_bwd(c["Q"], c["C"], c["E"], c["dH"], dR, S)
    for k in ("dQ", "dC", "dE", "ddH"):
        assert np.all(g[k] == 0.0), k


def test_bwd_matches_finite_differences(orc):
    check_bwd_finite_differences(orc, sma_case(60, Bt=1, L=40, S=8, N=4, P=3, H=4, G=2))


def test_bwd_finite_differences_ragged(orc):
    """A ragged last chunk and one head per group."""
    check_bwd_finite_differences(orc, sma_case(61, Bt=2, L=27, S=8, N=3, P=2, H=1, G=1))


@pytest.mark.parametrize("eps", [1e-6, 0.3])
def test_bwd_normalised_branch_matches_finite_differences(orc, eps):
    check_bwd_finite_differences(orc, sma_case(67, Bt=1, L=40, S=8, N=4, P=3, H=4, G=2), norm_eps=eps)


def test_bwd_grouped_e_is_the_sum_over_a_groups_heads(orc):
    """The grouped-E backward the GPU tests compare with: when the heads of a group read one E row
    (E_group repeated per head), the derivative of the loss by E_group, taken by central differences of
    the forward, is the oracle's per-head dE summed over the group's heads."""
    c = sma_case(63, Bt=1, L=40, S=8, N=4, P=3, H=4, G=2)
    EG, S = 2, c["S"]
    Eg = c["E"][:, :, :EG].copy()
    rep = lambda e: np.repeat(e, c["E"].shape[2] // EG, axis=2)  # noqa: E731
    dR = np.random.default_rng(81).standard_normal(c["E"].shape)
    dE = orc.sma_bwd(c["Q"], c["C"], rep(Eg), c["dH"], dR, S)["dE"]
    summed = dE.reshape(*Eg.shape[:2], EG, -1, Eg.shape[3]).sum(axis=3)

    def loss(e):
        return float(np.sum(orc.sma(c["Q"], c["C"], rep(e), c["dH"], S, threads=1)[0] * dR))

    h, fd = 1e-6, np.empty(Eg.size)
    for i in range(Eg.size):
        ep, em = Eg.copy().reshape(-1), Eg.copy().reshape(-1)
        ep[i] += h
        em[i] -= h
        fd[i] = (loss(ep.reshape(Eg.shape)) - loss(em.reshape(Eg.shape))) / (2 * h)
    close(summed, fd.reshape(Eg.shape), rtol=1e-7)


def test_bwd_single_history(orc):
    check_bwd_single_history(orc, sma_case(62, L=32, S=16, N=5, P=3, H=4, G=2))


def test_bwd_first_chunk(orc):
    check_bwd_first_chunk(orc, sma_case(63, L=48, S=16))


# ---------------------------------------------------------------------------
# mutation tests: a planted mistake in the oracle source must break a pin
# ---------------------------------------------------------------------------

MUTATIONS = {
    # decay applied after the write (a_t would scale B_t^T X_t): eq (2) order
    "decay_on_write": ("Hs[n * s->P + p] = a * Hs[n * s->P + p] + Bt[n] * Xt[p];",
                       "Hs[n * s->P + p] = a * (Hs[n * s->P + p] + Bt[n] * Xt[p]);", "quadratic"),
    # A_{s+1:e(c)} off by one (includes a_s): eq (5)
    "decay_window": ("for (i64 r = t + 1; r <= e; ++r)", "for (i64 r = t; r <= e; ++r)", "chunk_identity"),
    # logit scale 1/sqrt(P) instead of 1/sqrt(N): eq (9)
    "logit_scale": ("logit[c] = l / sqrt((double)d.N);", "logit[c] = l / sqrt((double)d.P);", "single_history"),
    # history includes the token's own chunk: eq (10) c < c(t)
    "history": ("t / s->S, R, lse, scratch);", "t / s->S + 1, R, lse, scratch);", "first_chunk"),
    # value read with the query instead of C_t: eq (8)
    "value_vector": ("acc += cr[n] * D[n * d.P + p];", "acc += q[n] * D[n * d.P + p];", "single_history"),
    # softmax with the wrong sign
    "softmax_sign": ("den += exp(logit[c] - m);", "den += exp(m - logit[c]);", "brute"),
    # key readout with the wrong operand (C_t in place of E_t): eq (8)
    "key_operand": ("acc += D[n * d.P + p] * e[p];", "acc += D[n * d.P + p] * cr[p % d.N];", "brute"),
    # gate strides swapped: eq (11)
    "gate_index": ("g[b * gsb + t * gst + h * gsh]", "g[b * gsb + h * gst + t * gsh]", "combine"),
    # decode step: the open chunk's memory accumulated without the decay (eq 5 in recurrent form)
    "step_acc_decay": ("ac[n * P + p] = a * ac[n * P + p] + Bv[n] * Xv[p];",
                       "ac[n * P + p] = ac[n * P + p] + Bv[n] * Xv[p];", "decode_steps"),
    # decode step: the state decayed after the write (eq 2 order)
    "step_state_order": ("st[n * P + p] = a * st[n * P + p] + Bv[n] * Xv[p];",
                         "st[n * P + p] = a * (st[n * P + p] + Bv[n] * Xv[p]);", "decode_steps"),
    # decode step: the memory of a closed chunk is not reset
    "step_close_reset": ("ac[e] = 0.0;", "ac[e] = ac[e];", "decode_steps"),
    # normalised branch: Q_t not normalised (eq 25)
    "norm_query": ("qb[n] = q[n] * inv_q;", "qb[n] = q[n];", "norm_invariances"),
    # normalised branch: E_t not normalised (eq 25)
    "norm_key_input": ("eb[p] = e[p] * inv_e;", "eb[p] = e[p];", "norm_invariances"),
    # backward: the softmax Jacobian without its mean term (dl = w dw)
    "bwd_softmax_jacobian": ("const double dl = w[ch] * (dw - dRR);", "const double dl = w[ch] * dw;", "bwd_fd"),
    # backward: dE contracted with C_t instead of Q_t
    "bwd_de_operand": ("for (i64 n = 0; n < N; ++n) acc += D[n * P + p] * q[n];",
                       "for (i64 n = 0; n < N; ++n) acc += D[n * P + p] * cr[n];", "bwd_fd"),
    # backward: dQ without the 1/sqrt(N) of eq (9)
    "bwd_dq_scale": ("dq[n] += dl * rs * K[ch * N + n];", "dq[n] += dl * K[ch * N + n];", "bwd_fd"),
    # backward: the value path of ddH transposed (dR_t^T C_t read as n x p with swapped indices)
    "bwd_ddh_value": ("dd[n * P + p] += w[ch] * cr[n] * dr[p]", "dd[n * P + p] += w[ch] * cr[p % N] * dr[n % P]",
                      "bwd_single"),
    # backward: dC summed over one head only (Q, C shared by a group's heads)
    "bwd_group_sum": ("dc[n] += w[ch] * acc;", "if (h == g * (s->H / s->G)) dc[n] += w[ch] * acc;", "bwd_single"),
    # normalised backward: the key rows' norm factor taken as constant (no d r / d dH term)
    "bwd_norm_key_factor": ("r * eb[p] - r * r * r * kv * D[n * P + p] / (double)P", "r * eb[p]", "bwd_norm_fd"),
    # normalised backward: dQ without the RMSNorm Jacobian's projection term
    "bwd_norm_q_jacobian": ("dq[n] += iq * dqb[n] - iq * iq * iq * q[n] * qd / (double)N;", "dq[n] += iq * dqb[n];",
                            "bwd_norm_fd"),
    # normalised branch: r averaged over the wrong axis length (N instead of P, eq 26)
    "norm_row_axis": ("double r = 1.0 / sqrt(row_sq / (double)d.P + eps);",
                      "double r = 1.0 / sqrt(row_sq / (double)d.N + eps);", "norm_plain"),
    # normalised branch: eps added outside the square root of each RMS (eq 25-26), or left out of r
    "norm_eps_q": ("double inv_q = 1.0 / sqrt(sq / (double)d.N + eps);",
                   "double inv_q = 1.0 / (sqrt(sq / (double)d.N) + eps);", "norm_eps"),
    "norm_eps_e": ("double inv_e = 1.0 / sqrt(se / (double)d.P + eps);",
                   "double inv_e = 1.0 / (sqrt(se / (double)d.P) + eps);", "norm_eps"),
    "norm_eps_r": ("double r = 1.0 / sqrt(row_sq / (double)d.P + eps);",
                   "double r = 1.0 / (sqrt(row_sq / (double)d.P) + eps);", "norm_eps"),
    "norm_eps_r_dropped": ("double r = 1.0 / sqrt(row_sq / (double)d.P + eps);",
                           "double r = 1.0 / sqrt(row_sq / (double)d.P);", "norm_eps"),
    # the same four mistakes in the normalised backward, caught by finite differences of the forward
    "bwd_norm_eps_q": ("const double iq = 1.0 / sqrt(sq / (double)N + eps);",
                       "const double iq = 1.0 / (sqrt(sq / (double)N) + eps);", "bwd_norm_fd_eps"),
    "bwd_norm_eps_e": ("const double ie = 1.0 / sqrt(se / (double)P + eps);",
                       "const double ie = 1.0 / (sqrt(se / (double)P) + eps);", "bwd_norm_fd_eps"),
    "bwd_norm_eps_r": ("const double r = 1.0 / sqrt(rowsq / (double)P + eps);",
                       "const double r = 1.0 / (sqrt(rowsq / (double)P) + eps);", "bwd_norm_fd_eps"),
    "bwd_norm_eps_r_dropped": ("const double r = 1.0 / sqrt(rowsq / (double)P + eps);",
                               "const double r = 1.0 / sqrt(rowsq / (double)P);", "bwd_norm_fd_eps"),
}


def _run_pin(orc, which):
    if which == "quadratic":
        check_quadratic_form(orc, rand_case(30, L=24))
    elif which == "chunk_identity":
        check_chunk_identity(orc, rand_case(31, L=40, S=16))
    elif which == "single_history":
        check_single_history(orc, sma_case(32, N=5, P=3))
    elif which == "first_chunk":
        check_first_chunk(orc, sma_case(33))
    elif which == "brute":
        c = sma_case(34, L=48, S=8)
        c["Q"] *= 3.0
        check_brute_force(orc, c)
    elif which == "combine":
        check_combine(orc)
    elif which == "decode_steps":
        check_decode_steps(orc, rand_case(35, L=29, S=8, G=1, H=2))
    elif which == "norm_invariances":
        check_norm_invariances(orc, sma_case(36, L=64, S=16, N=6, P=5, H=2, G=1))
    elif which == "norm_plain":
        check_norm_reduces_to_plain(orc, sma_case(37, L=64, S=16, N=6, P=5, H=2, G=1))
    elif which == "bwd_fd":
        check_bwd_finite_differences(orc, sma_case(64, Bt=1, L=24, S=8, N=3, P=2, H=2, G=1))
    elif which == "bwd_norm_fd":
        check_bwd_finite_differences(orc, sma_case(68, Bt=1, L=24, S=8, N=3, P=2, H=2, G=1), norm_eps=1e-3)
    elif which == "norm_eps":
        check_norm_eps_closed_form(orc)
    elif which == "bwd_norm_fd_eps":
        check_bwd_finite_differences(orc, sma_case(69, Bt=1, L=24, S=8, N=3, P=2, H=2, G=1), norm_eps=0.3)
    elif which == "bwd_single":
        check_bwd_single_history(orc, sma_case(65, L=32, S=16, N=5, P=3, H=4, G=2))
    else:
        raise KeyError(which)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new, pin = MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = oracle.build(str(mutated), str(tmp_path / "libmutant.so"), force=True)
    mutant = oracle.Oracle(lib)
    with pytest.raises(AssertionError):
        _run_pin(mutant, pin)


@pytest.mark.parametrize("pin", ["quadratic", "chunk_identity", "single_history", "first_chunk", "brute", "combine",
                                 "decode_steps", "norm_invariances", "norm_plain", "bwd_fd", "bwd_single",
                                 "bwd_norm_fd", "norm_eps", "bwd_norm_fd_eps"])
def test_pins_pass_on_the_oracle(orc, pin):
    _run_pin(orc, pin)


@pytest.mark.parametrize("norm_eps", [None, 0.3])
def test_bwd_sampled_modes_agree_with_the_full_backward(orc, norm_eps):
    """The sampled per-token and per-chunk-memory modes return the rows and memories of the full backward
    (plain, and with norm_eps the normalised score branch's)."""
    c = sma_case(66, Bt=2, L=56, S=8, N=4, P=3, H=4, G=2)
    dR = np.random.default_rng(80).standard_normal(c["E"].shape)
    full = orc.sma_bwd(c["Q"], c["C"], c["E"], c["dH"], dR, c["S"], norm_eps=norm_eps)
    tok = [0, 7, 8, 31, 55]
    part = orc.sma_bwd_tokens(c["Q"], c["C"], c["E"], c["dH"], dR, c["S"], tok, norm_eps=norm_eps)
    for k in ("dQ", "dC", "dE"):
        close(part[k], full[k][:, tok])
    trip = [(0, 0, 0), (1, 3, 5), (1, 2, 6)]
    dd = orc.sma_bwd_ddh(c["Q"], c["C"], c["E"], c["dH"], dR, c["S"], trip, norm_eps=norm_eps)
    for i, (b, h, ch) in enumerate(trip):
        close(dd[i], full["ddH"][b, h, ch])
