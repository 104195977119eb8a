"""Checks of the seeded input recipe (no GPU)."""
import math
import os

import numpy as np
import torch

import workloads as W


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0e38])]).astype(np.float32)
    mine = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, ref)
    back = W.bf16_bits_to_f32(mine)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_splitmix64_reference_vectors():
    path = os.path.join(os.path.dirname(__file__), "golden", "splitmix64_seed1234567.txt")
    ref = [int(l) for l in open(path) if l.strip() and not l.startswith("#")]
    got = W.splitmix64(1234567, np.arange(len(ref))).tolist()
    assert got == ref


def test_irwin_hall_moments_and_slicing():
    v = W.bf16_bits_to_f32(W.irwin_hall_bf16(W.cache_key(7), 0, 1 << 20, 0.027)).astype(np.float64)
    assert abs(v.mean()) < 1e-4
    assert abs(v.std() / 0.027 - 1.0) < 0.01
    # any window of counters reproduces the same values
    part = W.irwin_hall_bf16(W.cache_key(7), 12345, 1000, 0.027)
    np.testing.assert_array_equal(part, W.irwin_hall_bf16(W.cache_key(7), 0, 1 << 20, 0.027)[12345:13345])


def test_decode_cache_sigma_matches_chunk_memory_spread(orc):
    """The decode cache stands in for chunk memories of the mixer_bf16 distributions."""
    w = W.MIXER_BF16.with_(batch=1, nheads=8, seqlen=1024)
    inp = W.make_layer_inputs(w)
    dH = orc.chunk_states(inp["X"].f64, inp["B"].f64, inp["logA"], w.chunk)
    assert abs(dH.std() / W.DECODE_BF16.cache_sigma - 1.0) < 0.15


def test_layer_inputs_shapes_and_recipe():
    w = W.MIXER_BF16.with_(seqlen=512)
    a = W.make_layer_inputs(w)
    b = W.make_layer_inputs(w)
    assert a["X"].storage.dtype == np.uint16 and a["X"].shape == (2, 512, 8, 64)
    assert a["B"].shape == (2, 512, 1, 128)
    np.testing.assert_array_equal(a["X"].storage, b["X"].storage)  # seeded
    assert a["logA"].dtype == np.float32 and np.all(a["logA"] < 0)
    # per-head A is constant over (b, t): logA / softplus(...) ratio varies only through dt
    assert a["g"].tolist() == [1.0] and a["g_strides"] == (0, 0, 0)
    t = W.make_layer_inputs(W.TINY_F32)
    assert t["X"].storage.dtype == np.float32 and t["g"].tolist() == [0.5]
    x = a["X"].f64
    assert abs(x.std() * math.sqrt(64) - 1.0) < 0.01


def test_planted_pairs_have_cosine_0_9():
    w = W.LONG_BF16.with_(seqlen=4096, nheads=2)
    inp = W.make_layer_inputs(w)
    pl = inp["plant"]
    assert 1 <= pl["c_star"] <= 15
    assert len(set(pl["positions"].tolist())) == 16
    assert np.all(pl["positions"] // w.chunk == pl["c_star"])
    Q, B, E, X = inp["Q"].f64, inp["B"].f64, inp["E"].f64, inp["X"].f64
    for j, t in enumerate(pl["queries"]):
        s = pl["positions"][j % 16]
        cq = Q[0, t, 0] @ B[0, s, 0] / np.linalg.norm(Q[0, t, 0]) / np.linalg.norm(B[0, s, 0])
        ce = E[0, t, 1] @ X[0, s, 1] / np.linalg.norm(E[0, t, 1]) / np.linalg.norm(X[0, s, 1])
        assert abs(cq - 0.9) < 0.02 and abs(ce - 0.9) < 0.03  # bf16 rounding of the stored values
    assert np.all(inp["logA"] == np.float32(-1e-3))
