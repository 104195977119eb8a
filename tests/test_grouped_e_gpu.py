"""GPU parity of the grouped-E entry points (dart_sma_fwd_ge, dart_layer_fwd_ge, dart_sma_decode_ge).

E [b, L, e_groups, P] is shared by the heads of each E group (the grouped projections of the Fig. 2
caption and App. B.2). The oracle takes E per head, so the tests hand it the grouped E repeated over
each group's heads: the same E_t for every head of a group is the definition of the grouping.
"""
import numpy as np
import pytest

import workloads as W
from _util import TOL, assert_close, assert_lse, layer_inputs_dev, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dart():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import ssm_state_memory_b200 as d

    return d


def grouped(st: W.Stored, EG: int, axis: int, scale: float = 1.0):
    """The first EG per-head slices of a stored E (times a power of two, exact in storage) as its groups,
    and those groups repeated per head."""
    H = st.storage.shape[axis]
    g = W.store(np.take(st.f64, range(EG), axis=axis) * scale, st.dtype)
    full = np.repeat(g.f64, H // EG, axis=axis)
    return g, full


@pytest.mark.parametrize("shape", [
    # (batch, L, H, G, N, P, S, dtype, e_groups)
    (1, 3 * 256 + 37, 4, 1, 128, 64, 256, "bf16", 1),  # tensor cores, every head shares E
    (2, 5 * 128 + 90, 8, 2, 128, 64, 128, "bf16", 2),  # tensor cores, E groups = Q/C groups
    (1, 700, 4, 1, 128, 64, 64, "bf16", 2),             # tensor cores, tiles spanning chunks
    (2, 3 * 64 + 21, 4, 2, 16, 8, 64, "f32", 1),        # CUDA cores
    (1, 600, 6, 1, 128, 64, 128, "bf16", 2),            # tensor cores, 3 heads an E group: a head pair spans two
])
def test_sma_and_layer_with_grouped_e(dart, orc, shape):
    import torch

    Bt, L, H, G, N, P, S, dt, EG = shape
    tc = dt == "bf16" and (N, P) == (128, 64)
    w = W.LayerWorkload("ge", 21, Bt, H, G, L, S, N, P, dt, "mamba2", "per_token")
    inp = W.make_layer_inputs(w)
    # E scaled by 8 so that the logits spread and R depends clearly on which E a head reads
    Eg, Efull = grouped(inp["E"], EG, axis=2, scale=8.0)
    dv = layer_inputs_dev(inp)
    Egd = to_dev(Eg)
    X, B, C, Q = (inp[k].f64 for k in "XBCQ")
    ref = orc.layer(X, B, C, Q, Efull, inp["logA"], inp["g"], inp["g_strides"], S)
    dH_in = W.store(ref["dH"], dt)
    R_ref, lse_ref = orc.sma(Q, C, Efull, dH_in.f64, S)
    torch.cuda.synchronize()
    dart.dart_profile_reset()
    dart.dart_profile_enable(True)
    try:
        R, lse = dart.sma_fwd(dv["Q"], dv["C"], Egd, to_dev(dH_in), S)
        torch.cuda.synchronize()
    finally:
        dart.dart_profile_enable(False)
    used = {k for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    assert ("sma_fwd_tc" in used) == tc, used
    assert_close(to_f64(R), R_ref, dt, "dart_sma_fwd_ge R")
    assert_lse(to_f64(lse), lse_ref, dt, "dart_sma_fwd_ge lse")
    out, _, lse2 = dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], Egd, dv["logA"], dv["g"], inp["g_strides"], S)
    torch.cuda.synchronize()
    assert_close(to_f64(out), ref["out"], dt, "dart_layer_fwd_ge out")
    assert_lse(to_f64(lse2), ref["lse"], dt, "dart_layer_fwd_ge lse")
    # the grouping is not a no-op on these inputs: reading E per head would break the tolerance above
    R_head, _ = orc.sma(Q, C, inp["E"].f64 * 8.0, dH_in.f64, S)
    assert np.max(np.abs(R_head - R_ref)) > 2 * TOL[dt] * np.sqrt(np.mean(R_ref ** 2))


@pytest.mark.parametrize("EG", [1, 2])
def test_decode_with_grouped_e(dart, orc, EG):
    rng = np.random.default_rng(6)
    Bt, H, G, N, P, n = 3, 4, 1, 128, 64, 7
    dt = "bf16"
    Q = W.store(rng.standard_normal((Bt, G, N)) / np.sqrt(N) * 4, dt)
    C = W.store(rng.standard_normal((Bt, G, N)) / np.sqrt(N), dt)
    E = W.store(rng.standard_normal((Bt, H, P)) / np.sqrt(P) * 4, dt)
    Y = W.store(rng.standard_normal((Bt, H, P)) / np.sqrt(P), dt)
    cache = W.store(rng.standard_normal((Bt, H, n, N, P)) * 0.3, dt)
    g = rng.uniform(size=(Bt, H)).astype(np.float32)
    Eg, Efull = grouped(E, EG, axis=1)
    out, lse = dart.sma_decode(to_dev(Q), to_dev(C), to_dev(Eg), to_dev(Y), to_dev(g), (H, 1), to_dev(cache))
    ref_out, ref_lse = orc.decode(Q.f64, C.f64, Efull, Y.f64, g, (H, 1), cache.f64)
    assert_close(to_f64(out), ref_out, dt, "dart_sma_decode_ge out")
    assert_lse(to_f64(lse), ref_lse, dt, "dart_sma_decode_ge lse")


@pytest.mark.parametrize("shape", [
    # (batch, L, H, G, N, P, S, dtype, e_groups); bf16 with N = 128, P = 64 runs on the tensor cores
    (1, 3 * 256 + 37, 4, 1, 128, 64, 256, "bf16", 1),  # one E for every head; ragged last chunk
    (2, 5 * 128 + 90, 8, 2, 128, 64, 128, "bf16", 2),  # E groups = Q/C groups, 4 heads an item
    (1, 700, 6, 1, 128, 64, 64, "bf16", 2),            # 3 heads a group: the head pair (2, 3) spans two
    (2, 300, 4, 2, 32, 16, 64, "f32", 2),               # CUDA cores: E groups = Q/C groups
    (1, 200, 6, 2, 16, 8, 32, "bf16", 3),               # CUDA cores: an E group spans two Q/C groups
])
def test_sma_bwd_with_grouped_e(dart, orc, shape):
    """dart_sma_bwd_ge against the oracle's backward on E repeated per head: dQ, dC and ddH are the
    per-head oracle's, and the gradient of a group's E is the sum over its heads (the chain rule through
    the repetition). On the tensor-core shapes the heads of a group add their dE into its rows."""
    import torch

    Bt, L, H, G, N, P, S, dt, EG = shape
    tc = dt == "bf16" and (N, P) == (128, 64)
    w = W.LayerWorkload("geb", 23, Bt, H, G, L, S, N, P, dt, "mamba2", "per_token")
    inp = W.make_layer_inputs(w)
    Eg, Efull = grouped(inp["E"], EG, axis=2)
    X, B, C, Q = (inp[k].f64 for k in "XBCQ")
    dH_in = W.store(orc.chunk_states(X, B, inp["logA"], S), dt)
    dR = W.make_readout_grad(w)
    R, lse = orc.sma(Q, C, Efull, dH_in.f64, S)
    ref = orc.sma_bwd(Q, C, Efull, dH_in.f64, dR.astype(np.float64), S)
    dE_ref = ref["dE"].reshape(Bt, L, EG, H // EG, P).sum(axis=3)
    dv = layer_inputs_dev(inp)
    torch.cuda.synchronize()
    dart.dart_profile_reset()
    dart.dart_profile_enable(True)
    try:
        dQ, dC, dE, ddH = dart.sma_bwd(dv["Q"], dv["C"], to_dev(Eg), to_dev(dH_in),
                                       torch.from_numpy(R.astype(np.float32)).cuda(),
                                       torch.from_numpy(lse.astype(np.float32)).cuda(), torch.from_numpy(dR).cuda(), S)
        torch.cuda.synchronize()
    finally:
        dart.dart_profile_enable(False)
    used = {k for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    assert ({"sma_bwd_r_tc", "sma_bwd_dq_tc", "sma_bwd_ddh_tc"} <= used) == tc, used
    assert tuple(dE.shape) == (Bt, L, EG, P)
    assert_close(to_f64(dQ), ref["dQ"], dt, "dart_sma_bwd_ge dQ")
    assert_close(to_f64(dC), ref["dC"], dt, "dart_sma_bwd_ge dC")
    assert_close(to_f64(dE), dE_ref, dt, "dart_sma_bwd_ge dE")
    assert_close(to_f64(ddH), ref["ddH"], dt, "dart_sma_bwd_ge ddH")
