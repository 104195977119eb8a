"""GPU parity of dart_sma_bwd (SMA backward by recomputation) against the float64 oracle.

Both sides read the same seeded inputs: Q, C, E in the storage dtype, the oracle's chunk
memories rounded once to it, and a seeded fp32 dR. The GPU also takes R and lse; they
are the oracle's forward outputs rounded to fp32 (oracle-made inputs), and in a second
check the GPU forward's own outputs, as a caller would pass them.
"""
import numpy as np
import pytest

import workloads as W
from _util import assert_close, layer_inputs_dev, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dart():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import ssm_state_memory_b200 as d

    return d


def kernels_used(dart, fn):
    import torch

    torch.cuda.synchronize()
    dart.dart_profile_reset()
    dart.dart_profile_enable(True)
    try:
        out = fn()
        torch.cuda.synchronize()
    finally:
        dart.dart_profile_enable(False)
    used = {k: v[1] for k, v in dart.profile_table().items() if v[1] > 0}
    dart.dart_profile_reset()
    return out, used


SIMT = ("sma_bwd_delta", "sma_bwd_dq", "sma_bwd_ddh")
TC = ("sma_bwd_delta", "sma_bwd_f16", "sma_bwd_r_tc", "sma_bwd_dq_tc", "sma_bwd_ddh_tc")
SHAPES = [
    # (batch, L, H, G, N, P, S, dtype, kernels launched once each)
    (2, 3 * 64 + 21, 4, 2, 16, 8, 64, "f32", SIMT),
    (2, 300, 2, 1, 32, 16, 32, "bf16", SIMT),
    (1, 3 * 256 + 37, 2, 1, 128, 64, 256, "bf16", TC),     # ragged last chunk, 2 tiles a chunk
    (2, 5 * 128 + 90, 8, 2, 128, 64, 128, "bf16", TC),     # 4 heads an item, 2 groups
    (1, 11 * 128 + 5, 2, 1, 128, 64, 128, "bf16", TC),     # 12 chunks: two chunk blocks of the ddH kernel
    (1, 700, 8, 1, 128, 64, 128, "bf16", TC),              # two head groups share one Q/C group
    (1, 700, 4, 1, 128, 64, 64, "bf16", TC),               # S = 64: tiles spanning two chunks
    (2, 333, 2, 1, 128, 64, 32, "bf16", TC),               # S = 32: four chunks a tile, ragged
    (1, 300, 2, 1, 128, 64, 16, "bf16", TC),               # S = 16: eight chunks a tile
    (1, 40, 2, 1, 128, 64, 64, "bf16", ("sma_bwd_delta",)),  # a row inside its first chunk: all zero
    (1, 256, 2, 1, 128, 64, 256, "bf16", ("sma_bwd_delta",)),  # one chunk: nothing has history, all zero
]


def bwd_case(orc, shape):
    Bt, L, H, G, N, P, S, dt = shape[:8]
    w = W.LayerWorkload("bwd", 17, Bt, H, G, L, S, N, P, dt, "mamba2", "per_token")
    inp = W.make_layer_inputs(w)
    X, B, C, Q, E = (inp[k].f64 for k in "XBCQE")
    dH_in = W.store(orc.chunk_states(X, B, inp["logA"], S), dt)
    dR = W.make_readout_grad(w)
    R, lse = orc.sma(Q, C, E, dH_in.f64, S)
    ref = orc.sma_bwd(Q, C, E, dH_in.f64, dR.astype(np.float64), S)
    return w, inp, dH_in, dR, R, lse, ref


@pytest.mark.parametrize("shape", SHAPES)
def test_sma_bwd_matches_oracle(dart, orc, shape):
    import torch

    w, inp, dH_in, dR, R, lse, ref = bwd_case(orc, shape)
    dv = layer_inputs_dev(inp)
    dH_dev = to_dev(dH_in)
    R_dev = torch.from_numpy(R.astype(np.float32)).cuda()
    lse_dev = torch.from_numpy(lse.astype(np.float32)).cuda()
    dR_dev = torch.from_numpy(dR).cuda()
    grads, used = kernels_used(dart, lambda: dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, R_dev, lse_dev, dR_dev,
                                                          w.chunk))
    assert used == {k: 1 for k in shape[8]}, used
    for name, g in zip(("dQ", "dC", "dE", "ddH"), grads):
        assert_close(to_f64(g), ref[name], w.dtype, f"dart_sma_bwd {name}")
    # exact zeros where nothing flows: tokens of chunk 0 (Q, C, E) and the last chunk memory
    S = w.chunk
    for name, g in zip(("dQ", "dC", "dE"), grads[:3]):
        assert bool((g[:, :S] == 0).all()), name
    assert bool((grads[3][:, :, -1] == 0).all())


@pytest.mark.parametrize("k", [-30, 20])
def test_sma_bwd_gradient_scale_is_invisible(dart, orc, k):
    """The tensor-core gradient products take the rows w dR_t and dl E_t in fp16 after a power-of-two scale
    chosen from the largest |dR| and |dl E_t| of the call. Scaling dR by 2^k scales those maxima, the rows'
    scales and every output by 2^k exactly, so the gradients are 2^k times the unscaled ones bit for bit
    (one head group, so no output is summed in varying order): dR of 2^-30 does not sink into fp16's
    subnormals, dR of 2^20 does not overflow it. Both also match the oracle's (linear) backward."""
    import torch

    w, inp, dH_in, dR, R, lse, ref = bwd_case(orc, SHAPES[2])
    dv = layer_inputs_dev(inp)
    dH_dev = to_dev(dH_in)
    R_dev = torch.from_numpy(R.astype(np.float32)).cuda()
    lse_dev = torch.from_numpy(lse.astype(np.float32)).cuda()
    dR_dev = torch.from_numpy(dR).cuda()
    base = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, R_dev, lse_dev, dR_dev, w.chunk)
    scaled = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, R_dev, lse_dev, dR_dev * 2.0 ** k, w.chunk)
    for name, g0, g1 in zip(("dQ", "dC", "dE", "ddH"), base, scaled):
        assert torch.equal(g1, g0 * 2.0 ** k), name
        assert_close(to_f64(g1), ref[name] * 2.0 ** k, w.dtype, f"dart_sma_bwd {name}, dR x 2^{k}")


def test_sma_bwd_from_gpu_forward(dart, orc):
    """The chain a caller runs: GPU forward (R, lse), then the GPU backward."""
    w, inp, dH_in, dR, _, _, ref = bwd_case(orc, SHAPES[2])
    import torch

    dv = layer_inputs_dev(inp)
    dH_dev = to_dev(dH_in)
    R, lse = dart.sma_fwd(dv["Q"], dv["C"], dv["E"], dH_dev, w.chunk)
    grads = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, R, lse, torch.from_numpy(dR).cuda(), w.chunk)
    for name, g in zip(("dQ", "dC", "dE", "ddH"), grads):
        assert_close(to_f64(g), ref[name], w.dtype, f"dart_sma_bwd {name} (GPU forward)")


NORM_SIMT = {"sma_bwd_dq": 1, "sma_bwd_ddh": 1}
# tensor cores: key rows (with fp16 copies of them and of dH) and Q's RMS factors, fp16 copies of Q and C,
# two recompute passes, one dQ/dC GEMM run (dC against dH, dQ against the key rows), two ddH GEMM runs (key
# and value terms), dQ and ddH assembly
NORM_TC = {"sma_bwd_norm_aux": 4, "sma_bwd_f16": 1, "sma_bwd_rn_tc": 2, "sma_bwd_dq_tc": 1, "sma_bwd_ddh_tc": 2}
NORM_TC_NO_HISTORY = {"sma_bwd_norm_aux": 4}


@pytest.mark.parametrize("shape", [
    # (batch, L, H, G, N, P, S, dtype, eps, kernels)
    (2, 3 * 64 + 21, 4, 2, 16, 8, 64, "f32", 1e-6, NORM_SIMT),
    (2, 300, 2, 1, 32, 16, 32, "bf16", 1e-2, NORM_SIMT),
    (1, 150, 2, 2, 16, 8, 16, "bf16", 1e-6, NORM_SIMT),    # ten chunks of 16, a Q/C group per head
    (1, 100, 2, 1, 16, 8, 128, "f32", 1e-6, NORM_SIMT),    # one chunk: no history, every gradient zero
    (1, 3 * 256 + 37, 2, 1, 128, 64, 256, "bf16", 1e-6, NORM_TC),  # ragged last chunk, 2 tiles a chunk
    (2, 5 * 128 + 90, 8, 2, 128, 64, 128, "bf16", 1e-6, NORM_TC),  # 4 heads an item, 2 groups
    (1, 11 * 128 + 5, 2, 1, 128, 64, 128, "bf16", 1e-2, NORM_TC),  # 12 chunks: two chunk blocks of ddH
    (1, 700, 4, 1, 128, 64, 64, "bf16", 1e-6, NORM_TC),            # S = 64: tiles spanning two chunks
    (2, 333, 2, 1, 128, 64, 32, "bf16", 1e-6, NORM_TC),            # S = 32: four chunks a tile, ragged
    (1, 256, 2, 1, 128, 64, 256, "bf16", 1e-6, NORM_TC_NO_HISTORY),  # one chunk: every gradient zero
    (1, 4096, 2, 1, 128, 64, 256, "bf16", 1e-6, NORM_TC),          # the mixer workload's 16 chunks
])
def test_sma_bwd_normalised_branch(dart, orc, shape):
    """dart_sma_bwd_norm (the normalised score branch's backward) against the oracle's, on the CUDA-core
    kernels and on the tensor cores. Both recompute the softmax statistics, so R and lse filled with NaN give
    the same gradients bit for bit."""
    import torch

    Bt, L, H, G, N, P, S, dt, eps, kernels = shape
    w = W.LayerWorkload("bwdn", 19, Bt, H, G, L, S, N, P, dt, "mamba2", "per_token")
    inp = W.make_layer_inputs(w)
    X, B, C, Q, E = (inp[k].f64 for k in "XBCQE")
    dH_in = W.store(orc.chunk_states(X, B, inp["logA"], S), dt)
    dR = W.make_readout_grad(w)
    R, lse = orc.sma(Q, C, E, dH_in.f64, S, norm_eps=eps)
    ref = orc.sma_bwd(Q, C, E, dH_in.f64, dR.astype(np.float64), S, norm_eps=eps)
    dv = layer_inputs_dev(inp)
    dH_dev = to_dev(dH_in)
    dR_dev = torch.from_numpy(dR).cuda()
    grads, used = kernels_used(dart, lambda: dart.sma_bwd(
        dv["Q"], dv["C"], dv["E"], dH_dev, torch.from_numpy(R.astype(np.float32)).cuda(),
        torch.from_numpy(lse.astype(np.float32)).cuda(), dR_dev, S, norm_eps=eps))
    assert used == kernels, used
    for name, g in zip(("dQ", "dC", "dE", "ddH"), grads):
        assert_close(to_f64(g), ref[name], dt, f"dart_sma_bwd_norm {name}")
    Rn = torch.full((Bt, L, H, P), float("nan"), device="cuda")
    lsen = torch.full((Bt, H, L), float("nan"), device="cuda")
    again = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, Rn, lsen, dR_dev, S, norm_eps=eps)
    none = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], dH_dev, None, None, dR_dev, S, norm_eps=eps)
    for name, g, g2, g3 in zip(("dQ", "dC", "dE", "ddH"), grads, again, none):
        assert torch.equal(g, g2) and torch.equal(g, g3), f"dart_sma_bwd_norm {name} read R or lse"
    if L <= S:
        for name, g in zip(("dQ", "dC", "dE", "ddH"), grads):
            assert not bool(g.any()), f"dart_sma_bwd_norm {name}: one chunk has no history"
        return
    # the branch's backward differs from the plain one on these inputs
    plain = orc.sma_bwd(Q, C, E, dH_in.f64, dR.astype(np.float64), S)
    assert np.max(np.abs(plain["dQ"] - ref["dQ"])) > 0.1 * np.sqrt(np.mean(ref["dQ"] ** 2))
