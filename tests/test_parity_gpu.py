"""GPU parity of every C-ABI entry point against the float64 oracle.

Small cases compare every output element; the full-size workloads compare sampled
(batch, head) pairs and tokens that the oracle computes one by one. All inputs are
seeded (workloads/), identical bits on both sides.
"""
import math

import numpy as np
import pytest

import workloads as W
from _util import assert_close, assert_lse, assert_stored, layer_inputs_dev, rel_err, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dart():
    import torch

    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import ssm_state_memory_b200 as d

    return d


def run_layer_checks(dart, orc, w: W.LayerWorkload, inp=None, sample_tokens=None, dh_rms_bound=False):
    """Run all four layer entry points on the GPU; compare with the full oracle. dh_rms_bound adds the
    per-tensor bound max|err| <= tol * rms(ref) on the stored chunk memories to the element-by-element
    check (it holds for chunks of 64 tokens or more; shorter chunks make dH too heavy-tailed for one
    bf16 rounding to stay under 2e-2 of its rms)."""
    import torch

    inp = inp or W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    X, B, C, Q, E = (inp[k].f64 for k in "XBCQE")
    ref = orc.layer(X, B, C, Q, E, inp["logA"], inp["g"], inp["g_strides"], w.chunk)
    dt = w.dtype
    # 1. chunk states, eq (5)
    dH = dart.chunk_states(dv["X"], dv["B"], dv["logA"], w.chunk)
    assert_stored(to_f64(dH), ref["dH"], dt, "dart_chunk_states dH")
    if dh_rms_bound:
        assert_close(to_f64(dH), ref["dH"], dt, "dart_chunk_states dH (per-tensor bound)")
    # The next two entry points take dH as an input: both sides get the oracle's dH
    # rounded once to the storage dtype (an oracle-made input, never a GPU output).
    dH_in = W.store(ref["dH"], dt)
    dH_dev = to_dev(dH_in)
    # 2. SSD scan
    Y, fin = dart.ssd_scan(dv["X"], dv["B"], dv["C"], dv["logA"], dH_dev, w.chunk)
    assert_close(to_f64(Y), ref["Y"], dt, "dart_ssd_scan Y")
    assert_close(to_f64(fin), ref["Hfinal"], dt, "dart_ssd_scan final state")
    # 3. SMA
    R_ref, lse_ref = orc.sma(Q, C, E, dH_in.f64, w.chunk)
    R, lse = dart.sma_fwd(dv["Q"], dv["C"], dv["E"], dH_dev, w.chunk)
    assert_close(to_f64(R), R_ref, dt, "dart_sma_fwd R")
    assert_lse(to_f64(lse), lse_ref, dt, "dart_sma_fwd lse")
    # 4. the fused layer
    out, dH2, lse2 = dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], dv["logA"], dv["g"],
                                    inp["g_strides"], w.chunk)
    torch.cuda.synchronize()
    assert_close(to_f64(out), ref["out"], dt, "dart_layer_fwd out")
    assert torch.equal(dH2, dH), "layer dH differs from dart_chunk_states"
    assert_lse(to_f64(lse2), ref["lse"], dt, "dart_layer_fwd lse")
    return ref


def test_tiny_f32_workload(dart, orc):
    run_layer_checks(dart, orc, W.TINY_F32, dh_rms_bound=True)


def test_mixer_bf16_workload(dart, orc):
    run_layer_checks(dart, orc, W.MIXER_BF16, dh_rms_bound=True)


@pytest.mark.parametrize("shape", [
    # (batch, L, H, G, N, P, S, dtype)
    (2, 3 * 256 + 37, 4, 1, 128, 64, 256, "bf16"),   # ragged last chunk, tensor-core shape
    (1, 5 * 128, 3, 1, 128, 64, 128, "bf16"),        # S = 128
    (1, 200, 2, 1, 128, 64, 256, "bf16"),            # a single partial chunk
    (2, 101, 4, 2, 5, 3, 7, "f32"),                  # odd sizes, 2 groups
    (1, 300, 2, 1, 32, 16, 64, "bf16"),              # small bf16 shape on CUDA cores
    (1, 129, 2, 1, 256, 64, 32, "f32"),              # N = 256
    (1, 96, 1, 1, 8, 256, 16, "f32"),                # P = 256
    (2, 1000, 4, 1, 128, 64, 64, "bf16"),            # S = 64: SMA tiles span two chunks (tcgen05)
    (1, 700, 2, 1, 128, 64, 32, "bf16"),             # S = 32: four chunks per tile
    (1, 500, 3, 1, 128, 64, 64, "bf16"),             # S = 64, odd heads: chunk memories one head a unit
    (1, 300, 2, 1, 128, 64, 16, "bf16"),             # S = 16: eight chunks per tile
    (1, 40, 2, 1, 128, 64, 64, "bf16"),              # a row shorter than one chunk: no history at all
])
def test_generic_shapes(dart, orc, shape):
    Bt, L, H, G, N, P, S, dt = shape
    w = W.LayerWorkload("custom", 7, Bt, H, G, L, S, N, P, dt, "mamba2", "per_token")
    run_layer_checks(dart, orc, w, dh_rms_bound=S >= 128)


def test_strong_decays(dart, orc):
    """Decays far outside the sampled ones: -6 per token over whole 32-token blocks and across a 128-token
    tile boundary of sources (weights exp(cs_t - cs_s) underflow to zero within a few tokens), single -30
    steps inside a block and inside a ragged last chunk. Every entry point against the oracle."""
    w = W.MIXER_BF16.with_(batch=2, seqlen=3 * 256 + 37, nheads=4)
    inp = W.make_layer_inputs(w)
    logA = inp["logA"].copy()
    logA[0, 40:104, 1] = -6.0            # two whole blocks and parts of two more, chunk 0
    logA[1, 300:340, 2] = -6.0           # chunk 1, across a 128-token tile boundary of sources
    logA[0, 530, 0] = -30.0              # one step inside the block 512-543
    logA[1, 3 * 256 + 20, 3] = -30.0     # inside the ragged last chunk
    inp["logA"] = np.ascontiguousarray(logA.astype(np.float32))
    run_layer_checks(dart, orc, w, inp=inp)


def test_gate_zero_reproduces_mamba2_bitwise(dart, orc):
    import torch

    w = W.MIXER_BF16.with_(seqlen=1024, nheads=4)
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    g0 = torch.zeros(1, device="cuda")
    out, dH, _ = dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], dv["logA"], g0, (0, 0, 0), w.chunk)
    Y, _ = dart.ssd_scan(dv["X"], dv["B"], dv["C"], dv["logA"], dH, w.chunk)
    assert torch.equal(out, Y)
    Yref, _, _ = orc.recurrence(inp["X"].f64, inp["B"].f64, inp["C"].f64, inp["logA"], w.chunk)
    assert_close(to_f64(out), Yref, "bf16", "g=0 out vs pure Mamba-2")


def test_first_chunk_mask_and_single_history(dart, orc):
    """Chunk-0 tokens: R = 0, lse = -inf exactly; chunk-1 tokens: R = C_t dH[0] (one memory)."""
    import torch

    w = W.MIXER_BF16.with_(batch=1, seqlen=512, nheads=2)
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    dH_in = W.store(orc.chunk_states(inp["X"].f64, inp["B"].f64, inp["logA"], w.chunk), "bf16")
    R, lse = dart.sma_fwd(dv["Q"], dv["C"], dv["E"], to_dev(dH_in), w.chunk)
    assert torch.all(R[:, :256] == 0)
    assert torch.all(torch.isneginf(lse[:, :, :256]))
    assert torch.all(torch.isfinite(lse[:, :, 256:]))
    C = inp["C"].f64
    ref = np.einsum("tn,hnp->thp", C[0, 256:, 0], dH_in.f64[0, :, 0])
    assert_close(to_f64(R)[0, 256:], ref, "bf16", "single-history readout")


def test_launch_count_of_layer(dart):
    import torch

    w = W.MIXER_BF16.with_(batch=1, seqlen=512, nheads=2)
    dv = layer_inputs_dev(W.make_layer_inputs(w))
    before = dart.dart_kernel_launches()
    _, used = kernel_launches_of(dart, lambda: dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"],
                                                                dv["logA"], dv["g"], (0, 0, 0), w.chunk))
    torch.cuda.synchronize()
    assert used == {"chunk_cumsum": 1, "chunk_states_tc": 1, "state_pass": 1, "ssd_out_tc": 1, "sma_fwd_tc": 1}
    assert dart.dart_kernel_launches() - before == 5


def test_no_kernel_gave_up_a_wait(dart):
    """The tensor-core kernels bound every wait; none of the runs above may have hit the bound."""
    assert dart.dart_device_error() == 0


def kernel_launches_of(dart, fn):
    """Run fn with launch profiling on; {kernel name: launches} of the kernels it launched."""
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


@pytest.mark.parametrize("shape", [
    # (batch, L, H, G, N, P, S, dtype, eps, kernel)
    (2, 3 * 64 + 21, 4, 2, 16, 8, 64, "f32", 1e-6, "sma_fwd"),
    (1, 3 * 256 + 37, 2, 1, 128, 64, 256, "bf16", 1e-6, "sma_fwd_norm_tc"),  # ragged last chunk, 2 tiles a chunk
    (2, 5 * 128 + 90, 8, 2, 128, 64, 128, "bf16", 1e-6, "sma_fwd_norm_tc"),  # 4 heads an item, 2 groups
    (1, 3 * 256 + 37, 2, 1, 128, 64, 256, "bf16", 1e-2, "sma_fwd_norm_tc"),  # eps above mean dH^2: it matters
    (1, 700, 4, 1, 128, 64, 64, "bf16", 1e-6, "sma_fwd_norm_tc"),            # tiles spanning two chunks
    (2, 333, 2, 1, 128, 64, 32, "bf16", 1e-6, "sma_fwd_norm_tc"),            # tiles spanning four chunks
    (2, 300, 2, 1, 32, 16, 32, "bf16", 1e-6, "sma_fwd"),
])
def test_normalised_score_branch(dart, orc, shape):
    """dart_sma_fwd_norm_ws and dart_sma_fwd_norm (App. B.1 eq 25-27) against the oracle, on dH rounded
    once to the dtype: on the tensor cores the fp16 key rows and Q rows come from their own pass (with
    scratch) or from the SMA kernel's scaler warps (without)."""
    Bt, L, H, G, N, P, S, dt, eps, kernel = shape
    w = W.LayerWorkload("norm", 13, Bt, H, G, L, S, N, P, dt, "mamba2", "per_token")
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    X, B, C, Q, E = (inp[k].f64 for k in "XBCQE")
    dH_in = W.store(orc.chunk_states(X, B, inp["logA"], S), dt)
    R_ref, lse_ref = orc.sma(Q, C, E, dH_in.f64, S, norm_eps=eps)
    dH_dev = to_dev(dH_in)
    dH_before = dH_dev.clone()
    for pre in (True, False):
        (R, lse), used = kernel_launches_of(dart, lambda: dart.sma_fwd(dv["Q"], dv["C"], dv["E"], dH_dev, S,
                                                                       norm_eps=eps, prep_pass=pre))
        expect = {kernel: 1, "sma_norm_prep": 1} if (pre and kernel.endswith("_tc")) else {kernel: 1}
        assert used == expect, used
        assert_close(to_f64(R), R_ref, dt, f"dart_sma_fwd_norm R (key pass {pre})")
        assert_lse(to_f64(lse), lse_ref, dt, f"dart_sma_fwd_norm lse (key pass {pre})")
    # the key-side row scaling works on shared-memory copies: the caller's chunk memories are untouched
    assert bool((dH_dev == dH_before).all())
    # the branch differs from the plain SMA on these inputs (it is not a no-op), and so does eps
    tol = 2e-2 if dt == "bf16" else 1e-4
    R_plain, _ = orc.sma(Q, C, E, dH_in.f64, S)
    assert rel_err(R_ref, R_plain) > 10 * tol
    if eps != 1e-6:
        R_eps, _ = orc.sma(Q, C, E, dH_in.f64, S, norm_eps=1e-6)
        assert rel_err(R_ref, R_eps) > 10 * tol
