"""The fp16 range of the tensor-core scan kernels, as include/dart.h states it.

With bf16 inputs (N = 128, P = 64) the chunk-state kernel multiplies B and the
decay-scaled X rows in fp16, and the SSD-output kernel X and the intra-chunk
weights (C_t . B_s) exp(cs_t - cs_s). A value below 65504 is kept (to fp16
rounding); one past it becomes inf, so the outputs it reaches are inf or NaN and
the kernel raises its bit in dart_fp16_range_flags(). These tests plant such
values in otherwise ordinary inputs.
"""
import numpy as np
import pytest

import workloads as W
from _util import assert_stored, layer_inputs_dev, to_dev, to_f64

pytestmark = pytest.mark.gpu

CHUNK_STATES, SSD_OUT = 1, 2


@pytest.fixture(scope="module")
def dart():
    import ssm_state_memory_b200 as d

    return d


def small_inputs():
    w = W.MIXER_BF16.with_(batch=1, nheads=2, seqlen=512)
    return w, W.make_layer_inputs(w)


def with_value(inp, name, index, value):
    x = inp[name].f64.copy()
    x[index] = value
    return inp | {name: W.store(x, "bf16")}


def run_scan(dart, w, inp):
    import torch

    dv = layer_inputs_dev(inp)
    assert dart.dart_fp16_range_flags() >= 0  # clear what earlier calls left
    dH = dart.chunk_states(dv["X"], dv["B"], dv["logA"], w.chunk)
    Y, _ = dart.ssd_scan(dv["X"], dv["B"], dv["C"], dv["logA"], dH, w.chunk)
    torch.cuda.synchronize()
    return dH, Y, dart.dart_fp16_range_flags()


def test_values_just_inside_the_fp16_range_are_kept(dart, orc):
    """|X| = 60000 (below 65504) at the last token of chunk 0: no flag, every output finite, and the chunk
    memories and Y match the oracle. In chunk 0 the value reaches Y only through the fp16 intra-chunk
    product, so those rows are checked element by element (the one large value makes Y heavy-tailed):
    within 2^-8 of each value (fp16 keeps 2^-11 of the dominant product) plus 2e-2 of rms(Y). Later chunks
    see it through the state entering the chunk, stored in bf16, whose rounding of the one dominant term
    (2^-9 of each entry, over 128 entries) sets their error; they are not part of this check."""
    w, inp = small_inputs()
    inp = with_value(inp, "X", (0, 255, 0, 3), 60000.0)
    dH, Y, flags = run_scan(dart, w, inp)
    assert flags == 0
    X, B, C = (inp[k].f64 for k in "XBC")
    Yr, _, _ = orc.recurrence(X, B, C, inp["logA"], w.chunk)
    y = to_f64(Y)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(to_f64(dH)))
    assert_stored(to_f64(dH), orc.chunk_states(X, B, inp["logA"], w.chunk), "bf16", "dH with |X| = 6e4")
    assert_stored(y[:, :w.chunk], Yr[:, :w.chunk], "bf16", "Y of chunk 0 with |X| = 6e4", acc_tol=2e-2)


def test_x_past_the_fp16_range_is_flagged(dart):
    """|X| = 1e5 at token 255 of head 0, the last token of chunk 0 (decay weight 1 in its chunk memory):
    that head's first chunk memory and the Y rows of the token's 128-token block (whose products take X of
    the whole block, 0 * inf included) are not finite, both kernels raise their bit, and the earlier block
    and head 1 (which never read the value) stay finite. (At an earlier token of the chunk the memory would
    see X scaled by the decay to the chunk's end, which can bring it back into range.)"""
    w, inp = small_inputs()
    inp = with_value(inp, "X", (0, 255, 0, 3), 1.0e5)
    dH, Y, flags = run_scan(dart, w, inp)
    assert flags == CHUNK_STATES | SSD_OUT
    d, y = to_f64(dH), to_f64(Y)
    assert not np.all(np.isfinite(d[0, 0, 0]))
    assert np.all(np.isfinite(d[0, 1]))
    assert not np.all(np.isfinite(y[0, 255, 0]))
    assert np.all(np.isfinite(y[0, :128, 0])) and np.all(np.isfinite(y[0, :, 1]))


def test_intra_chunk_weight_past_the_fp16_range_is_flagged(dart):
    """C_t = B_s = 30 in every entry for two tokens of one chunk gives C_t . B_s = 115200 > 65504: the SSD
    output raises its bit and those rows are not finite; the chunk memories (B = 30 is in range) stay
    finite and raise nothing."""
    w, inp = small_inputs()
    for name in "BC":
        x = inp[name].f64.copy()
        x[0, 300:302] = 30.0
        inp = inp | {name: W.store(x, "bf16")}
    dH, Y, flags = run_scan(dart, w, inp)
    assert flags == SSD_OUT
    assert np.all(np.isfinite(to_f64(dH)))
    y = to_f64(Y)
    assert not np.all(np.isfinite(y[0, 301]))
    assert np.all(np.isfinite(y[0, :300]))


def test_layer_reports_the_same_flag(dart):
    """dart_layer_fwd runs the same kernels: the planted X of the test above raises both bits."""
    import torch

    w, inp = small_inputs()
    inp = with_value(inp, "X", (0, 255, 0, 3), 1.0e5)
    dv = layer_inputs_dev(inp)
    assert dart.dart_fp16_range_flags() >= 0
    out, _, _ = dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], dv["logA"], dv["g"],
                               inp["g_strides"], w.chunk)
    torch.cuda.synchronize()
    assert dart.dart_fp16_range_flags() == CHUNK_STATES | SSD_OUT
    assert not np.all(np.isfinite(to_f64(out)[0, 255, 0]))
    assert dart.dart_fp16_range_flags() == 0  # the read cleared them


def bwd_with_memory_value(dart, orc, value):
    """dart_sma_bwd on a small tensor-core shape with one chunk memory entry set to value (bf16)."""
    import torch

    w = W.MIXER_BF16.with_(batch=1, nheads=2, seqlen=3 * 256 + 37)
    inp = W.make_layer_inputs(w)
    X, B, C, Q, E = (inp[k].f64 for k in "XBCQE")
    dH = orc.chunk_states(X, B, inp["logA"], w.chunk)
    dH[0, 1, 0, 5, 7] = value
    dH_in = W.store(dH, "bf16")
    dR = W.make_readout_grad(w)
    R, lse = orc.sma(Q, C, E, dH_in.f64, w.chunk)
    dv = layer_inputs_dev(inp)
    assert dart.dart_fp16_range_flags() >= 0
    grads = dart.sma_bwd(dv["Q"], dv["C"], dv["E"], to_dev(dH_in),
                         torch.from_numpy(R.astype(np.float32)).cuda(), torch.from_numpy(lse.astype(np.float32)).cuda(),
                         torch.from_numpy(dR).cuda(), w.chunk)
    torch.cuda.synchronize()
    return grads, dart.dart_fp16_range_flags()


BWD_OPERANDS = 4


def test_backward_memory_inside_the_fp16_range(dart, orc):
    """A chunk memory entry of 65280 (the largest bf16 value below fp16's limit) converts exactly: no flag,
    every gradient finite."""
    grads, flags = bwd_with_memory_value(dart, orc, 65280.0)
    assert flags == 0
    for g in grads:
        assert bool(np.all(np.isfinite(to_f64(g))))


def test_backward_memory_past_the_fp16_range_is_flagged(dart, orc):
    """A chunk memory entry of 65536 becomes inf in the backward's fp16 copy: the flag is raised and the
    gradient products that read that memory are not finite (inf times the rows, inf - inf among them)."""
    grads, flags = bwd_with_memory_value(dart, orc, 65536.0)
    assert flags == BWD_OPERANDS
    dQ = to_f64(grads[0])
    assert not np.all(np.isfinite(dQ[0, 256:]))  # the memory is head 1's of chunk 0: every later token reads it
