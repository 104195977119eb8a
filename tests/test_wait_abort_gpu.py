"""The give-up path of the tensor-core kernels' bounded waits, taken on purpose.

Every wait inside the tcgen05 kernels is bounded (by default 2 s). A wait that
runs out records a code in the device error word, stops every role of the CTA,
lets the copies and tensor-core products it already started finish, releases
tensor memory and returns. This test shortens the limit to 1 ns through
dart_set_wait_limit, so that the first wait which is not satisfied at once gives
up, runs one small layer forward (chunk states, SSD output and SMA kernels, one
tile each), and checks that the kernels reported it and that the next call at the
default limit runs clean and correct on the same context.
"""
import pytest

import workloads as W
from _util import assert_close, layer_inputs_dev, to_f64

pytestmark = pytest.mark.gpu


def test_a_wait_that_runs_out_stops_the_kernels_cleanly(orc):
    import torch

    import ssm_state_memory_b200 as dart

    w = W.MIXER_BF16.with_(batch=1, nheads=2, seqlen=512)
    inp = W.make_layer_inputs(w)
    dv = layer_inputs_dev(inp)
    torch.cuda.synchronize()
    assert dart.dart_device_error() == 0
    dart.dart_set_wait_limit(1)
    try:
        dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], dv["logA"], dv["g"], inp["g_strides"], w.chunk)
        torch.cuda.synchronize()
        code = dart.dart_device_error()
    finally:
        dart.dart_set_wait_limit(0)
    assert code > 0, "no wait gave up under a 1 ns limit"
    out, _, _ = dart.layer_fwd(dv["X"], dv["B"], dv["C"], dv["Q"], dv["E"], dv["logA"], dv["g"], inp["g_strides"],
                               w.chunk)
    torch.cuda.synchronize()
    assert dart.dart_device_error() == 0
    ref = orc.layer(*(inp[k].f64 for k in "XBCQE"), inp["logA"], inp["g"], inp["g_strides"], w.chunk)
    assert_close(to_f64(out), ref["out"], "bf16", "layer out after the aborted call")
