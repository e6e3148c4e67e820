"""The device time-out path of the tensor-core kernel, made to run without any GPU fault.

``gdn_debug_stall`` makes the chunk kernel wait on a barrier that nothing arrives on, with a ~1 ms limit: the
wait runs out, the kernel sets the device error word and every warp leaves through its own bounded waits after
draining what it issued.  The host then reads GDN_ERR_TIMEOUT, the context stays usable, and the next ordinary
call is parity-green against the fp64 oracle.
"""
import pytest
import torch

from gated_delta_rule_105_b200 import binding as bd
from gated_delta_rule_105_b200.inputs import generate
from parity_util import TOL, f64, o_excess, relerr, run_cuda, run_oracle

pytestmark = pytest.mark.gpu


def test_stalled_wait_reports_timeout_and_the_next_call_is_correct():
    inp = generate(1, 130, 2, 128, 128, "bf16", seed=55, h0_std=0.05)
    bd.set_kernel("tc")
    try:
        bd.debug_stall(True)
        try:
            run_cuda(inp, "gdn")
        finally:
            bd.debug_stall(False)
        with pytest.raises(bd.GdnError) as ei:
            bd.check_error()
        assert ei.value.status == bd.GDN_ERR_TIMEOUT
        bd.check_error()  # the word was cleared and the context is still usable
        o, hT = run_cuda(inp, "gdn")
        bd.check_error()
        assert bd.last_kernel() == "tc"
    finally:
        bd.set_kernel("auto")
    ro, rh = run_oracle(inp, "gdn")
    assert o_excess(f64(o), ro, "bf16", "f32") <= 1.0
    assert relerr(f64(hT), rh) <= TOL["bf16"]


def test_stall_does_not_touch_the_simt_kernel():
    inp = generate(1, 70, 2, 64, 64, "f32", seed=56)
    bd.debug_stall(True)
    try:
        o, hT = run_cuda(inp, "gdn")
        bd.check_error()
    finally:
        bd.debug_stall(False)
    assert bd.last_kernel() == "simt"
    ro, rh = run_oracle(inp, "gdn")
    assert o_excess(f64(o), ro, "f32", "f32") <= 1.0
