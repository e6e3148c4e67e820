"""Per-kernel launch timing of the C ABI (gdn_profile_enable / gdn_profile_take)."""
import ctypes

import pytest
import torch

from gated_delta_rule_105_b200 import binding as bd
from gated_delta_rule_105_b200.inputs import generate


def test_profile_take_rejects_bad_ids(oracle_lib):
    lib = bd.load_library()
    n, ms = ctypes.c_int(7), ctypes.c_double(1.0)
    assert lib.gdn_profile_take(9, ctypes.byref(n), ctypes.byref(ms)) == 1
    assert lib.gdn_profile_take(-1, ctypes.byref(n), ctypes.byref(ms)) == 1
    assert lib.gdn_profile_take(0, None, ctypes.byref(ms)) == 1
    # nothing recorded: zero launches, no device work
    assert lib.gdn_profile_take(0, ctypes.byref(n), ctypes.byref(ms)) == 0 and n.value == 0


@pytest.mark.gpu
def test_profile_counts_both_tensor_core_launches():
    inp = generate(1, 256, 2, 128, 128, "bf16", 4242, "gdn", 0.02, 0, None)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    bd.set_kernel("tc")
    try:
        bd.profile_take()
        bd.profile_enable(True)
        for _ in range(3):
            bd.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"])
        torch.cuda.synchronize()
        bd.profile_enable(False)
        got = bd.profile_take()
    finally:
        bd.profile_enable(False)
        bd.set_kernel("auto")
    assert got["gdn_tc_wy_kernel"][0] == 3 and got["gdn_tc_fwd_kernel"][0] == 3
    assert got["gdn_tc_wy_kernel"][1] > 0 and got["gdn_tc_fwd_kernel"][1] > 0
    assert "gdn_simt_fwd_kernel" not in got
