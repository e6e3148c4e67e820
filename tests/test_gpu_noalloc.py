"""gdn_chunk_fwd_noalloc: the tensor-core path on the library's static scratch, no allocation."""
import pytest
import torch

from gated_delta_rule_105_b200 import binding as bd
from gated_delta_rule_105_b200.inputs import WORKLOADS, generate, generate_workload

STATIC_WS = 128 * 1024 * 1024


def _dev(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["gdn_bf16_b4h16t4096_dk128_dv256_h0", "gdn_bf16_b8h8t4096_dk128_dv128"])
def test_noalloc_matches_the_workspace_call_bit_for_bit(name):
    w = WORKLOADS[name]
    assert bd.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv) <= STATIC_WS
    d = _dev(generate_workload(w))
    o1, h1 = bd.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"], o_dtype=torch.float32)
    assert bd.last_kernel() == "tc"
    o2, h2 = bd.gdn_chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                                      o_dtype=torch.float32)
    assert bd.last_kernel() == "tc"
    bd.check_error()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


@pytest.mark.gpu
def test_noalloc_beyond_the_static_scratch_takes_the_simt_kernel():
    # 1025 chunk slots x 8 heads x 24 KB > 128 MiB: AUTO runs the SIMT kernel, forcing TC is refused
    inp = generate(1, 65536, 8, 128, 128, "bf16", 777, "gdn", 0.0, 0)
    assert bd.workspace_bytes(1, 65536, 8, 128, 128) > STATIC_WS
    d = _dev(inp)
    o1, h1 = bd.gdn_chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], None,
                                      o_dtype=torch.float32)
    assert bd.last_kernel() == "simt"
    o2, h2 = bd.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], None, o_dtype=torch.float32)
    assert bd.last_kernel() == "tc"
    rms = o2.float().pow(2).mean().sqrt()
    assert ((o1 - o2).abs().max() / rms).item() < 2e-2
    bd.set_kernel("tc")
    try:
        with pytest.raises(bd.GdnError):
            bd.gdn_chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], None)
    finally:
        bd.set_kernel("auto")
