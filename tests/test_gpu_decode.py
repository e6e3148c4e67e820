"""The recurrent decode step (one token per sequence, state in place) against the fp64 oracle.

One decode step is the token recurrence for T = 1 with the state as h0, so the oracle's recurrence with T = 1
is its definition; many steps in a row must reproduce the oracle's run over the whole token sequence.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_105_b200.inputs import generate
from parity_util import TOL, f64, kda_gates, o_excess, relerr

pytestmark = pytest.mark.gpu


def oracle_run(inp, variant, h0):
    import oracle
    q, k, v, g = (f64(inp[x]) for x in ("q", "k", "v", "g"))
    if variant == "gdn":
        return oracle.gdn_fwd(q, k, v, g, f64(inp["beta"]), inp["scale"], h0)
    if variant == "kda":
        b, w = kda_gates(inp)
        return oracle.gdn2_fwd(q, k, v, g, b, w, inp["scale"], h0)
    return oracle.gdn2_fwd(q, k, v, g, f64(inp["b"]), f64(inp["w"]), inp["scale"], h0)


def step(inp, t, state, variant, o_dtype):
    """Decode step for token t of a [N, T, H, ...] input set (the batch rows are the N sequences)."""
    from gated_delta_rule_105_b200 import decode_fwd
    sl = {key: (val[:, t].contiguous().cuda() if isinstance(val, torch.Tensor) and key not in ("h0", "cu_seqlens")
                else val) for key, val in inp.items()}
    return decode_fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl.get("beta"), state, inp["scale"], o_dtype=o_dtype,
                      b=sl.get("b"), w=sl.get("w"), variant=variant)


@pytest.mark.parametrize("variant", ["gdn", "gdn2", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 256), (64, 192)])
def test_single_step_matches_oracle(variant, dtype, dk, dv):
    inp = generate(3, 1, 2, dk, dv, dtype, seed=dk + dv + len(variant), variant=variant, h0_std=0.1)
    state = inp["h0"].clone().cuda()
    o = step(inp, 0, state, variant, torch.float32)
    ro, rh = oracle_run(inp, variant, f64(inp["h0"]))
    assert o_excess(f64(o), ro[:, 0], dtype, "f32") <= 1.0
    assert relerr(f64(state), rh) <= TOL[dtype]


@pytest.mark.parametrize("variant", ["gdn", "gdn2", "kda"])
def test_many_steps_equal_the_whole_sequence(variant):
    T = 70
    inp = generate(4, T, 2, 128, 128, "bf16", seed=77, variant=variant, h0_std=0.05)
    state = inp["h0"].clone().cuda()
    outs = [step(inp, t, state, variant, torch.bfloat16) for t in range(T)]
    torch.cuda.synchronize()
    o = torch.stack(outs, 1)
    ro, rh = oracle_run(inp, variant, f64(inp["h0"]))
    assert o_excess(f64(o), ro, "bf16", "bf16") <= 1.0
    assert relerr(f64(state), rh) <= TOL["bf16"]


def test_decode_leaves_the_other_sequences_alone_and_writes_in_place():
    inp = generate(2, 1, 1, 64, 64, "f32", seed=5, h0_std=0.2)
    state = inp["h0"].clone().cuda()
    ptr = state.data_ptr()
    step(inp, 0, state, "gdn", torch.float32)
    assert state.data_ptr() == ptr
    # per sequence, the update equals the single-sequence run
    for n in range(2):
        one = {key: (val[n:n + 1] if isinstance(val, torch.Tensor) else val) for key, val in inp.items()}
        s1 = inp["h0"][n:n + 1].clone().cuda()
        step(one, 0, s1, "gdn", torch.float32)
        assert torch.allclose(s1[0], state[n], rtol=0, atol=0)
