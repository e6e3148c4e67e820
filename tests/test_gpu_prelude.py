"""The mixer's prelude (short conv + SiLU, L2 norm, gates) and epilogue (RMSNorm x SiLU gate) against the fp64
oracle of oracle/prelude.py, on the same seeded inputs."""
import numpy as np
import pytest
import torch

from gated_delta_rule_105_b200.inputs import generate_prelude
from parity_util import f64

pytestmark = pytest.mark.gpu


def within(x, ref, dtype, what):
    """fp32 outputs: max error <= 1e-5 of the RMS; bf16 outputs: plus the format's rounding, 2^-8 of |ref|."""
    x, ref = f64(x) if isinstance(x, torch.Tensor) else x, np.asarray(ref, dtype=np.float64)
    assert np.isfinite(x).all(), what
    rms = max(np.sqrt(np.mean(ref ** 2)), 1e-30)
    allow = 1e-5 * rms + (2.0 ** -8 * np.abs(ref) if dtype == "bf16" else 0.0)
    excess = float(np.max(np.abs(x - ref) - allow)) if ref.size else -1.0
    assert excess <= 0, f"{what}: error exceeds the allowance by {excess:.3g} (rms {rms:.3g})"


def run_both(inp, eps=1e-6, in_place=False):
    from oracle import prelude as P
    from gated_delta_rule_105_b200 import prelude_fwd
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    cs = d["conv_state"]
    if cs is not None:
        cs_out = cs if in_place else torch.full_like(cs, float("nan"))
    else:
        n = inp["xq"].shape[0] if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
        H, dk, dv = inp["xq"].shape[2], inp["xq"].shape[3], inp["xv"].shape[3]
        cs_out = torch.full((n, 2 * H * dk + H * dv, 3), float("nan"), device="cuda")
    got = prelude_fwd(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["a"], d["A_log"], d["dt_bias"], d["b"],
                      d["c"], cs, cs_out, d["cu_seqlens"], eps)
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy()
    ref = P.prelude(f64(inp["xq"]), f64(inp["xk"]), f64(inp["xv"]), f64(inp["wq"]), f64(inp["wk"]), f64(inp["wv"]),
                    f64(inp["a"]), f64(inp["A_log"]), f64(inp["dt_bias"]), f64(inp["b"]), f64(inp["c"]),
                    f64(inp["conv_state"]), cu, eps)
    return got, ref


def check(got, ref, dtype):
    for key in ("q", "k", "v"):
        within(got[key], ref[key], dtype, key)
    for key in ("g", "beta", "w"):
        if key in ref:
            within(got[key], ref[key], "f32", key)
    # the cache holds raw inputs: exact
    assert np.array_equal(f64(got["conv_state_out"]), ref["conv_state"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 256), (64, 192)])
def test_prelude_dense(dtype, dk, dv):
    inp = generate_prelude(2, 37, 3, dk, dv, dtype, seed=dk + dv, conv_state=True)
    got, ref = run_both(inp)
    check(got, ref, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prelude_packed_with_empty_and_short_sequences(dtype):
    cu = np.array([0, 1, 1, 2, 5, 40, 40, 101], dtype=np.int32)
    inp = generate_prelude(1, int(cu[-1]), 2, 128, 128, dtype, seed=9, conv_state=True, cu_seqlens=cu)
    got, ref = run_both(inp)
    check(got, ref, dtype)
    inp["conv_state"] = None  # zero history
    got, ref = run_both(inp)
    check(got, ref, dtype)


def test_prelude_gdn2_gates():
    inp = generate_prelude(2, 20, 2, 128, 128, "bf16", seed=12, gate_width=128, write_gate=True)
    got, ref = run_both(inp)
    check(got, ref, "bf16")


def test_prelude_single_token_steps_update_the_cache_in_place():
    """Decode: one token per sequence per call, the cache read and rewritten in place, equals one long run."""
    full = generate_prelude(3, 9, 2, 64, 128, "f32", seed=13, conv_state=True)
    got_full, ref_full = run_both(full)
    cache = full["conv_state"].clone().cuda()
    from gated_delta_rule_105_b200 import prelude_fwd
    outs = []
    for t in range(9):
        d = {k: (v[:, t:t + 1].contiguous().cuda() if k in ("xq", "xk", "xv", "a", "b") else
                 (v.cuda() if isinstance(v, torch.Tensor) else v)) for k, v in full.items()}
        outs.append(prelude_fwd(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["a"], d["A_log"], d["dt_bias"],
                                d["b"], None, cache, cache))
    for key in ("q", "k", "v", "g", "beta"):
        within(torch.cat([o[key] for o in outs], 1), ref_full[key], "f32", f"stepped {key}")
    assert np.array_equal(f64(cache), ref_full["conv_state"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128, 192, 256])
def test_output_gate(dtype, dv):
    from oracle import prelude as P
    from gated_delta_rule_105_b200 import output_gate_fwd
    rng = np.random.default_rng(dv)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]
    o = torch.from_numpy(rng.standard_normal((2, 33, 3, dv)).astype(np.float32)).to(tdt)
    z = torch.from_numpy(rng.standard_normal((2, 33, 3, dv)).astype(np.float32)).to(tdt)
    wt = torch.from_numpy(rng.uniform(0.5, 1.5, dv).astype(np.float32))
    y = output_gate_fwd(o.cuda(), z.cuda(), wt.cuda(), eps=1e-5)
    ref = P.output_gate(f64(o), f64(z), f64(wt), eps=1e-5)
    within(y, ref, dtype, "output gate")
