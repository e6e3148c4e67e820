"""Backward pass (gdn_chunk_bwd) against the fp64 reverse-mode oracle (oracle.gdn_vjp), gradient by gradient.

Tolerance as for the forward: max |x - x_ref| / rms(x_ref) <= 1e-4 for fp32 inputs and 2e-2 for bf16 inputs
(the backward computes in fp32 on the rounded inputs; the oracle consumes the same rounded values).
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_105_b200.inputs import WORKLOADS, generate, generate_workload
from parity_util import TOL, cotangents, f64, relerr, seq_spans

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def run_gpu(inp, d_o, dhT):
    from gated_delta_rule_105_b200 import gdn_chunk_bwd
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out = gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(), d["scale"], d["h0"],
                        None if dhT is None else dhT.cuda(), d["cu_seqlens"])
    torch.cuda.synchronize()
    return {k: f64(v) for k, v in out.items()}


def run_oracle(inp, d_o, dhT, units=None, threads=8):
    import oracle
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy()
    return oracle.gdn_vjp(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["beta"]), inp["scale"],
                          f64(inp["h0"]), f64(d_o), f64(dhT), cu_seqlens=cu, units=units, threads=threads)


def check(got, ref, dtype, what, mask=None):
    for name in GRADS:
        r, x = ref[name], got[name]
        if mask is not None:
            r, x = r[mask[name]], x[mask[name]]
        assert np.isfinite(x).all(), f"{what}: {name} not finite"
        e = relerr(x, r)
        assert e <= TOL[dtype], f"{what}: {name} error {e:.3g} of its RMS (tol {TOL[dtype]})"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,dk,dv", [(1, 64, 64), (63, 64, 64), (130, 128, 128), (257, 128, 256), (97, 64, 192)])
def test_small_shapes(dtype, T, dk, dv):
    inp = generate(2, T, 2, dk, dv, dtype, seed=T + dk + dv, h0_std=0.05)
    d_o, dhT = cotangents(inp, T)
    got = run_gpu(inp, d_o, dhT)
    check(got, run_oracle(inp, d_o, dhT), dtype, f"bwd {dtype} T={T} dk={dk} dv={dv}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_packed_sequences_with_empty_and_short_ones(dtype):
    cu = np.array([0, 1, 1, 64, 129, 200, 330], dtype=np.int32)
    inp = generate(1, int(cu[-1]), 3, 128, 128, dtype, seed=17, h0_std=0.1, cu_seqlens=cu)
    d_o, dhT = cotangents(inp, 17)
    got = run_gpu(inp, d_o, dhT)
    ref = run_oracle(inp, d_o, dhT)
    check(got, ref, dtype, f"packed bwd {dtype}")
    assert np.array_equal(got["dh0"][1], f64(dhT)[1])  # an empty sequence passes dhT through


def test_zero_initial_state_and_no_final_state_cotangent():
    inp = generate(1, 100, 2, 128, 128, "f32", seed=19)
    d_o, _ = cotangents(inp, 19)
    got = run_gpu(inp, d_o, None)
    check(got, run_oracle(inp, d_o, None), "f32", "h0 = 0, dhT = 0")


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items() if w.variant == "gdn"])
def test_workload_full_size_sampled(name):
    """The GDN workloads at full size; sampled (sequence, head) units against the oracle, each unit's gradients
    depending only on that unit's inputs and cotangents."""
    w = WORKLOADS[name]
    inp = generate_workload(w)
    d_o, dhT = cotangents(inp, w.seed)
    got = run_gpu(inp, d_o, dhT)
    n_seq = got["dh0"].shape[0]
    units = [(0, 0), (n_seq - 1, w.H - 1)] if w.T > 256 else None
    ref = run_oracle(inp, d_o, dhT, units=units, threads=8)
    if units is None:
        check(got, ref, w.dtype, name)
        return
    spans = seq_spans(inp)
    for n, h in units:
        row, t0, t1 = spans[n]
        sl = {"dq": (row, slice(t0, t1), h), "dk": (row, slice(t0, t1), h), "dv": (row, slice(t0, t1), h),
              "dg": (row, slice(t0, t1), h), "dbeta": (row, slice(t0, t1), h), "dh0": (n, h)}
        check({k: got[k][sl[k]] for k in GRADS}, {k: ref[k][sl[k]] for k in GRADS}, w.dtype, f"{name} unit {(n, h)}")
