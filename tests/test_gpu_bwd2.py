"""Backward pass of GDN-2 (gdn2_chunk_bwd) and KDA (gdn_kda_chunk_bwd) against the fp64 reverse-mode oracle
(oracle.gdn2_vjp), gradient by gradient.

KDA is GDN-2 with the scalar beta broadcast to both gates, so its oracle is gdn2_vjp on the broadcast gates and
its dbeta the sum of the oracle's db over the key channels and dw over the value channels.  Tolerance as for the
forward: max |x - x_ref| / rms(x_ref) <= 1e-4 for fp32 inputs and 2e-2 for bf16 inputs.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_105_b200.inputs import WORKLOADS, generate, generate_workload
from parity_util import TOL, cotangents, f64, kda_gates, relerr, seq_spans

pytestmark = pytest.mark.gpu

GRADS2 = ("dq", "dk", "dv", "dg", "db", "dw", "dh0")
GRADS_KDA = ("dq", "dk", "dv", "dg", "dbeta", "dh0")


def run_gpu(inp, d_o, dhT, variant):
    from gated_delta_rule_105_b200 import gdn2_chunk_bwd, gdn_kda_chunk_bwd
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    dhT = None if dhT is None else dhT.cuda()
    if variant == "kda":
        out = gdn_kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o.cuda(), d["scale"], d["h0"], dhT,
                                d["cu_seqlens"])
    else:
        out = gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d_o.cuda(), d["scale"], d["h0"], dhT,
                             d["cu_seqlens"])
    torch.cuda.synchronize()
    return {k: f64(v) for k, v in out.items()}


def run_oracle(inp, d_o, dhT, variant, units=None, threads=8):
    import oracle
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy()
    b, w = kda_gates(inp) if variant == "kda" else (f64(inp["b"]), f64(inp["w"]))
    ref = oracle.gdn2_vjp(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), b, w, inp["scale"],
                          f64(inp["h0"]), f64(d_o), f64(dhT), cu_seqlens=cu, units=units, threads=threads)
    if variant == "kda":
        ref["dbeta"] = ref.pop("db").sum(-1) + ref.pop("dw").sum(-1)
    return ref


def check(got, ref, dtype, what, names):
    for name in names:
        r, x = ref[name], got[name]
        assert np.isfinite(x).all(), f"{what}: {name} not finite"
        e = relerr(x, r)
        assert e <= TOL[dtype], f"{what}: {name} error {e:.3g} of its RMS (tol {TOL[dtype]})"


@pytest.mark.parametrize("variant", ["gdn2", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,dk,dv", [(1, 64, 64), (63, 64, 64), (130, 128, 128), (257, 128, 256), (97, 64, 192)])
def test_small_shapes(variant, dtype, T, dk, dv):
    inp = generate(2, T, 2, dk, dv, dtype, seed=T + dk + dv + 3, variant=variant, h0_std=0.05)
    d_o, dhT = cotangents(inp, T + 1)
    got = run_gpu(inp, d_o, dhT, variant)
    names = GRADS_KDA if variant == "kda" else GRADS2
    check(got, run_oracle(inp, d_o, dhT, variant), dtype, f"{variant} bwd {dtype} T={T} dk={dk} dv={dv}", names)


@pytest.mark.parametrize("variant", ["gdn2", "kda"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_packed_sequences_with_empty_and_short_ones(variant, dtype):
    cu = np.array([0, 1, 1, 64, 129, 200, 330], dtype=np.int32)
    inp = generate(1, int(cu[-1]), 3, 128, 128, dtype, seed=23, variant=variant, h0_std=0.1, cu_seqlens=cu)
    d_o, dhT = cotangents(inp, 23)
    got = run_gpu(inp, d_o, dhT, variant)
    names = GRADS_KDA if variant == "kda" else GRADS2
    check(got, run_oracle(inp, d_o, dhT, variant), dtype, f"packed {variant} bwd {dtype}", names)
    assert np.array_equal(got["dh0"][1], f64(dhT)[1])  # an empty sequence passes dhT through


def test_zero_initial_state_and_no_final_state_cotangent():
    inp = generate(1, 100, 2, 128, 128, "f32", seed=29, variant="gdn2")
    d_o, _ = cotangents(inp, 29)
    got = run_gpu(inp, d_o, None, "gdn2")
    check(got, run_oracle(inp, d_o, None, "gdn2"), "f32", "gdn2 h0 = 0, dhT = 0", GRADS2)


def test_kda_backward_equals_gdn2_backward_on_broadcast_gates():
    """The KDA entry and the GDN-2 entry given beta broadcast to b and w run the same arithmetic on the same
    values, so dq, dk, dv, dg and dh0 agree exactly and dbeta is the sum of db and dw."""
    inp = generate(2, 150, 2, 128, 128, "bf16", seed=31, variant="kda", h0_std=0.05)
    d_o, dhT = cotangents(inp, 31)
    got = run_gpu(inp, d_o, dhT, "kda")
    b, w = kda_gates(inp)
    inp2 = dict(inp, b=torch.from_numpy(b.astype(np.float32)), w=torch.from_numpy(w.astype(np.float32)))
    got2 = run_gpu(inp2, d_o, dhT, "gdn2")
    for name in ("dq", "dk", "dv", "dg", "dh0"):
        assert np.array_equal(got[name], got2[name]), name
    np.testing.assert_allclose(got["dbeta"], got2["db"].sum(-1) + got2["dw"].sum(-1), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("name", [n for n, w in WORKLOADS.items() if w.variant == "gdn2"])
def test_workload_full_size_sampled(name):
    """The GDN-2 workload at full size; sampled (sequence, head) units against the oracle, each unit's gradients
    depending only on that unit's inputs and cotangents."""
    w = WORKLOADS[name]
    inp = generate_workload(w)
    d_o, dhT = cotangents(inp, w.seed)
    got = run_gpu(inp, d_o, dhT, "gdn2")
    n_seq = got["dh0"].shape[0]
    units = [(0, 0), (n_seq - 1, w.H - 1)]
    ref = run_oracle(inp, d_o, dhT, "gdn2", units=units, threads=8)
    spans = seq_spans(inp)
    for n, h in units:
        row, t0, t1 = spans[n]
        tok = (row, slice(t0, t1), h)
        sl = {k: tok for k in GRADS2}
        sl["dh0"] = (n, h)
        check({k: got[k][sl[k]] for k in GRADS2}, {k: ref[k][sl[k]] for k in GRADS2}, w.dtype, f"{name} unit {(n, h)}",
              GRADS2)
