"""Pins of the reverse-mode oracle (oracle.gdn_vjp / gdn2_vjp) against central finite differences of the
forward recurrence oracle, the GDN-2 -> GDN reduction, and inputs that cannot matter."""
import numpy as np
import pytest

import oracle

IN_GDN = ("q", "k", "v", "g", "beta", "h0")
IN_GDN2 = ("q", "k", "v", "g", "b", "w", "h0")


def tiny(variant, B=1, T=7, H=2, dk=3, dv=4, seed=0, n_seqs=None):
    rng = np.random.default_rng(seed)
    x = {"q": rng.standard_normal((B, T, H, dk)), "k": rng.standard_normal((B, T, H, dk)) * 0.6,
         "v": rng.standard_normal((B, T, H, dv))}
    if variant == "gdn":
        x["g"] = -rng.uniform(0.05, 1.5, (B, T, H))
        x["beta"] = rng.uniform(0.1, 0.9, (B, T, H))
    else:
        x["g"] = -rng.uniform(0.05, 1.5, (B, T, H, dk))
        x["b"] = rng.uniform(0.1, 0.9, (B, T, H, dk))
        x["w"] = rng.uniform(0.1, 0.9, (B, T, H, dv))
    n = B if n_seqs is None else len(n_seqs) - 1
    x["h0"] = rng.standard_normal((n, H, dk, dv)) * 0.3
    do = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((n, H, dk, dv))
    return x, do, dhT


def loss(variant, x, do, dhT, cu=None):
    if variant == "gdn":
        o, hT = oracle.gdn_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], 0.7, x["h0"], cu_seqlens=cu)
    else:
        o, hT = oracle.gdn2_fwd(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], 0.7, x["h0"], cu_seqlens=cu)
    return float(np.sum(do * o) + np.sum(dhT * hT))


def grads(variant, x, do, dhT, cu=None):
    if variant == "gdn":
        r = oracle.gdn_vjp(x["q"], x["k"], x["v"], x["g"], x["beta"], 0.7, x["h0"], do, dhT, cu_seqlens=cu)
        return {"q": r["dq"], "k": r["dk"], "v": r["dv"], "g": r["dg"], "beta": r["dbeta"], "h0": r["dh0"]}
    r = oracle.gdn2_vjp(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], 0.7, x["h0"], do, dhT, cu_seqlens=cu)
    return {"q": r["dq"], "k": r["dk"], "v": r["dv"], "g": r["dg"], "b": r["db"], "w": r["dw"], "h0": r["dh0"]}


def fd_check(variant, x, do, dhT, cu=None, eps=1e-6, n_dirs=2, seed=1):
    rng = np.random.default_rng(seed)
    gr = grads(variant, x, do, dhT, cu)
    for name in (IN_GDN if variant == "gdn" else IN_GDN2):
        for _ in range(n_dirs):
            d = rng.standard_normal(x[name].shape)
            xp = dict(x)
            xm = dict(x)
            xp[name] = x[name] + eps * d
            xm[name] = x[name] - eps * d
            fd = (loss(variant, xp, do, dhT, cu) - loss(variant, xm, do, dhT, cu)) / (2 * eps)
            an = float(np.sum(gr[name] * d))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"{variant} d{name}: fd {fd:.10g} vs vjp {an:.10g}"


@pytest.mark.parametrize("variant", ["gdn", "gdn2"])
def test_vjp_matches_central_differences(variant):
    x, do, dhT = tiny(variant, seed=3)
    fd_check(variant, x, do, dhT)


@pytest.mark.parametrize("variant", ["gdn", "gdn2"])
def test_vjp_across_checkpoint_blocks(variant):
    """T = 150 spans three 64-token recomputation blocks."""
    x, do, dhT = tiny(variant, T=150, H=1, dk=2, dv=3, seed=4)
    fd_check(variant, x, do, dhT, n_dirs=1)


@pytest.mark.parametrize("variant", ["gdn", "gdn2"])
def test_vjp_packed_sequences(variant):
    cu = np.array([0, 2, 2, 9, 13], dtype=np.int32)
    x, do, dhT = tiny(variant, T=13, seed=5, n_seqs=cu)
    fd_check(variant, x, do, dhT, cu=cu, n_dirs=1)
    gr = grads(variant, x, do, dhT, cu)
    assert np.array_equal(gr["h0"][1], dhT[1])  # an empty sequence passes its state's cotangent through


def test_gdn2_with_scalar_gates_reduces_to_gdn():
    x, do, dhT = tiny("gdn", seed=6)
    dk, dv = x["q"].shape[-1], x["v"].shape[-1]
    x2 = {"q": x["q"], "k": x["k"], "v": x["v"], "h0": x["h0"],
          "g": np.repeat(x["g"][..., None], dk, -1), "b": np.repeat(x["beta"][..., None], dk, -1),
          "w": np.repeat(x["beta"][..., None], dv, -1)}
    g1 = grads("gdn", x, do, dhT)
    g2 = grads("gdn2", x2, do, dhT)
    for name in ("q", "k", "v", "h0"):
        assert np.allclose(g1[name], g2[name], rtol=1e-12, atol=1e-12)
    assert np.allclose(g1["beta"], g2["b"].sum(-1) + g2["w"].sum(-1), rtol=1e-12, atol=1e-12)
    assert np.allclose(g1["g"], g2["g"].sum(-1), rtol=1e-12, atol=1e-12)


def test_inputs_that_cannot_matter_get_zero_gradient():
    x, do, dhT = tiny("gdn", seed=7)
    x["beta"] = np.zeros_like(x["beta"])  # nothing is written: v never reaches o or hT
    gr = grads("gdn", x, do, dhT)
    assert np.all(gr["v"] == 0.0)
    z = grads("gdn", tiny("gdn", seed=8)[0], np.zeros_like(do), np.zeros_like(dhT))
    for name in IN_GDN:
        assert np.all(z[name] == 0.0)  # zero cotangents, zero gradients
