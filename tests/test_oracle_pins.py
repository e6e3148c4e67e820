"""Pins for the fp64 oracle: facts fixed by the pages and by the mathematics, not by the oracle.

Each test is chosen so that a plausible slip in the oracle (a dropped decay, beta on the wrong side,
a transposed state, read-out before the write, a sign error, a missed reset at a sequence start)
fails at least one of them.  Definitions: GatedDeltaNet data-flow walkthrough (yfxerp.com/news/
367755), section "Delta Rule: predict first, then correct"; Gated DeltaNet-2 article (7minutos.es),
section "Regla-2 del Delta cerrado"; chunked form: walkthrough section "Chunked parallelism".
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rnd(rng, *shape):
    return rng.standard_normal(shape)


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def gdn_inputs(rng, B=1, T=20, H=2, dk=5, dv=7, h0=True):
    q = unit(rnd(rng, B, T, H, dk))
    k = unit(rnd(rng, B, T, H, dk))
    v = rnd(rng, B, T, H, dv)
    g = -np.abs(rnd(rng, B, T, H)) * 0.7
    beta = 1.0 / (1.0 + np.exp(-rnd(rng, B, T, H)))
    hz = rnd(rng, B, H, dk, dv) * 0.3 if h0 else None
    return q, k, v, g, beta, hz


def gdn2_inputs(rng, B=1, T=20, H=2, dk=5, dv=7, h0=True):
    q = unit(rnd(rng, B, T, H, dk))
    k = unit(rnd(rng, B, T, H, dk))
    v = rnd(rng, B, T, H, dv)
    g = -np.abs(rnd(rng, B, T, H, dk)) * 0.7
    b = 1.0 / (1.0 + np.exp(-rnd(rng, B, T, H, dk)))
    w = 1.0 / (1.0 + np.exp(-rnd(rng, B, T, H, dv)))
    hz = rnd(rng, B, H, dk, dv) * 0.3 if h0 else None
    return q, k, v, g, b, w, hz


def relerr(x, ref):
    return np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-300)


# ---------------------------------------------------------------- hand-worked golden values
def test_handworked_golden(oracle_lib):
    with open(os.path.join(HERE, "golden", "handworked_small.json")) as f:
        gold = json.load(f)
    c = gold["gdn"]
    toks = c["tokens"]
    T = len(toks)
    q = np.array([t["q"] for t in toks])[None, :, None, :]
    k = np.array([t["k"] for t in toks])[None, :, None, :]
    v = np.array([t["v"] for t in toks])[None, :, None, :]
    g = np.log(np.array([t["exp_g"] for t in toks]))[None, :, None]
    beta = np.array([t["beta"] for t in toks])[None, :, None]
    h0 = np.array(c["h0"])[None, None]
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 1.0, h0)
    np.testing.assert_allclose(o[0, :, 0], np.array(c["o"]), rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(hT[0, 0], np.array(c["hT"]), rtol=1e-15, atol=1e-15)
    assert T == 2

    c = gold["gdn2"]
    toks = c["tokens"]
    q = np.array([t["q"] for t in toks])[None, :, None, :]
    k = np.array([t["k"] for t in toks])[None, :, None, :]
    v = np.array([t["v"] for t in toks])[None, :, None, :]
    g = np.log(np.array([t["alpha"] for t in toks]))[None, :, None, :]
    b = np.array([t["b"] for t in toks])[None, :, None, :]
    w = np.array([t["w"] for t in toks])[None, :, None, :]
    h0 = np.array(c["h0"])[None, None]
    o, hT = oracle_lib.gdn2_fwd(q, k, v, g, b, w, 1.0, h0)
    np.testing.assert_allclose(o[0, :, 0], np.array(c["o"]), rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(hT[0, 0], np.array(c["hT"]), rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------- P1: no write, no decay
def test_p1_identity_when_beta_and_g_zero(oracle_lib):
    rng = np.random.default_rng(1)
    q, k, v, g, beta, h0 = gdn_inputs(rng)
    g[:] = 0.0
    beta[:] = 0.0
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.25, h0)
    assert np.array_equal(hT, h0)  # bit-exact: 1*x = x, 0*x = 0, x + 0 = x
    expect = 0.25 * np.einsum("btnk,bnkv->btnv", q, h0)
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- P2: exact retrieval after a full write
def test_p2_basis_key_full_write_is_exact(oracle_lib):
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 1, 16, 2, 6, 5
    q, k, v, g, beta, h0 = gdn_inputs(rng, B, T, H, dk, dv)
    g[:] = 0.0
    beta[:] = 1.0
    idx = rng.integers(0, dk, size=(B, T, H))
    k = np.zeros((B, T, H, dk))
    np.put_along_axis(k, idx[..., None], 1.0, axis=-1)
    q = k.copy()  # read back with the key just written
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 1.0, h0)
    # k_t^T S_t == v_t: the write stores x + (v - x) in the addressed row, which is v up to the one
    # rounding of (v - x) -- at most an ulp or two of |v|.
    tol = 4 * np.finfo(np.float64).eps * np.max(np.abs(v))
    np.testing.assert_allclose(o, v, rtol=0, atol=tol)
    for hh in range(H):
        np.testing.assert_allclose(hT[0, hh, idx[0, -1, hh]], v[0, -1, hh], rtol=0, atol=tol)
    # from a zero state the first write to a row is exact: S_i = 0 + (v - 0)
    o0, _ = oracle_lib.gdn_fwd(q[:, :1], k[:, :1], v[:, :1], g[:, :1], beta[:, :1], 1.0, None)
    assert np.array_equal(o0, v[:, :1])


def test_p2_unit_key_full_write(oracle_lib):
    rng = np.random.default_rng(3)
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=24)
    g[:] = 0.0
    beta[:] = 1.0
    o, _ = oracle_lib.gdn_fwd(k, k, v, g, beta, 1.0, h0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- read-out after the write, scale, beta on v
def test_readout_single_token_closed_form(oracle_lib):
    rng = np.random.default_rng(4)
    q, k, v, g, beta, _ = gdn_inputs(rng, T=1, H=3, dk=4, dv=6)
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.5, None)
    # from a zero state: S_0 = beta k v^T, o_0 = scale beta (k.q) v
    expect = 0.5 * beta[..., None] * np.sum(k * q, -1, keepdims=True) * v
    np.testing.assert_allclose(o, expect, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(hT[0], beta[0, 0][:, None, None] * np.einsum("hk,hv->hkv", k[0, 0], v[0, 0]),
                               rtol=1e-15, atol=1e-16)


# ---------------------------------------------------------------- P3: GDN-2 reduces to GDN bit-for-bit
def test_p3_gdn2_scalar_gates_equal_gdn_bitwise(oracle_lib):
    rng = np.random.default_rng(5)
    q, k, v, g, beta, h0 = gdn_inputs(rng, B=2, T=33, dk=6, dv=4)
    dk, dv = q.shape[-1], v.shape[-1]
    o1, h1 = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.4, h0)
    o2, h2 = oracle_lib.gdn2_fwd(q, k, v, np.repeat(g[..., None], dk, -1), np.repeat(beta[..., None], dk, -1),
                                 np.repeat(beta[..., None], dv, -1), 0.4, h0)
    assert np.array_equal(o1, o2) and np.array_equal(h1, h2)


def test_literal_page_form_matches(oracle_lib):
    rng = np.random.default_rng(6)
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=50)
    o0, h0_ = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0, form=0)
    o1, h1 = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0, form=1)
    assert relerr(o1, o0) < 1e-12 and relerr(h1, h0_) < 1e-12


# ---------------------------------------------------------------- P4: chunked form agrees with the recurrence
@pytest.mark.parametrize("C", [4, 8, 64])
@pytest.mark.parametrize("T", [1, 7, 64, 65, 130])
def test_p4_chunked_matches_recurrence_gdn(oracle_lib, C, T):
    from oracle.chunked import gdn_fwd_chunked
    rng = np.random.default_rng(100 + T + C)
    q, k, v, g, beta, h0 = gdn_inputs(rng, B=1, T=T, H=2, dk=8, dv=6)
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.35, h0)
    oc, hc = gdn_fwd_chunked(q, k, v, g, beta, 0.35, h0, C=C)
    assert relerr(oc, o) < 1e-10 and relerr(hc, hT) < 1e-10


@pytest.mark.parametrize("C,T", [(4, 13), (16, 64), (64, 130)])
def test_p4_chunked_matches_recurrence_gdn2(oracle_lib, C, T):
    from oracle.chunked import gdn2_fwd_chunked
    rng = np.random.default_rng(200 + T + C)
    q, k, v, g, b, w, h0 = gdn2_inputs(rng, B=1, T=T, H=2, dk=8, dv=6)
    o, hT = oracle_lib.gdn2_fwd(q, k, v, g, b, w, 0.35, h0)
    oc, hc = gdn2_fwd_chunked(q, k, v, g, b, w, 0.35, h0, C=C)
    assert relerr(oc, o) < 1e-10 and relerr(hc, hT) < 1e-10


def test_p4_chunked_varlen(oracle_lib):
    from oracle.chunked import gdn_fwd_chunked
    rng = np.random.default_rng(7)
    q, k, v, g, beta, _ = gdn_inputs(rng, B=1, T=150, H=2, dk=8, dv=6)
    cu = [0, 5, 69, 70, 150]
    h0 = rnd(rng, 4, 2, 8, 6) * 0.2
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.35, h0, cu_seqlens=cu)
    oc, hc = gdn_fwd_chunked(q, k, v, g, beta, 0.35, h0, cu_seqlens=cu, C=16)
    assert relerr(oc, o) < 1e-10 and relerr(hc, hT) < 1e-10


# ---------------------------------------------------------------- P5: full forget
def test_p5_full_forget(oracle_lib):
    rng = np.random.default_rng(8)
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=9)
    g[0, -1] = -np.inf
    _, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0)
    kt, vt, bt = k[0, -1], v[0, -1], beta[0, -1]
    for hh in range(q.shape[2]):
        assert np.array_equal(hT[0, hh], kt[hh][:, None] * (bt[hh] * vt[hh])[None, :])

    q, k, v, g, b, w, h0 = gdn2_inputs(rng, T=9)
    g[0, -1] = -np.inf
    _, hT = oracle_lib.gdn2_fwd(q, k, v, g, b, w, 0.3, h0)
    for hh in range(q.shape[2]):
        assert np.array_equal(hT[0, hh], k[0, -1, hh][:, None] * (w[0, -1, hh] * v[0, -1, hh])[None, :])


# ---------------------------------------------------------------- P6: pure decay closed form
def test_p6_pure_decay(oracle_lib):
    rng = np.random.default_rng(9)
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=40)
    beta[:] = 0.0
    _, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0)
    expect = np.exp(g.sum(axis=1))[..., None, None] * h0
    # 40 steps, each one exp and one multiply rounded: elementwise error <= ~80 ulp
    np.testing.assert_allclose(hT, expect, rtol=100 * np.finfo(np.float64).eps, atol=0)

    q, k, v, g, b, w, h0 = gdn2_inputs(rng, T=40)
    b[:] = 0.0
    w[:] = 0.0
    _, hT = oracle_lib.gdn2_fwd(q, k, v, g, b, w, 0.3, h0)
    expect = np.exp(g.sum(axis=1))[..., None] * h0  # row i (key channel) decays by prod exp(g_ti)
    np.testing.assert_allclose(hT, expect, rtol=100 * np.finfo(np.float64).eps, atol=0)


# ---------------------------------------------------------------- P7: split continuation (h0/hT resume)
def test_p7_split_continuation_bitwise(oracle_lib):
    rng = np.random.default_rng(10)
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=37)
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0)
    t0 = 15
    oa, ha = oracle_lib.gdn_fwd(q[:, :t0], k[:, :t0], v[:, :t0], g[:, :t0], beta[:, :t0], 0.3, h0)
    ob, hb = oracle_lib.gdn_fwd(q[:, t0:], k[:, t0:], v[:, t0:], g[:, t0:], beta[:, t0:], 0.3, ha)
    assert np.array_equal(np.concatenate([oa, ob], 1), o) and np.array_equal(hb, hT)


# ---------------------------------------------------------------- P8: brute force dense matrix products
def test_p8_dense_matrix_form(oracle_lib):
    rng = np.random.default_rng(11)
    dk, dv = 3, 5  # unequal, so a transposed state cannot pass
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=12, H=1, dk=dk, dv=dv)
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.6, h0)
    S = h0[0, 0].copy()
    for t in range(12):
        kt, vt, bt = k[0, t, 0], v[0, t, 0], beta[0, t, 0]
        S = (np.eye(dk) - bt * np.outer(kt, kt)) @ (np.exp(g[0, t, 0]) * S) + bt * np.outer(kt, vt)
        np.testing.assert_allclose(o[0, t, 0], 0.6 * S.T @ q[0, t, 0], rtol=1e-12, atol=1e-13)
    assert relerr(hT[0, 0], S) < 1e-13

    q, k, v, g, b, w, h0 = gdn2_inputs(rng, T=12, H=1, dk=dk, dv=dv)
    o, hT = oracle_lib.gdn2_fwd(q, k, v, g, b, w, 0.6, h0)
    S = h0[0, 0].copy()
    for t in range(12):
        kt = k[0, t, 0]
        S = (np.eye(dk) - np.outer(kt, b[0, t, 0] * kt)) @ np.diag(np.exp(g[0, t, 0])) @ S \
            + np.outer(kt, w[0, t, 0] * v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], 0.6 * S.T @ q[0, t, 0], rtol=1e-12, atol=1e-13)
    assert relerr(hT[0, 0], S) < 1e-13


# ---------------------------------------------------------------- P9: value columns are independent
def test_p9_value_column_permutation(oracle_lib):
    rng = np.random.default_rng(12)
    q, k, v, g, beta, h0 = gdn_inputs(rng, T=21)
    perm = rng.permutation(v.shape[-1])
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0)
    op, hp = oracle_lib.gdn_fwd(q, k, v[..., perm], g, beta, 0.3, h0[..., perm])
    assert np.array_equal(op, o[..., perm]) and np.array_equal(hp, hT[..., perm])


# ---------------------------------------------------------------- varlen: state resets at each boundary
def test_varlen_equals_separate_sequences(oracle_lib):
    rng = np.random.default_rng(13)
    q, k, v, g, beta, _ = gdn_inputs(rng, B=1, T=30, H=2)
    cu = [0, 7, 7, 30]  # includes an empty sequence
    h0 = rnd(rng, 3, 2, q.shape[-1], v.shape[-1])
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0, cu_seqlens=cu)
    for n in range(3):
        a, b_ = cu[n], cu[n + 1]
        if b_ == a:
            assert np.array_equal(hT[n], h0[n])  # zero-length sequence: hT = h0
            continue
        on, hn = oracle_lib.gdn_fwd(q[:, a:b_], k[:, a:b_], v[:, a:b_], g[:, a:b_], beta[:, a:b_], 0.3, h0[n:n + 1])
        assert np.array_equal(o[:, a:b_], on) and np.array_equal(hT[n], hn[0])


def test_units_subset_and_threads(oracle_lib):
    rng = np.random.default_rng(14)
    q, k, v, g, beta, h0 = gdn_inputs(rng, B=2, T=10, H=3)
    o, hT = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0)
    os_, hs = oracle_lib.gdn_fwd(q, k, v, g, beta, 0.3, h0, units=[(1, 2), (0, 1)], threads=2)
    assert np.array_equal(os_[1, :, 2], o[1, :, 2]) and np.array_equal(hs[0, 1], hT[0, 1])
    assert np.isnan(os_[0, :, 0]).all()
