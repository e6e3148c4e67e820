"""Pins of the prelude / epilogue oracle (oracle/prelude.py) against facts other than its own formulas:
numpy.convolve, one-hot taps, closed forms and identities of SiLU, sigmoid and softplus, split continuation
through the conv cache, packed = separate sequences, and scale invariance of the RMS norm."""
import math

import numpy as np
import pytest

from oracle import prelude as P


def test_short_conv_is_numpy_convolve_per_channel():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 37, 5))
    w = rng.standard_normal((5, 4))
    y, _ = P.short_conv(x, w, activation=False)
    for b in range(2):
        for c in range(5):
            # causal Conv1d with 3 zeros of left padding == full convolution with the reversed taps, first T terms
            ref = np.convolve(x[b, :, c], w[c, ::-1])[:37]
            assert np.allclose(y[b, :, c], ref, rtol=0, atol=1e-12)


def test_one_hot_taps_are_identity_and_delay():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 9, 3))
    cur = np.zeros((3, 4))
    cur[:, 3] = 1.0
    y, st = P.short_conv(x, cur, activation=False)
    assert np.array_equal(y, x)
    assert np.array_equal(st[0], x[0, -3:].T)  # the cache is the last three inputs, oldest first
    old = np.zeros((3, 4))
    old[:, 0] = 1.0
    y, _ = P.short_conv(x, old, activation=False)
    assert np.array_equal(y[0, 3:], x[0, :-3]) and np.array_equal(y[0, :3], np.zeros((3, 3)))


def test_split_continuation_through_the_cache_is_exact():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((2, 20, 6))
    w = rng.standard_normal((6, 4))
    s0 = rng.standard_normal((2, 6, 3))
    y, s = P.short_conv(x, w, s0)
    for t0 in (1, 2, 3, 7):
        ya, sa = P.short_conv(x[:, :t0], w, s0)
        yb, sb = P.short_conv(x[:, t0:], w, sa)
        assert np.array_equal(np.concatenate([ya, yb], 1), y) and np.array_equal(sb, s)


def test_packed_sequences_equal_separate_ones():
    rng = np.random.default_rng(3)
    lens = [5, 1, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = rng.standard_normal((1, int(cu[-1]), 4))
    w = rng.standard_normal((4, 4))
    st = rng.standard_normal((4, 4, 3))
    y, s = P.short_conv(x, w, st, cu_seqlens=cu)
    for n in range(4):
        yn, sn = P.short_conv(x[:, cu[n]:cu[n + 1]], w, st[n:n + 1])
        assert np.array_equal(y[:, cu[n]:cu[n + 1]], yn) and np.array_equal(s[n], sn[0])
    assert np.array_equal(s[2], st[2])  # an empty sequence keeps its cache


def test_activation_and_gate_identities():
    x = np.linspace(-30, 30, 121)
    assert np.allclose(P.silu(x) - P.silu(-x), x, rtol=0, atol=1e-12)
    assert P.silu(0.0) == 0.0
    assert np.allclose(P.sigmoid(x) + P.sigmoid(-x), 1.0, rtol=0, atol=1e-15)
    assert P.sigmoid(0.0) == 0.5
    assert np.allclose(P.softplus(x) - P.softplus(-x), x, rtol=0, atol=1e-12)
    assert abs(P.softplus(0.0) - math.log(2.0)) < 1e-15
    A_log = np.log(np.array([1.0, 4.0, 16.0]))
    dt_bias = np.array([0.1, -0.2, 0.3])
    g = P.decay_gate(-dt_bias[None, None, :] * np.ones((2, 3, 3)), A_log, dt_bias)
    assert np.allclose(g, -np.exp(A_log) * math.log(2.0), rtol=1e-15, atol=0)  # softplus(0) = ln 2
    g_deep = P.decay_gate(np.full((1, 1, 3), -60.0), A_log, dt_bias)
    assert np.all(g_deep < 0) and np.all(g_deep > -1e-20)  # no decay for very negative inputs
    g_ch = P.decay_gate(np.zeros((1, 2, 3, 8)), A_log, dt_bias)  # per-channel form broadcasts per head
    assert np.allclose(g_ch[..., 0], g_ch[..., 5]) and g_ch.shape == (1, 2, 3, 8)


def test_l2norm_unit_length_and_direction():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 4, 128)) * 7.0
    y = P.l2norm(x, eps=0.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=0, atol=1e-14)
    assert np.allclose(y * np.linalg.norm(x, axis=-1, keepdims=True), x, rtol=1e-14, atol=0)


def test_output_gate_rms_and_scale_invariance():
    rng = np.random.default_rng(5)
    o = rng.standard_normal((2, 3, 4, 64))
    z = rng.standard_normal((2, 3, 4, 64))
    wt = rng.uniform(0.5, 1.5, 64)
    y = P.output_gate(o, z, wt, eps=0.0)
    assert np.allclose(P.output_gate(o * 37.5, z, wt, eps=0.0), y, rtol=1e-13, atol=0)
    n = y / (wt * P.silu(z))
    assert np.allclose(np.sqrt(np.mean(n * n, axis=-1)), 1.0, rtol=1e-13, atol=0)
    # with weight 1 and z -> large, silu(z) -> z: the gate passes the normalised output scaled by z
    big = np.full_like(z, 40.0)
    yb = P.output_gate(o, big, np.ones(64), eps=0.0)
    assert np.allclose(yb / 40.0, o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True)), rtol=1e-12, atol=0)


def test_prelude_wires_each_path():
    rng = np.random.default_rng(6)
    B, T, H, dk, dv = 1, 10, 2, 8, 16
    xq, xk = rng.standard_normal((2, B, T, H, dk))
    xv = rng.standard_normal((B, T, H, dv))
    wq, wk = rng.standard_normal((2, H * dk, 4))
    wv = rng.standard_normal((H * dv, 4))
    a, b = rng.standard_normal((2, B, T, H))
    out = P.prelude(xq, xk, xv, wq, wk, wv, a, np.zeros(H), np.zeros(H), b)
    assert np.allclose(np.linalg.norm(out["q"], axis=-1), 1.0, atol=1e-6)
    v_ref, _ = P.short_conv(xv.reshape(B, T, H * dv), wv)
    assert np.array_equal(out["v"].reshape(B, T, H * dv), v_ref)  # the value path has no normalisation
    assert out["conv_state"].shape == (B, 2 * H * dk + H * dv, 3)
    assert np.all(out["g"] < 0) and np.all((out["beta"] > 0) & (out["beta"] < 1))
