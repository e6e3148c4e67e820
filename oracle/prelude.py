"""fp64 oracle of the token mixer's prelude and epilogue (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import this module; it shares no
code with the CUDA path.  What it computes, in the order the pages give it:

  * Short convolution (GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755, section "Short
    convolution": q, k and v each pass a depthwise causal convolution with kernel size 4 and a SiLU activation;
    at inference the 3 previous inputs are cached).  Per channel c, with taps w[c, 0..3] and no bias:
        y[t, c] = silu( sum_{j=0..3} w[c, j] * x[t - 3 + j, c] )
    so w[c, 3] weighs the current token (a causal Conv1d with 3 zeros of left padding).  Inputs before the
    sequence start are the cached state (oldest first) or 0; the returned state is the last 3 inputs.
  * L2 normalisation of q and k over each head's channels (same section of the walkthrough, qk_norm = l2;
    the Gated DeltaNet-2 article, section "Diseno de bloques y modelo hibrido": the query and key paths use
    projection, short causal convolution, SiLU and L2 normalisation; the value path has no normalisation):
        x / sqrt(sum x^2 + eps)
  * Gates (walkthrough, section "Gating"): g = -exp(A_log) * softplus(a + dt_bias) with A_log and dt_bias per
    head, beta = sigmoid(b); the Gated DeltaNet-2 erase and write gates are sigmoids of their own branches.
  * Output gate (walkthrough, section "Data flow" step 5: a fused RMSNorm with a Swish gate; the Gated
    DeltaNet-2 article: the recurrent output is RMS-normalised and multiplied by a SiLU output gate):
        y = o / sqrt(mean(o^2) + eps) * weight * silu(z)     (per token and head, over the dv channels)

Readings where the pages are silent: the tap order above, no convolution bias, eps = 1e-6 for the L2 norm and
1e-5 for the RMS norm (both arguments), one RMS-norm weight vector of length dv shared by the heads.
Pinned by ``tests/test_oracle_prelude.py`` (numpy.convolve, closed forms, invariants, split continuation).
"""
from __future__ import annotations

import numpy as np

K = 4  # taps of the short convolution


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def softplus(x):
    return np.logaddexp(0.0, np.asarray(x, dtype=np.float64))


def _spans(B, T, cu_seqlens):
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in cu_seqlens]
    return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def short_conv(x, w, state=None, cu_seqlens=None, activation=True):
    """Causal depthwise convolution of x [B, T, C] with taps w [C, 4], then SiLU (if ``activation``).

    ``state`` [N, C, 3] (N sequences: B rows, or the packed sequences of ``cu_seqlens``) holds the 3 inputs before
    each sequence, oldest first; None means zeros.  Returns (y [B, T, C], final state [N, C, 3]).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, T, C = x.shape
    spans = _spans(B, T, cu_seqlens)
    y = np.zeros_like(x)
    out_state = np.zeros((len(spans), C, K - 1))
    for n, (row, t0, t1) in enumerate(spans):
        hist = np.zeros((K - 1, C)) if state is None else np.asarray(state[n], dtype=np.float64).T
        seq = np.concatenate([hist, x[row, t0:t1]], axis=0)  # [3 + L, C]
        for t in range(t1 - t0):
            window = seq[t:t + K]  # inputs t-3 .. t of the sequence
            y[row, t0 + t] = np.sum(window * w.T, axis=0)
        out_state[n] = seq[-(K - 1):].T
    return (silu(y) if activation else y), out_state


def l2norm(x, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def decay_gate(a, A_log, dt_bias):
    """g = -exp(A_log) * softplus(a + dt_bias) for a [B, T, H] or [B, T, H, G] (A_log, dt_bias per head)."""
    a = np.asarray(a, dtype=np.float64)
    shape = (1, 1, -1) + (1,) * (a.ndim - 3)
    A = np.exp(np.asarray(A_log, dtype=np.float64)).reshape(shape)
    return -A * softplus(a + np.asarray(dt_bias, dtype=np.float64).reshape(shape))


def prelude(xq, xk, xv, wq, wk, wv, a, A_log, dt_bias, b, c=None, conv_state=None, cu_seqlens=None, eps=1e-6):
    """The whole prelude.  xq, xk [B, T, H, dk], xv [B, T, H, dv]; wq, wk [H*dk, 4], wv [H*dv, 4]; conv_state
    [N, 2 H dk + H dv, 3] (q channels, then k, then v) or None; a [B, T, H(, G)]; b [B, T, H(, Gb)]; optional c.

    Returns dict q, k [B, T, H, dk] (L2-normalised), v [B, T, H, dv], g, beta (, w) and conv_state.
    """
    B, T, H, dk = np.shape(xq)
    dv = np.shape(xv)[-1]
    st = [None, None, None]
    if conv_state is not None:
        cs = np.asarray(conv_state, dtype=np.float64)
        st = [cs[:, :H * dk], cs[:, H * dk:2 * H * dk], cs[:, 2 * H * dk:]]
    q, sq = short_conv(np.reshape(xq, (B, T, H * dk)), wq, st[0], cu_seqlens)
    k, sk = short_conv(np.reshape(xk, (B, T, H * dk)), wk, st[1], cu_seqlens)
    v, sv = short_conv(np.reshape(xv, (B, T, H * dv)), wv, st[2], cu_seqlens)
    out = {"q": l2norm(q.reshape(B, T, H, dk), eps), "k": l2norm(k.reshape(B, T, H, dk), eps),
           "v": v.reshape(B, T, H, dv), "g": decay_gate(a, A_log, dt_bias), "beta": sigmoid(b),
           "conv_state": np.concatenate([sq, sk, sv], axis=1)}
    if c is not None:
        out["w"] = sigmoid(c)
    return out


def output_gate(o, z, weight, eps=1e-5):
    """y = o / sqrt(mean(o^2) + eps) * weight * silu(z), over the last axis (dv) of o, z [..., dv]."""
    o = np.asarray(o, dtype=np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o / rms * np.asarray(weight, dtype=np.float64) * silu(z)
