"""Naive chunked form of the GDN / GDN-2 forward pass in numpy fp64 (TEST INFRASTRUCTURE ONLY).

This restates the chunkwise-parallel algorithm the kernels follow -- parallel inside a chunk of C
tokens, one state matrix handed from chunk to chunk (GatedDeltaNet data-flow walkthrough,
yfxerp.com/news/367755, section "Chunked parallelism: how the Triton kernels turn serial into
parallel"; Gated DeltaNet-2 article, 7minutos.es, section "Entrenamiento fragmentado", C = 64) --
in the plainest form, so that its agreement with the token recurrence (``oracle.gdn_fwd``) checks
the algebra.  It is slow on purpose: no blocking, Gamma computed as exp(G_r - G_s) directly, and
(I + A)^-1 formed by explicit forward substitution.

Per chunk with incoming state h (dk x dv) and chunk-local cumulative log-decay G_r = sum_{s<=r} g_s:
  GDN   A_rs = beta_r (k_r . k_s) exp(G_r - G_s)                     (s < r, else 0)
        W = (I+A)^-1 diag(beta e^G) K ,   U~ = (I+A)^-1 diag(beta) V
  GDN-2 A_rs = sum_i b_ri k_ri k_si exp(G_ri - G_si)                  (s < r)
        W = (I+A)^-1 (e^G . b . K) ,        U~ = (I+A)^-1 (w . V)
  U = U~ - W h
  O = scale [ (Q . e^G) h + (P . M<=) U ],  P_rs = sum_i q_ri k_si exp(G_ri - G_si)  (scalar G for GDN)
  h <- Diag(e^{G_last}) h + sum_s (k_s . e^{G_last - G_s}) u_s^T
Chunks start at each sequence start; the last chunk of a sequence may be partial.
"""
from __future__ import annotations

import numpy as np

from . import seq_ranges


def unit_lower_inverse(A):
    """(I + A)^-1 for strictly lower-triangular A, by forward substitution on the identity."""
    n = A.shape[0]
    Tm = np.zeros_like(A)
    for r in range(n):
        e = np.zeros(n)
        e[r] = 1.0
        # row r of T solves T_r + sum_{s<r} A_rs T_s = e_r  (T is unit lower triangular)
        Tm[r] = e - A[r, :r] @ Tm[:r]
    return Tm


def _chunk(qc, kc, vc, Gc, bk, wv, h, scale):
    """One chunk.  Gc: [L] (GDN) or [L,dk] (GDN-2) cumulative log-decay; bk: [L,dk] erase-side
    weights (beta_r broadcast, or b); wv: [L,dv] write-side scaled values (beta.v or w.v)."""
    L, dk = kc.shape
    Gm = Gc if Gc.ndim == 2 else np.repeat(Gc[:, None], dk, axis=1)
    A = np.zeros((L, L))
    P = np.zeros((L, L))
    for r in range(L):
        for s in range(L):
            dec = np.exp(Gm[r] - Gm[s]) if s <= r else None
            if s < r:
                A[r, s] = np.sum(bk[r] * kc[r] * kc[s] * dec)
            if s <= r:
                P[r, s] = np.sum(qc[r] * kc[s] * dec)
    Tm = unit_lower_inverse(A)
    W = Tm @ (np.exp(Gm) * bk * kc)
    Ut = Tm @ wv
    U = Ut - W @ h
    O = scale * ((qc * np.exp(Gm)) @ h + P @ U)
    Kt = kc * np.exp(Gm[L - 1][None, :] - Gm)
    h_new = np.exp(Gm[L - 1])[:, None] * h + Kt.T @ U
    return O, h_new


def _run(q, k, v, gate_fn, scale, h0, cu_seqlens, C):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    seqs = seq_ranges(B, T, cu_seqlens)
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((len(seqs), H, dk, dv))
    for n, (row, t0, t1) in enumerate(seqs):
        for hh in range(H):
            h = np.zeros((dk, dv)) if h0 is None else np.array(h0[n, hh], dtype=np.float64)
            for c0 in range(t0, t1, C):
                c1 = min(c0 + C, t1)
                sl = (row, slice(c0, c1), hh)
                Gc, bk, wv = gate_fn(sl)
                O, h = _chunk(q[sl], k[sl], v[sl], Gc, bk, wv, h, scale)
                o[sl] = O
            hT[n, hh] = h
    return o, hT


def gdn_fwd_chunked(q, k, v, g, beta, scale, h0=None, cu_seqlens=None, C=64):
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    dk = q.shape[-1]

    def gate(sl):
        G = np.cumsum(g[sl])
        bt = beta[sl]
        return G, np.repeat(bt[:, None], dk, axis=1), bt[:, None] * v[sl]

    return _run(q, k, v, gate, scale, h0, cu_seqlens, C)


def gdn2_fwd_chunked(q, k, v, g, b, w, scale, h0=None, cu_seqlens=None, C=64):
    q, k, v, g, b, w = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, b, w))

    def gate(sl):
        return np.cumsum(g[sl], axis=0), b[sl], w[sl] * v[sl]

    return _run(q, k, v, gate, scale, h0, cu_seqlens, C)
