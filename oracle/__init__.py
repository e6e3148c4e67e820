"""fp64 oracle for the gated delta rule forward pass (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this
package.  It shares no code with the CUDA path: the recurrence lives in ``gdn_oracle.c`` (plain C,
fp64, compiled by ``oracle/build.py``); the naive chunked restatement used to self-check the
algebra lives in ``oracle/chunked.py`` (numpy fp64).

Definitions followed (see the C file's header for the step-by-step statement):
  * GDN -- GatedDeltaNet data-flow walkthrough (yfxerp.com/news/367755), section "Delta Rule:
    predict first, then correct" (the token loop) and section "Gating" (g < 0, beta in (0,1)).
  * GDN-2 -- NVIDIA Gated DeltaNet-2 article (7minutos.es), section "Regla-2 del Delta cerrado".

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py`` (closed forms,
invariants, a hand-worked example under ``tests/golden/`` and brute-force dense products); the reverse
mode (``gdn_vjp`` / ``gdn2_vjp``, ``gdn_vjp.c``) by ``tests/test_oracle_vjp.py`` (central finite differences
of the forward recurrence, the GDN-2 -> GDN reduction, and zero gradients where an input cannot matter).
"""
from __future__ import annotations

import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None

_dp = ctypes.POINTER(ctypes.c_double)


def _load():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "liboracle.so")
        if not os.path.exists(path):
            from . import build as _b
            _b.build()
        lib = ctypes.CDLL(path)
        i = ctypes.c_int
        lib.oracle_gdn_unit.argtypes = [_dp] * 5 + [ctypes.c_double, _dp, _dp, _dp] + [i] * 10 + [_dp, _dp]
        lib.oracle_gdn_unit.restype = None
        lib.oracle_gdn2_unit.argtypes = [_dp] * 6 + [ctypes.c_double, _dp, _dp, _dp] + [i] * 9 + [_dp, _dp]
        lib.oracle_gdn2_unit.restype = None
        lib.oracle_vjp_unit.argtypes = [i] + [_dp] * 6 + [ctypes.c_double] + [_dp] * 10 + [i] * 9
        lib.oracle_vjp_unit.restype = i
        _LIB = lib
    return _LIB


def _ptr(a):
    if a is None:
        return ctypes.cast(None, _dp)
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_dp)


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def seq_ranges(B: int, T: int, cu_seqlens=None):
    """(row, t0, t1) for every sequence: the batch rows, or the packed spans of ``cu_seqlens``."""
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in cu_seqlens]
    assert B == 1 and cu[0] == 0 and cu[-1] == T
    return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def gdn_fwd(q, k, v, g, beta, scale, h0=None, cu_seqlens=None, units=None, threads=1, form=0):
    """fp64 GDN recurrence.  Returns (o [B,T,H,dv], hT [n_seq,H,dk,dv]).

    ``units`` optionally restricts the work to a list of (n, h) pairs; rows of ``o`` and ``hT``
    outside those units are left NaN.  ``threads`` runs independent units concurrently.
    """
    q, k, v, g, beta, h0 = map(_f64, (q, k, v, g, beta, h0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    seqs = seq_ranges(B, T, cu_seqlens)
    o = np.full((B, T, H, dv), np.nan)
    hT = np.full((len(seqs), H, dk, dv), np.nan)
    lib = _load()
    if units is None:
        units = [(n, h) for n in range(len(seqs)) for h in range(H)]

    def run(unit):
        n, h = unit
        row, t0, t1 = seqs[n]
        S = np.empty(dk * dv)
        u = np.empty(dv)
        lib.oracle_gdn_unit(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(h0),
                            _ptr(o), _ptr(hT), T, H, dk, dv, row, t0, t1, n, h, form, _ptr(S), _ptr(u))

    _map(run, units, threads)
    return o, hT


def gdn2_fwd(q, k, v, g, b, w, scale, h0=None, cu_seqlens=None, units=None, threads=1):
    """fp64 GDN-2 recurrence with per-channel decay g[..,dk], erase gate b[..,dk], write gate w[..,dv]."""
    q, k, v, g, b, w, h0 = map(_f64, (q, k, v, g, b, w, h0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    seqs = seq_ranges(B, T, cu_seqlens)
    o = np.full((B, T, H, dv), np.nan)
    hT = np.full((len(seqs), H, dk, dv), np.nan)
    lib = _load()
    if units is None:
        units = [(n, h) for n in range(len(seqs)) for h in range(H)]

    def run(unit):
        n, h = unit
        row, t0, t1 = seqs[n]
        S = np.empty(dk * dv)
        u = np.empty(dv)
        lib.oracle_gdn2_unit(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), float(scale), _ptr(h0),
                             _ptr(o), _ptr(hT), T, H, dk, dv, row, t0, t1, n, h, _ptr(S), _ptr(u))

    _map(run, units, threads)
    return o, hT


def _map(fn, items, threads):
    if threads <= 1 or len(items) <= 1:
        for it in items:
            fn(it)
        return
    # ctypes releases the GIL for the duration of each C call, so threads run units in parallel.
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fn, items))


def _vjp(mode, q, k, v, g, b, w, scale, h0, d_o, dhT, cu_seqlens, units, threads):
    q, k, v, g, b, w, h0, d_o, dhT = map(_f64, (q, k, v, g, b, w, h0, d_o, dhT))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    seqs = seq_ranges(B, T, cu_seqlens)
    out = {"dq": np.full(q.shape, np.nan), "dk": np.full(k.shape, np.nan), "dv": np.full(v.shape, np.nan),
           "dg": np.full(g.shape, np.nan), "db": np.full(b.shape, np.nan),
           "dw": None if w is None else np.full(w.shape, np.nan), "dh0": np.full((len(seqs), H, dk, dv), np.nan)}
    lib = _load()
    if units is None:
        units = [(n, h) for n in range(len(seqs)) for h in range(H)]

    def run(unit):
        n, h = unit
        row, t0, t1 = seqs[n]
        rc = lib.oracle_vjp_unit(mode, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), float(scale), _ptr(h0),
                                 _ptr(d_o), _ptr(dhT), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                 _ptr(out["dg"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dh0"]), T, H, dk, dv,
                                 row, t0, t1, n, h)
        if rc != 0:
            raise MemoryError("oracle_vjp_unit: scratch allocation failed")

    _map(run, units, threads)
    return out


def gdn_vjp(q, k, v, g, beta, scale, h0, d_o, dhT=None, cu_seqlens=None, units=None, threads=1):
    """fp64 reverse mode of :func:`gdn_fwd`: gradients of <d_o, o> + <dhT, hT> with respect to every input.

    Returns dict dq, dk [B,T,H,dk], dv [B,T,H,dv], dg, dbeta [B,T,H], dh0 [n_seq,H,dk,dv].
    """
    out = _vjp(0, q, k, v, g, beta, None, scale, h0, d_o, dhT, cu_seqlens, units, threads)
    out["dbeta"] = out.pop("db")
    out.pop("dw")
    return out


def gdn2_vjp(q, k, v, g, b, w, scale, h0, d_o, dhT=None, cu_seqlens=None, units=None, threads=1):
    """fp64 reverse mode of :func:`gdn2_fwd`.  Returns dq, dk, dv, dg, db [B,T,H,dk], dw [B,T,H,dv], dh0."""
    return _vjp(1, q, k, v, g, b, w, scale, h0, d_o, dhT, cu_seqlens, units, threads)
