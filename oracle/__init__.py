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
invariants, a hand-worked example under ``tests/golden/`` and brute-force dense products).
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
