"""Thin Python binding over libgdn's C ABI (argument marshalling only).

Every step of the forward pass runs in libgdn's CUDA kernels; this module only checks torch tensors,
allocates outputs with torch and passes raw pointers and the current CUDA stream.  There is no CPU
fallback: without the built library or a CUDA device every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, GDN_ERR_DEVICE_ARG = range(6)
GDN_F32, GDN_BF16 = 0, 1
KERNELS = {"auto": 0, "simt": 1, "tc": 2}
KERNEL_NAMES = {v: k for k, v in KERNELS.items()}

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"libgdn status {status}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgdn.so and declare its signatures.  Raises if the library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libgdn.so not found at {path}: build it with "
                           "`python -m gated_delta_rule_105_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, fp, i, f, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.gdn_workspace_bytes.argtypes = [i] * 7
    lib.gdn_workspace_bytes.restype = sz
    lib.gdn2_workspace_bytes.argtypes = [i] * 7
    lib.gdn2_workspace_bytes.restype = sz
    lib.gdn_kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp] + [i] * 8 + [vp, i, vp, sz, vp]
    lib.gdn_kda_chunk_fwd.restype = i
    lib.gdn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp] + [i] * 8 + [vp, i, vp, sz, vp]
    lib.gdn_chunk_fwd.restype = i
    lib.gdn_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp] + [i] * 8 + [vp, i, vp]
    lib.gdn_chunk_fwd_noalloc.restype = i
    lib.gdn2_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, f, fp, vp, fp] + [i] * 8 + [vp, i, vp, sz, vp]
    lib.gdn2_chunk_fwd.restype = i
    lib.gdn_set_kernel.argtypes = [i]
    lib.gdn_set_kernel.restype = i
    lib.gdn_last_kernel.argtypes = []
    lib.gdn_last_kernel.restype = i
    lib.gdn_check_error.argtypes = [vp]
    lib.gdn_check_error.restype = i
    lib.gdn_status_string.argtypes = [i]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_last_error.argtypes = []
    lib.gdn_last_error.restype = ctypes.c_char_p
    lib.gdn_debug_umma_selftest.argtypes = [vp, vp, vp, i, vp]
    lib.gdn_debug_umma_selftest.restype = i
    lib.gdn_profile_enable.argtypes = [i]
    lib.gdn_profile_enable.restype = i
    lib.gdn_profile_take.argtypes = [i, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]
    lib.gdn_profile_take.restype = i
    for name in ("gdn_decode_fwd", "gdn_kda_decode_fwd"):
        getattr(lib, name).argtypes = [vp, vp, vp, fp, fp, f, fp, vp] + [i] * 6 + [vp]
        getattr(lib, name).restype = i
    lib.gdn2_decode_fwd.argtypes = [vp, vp, vp, fp, fp, fp, f, fp, vp] + [i] * 6 + [vp]
    lib.gdn2_decode_fwd.restype = i
    lib.gdn_prelude_fwd.argtypes = [vp] * 11 + [fp, i, fp, fp, i, fp, fp, i, vp, vp, vp] + [i] * 5 + [i, f, vp, i, vp]
    lib.gdn_prelude_fwd.restype = i
    lib.gdn_output_gate_fwd.argtypes = [vp, vp, fp, vp, ctypes.c_longlong, i, i, f, vp]
    lib.gdn_output_gate_fwd.restype = i
    lib.gdn_bwd_workspace_bytes.argtypes = [i] * 7
    lib.gdn_bwd_workspace_bytes.restype = sz
    lib.gdn_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp] + [fp] * 6 + [i] * 6 + [i, vp, i, vp, sz, vp]
    lib.gdn_chunk_bwd.restype = i
    lib.gdn2_bwd_workspace_bytes.argtypes = [i] * 7
    lib.gdn2_bwd_workspace_bytes.restype = sz
    lib.gdn2_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, f, fp, vp, fp] + [fp] * 7 + [i] * 6 + [i, vp, i, vp, sz, vp]
    lib.gdn2_chunk_bwd.restype = i
    lib.gdn_kda_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp] + [fp] * 6 + [i] * 6 + [i, vp, i, vp, sz, vp]
    lib.gdn_kda_chunk_bwd.restype = i
    lib.gdn_debug_stall.argtypes = [i]
    lib.gdn_debug_stall.restype = i
    _lib = lib
    return lib


def _raise_on(status: int):
    if status != GDN_OK:
        lib = load_library()
        raise GdnError(status, f"{lib.gdn_status_string(status).decode()}: {lib.gdn_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_dev(name, t, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libgdn has no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _dtype_code(t):
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise ValueError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def set_kernel(name: str) -> None:
    """Select the kernel family ("auto", "simt" or "tc") for later calls (process-wide)."""
    _raise_on(load_library().gdn_set_kernel(KERNELS[name]))


def last_kernel() -> str:
    return KERNEL_NAMES[load_library().gdn_last_kernel()]


def debug_stall(on: bool) -> None:
    """Diagnostic of the device time-out path (``gdn_debug_stall``): while on, tensor-core GDN calls make a
    pipeline wait run out; ``check_error`` then raises with status GDN_ERR_TIMEOUT."""
    _raise_on(load_library().gdn_debug_stall(1 if on else 0))


def check_error(stream=None) -> None:
    """Synchronise the stream and raise if a kernel reported a device-side error."""
    s = torch.cuda.current_stream() if stream is None else stream
    _raise_on(load_library().gdn_check_error(ctypes.c_void_p(s.cuda_stream)))


PROFILE_KERNELS = {"gdn_simt_fwd_kernel": 0, "gdn_tc_wy_kernel": 1, "gdn_tc_fwd_kernel": 2, "gdn2_tc_prep_kernel": 3,
                   "gdn2_tc_fwd_kernel": 4, "gdn_decode_kernel": 5, "gdn_prelude_kernel": 6,
                   "gdn_output_gate_kernel": 7, "gdn_bwd_kernels": 8}


def profile_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events on its stream (see ``gdn_profile_take``)."""
    _raise_on(load_library().gdn_profile_enable(1 if on else 0))


def profile_take() -> dict:
    """{kernel name: (launches, total device ms)} of the launches recorded since the last take."""
    out = {}
    for name, kid in PROFILE_KERNELS.items():
        n, ms = ctypes.c_int(0), ctypes.c_double(0.0)
        _raise_on(load_library().gdn_profile_take(kid, ctypes.byref(n), ctypes.byref(ms)))
        if n.value:
            out[name] = (n.value, ms.value)
    return out


def umma_selftest(A, B, mode):
    """Runs the tensor-core layout self-test (see ``gdn_debug_umma_selftest``); returns D = A B (fp32)."""
    _check_dev("A", A, torch.float32)
    _check_dev("B", B, torch.float32)
    D = torch.empty((A.shape[0], B.shape[1]), dtype=torch.float32, device=A.device)
    st = load_library().gdn_debug_umma_selftest(_ptr(A), _ptr(B), _ptr(D), int(mode),
                                                 ctypes.c_void_p(torch.cuda.current_stream(A.device).cuda_stream))
    _raise_on(st)
    return D


def _prep(q, k, v, h0, cu_seqlens, o, hT, output_final_state, o_dtype):
    _check_dev("q", q)
    dt = q.dtype
    o_dtype = dt if o_dtype is None else o_dtype
    if o_dtype not in (torch.float32, dt):
        raise ValueError(f"o_dtype must be float32 or q's dtype, got {o_dtype}")
    _check_dev("k", k, dt)
    _check_dev("v", v, dt)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B,T,H,dk] and v [B,T,H,dv] with matching B, T, H")
    n_seq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None:
        _check_dev("cu_seqlens", cu_seqlens, torch.int32)
    _check_dev("h0", h0, torch.float32)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=o_dtype, device=q.device)
    elif o.dtype != o_dtype:
        raise ValueError(f"o must be {o_dtype}")
    if hT is None and output_final_state:
        hT = torch.empty((n_seq, H, dk, dv), dtype=torch.float32, device=q.device)
    return B, T, H, dk, dv, n_seq, o, hT


def workspace_bytes(B, T, H, dk, dv, BT=64, n_seqs=0) -> int:
    """Device workspace (bytes) a call with these sizes can use: the tensor-core path of bf16 inputs keeps the
    WY factors of every chunk there; 0 when no path needs any."""
    return int(load_library().gdn_workspace_bytes(B, T, H, dk, dv, BT, n_seqs))


def gdn2_workspace_bytes(B, T, H, dk, dv, BT=64, n_seqs=0) -> int:
    """Device workspace (bytes) the tensor-core path of ``gdn2_chunk_fwd`` / ``gdn_kda_chunk_fwd`` can use."""
    return int(load_library().gdn2_workspace_bytes(B, T, H, dk, dv, BT, n_seqs))


def _workspace(q, B, T, H, dk, dv, BT, n_seqs, workspace, gdn2=False):
    if workspace is not None:
        _check_dev("workspace", workspace, torch.uint8)
        return workspace
    if q.dtype != torch.bfloat16:
        return None
    nbytes = (gdn2_workspace_bytes if gdn2 else workspace_bytes)(B, T, H, dk, dv, BT, n_seqs)
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes > 0 else None


def gdn_chunk_fwd(q, k, v, g, beta, scale=None, h0=None, output_final_state=True, cu_seqlens=None, BT=64,
                  o=None, hT=None, o_dtype=None, workspace=None):
    """Chunked gated delta rule forward through ``gdn_chunk_fwd`` of the C ABI.

    q, k [B,T,H,dk] and v [B,T,H,dv] (fp32 or bf16), g, beta [B,T,H] fp32, h0 [N,H,dk,dv] fp32 or None,
    cu_seqlens int32 [N+1] (B == 1) or None.  Returns (o [B,T,H,dv], hT [N,H,dk,dv] fp32); o is in
    ``o_dtype`` (float32, or q's dtype -- the default).  ``workspace`` (uint8 on the device, at least
    :func:`workspace_bytes`) is allocated per call when not given.
    """
    B, T, H, dk, dv, n_seq, o, hT = _prep(q, k, v, h0, cu_seqlens, o, hT, output_final_state, o_dtype)
    _check_dev("g", g, torch.float32)
    _check_dev("beta", beta, torch.float32)
    if g.shape != (B, T, H) or beta.shape != (B, T, H):
        raise ValueError("g and beta must be [B,T,H]")
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    n_seqs = 0 if cu_seqlens is None else n_seq
    ws = _workspace(q, B, T, H, dk, dv, BT, n_seqs, workspace)
    st = load_library().gdn_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(o), _ptr(hT),
        B, T, H, dk, dv, BT, _dtype_code(q), _dtype_code(o), _ptr(cu_seqlens),
        n_seqs, _ptr(ws), 0 if ws is None else ws.numel(), ctypes.c_void_p(stream))
    _raise_on(st)
    return o, hT


def gdn_chunk_fwd_noalloc(q, k, v, g, beta, scale=None, h0=None, output_final_state=True, cu_seqlens=None,
                          BT=64, o=None, hT=None, o_dtype=None):
    """As :func:`gdn_chunk_fwd`, through ``gdn_chunk_fwd_noalloc``, for callers that may not allocate device
    memory (an engine that owns all of it, a host framework's allocator): no workspace is allocated, the
    library's static 256 MiB scratch serves the tensor-core path, sizes that need more are refused, and calls
    must not overlap on the device.  The outputs ``o`` and ``hT`` are still allocated here unless passed in."""
    B, T, H, dk, dv, n_seq, o, hT = _prep(q, k, v, h0, cu_seqlens, o, hT, output_final_state, o_dtype)
    _check_dev("g", g, torch.float32)
    _check_dev("beta", beta, torch.float32)
    if g.shape != (B, T, H) or beta.shape != (B, T, H):
        raise ValueError("g and beta must be [B,T,H]")
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    st = load_library().gdn_chunk_fwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(o), _ptr(hT),
        B, T, H, dk, dv, BT, _dtype_code(q), _dtype_code(o), _ptr(cu_seqlens),
        0 if cu_seqlens is None else n_seq, ctypes.c_void_p(stream))
    _raise_on(st)
    return o, hT


def gdn2_chunk_fwd(q, k, v, g, b, w, scale=None, h0=None, output_final_state=True, cu_seqlens=None, BT=64,
                   o=None, hT=None, o_dtype=None, workspace=None):
    """Gated Delta Rule-2 forward through ``gdn2_chunk_fwd`` of the C ABI.

    g (per-channel log-decay) and b (erase gate) are [B,T,H,dk] fp32, w (write gate) is [B,T,H,dv] fp32.
    ``workspace`` (uint8, at least :func:`gdn2_workspace_bytes`) is allocated per call when not given.
    """
    B, T, H, dk, dv, n_seq, o, hT = _prep(q, k, v, h0, cu_seqlens, o, hT, output_final_state, o_dtype)
    for name, t, shape in (("g", g, (B, T, H, dk)), ("b", b, (B, T, H, dk)), ("w", w, (B, T, H, dv))):
        _check_dev(name, t, torch.float32)
        if t.shape != shape:
            raise ValueError(f"{name} must be {list(shape)}")
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    n_seqs = 0 if cu_seqlens is None else n_seq
    ws = _workspace(q, B, T, H, dk, dv, BT, n_seqs, workspace, gdn2=True)
    st = load_library().gdn2_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), scale, _ptr(h0), _ptr(o), _ptr(hT),
        B, T, H, dk, dv, BT, _dtype_code(q), _dtype_code(o), _ptr(cu_seqlens),
        n_seqs, _ptr(ws), 0 if ws is None else ws.numel(), ctypes.c_void_p(stream))
    _raise_on(st)
    return o, hT


def gdn_kda_chunk_fwd(q, k, v, g, beta, scale=None, h0=None, output_final_state=True, cu_seqlens=None, BT=64,
                      o=None, hT=None, o_dtype=None, workspace=None):
    """KDA forward through ``gdn_kda_chunk_fwd``: per-channel log-decay g [B,T,H,dk] fp32 and one scalar
    beta [B,T,H] fp32 as both the erase and the write gate (GDN-2 with b = w = beta)."""
    B, T, H, dk, dv, n_seq, o, hT = _prep(q, k, v, h0, cu_seqlens, o, hT, output_final_state, o_dtype)
    for name, t, shape in (("g", g, (B, T, H, dk)), ("beta", beta, (B, T, H))):
        _check_dev(name, t, torch.float32)
        if t.shape != shape:
            raise ValueError(f"{name} must be {list(shape)}")
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    n_seqs = 0 if cu_seqlens is None else n_seq
    ws = _workspace(q, B, T, H, dk, dv, BT, n_seqs, workspace, gdn2=True)
    st = load_library().gdn_kda_chunk_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(o), _ptr(hT),
        B, T, H, dk, dv, BT, _dtype_code(q), _dtype_code(o), _ptr(cu_seqlens),
        n_seqs, _ptr(ws), 0 if ws is None else ws.numel(), ctypes.c_void_p(stream))
    _raise_on(st)
    return o, hT


def chunk_gated_delta_rule(q, k, v, g, beta, scale=None, initial_state=None, output_final_state=True,
                           cu_seqlens=None):
    """The token mixer call by the name the pages use; same as :func:`gdn_chunk_fwd`."""
    return gdn_chunk_fwd(q, k, v, g, beta, scale, initial_state, output_final_state, cu_seqlens)


def decode_fwd(q, k, v, g, beta, state, scale=None, o=None, o_dtype=None, b=None, w=None, variant="gdn"):
    """One recurrent decode step (``gdn_decode_fwd`` / ``gdn2_decode_fwd`` / ``gdn_kda_decode_fwd``).

    q, k [N,H,dk] and v [N,H,dv] (fp32 or bf16); ``state`` [N,H,dk,dv] fp32 is updated in place.  GDN: g, beta
    [N,H]; KDA: g [N,H,dk], beta [N,H]; GDN-2: g, b [N,H,dk], w [N,H,dv] (pass beta=None).  Returns o [N,H,dv].
    """
    _check_dev("q", q)
    dt = q.dtype
    o_dtype = dt if o_dtype is None else o_dtype
    _check_dev("k", k, dt)
    _check_dev("v", v, dt)
    _check_dev("state", state, torch.float32)
    N, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:2] != (N, H) or state.shape != (N, H, dk, dv):
        raise ValueError("q, k [N,H,dk], v [N,H,dv] and state [N,H,dk,dv] must agree")
    gate_shapes = {"gdn": {"g": (N, H), "beta": (N, H)}, "kda": {"g": (N, H, dk), "beta": (N, H)},
                   "gdn2": {"g": (N, H, dk), "b": (N, H, dk), "w": (N, H, dv)}}[variant]
    gates = {"g": g, "beta": beta, "b": b, "w": w}
    for name, shape in gate_shapes.items():
        _check_dev(name, gates[name], torch.float32)
        if gates[name] is None or gates[name].shape != shape:
            raise ValueError(f"{name} must be {list(shape)}")
    if o is None:
        o = torch.empty((N, H, dv), dtype=o_dtype, device=q.device)
    _check_dev("o", o, o_dtype)
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    lib = load_library()
    tail = (scale, _ptr(state), _ptr(o), N, H, dk, dv, _dtype_code(q), _dtype_code(o), stream)
    if variant == "gdn2":
        st = lib.gdn2_decode_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), *tail)
    else:
        fn = lib.gdn_decode_fwd if variant == "gdn" else lib.gdn_kda_decode_fwd
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), *tail)
    _raise_on(st)
    return o


def prelude_fwd(xq, xk, xv, wq, wk, wv, a, A_log, dt_bias, b, c=None, conv_state=None, conv_state_out=None,
                cu_seqlens=None, l2_eps=1e-6):
    """The mixer's prelude through ``gdn_prelude_fwd`` (one launch): causal 4-tap conv + SiLU of xq, xk [B,T,H,dk]
    and xv [B,T,H,dv] (taps wq, wk [H*dk, 4], wv [H*dv, 4], fp32), L2 norm of q and k, and the gates
    g = -exp(A_log) softplus(a + dt_bias) (a [B,T,H] or [B,T,H,G]), beta = sigmoid(b), optional w = sigmoid(c).
    ``conv_state`` [N, 2 H dk + H dv, 3] fp32 is the cache before each sequence (None: zeros);
    ``conv_state_out`` (may be ``conv_state`` itself when T == 1) receives the cache after it.
    Returns a dict with q, k, v, g, beta (, w) and conv_state_out."""
    _check_dev("xq", xq)
    dt = xq.dtype
    for name, t in (("xk", xk), ("xv", xv)):
        _check_dev(name, t, dt)
    for name, t in (("wq", wq), ("wk", wk), ("wv", wv), ("a", a), ("A_log", A_log), ("dt_bias", dt_bias), ("b", b),
                    ("c", c), ("conv_state", conv_state), ("conv_state_out", conv_state_out)):
        _check_dev(name, t, torch.float32)
    B, T, H, dk = xq.shape
    dv = xv.shape[-1]
    if cu_seqlens is not None:
        _check_dev("cu_seqlens", cu_seqlens, torch.int32)
    n_seq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    q = torch.empty_like(xq)
    k = torch.empty_like(xk)
    v = torch.empty_like(xv)
    g = torch.empty_like(a)
    beta = torch.empty_like(b)
    w = None if c is None else torch.empty_like(c)
    gw = 1 if a.dim() == 3 else a.shape[-1]
    bw = 1 if b.dim() == 3 else b.shape[-1]
    cw = 0 if c is None else (1 if c.dim() == 3 else c.shape[-1])
    stream = ctypes.c_void_p(torch.cuda.current_stream(xq.device).cuda_stream)
    st = load_library().gdn_prelude_fwd(
        _ptr(xq), _ptr(xk), _ptr(xv), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(conv_state), _ptr(conv_state_out), _ptr(a),
        _ptr(A_log), _ptr(dt_bias), _ptr(g), gw, _ptr(b), _ptr(beta), bw, _ptr(c), _ptr(w), cw, _ptr(q), _ptr(k),
        _ptr(v), B, T, H, dk, dv, _dtype_code(xq), float(l2_eps), _ptr(cu_seqlens),
        0 if cu_seqlens is None else n_seq, stream)
    _raise_on(st)
    out = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "conv_state_out": conv_state_out}
    if w is not None:
        out["w"] = w
    return out


def output_gate_fwd(o, z, weight, eps=1e-5, y=None):
    """The mixer's epilogue through ``gdn_output_gate_fwd``: y = o / sqrt(mean(o^2) + eps) * weight * silu(z) over the
    last axis (dv) of o, z [..., dv] (fp32 or bf16, same dtype); weight [dv] fp32."""
    _check_dev("o", o)
    _check_dev("z", z, o.dtype)
    _check_dev("weight", weight, torch.float32)
    if z.shape != o.shape or weight.shape != (o.shape[-1],):
        raise ValueError("o and z must have one shape and weight [dv]")
    y = torch.empty_like(o) if y is None else y
    _check_dev("y", y, o.dtype)
    dv = o.shape[-1]
    stream = ctypes.c_void_p(torch.cuda.current_stream(o.device).cuda_stream)
    st = load_library().gdn_output_gate_fwd(_ptr(o), _ptr(z), _ptr(weight), _ptr(y), o.numel() // dv, dv,
                                            _dtype_code(o), float(eps), stream)
    _raise_on(st)
    return y


def bwd_workspace_bytes(B, T, H, dk, dv, BT=64, n_seqs=0) -> int:
    """Device workspace (bytes) ``gdn_chunk_bwd`` needs: two fp32 states and the fp32 T and P of every chunk slot
    and head."""
    return int(load_library().gdn_bwd_workspace_bytes(B, T, H, dk, dv, BT, n_seqs))


def gdn_chunk_bwd(q, k, v, g, beta, d_o, scale=None, h0=None, dhT=None, cu_seqlens=None, BT=64, workspace=None,
                  want_dh0=True):
    """Backward pass of :func:`gdn_chunk_fwd` through ``gdn_chunk_bwd``: the gradients of <d_o, o> + <dhT, hT>.

    d_o [B,T,H,dv] in q's dtype; dhT [N,H,dk,dv] fp32 or None.  Returns a dict of fp32 tensors dq, dk, dv, dg,
    dbeta and (when ``want_dh0``) dh0.
    """
    _check_dev("q", q)
    dt = q.dtype
    for name, t in (("k", k), ("v", v), ("d_o", d_o)):
        _check_dev(name, t, dt)
    for name, t in (("g", g), ("beta", beta), ("h0", h0), ("dhT", dhT)):
        _check_dev(name, t, torch.float32)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        _check_dev("cu_seqlens", cu_seqlens, torch.int32)
    n_seq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    n_seqs = 0 if cu_seqlens is None else n_seq
    f32 = dict(dtype=torch.float32, device=q.device)
    out = {"dq": torch.empty((B, T, H, dk), **f32), "dk": torch.empty((B, T, H, dk), **f32),
           "dv": torch.empty((B, T, H, dv), **f32), "dg": torch.empty((B, T, H), **f32),
           "dbeta": torch.empty((B, T, H), **f32),
           "dh0": torch.empty((n_seq, H, dk, dv), **f32) if want_dh0 else None}
    if workspace is None:
        workspace = torch.empty(bwd_workspace_bytes(B, T, H, dk, dv, BT, n_seqs), dtype=torch.uint8, device=q.device)
    _check_dev("workspace", workspace, torch.uint8)
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    st = load_library().gdn_chunk_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), scale, _ptr(h0), _ptr(d_o), _ptr(dhT), _ptr(out["dq"]),
        _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dh0"]), B, T, H, dk, dv,
        BT, _dtype_code(q), _ptr(cu_seqlens), n_seqs, _ptr(workspace), workspace.numel(), stream)
    _raise_on(st)
    return out


def gdn2_bwd_workspace_bytes(B, T, H, dk, dv, BT=64, n_seqs=0) -> int:
    """Device workspace (bytes) ``gdn2_chunk_bwd`` and ``gdn_kda_chunk_bwd`` need: two fp32 states and the fp32
    T and P of every chunk slot and head."""
    return int(load_library().gdn2_bwd_workspace_bytes(B, T, H, dk, dv, BT, n_seqs))


def _bwd2(kda, q, k, v, g, b, w, d_o, scale, h0, dhT, cu_seqlens, BT, workspace, want_dh0):
    _check_dev("q", q)
    dt = q.dtype
    for name, t in (("k", k), ("v", v), ("d_o", d_o)):
        _check_dev(name, t, dt)
    for name, t in (("g", g), ("b" if not kda else "beta", b), ("w", w), ("h0", h0), ("dhT", dhT)):
        _check_dev(name, t, torch.float32)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        _check_dev("cu_seqlens", cu_seqlens, torch.int32)
    n_seq = B if cu_seqlens is None else cu_seqlens.numel() - 1
    n_seqs = 0 if cu_seqlens is None else n_seq
    f32 = dict(dtype=torch.float32, device=q.device)
    out = {"dq": torch.empty((B, T, H, dk), **f32), "dk": torch.empty((B, T, H, dk), **f32),
           "dv": torch.empty((B, T, H, dv), **f32), "dg": torch.empty((B, T, H, dk), **f32)}
    if kda:
        out["dbeta"] = torch.empty((B, T, H), **f32)
    else:
        out["db"] = torch.empty((B, T, H, dk), **f32)
        out["dw"] = torch.empty((B, T, H, dv), **f32)
    out["dh0"] = torch.empty((n_seq, H, dk, dv), **f32) if want_dh0 else None
    if workspace is None:
        workspace = torch.empty(gdn2_bwd_workspace_bytes(B, T, H, dk, dv, BT, n_seqs), dtype=torch.uint8,
                                device=q.device)
    _check_dev("workspace", workspace, torch.uint8)
    scale = dk ** -0.5 if scale is None else float(scale)
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    lib = load_library()
    tail = (B, T, H, dk, dv, BT, _dtype_code(q), _ptr(cu_seqlens), n_seqs, _ptr(workspace), workspace.numel(), stream)
    if kda:
        st = lib.gdn_kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), scale, _ptr(h0), _ptr(d_o), _ptr(dhT),
                                   _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                   _ptr(out["dbeta"]), _ptr(out["dh0"]), *tail)
    else:
        st = lib.gdn2_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), scale, _ptr(h0), _ptr(d_o),
                                _ptr(dhT), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
                                _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dh0"]), *tail)
    _raise_on(st)
    return out


def gdn2_chunk_bwd(q, k, v, g, b, w, d_o, scale=None, h0=None, dhT=None, cu_seqlens=None, BT=64, workspace=None,
                   want_dh0=True):
    """Backward pass of :func:`gdn2_chunk_fwd` through ``gdn2_chunk_bwd``: the gradients of <d_o, o> + <dhT, hT>.

    g, b [B,T,H,dk] and w [B,T,H,dv] fp32; d_o in q's dtype.  Returns fp32 dq, dk, dv, dg, db, dw and dh0.
    """
    return _bwd2(False, q, k, v, g, b, w, d_o, scale, h0, dhT, cu_seqlens, BT, workspace, want_dh0)


def gdn_kda_chunk_bwd(q, k, v, g, beta, d_o, scale=None, h0=None, dhT=None, cu_seqlens=None, BT=64, workspace=None,
                      want_dh0=True):
    """Backward pass of :func:`gdn_kda_chunk_fwd` through ``gdn_kda_chunk_bwd``.  g [B,T,H,dk] and beta [B,T,H]
    fp32.  Returns fp32 dq, dk, dv, dg [B,T,H,dk], dbeta [B,T,H] and dh0."""
    return _bwd2(True, q, k, v, g, beta, None, d_o, scale, h0, dhT, cu_seqlens, BT, workspace, want_dh0)
