"""gdn_chunk_fwd_noalloc: the forward pass for callers that cannot allocate device memory.

Some callers of this library may not call cudaMalloc: serving engines that give all free device memory to their
own pool at start-up, plug-ins inside a host framework that owns the allocator, and latency-critical loops where
an allocation may synchronise the device.  ``gdn_chunk_fwd_noalloc`` serves them: it takes no workspace and keeps
the tensor-core path's per-chunk WY factors in a scratch array compiled into the library (256 MiB per device).
These tests call it through the C ABI (ctypes, no binding helper) and compare it with ``gdn_chunk_fwd`` given its
own workspace, on two calls in a row, so the second call runs on whatever the first left in the shared array.

This file is collected last on purpose: it runs alone in a fresh process as well as after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_util import TOL, f64, relerr

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 256 * 1024 * 1024  # GDN_STATIC_WS_BYTES in include/gdn.h
GDN_OK, GDN_ERR_UNSUPPORTED, GDN_F32, GDN_BF16 = 0, 2, 0, 1


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_105_b200 import build
    build.build()
    from gated_delta_rule_105_b200.binding import load_library
    return load_library()


def _p(t):
    return ctypes.c_void_p(None if t is None else t.data_ptr())


def _outputs(d, n_seq):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    o = torch.full((B, T, H, dv), float("nan"), dtype=torch.float32, device="cuda")
    hT = torch.full((n_seq, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
    return o, hT


def _args(d, o, hT, n_seqs):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    return [_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["g"]), _p(d["beta"]), ctypes.c_float(d["scale"]), _p(d["h0"]),
            _p(o), _p(hT), B, T, H, dk, dv, 64, GDN_BF16, GDN_F32, _p(d["cu_seqlens"]), n_seqs]


def call_noalloc(lib, d, n_seq, n_seqs):
    o, hT = _outputs(d, n_seq)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.gdn_chunk_fwd_noalloc(*_args(d, o, hT, n_seqs), stream)
    assert st == GDN_OK, lib.gdn_last_error().decode()
    assert lib.gdn_check_error(stream) == GDN_OK, lib.gdn_last_error().decode()
    return o, hT


def call_with_workspace(lib, d, n_seq, n_seqs):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    nbytes = lib.gdn_workspace_bytes(B, T, H, dk, dv, 64, n_seqs)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o, hT = _outputs(d, n_seq)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.gdn_chunk_fwd(*_args(d, o, hT, n_seqs), _p(ws), ctypes.c_size_t(nbytes), stream)
    assert st == GDN_OK, lib.gdn_last_error().decode()
    assert lib.gdn_check_error(stream) == GDN_OK, lib.gdn_last_error().decode()
    return o, hT


def _dev(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def _same_within_tolerance(got, ref, what):
    for x, r, name in ((got[0], ref[0], "o"), (got[1], ref[1], "hT")):
        assert torch.isfinite(x).all(), f"{what}: {name} not finite"
        e = relerr(f64(x), f64(r))
        assert e <= TOL["bf16"], f"{what}: {name} differs from gdn_chunk_fwd by {e:.3g} of its RMS"


def test_noalloc_matches_the_workspace_call_twice_in_a_row(lib):
    """The bench workload (bf16, B4 H16 T4096, dk 128, dv 256, h0 given): 170 MB of WY factors and P, which fit."""
    from gated_delta_rule_105_b200.inputs import WORKLOADS, generate_workload
    w = WORKLOADS["gdn_bf16_b4h16t4096_dk128_dv256_h0"]
    assert lib.gdn_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, 64, 0) <= STATIC_WS_BYTES
    d = _dev(generate_workload(w))
    ref = call_with_workspace(lib, d, w.B, 0)
    for call in range(2):
        got = call_noalloc(lib, d, w.B, 0)
        assert lib.gdn_last_kernel() == 2  # the tensor-core path, on the static scratch
        _same_within_tolerance(got, ref, f"call {call + 1}")


def test_noalloc_packed_sequences_with_empty_and_ragged_ones(lib):
    """Packed variable-length input numbers its scratch slots per sequence start; two calls in a row."""
    from gated_delta_rule_105_b200.inputs import generate
    cu = np.array([0, 1, 1, 64, 129, 200, 330, 330, 777], dtype=np.int32)
    inp = generate(1, int(cu[-1]), 3, 128, 128, "bf16", seed=31, h0_std=0.1, cu_seqlens=cu)
    d = _dev(inp)
    n = len(cu) - 1
    ref = call_with_workspace(lib, d, n, n)
    for call in range(2):
        got = call_noalloc(lib, d, n, n)
        assert lib.gdn_last_kernel() == 2
        _same_within_tolerance(got, ref, f"packed call {call + 1}")
        assert torch.equal(got[1][1].cpu(), inp["h0"][1])  # zero-length sequence: hT = h0


def test_noalloc_refuses_sizes_beyond_the_static_scratch(lib):
    """1025 chunk slots x 8 heads x 40 KB > 256 MiB: refused on the host with a message, nothing enqueued."""
    from gated_delta_rule_105_b200.inputs import generate
    assert lib.gdn_workspace_bytes(1, 65536, 8, 128, 128, 64, 0) > STATIC_WS_BYTES
    d = _dev(generate(1, 65536, 8, 128, 128, "bf16", 777, "gdn", 0.0, 0))
    o, hT = _outputs(d, 1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.gdn_chunk_fwd_noalloc(*_args(d, o, hT, 0), stream)
    assert st == GDN_ERR_UNSUPPORTED
    assert b"static scratch" in lib.gdn_last_error()
    torch.cuda.synchronize()
    assert torch.isnan(o).all()  # nothing ran
