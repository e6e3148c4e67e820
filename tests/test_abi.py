"""CPU tests of the C ABI: the library loads, exports what include/gdn.h declares, and rejects bad
arguments on the host before touching a device (no compute call runs here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_105_b200 import build
    build.build()
    from gated_delta_rule_105_b200.binding import load_library
    return load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn\w*)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["gdn_chunk_fwd", "gdn2_chunk_fwd", "gdn_workspace_bytes", "gdn_check_error", "gdn_status_string",
              "gdn_last_error", "gdn_set_kernel", "gdn_last_kernel", "gdn_debug_umma_selftest",
              "gdn_chunk_fwd_noalloc", "gdn_profile_enable", "gdn_profile_take", "gdn2_workspace_bytes",
              "gdn_kda_chunk_fwd", "gdn_debug_stall", "gdn_decode_fwd", "gdn2_decode_fwd",
              "gdn_kda_decode_fwd", "gdn_prelude_fwd", "gdn_output_gate_fwd", "gdn_bwd_workspace_bytes",
              "gdn_chunk_bwd", "gdn2_bwd_workspace_bytes", "gdn2_chunk_bwd", "gdn_kda_chunk_bwd"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libgdn.so does not export {name}"


def test_exported_symbols_are_unmangled_c():
    out = os.popen(f"nm -D --defined-only {os.path.join(ROOT, 'gated_delta_rule_105_b200', 'libgdn.so')}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


A = 0x10000  # a 16-byte aligned fake device address; never dereferenced by the host checks


def call(lib, **kw):
    args = dict(q=A, k=A, v=A, g=A, beta=A, scale=0.125, h0=None, o=A, hT=None, B=1, T=64, H=1, dk=64, dv=64,
                BT=64, dt=1, odt=0, cu=None, n_seqs=0, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    vp = ctypes.c_void_p
    return lib.gdn_chunk_fwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["beta"]),
                             args["scale"], vp(args["h0"]), vp(args["o"]), vp(args["hT"]), args["B"], args["T"],
                             args["H"], args["dk"], args["dv"], args["BT"], args["dt"], args["odt"], vp(args["cu"]),
                             args["n_seqs"], vp(args["ws"]), args["ws_bytes"], vp(args["stream"]))


def call2(lib, **kw):
    args = dict(q=A, k=A, v=A, g=A, b=A, w=A, B=1, T=64, H=1, dk=64, dv=64, BT=64, dt=1)
    args.update(kw)
    vp = ctypes.c_void_p
    return lib.gdn2_chunk_fwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["b"]),
                              vp(args["w"]), 0.125, None, vp(A), None, args["B"], args["T"], args["H"], args["dk"],
                              args["dv"], args["BT"], args["dt"], 0, None, 0, None, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(beta=None), 1),
    (dict(q=A + 8), 1), (dict(hT=A + 4), 1), (dict(h0=A + 2), 1),
    (dict(B=0), 1), (dict(H=0), 1), (dict(T=-1), 1),
    (dict(BT=32), 2), (dict(dk=96), 2), (dict(dk=256), 2), (dict(dv=32), 2), (dict(dv=320), 2), (dict(dv=96), 2),
    (dict(dt=7), 2), (dict(dt=0, odt=1), 2), (dict(odt=5), 2), (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1),
    (dict(cu=A, B=2, n_seqs=2), 1), (dict(cu=A, n_seqs=0), 1), (dict(n_seqs=3), 1),
    (dict(ws=None, ws_bytes=64), 1),
])
def test_host_checks_reject_bad_arguments(lib, kw, status):
    assert call(lib, **kw) == status
    assert lib.gdn_last_error().decode() != ""


@pytest.mark.parametrize("kw,status", [(dict(w=None), 1), (dict(b=None), 1), (dict(w=A + 8), 1), (dict(dk=32), 2)])
def test_host_checks_gdn2(lib, kw, status):
    assert call2(lib, **kw) == status


def call_kda(lib, **kw):
    args = dict(q=A, k=A, v=A, g=A, beta=A, B=1, T=64, H=1, dk=128, dv=128, BT=64, dt=1)
    args.update(kw)
    vp = ctypes.c_void_p
    return lib.gdn_kda_chunk_fwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["beta"]),
                                 0.125, None, vp(A), None, args["B"], args["T"], args["H"], args["dk"], args["dv"],
                                 args["BT"], args["dt"], 0, None, 0, None, 0, None)


@pytest.mark.parametrize("kw,status", [(dict(beta=None), 1), (dict(g=None), 1), (dict(beta=A + 4), 1),
                                       (dict(dk=32), 2), (dict(BT=16), 2)])
def test_host_checks_kda(lib, kw, status):
    assert call_kda(lib, **kw) == status
    assert lib.gdn_last_error().decode() != ""


def call_decode(lib, name="gdn_decode_fwd", **kw):
    args = dict(q=A, k=A, v=A, g=A, beta=A, state=A, o=A, N=2, H=1, dk=128, dv=128, dt=1, odt=0)
    args.update(kw)
    vp = ctypes.c_void_p
    head = [vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["beta"])]
    if name == "gdn2_decode_fwd":
        head.append(vp(A))
    return getattr(lib, name)(*head, ctypes.c_float(0.125), vp(args["state"]), vp(args["o"]), args["N"], args["H"],
                              args["dk"], args["dv"], args["dt"], args["odt"], None)


@pytest.mark.parametrize("name", ["gdn_decode_fwd", "gdn2_decode_fwd", "gdn_kda_decode_fwd"])
@pytest.mark.parametrize("kw,status", [(dict(state=None), 1), (dict(state=A + 4), 1), (dict(q=None), 1),
                                       (dict(N=0), 1), (dict(dk=96), 2), (dict(dv=320), 2), (dict(dv=96), 2),
                                       (dict(dt=0, odt=1), 2)])
def test_host_checks_decode(lib, name, kw, status):
    assert call_decode(lib, name, **kw) == status
    assert lib.gdn_last_error().decode() != ""


def test_status_strings_and_kernel_choice(lib):
    for s in range(6):
        assert lib.gdn_status_string(s).decode() not in ("", "unknown status")
    assert lib.gdn_set_kernel(9) == 1
    assert lib.gdn_set_kernel(0) == 0
    # the tensor-core path keeps 40 KB of WY factors and P per (chunk slot, head); slots = ceil(B T / 64) + sequences
    assert lib.gdn_workspace_bytes(4, 4096, 16, 128, 256, 64, 0) == (256 + 4) * 16 * 40960
    assert lib.gdn_workspace_bytes(1, 65536, 16, 128, 256, 64, 16) == (1024 + 16) * 16 * 40960
    assert lib.gdn_workspace_bytes(1, 100, 2, 128, 128, 64, 0) == (2 + 1) * 2 * 40960
    assert lib.gdn_workspace_bytes(4, 4096, 16, 64, 64, 64, 0) == 0  # shapes only the SIMT kernel takes
    assert lib.gdn_workspace_bytes(4, 0, 16, 128, 256, 64, 0) == 0
    # GDN-2 / KDA: one 82432-byte unit (T hi/lo, -W^T, P, Q', K~, Lambda) per chunk slot and head
    assert lib.gdn2_workspace_bytes(4, 4096, 16, 128, 128, 64, 0) == (256 + 4) * 16 * 82432
    assert lib.gdn2_workspace_bytes(1, 100, 2, 128, 256, 64, 0) == (2 + 1) * 2 * 82432
    assert lib.gdn2_workspace_bytes(4, 4096, 16, 64, 64, 64, 0) == 0


def test_binding_refuses_cpu_tensors(lib):
    import torch
    from gated_delta_rule_105_b200 import gdn_chunk_fwd
    q = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gdn_chunk_fwd(q, q, q, torch.zeros(1, 4, 1), torch.zeros(1, 4, 1))


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(q=A + 8), 1), (dict(B=0), 1), (dict(BT=32), 2), (dict(dk=96), 2), (dict(dv=320), 2),
    (dict(dt=7), 2), (dict(scale=float("nan")), 1), (dict(cu=A, B=2, n_seqs=2), 1), (dict(n_seqs=3), 1),
])
def test_noalloc_entry_checks_arguments_before_touching_the_device(lib, kw, status):
    args = dict(q=A, k=A, v=A, g=A, beta=A, scale=0.125, h0=None, o=A, hT=None, B=1, T=64, H=1, dk=64, dv=64,
                BT=64, dt=1, odt=0, cu=None, n_seqs=0)
    args.update(kw)
    vp = ctypes.c_void_p
    st = lib.gdn_chunk_fwd_noalloc(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["beta"]),
                                   args["scale"], vp(args["h0"]), vp(args["o"]), vp(args["hT"]), args["B"], args["T"],
                                   args["H"], args["dk"], args["dv"], args["BT"], args["dt"], args["odt"],
                                   vp(args["cu"]), args["n_seqs"], None)
    assert st == status
    assert lib.gdn_last_error().decode() != ""


def test_bwd_workspace_holds_two_states_and_t_and_p_of_every_chunk(lib):
    lib.gdn_bwd_workspace_bytes.restype = lib.gdn2_bwd_workspace_bytes.restype = ctypes.c_size_t
    B, T, H, dk, dv = 2, 130, 3, 128, 64
    slots = -(-B * T // 64) + B
    need = 2 * slots * H * dk * dv * 4 + slots * H * 2 * 64 * 64 * 4
    assert lib.gdn_bwd_workspace_bytes(B, T, H, dk, dv, 64, 0) == need
    assert lib.gdn2_bwd_workspace_bytes(B, T, H, dk, dv, 64, 0) == need
    assert lib.gdn2_bwd_workspace_bytes(B, T, H, 96, dv, 64, 0) == 0  # unsupported dk


def call_bwd2(lib, kda=False, **kw):
    args = dict(q=A, k=A, v=A, g=A, b=A, w=A, d_o=A, dq=A, dk=A, dv=A, dg=A, db=A, dw=A, B=1, T=64, H=1, dk_=64,
                dv_=64, dt=1, ws=A, ws_bytes=1 << 30)
    args.update(kw)
    vp = ctypes.c_void_p
    tail = (args["B"], args["T"], args["H"], args["dk_"], args["dv_"], 64, args["dt"], None, 0, vp(args["ws"]),
            ctypes.c_size_t(args["ws_bytes"]), None)
    if kda:
        return lib.gdn_kda_chunk_bwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["b"]),
                                     ctypes.c_float(0.125), None, vp(args["d_o"]), None, vp(args["dq"]),
                                     vp(args["dk"]), vp(args["dv"]), vp(args["dg"]), vp(args["db"]), None, *tail)
    return lib.gdn2_chunk_bwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]), vp(args["b"]),
                              vp(args["w"]), ctypes.c_float(0.125), None, vp(args["d_o"]), None, vp(args["dq"]),
                              vp(args["dk"]), vp(args["dv"]), vp(args["dg"]), vp(args["db"]), vp(args["dw"]), None,
                              *tail)


@pytest.mark.parametrize("kda", [False, True])
@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(d_o=None), 1), (dict(g=None), 1), (dict(b=None), 1), (dict(dq=None), 1),
    (dict(db=None), 1), (dict(dg=A + 4), 1), (dict(ws_bytes=1024), 1), (dict(ws=None, ws_bytes=0), 1),
    (dict(dk_=96), 2), (dict(dv_=320), 2), (dict(dt=5), 2),
])
def test_gdn2_bwd_host_checks(lib, kda, kw, status):
    lib.gdn2_chunk_bwd.restype = lib.gdn_kda_chunk_bwd.restype = ctypes.c_int
    assert call_bwd2(lib, kda, **kw) == status
    assert lib.gdn_last_error().decode() != ""


def test_gdn2_bwd_needs_the_write_gate_and_its_gradient(lib):
    lib.gdn2_chunk_bwd.restype = ctypes.c_int
    assert call_bwd2(lib, w=None) == 1
    assert call_bwd2(lib, dw=None) == 1
