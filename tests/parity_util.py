"""Helpers shared by the parity tests: run the CUDA path and the fp64 oracle on the same inputs.

Tolerance (stated for this method): max |x - x_ref| / rms(x_ref), separately for o and hT, at most
1e-4 for fp32 inputs and 2e-2 for bf16 inputs with fp32 gates and state.  That bound applies as stated
to hT (always fp32) and to an fp32 o.  A bf16 o cannot meet it as stated: rounding the exact output to
bf16 alone moves an element by up to 2^-9 of its own size, and the outputs' largest elements are ~10-12
times their RMS, so the exactly rounded oracle output itself is ~2e-2 away.  For a bf16 o the allowance
per element is therefore the stated bound plus one bf16 ulp (2^-8) of |o_ref|.
"""
import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}
BF16_ULP = 2.0 ** -8


def o_excess(o, ref, in_dtype, o_dtype):
    """max_i |o_i - ref_i| / allowance_i  (<= 1 passes); allowance described in the module docstring."""
    o = np.asarray(o, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    allow = TOL[in_dtype] * max(np.sqrt(np.mean(ref ** 2)), 1e-30)
    if o_dtype == "bf16":
        allow = allow + BF16_ULP * np.abs(ref)
    return float(np.max(np.abs(o - ref) / allow))


def relerr(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(x - ref)) / max(rms, 1e-30)) if ref.size else 0.0


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def to_dev(inp, device="cuda"):
    out = {}
    for key, val in inp.items():
        out[key] = val.to(device) if isinstance(val, torch.Tensor) else val
    return out


def run_cuda(inp, variant, output_final_state=True, o_dtype="f32"):
    """Run the C ABI through the binding on device copies of ``inp``; returns (o, hT) on the device."""
    from gated_delta_rule_105_b200 import gdn2_chunk_fwd, gdn_chunk_fwd, gdn_kda_chunk_fwd
    d = to_dev(inp)
    odt = {"f32": torch.float32, "bf16": torch.bfloat16}[o_dtype]
    if variant == "gdn":
        return gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                             output_final_state, d["cu_seqlens"], o_dtype=odt)
    if variant == "kda":
        return gdn_kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["scale"], d["h0"],
                                 output_final_state, d["cu_seqlens"], o_dtype=odt)
    return gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d["scale"], d["h0"],
                          output_final_state, d["cu_seqlens"], o_dtype=odt)


def seq_spans(inp):
    B, T = inp["q"].shape[:2]
    cu = inp["cu_seqlens"]
    if cu is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in cu]
    return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def kda_gates(inp):
    """KDA as GDN-2: the scalar beta broadcast to the erase gate b [..,dk] and the write gate w [..,dv]."""
    beta = f64(inp["beta"])[..., None]
    dk, dv = inp["q"].shape[-1], inp["v"].shape[-1]
    return np.repeat(beta, dk, axis=-1), np.repeat(beta, dv, axis=-1)


def run_oracle(inp, variant, threads=8):
    """Whole-input fp64 oracle run (small inputs)."""
    import oracle
    cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy()
    if variant == "kda":
        b, w = kda_gates(inp)
        return oracle.gdn2_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), b, w, inp["scale"],
                               f64(inp["h0"]), cu_seqlens=cu, threads=threads)
    if variant == "gdn":
        return oracle.gdn_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["beta"]),
                              inp["scale"], f64(inp["h0"]), cu_seqlens=cu, threads=threads)
    return oracle.gdn2_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]), f64(inp["b"]),
                           f64(inp["w"]), inp["scale"], f64(inp["h0"]), cu_seqlens=cu, threads=threads)


def oracle_units(inp, variant, units, threads=8):
    """fp64 oracle on a few (sequence n, head h) units of a large input, each sliced out on its own.

    Returns {(n, h): (o [L, dv], hT [dk, dv])}.
    """
    import oracle
    spans = seq_spans(inp)
    results = {}

    def one(unit):
        n, h = unit
        row, t0, t1 = spans[n]

        def sl(t):
            return None if t is None else f64(t[row:row + 1, t0:t1, h:h + 1])

        h0 = None if inp["h0"] is None else f64(inp["h0"][n:n + 1, h:h + 1])
        if variant == "gdn":
            o, hT = oracle.gdn_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]),
                                   inp["scale"], h0)
        elif variant == "kda":
            bt = sl(inp["beta"])[..., None]
            dk, dv = inp["q"].shape[-1], inp["v"].shape[-1]
            o, hT = oracle.gdn2_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]),
                                    np.repeat(bt, dk, axis=-1), np.repeat(bt, dv, axis=-1), inp["scale"], h0)
        else:
            o, hT = oracle.gdn2_fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["b"]),
                                    sl(inp["w"]), inp["scale"], h0)
        results[unit] = (o[0, :, 0], hT[0, 0])

    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=max(1, min(threads, len(units)))) as ex:
        list(ex.map(one, units))
    return results


def unit_slices(inp, o, hT, unit):
    """The CUDA outputs of one (n, h) unit as fp64 numpy: (o [L, dv], hT [dk, dv])."""
    n, h = unit
    row, t0, t1 = seq_spans(inp)[n]
    return f64(o[row, t0:t1, h]), f64(hT[n, h])


def cotangents(inp, seed):
    """Seeded output and final-state cotangents of a backward test: d_o in q's dtype, dhT fp32."""
    rng = np.random.default_rng(seed)
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    n = B if inp["cu_seqlens"] is None else inp["cu_seqlens"].numel() - 1
    d_o = torch.from_numpy(rng.standard_normal((B, T, H, dv)).astype(np.float32)).to(inp["q"].dtype)
    dhT = torch.from_numpy((rng.standard_normal((n, H, dk, dv)) * 0.5).astype(np.float32))
    return d_o, dhT
