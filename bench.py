#!/usr/bin/env python
"""Throughput of the chunked gated delta rule forward pass on B200 (tokens/s, TFLOP/s, roofline fraction).

One step is one ``gdn_chunk_fwd`` (or ``gdn2_chunk_fwd``) call over the whole batch of the workload:
every step of the path (gate cumsum, intra-chunk WY solve, chunk-to-chunk state pass, output, final
state) runs inside it.  Inputs are seeded synthetic tensors (``gated_delta_rule_105_b200.inputs``)
resident in HBM before timing; per-step traffic is larger than the 126 MB L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--kernel auto|simt|tc]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample (rank 0 only)

For N > 1 (torchrun, one rank per GPU) every rank runs its own batch of the workload (the (sequence,
head) units are independent, so there is no data-path collective); time is the max over ranks and
``value`` counts the tokens of all ranks ("weak" scaling).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule fwd tokens/s and TFLOP/s, % of B200 roofline (1 GPU)"
DEFAULT_WORKLOAD = "gdn_bf16_b4h16t4096_dk128_dv256_h0"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
C = 64  # tokens per chunk


# ------------------------------------------------------------------------------------------ work model
def n_sequences(w, inp=None):
    if w.n_seqs:
        return w.n_seqs
    return w.B


def algorithmic(w):
    """Algorithmic FLOPs and HBM bytes of one launch over the whole workload.

    Per head-token: F = 2 (3 C dk + 2 C dv + 3 dk dv) + C^2/3 (chunk products counted dense, the
    64x64 triangular solve as C^2/3); bytes = s (2 dk + dv) read + s dv written (s = the input element
    size: o is counted in q's dtype, as the operation defines it) + gates (GDN: g, beta fp32 = 8 B;
    GDN-2: g, b, w fp32 = 4 (2 dk + dv) B); plus one fp32 state per (sequence, head) written, and read
    when h0 is given.
    """
    s = 2 if w.dtype == "bf16" else 4
    dk, dv = w.dk, w.dv
    head_tokens = w.B * w.T * w.H
    f_ht = 2 * (3 * C * dk + 2 * C * dv + 3 * dk * dv) + C * C / 3
    gate = 8 if w.variant == "gdn" else 4 * (2 * dk + dv)
    b_ht = s * (2 * dk + dv) + s * dv + gate
    state = n_sequences(w) * w.H * dk * dv * 4
    n_states = 2 if w.h0_std > 0 else 1
    return f_ht * head_tokens, b_ht * head_tokens + n_states * state


def output_overhead_bytes(w, o_dtype):
    """Bytes written beyond the algorithmic count when o is wider than q's dtype (an fp32 o for bf16 inputs)."""
    s = 2 if w.dtype == "bf16" else 4
    s_o = 2 if o_dtype == "bf16" else 4
    return max(0, s_o - s) * w.B * w.T * w.H * w.dv


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Source files each timed kernel family is compiled from (its own header and what that header includes);
# a recorded DRAM traffic figure stays valid while these are unchanged.
KERNEL_SOURCES = {
    "gdn_tc_wy_kernel+gdn_tc_fwd_kernel": ["gdn_common.cuh", "gdn_sm100.cuh", "gdn_tc.cuh"],
    "gdn2_tc_prep_kernel+gdn2_tc_fwd_kernel": ["gdn_common.cuh", "gdn_sm100.cuh", "gdn_tc.cuh", "gdn2_tc.cuh"],
    "gdn_simt_fwd_kernel": ["gdn_common.cuh", "gdn_simt.cuh"],
}


def kernel_source_hash(kernel=None):
    """sha256[:16] over the named kernel's source files (every file under csrc/ for an unknown kernel)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_105_b200", "csrc")
    for f in KERNEL_SOURCES.get(kernel) or sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash(kernel)
    for line in open(path):
        parts = dict(p.split("=", 1) for p in line.split() if "=" in p)
        if parts.get("kernel") == kernel and parts.get("workload") == workload and parts.get("sources") == src:
            return float(parts["bytes_per_launch"])
    return None


# ------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index, period_s=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML (CPU machine): clocks are reported as unavailable
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------------ distributed
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, ws: int, ms_per_step_max: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch; time is the slowest rank's."""
    return ws * tokens_per_rank / (ms_per_step_max * 1e-3)


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------------------------ oracle (CPU)
def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def seq_spans(inp):
    B, T = inp["q"].shape[:2]
    if inp["cu_seqlens"] is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in inp["cu_seqlens"]]
    return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]


def oracle_sample_run(inp, w, units, threads):
    """Run the fp64 oracle on ``units`` (sequence, head) pairs of ``inp``; returns head-tokens done."""
    import numpy as np
    import torch
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    spans = seq_spans(inp)

    def f64(t):
        return None if t is None else np.ascontiguousarray(t.to(torch.float64).numpy())

    def one(unit):
        n, h = unit
        row, t0, t1 = spans[n]
        sl = {k: f64(inp[k][row:row + 1, t0:t1, h:h + 1]) for k in ("q", "k", "v", "g", "beta", "b", "w")
              if inp.get(k) is not None}
        h0 = None if inp["h0"] is None else f64(inp["h0"][n:n + 1, h:h + 1])
        if w.variant == "gdn":
            oracle.gdn_fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], inp["scale"], h0)
        else:
            oracle.gdn2_fwd(sl["q"], sl["k"], sl["v"], sl["g"], sl["b"], sl["w"], inp["scale"], h0)
        return t1 - t0

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        return sum(ex.map(one, units))


def all_units(inp, w):
    return [(n, h) for n in range(len(seq_spans(inp))) for h in range(w.H)]


def cpu_baseline(inp, w, budget_s=15.0):
    """Times the oracle on a bounded sample of the workload: whole (sequence, head) units, one per core."""
    from oracle import build as obuild
    obuild.build()
    cores = cpu_cores()
    units = all_units(inp, w)
    t0 = time.perf_counter()
    done1 = oracle_sample_run(inp, w, units[:1], 1)
    t_unit = time.perf_counter() - t0
    n = max(1, min(len(units), int(budget_s / max(t_unit, 1e-3) * cores)))
    n = max(min(n, len(units)), 1)
    sample = units[1:1 + n] if len(units) > n else units[:n]
    threads = min(cores, len(sample))
    t0 = time.perf_counter()
    done = oracle_sample_run(inp, w, sample, threads)
    dt = time.perf_counter() - t0
    return {"value": done / w.H / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(sample)} of {len(units)} (sequence, head) units at full length "
                      f"({done} head-tokens), fp64 C recurrence, {threads} threads; tokens/s = head-tokens/s / H",
            "seconds": round(dt, 3),
            "single_thread": {"value": done1 / w.H / t_unit, "unit": "tokens/s", "cores": 1,
                              "sample": f"1 (sequence, head) unit at full length ({done1} head-tokens), 1 thread",
                              "seconds": round(t_unit, 3)}}


# ------------------------------------------------------------------------------------------ arms
def run_reference(args, w):
    rank, _, ws = dist_env()
    if rank != 0:
        return 0
    from gated_delta_rule_105_b200.inputs import generate_workload
    from oracle import build as obuild
    obuild.build()
    inp = generate_workload(w)
    units = all_units(inp, w)
    cores = cpu_cores()
    t0 = time.perf_counter()
    oracle_sample_run(inp, w, units[:1], 1)
    t_unit = time.perf_counter() - t0
    per_step = max(1, min(len(units), int(args.ref_budget / (args.steps + args.warmup) / t_unit * cores)))
    threads = min(cores, per_step)
    step_units = [units[(i * per_step + j) % len(units)] for i in range(args.steps + args.warmup)
                  for j in range(per_step)]
    for i in range(args.warmup):
        oracle_sample_run(inp, w, step_units[i * per_step:(i + 1) * per_step], threads)
    done = 0
    t0 = time.perf_counter()
    for i in range(args.warmup, args.warmup + args.steps):
        done += oracle_sample_run(inp, w, step_units[i * per_step:(i + 1) * per_step], threads)
    dt = time.perf_counter() - t0
    value = done / w.H / dt
    sample = (f"each step {per_step} of {len(units)} (sequence, head) units at full length, fp64 C recurrence, "
              f"{threads} threads; tokens/s = head-tokens/s / H")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv, "BT": C},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    import torch
    rank, local_rank, ws = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    from gated_delta_rule_105_b200 import (gdn2_chunk_fwd, gdn2_workspace_bytes, gdn_chunk_fwd, last_kernel,
                                           set_kernel, check_error,
                                           profile_enable, profile_take, workspace_bytes)
    from gated_delta_rule_105_b200.inputs import generate
    set_kernel(args.kernel)
    o_dtype = "f32" if w.dtype == "f32" else args.o_dtype
    o_torch = torch.float32 if o_dtype == "f32" else torch.bfloat16

    # each rank draws its own batch (seed offset by rank): independent units, weak scaling
    inp = generate(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.seed + 7919 * rank, w.variant, w.h0_std, w.n_seqs,
                   w.len_range)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    n_seq = w.B if d["cu_seqlens"] is None else d["cu_seqlens"].numel() - 1
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=o_torch, device=dev)
    hT = torch.empty((n_seq, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)

    # the tensor-core path's scratch (WY factors of every chunk), allocated once like a caller would
    n_ws = (workspace_bytes if w.variant == "gdn" else gdn2_workspace_bytes)(
        w.B, w.T, w.H, w.dk, w.dv, C, 0 if d["cu_seqlens"] is None else n_seq)
    wsp = torch.empty(n_ws, dtype=torch.uint8, device=dev) if (n_ws and w.dtype == "bf16") else None

    if w.variant == "gdn":
        def step(dd, oo, hh):
            return gdn_chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], dd["scale"], dd["h0"], True,
                                 dd["cu_seqlens"], o=oo, hT=hh, o_dtype=o_torch, workspace=wsp)
    else:
        def step(dd, oo, hh):
            return gdn2_chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["b"], dd["w"], dd["scale"], dd["h0"],
                                  True, dd["cu_seqlens"], o=oo, hT=hh, o_dtype=o_torch, workspace=wsp)

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step(d, o, hT)
    check_error(stream)
    kernel = last_kernel()

    # ---- per-kernel durations: a short pass with the library's own event pair around each of its kernel
    # launches (same stream); these events serialise the launches, so the timed region below runs without
    n_prof = max(3, min(args.steps, 20))
    torch.cuda.synchronize(dev)
    profile_take()
    profile_enable(True)
    for _ in range(n_prof):
        step(d, o, hT)
    torch.cuda.synchronize(dev)
    profile_enable(False)
    per_kernel = profile_take()
    kernels_per_step = max(1, round(sum(n for n, _ in per_kernel.values()) / n_prof))
    kernel_ms = {name: round(max_over_ranks(ms / n, ws), 5) for name, (n, ms) in per_kernel.items()}

    # ---- device-resident timing: one event pair per step on the launching stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local_rank)
    launches = 0
    with sampler:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step(d, o, hT)
            launches += kernels_per_step
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(ws)
    check_error(stream)
    elapsed_ms = t_start.elapsed_time(t_end)
    per_launch = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    elapsed_ms = max_over_ranks(elapsed_ms, ws)
    launch_ms = max_over_ranks(statistics.mean(per_launch), ws)

    # ---- end to end through the public API: pinned host inputs -> device -> call -> host outputs
    in_keys = [k for k in ("q", "k", "v", "g", "beta", "b", "w", "h0", "cu_seqlens") if inp.get(k) is not None]
    host = {k: inp[k].pin_memory() for k in in_keys}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    h_host = torch.empty(hT.shape, dtype=hT.dtype).pin_memory()
    h2d = sum(host[k].numel() * host[k].element_size() for k in in_keys)
    d2h = o_host.numel() * o_host.element_size() + h_host.numel() * h_host.element_size()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        dd = dict(inp)
        for k in in_keys:
            dd[k] = host[k].to(dev, non_blocking=True)
        oo, hh = step(dd, None, None)
        o_host.copy_(oo, non_blocking=True)
        h_host.copy_(hh, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws)

    flops, nbytes = algorithmic(w)
    overhead = output_overhead_bytes(w, o_dtype)
    tokens = w.B * w.T
    ms_per_step = elapsed_ms / args.steps
    value = job_throughput(tokens, ws, ms_per_step)
    peaks, peaks_src = load_peaks()
    t_launch = launch_ms * 1e-3
    gbs = nbytes / t_launch / 1e9
    tflops = flops / t_launch / 1e12
    hbm_frac = gbs / peaks["hbm_gbs"]
    flop_frac = tflops / peaks["bf16_tflops"]
    bound = "hbm" if nbytes / peaks["hbm_gbs"] >= flops / (peaks["bf16_tflops"] * 1e3) else "tensor"
    # the path's kernels: on the tensor-core path the WY kernel and then the chunk kernel run one after the
    # other on the stream, with no overlap; the roofline is taken over the whole step: the operation's
    # algorithmic bytes (o in q's dtype) against the step's device time
    kname = {"tc": "gdn_tc_wy_kernel+gdn_tc_fwd_kernel" if w.variant == "gdn"
             else "gdn2_tc_prep_kernel+gdn2_tc_fwd_kernel", "simt": "gdn_simt_fwd_kernel"}.get(kernel, kernel)
    traffic = recorded_traffic(kname, w.name)
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(hbm_frac, 4), "traffic": traffic}
    else:
        roof = {"bound": "tensor", "achieved": round(tflops, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(flop_frac, 4), "traffic": traffic}
    roof.update({"peak_source": f"{peaks_src} (MEASURED_PEAKS.json burst figures)" if peaks_src == "measured"
                 else "fallback", "kernel": kname, "algorithmic_bytes": int(nbytes),
                 "algorithmic_flops": int(flops), "overhead_bytes": int(overhead),
                 "launch_ms": round(launch_ms, 5), "kernel_ms": kernel_ms,
                 "tflops": round(tflops, 2), "tensor_frac": round(flop_frac, 4),
                 "frac_of_roofline": round(max(hbm_frac, flop_frac), 4)})

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "variant": w.variant, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk,
                       "dv": w.dv, "BT": C, "n_seqs": n_seq, "kernel": kernel, "o_dtype": o_dtype,
                       "state_dtype": "f32", "parallelism": f"dp{ws} (independent batches per rank)",
                       "l2": f"no flush: {(nbytes + overhead) / 1e6:.0f} MB of HBM traffic per step > 126 MB L2"},
            "tflops": round(ws * flops / (ms_per_step * 1e-3) / 1e12, 2),
            "roofline": roof,
            "e2e": {"value": job_throughput(tokens, ws, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "clocks": sampler.summary()}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp, w, args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------------------ the other rows
def run_row(args, w):
    """Device throughput of one of the path's other kernels on the bench workload's shape (1 GPU, rank 0 prints):
    ``decode`` -- one recurrent decode step for 64 sequences of the workload's heads (state read and written in
    place); ``prelude`` -- short conv + SiLU + L2 norm + gates over the whole workload; ``output_gate`` -- the
    RMSNorm x SiLU epilogue over the workload's output; ``bwd`` -- the backward pass of the workload (GDN or
    GDN-2).  Each is reported against the HBM roofline of its bytes per launch."""
    import torch
    from gated_delta_rule_105_b200 import decode_fwd, output_gate_fwd, prelude_fwd, profile_enable, profile_take
    from gated_delta_rule_105_b200.inputs import generate, generate_prelude
    rank, local_rank, ws = dist_env()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    if args.path == "decode":
        N = 64
        inp = generate(N, 1, H, dk, dv, w.dtype, w.seed, w.variant if w.variant != "gdn2" else "gdn2", 0.02)
        d = {k: (v[:, 0].contiguous().to(dev) if isinstance(v, torch.Tensor) and k not in ("h0", "cu_seqlens")
                 else v) for k, v in inp.items()}
        state = inp["h0"].to(dev)
        o = torch.empty((N, H, dv), dtype=d["q"].dtype, device=dev)
        variant = w.variant

        def step():
            decode_fwd(d["q"], d["k"], d["v"], d["g"], d.get("beta"), state, d["scale"], o=o, b=d.get("b"),
                       w=d.get("w"), variant=variant)
        s = 2 if w.dtype == "bf16" else 4
        gate_b = 8 if variant == "gdn" else 4 * (2 * dk + dv)
        nbytes = N * H * (2 * 4 * dk * dv + s * (2 * dk + 2 * dv) + gate_b)
        tokens, kname, workload = N, "gdn_decode_kernel", f"decode N{N} H{H} dk{dk} dv{dv} ({w.name} heads)"
    elif args.path == "prelude":
        inp = generate_prelude(B, T, H, dk, dv, w.dtype, w.seed)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}

        def step():
            prelude_fwd(d["xq"], d["xk"], d["xv"], d["wq"], d["wk"], d["wv"], d["a"], d["A_log"], d["dt_bias"], d["b"])
        s = 2 if w.dtype == "bf16" else 4
        nbytes = B * T * H * (2 * s * (2 * dk + dv) + 4 * 4)
        tokens, kname, workload = B * T, "gdn_prelude_kernel", f"prelude B{B} T{T} H{H} dk{dk} dv{dv}"
    elif args.path == "bwd":
        from gated_delta_rule_105_b200 import (bwd_workspace_bytes, gdn2_bwd_workspace_bytes, gdn2_chunk_bwd,
                                               gdn_chunk_bwd)
        gdn2 = w.variant == "gdn2"
        inp = generate(B, T, H, dk, dv, w.dtype, w.seed, w.variant, w.h0_std or 0.02, w.n_seqs, w.len_range)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        gen = torch.Generator().manual_seed(w.seed + 1)
        d_o = torch.randn((B, T, H, dv), generator=gen).to(d["q"].dtype).to(dev)
        n_seq = d["h0"].shape[0]
        dhT = torch.randn((n_seq, H, dk, dv), generator=gen).mul_(0.5).to(dev)
        n_ws = (gdn2_bwd_workspace_bytes if gdn2 else bwd_workspace_bytes)(
            B, T, H, dk, dv, C, 0 if d["cu_seqlens"] is None else n_seq)
        wsp = torch.empty(n_ws, dtype=torch.uint8, device=dev)

        def step():
            if gdn2:
                gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["b"], d["w"], d_o, d["scale"], d["h0"], dhT,
                               d["cu_seqlens"], workspace=wsp)
            else:
                gdn_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d_o, d["scale"], d["h0"], dhT,
                              d["cu_seqlens"], workspace=wsp)
        s = 2 if w.dtype == "bf16" else 4
        if gdn2:  # read q, k, v, d_o, g, b, w, h0, dhT; write dq, dk, dg, db, dv, dw (fp32), dh0
            nbytes = B * T * H * (s * (2 * dk + 2 * dv) + 4 * (2 * dk + dv) + 4 * (4 * dk + 2 * dv))
        else:  # read q, k, v, d_o, g, beta, h0, dhT; write dq, dk, dv (fp32), dg, dbeta, dh0
            nbytes = B * T * H * (s * (2 * dk + 2 * dv) + 8 + 4 * (2 * dk + dv) + 8)
        nbytes += 3 * n_seq * H * dk * dv * 4
        tokens, kname, workload = B * T, "gdn_bwd_kernels", f"backward {w.name}"
    else:
        gen = torch.Generator().manual_seed(w.seed)
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        o_in = torch.randn((B, T, H, dv), generator=gen).to(tdt).to(dev)
        z = torch.randn((B, T, H, dv), generator=gen).to(tdt).to(dev)
        wt = torch.rand(dv, generator=gen).add_(0.5).to(dev)
        y = torch.empty_like(o_in)

        def step():
            output_gate_fwd(o_in, z, wt, y=y)
        nbytes = B * T * H * dv * 3 * o_in.element_size()
        tokens, kname, workload = B * T, "gdn_output_gate_kernel", f"output gate B{B} T{T} H{H} dv{dv}"
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    profile_take()
    profile_enable(True)
    for _ in range(max(3, min(args.steps, 20))):
        step()
    torch.cuda.synchronize(dev)
    profile_enable(False)
    taken = profile_take()
    n_l, ms_l = taken[kname]
    if args.path == "bwd":  # the backward's forward recompute (SIMT or tensor-core kernels) belongs to the same step
        ms_l = sum(ms * n_l / max(n, 1) for name, (n, ms) in taken.items() if name != kname) + ms_l
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    with sampler:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    peaks, src = load_peaks()
    kernel_ms = ms_l / n_l
    gbs = nbytes / (kernel_ms * 1e-3) / 1e9
    line = {"metric": f"{args.path} tokens/s, % of B200 HBM roofline (1 GPU)", "value": tokens / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": workload, "path": args.path},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": None, "kernel": kname,
                         "algorithmic_bytes": int(nbytes), "kernel_ms": round(kernel_ms, 5),
                         "peak_source": src},
            "gpu_launches": args.steps, "clocks": sampler.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--o-dtype", default="bf16", choices=["f32", "bf16"],
                    help="output dtype for bf16 inputs: bf16 (q's dtype, as the operation defines o) or f32 "
                         "(its extra bytes are reported as roofline.overhead_bytes, not as algorithmic work)")
    ap.add_argument("--path", default="chunk", choices=["chunk", "decode", "prelude", "output_gate", "bwd"],
                    help="chunk: the chunked forward (the headline); the others time that row's kernel alone")
    ap.add_argument("--batch", type=int, default=0,
                    help="run the workload with this many sequences instead of its own B (a smaller case of the same "
                         "shapes, e.g. for an ncu capture); not for packed-sequence workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=120.0, help="seconds for the whole reference arm")
    args = ap.parse_args(argv)
    from gated_delta_rule_105_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.batch:
        if w.n_seqs or args.batch < 1:
            ap.error("--batch needs a positive count and a workload of equal-length sequences")
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name}_batch{args.batch}")
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args, w)
    if args.path != "chunk":
        return run_row(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
