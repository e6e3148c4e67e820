"""Seeded synthetic inputs for the gated delta rule forward pass.

This module holds only input generation: it draws the tensors a Gated DeltaNet layer would hand to
its token mixer, using the layer's own gate recipe, and none of the mixer's arithmetic.  Both the
CUDA path (tests, bench) and the fp64 oracle consume what it returns.

Recipe (gate math from the GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755, section
"Gating"; GDN-2 gates from the Gated DeltaNet-2 article, 7minutos.es, section "Regla-2 del Delta
cerrado" and "Diseno de bloques"):
  * generator: numpy PCG64 seeded with ``seed``; draw order A_log[H], dt_bias[H], q, k, v, gate
    noise, beta noise (GDN-2: erase-gate noise, write-gate noise), h0 -- each row-major over its
    layout.  Bulk normals are drawn in float64 for fp32 inputs and float32 for bf16 inputs.
  * q, k ~ N(0,1), then L2-normalised over the head dimension; v ~ N(0,1).
  * A_log = log(U(1,16)) and dt_bias ~ N(0, 0.1) per head (0.1 read as a standard deviation).
  * g = -exp(A_log) * softplus(N(0,1) + dt_bias): per token (GDN) or per token and key channel (GDN-2).
  * beta = sigmoid(N(0,1)); GDN-2 erase gate b[..,dk] and write gate w[..,dv] = sigmoid(N(0,1)).
  * h0 = 0, or N(0, h0_std) when ``h0_std`` > 0; scale = dk^-1/2.
  * q, k, v are rounded (round-to-nearest-even) to the input dtype; g, beta, b, w, h0 stay fp32.
  * packed variable-length batches: n_seqs lengths drawn uniformly from [lo, hi], rescaled to the
    total, rounded, remainder into the last; redrawn until every length lies in [lo, hi].
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    variant: str  # "gdn" or "gdn2"
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str  # "f32" or "bf16" (q, k, v, o)
    seed: int
    h0_std: float = 0.0
    n_seqs: int = 0  # > 0: one packed row of T tokens split into n_seqs sequences
    len_range: tuple = field(default=(512, 8192))

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads the method is measured on, by what they are.
WORKLOADS = {
    "gdn_tiny_f32_b1h2t256_d64": Workload("gdn_tiny_f32_b1h2t256_d64", "gdn", 1, 256, 2, 64, 64, "f32", 1000),
    "gdn_bf16_b8h8t4096_dk128_dv128": Workload("gdn_bf16_b8h8t4096_dk128_dv128", "gdn", 8, 4096, 8, 128, 128,
                                               "bf16", 1001),
    "gdn_bf16_b4h16t4096_dk128_dv256_h0": Workload("gdn_bf16_b4h16t4096_dk128_dv256_h0", "gdn", 4, 4096, 16, 128,
                                                   256, "bf16", 1002, h0_std=0.02),
    "gdn_bf16_varlen65536x16_h16_dk128_dv256": Workload("gdn_bf16_varlen65536x16_h16_dk128_dv256", "gdn", 1, 65536,
                                                        16, 128, 256, "bf16", 1003, n_seqs=16),
    "gdn2_bf16_b4h16t4096_dk128_dv128": Workload("gdn2_bf16_b4h16t4096_dk128_dv128", "gdn2", 4, 4096, 16, 128, 128,
                                                 "bf16", 1004),
}
WORKLOAD_ORDER = list(WORKLOADS)


def _softplus(x):
    return np.logaddexp(0.0, x)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def draw_lengths(rng, n, total, lo, hi):
    """n sequence lengths in [lo, hi] summing to ``total`` (see module docstring)."""
    while True:
        raw = rng.integers(lo, hi + 1, size=n).astype(np.float64)
        lens = np.rint(raw * (total / raw.sum())).astype(np.int64)
        lens[-1] = total - lens[:-1].sum()
        if lens.min() >= lo and lens.max() <= hi:
            return lens


def _torch_dtype(dt):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dt]


def generate(B, T, H, dk, dv, dtype="bf16", seed=0, variant="gdn", h0_std=0.0, n_seqs=0,
             len_range=(512, 8192), cu_seqlens=None):
    """Draw one input set.  Returns a dict of CPU torch tensors plus ``scale`` and ``cu_seqlens``.

    q,k [B,T,H,dk] and v [B,T,H,dv] in ``dtype``; GDN: g, beta [B,T,H] fp32; GDN-2: g, b [B,T,H,dk]
    and w [B,T,H,dv] fp32; KDA: g [B,T,H,dk] and beta [B,T,H] fp32; h0 [n_seq,H,dk,dv] fp32 or None;
    cu_seqlens int32 [n_seq+1] or None.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    fdt = np.float64 if dtype == "f32" else np.float32
    A_log = np.log(rng.uniform(1.0, 16.0, size=H))
    dt_bias = rng.normal(0.0, 0.1, size=H)

    def normal(shape):
        return rng.standard_normal(size=shape, dtype=fdt)

    def l2n(x):
        return x / np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True)).astype(fdt)

    q = l2n(normal((B, T, H, dk)))
    k = l2n(normal((B, T, H, dk)))
    v = normal((B, T, H, dv))
    A = np.exp(A_log)
    out = {}
    if variant == "gdn":
        gn = normal((B, T, H)).astype(np.float64)
        g = -A[None, None, :] * _softplus(gn + dt_bias[None, None, :])
        beta = _sigmoid(normal((B, T, H)).astype(np.float64))
        out["g"] = torch.from_numpy(g.astype(np.float32))
        out["beta"] = torch.from_numpy(beta.astype(np.float32))
    elif variant == "gdn2":
        gn = normal((B, T, H, dk)).astype(np.float64)
        g = -A[None, None, :, None] * _softplus(gn + dt_bias[None, None, :, None])
        b = _sigmoid(normal((B, T, H, dk)).astype(np.float64))
        w = _sigmoid(normal((B, T, H, dv)).astype(np.float64))
        out["g"] = torch.from_numpy(g.astype(np.float32))
        out["b"] = torch.from_numpy(b.astype(np.float32))
        out["w"] = torch.from_numpy(w.astype(np.float32))
    elif variant == "kda":  # per-channel decay as GDN-2, one scalar beta per token as GDN
        gn = normal((B, T, H, dk)).astype(np.float64)
        g = -A[None, None, :, None] * _softplus(gn + dt_bias[None, None, :, None])
        beta = _sigmoid(normal((B, T, H)).astype(np.float64))
        out["g"] = torch.from_numpy(g.astype(np.float32))
        out["beta"] = torch.from_numpy(beta.astype(np.float32))
    else:
        raise ValueError(variant)
    if n_seqs > 0 and cu_seqlens is None:
        assert B == 1
        lens = draw_lengths(rng, n_seqs, T, *len_range)
        cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    n_seq = B if cu_seqlens is None else len(cu_seqlens) - 1
    h0 = None
    if h0_std > 0:
        h0 = torch.from_numpy((rng.standard_normal(size=(n_seq, H, dk, dv)) * h0_std).astype(np.float32))
    tdt = _torch_dtype(dtype)
    out.update(
        q=torch.from_numpy(q).to(tdt), k=torch.from_numpy(k).to(tdt), v=torch.from_numpy(v).to(tdt),
        h0=h0, scale=float(dk) ** -0.5,
        cu_seqlens=None if cu_seqlens is None else torch.as_tensor(np.asarray(cu_seqlens, dtype=np.int32)),
    )
    return out


def generate_workload(w: Workload):
    return generate(w.B, w.T, w.H, w.dk, w.dv, w.dtype, w.seed, w.variant, w.h0_std, w.n_seqs, w.len_range)


def generate_prelude(B, T, H, dk, dv, dtype="bf16", seed=0, gate_width=1, write_gate=False, conv_state=False,
                     n_seqs=0, cu_seqlens=None, len_range=(1, 64)):
    """Inputs of the mixer's prelude (projection outputs, conv taps, gate pre-activations, cache), seeded.

    xq, xk [B,T,H,dk] and xv [B,T,H,dv] ~ N(0,1) in ``dtype``; taps wq, wk [H*dk,4], wv [H*dv,4] ~ N(0, 0.5^2);
    a [B,T,H(,gate_width)], b [B,T,H(,gate_width)] ~ N(0,1); c [B,T,H,dv] ~ N(0,1) when ``write_gate``;
    A_log = log U(1,16) and dt_bias ~ N(0, 0.1^2) per head; conv_state [N, 2 H dk + H dv, 3] ~ N(0,1) if asked.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    A_log = np.log(rng.uniform(1.0, 16.0, size=H)).astype(np.float32)
    dt_bias = rng.normal(0.0, 0.1, size=H).astype(np.float32)
    tdt = _torch_dtype(dtype)

    def t(x, dt=torch.float32):
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dt)

    out = {"xq": t(rng.standard_normal((B, T, H, dk)), tdt), "xk": t(rng.standard_normal((B, T, H, dk)), tdt),
           "xv": t(rng.standard_normal((B, T, H, dv)), tdt),
           "wq": t(rng.normal(0, 0.5, (H * dk, 4))), "wk": t(rng.normal(0, 0.5, (H * dk, 4))),
           "wv": t(rng.normal(0, 0.5, (H * dv, 4))),
           "A_log": t(A_log), "dt_bias": t(dt_bias)}
    gshape = (B, T, H) if gate_width == 1 else (B, T, H, gate_width)
    out["a"] = t(rng.standard_normal(gshape))
    out["b"] = t(rng.standard_normal(gshape))
    out["c"] = t(rng.standard_normal((B, T, H, dv))) if write_gate else None
    if n_seqs > 0 and cu_seqlens is None:
        assert B == 1
        lens = draw_lengths(rng, n_seqs, T, *len_range)
        cu_seqlens = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    out["cu_seqlens"] = None if cu_seqlens is None else torch.as_tensor(np.asarray(cu_seqlens, dtype=np.int32))
    n_seq = B if cu_seqlens is None else len(cu_seqlens) - 1
    out["conv_state"] = t(rng.standard_normal((n_seq, 2 * H * dk + H * dv, 3))) if conv_state else None
    return out
