// SIMT (fp32 FMA) chunked forward kernel for GDN and GDN-2.
//
// One CTA owns one (sequence n, head h, block of DVT value columns) and walks that sequence's chunks of
// 64 tokens in order, keeping its DK x DVT slice of the state in shared memory (fp32).  The value columns
// of the state never interact (every update is a left-multiplication on the key axis plus a rank-one
// write), so slicing dv across CTAs is exact.  All arithmetic is fp32 on CUDA cores: this is the path
// for fp32 inputs (tensor-core operand rounding would exceed a 1e-4 error budget) and the simple
// reference path for bf16 inputs.
//
// Per chunk (rows r, s < 64; zero rows pad a partial chunk, which makes them inert: k = v = 0,
// beta = b = w = 0 and g = 0 so the padded cumulative gate stays at the last real token's value):
//   G_r   = log2(e) * sum_{s<=r} g_s                           (GDN-2: per key channel)
// For fp32 inputs G is accumulated and differenced in fp64: with strong decay |G| reaches ~10^3 inside a
// chunk, where an fp32 cumsum loses ~1e-4 absolute in G_r - G_s for nearby r, s -- as much as the whole
// fp32 error budget; only the (small) differences are rounded to fp32 before exp2.  For bf16 inputs
// (a 2e-2 budget) the per-channel GDN-2 gate is kept in fp32, which halves its shared-memory traffic.
//   A_rs  = beta_r (k_r . k_s) 2^(G_r - G_s)        s < r      (GDN-2: sum_i b_ri k_ri k_si 2^(G_ri - G_si))
//   P_rs  = (q_r . k_s) 2^(G_r - G_s)               s <= r     (GDN-2: per-channel factor inside the sum)
//   Tm    = (I + A)^-1                               forward substitution row by row, each row's sums
//                                                    split over four threads per column
//   X     = beta V - diag(beta 2^G) K h              (GDN-2: w.V - (b.2^G.K) h)
//   U     = Tm X
//   O     = scale [ (Q . 2^G) h + P U ]
//   h    <- 2^(G_last) h + (K . 2^(G_last - G))^T U  (GDN-2: Diag(2^G_last) h + (K . 2^(G_last - G))^T U)
// This is the WY form of the intra-chunk dependency and the chunk-to-chunk state pass described in the
// GatedDeltaNet data-flow walkthrough (yfxerp.com/news/367755), section "Chunked parallelism", and for
// GDN-2 in the Gated DeltaNet-2 article (7minutos.es), section "Entrenamiento fragmentado".
#pragma once

#include "gdn_common.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;
// value columns per CTA: GDN-2 keeps a per-channel fp64 gate in shared memory, so it takes a narrower slice
template <bool GDN2> struct SimtDVT { static constexpr int value = GDN2 ? 16 : 32; };

// Shared-memory map in 4-byte words.  The fp64 gate block comes first so it is 8-byte aligned.
template <int DK, int DVT, bool GDN2, int GW = 2>
struct SimtSmem {  // GW: 4-byte words per cumulative-gate element (2: fp64, 1: fp32)
    static constexpr int LDK = DK + 1;  // padded row stride: conflict-free column walks
    static constexpr int LDT = kChunk + 1;
    static constexpr int nK = kChunk * LDK;
    static constexpr int oGd = 0;                               // cumulative gate: GDN-2 [64][LDK], GDN [64] (fp64)
    static constexpr int oK = oGd + (GDN2 ? GW * nK : 2 * kChunk);  // K [64][LDK]
    static constexpr int oQ = oK + nK;                         // Q, then Q.2^G (GDN-2)
    static constexpr int oBK = oQ + nK;                        // GDN-2: b.K, then b.K.2^G, then K.2^(G_last-G)
    static constexpr int oV = oBK + (GDN2 ? nK : 0);           // scaled V, then X
    static constexpr int oH = oV + kChunk * DVT;               // state slice [DK][DVT]
    static constexpr int oA = oH + DK * DVT;                   // A [64][LDT]; its space then holds U [64][DVT]
    static constexpr int oT = oA + kChunk * LDT;               // (I+A)^-1
    static constexpr int oP = oT + kChunk * LDT;               // P
    static constexpr int oB1 = oP + kChunk * LDT;              // GDN: beta [64]
    static constexpr int oF = oB1 + kChunk;                    // GDN: 2^(G_last - G_s) [64]
    static constexpr int total = oF + kChunk;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
    static_assert(kChunk * DVT <= kChunk * LDT, "U must fit in the space of A");
};

// Per-channel (GDN-2) cumulative-gate type: fp64 for fp32 inputs, fp32 for bf16 inputs.
template <typename TIn> struct SimtGate { using type = double; };
template <> struct SimtGate<__nv_bfloat16> { using type = float; };

template <typename TIn, typename TOut, int DK, int DVT, bool GDN2>
__global__ void __launch_bounds__(kSimtThreads)
gdn_simt_fwd_kernel(FwdParams p, unsigned* err) {
    using GT = typename SimtGate<TIn>::type;
    using L = SimtSmem<DK, DVT, GDN2, sizeof(GT) / 4>;
    constexpr int LDK = L::LDK, LDT = L::LDT, NT = kSimtThreads;
    constexpr int PER = kChunk * DVT / NT;  // (row, column) outputs per thread
    static_assert(kChunk * DVT % NT == 0, "tile must divide evenly");
    extern __shared__ __align__(16) float sm[];
    GT* sG = reinterpret_cast<GT*>(sm + L::oGd);              // GDN-2 [64][LDK]
    double* sG1 = reinterpret_cast<double*>(sm + L::oGd);     // GDN [64]
    float* sK = sm + L::oK;
    float* sQ = sm + L::oQ;
    float* sBK = sm + L::oBK;
    float* sV = sm + L::oV;
    float* sH = sm + L::oH;
    float* sA = sm + L::oA;
    float* sU = sm + L::oA;  // U is formed after (I+A)^-1, when A is no longer needed
    float* sT = sm + L::oT;
    float* sP = sm + L::oP;
    float* sB1 = sm + L::oB1;
    float* sF = sm + L::oF;

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * DVT;
    const int h = blockIdx.y;
    const int n = blockIdx.z;
    const int H = p.H, dv = p.dv, T = p.T;
    const TIn* __restrict__ q = static_cast<const TIn*>(p.q);
    const TIn* __restrict__ k = static_cast<const TIn*>(p.k);
    const TIn* __restrict__ v = static_cast<const TIn*>(p.v);
    TOut* __restrict__ o = static_cast<TOut*>(p.o);

    int row, bos, eos;
    if (p.cu_seqlens) {
        row = 0;
        bos = p.cu_seqlens[n];
        eos = p.cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > T) {
            if (tid == 0) atomicOr(err, kErrSeqlens);
            return;
        }
    } else {
        row = n;
        bos = 0;
        eos = T;
    }

    const size_t state_base = ((size_t)n * H + h) * DK * (size_t)dv + j0;
    for (int e = tid; e < DK * DVT; e += NT) {
        const int i = e / DVT, j = e % DVT;
        sH[e] = p.h0 ? p.h0[state_base + (size_t)i * dv + j] : 0.f;
    }

    for (int c0 = bos; c0 < eos; c0 += kChunk) {
        const int Lc = min(kChunk, eos - c0);
        __syncthreads();  // the previous chunk is done with every buffer
        if (p.h_chunks) {  // the state at this chunk's start, for the backward pass
            float* hc = p.h_chunks + ((size_t)wy_slot(n, (long long)row * T + bos, (c0 - bos) / kChunk) * H + h) *
                                         DK * (size_t)dv + j0;
            for (int e = tid; e < DK * DVT; e += NT) hc[(size_t)(e / DVT) * dv + e % DVT] = sH[e];
        }
        // ---- load the chunk (zero-padded past Lc); unrolled so that many global loads are in flight
#pragma unroll 8
        for (int e = tid; e < kChunk * DK; e += NT) {
            const int r = e / DK, i = e % DK;
            float kv = 0.f, qv = 0.f, gv = 0.f, bv = 0.f;
            if (r < Lc) {
                const size_t tok = ((size_t)row * T + c0 + r) * H + h;
                kv = to_f32(k[tok * DK + i]);
                qv = to_f32(q[tok * DK + i]);
                if (GDN2) {
                    gv = p.g[tok * DK + i];
                    bv = p.kda ? p.beta[tok] : p.beta[tok * DK + i];
                }
            }
            sK[r * LDK + i] = kv;
            sQ[r * LDK + i] = qv;
            if (GDN2) {
                sG[r * LDK + i] = (GT)gv;
                sBK[r * LDK + i] = bv * kv;
            }
        }
#pragma unroll
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float x = 0.f;
            if (r < Lc) {
                const size_t tok = ((size_t)row * T + c0 + r) * H + h;
                const float vv = to_f32(v[tok * dv + j0 + j]);
                x = (GDN2 && !p.kda ? p.w[tok * dv + j0 + j] : p.beta[tok]) * vv;
            }
            sV[e] = x;
        }
        if (!GDN2 && tid < kChunk) {
            const int r = tid;
            const size_t tok = ((size_t)row * T + c0 + r) * H + h;
            sG1[r] = r < Lc ? (double)p.g[tok] : 0.0;
            sB1[r] = r < Lc ? p.beta[tok] : 0.f;
        }
        __syncthreads();
        // ---- chunk-local cumulative gate, base 2
        if (GDN2) {
            for (int i = tid; i < DK; i += NT) {
                double acc = 0.0;
                for (int r = 0; r < kChunk; ++r) {
                    acc += (double)sG[r * LDK + i];
                    sG[r * LDK + i] = (GT)(acc * kLog2eD);
                }
            }
        } else if (tid == 0) {
            double acc = 0.0;
            for (int r = 0; r < kChunk; ++r) {
                acc += sG1[r];
                sG1[r] = acc * kLog2eD;
            }
        }
        __syncthreads();
        // ---- A (strictly lower) and P (lower incl. diagonal)
        if (GDN2) {
            // 2x2 tiles (rows 2R, 2R+1; columns 2S, 2S+1) on and below the diagonal, S <= R: each channel's
            // operands are loaded once per tile instead of once per entry.  Entries above the diagonal of a
            // diagonal tile are computed and then discarded.
            constexpr int kTiles = (kChunk / 2) * (kChunk / 2 + 1) / 2;
            for (int tt = tid; tt < kTiles; tt += NT) {
                int R = (int)((sqrtf(8.f * (float)tt + 1.f) - 1.f) * 0.5f);
                while (R * (R + 1) / 2 > tt) --R;
                while ((R + 1) * (R + 2) / 2 <= tt) ++R;
                const int S = tt - R * (R + 1) / 2;
                const int r0 = 2 * R, s0 = 2 * S;
                float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f, p00 = 0.f, p01 = 0.f, p10 = 0.f, p11 = 0.f;
                for (int i = 0; i < DK; ++i) {
                    const GT gr0 = sG[r0 * LDK + i], gr1 = sG[(r0 + 1) * LDK + i];
                    const GT gs0 = sG[s0 * LDK + i], gs1 = sG[(s0 + 1) * LDK + i];
                    const float k0 = sK[s0 * LDK + i], k1 = sK[(s0 + 1) * LDK + i];
                    const float b0 = sBK[r0 * LDK + i], b1 = sBK[(r0 + 1) * LDK + i];
                    const float q0 = sQ[r0 * LDK + i], q1 = sQ[(r0 + 1) * LDK + i];
                    const float k00 = k0 * exp2f((float)(gr0 - gs0)), k01 = k1 * exp2f((float)(gr0 - gs1));
                    const float k10 = k0 * exp2f((float)(gr1 - gs0)), k11 = k1 * exp2f((float)(gr1 - gs1));
                    a00 = fmaf(b0, k00, a00);
                    a01 = fmaf(b0, k01, a01);
                    a10 = fmaf(b1, k10, a10);
                    a11 = fmaf(b1, k11, a11);
                    p00 = fmaf(q0, k00, p00);
                    p01 = fmaf(q0, k01, p01);
                    p10 = fmaf(q1, k10, p10);
                    p11 = fmaf(q1, k11, p11);
                }
                const bool diag = R == S;  // then (r0, s0 + 1) is above the diagonal
                sA[r0 * LDT + s0] = diag ? 0.f : a00;
                sA[r0 * LDT + s0 + 1] = diag ? 0.f : a01;
                sA[(r0 + 1) * LDT + s0] = a10;
                sA[(r0 + 1) * LDT + s0 + 1] = diag ? 0.f : a11;
                sP[r0 * LDT + s0] = p00;
                sP[r0 * LDT + s0 + 1] = diag ? 0.f : p01;
                sP[(r0 + 1) * LDT + s0] = p10;
                sP[(r0 + 1) * LDT + s0 + 1] = p11;
                if (!diag) {  // the mirrored tile above the diagonal is zero
                    sA[s0 * LDT + r0] = 0.f;
                    sA[s0 * LDT + r0 + 1] = 0.f;
                    sA[(s0 + 1) * LDT + r0] = 0.f;
                    sA[(s0 + 1) * LDT + r0 + 1] = 0.f;
                    sP[s0 * LDT + r0] = 0.f;
                    sP[s0 * LDT + r0 + 1] = 0.f;
                    sP[(s0 + 1) * LDT + r0] = 0.f;
                    sP[(s0 + 1) * LDT + r0 + 1] = 0.f;
                }
            }
        } else {
        for (int e = tid; e < kChunk * kChunk; e += NT) {
            const int r = e / kChunk, s = e % kChunk;
            float a = 0.f, pp = 0.f;
            if (s <= r) {
                {
                    float dkk = 0.f, dqk = 0.f;
                    for (int i = 0; i < DK; ++i) {
                        const float ks = sK[s * LDK + i];
                        dkk = fmaf(sK[r * LDK + i], ks, dkk);
                        dqk = fmaf(sQ[r * LDK + i], ks, dqk);
                    }
                    const float f = exp2f((float)(sG1[r] - sG1[s]));
                    a = sB1[r] * f * dkk;
                    pp = f * dqk;
                }
                if (s == r) a = 0.f;
            }
            sA[r * LDT + s] = a;
            sP[r * LDT + s] = pp;
        }
        }
        __syncthreads();
        // ---- GDN-2: fold 2^G into Q and b.K (in place); (I + A)^-1 by forward substitution
        if (GDN2) {
            for (int e = tid; e < kChunk * DK; e += NT) {
                const int r = e / DK, i = e % DK;
                const float f = exp2f((float)sG[r * LDK + i]);
                sQ[r * LDK + i] *= f;
                sBK[r * LDK + i] *= f;
            }
        }
        // T[r][c] = [r == c] - sum_{c <= s < r} A[r][s] T[s][c], row by row: the four threads of column c
        // take every fourth s and add their sums by shuffles (they are adjacent lanes of one warp)
        {
            static_assert(NT == 4 * kChunk, "four threads per column");
            const int c = tid >> 2, part = tid & 3;
            for (int r = 0; r < kChunk; ++r) {
                float acc = 0.f;
                for (int s = c + part; s < r; s += 4) acc = fmaf(sA[r * LDT + s], sT[s * LDT + c], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                if (part == 0) sT[r * LDT + c] = r < c ? 0.f : (r == c ? 1.f : -acc);
                __syncthreads();
            }
        }
        // ---- X = (scaled V) - (erase-side keys . 2^G) h ;  Oi = (Q . 2^G) h  (kept in registers)
        float oi[PER];
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int e = tid + m * NT;
            const int r = e / DVT, j = e % DVT;
            float kh = 0.f, qh = 0.f;
            if (GDN2) {
                for (int i = 0; i < DK; ++i) {
                    const float hv = sH[i * DVT + j];
                    kh = fmaf(sBK[r * LDK + i], hv, kh);
                    qh = fmaf(sQ[r * LDK + i], hv, qh);
                }
                sV[e] -= kh;
                oi[m] = qh;
            } else {
                for (int i = 0; i < DK; ++i) {
                    const float hv = sH[i * DVT + j];
                    kh = fmaf(sK[r * LDK + i], hv, kh);
                    qh = fmaf(sQ[r * LDK + i], hv, qh);
                }
                const float f = exp2f((float)sG1[r]);
                sV[e] -= sB1[r] * f * kh;
                oi[m] = f * qh;
            }
        }
        __syncthreads();
        // ---- U = (I+A)^-1 X ; decay factors for the state update
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int e = tid + m * NT;
            const int r = e / DVT, j = e % DVT;
            float u = 0.f;
            for (int s = 0; s <= r; ++s) u = fmaf(sT[r * LDT + s], sV[s * DVT + j], u);
            sU[e] = u;
        }
        if (GDN2) {
            for (int e = tid; e < kChunk * DK; e += NT) {
                const int s = e / DK, i = e % DK;
                sBK[s * LDK + i] = sK[s * LDK + i] * exp2f((float)(sG[(kChunk - 1) * LDK + i] - sG[s * LDK + i]));
            }
        } else if (tid < kChunk) {
            sF[tid] = exp2f((float)(sG1[kChunk - 1] - sG1[tid]));
        }
        __syncthreads();
        // ---- O = scale (Oi + P U) ; h <- 2^G_last h + Ktilde^T U
#pragma unroll
        for (int m = 0; m < PER; ++m) {
            const int e = tid + m * NT;
            const int r = e / DVT, j = e % DVT;
            float acc = oi[m];
            for (int s = 0; s <= r; ++s) acc = fmaf(sP[r * LDT + s], sU[s * DVT + j], acc);
            if (o && r < Lc) {  // o is null when only the chunk states are wanted (backward pass)
                const size_t tok = ((size_t)row * T + c0 + r) * H + h;
                o[tok * dv + j0 + j] = from_f32<TOut>(p.scale * acc);
            }
        }
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            float acc;
            if (GDN2) {
                acc = exp2f((float)sG[(kChunk - 1) * LDK + i]) * sH[e];
                for (int s = 0; s < kChunk; ++s) acc = fmaf(sBK[s * LDK + i], sU[s * DVT + j], acc);
            } else {
                acc = exp2f((float)sG1[kChunk - 1]) * sH[e];
                for (int s = 0; s < kChunk; ++s) acc = fmaf(sK[s * LDK + i] * sF[s], sU[s * DVT + j], acc);
            }
            sH[e] = acc;
        }
    }
    __syncthreads();
    if (p.hT) {
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            p.hT[state_base + (size_t)i * dv + j] = sH[e];
        }
    }
}

}  // namespace gdn
