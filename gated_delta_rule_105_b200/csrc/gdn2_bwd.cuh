// Backward pass (reverse mode) of the chunked Gated Delta Rule-2 and of KDA (per-key-channel gates): fp32 on CUDA
// cores.
//
// The forward per chunk of C = 64 tokens (Gated DeltaNet-2 article, 7minutos.es, section "Regla-2 del Delta
// cerrado" for the token recurrence; section "Entrenamiento fragmentado y reconocimiento de puertas hacia atras"
// for the chunked form with the channel decay inside both erase factors), with G the chunk-local cumulative gate
// of every key channel (base 2), D_rsi = 2^(G_ri - G_si), F = 2^G, f_ri = 2^(G_Li - G_ri), Lambda_i = 2^(G_Li), L
// the chunk's last row, E = b . K (KDA: beta_r K_r) and Z = w . V (KDA: beta_r V_r):
//   A_rs = sum_i E_ri K_si D_rsi (s < r),   T = (I + A)^-1,   P_rs = sum_i Q_ri K_si D_rsi (s <= r)
//   X = Z - (E . F) h,  U = T X,  O = scale ((Q . F) h + P U),  h' = Diag(Lambda) h + (K . f)^T U
// Given the cotangents dO and dh' (the article's section on chunked training says that the gate factors enter
// the gradient's dot products; the GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755, section "Chunked
// parallelism", names the full backward of q, k, v, beta and g):
//   dU = scale P^T dO + (K . f) dh'      dX = T^T dU      dZ = dX
//   dh = scale (Q . F)^T dO + Diag(Lambda) dh' - (E . F)^T dX      (chunk to chunk)
//   dT = dU X^T -> dA = -T^T dT T^T (strictly lower),   dP = scale dO U^T (lower)
//   dQ = F . (scale dO h^T) + dP-path,   dE = -F . (dX h^T) + dA-path,   dK = f . (U dh'^T) + dA- and dP-paths
// Every occurrence of Q and E carries 2^(+G_r) and every occurrence of K carries 2^(-G_r), so the gradient of the
// natural-log cumulative gate is  dGn_ri = Q_ri dQ_ri + E_ri dE_ri - K_ri dK_ri, plus, on row L, the terms of
// G_L: sum_r K_ri f_ri (U dh'^T)_ri + Lambda_i sum_j h_ij dh'_ij.  dg is its reverse cumulative sum inside the
// chunk; db = K . dE and dk = dK + b . dE; dv = w . dX and dw = V . dX (KDA: dbeta_r = sum_i K_ri dE_ri +
// sum_j V_rj dX_rj, dv = beta dX).
//
// Four kernels: (1) gdn2_bwd_prep_kernel forms T and P of every (chunk, head) into the workspace;
// (2) gdn2_bwd_states_kernel walks each sequence's chunks forward with T and writes the state at every chunk start;
// (3) gdn2_bwd_dh_kernel walks them backwards with dh in shared memory (one CTA per (sequence, head, 32 value
// columns)) and writes dh' of every chunk; (4) gdn2_bwd_chunk_kernel forms every input gradient of one
// (chunk, head).
#pragma once

#include "gdn_common.cuh"

namespace gdn {

constexpr int kBw2Threads = 256;

struct Bwd2Params {
    const void* q;            // [B,T,H,dk]   (dtype TIn)
    const void* k;
    const void* v;            // [B,T,H,dv]
    const float* g;           // [B,T,H,dk] natural-log decay
    const float* b;           // GDN-2: erase gate [B,T,H,dk]; KDA: beta [B,T,H]
    const float* w;           // GDN-2: write gate [B,T,H,dv]; KDA: unused
    const void* dout;         // dO [B,T,H,dv] (dtype TIn)
    const float* dhT;         // [N,H,dk,dv] or null
    const float* h_chunks;    // [slot][H][dk][dv]: the state at each chunk's start
    float* dh_chunks;         // [slot][H][dk][dv]: the cotangent of each chunk's end state
    float* tp;                // [slot][H][2][64][64]: T, then P, of every chunk
    float* dq;                // [B,T,H,dk] fp32
    float* dk;
    float* dv;                // [B,T,H,dv] fp32
    float* dg;                // [B,T,H,dk] fp32
    float* db;                // GDN-2: [B,T,H,dk]; KDA: dbeta [B,T,H]
    float* dw;                // GDN-2: [B,T,H,dv]; KDA: unused
    float* dh0;               // [N,H,dk,dv] fp32 or null
    const int32_t* cu_seqlens;
    float scale;
    int B, T, H, kdim, vdim, n_seq, kda;
    const float* h0;          // [N,H,dk,dv] or null (zeros): the initial state of the forward walk
};

// Sequence bounds (row, first token, end) of sequence n; false (and the error word) for a bad cu_seqlens entry.
__device__ __forceinline__ bool bw2_seq_bounds(const Bwd2Params& p, int n, int& row, int& bos, int& eos,
                                               unsigned* err) {
    if (p.cu_seqlens) {
        row = 0;
        bos = p.cu_seqlens[n];
        eos = p.cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > p.T) {
            if (threadIdx.x == 0) atomicOr(err, kErrSeqlens);
            return false;
        }
    } else {
        row = n;
        bos = 0;
        eos = p.T;
    }
    return true;
}

// The (first global token, length) of the chunk in workspace slot `slot`; length 0 for a slot no chunk uses.
// Thread 0 decides (binary search over the sequence starts); the result is shared through `info`.
__device__ __forceinline__ void bw2_slot_chunk(const Bwd2Params& p, long long slot, int* info, unsigned* err) {
    if (threadIdx.x == 0) {
        int lo = 0, hi = p.n_seq - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            const long long st0 = p.cu_seqlens ? (long long)p.cu_seqlens[mid] : (long long)mid * p.T;
            if (wy_slot(mid, st0, 0) <= slot) lo = mid;
            else hi = mid - 1;
        }
        int row, bos, eos, Lc = 0;
        if (bw2_seq_bounds(p, lo, row, bos, eos, err)) {
            const long long start = (long long)row * p.T + bos;
            const long long cc = slot - wy_slot(lo, start, 0);
            if (cc >= 0 && cc * kChunk < eos - bos) {
                Lc = min(kChunk, (int)(eos - bos - cc * kChunk));
                info[0] = (int)(start + cc * kChunk);
            }
        }
        info[1] = Lc;
    }
    __syncthreads();
}

// Erase-gate value b_ri of token `tok` (global token index), channel i.
__device__ __forceinline__ float bw2_b(const Bwd2Params& p, size_t tok, int h, int i) {
    return p.kda ? p.b[tok * p.H + h] : p.b[(tok * p.H + h) * p.kdim + i];
}
// Write-gate value w_rj.
__device__ __forceinline__ float bw2_w(const Bwd2Params& p, size_t tok, int h, int j) {
    return p.kda ? p.b[tok * p.H + h] : p.w[(tok * p.H + h) * p.vdim + j];
}

// Chunk-local cumulative gate of channel i, in base 2: the value of row 63 (G_L; rows past Lc add 0).  The sum
// runs in fp64; every kernel rounds it the same way, so T and P from the prep kernel and the gate terms of the
// gradient kernel see identical G.
__device__ __forceinline__ double bw2_gate_last(const Bwd2Params& p, size_t tok0, int h, int i, int Lc) {
    double acc = 0.0;
    for (int r = 0; r < Lc; ++r) acc += (double)p.g[((tok0 + r) * p.H + h) * p.kdim + i];
    return acc * kLog2eD;
}

// T = (I + A)^-1 of a strictly lower A (row-major, leading dimension ldt), row by row, four adjacent threads per
// column splitting each row's sum.  Needs 4 * 64 = 256 threads.
__device__ __forceinline__ void bw2_invert_lower(const float* A, float* T, int ldt) {
    const int col = threadIdx.x >> 2, part = threadIdx.x & 3;
    for (int r = 0; r < kChunk; ++r) {
        float acc = 0.f;
        for (int s = col + part; s < r; s += 4) acc = fmaf(A[r * ldt + s], T[s * ldt + col], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (part == 0) T[r * ldt + col] = r < col ? 0.f : (r == col ? 1.f : -acc);
        __syncthreads();
    }
}

// (0) One CTA per (chunk slot, head): T and P of the chunk into the workspace.
template <int DK>
struct Bw2PrepSmem {  // 4-byte words; the cumulative gate is fp64, transposed [channel][row]
    static constexpr int LDK = DK + 1, LDT = kChunk + 1;
    static constexpr int oGd = 0;  // double [DK][64]
    static constexpr int oK = oGd + 2 * DK * kChunk, oQ = oK + kChunk * LDK, oE = oQ + kChunk * LDK;
    static constexpr int oA = oE + kChunk * LDK, oT = oA + kChunk * LDT;
    static constexpr int total = oT + kChunk * LDT;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads) gdn2_bwd_prep_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2PrepSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, NT = kBw2Threads;
    extern __shared__ __align__(16) float bsm[];
    double* sGd = reinterpret_cast<double*>(bsm + L::oGd);
    float* sK = bsm + L::oK;
    float* sQ = bsm + L::oQ;
    float* sE = bsm + L::oE;
    float* sA = bsm + L::oA;
    float* sT = bsm + L::oT;
    __shared__ int info[2];
    const int tid = threadIdx.x, H = p.H;
    const long long slot = blockIdx.x / H;
    const int h = blockIdx.x % H;
    bw2_slot_chunk(p, slot, info, err);
    const int Lc = info[1];
    if (Lc == 0) return;
    const size_t tok0 = (size_t)info[0];
    const TIn* q = static_cast<const TIn*>(p.q);
    const TIn* k = static_cast<const TIn*>(p.k);
    for (int e = tid; e < kChunk * DK; e += NT) {
        const int r = e / DK, i = e % DK;
        float kv = 0.f, qv = 0.f, bv = 0.f;
        if (r < Lc) {
            const size_t idx = ((tok0 + r) * H + h) * DK + i;
            kv = to_f32(k[idx]);
            qv = to_f32(q[idx]);
            bv = bw2_b(p, tok0 + r, h, i);
        }
        sK[r * LDK + i] = kv;
        sQ[r * LDK + i] = qv;
        sE[r * LDK + i] = bv * kv;
    }
    for (int i = tid; i < DK; i += NT) {
        double acc = 0.0;
        for (int r = 0; r < kChunk; ++r) {
            if (r < Lc) acc += (double)p.g[((tok0 + r) * H + h) * DK + i];
            sGd[i * kChunk + r] = acc * kLog2eD;
        }
    }
    __syncthreads();
    // A and P: thread column s = tid % 64, rows r = tid / 64 + 4 m.  The decay 2^(G_r - G_s) comes from the fp64
    // difference: an fp32 G of a strongly decaying channel (hundreds in magnitude) would cost ~1e-5 of it.
    float* P = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk + kChunk * kChunk;
    const int s = tid & (kChunk - 1);
    for (int r = tid >> 6; r < kChunk; r += NT / kChunk) {
        float a = 0.f, pp = 0.f;
        if (s <= r) {
            for (int i = 0; i < DK; ++i) {
                const float d = exp2f((float)(sGd[i * kChunk + r] - sGd[i * kChunk + s])), ks = sK[s * LDK + i] * d;
                a = fmaf(sE[r * LDK + i], ks, a);
                pp = fmaf(sQ[r * LDK + i], ks, pp);
            }
        }
        sA[r * LDT + s] = s < r ? a : 0.f;
        P[r * kChunk + s] = pp;
    }
    __syncthreads();
    bw2_invert_lower(sA, sT, LDT);
    float* Tg = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk;
    for (int e = tid; e < kChunk * kChunk; e += NT) Tg[e] = sT[(e / kChunk) * LDT + e % kChunk];
}

// Per-channel chunk quantities from the inputs: QF = Q . F, EF = E . F, Kf = K . f and Lambda (any pointer may be
// null).  One thread per channel walks the rows (the cumulative sum runs along them).
template <typename TIn, int DK>
__device__ void bw2_scaled_rows(const Bwd2Params& p, size_t tok0, int h, int Lc, float* QF, float* EF, float* Kf,
                                float* Lam, int ldk) {
    const TIn* q = static_cast<const TIn*>(p.q);
    const TIn* k = static_cast<const TIn*>(p.k);
    for (int i = threadIdx.x; i < DK; i += blockDim.x) {
        const double gl = bw2_gate_last(p, tok0, h, i, Lc);
        if (Lam) Lam[i] = exp2f((float)gl);
        double acc = 0.0;
        for (int r = 0; r < kChunk; ++r) {
            float kv = 0.f, qv = 0.f, bv = 0.f;
            if (r < Lc) {
                const size_t tok = tok0 + r, idx = (tok * p.H + h) * DK + i;
                acc += (double)p.g[idx];
                kv = to_f32(k[idx]);
                if (QF) qv = to_f32(q[idx]);
                bv = bw2_b(p, tok, h, i);
            }
            const double G = acc * kLog2eD;
            const float F = exp2f((float)G), f = exp2f((float)(gl - G));
            if (QF) QF[r * ldk + i] = qv * F;
            if (EF) EF[r * ldk + i] = bv * kv * F;
            if (Kf) Kf[r * ldk + i] = kv * f;
        }
    }
}

// (1) One CTA per (sequence, head, 32 value columns): the state at every chunk start, walked forward with T from
// the prep kernel (the forward's recurrence without its output): X = Z - (E . F) h, U = T X,
// h' = Diag(Lambda) h + (K . f)^T U.  The value columns of the state never mix, so the slices are exact.
template <int DK>
struct Bw2StSmem {  // 4-byte words
    static constexpr int LDK = DK + 1, LDT = kChunk + 1, DVT = 32, LDV = DVT + 1;
    static constexpr int oT = 0, oEF = oT + kChunk * LDT, oKf = oEF + kChunk * LDK, oLam = oKf + kChunk * LDK;
    static constexpr int oH = oLam + DK;         // h [DK][LDV]
    static constexpr int oZ = oH + DK * LDV;     // Z = w . V [64][LDV]
    static constexpr int oX = oZ + kChunk * LDV, oU = oX + kChunk * LDV;
    static constexpr int total = oU + kChunk * LDV;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads) gdn2_bwd_states_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2StSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, NT = kBw2Threads;
    extern __shared__ __align__(16) float bsm[];
    float* sT = bsm + L::oT;
    float* sEF = bsm + L::oEF;
    float* sKf = bsm + L::oKf;
    float* sLam = bsm + L::oLam;
    float* sH = bsm + L::oH;
    float* sZ = bsm + L::oZ;
    float* sX = bsm + L::oX;
    float* sU = bsm + L::oU;
    const int tid = threadIdx.x, j0 = blockIdx.x * DVT, h = blockIdx.y, n = blockIdx.z;
    const int H = p.H, dv = p.vdim;
    int row, bos, eos;
    if (!bw2_seq_bounds(p, n, row, bos, eos, err)) return;
    const long long start = (long long)row * p.T + bos;
    const size_t state_base = ((size_t)n * H + h) * DK * (size_t)dv + j0;
    for (int e = tid; e < DK * DVT; e += NT) {
        const int i = e / DVT, j = e % DVT;
        sH[i * LDV + j] = p.h0 ? p.h0[state_base + (size_t)i * dv + j] : 0.f;
    }
    // the states go into the workspace this launch owns (the parameter block holds them as read-only for the
    // kernels that read them)
    float* h_chunks = const_cast<float*>(p.h_chunks);
    const TIn* vin = static_cast<const TIn*>(p.v);
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    for (int ci = 0; ci < nc; ++ci) {
        const int Lc = min(kChunk, eos - bos - ci * kChunk);
        const size_t tok0 = (size_t)(start + (long long)ci * kChunk);
        const long long slot = wy_slot(n, start, ci);
        __syncthreads();  // the previous chunk is done with every buffer
        float* h_out = h_chunks + ((size_t)slot * H + h) * DK * (size_t)dv + j0;
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            h_out[(size_t)i * dv + j] = sH[i * LDV + j];
        }
        const float* tp = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk;
        for (int e = tid; e < kChunk * kChunk; e += NT) sT[(e / kChunk) * LDT + e % kChunk] = tp[e];
        bw2_scaled_rows<TIn, DK>(p, tok0, h, Lc, nullptr, sEF, sKf, sLam, LDK);
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float z = 0.f;
            if (r < Lc) {
                const size_t tok = tok0 + r;
                z = bw2_w(p, tok, h, j0 + j) * to_f32(vin[(tok * H + h) * dv + j0 + j]);
            }
            sZ[r * LDV + j] = z;
        }
        __syncthreads();
        // X = Z - (E . F) h
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float acc = 0.f;
            for (int i = 0; i < DK; ++i) acc = fmaf(sEF[r * LDK + i], sH[i * LDV + j], acc);
            sX[r * LDV + j] = sZ[r * LDV + j] - acc;
        }
        __syncthreads();
        // U = T X
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float acc = 0.f;
            for (int s2 = 0; s2 <= r; ++s2) acc = fmaf(sT[r * LDT + s2], sX[s2 * LDV + j], acc);
            sU[r * LDV + j] = acc;
        }
        __syncthreads();
        // h' = Diag(Lambda) h + (K . f)^T U
        float nh[DK * DVT / NT];
#pragma unroll
        for (int m = 0; m < DK * DVT / NT; ++m) {
            const int e = tid + m * NT, i = e / DVT, j = e % DVT;
            float acc = sLam[i] * sH[i * LDV + j];
            for (int r = 0; r < kChunk; ++r) acc = fmaf(sKf[r * LDK + i], sU[r * LDV + j], acc);
            nh[m] = acc;
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < DK * DVT / NT; ++m) {
            const int e = tid + m * NT;
            sH[(e / DVT) * LDV + e % DVT] = nh[m];
        }
    }
}

template <int DK>
struct Bw2DhSmem {  // 4-byte words
    static constexpr int LDK = DK + 1, LDT = kChunk + 1, DVT = 32, LDV = DVT + 1;
    static constexpr int oT = 0, oP = oT + kChunk * LDT, oQF = oP + kChunk * LDT, oEF = oQF + kChunk * LDK;
    static constexpr int oKf = oEF + kChunk * LDK, oLam = oKf + kChunk * LDK;
    static constexpr int oDh = oLam + DK;        // dh [DK][LDV]
    static constexpr int oDo = oDh + DK * LDV;   // dO [64][LDV]
    static constexpr int oDu = oDo + kChunk * LDV, oDx = oDu + kChunk * LDV;
    static constexpr int total = oDx + kChunk * LDV;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// (3) One CTA per (sequence, head, 32 value columns): the state cotangent, walked from the last chunk to the first.
template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads) gdn2_bwd_dh_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2DhSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, NT = kBw2Threads;
    extern __shared__ __align__(16) float bsm[];
    float* sT = bsm + L::oT;
    float* sP = bsm + L::oP;
    float* sQF = bsm + L::oQF;
    float* sEF = bsm + L::oEF;
    float* sKf = bsm + L::oKf;
    float* sLam = bsm + L::oLam;
    float* sDh = bsm + L::oDh;
    float* sDo = bsm + L::oDo;
    float* sDu = bsm + L::oDu;
    float* sDx = bsm + L::oDx;
    const int tid = threadIdx.x, j0 = blockIdx.x * DVT, h = blockIdx.y, n = blockIdx.z;
    const int H = p.H, dv = p.vdim;
    int row, bos, eos;
    if (!bw2_seq_bounds(p, n, row, bos, eos, err)) return;
    const long long start = (long long)row * p.T + bos;
    const size_t state_base = ((size_t)n * H + h) * DK * (size_t)dv + j0;
    for (int e = tid; e < DK * DVT; e += NT) {
        const int i = e / DVT, j = e % DVT;
        sDh[i * LDV + j] = p.dhT ? p.dhT[state_base + (size_t)i * dv + j] : 0.f;
    }
    const TIn* dout = static_cast<const TIn*>(p.dout);
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    for (int ci = nc - 1; ci >= 0; --ci) {
        const int Lc = min(kChunk, eos - bos - ci * kChunk);
        const size_t tok0 = (size_t)(start + (long long)ci * kChunk);
        const long long slot = wy_slot(n, start, ci);
        __syncthreads();  // the previous chunk is done with every buffer
        const float* tp = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk;
        for (int e = tid; e < kChunk * kChunk; e += NT) {
            sT[(e / kChunk) * LDT + e % kChunk] = tp[e];
            sP[(e / kChunk) * LDT + e % kChunk] = tp[kChunk * kChunk + e];
        }
        bw2_scaled_rows<TIn, DK>(p, tok0, h, Lc, sQF, sEF, sKf, sLam, LDK);
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            sDo[r * LDV + j] = r < Lc ? to_f32(dout[((tok0 + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        // dh' of this chunk (its end state's cotangent) for the gradient kernel
        float* dh_out = p.dh_chunks + ((size_t)slot * H + h) * DK * (size_t)dv + j0;
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            dh_out[(size_t)i * dv + j] = sDh[i * LDV + j];
        }
        __syncthreads();
        // dU = scale P^T dO + (K . f) dh'
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int s = e / DVT, j = e % DVT;
            float acc = 0.f;
            for (int r = s; r < kChunk; ++r) acc = fmaf(sP[r * LDT + s], sDo[r * LDV + j], acc);
            float kd = 0.f;
            for (int i = 0; i < DK; ++i) kd = fmaf(sKf[s * LDK + i], sDh[i * LDV + j], kd);
            sDu[s * LDV + j] = p.scale * acc + kd;
        }
        __syncthreads();
        // dX = T^T dU
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int s = e / DVT, j = e % DVT;
            float acc = 0.f;
            for (int r = s; r < kChunk; ++r) acc = fmaf(sT[r * LDT + s], sDu[r * LDV + j], acc);
            sDx[s * LDV + j] = acc;
        }
        __syncthreads();
        // dh = scale (Q . F)^T dO + Diag(Lambda) dh' - (E . F)^T dX
        float nd[DK * DVT / NT];
#pragma unroll
        for (int m = 0; m < DK * DVT / NT; ++m) {
            const int e = tid + m * NT, i = e / DVT, j = e % DVT;
            float a = 0.f;
            for (int r = 0; r < kChunk; ++r) {
                a = fmaf(p.scale * sQF[r * LDK + i], sDo[r * LDV + j], a);
                a = fmaf(-sEF[r * LDK + i], sDx[r * LDV + j], a);
            }
            nd[m] = a + sLam[i] * sDh[i * LDV + j];
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < DK * DVT / NT; ++m) {
            const int e = tid + m * NT;
            sDh[(e / DVT) * LDV + e % DVT] = nd[m];
        }
    }
    __syncthreads();
    if (p.dh0)
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            p.dh0[state_base + (size_t)i * dv + j] = sDh[i * LDV + j];
        }
}

template <int DK>
struct Bw2ChunkSmem {  // 4-byte words
    static constexpr int LDK = DK + 1, LDT = kChunk + 1, DVT = 16, LDV = DVT + 1;
    // T and dT adjacent: after dA is formed they hold dGn [64][LDK]
    static constexpr int oT = 0, odT = oT + kChunk * LDT, oP = odT + kChunk * LDT, odP = oP + kChunk * LDT;
    static constexpr int odA = odP + kChunk * LDT;
    static constexpr int oLam = odA + kChunk * LDT, odLam = oLam + DK;
    static constexpr int odB = odLam + DK;  // KDA: dbeta per row
    static constexpr int oR = odB + kChunk;
    // region R, gradient phase: EF, Kf [64][LDK]; h, dh' [DK][LDV]; V, W (write gate), dO, X, U, dU, dX [64][LDV]
    static constexpr int rEF = oR, rKf = rEF + kChunk * LDK, rH = rKf + kChunk * LDK, rDH = rH + DK * LDV;
    static constexpr int rV = rDH + DK * LDV, rW = rV + kChunk * LDV, rDO = rW + kChunk * LDV;
    static constexpr int rX = rDO + kChunk * LDV, rU = rX + kChunk * LDV, rDU = rU + kChunk * LDV;
    static constexpr int rDX = rDU + kChunk * LDV, rEnd1 = rDX + kChunk * LDV;
    static constexpr int rM = rH;  // dT T^T scratch [64][LDT] once the tiles are done
    // region R, gate phase: K, Q, E and the per-token decays a = exp(g) [64][LDK]
    static constexpr int rK = oR, rQ = rK + kChunk * LDK, rE = rQ + kChunk * LDK, rA = rE + kChunk * LDK;
    static constexpr int rEnd2 = rA + kChunk * LDK;
    static constexpr int total = rEnd1 > rEnd2 ? rEnd1 : rEnd2;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
    static_assert(kChunk * LDK <= 2 * kChunk * LDT, "dGn fits over T and dT");
    static_assert(rM + kChunk * LDT <= rEnd1, "the dT T^T scratch fits over the tiles");
};

// (4) One CTA per (chunk slot, head): every input gradient of the chunk.
template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads, 1) gdn2_bwd_chunk_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2ChunkSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, NT = kBw2Threads;
    constexpr int ACC = DK / 4;            // key channels per thread in the register sums (row tid / 4)
    constexpr int TPC = NT / DK;           // threads per channel in the Lambda sums
    extern __shared__ __align__(16) float bsm[];
    float* sT = bsm + L::oT;
    float* sdT = bsm + L::odT;
    float* sP = bsm + L::oP;
    float* sdP = bsm + L::odP;
    float* sdA = bsm + L::odA;
    float* sLam = bsm + L::oLam;
    float* sdLam = bsm + L::odLam;
    float* sdB = bsm + L::odB;
    float* sEF = bsm + L::rEF;
    float* sKf = bsm + L::rKf;
    float* sH = bsm + L::rH;
    float* sDH = bsm + L::rDH;
    float* sV = bsm + L::rV;
    float* sW = bsm + L::rW;
    float* sDO = bsm + L::rDO;
    float* sX = bsm + L::rX;
    float* sU = bsm + L::rU;
    float* sDU = bsm + L::rDU;
    float* sDX = bsm + L::rDX;
    __shared__ int info[2];
    const int tid = threadIdx.x, H = p.H, dv = p.vdim;
    const long long slot = blockIdx.x / H;
    const int h = blockIdx.x % H;
    bw2_slot_chunk(p, slot, info, err);
    const int Lc = info[1];
    if (Lc == 0) return;
    const size_t tok0 = (size_t)info[0];
    const TIn* vin = static_cast<const TIn*>(p.v);
    const TIn* dout = static_cast<const TIn*>(p.dout);
    const float* hc = p.h_chunks + ((size_t)slot * H + h) * DK * (size_t)dv;
    const float* dhc = p.dh_chunks + ((size_t)slot * H + h) * DK * (size_t)dv;
    const float* tp = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk;

    for (int e = tid; e < kChunk * kChunk; e += NT) {
        const int r = e / kChunk, s = e % kChunk;
        sT[r * LDT + s] = tp[e];
        sP[r * LDT + s] = tp[kChunk * kChunk + e];
        sdT[r * LDT + s] = 0.f;
        sdP[r * LDT + s] = 0.f;
    }
    if (tid < kChunk) sdB[tid] = 0.f;
    bw2_scaled_rows<TIn, DK>(p, tok0, h, Lc, nullptr, sEF, sKf, sLam, LDK);

    const int ar = tid >> 2, ai = tid & 3;  // register sums: row ar, channels ai + 4 m
    float aQ[ACC], aE[ACC], aK[ACC];        // (dO h^T), (dX h^T), (U dh'^T) of row ar
#pragma unroll
    for (int m = 0; m < ACC; ++m) aQ[m] = aE[m] = aK[m] = 0.f;
    const int lc = tid / TPC, lpart = tid % TPC;  // Lambda sums: channel lc, value columns lpart + TPC * x
    float dlam = 0.f;

    for (int j0 = 0; j0 < dv; j0 += DVT) {
        __syncthreads();  // the previous tile is done (and, the first time, the scaled rows are in place)
        for (int e = tid; e < DK * DVT; e += NT) {
            const int i = e / DVT, j = e % DVT;
            sH[i * LDV + j] = hc[(size_t)i * dv + j0 + j];
            sDH[i * LDV + j] = dhc[(size_t)i * dv + j0 + j];
        }
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            const bool ok = r < Lc;
            const size_t tok = tok0 + r, idx = (tok * H + h) * dv + j0 + j;
            sV[r * LDV + j] = ok ? to_f32(vin[idx]) : 0.f;
            sW[r * LDV + j] = ok ? bw2_w(p, tok, h, j0 + j) : 0.f;
            sDO[r * LDV + j] = ok ? to_f32(dout[idx]) : 0.f;
        }
        __syncthreads();
        // X = w . V - (E . F) h ; (K . f) dh' (into dU for now).  Each thread forms a 2 x 2 block (rows ra, ra + 32;
        // columns jb, jb + 8), so every shared-memory operand it loads feeds two products.
        static_assert(kChunk * DVT == 4 * NT && DVT == 16, "2 x 2 blocks cover the tile");
        {
            const int ra = tid >> 3, jb = tid & 7;
            float eh[2][2] = {}, kd[2][2] = {};
#pragma unroll 4
            for (int i = 0; i < DK; ++i) {
                const float h0 = sH[i * LDV + jb], h1 = sH[i * LDV + jb + 8];
                const float d0 = sDH[i * LDV + jb], d1 = sDH[i * LDV + jb + 8];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    const float ev = sEF[(ra + 32 * a) * LDK + i], kv = sKf[(ra + 32 * a) * LDK + i];
                    eh[a][0] = fmaf(ev, h0, eh[a][0]);
                    eh[a][1] = fmaf(ev, h1, eh[a][1]);
                    kd[a][0] = fmaf(kv, d0, kd[a][0]);
                    kd[a][1] = fmaf(kv, d1, kd[a][1]);
                }
            }
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int r = ra + 32 * a, j = jb + 8 * b;
                    sX[r * LDV + j] = sW[r * LDV + j] * sV[r * LDV + j] - eh[a][b];
                    sDU[r * LDV + j] = kd[a][b];
                }
        }
        __syncthreads();
        // U = T X ; dU = scale P^T dO + (K . f) dh'
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int r = e / DVT, j = e % DVT;
            float u = 0.f, du = 0.f;
            for (int s = 0; s <= r; ++s) u = fmaf(sT[r * LDT + s], sX[s * LDV + j], u);
            for (int t = r; t < kChunk; ++t) du = fmaf(sP[t * LDT + r], sDO[t * LDV + j], du);
            sU[r * LDV + j] = u;
            sDU[r * LDV + j] = fmaf(p.scale, du, sDU[r * LDV + j]);
        }
        __syncthreads();
        // dX = T^T dU ; dv = w . dX ; dw = V . dX (KDA: summed into dbeta)
        for (int e = tid; e < kChunk * DVT; e += NT) {
            const int s = e / DVT, j = e % DVT;
            float acc = 0.f;
            for (int r = s; r < kChunk; ++r) acc = fmaf(sT[r * LDT + s], sDU[r * LDV + j], acc);
            sDX[s * LDV + j] = acc;
            if (s < Lc) {
                const size_t idx = ((tok0 + s) * H + h) * dv + j0 + j;
                p.dv[idx] = sW[s * LDV + j] * acc;
                if (!p.kda) p.dw[idx] = sV[s * LDV + j] * acc;
            }
        }
        __syncthreads();
        // dT += dU X^T, dP += scale dO U^T (lower parts)
        for (int e = tid; e < kChunk * kChunk; e += NT) {
            const int r = e / kChunk, s = e % kChunk;
            if (s > r) continue;
            float t = 0.f, pp = 0.f;
#pragma unroll
            for (int j = 0; j < DVT; ++j) {
                t = fmaf(sDU[r * LDV + j], sX[s * LDV + j], t);
                pp = fmaf(sDO[r * LDV + j], sU[s * LDV + j], pp);
            }
            sdT[r * LDT + s] += t;
            sdP[r * LDT + s] += p.scale * pp;
        }
        if (p.kda && tid < kChunk) {  // the write gate's share of dbeta
            float a = 0.f;
#pragma unroll
            for (int j = 0; j < DVT; ++j) a = fmaf(sV[tid * LDV + j], sDX[tid * LDV + j], a);
            sdB[tid] += a;
        }
        // sum_j h_ij dh'_ij
#pragma unroll
        for (int x = 0; x < DVT / TPC; ++x) {
            const int j = lpart + TPC * x;
            dlam = fmaf(sH[lc * LDV + j], sDH[lc * LDV + j], dlam);
        }
        // register sums of row ar: dO h^T, dX h^T, U dh'^T
#pragma unroll
        for (int m = 0; m < ACC; ++m) {
            const int i = ai + 4 * m;
            float q1 = 0.f, e1 = 0.f, k1 = 0.f;
#pragma unroll
            for (int j = 0; j < DVT; ++j) {
                const float hv = sH[i * LDV + j];
                q1 = fmaf(sDO[ar * LDV + j], hv, q1);
                e1 = fmaf(sDX[ar * LDV + j], hv, e1);
                k1 = fmaf(sU[ar * LDV + j], sDH[i * LDV + j], k1);
            }
            aQ[m] += q1;
            aE[m] += e1;
            aK[m] += k1;
        }
    }
#pragma unroll
    for (int o = 1; o < TPC; o <<= 1) dlam += __shfl_xor_sync(0xffffffffu, dlam, o);
    if (lpart == 0) sdLam[lc] = dlam;
    __syncthreads();
    // dA = -T^T dT T^T on the strictly lower part (dT's diagonal and upper part do not reach A)
    float* sM = bsm + L::rM;
    for (int e = tid; e < kChunk * kChunk; e += NT) {  // M = dT T^T, dT strictly lower
        const int r = e / kChunk, s = e % kChunk;
        float m = 0.f;
        const int tmax = min(r - 1, s);
        for (int t = 0; t <= tmax; ++t) m = fmaf(sdT[r * LDT + t], sT[s * LDT + t], m);
        sM[r * LDT + s] = m;
    }
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += NT) {
        const int r = e / kChunk, s = e % kChunk;
        float a = 0.f;
        if (s < r)
            for (int t = r; t < kChunk; ++t) a = fmaf(sT[t * LDT + r], sM[t * LDT + s], a);
        sdA[r * LDT + s] = -a;
    }
    __syncthreads();
    // gate phase: the raw K, Q, E and the per-token decays a = exp(g) over the region
    float* sK = bsm + L::rK;
    float* sQ = bsm + L::rQ;
    float* sE = bsm + L::rE;
    float* sAd = bsm + L::rA;
    {
        const TIn* q = static_cast<const TIn*>(p.q);
        const TIn* k = static_cast<const TIn*>(p.k);
        for (int e = tid; e < kChunk * DK; e += NT) {
            const int r = e / DK, i = e % DK;
            float kv = 0.f, qv = 0.f, bv = 0.f, gv = 0.f;
            if (r < Lc) {
                const size_t idx = ((tok0 + r) * H + h) * DK + i;
                kv = to_f32(k[idx]);
                qv = to_f32(q[idx]);
                bv = bw2_b(p, tok0 + r, h, i);
                gv = p.g[idx];
            }
            sK[r * LDK + i] = kv;
            sQ[r * LDK + i] = qv;
            sE[r * LDK + i] = bv * kv;
            sAd[r * LDK + i] = expf(gv);
        }
    }
    __syncthreads();
    // through A and P, then the complete dQ, dE, dK of row ar.  D_rsi = a_(s+1)i ... a_ri is a running product
    // along the row (columns s from ar down) or the column (rows r from ar up); the finished products are
    // F = 2^(G_ar) and f = 2^(G_L - G_ar) of the row.  Two pairs of terms cancel exactly in dGn and are left out
    // of it (not of dq and dk): P's diagonal (q_r . k_r, no decay) and, on row L, the row's own share of the
    // G_L terms.
    float* sDG = sT;  // dGn [64][LDK] over T and dT (both done)
    float* sLr = sQ;  // the G_L terms of every row [64][LDK], once Q is no longer read
    float dGn[ACC], lt[ACC];
    float kdb = 0.f;  // KDA: this thread's share of sum_i k_ri dE_ri
#pragma unroll
    for (int m = 0; m < ACC; ++m) {
        const int i = ai + 4 * m;
        const float kv = sK[ar * LDK + i], qv = sQ[ar * LDK + i], ev = sE[ar * LDK + i];
        float dEa = 0.f, dQp = 0.f, dKap = 0.f, F = sAd[ar * LDK + i], f = 1.f;
        for (int s = ar - 1; s >= 0; --s) {
            const float ks = sK[s * LDK + i] * F;
            dEa = fmaf(sdA[ar * LDT + s], ks, dEa);
            dQp = fmaf(sdP[ar * LDT + s], ks, dQp);
            F *= sAd[s * LDK + i];
        }
        for (int r = ar + 1; r < kChunk; ++r) {
            f *= sAd[r * LDK + i];
            dKap = fmaf(fmaf(sdA[r * LDT + ar], sE[r * LDK + i], sdP[r * LDT + ar] * sQ[r * LDK + i]), f, dKap);
        }
        const float pd = sdP[ar * LDT + ar];
        const float dQo = fmaf(p.scale * F, aQ[m], dQp);  // without P's diagonal
        const float dE = fmaf(-F, aE[m], dEa);
        const float kf = f * aK[m];
        const bool last = ar == kChunk - 1;
        const float dKo = (last ? 0.f : kf) + dKap;  // without P's diagonal (and, on row L, without its G_L share)
        dGn[m] = (float)((double)qv * dQo + (double)ev * dE - (double)kv * dKo);
        lt[m] = last ? 0.f : kv * kf;
        if (ar < Lc) {
            const size_t tok = tok0 + ar, idx = (tok * H + h) * DK + i;
            const float bv = bw2_b(p, tok, h, i);
            const float dK = kf + dKap + pd * qv;
            p.dq[idx] = fmaf(pd, kv, dQo);
            p.dk[idx] = fmaf(bv, dE, dK);
            if (p.kda) kdb = fmaf(kv, dE, kdb);
            else p.db[idx] = kv * dE;
        }
    }
    kdb += __shfl_xor_sync(0xffffffffu, kdb, 1);  // the four threads of row ar are adjacent lanes
    kdb += __shfl_xor_sync(0xffffffffu, kdb, 2);
    __syncthreads();  // every thread is done reading T, dT and Q
#pragma unroll
    for (int m = 0; m < ACC; ++m) {
        sDG[ar * LDK + ai + 4 * m] = dGn[m];
        sLr[ar * LDK + ai + 4 * m] = lt[m];
    }
    if (p.kda && ai == 0) sdB[ar] += kdb;
    __syncthreads();
    // dg: reverse cumulative sum of dGn along the rows, with the terms of G_L on row 63
    for (int i = tid; i < DK; i += NT) {
        double acc = (double)sLam[i] * sdLam[i];
        for (int r = 0; r < kChunk; ++r) acc += sLr[r * LDK + i];
        for (int r = kChunk - 1; r >= 0; --r) {
            acc += sDG[r * LDK + i];
            if (r < Lc) p.dg[((tok0 + r) * H + h) * DK + i] = (float)acc;
        }
    }
    if (p.kda && tid < Lc) p.db[(tok0 + tid) * H + h] = sdB[tid];
}

}  // namespace gdn
