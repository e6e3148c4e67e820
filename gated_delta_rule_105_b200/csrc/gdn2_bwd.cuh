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

#include "gdn_bwd_tiles.cuh"
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

// (0) One CTA per (chunk slot, head): T and P of the chunk into the workspace.
template <int DK>
struct Bw2PrepSmem {  // 4-byte words; the cumulative gate is fp64, transposed [channel][row]
    static constexpr int LDK = DK + 1, LDT = kChunk + 1;
    static constexpr int oGd = 0;  // double [DK][64]
    static constexpr int oK = oGd + 2 * DK * kChunk, oQ = oK + kChunk * LDK, oE = oQ + kChunk * LDK;
    static constexpr int oA = oE + kChunk * LDK, oT = oA + kChunk * LDT;
    static constexpr int oAd = oT + kChunk * LDT;  // per-token decays of 64 channels [row][channel], LDT apart
    static constexpr int total = oAd + kChunk * LDT;
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
    // Every load of the chunk in one round trip, as 16-byte vectors: k, q into their buffers, the erase gate into
    // E (multiplied by k below), the raw gate rows into A, T and the decay buffer (free until the A and P sweep).
    float* sGr = sA;
    static_assert(L::oA + kChunk * LDK <= L::total, "the raw gate rows fit over A, T and the decays");
    {
        RowBlock<TIn, DK> rk, rq;
        RowBlock<float, DK> rg, rb;
        const size_t base = (tok0 * H + h) * DK, rs = (size_t)H * DK;
        rk.load(k + base, rs, Lc);
        rq.load(q + base, rs, Lc);
        rg.load(p.g + base, rs, Lc);
        if (!p.kda) rb.load(p.b + base, rs, Lc);
        rk.store_scalar(sK, LDK);
        rq.store_scalar(sQ, LDK);
        rg.store_scalar(sGr, LDK);
        if (!p.kda) rb.store_scalar(sE, LDK);
        else
            for (int e = tid; e < kChunk * DK; e += NT) {  // KDA: beta of the row
                const int r = e / DK;
                sE[r * LDK + e % DK] = r < Lc ? p.b[(tok0 + r) * H + h] : 0.f;
            }
    }
    __syncthreads();
    {  // G of every row and channel: the fp64 running sum from row 0 (rows past Lc add nothing), two threads per
       // channel, the first half's total handed to the second half through shared memory; E = b . k on the way
        constexpr int RH = kChunk / 2;
        __shared__ double carry[DK];
        const int i = tid % DK, half = tid / DK, r0 = half * RH;
        double acc = 0.0;
        if (half == 0) {
#pragma unroll 8
            for (int m = 0; m < RH; ++m) {
                acc += (double)sGr[m * LDK + i];
                sGd[i * kChunk + m] = acc * kLog2eD;
            }
            carry[i] = acc;
        }
        __syncthreads();
        if (half == 1) {
            acc = carry[i];
#pragma unroll 8
            for (int m = 0; m < RH; ++m) {
                acc += (double)sGr[(r0 + m) * LDK + i];
                sGd[i * kChunk + r0 + m] = acc * kLog2eD;
            }
        }
        if (half < 2)
            for (int m = 0; m < RH; ++m) sE[(r0 + m) * LDK + i] *= sK[(r0 + m) * LDK + i];
    }
    __syncthreads();
    // A and P: thread column s = tid % 64, rows 16 rb .. 16 rb + 15 (rb = tid / 64).  Per channel the decay
    // 2^(G_r - G_s) starts at the block's first row r0 at or below s (1 when r0 = s, else exp2 of the fp64
    // difference: an fp32 G of a strongly decaying channel, hundreds in magnitude, would cost ~1e-5 of it) and is
    // carried down the block by the per-token decays a_r = 2^(G_r - G_(r-1)), shared by the warp through shared
    // memory, 64 channels at a time (at most 15 roundings more than one exp2 per entry: ~1e-6).
    float* P = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk + kChunk * kChunk;
    float* sAd = bsm + L::oAd;
    const int s = tid & (kChunk - 1), rb = tid >> 6, r0 = max(16 * rb, s);
    const bool act = r0 < 16 * rb + 16;
    float accA[16], accP[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) accA[u] = accP[u] = 0.f;
    for (int i0 = 0; i0 < DK; i0 += 64) {
        __syncthreads();  // the previous channels' decays are no longer read
        for (int e = tid; e < 64 * kChunk; e += NT) {
            const int ii = e / kChunk, r = e % kChunk;
            const double* gd = sGd + (i0 + ii) * kChunk;
            sAd[r * LDT + ii] = r == 0 ? 1.f : exp2f((float)(gd[r] - gd[r - 1]));
        }
        __syncthreads();
        if (act)
            for (int ii = 0; ii < 64; ++ii) {
                const int i = i0 + ii;
                const float ks = sK[s * LDK + i];
                float D = r0 == s ? 1.f : exp2f((float)(sGd[i * kChunk + r0] - sGd[i * kChunk + s]));
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int r = 16 * rb + u;
                    if (r > r0) D *= sAd[r * LDT + ii];
                    if (r >= r0) {
                        const float kd = ks * D;
                        accA[u] = fmaf(sE[r * LDK + i], kd, accA[u]);
                        accP[u] = fmaf(sQ[r * LDK + i], kd, accP[u]);
                    }
                }
            }
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        const int r = 16 * rb + u;
        sA[r * LDT + s] = s < r ? accA[u] : 0.f;
        P[r * kChunk + s] = accP[u];
    }
    __syncthreads();
    inv_unit_lower64(sA, sT, LDT, sK);  // K is no longer read: it holds the inverse's scratch
    float* Tg = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk;
    for (int e = tid; e < kChunk * kChunk; e += NT) Tg[e] = sT[(e / kChunk) * LDT + e % kChunk];
}

// Per-channel chunk quantities from raw rows in shared memory ([64][ldk]: g in G, q in QF, the erase gate b in EF
// or, for KDA, beta per row in bt, k in Kf; rows past the chunk's end zero), in place: QF <- q F, EF <- b k F,
// Kf <- k f, Lambda = 2^G_L (QF and Lam may be null).  Two threads per channel, one per half of the rows (threads
// past 2 * DK idle).  The cumulative sum runs along the rows in fp64 in the prep kernel's order (row 0 first, rows
// past the chunk's end adding nothing): the first half's total is handed to the second half, whose total is G_L.
// Called by every thread of the block (it synchronises twice).
template <int DK>
__device__ void bw2_scale_rows_smem(const float* G, float* QF, float* EF, float* Kf, const float* bt, float* Lam,
                                    int ldk) {
    constexpr int RH = kChunk / 2;
    __shared__ double carry[2 * DK];
    const int i = threadIdx.x % DK, half = threadIdx.x / DK, r0 = half * RH;
    double acc = 0.0;
    if (half == 0) {
#pragma unroll 8
        for (int m = 0; m < RH; ++m) acc += (double)G[(r0 + m) * ldk + i];
        carry[i] = acc;
    }
    __syncthreads();
    if (half == 1) {
        acc = carry[i];
#pragma unroll 8
        for (int m = 0; m < RH; ++m) acc += (double)G[(r0 + m) * ldk + i];
        carry[DK + i] = acc;
    }
    __syncthreads();
    if (half >= 2) return;
    const double gl = carry[DK + i] * kLog2eD;
    if (Lam && half == 0) Lam[i] = exp2f((float)gl);
    acc = half == 0 ? 0.0 : carry[i];
#pragma unroll 4
    for (int m = 0; m < RH; ++m) {
        const int e = (r0 + m) * ldk + i;
        acc += (double)G[e];
        const double Gd = acc * kLog2eD;
        const float F = exp2f((float)Gd), f = exp2f((float)(gl - Gd));
        const float kv = Kf[e];
        if (QF) QF[e] *= F;
        EF[e] = (bt ? bt[r0 + m] : EF[e]) * kv * F;
        Kf[e] = kv * f;
    }
}

// (1) One CTA per (sequence, head, 32 value columns): the state at every chunk start, walked forward with T from
// the prep kernel (the forward's recurrence without its output): X = Z - (E . F) h, U = T X,
// h' = Diag(Lambda) h + (K . f)^T U, each as register tiles (gdn_bwd_tiles.cuh).  The value columns of the state
// never mix, so the slices are exact.
template <int DK>
struct Bw2StSmem {  // 4-byte words; row strides padded to 16 bytes
    static constexpr int LDK = DK + 4, LDT = kChunk + 4, DVT = kTileDv, LDV = kTileLdv;
    static constexpr int oT = 0, oEF = oT + kChunk * LDT, oKf = oEF + kChunk * LDK, oG = oKf + kChunk * LDK;
    static constexpr int oLam = oG + kChunk * LDK, oBt = oLam + DK;  // Lambda [DK]; KDA beta [64]
    static constexpr int oH = oBt + kChunk;      // h [DK][LDV]
    static constexpr int oZ = oH + DK * LDV;     // V [64][LDV]
    static constexpr int oX = oZ + kChunk * LDV, oU = oX + kChunk * LDV;  // X (first the write gate w) and U
    static constexpr int total = oU + kChunk * LDV;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads) gdn2_bwd_states_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2StSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, IP = DK / 32;
    static_assert(kBw2Threads == kTileThreads, "the register tiles assume 256 threads");
    extern __shared__ __align__(16) float bsm[];
    float* sT = bsm + L::oT;
    float* sEF = bsm + L::oEF;
    float* sKf = bsm + L::oKf;
    float* sG = bsm + L::oG;
    float* sLam = bsm + L::oLam;
    float* sBt = bsm + L::oBt;
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
    tile_load_state(sH, p.h0 ? p.h0 + state_base : nullptr, dv, DK);
    // the states go into the workspace this launch owns (the parameter block holds them as read-only for the
    // kernels that read them)
    float* h_chunks = const_cast<float*>(p.h_chunks);
    const TIn* vin = static_cast<const TIn*>(p.v);
    const TIn* k = static_cast<const TIn*>(p.k);
    const int s0 = tile_s0(), tj = tile_j0(), wr = tile_warp_row(), i0 = tile_i0<DK>();
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    // the next chunk's operands, loaded into registers while the current one computes
    RowBlock<float, kChunk> rt;
    RowBlock<TIn, DVT> rv;
    RowBlock<float, DVT> rw;
    RowBlock<float, DK> rg, rb;
    RowBlock<TIn, DK> rk;
    float rbt = 0.f;
    auto fetch = [&](int ci) {
        const int Lc = min(kChunk, eos - bos - ci * kChunk);
        const size_t tok0 = (size_t)(start + (long long)ci * kChunk), rs = (size_t)H * DK;
        rt.load(p.tp + ((size_t)wy_slot(n, start, ci) * H + h) * 2 * kChunk * kChunk, kChunk, kChunk);
        rv.load(vin + (tok0 * H + h) * dv + j0, (size_t)H * dv, Lc);
        rg.load(p.g + (tok0 * H + h) * DK, rs, Lc);
        rk.load(k + (tok0 * H + h) * DK, rs, Lc);
        if (p.kda) {
            if (tid < kChunk) rbt = tid < Lc ? p.b[(tok0 + tid) * H + h] : 0.f;
        } else {
            rw.load(p.w + (tok0 * H + h) * dv + j0, (size_t)H * dv, Lc);
            rb.load(p.b + (tok0 * H + h) * DK, rs, Lc);
        }
    };
    if (nc > 0) fetch(0);
    for (int ci = 0; ci < nc; ++ci) {
        const long long slot = wy_slot(n, start, ci);
        __syncthreads();  // the previous chunk is done with every buffer
        tile_store_state(h_chunks + ((size_t)slot * H + h) * DK * (size_t)dv + j0, dv, sH, DK);
        rt.store(sT, LDT);
        rv.store(sZ, LDV);
        rg.store(sG, LDK);
        rk.store(sKf, LDK);
        if (p.kda) {
            if (tid < kChunk) sBt[tid] = rbt;
        } else {
            rw.store(sX, LDV);
            rb.store(sEF, LDK);
        }
        __syncthreads();
        if (ci + 1 < nc) fetch(ci + 1);
        bw2_scale_rows_smem<DK>(sG, nullptr, sEF, sKf, p.kda ? sBt : nullptr, sLam, LDK);
        __syncthreads();
        {  // X = w . V - (E . F) h (KDA: w = beta of the row); sX holds w until the thread's own tile is read
            float a[2][4] = {};
            tile_acc_AD_split<DK, LDK>(sEF, sH, a);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int s = s0 + u;
                const float4 v = lds4(sZ + s * LDV + tj);
                const float4 w = p.kda ? make_float4(sBt[s], sBt[s], sBt[s], sBt[s]) : lds4(sX + s * LDV + tj);
                sts4(sX + s * LDV + tj, w.x * v.x - a[u][0], w.y * v.y - a[u][1], w.z * v.z - a[u][2],
                     w.w * v.w - a[u][3]);
            }
        }
        __syncthreads();
        {  // U = T X (T lower triangular: the warp's rows reach column 8w + 7 at most)
            float a[2][4] = {};
            tile_acc_AD<LDT>(sT, sX, wr + 8, a);
#pragma unroll
            for (int u = 0; u < 2; ++u) sts4(sU + (s0 + u) * LDV + tj, a[u][0], a[u][1], a[u][2], a[u][3]);
        }
        __syncthreads();
        {  // h' = Diag(Lambda) h + (K . f)^T U on the thread's own rows and columns of h
            float a[IP][4];
#pragma unroll
            for (int u = 0; u < IP; ++u) {
                const float lam = sLam[i0 + u];
                const float4 d = lds4(sH + (i0 + u) * LDV + tj);
                a[u][0] = lam * d.x;
                a[u][1] = lam * d.y;
                a[u][2] = lam * d.z;
                a[u][3] = lam * d.w;
            }
            tile_acc_KtX_split<DK, LDK>(sKf, sU, nullptr, nullptr, a);
#pragma unroll
            for (int u = 0; u < IP; ++u) sts4(sH + (i0 + u) * LDV + tj, a[u][0], a[u][1], a[u][2], a[u][3]);
        }
    }
}

template <int DK>
struct Bw2DhSmem {  // 4-byte words; row strides padded to 16 bytes
    static constexpr int LDK = DK + 4, LDT = kChunk + 4, DVT = kTileDv, LDV = kTileLdv;
    static constexpr int oT = 0, oP = oT + kChunk * LDT, oQF = oP + kChunk * LDT, oEF = oQF + kChunk * LDK;
    static constexpr int oKf = oEF + kChunk * LDK, oG = oKf + kChunk * LDK, oLam = oG + kChunk * LDK;
    static constexpr int oBt = oLam + DK;        // KDA beta [64]
    static constexpr int oDh = oBt + kChunk;     // dh [DK][LDV]
    static constexpr int oDo = oDh + DK * LDV;   // dO [64][LDV], then scale dO
    static constexpr int oDu = oDo + kChunk * LDV, oDx = oDu + kChunk * LDV;  // dU; -dX
    static constexpr int total = oDx + kChunk * LDV;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// (3) One CTA per (sequence, head, 32 value columns): the state cotangent, walked from the last chunk to the first.
// Per chunk: dU = scale P^T dO + (K . f) dh', dX = T^T dU, dh = (Q . F)^T (scale dO) + (E . F)^T (-dX)
// + Diag(Lambda) dh', each as register tiles.
template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads) gdn2_bwd_dh_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2DhSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, IP = DK / 32;
    static_assert(kBw2Threads == kTileThreads, "the register tiles assume 256 threads");
    extern __shared__ __align__(16) float bsm[];
    float* sT = bsm + L::oT;
    float* sP = bsm + L::oP;
    float* sQF = bsm + L::oQF;
    float* sEF = bsm + L::oEF;
    float* sKf = bsm + L::oKf;
    float* sG = bsm + L::oG;
    float* sLam = bsm + L::oLam;
    float* sBt = bsm + L::oBt;
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
    tile_load_state(sDh, p.dhT ? p.dhT + state_base : nullptr, dv, DK);
    const TIn* q = static_cast<const TIn*>(p.q);
    const TIn* k = static_cast<const TIn*>(p.k);
    const TIn* dout = static_cast<const TIn*>(p.dout);
    const int s0 = tile_s0(), tj = tile_j0(), wr = tile_warp_row(), i0 = tile_i0<DK>();
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    // the next chunk's operands, loaded into registers while the current one computes
    RowBlock<float, kChunk> rt, rp;
    RowBlock<TIn, DVT> rdo;
    RowBlock<float, DK> rg, rb;
    RowBlock<TIn, DK> rk, rq;
    float rbt = 0.f;
    auto fetch = [&](int ci) {
        const int Lc = min(kChunk, eos - bos - ci * kChunk);
        const size_t tok0 = (size_t)(start + (long long)ci * kChunk), rs = (size_t)H * DK;
        const float* tp = p.tp + ((size_t)wy_slot(n, start, ci) * H + h) * 2 * kChunk * kChunk;
        rt.load(tp, kChunk, kChunk);
        rp.load(tp + kChunk * kChunk, kChunk, kChunk);
        rdo.load(dout + (tok0 * H + h) * dv + j0, (size_t)H * dv, Lc);
        rg.load(p.g + (tok0 * H + h) * DK, rs, Lc);
        rk.load(k + (tok0 * H + h) * DK, rs, Lc);
        rq.load(q + (tok0 * H + h) * DK, rs, Lc);
        if (p.kda) {
            if (tid < kChunk) rbt = tid < Lc ? p.b[(tok0 + tid) * H + h] : 0.f;
        } else {
            rb.load(p.b + (tok0 * H + h) * DK, rs, Lc);
        }
    };
    if (nc > 0) fetch(nc - 1);
    for (int ci = nc - 1; ci >= 0; --ci) {
        const long long slot = wy_slot(n, start, ci);
        __syncthreads();  // the previous chunk is done with every buffer
        rt.store(sT, LDT);
        rp.store(sP, LDT);
        rdo.store(sDo, LDV);
        rg.store(sG, LDK);
        rk.store(sKf, LDK);
        rq.store(sQF, LDK);
        if (p.kda) {
            if (tid < kChunk) sBt[tid] = rbt;
        } else {
            rb.store(sEF, LDK);
        }
        // dh' of this chunk (its end state's cotangent) for the gradient kernel
        tile_store_state(p.dh_chunks + ((size_t)slot * H + h) * DK * (size_t)dv + j0, dv, sDh, DK);
        __syncthreads();
        if (ci > 0) fetch(ci - 1);
        bw2_scale_rows_smem<DK>(sG, sQF, sEF, sKf, p.kda ? sBt : nullptr, sLam, LDK);
        __syncthreads();
        {  // dU = scale P^T dO + (K . f) dh'
            float a[2][4] = {};
            tile_acc_AtX<LDT>(sP, sDo, wr, a);
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int c = 0; c < 4; ++c) a[u][c] *= p.scale;
            tile_acc_AD_split<DK, LDK>(sKf, sDh, a);
#pragma unroll
            for (int u = 0; u < 2; ++u) sts4(sDu + (s0 + u) * LDV + tj, a[u][0], a[u][1], a[u][2], a[u][3]);
        }
        __syncthreads();
        {  // dX = T^T dU, kept as -dX; the thread's own tile of dO becomes scale dO
            float x[2][4] = {};
            tile_acc_AtX<LDT>(sT, sDu, wr, x);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int s = s0 + u;
                sts4(sDx + s * LDV + tj, -x[u][0], -x[u][1], -x[u][2], -x[u][3]);
                const float4 d = lds4(sDo + s * LDV + tj);
                sts4(sDo + s * LDV + tj, p.scale * d.x, p.scale * d.y, p.scale * d.z, p.scale * d.w);
            }
        }
        __syncthreads();
        {  // dh = (Q . F)^T (scale dO) + (E . F)^T (-dX) + Diag(Lambda) dh' on the thread's own tile of dh
            float a[IP][4];
#pragma unroll
            for (int u = 0; u < IP; ++u) {
                const float lam = sLam[i0 + u];
                const float4 d = lds4(sDh + (i0 + u) * LDV + tj);
                a[u][0] = lam * d.x;
                a[u][1] = lam * d.y;
                a[u][2] = lam * d.z;
                a[u][3] = lam * d.w;
            }
            tile_acc_KtX_split<DK, LDK>(sQF, sDo, sEF, sDx, a);
#pragma unroll
            for (int u = 0; u < IP; ++u) sts4(sDh + (i0 + u) * LDV + tj, a[u][0], a[u][1], a[u][2], a[u][3]);
        }
    }
    __syncthreads();
    if (p.dh0) tile_store_state(p.dh0 + state_base, dv, sDh, DK);
}

template <int DK>
struct Bw2ChunkSmem {  // 4-byte words
    static constexpr int LDK = DK + 1, LDT = kChunk + 1, DVT = 16, LDV = DVT + 4;  // value tiles: 16-byte rows
    // T and dT adjacent: after dA is formed they hold dGn [64][LDK]
    static constexpr int oT = 0, odT = oT + kChunk * LDT, oP = odT + kChunk * LDT, odP = oP + kChunk * LDT;
    static constexpr int odA = odP + kChunk * LDT;
    static constexpr int oLam = odA + kChunk * LDT, odLam = oLam + DK;
    static constexpr int odB = odLam + DK;  // KDA: dbeta per row
    static constexpr int oR = odB + kChunk;
    // region R, gradient phase: EF, Kf [64][LDK]; h, dh' [DK][LDV]; dO, X, U, dU, dX [64][LDV]
    static constexpr int rEF = oR, rKf = rEF + kChunk * LDK, rH = rKf + kChunk * LDK, rDH = rH + DK * LDV;
    static constexpr int rDO = rDH + DK * LDV;
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
    static_assert(rH % 4 == 0 && rDO % 4 == 0, "16-byte aligned value tiles");
};

// (4) One CTA per (chunk slot, head): every input gradient of the chunk.
template <typename TIn, int DK>
__global__ void __launch_bounds__(kBw2Threads, 1) gdn2_bwd_chunk_kernel(const Bwd2Params p, unsigned* err) {
    using L = Bw2ChunkSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, NT = kBw2Threads;
    constexpr int CM = DK / 32;            // key channels per thread in the register sums (8 rows each)
    constexpr int QA = kChunk / (NT / 32); // rows per thread in the register sums
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

#pragma unroll 8
    for (int m = 0; m < kChunk * kChunk / NT; ++m) {
        const int e = tid + m * NT, r = e / kChunk, s = e % kChunk;
        sT[r * LDT + s] = tp[e];
        sP[r * LDT + s] = tp[kChunk * kChunk + e];
        sdT[r * LDT + s] = 0.f;
        sdP[r * LDT + s] = 0.f;
    }
    if (tid < kChunk) sdB[tid] = 0.f;
    {  // the raw rows of g, the erase gate (KDA: beta per row) and k, then E . F, K . f and Lambda in place
        float* sG = bsm + L::rH;  // the value tiles are free until the first tile
        float* sBt = sG + kChunk * LDK;
        static_assert(L::rH + kChunk * LDK + kChunk <= L::rEnd1, "raw gate rows fit over the value tiles");
        const TIn* k = static_cast<const TIn*>(p.k);
        constexpr int PER = kChunk * DK / NT, BATCH = 8;
        for (int m0 = 0; m0 < PER; m0 += BATCH) {
            float gv[BATCH], bv[BATCH], kv[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int e = tid + (m0 + u) * NT, r = e / DK, i = e % DK;
                gv[u] = bv[u] = kv[u] = 0.f;
                if (r < Lc) {
                    const size_t idx = ((tok0 + r) * H + h) * DK + i;
                    gv[u] = p.g[idx];
                    if (!p.kda) bv[u] = p.b[idx];
                    kv[u] = to_f32(k[idx]);
                }
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int e = tid + (m0 + u) * NT, r = e / DK, i = e % DK;
                sG[r * LDK + i] = gv[u];
                sEF[r * LDK + i] = bv[u];
                sKf[r * LDK + i] = kv[u];
            }
        }
        if (p.kda && tid < kChunk) sBt[tid] = tid < Lc ? p.b[(tok0 + tid) * H + h] : 0.f;
        __syncthreads();
        bw2_scale_rows_smem<DK>(sG, nullptr, sEF, sKf, p.kda ? sBt : nullptr, sLam, LDK);
    }

    // Thread roles over a 64 x 16 value tile: row tr, columns tc .. tc + 3 (the row products; (E . F) h and
    // (K . f) dh' run as 4 x 4 blocks, rows pb .. pb + 3, the sum over the key channels split over the block's four
    // threads, channels kq + 4 t, each thread keeping row tr = pb + kq); rows qw + 8 a and channels lane + 32 m (the
    // key-side register sums, and later the gate phase: a warp's lanes share their rows); rows 4 (tid / 16) .. + 3
    // and columns tid % 16 + 16 v (the dT, dP blocks).
    const int kq = tid & 3, tc = 4 * ((tid >> 2) & 3), pb = 4 * (tid >> 4), tr = pb + kq;
    const int qw = tid >> 5, lane = tid & 31;
    const int pr = 4 * (tid >> 4), pc = tid & 15;
    constexpr int HV = DK * DVT / 4 / NT;  // float4 of each state slice per thread (channels tid / 4 + 64 m)
    static_assert(DK * DVT == 4 * NT * HV && kChunk * DVT == 4 * NT, "tile shapes");
    float aQ[QA][CM], aE[QA][CM], aK[QA][CM];  // (dO h^T), (dX h^T), (U dh'^T) of rows qw + 8 a
#pragma unroll
    for (int a = 0; a < QA; ++a)
#pragma unroll
        for (int m = 0; m < CM; ++m) aQ[a][m] = aE[a][m] = aK[a][m] = 0.f;
    float dlam[HV], rdb = 0.f;  // sum_j h dh' of this thread's channels; KDA: row tr's share of dbeta
#pragma unroll
    for (int m = 0; m < HV; ++m) dlam[m] = 0.f;

    for (int j0 = 0; j0 < dv; j0 += DVT) {
        __syncthreads();  // the previous tile is done (and, the first time, the scaled rows are in place)
        float4 vv, wv, dov;  // row tr, columns tc .. tc + 3 of V, the write gate and dO
        {  // every load of the tile first, then the stores
            float4 hv[HV], dhv[HV];
#pragma unroll
            for (int m = 0; m < HV; ++m) {
                const int e = tid + m * NT, i = e / (DVT / 4), cc = 4 * (e % (DVT / 4));
                hv[m] = __ldg(reinterpret_cast<const float4*>(hc + (size_t)i * dv + j0 + cc));
                dhv[m] = __ldg(reinterpret_cast<const float4*>(dhc + (size_t)i * dv + j0 + cc));
            }
            const bool ok = tr < Lc;
            const size_t tok = tok0 + tr, idx = (tok * H + h) * dv + j0 + tc;
            const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
            vv = ok ? ldg4(vin + idx) : z4;
            dov = ok ? ldg4(dout + idx) : z4;
            if (p.kda) {
                const float bt = ok ? p.b[tok * H + h] : 0.f;
                wv = make_float4(bt, bt, bt, bt);
            } else {
                wv = ok ? ldg4(p.w + idx) : z4;
            }
#pragma unroll
            for (int m = 0; m < HV; ++m) {
                const int e = tid + m * NT, i = e / (DVT / 4), cc = 4 * (e % (DVT / 4));
                *reinterpret_cast<float4*>(sH + i * LDV + cc) = hv[m];
                *reinterpret_cast<float4*>(sDH + i * LDV + cc) = dhv[m];
                dlam[m] = fmaf(hv[m].x, dhv[m].x, dlam[m]);
                dlam[m] = fmaf(hv[m].y, dhv[m].y, dlam[m]);
                dlam[m] = fmaf(hv[m].z, dhv[m].z, dlam[m]);
                dlam[m] = fmaf(hv[m].w, dhv[m].w, dlam[m]);
            }
            *reinterpret_cast<float4*>(sDO + tr * LDV + tc) = dov;
        }
        __syncthreads();
        // X = w . V - (E . F) h ; (K . f) dh' of row tr
        float eh[4], kd[4];
        {
            float be[4][4] = {}, bd[4][4] = {};
#pragma unroll 2
            for (int t = 0; t < DK / 4; ++t) {
                const int i = kq + 4 * t;
                const float4 hv = lds4(sH + i * LDV + tc), dhv = lds4(sDH + i * LDV + tc);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    fma4(be[u], sEF[(pb + u) * LDK + i], hv);
                    fma4(bd[u], sKf[(pb + u) * LDK + i], dhv);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int o = 1; o <= 2; o <<= 1) {
                        be[u][q] += __shfl_xor_sync(0xffffffffu, be[u][q], o);
                        bd[u][q] += __shfl_xor_sync(0xffffffffu, bd[u][q], o);
                    }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                eh[q] = kq == 0 ? be[0][q] : kq == 1 ? be[1][q] : kq == 2 ? be[2][q] : be[3][q];
                kd[q] = kq == 0 ? bd[0][q] : kq == 1 ? bd[1][q] : kq == 2 ? bd[2][q] : bd[3][q];
            }
        }
        const float vr[4] = {vv.x, vv.y, vv.z, vv.w}, wr4[4] = {wv.x, wv.y, wv.z, wv.w};
        sts4(sX + tr * LDV + tc, wr4[0] * vr[0] - eh[0], wr4[1] * vr[1] - eh[1], wr4[2] * vr[2] - eh[2],
             wr4[3] * vr[3] - eh[3]);
        __syncthreads();
        // U = T X ; dU = scale P^T dO + (K . f) dh'
        {
            float ur[4], du[4];
            blk_tri_TX<LDT, LDV>(sT, sX, pb, kq, tc, ur);
            blk_tri_TtX<LDT, LDV>(sP, sDO, pb, kq, tc, du);
            sts4(sU + tr * LDV + tc, ur[0], ur[1], ur[2], ur[3]);
            sts4(sDU + tr * LDV + tc, fmaf(p.scale, du[0], kd[0]), fmaf(p.scale, du[1], kd[1]),
                 fmaf(p.scale, du[2], kd[2]), fmaf(p.scale, du[3], kd[3]));
        }
        __syncthreads();
        // dX = T^T dU ; dv = w . dX ; dw = V . dX (KDA: summed into dbeta)
        {
            float dx[4];
            blk_tri_TtX<LDT, LDV>(sT, sDU, pb, kq, tc, dx);
            sts4(sDX + tr * LDV + tc, dx[0], dx[1], dx[2], dx[3]);
            if (tr < Lc) {
                const size_t idx = ((tok0 + tr) * H + h) * dv + j0 + tc;
                *reinterpret_cast<float4*>(p.dv + idx) =
                    make_float4(wr4[0] * dx[0], wr4[1] * dx[1], wr4[2] * dx[2], wr4[3] * dx[3]);
                if (!p.kda)
                    *reinterpret_cast<float4*>(p.dw + idx) =
                        make_float4(vr[0] * dx[0], vr[1] * dx[1], vr[2] * dx[2], vr[3] * dx[3]);
            }
            if (p.kda)
#pragma unroll
                for (int q = 0; q < 4; ++q) rdb = fmaf(vr[q], dx[q], rdb);
        }
        __syncthreads();
        {  // dT += dU X^T, dP += scale dO U^T: 4 x 4 blocks, the lower parts kept
            float bt[4][4] = {}, bp[4][4] = {};
#pragma unroll
            for (int jg = 0; jg < DVT; jg += 4) {
                float4 xa[4], ua[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    xa[v] = lds4(sX + (pc + 16 * v) * LDV + jg);
                    ua[v] = lds4(sU + (pc + 16 * v) * LDV + jg);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 dua = lds4(sDU + (pr + u) * LDV + jg), doa = lds4(sDO + (pr + u) * LDV + jg);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        bt[u][v] = fmaf(dua.x, xa[v].x, fmaf(dua.y, xa[v].y, fmaf(dua.z, xa[v].z,
                                   fmaf(dua.w, xa[v].w, bt[u][v]))));
                        bp[u][v] = fmaf(doa.x, ua[v].x, fmaf(doa.y, ua[v].y, fmaf(doa.z, ua[v].z,
                                   fmaf(doa.w, ua[v].w, bp[u][v]))));
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int r = pr + u, s2 = pc + 16 * v;
                    if (s2 <= r) {
                        sdT[r * LDT + s2] += bt[u][v];
                        sdP[r * LDT + s2] += p.scale * bp[u][v];
                    }
                }
        }
        // register sums of rows qw + 8 a: dO h^T, dX h^T, U dh'^T
#pragma unroll
        for (int jg = 0; jg < DVT; jg += 4) {
            float4 hv[CM], dhv[CM];
#pragma unroll
            for (int m = 0; m < CM; ++m) {
                hv[m] = lds4(sH + (lane + 32 * m) * LDV + jg);
                dhv[m] = lds4(sDH + (lane + 32 * m) * LDV + jg);
            }
#pragma unroll
            for (int a = 0; a < QA; ++a) {
                const int r = qw + 8 * a;
                const float4 o = lds4(sDO + r * LDV + jg), x = lds4(sDX + r * LDV + jg), u4 = lds4(sU + r * LDV + jg);
#pragma unroll
                for (int m = 0; m < CM; ++m) {
                    aQ[a][m] = fmaf(o.x, hv[m].x, fmaf(o.y, hv[m].y, fmaf(o.z, hv[m].z, fmaf(o.w, hv[m].w, aQ[a][m]))));
                    aE[a][m] = fmaf(x.x, hv[m].x, fmaf(x.y, hv[m].y, fmaf(x.z, hv[m].z, fmaf(x.w, hv[m].w, aE[a][m]))));
                    aK[a][m] = fmaf(u4.x, dhv[m].x, fmaf(u4.y, dhv[m].y, fmaf(u4.z, dhv[m].z,
                               fmaf(u4.w, dhv[m].w, aK[a][m]))));
                }
            }
        }
    }
    // the sums over the four threads that share a channel (dLambda, adjacent lanes) or a row (KDA dbeta)
#pragma unroll
    for (int m = 0; m < HV; ++m) {
        dlam[m] += __shfl_xor_sync(0xffffffffu, dlam[m], 1);
        dlam[m] += __shfl_xor_sync(0xffffffffu, dlam[m], 2);
        if ((tid & 3) == 0) sdLam[(tid + m * NT) / (DVT / 4)] = dlam[m];
    }
    rdb += __shfl_xor_sync(0xffffffffu, rdb, 4);  // the four threads of row tr: lanes 4 and 8 apart
    rdb += __shfl_xor_sync(0xffffffffu, rdb, 8);
    if (p.kda && tc == 0) sdB[tr] = rdb;
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
    {  // eight elements of each tensor in flight per thread
        const TIn* q = static_cast<const TIn*>(p.q);
        const TIn* k = static_cast<const TIn*>(p.k);
        constexpr int PER = kChunk * DK / NT, BATCH = 8;
        for (int m0 = 0; m0 < PER; m0 += BATCH) {
            float kv[BATCH], qv[BATCH], bv[BATCH], gv[BATCH];
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int e = tid + (m0 + u) * NT, r = e / DK, i = e % DK;
                kv[u] = qv[u] = bv[u] = gv[u] = 0.f;
                if (r < Lc) {
                    const size_t idx = ((tok0 + r) * H + h) * DK + i;
                    kv[u] = to_f32(k[idx]);
                    qv[u] = to_f32(q[idx]);
                    bv[u] = bw2_b(p, tok0 + r, h, i);
                    gv[u] = p.g[idx];
                }
            }
#pragma unroll
            for (int u = 0; u < BATCH; ++u) {
                const int e = tid + (m0 + u) * NT, r = e / DK, i = e % DK;
                sK[r * LDK + i] = kv[u];
                sQ[r * LDK + i] = qv[u];
                sE[r * LDK + i] = bv[u] * kv[u];
                sAd[r * LDK + i] = expf(gv[u]);
            }
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
    float lt[QA][CM];
    float kdb[QA];  // KDA: this thread's share of sum_i k_ri dE_ri of its rows
#pragma unroll
    for (int a = 0; a < QA; ++a) kdb[a] = 0.f;
#pragma unroll
    for (int m = 0; m < CM; ++m) {
        const int i = lane + 32 * m;
        // one sweep down and one up channel i's column for all the thread's rows ar = qw + 8 a, sharing the loads
        // of K, E, Q and a; each row's running product multiplies in the same order as a walk from its own row
        float Fa[QA], dEa[QA], dQp[QA], fa[QA], dKap[QA];
#pragma unroll
        for (int a = 0; a < QA; ++a) {
            Fa[a] = fa[a] = 1.f;
            dEa[a] = dQp[a] = dKap[a] = 0.f;
        }
        for (int s = kChunk - 2; s >= 0; --s) {  // Fa = a_(s+1) ... a_ar for the rows below s
            const float an = sAd[(s + 1) * LDK + i], k0 = sK[s * LDK + i];
#pragma unroll
            for (int a = 0; a < QA; ++a) {
                const int ar = qw + 8 * a;
                if (s < ar) {
                    Fa[a] *= an;
                    const float ks = k0 * Fa[a];
                    dEa[a] = fmaf(sdA[ar * LDT + s], ks, dEa[a]);
                    dQp[a] = fmaf(sdP[ar * LDT + s], ks, dQp[a]);
                }
            }
        }
        for (int r = 1; r < kChunk; ++r) {  // fa = a_(ar+1) ... a_r for the rows above r
            const float ad = sAd[r * LDK + i], er = sE[r * LDK + i], qr = sQ[r * LDK + i];
#pragma unroll
            for (int a = 0; a < QA; ++a) {
                const int ar = qw + 8 * a;
                if (r > ar) {
                    fa[a] *= ad;
                    dKap[a] = fmaf(fmaf(sdA[r * LDT + ar], er, sdP[r * LDT + ar] * qr), fa[a], dKap[a]);
                }
            }
        }
        const float a0 = sAd[i];  // a_0: F = a_ar ... a_1 a_0
#pragma unroll
        for (int a = 0; a < QA; ++a) {
            const int ar = qw + 8 * a;
            const float kv = sK[ar * LDK + i], qv = sQ[ar * LDK + i], ev = sE[ar * LDK + i];
            const float F = Fa[a] * a0, f = fa[a];
            const float pd = sdP[ar * LDT + ar];
            const float dQo = fmaf(p.scale * F, aQ[a][m], dQp[a]);  // without P's diagonal
            const float dE = fmaf(-F, aE[a][m], dEa[a]);
            const float kf = f * aK[a][m];
            const bool last = ar == kChunk - 1;
            const float dKo = (last ? 0.f : kf) + dKap[a];  // without P's diagonal (and, on row L, its G_L share)
            sDG[ar * LDK + i] = (float)((double)qv * dQo + (double)ev * dE - (double)kv * dKo);  // T, dT unread
            lt[a][m] = last ? 0.f : kv * kf;
            if (ar < Lc) {
                const size_t tok = tok0 + ar, idx = (tok * H + h) * DK + i;
                const float bv = bw2_b(p, tok, h, i);
                const float dK = kf + dKap[a] + pd * qv;
                p.dq[idx] = fmaf(pd, kv, dQo);
                p.dk[idx] = fmaf(bv, dE, dK);
                if (p.kda) kdb[a] = fmaf(kv, dE, kdb[a]);
                else p.db[idx] = kv * dE;
            }
        }
    }
#pragma unroll
    for (int a = 0; a < QA; ++a)  // a row's channels are the 32 lanes of one warp, summed in a fixed order
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) kdb[a] += __shfl_xor_sync(0xffffffffu, kdb[a], o);
    __syncthreads();  // every thread is done reading Q
#pragma unroll
    for (int a = 0; a < QA; ++a)
#pragma unroll
        for (int m = 0; m < CM; ++m) sLr[(qw + 8 * a) * LDK + lane + 32 * m] = lt[a][m];
    if (p.kda && lane == 0)
#pragma unroll
        for (int a = 0; a < QA; ++a) sdB[qw + 8 * a] += kdb[a];
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
