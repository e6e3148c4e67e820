// Backward pass (reverse mode) of the chunked gated delta rule, GDN (scalar gates): fp32 on CUDA cores.
//
// The forward per chunk of C = 64 tokens (the WY form of the SIMT forward kernel; GatedDeltaNet data-flow
// walkthrough, yfxerp.com/news/367755, section "Chunked parallelism", which also names the full backward --
// gradients of q, k, v, beta and g), with Gamma_rs = 2^(G_r - G_s), F = 2^G, f = 2^(G_last - G), gamma = 2^(G_last):
//   A = strict_lower(diag(beta) (K K^T) . Gamma),  T = (I + A)^-1,  P = lower((Q K^T) . Gamma)
//   X = diag(beta) V - diag(beta F) K h,  U = T X
//   O = scale (diag(F) Q h + P U),  h' = gamma h + (diag(f) K)^T U
// Given the cotangents dO of the output and dh' of the chunk's end state:
//   dU = scale P^T dO + diag(f) K dh'      dX = T^T dU
//   dh = scale (diag(F) Q)^T dO + gamma dh' - K^T diag(beta F) dX       (the state recurrence, chunk to chunk)
//   dT = dU X^T  ->  dA = -T^T dT T^T (strictly lower part),   dP = scale dO U^T (lower part)
// and from A, P, X, F, f, gamma to q, k, v, beta and the chunk-local cumulative gate; dg is the reverse cumulative
// sum of the gate's gradient inside the chunk.
//
// Four kernels: (1) a forward kernel (the tensor-core one for bf16 inputs, else the SIMT one) writes the state at
// every chunk start (FwdParams::h_chunks); (2) gdn_bwd_prep_kernel forms T and P of every chunk into the
// workspace; (3) gdn_bwd_dh_kernel walks each sequence's chunks backwards with the state cotangent dh in shared
// memory (one CTA per (sequence, head, 32 value columns), the value columns of dh never mix) and writes dh' of
// every chunk; (4) gdn_bwd_chunk_kernel forms every input gradient of one (chunk, head), all chunks at once,
// walking the value columns in tiles of 16 and keeping the key-side sums in registers.
#pragma once

#include "gdn_bwd_tiles.cuh"
#include "gdn_common.cuh"

namespace gdn {

constexpr int kBwThreads = 256;

struct BwdParams {
    const void* q;            // [B,T,H,dk]   (dtype TIn)
    const void* k;
    const void* v;            // [B,T,H,dv]
    const float* g;           // [B,T,H]
    const float* beta;        // [B,T,H]
    const void* dout;         // dO [B,T,H,dv] (dtype TIn)
    const float* dhT;         // [N,H,dk,dv] or null
    const float* h_chunks;    // [slot][H][dk][dv]: the state at each chunk's start (from the forward)
    float* dh_chunks;         // [slot][H][dk][dv]: the cotangent of the state at each chunk's end
    float* tp;                // [slot][H][2][64][64]: T, then P, of every chunk (from the prep kernel)
    float* dq;                // [B,T,H,dk] fp32
    float* dk;
    float* dv;                // [B,T,H,dv] fp32
    float* dg;                // [B,T,H] fp32
    float* dbeta;             // [B,T,H] fp32
    float* dh0;               // [N,H,dk,dv] fp32 or null
    const int32_t* cu_seqlens;
    float scale;
    int B, T, H, kdim, vdim, n_seq;
};

// Shared per-chunk quantities of the backward kernels (pointers into shared memory).
template <int DK>
struct BwChunk {
    static constexpr int LDK = DK + 1, LDT = kChunk + 1;
    float* K;      // [64][LDK]
    float* Q;      // [64][LDK]
    float* Gm;     // Gamma [64][LDT], 0 above the diagonal
    float* T;      // (I + A)^-1 [64][LDT]
    float* P;      // [64][LDT], 0 above the diagonal
    float* A;      // scratch [64][LDT] (A while inverting)
    double* G;     // [64] log2(e) * chunk-local cumsum of g
    float* beta;   // [64]
    float* F;      // [64] 2^G
    float* f;      // [64] 2^(G_last - G)
    float* gamma;  // [1]
};

// K and Q rows of a chunk into shared memory ([64][ldk], rows past Lc zero), eight elements of each in flight per
// thread.
template <typename TIn, int DK>
__device__ __forceinline__ void bw_load_kq(float* K, float* Q, int ldk, const TIn* k, const TIn* q, size_t tok0,
                                           int H, int h, int Lc) {
    constexpr int PER = kChunk * DK / kBwThreads, BATCH = 8;
    static_assert(PER % BATCH == 0, "batches");
    for (int m0 = 0; m0 < PER; m0 += BATCH) {
        float kv[BATCH], qv[BATCH];
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int e = threadIdx.x + (m0 + u) * kBwThreads, r = e / DK, i = e % DK;
            kv[u] = qv[u] = 0.f;
            if (r < Lc) {
                const size_t idx = ((tok0 + r) * H + h) * DK + i;
                kv[u] = to_f32(k[idx]);
                qv[u] = to_f32(q[idx]);
            }
        }
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
            const int e = threadIdx.x + (m0 + u) * kBwThreads, r = e / DK, i = e % DK;
            K[r * ldk + i] = kv[u];
            Q[r * ldk + i] = qv[u];
        }
    }
}

// Loads one chunk (rows past Lc zero: k = q = beta = g = 0), forms G, F, f, gamma and T = (I + A)^-1 in shared
// memory (A in c.A while inverting; c.Gm and c.P unused) and writes P, row stride 64, to Pg.
template <typename TIn, int DK>
__device__ void bw_chunk_prep(const BwChunk<DK>& c, const BwdParams& p, size_t tok0, int h, int Lc, float* Pg) {
    constexpr int LDK = BwChunk<DK>::LDK, LDT = BwChunk<DK>::LDT, NT = kBwThreads;
    const int tid = threadIdx.x, H = p.H;
    const TIn* q = static_cast<const TIn*>(p.q);
    const TIn* k = static_cast<const TIn*>(p.k);
    __syncthreads();  // the previous user of these buffers is done
    bw_load_kq<TIn, DK>(c.K, c.Q, LDK, k, q, tok0, H, h, Lc);
    if (tid < kChunk) {
        const bool ok = tid < Lc;
        c.beta[tid] = ok ? p.beta[(tok0 + tid) * H + h] : 0.f;
        c.G[tid] = ok ? (double)p.g[(tok0 + tid) * H + h] : 0.0;
    }
    __syncthreads();
    if (tid == 0) {
        double acc = 0.0;
        for (int r = 0; r < kChunk; ++r) {
            acc += c.G[r];
            c.G[r] = acc * kLog2eD;
        }
    }
    __syncthreads();
    if (tid < kChunk) {
        c.F[tid] = exp2f((float)c.G[tid]);
        c.f[tid] = exp2f((float)(c.G[kChunk - 1] - c.G[tid]));
        if (tid == 0) c.gamma[0] = exp2f((float)c.G[kChunk - 1]);
    }
    {  // K K^T and Q K^T as 4 x 4 blocks: rows pr .. pr + 3, columns pc + 16 v
        static_assert(NT == 256, "16 x 16 blocks of 4 x 4 entries");
        const int pr = 4 * (tid >> 4), pc = tid & 15;
        float kk[4][4] = {}, qk[4][4] = {};
#pragma unroll 2
        for (int i = 0; i < DK; ++i) {
            float ks[4], kr[4], qv[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) ks[v] = c.K[(pc + 16 * v) * LDK + i];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                kr[u] = c.K[(pr + u) * LDK + i];
                qv[u] = c.Q[(pr + u) * LDK + i];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    kk[u][v] = fmaf(kr[u], ks[v], kk[u][v]);
                    qk[u][v] = fmaf(qv[u], ks[v], qk[u][v]);
                }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int r = pr + u, s = pc + 16 * v;
                float gm = 0.f, a = 0.f, pp = 0.f;
                if (s <= r) {
                    gm = exp2f((float)(c.G[r] - c.G[s]));
                    a = s < r ? c.beta[r] * gm * kk[u][v] : 0.f;
                    pp = gm * qk[u][v];
                }
                c.A[r * LDT + s] = a;
                Pg[r * kChunk + s] = pp;
            }
    }
    __syncthreads();
    inv_unit_lower64(c.A, c.T, LDT, c.K);  // K is no longer read: it holds the inverse's scratch
}

// Loads one chunk as bw_chunk_prep does, but takes T and P from the prep kernel's output (`tp`: T then P,
// [64][64] each) instead of forming A, P and the inverse again; Gamma (0 above the diagonal) is formed only when
// `want_gm`.  The padded rows of K and Q are zero, as there.
template <typename TIn, int DK>
__device__ void bw_chunk_load(const BwChunk<DK>& c, const BwdParams& p, size_t tok0, int h, int Lc, const float* tp,
                              bool want_gm) {
    constexpr int LDK = BwChunk<DK>::LDK, LDT = BwChunk<DK>::LDT, NT = kBwThreads;
    const int tid = threadIdx.x, H = p.H;
    const TIn* q = static_cast<const TIn*>(p.q);
    const TIn* k = static_cast<const TIn*>(p.k);
    __syncthreads();  // the previous user of these buffers is done
    bw_load_kq<TIn, DK>(c.K, c.Q, LDK, k, q, tok0, H, h, Lc);
#pragma unroll 8
    for (int m = 0; m < kChunk * kChunk / NT; ++m) {
        const int e = tid + m * NT;
        c.T[(e / kChunk) * LDT + e % kChunk] = tp[e];
        c.P[(e / kChunk) * LDT + e % kChunk] = tp[kChunk * kChunk + e];
    }
    if (tid < kChunk) {
        const bool ok = tid < Lc;
        c.beta[tid] = ok ? p.beta[(tok0 + tid) * H + h] : 0.f;
        c.G[tid] = ok ? (double)p.g[(tok0 + tid) * H + h] : 0.0;
    }
    __syncthreads();
    if (tid == 0) {
        double acc = 0.0;
        for (int r = 0; r < kChunk; ++r) {
            acc += c.G[r];
            c.G[r] = acc * kLog2eD;
        }
    }
    __syncthreads();
    if (tid < kChunk) {
        c.F[tid] = exp2f((float)c.G[tid]);
        c.f[tid] = exp2f((float)(c.G[kChunk - 1] - c.G[tid]));
        if (tid == 0) c.gamma[0] = exp2f((float)c.G[kChunk - 1]);
    }
    if (want_gm)
        for (int e = tid; e < kChunk * kChunk; e += NT) {
            const int r = e / kChunk, s2 = e % kChunk;
            c.Gm[r * LDT + s2] = s2 <= r ? exp2f((float)(c.G[r] - c.G[s2])) : 0.f;
        }
    __syncthreads();
}

// Sequence bounds (row, first token, end) of sequence n; false (and the error word) for a bad cu_seqlens entry.
__device__ __forceinline__ bool bw_seq_bounds(const BwdParams& p, int n, int& row, int& bos, int& eos, unsigned* err) {
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

// The (first global token, length) of the chunk in workspace slot `slot` into info[0], info[1] (length 0 for a slot
// no chunk uses): the largest sequence n with wy_slot(n, start_n, 0) <= slot, then the chunk within it.
__device__ __forceinline__ void bw_slot_chunk(const BwdParams& p, long long slot, int* info, unsigned* err) {
    int lo = 0, hi = p.n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const long long st0 = p.cu_seqlens ? (long long)p.cu_seqlens[mid] : (long long)mid * p.T;
        if (wy_slot(mid, st0, 0) <= slot) lo = mid;
        else hi = mid - 1;
    }
    int row, bos, eos, Lc = 0;
    if (bw_seq_bounds(p, lo, row, bos, eos, err)) {
        const long long start = (long long)row * p.T + bos;
        const long long cc = slot - wy_slot(lo, start, 0);
        if (cc >= 0 && cc * kChunk < eos - bos) {
            Lc = min(kChunk, (int)(eos - bos - cc * kChunk));
            info[0] = (int)(start + cc * kChunk);
        }
    }
    info[1] = Lc;
}

template <int DK>
struct BwDhSmem {  // 4-byte words; row strides padded to 16 bytes for the register-blocked products
    static constexpr int LDK = DK + 4, LDT = kChunk + 4, DVT = kTileDv, LDV = kTileLdv;
    static constexpr int oK = 0, oQ = oK + kChunk * LDK, oT = oQ + kChunk * LDK, oP = oT + kChunk * LDT;
    static constexpr int oG = oP + kChunk * LDT;  // double [64]
    static constexpr int oBeta = oG + 2 * kChunk, oF = oBeta + kChunk, of = oF + kChunk, oGam = of + kChunk;
    static constexpr int oDh = oGam + 4;          // dh [DK][LDV]
    static constexpr int oDo = oDh + DK * LDV;    // dO [64][LDV], then scale F dO
    static constexpr int oDu = oDo + kChunk * LDV;
    static constexpr int oDx = oDu + kChunk * LDV;  // -beta F dX
    static constexpr int total = oDx + kChunk * LDV;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// Warp 0 of the block: G <- log2(e) * (chunk-local cumulative sum of g) in fp64 (G holds g on entry, 0 past the
// chunk's end), F = 2^G, f = 2^(G_63 - G), gamma = 2^G_63.  A scan over the lanes, two rows a lane.
__device__ __forceinline__ void bw_gate_scan(double* G, float* F, float* f, float* gam) {
    const int l = threadIdx.x & 31;
    const double a = G[2 * l], b = G[2 * l + 1];
    double incl = a + b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, incl, o);
        if (l >= o) incl += t;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (l == 0) excl = 0.0;
    const double g0 = (excl + a) * kLog2eD, g1 = incl * kLog2eD;
    const double gl = __shfl_sync(0xffffffffu, incl, 31) * kLog2eD;
    G[2 * l] = g0;
    G[2 * l + 1] = g1;
    F[2 * l] = exp2f((float)g0);
    F[2 * l + 1] = exp2f((float)g1);
    f[2 * l] = exp2f((float)(gl - g0));
    f[2 * l + 1] = exp2f((float)(gl - g1));
    if (l == 31) gam[0] = exp2f((float)gl);
}

// (2) One CTA per (sequence, head, 32 value columns): the state cotangent, walked from the last chunk to the first.
// Per chunk: dU = scale P^T dO + diag(f) K dh', dX = T^T dU, dh = Q^T (scale F dO) + K^T (-beta F dX) + gamma dh',
// each as register tiles (gdn_bwd_tiles.cuh).
template <typename TIn, int DK>
__global__ void __launch_bounds__(kBwThreads) gdn_bwd_dh_kernel(const BwdParams p, unsigned* err) {
    using L = BwDhSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, IP = DK / 32;
    static_assert(kBwThreads == kTileThreads, "the register tiles assume 256 threads");
    extern __shared__ __align__(16) float bsm[];
    float* sK = bsm + L::oK;
    float* sQ = bsm + L::oQ;
    float* sT = bsm + L::oT;
    float* sP = bsm + L::oP;
    double* sG = reinterpret_cast<double*>(bsm + L::oG);
    float* sBeta = bsm + L::oBeta;
    float* sF = bsm + L::oF;
    float* sf = bsm + L::of;
    float* sGam = bsm + L::oGam;
    float* sDh = bsm + L::oDh;
    float* sDo = bsm + L::oDo;
    float* sDu = bsm + L::oDu;
    float* sDx = bsm + L::oDx;
    const int tid = threadIdx.x, j0 = blockIdx.x * DVT, h = blockIdx.y, n = blockIdx.z;
    const int H = p.H, dv = p.vdim;
    int row, bos, eos;
    if (!bw_seq_bounds(p, n, row, bos, eos, err)) return;
    const long long start = (long long)row * p.T + bos;
    const size_t state_base = ((size_t)n * H + h) * DK * (size_t)dv + j0;
    tile_load_state(sDh, p.dhT ? p.dhT + state_base : nullptr, dv, DK);
    const TIn* q = static_cast<const TIn*>(p.q);
    const TIn* k = static_cast<const TIn*>(p.k);
    const TIn* dout = static_cast<const TIn*>(p.dout);
    const int s0 = tile_s0(), tj = tile_j0(), wr = tile_warp_row(), i0 = tile_i0<DK>();
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    // the next chunk's operands, loaded into registers while the current one computes
    RowBlock<TIn, DK> rk, rq;
    RowBlock<float, kChunk> rt, rp;
    RowBlock<TIn, DVT> rdo;
    float rbeta = 0.f, rg = 0.f;
    auto fetch = [&](int ci) {
        const int Lc = min(kChunk, eos - bos - ci * kChunk);
        const size_t tok0 = (size_t)(start + (long long)ci * kChunk);
        const float* tp = p.tp + ((size_t)wy_slot(n, start, ci) * H + h) * 2 * kChunk * kChunk;
        rk.load(k + (tok0 * H + h) * DK, (size_t)H * DK, Lc);
        rq.load(q + (tok0 * H + h) * DK, (size_t)H * DK, Lc);
        rt.load(tp, kChunk, kChunk);
        rp.load(tp + kChunk * kChunk, kChunk, kChunk);
        rdo.load(dout + (tok0 * H + h) * dv + j0, (size_t)H * dv, Lc);
        if (tid < kChunk) {
            const bool ok = tid < Lc;
            rbeta = ok ? p.beta[(tok0 + tid) * H + h] : 0.f;
            rg = ok ? p.g[(tok0 + tid) * H + h] : 0.f;
        }
    };
    if (nc > 0) fetch(nc - 1);
    for (int ci = nc - 1; ci >= 0; --ci) {
        const long long slot = wy_slot(n, start, ci);
        __syncthreads();  // the previous chunk is done with every buffer
        rk.store(sK, LDK);
        rq.store(sQ, LDK);
        rt.store(sT, LDT);
        rp.store(sP, LDT);
        rdo.store(sDo, LDV);
        if (tid < kChunk) {
            sBeta[tid] = rbeta;
            sG[tid] = (double)rg;
        }
        // dh' of this chunk (its end state's cotangent) for the gradient kernel
        tile_store_state(p.dh_chunks + ((size_t)slot * H + h) * DK * (size_t)dv + j0, dv, sDh, DK);
        __syncthreads();
        if (ci > 0) fetch(ci - 1);
        if (tid < 32) bw_gate_scan(sG, sF, sf, sGam);
        __syncthreads();
        {  // dU = scale P^T dO + diag(f) K dh'
            float a[2][4] = {}, b[2][4] = {};
            tile_acc_AtX<LDT>(sP, sDo, wr, a);
            tile_acc_AD_split<DK, LDK>(sK, sDh, b);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float fs = sf[s0 + u];
                sts4(sDu + (s0 + u) * LDV + tj, fmaf(p.scale, a[u][0], fs * b[u][0]),
                     fmaf(p.scale, a[u][1], fs * b[u][1]), fmaf(p.scale, a[u][2], fs * b[u][2]),
                     fmaf(p.scale, a[u][3], fs * b[u][3]));
            }
        }
        __syncthreads();
        {  // dX = T^T dU, kept as -beta F dX; the thread's own tile of dO becomes scale F dO
            float x[2][4] = {};
            tile_acc_AtX<LDT>(sT, sDu, wr, x);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int s = s0 + u;
                const float xs = -sBeta[s] * sF[s], ds = p.scale * sF[s];
                sts4(sDx + s * LDV + tj, xs * x[u][0], xs * x[u][1], xs * x[u][2], xs * x[u][3]);
                const float4 d = lds4(sDo + s * LDV + tj);
                sts4(sDo + s * LDV + tj, ds * d.x, ds * d.y, ds * d.z, ds * d.w);
            }
        }
        __syncthreads();
        {  // dh = Q^T (scale F dO) + K^T (-beta F dX) + gamma dh' on the thread's own rows and columns of dh
            const float gam = sGam[0];
            float a[IP][4];
#pragma unroll
            for (int u = 0; u < IP; ++u) {
                const float4 d = lds4(sDh + (i0 + u) * LDV + tj);
                a[u][0] = gam * d.x;
                a[u][1] = gam * d.y;
                a[u][2] = gam * d.z;
                a[u][3] = gam * d.w;
            }
            tile_acc_KtX_split<DK, LDK>(sQ, sDo, sK, sDx, a);
#pragma unroll
            for (int u = 0; u < IP; ++u) sts4(sDh + (i0 + u) * LDV + tj, a[u][0], a[u][1], a[u][2], a[u][3]);
        }
    }
    __syncthreads();
    if (p.dh0) tile_store_state(p.dh0 + state_base, dv, sDh, DK);
}

// (2) One CTA per (chunk slot, head): T = (I + A)^-1 and P of the chunk (bw_chunk_prep) into the workspace, so
// that the state-cotangent kernel (every value slice of every chunk) and the gradient kernel read them instead
// of forming them again.
template <int DK>
struct BwPrepSmem {  // 4-byte words: the bw_chunk_prep operands (~100 KB for dk = 128: two CTAs per SM)
    static constexpr int LDK = DK + 1, LDT = kChunk + 1;
    static constexpr int oK = 0, oQ = oK + kChunk * LDK, oT = oQ + kChunk * LDK, oA = oT + kChunk * LDT;
    static constexpr int oG = oA + kChunk * LDT;  // double [64]
    static constexpr int oBeta = oG + 2 * kChunk, oF = oBeta + kChunk, of = oF + kChunk, oGam = of + kChunk;
    static constexpr int total = oGam + 4;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

template <typename TIn, int DK>
__global__ void __launch_bounds__(kBwThreads) gdn_bwd_prep_kernel(const BwdParams p, unsigned* err) {
    using L = BwPrepSmem<DK>;
    extern __shared__ __align__(16) float bsm[];
    const BwChunk<DK> c{bsm + L::oK, bsm + L::oQ, nullptr, bsm + L::oT, nullptr, bsm + L::oA,
                        reinterpret_cast<double*>(bsm + L::oG), bsm + L::oBeta, bsm + L::oF, bsm + L::of,
                        bsm + L::oGam};
    __shared__ int info[2];
    const int tid = threadIdx.x, H = p.H;
    const long long slot = blockIdx.x / H;
    const int h = blockIdx.x % H;
    if (tid == 0) bw_slot_chunk(p, slot, info, err);
    __syncthreads();
    const int Lc = info[1];
    if (Lc == 0) return;
    float* out = p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk;  // T, then P
    bw_chunk_prep<TIn, DK>(c, p, (size_t)info[0], h, Lc, out + kChunk * kChunk);
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += kBwThreads) out[e] = c.T[(e / kChunk) * L::LDT + e % kChunk];
}

template <int DK>
struct BwChunkSmem {  // 4-byte words
    static constexpr int LDK = DK + 1, LDT = kChunk + 1, DVT = 16, LDV = DVT + 4;  // value tiles: 16-byte rows
    static constexpr int oK = 0, oQ = oK + kChunk * LDK, oGm = oQ + kChunk * LDK, oT = oGm + kChunk * LDT;
    static constexpr int oP = oT + kChunk * LDT, oA = oP + kChunk * LDT;  // A, then dT
    static constexpr int odP = oA + kChunk * LDT;
    static constexpr int oG = odP + kChunk * LDT;  // double [64]
    static constexpr int oBeta = oG + 2 * kChunk, oF = oBeta + kChunk, of = oF + kChunk, oGam = of + kChunk;
    static constexpr int odBeta = oGam + 4, odF = odBeta + kChunk, odf = odF + kChunk, odGn = odf + kChunk;
    static constexpr int odGam = odGn + kChunk;
    static constexpr int oH = (odGam + 4 + 3) / 4 * 4;  // h tile [DK][LDV] (16-byte aligned)
    static constexpr int oDH = oH + DK * LDV;           // dh' tile [DK][LDV]
    static constexpr int oDO = oDH + DK * LDV;          // [64][LDV] tiles: dO, X, U, dU, dX
    static constexpr int oX = oDO + kChunk * LDV, oU = oX + kChunk * LDV;
    static constexpr int oDU = oU + kChunk * LDV, oDX = oDU + kChunk * LDV;
    static constexpr int total = oDX + kChunk * LDV;
    static constexpr size_t bytes = sizeof(float) * (size_t)total;
};

// (3) One CTA per (chunk slot, head): every input gradient of the chunk.
template <typename TIn, int DK>
__global__ void __launch_bounds__(kBwThreads) gdn_bwd_chunk_kernel(const BwdParams p, unsigned* err) {
    using L = BwChunkSmem<DK>;
    constexpr int LDK = L::LDK, LDT = L::LDT, DVT = L::DVT, LDV = L::LDV, NT = kBwThreads;
    extern __shared__ __align__(16) float bsm[];
    const BwChunk<DK> c{bsm + L::oK, bsm + L::oQ, bsm + L::oGm, bsm + L::oT, bsm + L::oP, bsm + L::oA,
                        reinterpret_cast<double*>(bsm + L::oG), bsm + L::oBeta, bsm + L::oF, bsm + L::of,
                        bsm + L::oGam};
    float* sdT = bsm + L::oA;
    float* sdP = bsm + L::odP;
    float* sdBeta = bsm + L::odBeta;
    float* sdF = bsm + L::odF;
    float* sdf = bsm + L::odf;
    float* sdGn = bsm + L::odGn;
    float* sdGam = bsm + L::odGam;
    float* sH = bsm + L::oH;
    float* sDH = bsm + L::oDH;
    float* sDO = bsm + L::oDO;
    float* sX = bsm + L::oX;
    float* sU = bsm + L::oU;
    float* sDU = bsm + L::oDU;
    float* sDX = bsm + L::oDX;
    __shared__ int info[4];
    const int tid = threadIdx.x, H = p.H, dv = p.vdim;
    const long long slot = blockIdx.x / H;
    const int h = blockIdx.x % H;
    if (tid == 0) bw_slot_chunk(p, slot, info, err);
    __syncthreads();
    const int Lc = info[1];
    if (Lc == 0) return;
    const size_t tok0 = (size_t)info[0];
    const TIn* vin = static_cast<const TIn*>(p.v);
    const TIn* dout = static_cast<const TIn*>(p.dout);
    const float* hc = p.h_chunks + ((size_t)slot * H + h) * DK * (size_t)dv;
    const float* dhc = p.dh_chunks + ((size_t)slot * H + h) * DK * (size_t)dv;

    bw_chunk_load<TIn, DK>(c, p, tok0, h, Lc, p.tp + ((size_t)slot * H + h) * 2 * kChunk * kChunk, true);
    for (int e = tid; e < kChunk * LDT; e += NT) {
        sdT[e] = 0.f;
        sdP[e] = 0.f;
    }
    if (tid == 0) sdGam[0] = 0.f;
    // Thread roles over a 64 x 16 value tile: row tr, columns tc .. tc + 3 (the row products and the per-row sums;
    // K h, Q h and K dh' run as 4 x 4 blocks, rows pb .. pb + 3, the sum over the key channels split over the
    // block's four threads, channels kq + 4 t, each thread keeping row tr = pb + kq); rows qr, qr + 32 and channels
    // qc + 8 m (the key-side register sums); rows 4 (tid / 16) .. + 3 and columns tid % 16 + 16 v (dT, dP blocks).
    const int kq = tid & 3, tc = 4 * ((tid >> 2) & 3), pb = 4 * (tid >> 4), tr = pb + kq;
    const int qr = tid >> 3, qc = tid & 7;
    const int pr = 4 * (tid >> 4), pc = tid & 15;
    constexpr int HV = DK * DVT / 4 / NT;  // float4 of each state slice per thread
    static_assert(DK * DVT == 4 * NT * HV && kChunk * DVT == 4 * NT, "tile shapes");
    float aQ[2][16], aK[2][16];            // dq, dk of rows qr, qr + 32, channels qc + 8 m (DK / 8 of them)
    static_assert(DK / 8 <= 16, "register sums");
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int m = 0; m < 16; ++m) aQ[a][m] = aK[a][m] = 0.f;
    float dgam = 0.f, rdb = 0.f, rdF = 0.f, rdf = 0.f;  // <h, dh'>; row tr's partial dbeta, dF, df

    for (int j0 = 0; j0 < dv; j0 += DVT) {
        __syncthreads();  // the previous tile is done
        float4 vv, dov;   // row tr, columns tc .. tc + 3 of V and dO
        {  // every load of the tile first, then the stores
            float4 hv[HV], dhv[HV];
#pragma unroll
            for (int m = 0; m < HV; ++m) {
                const int e = tid + m * NT, i = e / (DVT / 4), cc = 4 * (e % (DVT / 4));
                hv[m] = __ldg(reinterpret_cast<const float4*>(hc + (size_t)i * dv + j0 + cc));
                dhv[m] = __ldg(reinterpret_cast<const float4*>(dhc + (size_t)i * dv + j0 + cc));
            }
            const bool ok = tr < Lc;
            const size_t idx = ((tok0 + tr) * H + h) * dv + j0 + tc;
            vv = ok ? ldg4(vin + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
            dov = ok ? ldg4(dout + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int m = 0; m < HV; ++m) {
                const int e = tid + m * NT, i = e / (DVT / 4), cc = 4 * (e % (DVT / 4));
                *reinterpret_cast<float4*>(sH + i * LDV + cc) = hv[m];
                *reinterpret_cast<float4*>(sDH + i * LDV + cc) = dhv[m];
                dgam = fmaf(hv[m].x, dhv[m].x, dgam);
                dgam = fmaf(hv[m].y, dhv[m].y, dgam);
                dgam = fmaf(hv[m].z, dhv[m].z, dgam);
                dgam = fmaf(hv[m].w, dhv[m].w, dgam);
            }
            *reinterpret_cast<float4*>(sDO + tr * LDV + tc) = dov;
        }
        __syncthreads();
        // K h, Q h, K dh' of row tr ; X = beta V - beta F (K h)
        float kh[4], qh[4], kd[4];
        {
            float bk[4][4] = {}, bq[4][4] = {}, bd[4][4] = {};
#pragma unroll 2
            for (int t = 0; t < DK / 4; ++t) {
                const int i = kq + 4 * t;
                const float4 hv = lds4(sH + i * LDV + tc), dhv = lds4(sDH + i * LDV + tc);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float kv = c.K[(pb + u) * LDK + i], qv = c.Q[(pb + u) * LDK + i];
                    fma4(bk[u], kv, hv);
                    fma4(bq[u], qv, hv);
                    fma4(bd[u], kv, dhv);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int o = 1; o <= 2; o <<= 1) {
                        bk[u][q] += __shfl_xor_sync(0xffffffffu, bk[u][q], o);
                        bq[u][q] += __shfl_xor_sync(0xffffffffu, bq[u][q], o);
                        bd[u][q] += __shfl_xor_sync(0xffffffffu, bd[u][q], o);
                    }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                kh[q] = kq == 0 ? bk[0][q] : kq == 1 ? bk[1][q] : kq == 2 ? bk[2][q] : bk[3][q];
                qh[q] = kq == 0 ? bq[0][q] : kq == 1 ? bq[1][q] : kq == 2 ? bq[2][q] : bq[3][q];
                kd[q] = kq == 0 ? bd[0][q] : kq == 1 ? bd[1][q] : kq == 2 ? bd[2][q] : bd[3][q];
            }
        }
        const float br = c.beta[tr], Fr = c.F[tr], fr = c.f[tr];
        const float vr[4] = {vv.x, vv.y, vv.z, vv.w}, dor[4] = {dov.x, dov.y, dov.z, dov.w};
        float xr[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xr[q] = br * (vr[q] - Fr * kh[q]);
        sts4(sX + tr * LDV + tc, xr[0], xr[1], xr[2], xr[3]);
        __syncthreads();
        // U = T X ; dU = scale P^T dO + diag(f) K dh'
        float ur[4], du[4];
        blk_tri_TX<LDT, LDV>(c.T, sX, pb, kq, tc, ur);
        blk_tri_TtX<LDT, LDV>(c.P, sDO, pb, kq, tc, du);
#pragma unroll
        for (int q = 0; q < 4; ++q) du[q] = p.scale * du[q] + fr * kd[q];
        sts4(sU + tr * LDV + tc, ur[0], ur[1], ur[2], ur[3]);
        sts4(sDU + tr * LDV + tc, du[0], du[1], du[2], du[3]);
        __syncthreads();
        // dX = T^T dU ; dv = beta dX ; the per-row sums of dbeta, dF, df
        {
            float dx[4];
            blk_tri_TtX<LDT, LDV>(c.T, sDU, pb, kq, tc, dx);
            sts4(sDX + tr * LDV + tc, dx[0], dx[1], dx[2], dx[3]);
            if (tr < Lc)
                *reinterpret_cast<float4*>(p.dv + ((tok0 + tr) * H + h) * dv + j0 + tc) =
                    make_float4(br * dx[0], br * dx[1], br * dx[2], br * dx[3]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                rdb = fmaf(dx[q], vr[q] - Fr * kh[q], rdb);
                rdF = fmaf(-br * dx[q], kh[q], rdF);
                rdF = fmaf(p.scale * dor[q], qh[q], rdF);
                rdf = fmaf(ur[q], kd[q], rdf);
            }
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
        {  // register sums: dq += scale F_r dO h^T ; dk += f_r U dh'^T - beta_r F_r dX h^T
#pragma unroll
            for (int jg = 0; jg < DVT; jg += 4) {
                float4 o[2], x[2], u4[2];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    const int r = qr + 32 * a;
                    const float so = p.scale * c.F[r], sx = -c.beta[r] * c.F[r], su = c.f[r];
                    const float4 o0 = lds4(sDO + r * LDV + jg), x0 = lds4(sDX + r * LDV + jg);
                    const float4 u0 = lds4(sU + r * LDV + jg);
                    o[a] = make_float4(so * o0.x, so * o0.y, so * o0.z, so * o0.w);
                    x[a] = make_float4(sx * x0.x, sx * x0.y, sx * x0.z, sx * x0.w);
                    u4[a] = make_float4(su * u0.x, su * u0.y, su * u0.z, su * u0.w);
                }
#pragma unroll
                for (int m = 0; m < DK / 8; ++m) {
                    const int i = qc + 8 * m;
                    const float4 hv = lds4(sH + i * LDV + jg), dhv = lds4(sDH + i * LDV + jg);
#pragma unroll
                    for (int a = 0; a < 2; ++a) {
                        aQ[a][m] = fmaf(o[a].x, hv.x, fmaf(o[a].y, hv.y, fmaf(o[a].z, hv.z, fmaf(o[a].w, hv.w,
                                   aQ[a][m]))));
                        aK[a][m] = fmaf(u4[a].x, dhv.x, fmaf(u4[a].y, dhv.y, fmaf(u4[a].z, dhv.z,
                                   fmaf(u4[a].w, dhv.w, aK[a][m]))));
                        aK[a][m] = fmaf(x[a].x, hv.x, fmaf(x[a].y, hv.y, fmaf(x[a].z, hv.z, fmaf(x[a].w, hv.w,
                                   aK[a][m]))));
                    }
                }
            }
        }
    }
    // the per-row sums over the four threads of a row (lanes 4 and 8 apart); dgamma over the CTA
    rdb += __shfl_xor_sync(0xffffffffu, rdb, 4);
    rdb += __shfl_xor_sync(0xffffffffu, rdb, 8);
    rdF += __shfl_xor_sync(0xffffffffu, rdF, 4);
    rdF += __shfl_xor_sync(0xffffffffu, rdF, 8);
    rdf += __shfl_xor_sync(0xffffffffu, rdf, 4);
    rdf += __shfl_xor_sync(0xffffffffu, rdf, 8);
    if (tc == 0) {
        sdBeta[tr] = rdb;
        sdF[tr] = rdF;
        sdf[tr] = rdf;
    }
    for (int o = 16; o > 0; o >>= 1) dgam += __shfl_xor_sync(0xffffffffu, dgam, o);
    __syncthreads();
    if ((tid & 31) == 0) atomicAdd(sdGam, dgam);
    // dA = -T^T dT T^T on the strictly lower part (dT's diagonal and upper part do not reach A)
    float* sM = sDO;  // [64][LDT] scratch over the tile buffers (dO, X, U ... are no longer needed)
    static_assert(kChunk * (kChunk + 1) <= 5 * kChunk * L::LDV, "scratch fits the tile buffers");
    __syncthreads();
    for (int e = tid; e < kChunk * kChunk; e += NT) {  // M = dT T^T, dT strictly lower
        const int r = e / kChunk, s = e % kChunk;
        float m = 0.f;
        const int tmax = min(r - 1, s);
        for (int t = 0; t <= tmax; ++t) m = fmaf(sdT[r * LDT + t], c.T[s * LDT + t], m);
        sM[r * LDT + s] = m;
    }
    __syncthreads();
    float* sdA = c.A;  // A is no longer needed
    for (int e = tid; e < kChunk * kChunk; e += NT) {
        const int r = e / kChunk, s = e % kChunk;
        float a = 0.f;
        if (s < r)
            for (int t = r; t < kChunk; ++t) a = fmaf(c.T[t * LDT + r], sM[t * LDT + s], a);
        sdA[r * LDT + s] = -a;
    }
    __syncthreads();
    // through A and P to K, Q, beta and Gamma: dKK = dA beta_r Gamma, dQK = dP Gamma; W = dGamma . Gamma.  K K^T
    // and Q K^T are formed again as 4 x 4 blocks (rows pr .. pr + 3, columns pc + 16 v).
    float* sW = sM;
    {
        float kk[4][4] = {}, qk[4][4] = {};
#pragma unroll 2
        for (int i = 0; i < DK; ++i) {
            float ks[4], kr[4], qv[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) ks[v] = c.K[(pc + 16 * v) * LDK + i];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                kr[u] = c.K[(pr + u) * LDK + i];
                qv[u] = c.Q[(pr + u) * LDK + i];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    kk[u][v] = fmaf(kr[u], ks[v], kk[u][v]);
                    qk[u][v] = fmaf(qv[u], ks[v], qk[u][v]);
                }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = pr + u;
            float dbs = 0.f;  // this thread's share of dbeta_r
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int s2 = pc + 16 * v;
                float dkk = 0.f, dqk = 0.f, w = 0.f;
                if (s2 <= r) {
                    const float gm = c.Gm[r * LDT + s2], da = sdA[r * LDT + s2], dp = sdP[r * LDT + s2];
                    if (s2 < r) {
                        dkk = da * c.beta[r] * gm;
                        dbs = fmaf(da * gm, kk[u][v], dbs);
                    }
                    dqk = dp * gm;
                    w = (da * c.beta[r] * kk[u][v] + dp * qk[u][v]) * gm;
                }
                sdT[r * LDT + s2] = dkk;  // dT holds dKK from here on
                sdP[r * LDT + s2] = dqk;  // dP holds dQK
                sW[r * LDT + s2] = w;
            }
            atomicAdd(&sdBeta[r], dbs);
        }
    }
    __syncthreads();
    // gradient of the natural-log cumulative gate Gn (Gamma_rs = exp(Gn_r - Gn_s), F = exp(Gn), f = exp(Gn_L - Gn),
    // gamma = exp(Gn_L), L the chunk's last row 63: padded rows add nothing)
    if (tid < kChunk) {
        const int r = tid;
        float d = c.F[r] * sdF[r] - c.f[r] * sdf[r];
        for (int s = 0; s <= r; ++s) d += sW[r * LDT + s];
        for (int t = r; t < kChunk; ++t) d -= sW[t * LDT + r];
        if (r == kChunk - 1) {
            float fs = 0.f;
            for (int s = 0; s < kChunk; ++s) fs = fmaf(c.f[s], sdf[s], fs);
            d += fs + c.gamma[0] * sdGam[0];
        }
        sdGn[r] = d;
    }
    // dQ += dQK K ; dK += dQK^T Q + dKK^T K + dKK K   (register sums of rows qr, qr + 32)
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const int r = qr + 32 * a;
        for (int s2 = 0; s2 <= r; ++s2) {
            const float wq = sdP[r * LDT + s2], wk = sdT[r * LDT + s2];
#pragma unroll
            for (int m = 0; m < DK / 8; ++m) {
                const float kv = c.K[s2 * LDK + qc + 8 * m];
                aQ[a][m] = fmaf(wq, kv, aQ[a][m]);
                aK[a][m] = fmaf(wk, kv, aK[a][m]);
            }
        }
        // from the warp's first row, so that the warp's four row groups read the same K and Q rows (the rows
        // before r add zero)
        for (int t = (tid >> 5) * 4 + 32 * a; t < kChunk; ++t) {
            const float wq = t >= r ? sdP[t * LDT + r] : 0.f, wk = t >= r ? sdT[t * LDT + r] : 0.f;
#pragma unroll
            for (int m = 0; m < DK / 8; ++m)
                aK[a][m] = fmaf(wq, c.Q[t * LDK + qc + 8 * m], fmaf(wk, c.K[t * LDK + qc + 8 * m], aK[a][m]));
        }
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const int r = qr + 32 * a;
        if (r < Lc) {
#pragma unroll
            for (int m = 0; m < DK / 8; ++m) {
                const size_t idx = ((tok0 + r) * H + h) * DK + qc + 8 * m;
                p.dq[idx] = aQ[a][m];
                p.dk[idx] = aK[a][m];
            }
        }
    }
    if (tid < Lc) {
        const int t = tid;
        float dg = 0.f;
        for (int r = t; r < kChunk; ++r) dg += sdGn[r];
        p.dg[(tok0 + t) * H + h] = dg;
        p.dbeta[(tok0 + t) * H + h] = sdBeta[t];
    }
}

}  // namespace gdn
