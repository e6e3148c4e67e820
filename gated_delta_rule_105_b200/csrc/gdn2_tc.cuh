// tcgen05 chunked forward of Gated Delta Rule-2 (per-channel gates), bf16 inputs, dk = 128: two kernels.
//
// Per chunk of C = 64 tokens (r, s = token rows, i = key channel, j = value column; G_ri = log2(e) times the
// chunk-local cumulative g_ri; e_r = b_r . k_r the erase key; L = the chunk's last row):
//   A_rs = sum_i e_ri k_si 2^(G_ri - G_si)   (s < r)        T = (I + A)^-1
//   P_rs = sum_i q_ri k_si 2^(G_ri - G_si)   (s <= r)
//   W = T (e . 2^G) ;  U = T (w . V) - W h
//   O = scale ((q . 2^G) h + P U)
//   h <- Diag(2^G_L) h + (k . 2^(G_L - G))^T U
// (Gated DeltaNet-2 article, 7minutos.es: the recurrence in section "Regla-2 del Delta cerrado", the chunked
// form with both erase factors carrying the channel decay in section "Entrenamiento fragmentado y
// reconocimiento de puertas hacia atras".)
//
// The per-channel factor 2^(G_ri - G_si) sits inside the sums over i, so A and P are not one product with a
// scaled result as in GDN.  Between 16-token sub-chunks it splits through the first row m of the later
// sub-chunk: 2^(G_ri - G_mi) 2^(G_mi - G_si), both factors <= 1 because g <= 0, so those blocks are plain
// products of scaled bf16 rows (q . 2^(G_r - G_m), e . 2^(G_r - G_m), k . 2^(G_m - G_s)).  Inside the four
// diagonal 16x16 blocks a fixed reference row could overflow fp32 (the decay of one sub-chunk can pass 2^-126),
// so they are summed on CUDA cores with the exact factor, a running product of the per-token decays.
//
// The prep kernel (gdn2_tc_prep_kernel) does every step that does not depend on the state, for all chunks of
// all sequences at once, and writes one workspace unit per (chunk, head) in the exact shared-memory form the
// chunk kernel's MMAs read: T (bf16 hi + lo), -W^T, P (tf32), Q' = q . 2^G, K~ = k . 2^(G_L - G) (bf16) and
// Lambda = 2^G_L.  The chunk kernel (gdn2_tc_fwd_kernel) walks each sequence's chunks with the state h^T fp32 in
// TMEM, as the GDN chunk kernel does: U^T = (w.V)^T T^T - h^T W^T, h^T <- h^T Diag(Lambda) + U^T K~,
// O^T = h^T Q'^T + U^T P^T.  w . V is formed in the chunk kernel (per value tile) as a bf16 hi + lo pair.
// Precision: a numpy emulation of these rounding sites on the GDN-2 workload's inputs gave o and hT errors of
// 0.4-1.0e-2 of RMS; splitting w . V into hi + lo was needed (without it: 4-5e-2), Q' and W need no lo part.
#pragma once

#include "gdn_tc.cuh"

namespace gdn {

constexpr int kG2Threads = 512;

// Workspace unit of one (chunk slot, head), byte offsets.  Every swizzled region is 1024-byte aligned inside the
// unit, so a bulk copy into a 1024-aligned shared-memory buffer keeps the 128-byte swizzle pattern.
struct G2Unit {
    static constexpr uint32_t TH = 0;       // T hi: [r][s] bf16, K-major, 128B swizzle (8 KB)
    static constexpr uint32_t TL = 8192;    // T lo = bf16(T - T hi)
    static constexpr uint32_t WT = 16384;   // -W^T: lines i (128) x 64 r bf16, MN-major B operand (16 KB)
    static constexpr uint32_t PH = 32768;   // P columns s 0-31: [r][s] fp32 (tf32-rounded), K-major (8 KB)
    static constexpr uint32_t PL = 40960;   // P columns s 32-63
    static constexpr uint32_t QP = 49152;   // Q' = q . 2^G: [r][i] bf16, channel panels 0-63 | 64-127 (8 KB each)
    static constexpr uint32_t KT = 65536;   // K~ = k . 2^(G_L - G): [s][i] bf16, same layout
    static constexpr uint32_t LAM = 81920;  // Lambda_i = 2^(G_L,i), fp32 [128]
    static constexpr uint32_t BYTES = 82432;
};

inline size_t tc2_workspace_bytes(int B, int T, int H, int n_seqs) {
    return (size_t)wy_slots(B, T, n_seqs) * (size_t)H * G2Unit::BYTES;
}

// ------------------------------------------------------------------------------------------ warp-level MMA
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr)
                 : "memory");
}
// D(16x8) += A(16x16) B(16x8), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Element (r, s) of P, rounded to tf32, into a unit image (G2Unit::PH / PL layout).
__device__ __forceinline__ void st_p_tf32(uint8_t* unit, int r, int s, float x) {
    uint8_t* panel = unit + ((s & 32) ? G2Unit::PL : G2Unit::PH);
    *reinterpret_cast<uint32_t*>(panel + sm100::sw128(r, (s & 31) >> 2) + (s & 3) * 4) = f2tf32(x);
}

// ------------------------------------------------------------------------------------------ the prep kernel
// Shared-memory map (bytes from a 1024-aligned base).
struct G2PrepSmem {
    static constexpr uint32_t STG = 0;                // the unit image, bulk-stored at the end; its Q' and K~ places
                                                      // first receive q and k themselves (TMA, 0 past the chunk end)
    static constexpr uint32_t SG = 82944;             // g (TMA), then G, fp32 [64][128]
    static constexpr uint32_t SE = SG + 32768;        // b (TMA), then e = b . k, fp32 [64][128]
    static constexpr uint32_t SA = SE + 32768;        // A, then (I + A)^-1, fp32 [64][kAsLd]
    static constexpr uint32_t SOP = SA + 64 * kAsLd * 4;  // scaled rows of the off-diagonal products; then the
                                                          // per-token decays fp32 [64][128]; then E' bf16
    static constexpr uint32_t OP_LD = 272;            // row pitch (bytes) of the bf16 operand rows (ldmatrix)
    static constexpr uint32_t TOT = SOP + 192 * OP_LD;  // per-sub-chunk sums of g [4][128]
    static constexpr uint32_t BETA = TOT + 2048;        // KDA: beta of the chunk's rows [64]
    static constexpr uint32_t MISC = BETA + 256;        // unit info, mbarrier, abort flag
    static constexpr uint32_t END = MISC + 64;
    static constexpr uint32_t ALLOC = END + 1024;
};
static_assert(G2PrepSmem::STG + G2Unit::BYTES <= G2PrepSmem::SG, "unit image");
static_assert(64 * 128 * 4 <= 192 * G2PrepSmem::OP_LD, "decay table fits the operand rows");
static_assert(G2PrepSmem::ALLOC <= 232448, "shared memory budget");

// One CTA per (workspace slot, head), 16 warps.  Phases (each ends at a CTA barrier):
//   1  TMA of q, k, g, b; the chunk-local cumulative gate G and e = b . k (thread: channel i, sub-chunk of 16
//      tokens; the thread keeps its per-token decays 2^(log2(e) g) in registers for phase 3), Lambda
//   2  scaled rows for the off-diagonal sub-chunk blocks, then those blocks of A and P on mma.sync
//   3  per-token decays, then the diagonal 16x16 blocks of A and P (running products, CUDA cores)
//   4  warps 0-3: T = (I + A)^-1 (blocked, emitted as T hi / lo); warps 4-15: Q', K~ and E' = e . 2^G
//   5  -W^T = -(T_hi E')^T on mma.sync; bulk store of the unit
// Rows past the chunk end carry zero q, k and erase gate, so their rows and columns of A, P, W, Q', K~ are 0.
__global__ void __launch_bounds__(kG2Threads, 1)
gdn2_tc_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_b, const FwdParams p,
                    uint8_t* ws, unsigned* err) {
    using namespace sm100;
    using L = G2PrepSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int* info = reinterpret_cast<int*>(sm + L::MISC);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::MISC + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 32);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long slot = blockIdx.x / p.H;
    const int h = blockIdx.x % p.H, H = p.H;
    if (tid == 0) {
        int Lc = 0;
        wy_unit_of_slot(p, slot, &info[0], &Lc, err);
        info[1] = Lc;
        if (Lc > 0) {
            const int tok0 = info[0];
            uint8_t* stg = sm + L::STG;
            mbar_init(bar, 1);
            *abort_flag = 0;
            fence_barrier_init();
            mbar_expect_tx(bar, p.kda ? 65536u : 98304u);
            tma_load_3d(stg + G2Unit::QP, &tm_q, bar, 0, h, tok0);
            tma_load_3d(stg + G2Unit::QP + 8192, &tm_q, bar, 64, h, tok0);
            tma_load_3d(stg + G2Unit::KT, &tm_k, bar, 0, h, tok0);
            tma_load_3d(stg + G2Unit::KT + 8192, &tm_k, bar, 64, h, tok0);
            tma_load_3d(sm + L::SG, &tm_g, bar, 0, h, tok0);
            if (!p.kda) tma_load_3d(sm + L::SE, &tm_b, bar, 0, h, tok0);
        }
    }
    __syncthreads();
    const int tok0 = info[0], Lc = info[1];
    if (Lc == 0) return;  // unused slot

    float* sG = reinterpret_cast<float*>(sm + L::SG);
    float* sE = reinterpret_cast<float*>(sm + L::SE);
    float* sA = reinterpret_cast<float*>(sm + L::SA);
    float* tot = reinterpret_cast<float*>(sm + L::TOT);
    float* sBeta = reinterpret_cast<float*>(sm + L::BETA);
    uint8_t* stg = sm + L::STG;
    // q and k of row r, channel i, in the 128B-swizzled [r][i] layout of the unit's Q' / K~ places
    auto qk_off = [](int r, int i) -> uint32_t {
        return (uint32_t)(i >> 6) * 8192u + sm100::sw128(r, (i & 63) >> 3) + (i & 7) * 2;
    };
    if (p.kda && tid < 64) sBeta[tid] = tid < Lc ? p.beta[(size_t)(tok0 + tid) * H + h] : 0.f;
    for (int e = tid; e < 64 * kAsLd; e += kG2Threads) sA[e] = 0.f;
    const bool landed = mbar_wait(bar, 0, abort_flag, err);
    if (!__syncthreads_and(landed)) return;

    // ---- phase 1: G, e, decays.  Rows past the chunk end (the next sequence's tokens, or TMA zero fill) are
    // cleared: g = 0 there, and q = k = e = 0.
    float al[16];
    {
        const int i = tid & 127, ps = tid >> 7;
        float run = 0.f;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const int r = 16 * ps + rr, e = r * 128 + i;
            const bool ok = r < Lc;
            const float gv = ok ? sG[e] : 0.f;
            al[rr] = (ok && rr != 0) ? ex2_approx(gv * kLog2e) : 1.f;
            run += gv;
            sG[e] = run;
            __nv_bfloat16* qp = reinterpret_cast<__nv_bfloat16*>(stg + G2Unit::QP + qk_off(r, i));
            __nv_bfloat16* kp = reinterpret_cast<__nv_bfloat16*>(stg + G2Unit::KT + qk_off(r, i));
            float kv = 0.f;
            if (ok) {
                kv = __bfloat162float(*kp);
            } else {
                *qp = __float2bfloat16_rn(0.f);
                *kp = __float2bfloat16_rn(0.f);
            }
            const float bv = ok ? (p.kda ? sBeta[r] : sE[e]) : 0.f;
            sE[e] = bv * kv;
        }
        tot[ps * 128 + i] = run;
    }
    __syncthreads();
    {
        const int i = tid & 127, ps = tid >> 7;
        float pre = 0.f;
        for (int q2 = 0; q2 < ps; ++q2) pre += tot[q2 * 128 + i];
#pragma unroll 4
        for (int rr = 0; rr < 16; ++rr) {
            const int e = (16 * ps + rr) * 128 + i;
            sG[e] = (sG[e] + pre) * kLog2e;
        }
    }
    __syncthreads();
    if (tid < 128) reinterpret_cast<float*>(stg + G2Unit::LAM)[tid] = ex2_approx(sG[63 * 128 + tid]);

    // ---- phase 2: off-diagonal sub-chunk blocks.  Rows 0-95: for I = 1, 2, 3 (m = 16 I), 16 rows of
    // e . 2^(G_r - G_m) then 16 rows of q . 2^(G_r - G_m) for r in [m, m + 16); rows 96-191: k . 2^(G_m - G_s) for
    // s < m (16, 32 and 48 rows).
    // Work item: one row and 8 consecutive channels (one 16-byte chunk of the q / k layout, two float4 of G and e).
    {
        for (int item = tid; item < 192 * 16; item += kG2Threads) {
            const int row = item >> 4, ch = item & 15, c0 = 8 * ch;
            const uint32_t qk_chunk = (uint32_t)(ch >> 3) * 8192u;  // panel of channels c0 .. c0 + 7
            int src, m;
            bool side_r, use_e = false;
            if (row < 96) {
                const int I = row / 32 + 1, w = row % 32;
                m = 16 * I;
                src = m + (w & 15);
                side_r = true;
                use_e = w < 16;
            } else {
                const int y = row - 96;
                const int I = y < 16 ? 1 : (y < 48 ? 2 : 3);
                m = 16 * I;
                src = y - (I == 1 ? 0 : (I == 2 ? 16 : 48));
                side_r = false;
            }
            const float4* gs = reinterpret_cast<const float4*>(sG + src * 128 + c0);
            const float4* gm = reinterpret_cast<const float4*>(sG + m * 128 + c0);
            const float4 gs0 = gs[0], gs1 = gs[1], gm0 = gm[0], gm1 = gm[1];
            const float dg[8] = {gs0.x - gm0.x, gs0.y - gm0.y, gs0.z - gm0.z, gs0.w - gm0.w,
                                 gs1.x - gm1.x, gs1.y - gm1.y, gs1.z - gm1.z, gs1.w - gm1.w};
            float x[8];
            if (use_e) {
                const float4* ep = reinterpret_cast<const float4*>(sE + src * 128 + c0);
                const float4 e0 = ep[0], e1 = ep[1];
                x[0] = e0.x, x[1] = e0.y, x[2] = e0.z, x[3] = e0.w, x[4] = e1.x, x[5] = e1.y, x[6] = e1.z, x[7] = e1.w;
            } else {
                const uint8_t* base = stg + (side_r ? G2Unit::QP : G2Unit::KT) + qk_chunk;
                const uint4 u = *reinterpret_cast<const uint4*>(base + sw128(src, ch & 7));
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int c2 = 0; c2 < 4; ++c2) {
                    const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[c2]));
                    x[2 * c2] = f2.x;
                    x[2 * c2 + 1] = f2.y;
                }
            }
            // r side: 2^(G_r - G_m); s side: 2^(G_m - G_s)
            uint32_t o4[4];
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
                const float f0 = ex2_approx(side_r ? dg[2 * c2] : -dg[2 * c2]);
                const float f1 = ex2_approx(side_r ? dg[2 * c2 + 1] : -dg[2 * c2 + 1]);
                o4[c2] = pack_bf16(x[2 * c2] * f0, x[2 * c2 + 1] * f1);
            }
            *reinterpret_cast<uint4*>(sm + L::SOP + row * L::OP_LD + 16 * ch) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
    }
    __syncthreads();
    {
        // 24 output tiles of 16 x 8: (I, mt, nt) with mt 0 = the e rows (A), 1 = the q rows (P), nt over s < 16 I
        const uint32_t sop = smem_u32(sm + L::SOP);
        const int g = lane >> 2, t4 = lane & 3;
        for (int tix = warp; tix < 24; tix += 16) {
            int I, mt, nt;
            if (tix < 4) {
                I = 1, mt = tix >> 1, nt = tix & 1;
            } else if (tix < 12) {
                I = 2, mt = (tix - 4) >> 2, nt = (tix - 4) & 3;
            } else {
                I = 3, mt = (tix - 12) / 6, nt = (tix - 12) % 6;
            }
            const int kbase = I == 1 ? 0 : (I == 2 ? 16 : 48);
            const uint32_t a_row = (I - 1) * 32 + mt * 16 + (lane & 15);
            const uint32_t b_row = 96 + kbase + nt * 8 + (lane & 7);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                uint32_t a[4], b[2];
                ldsm_x4(sop + a_row * L::OP_LD + (ks * 16 + (lane >> 4) * 8) * 2, a);
                ldsm_x2(sop + b_row * L::OP_LD + (ks * 16 + ((lane >> 3) & 1) * 8) * 2, b);
                mma_bf16_16816(d, a, b);
            }
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 16 * I + g + 8 * hr, s = nt * 8 + 2 * t4;
                if (mt == 0) {
                    sA[r * kAsLd + s] = d[2 * hr];
                    sA[r * kAsLd + s + 1] = d[2 * hr + 1];
                } else {
                    st_p_tf32(stg, r, s, d[2 * hr]);
                    st_p_tf32(stg, r, s + 1, d[2 * hr + 1]);
                }
            }
        }
    }
    __syncthreads();

    // ---- phase 3: the diagonal blocks.  alpha_t = 2^(log2(e) g_t) per channel, from the registers of phase 1
    // (rows that start a block are unused).
    float* sAl = reinterpret_cast<float*>(sm + L::SOP);
    {
        const int i = tid & 127, ps = tid >> 7;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) sAl[(16 * ps + rr) * 128 + i] = al[rr];
    }
    __syncthreads();
    {
        // thread: block I, row r, channels [16 cg, 16 cg + 16); the 8 threads of a row are consecutive lanes.
        // EF, QF hold e_r . F and q_r . F with F_s = prod_{t = s+1..r} alpha_t, updated as s walks down from r.
        const int cg = tid & 7, I = tid >> 7, r = 16 * I + ((tid >> 3) & 15), c0 = 16 * cg;
        float EF[16], QF[16];
        const uint32_t kq_panel = (uint32_t)(c0 >> 6) * 8192u, kq_ch = (uint32_t)(c0 & 63) >> 3;
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const uint4 u = *reinterpret_cast<const uint4*>(stg + G2Unit::QP + kq_panel + sw128(r, kq_ch + h8));
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
                const float2 qv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[c2]));
                QF[8 * h8 + 2 * c2] = qv.x;
                QF[8 * h8 + 2 * c2 + 1] = qv.y;
            }
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) EF[c] = sE[r * 128 + c0 + c];
        const int steps = 4 * (warp & 3) + 4;  // rows of this warp: 4 (warp & 3) .. + 3 within the block
        for (int d = 0; d < steps; ++d) {
            const int s = r - d;
            const bool act = s >= 16 * I;
            const int sc = act ? s : 16 * I;
            if (d > 0 && act) {
                const float4* al = reinterpret_cast<const float4*>(sAl + (sc + 1) * 128 + c0);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float4 a4 = al[c4];
                    EF[4 * c4 + 0] *= a4.x, QF[4 * c4 + 0] *= a4.x;
                    EF[4 * c4 + 1] *= a4.y, QF[4 * c4 + 1] *= a4.y;
                    EF[4 * c4 + 2] *= a4.z, QF[4 * c4 + 2] *= a4.z;
                    EF[4 * c4 + 3] *= a4.w, QF[4 * c4 + 3] *= a4.w;
                }
            }
            float accA = 0.f, accP = 0.f;
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const uint4 u = *reinterpret_cast<const uint4*>(stg + G2Unit::KT + kq_panel + sw128(sc, kq_ch + h8));
                const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int c2 = 0; c2 < 4; ++c2) {
                    const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[c2]));
                    const int c = 8 * h8 + 2 * c2;
                    accA = fmaf(EF[c], kv.x, accA);
                    accA = fmaf(EF[c + 1], kv.y, accA);
                    accP = fmaf(QF[c], kv.x, accP);
                    accP = fmaf(QF[c + 1], kv.y, accP);
                }
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                accA += __shfl_xor_sync(0xffffffffu, accA, o);
                accP += __shfl_xor_sync(0xffffffffu, accP, o);
            }
            if (cg == 0 && act) {
                if (d > 0) sA[r * kAsLd + s] = accA;
                st_p_tf32(stg, r, s, accP);
            }
        }
        // P above the diagonal inside the block is read by the chunk kernel's triangular MMAs: zero it
        if (cg == 0)
            for (int s = r + 1; s < 16 * I + 16; ++s) st_p_tf32(stg, r, s, 0.f);
    }
    __syncthreads();

    // ---- phase 4: the inverse (warps 0-3) and the scaled operands of the chunk kernel (warps 4-15)
    uint8_t* sEp = sm + L::SOP;  // E' = e . 2^G, bf16 [s][i], pitch OP_LD (the decays are no longer needed)
    if (warp < 4) {
        const TEmitPlain em{stg + G2Unit::TH, stg + G2Unit::TL};
        invert_unit_lower64(sA, warp, lane, 1, em);
    } else {
        // q and k are turned into Q' and K~ in place (each 16-byte chunk read and written by the same thread)
        for (int item = tid - 128; item < 64 * 16; item += kG2Threads - 128) {
            const int r = item >> 4, ch = item & 15, c0 = 8 * ch;
            const float4* gp = reinterpret_cast<const float4*>(sG + r * 128 + c0);
            const float4* gl = reinterpret_cast<const float4*>(sG + 63 * 128 + c0);
            const float4* ep = reinterpret_cast<const float4*>(sE + r * 128 + c0);
            const float4 g0 = gp[0], g1 = gp[1], l0 = gl[0], l1 = gl[1], e0 = ep[0], e1 = ep[1];
            const float G[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const float GL[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
            const float E[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
            const uint32_t off = (uint32_t)(ch >> 3) * 8192u + sw128(r, ch & 7);
            uint4* qp = reinterpret_cast<uint4*>(stg + G2Unit::QP + off);
            uint4* kp = reinterpret_cast<uint4*>(stg + G2Unit::KT + off);
            const uint4 qu = *qp, ku = *kp;
            const uint32_t qw[4] = {qu.x, qu.y, qu.z, qu.w}, kw[4] = {ku.x, ku.y, ku.z, ku.w};
            uint32_t qo[4], ko[4], eo[4];
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
                const float2 qv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw[c2]));
                const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw[c2]));
                const int a = 2 * c2, b = a + 1;
                const float f1a = ex2_approx(G[a]), f1b = ex2_approx(G[b]);
                qo[c2] = pack_bf16(qv.x * f1a, qv.y * f1b);
                ko[c2] = pack_bf16(kv.x * ex2_approx(GL[a] - G[a]), kv.y * ex2_approx(GL[b] - G[b]));
                eo[c2] = pack_bf16(E[a] * f1a, E[b] * f1b);
            }
            *qp = make_uint4(qo[0], qo[1], qo[2], qo[3]);
            *kp = make_uint4(ko[0], ko[1], ko[2], ko[3]);
            *reinterpret_cast<uint4*>(sEp + r * L::OP_LD + 16 * ch) = make_uint4(eo[0], eo[1], eo[2], eo[3]);
        }
    }
    __syncthreads();

    // ---- phase 5: W = T_hi E' (T lower triangular: k-steps above the row block skipped); -W^T into the unit
    {
        const int mt = warp & 3;
        const uint32_t th = smem_u32(stg + G2Unit::TH), ep = smem_u32(sEp);
        const int g = lane >> 2, t4 = lane & 3;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
            const int nt = (warp >> 2) * 4 + q4;  // channels [8 nt, 8 nt + 8)
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            for (int ks = 0; ks <= mt; ++ks) {
                uint32_t a[4], b[2];
                ldsm_x4(th + sw128(16 * mt + (lane & 15), 2 * ks + (lane >> 4)), a);
                ldsm_x2_trans(ep + (16 * ks + (lane & 15)) * L::OP_LD + nt * 16, b);
                mma_bf16_16816(d, a, b);
            }
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 16 * mt + g + 8 * hr, i = 8 * nt + 2 * t4;
                const uint32_t o0 = sw128(i, r >> 3) + (r & 7) * 2, o1 = sw128(i + 1, r >> 3) + (r & 7) * 2;
                *reinterpret_cast<__nv_bfloat16*>(stg + G2Unit::WT + o0) = __float2bfloat16_rn(-d[2 * hr]);
                *reinterpret_cast<__nv_bfloat16*>(stg + G2Unit::WT + o1) = __float2bfloat16_rn(-d[2 * hr + 1]);
            }
        }
    }
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        bulk_store(ws + ((size_t)slot * H + h) * G2Unit::BYTES, stg, G2Unit::BYTES);
        bulk_commit();
        bulk_wait_read();  // the CTA may exit once the store has read shared memory
    }
}

// ------------------------------------------------------------------------------------------ the chunk kernel
struct G2Smem {
    static constexpr uint32_t VH = 0;         // V tile (TMA: value columns 0-63 | 64-127, [64 s][128 B] each), then
                                              // (w . V) hi in place (MN-major A of the U~ MMA)
    static constexpr uint32_t VL = 16384;     // (w . V) lo, same layout
    static constexpr uint32_t W32 = 32768;    // w tile (TMA), fp32 [64 s][128 j]
    static constexpr uint32_t TW = 65536;     // T hi | T lo
    static constexpr uint32_t WT = 81920;     // -W^T
    static constexpr uint32_t P = 98304;      // P: PH | PL
    static constexpr uint32_t QP = 114688;    // Q'
    static constexpr uint32_t KT = 131072;    // K~
    static constexpr uint32_t HT = 147456;    // h^T bf16 [2]: [j][i] K-major, channel panels 0-63 | 64-127
    static constexpr uint32_t HT_STAGE = 32768;
    static constexpr uint32_t LAM = HT + 2 * HT_STAGE;  // Lambda [2] x 512 B
    static constexpr uint32_t BARS = LAM + 1024;
    static constexpr uint32_t N_BARS = 24;
    static constexpr uint32_t MISC = BARS + 8 * N_BARS;  // tmem base, abort flag
    static constexpr uint32_t END = MISC + 64;
    static constexpr uint32_t ALLOC = END + 1024;
};
static_assert(G2Smem::ALLOC <= 232448, "shared memory budget");

enum G2Bar : int {
    G_VR_FULL = 0,    // V and w landed (tx)
    G_VW_FULL = 2,    // w . V hi / lo written (128)
    G_UT_DONE = 3,    // U~ MMA done (w . V and T read)
    G_TW_FULL = 4,    // T hi | lo landed (tx)
    G_WT_FULL = 5,    // -W^T landed (tx)
    G_KT_FULL = 6,    // K~ landed (tx)
    G_QP_FULL = 7,    // Q' landed (tx)
    G_P_FULL = 8,     // P landed (tx)
    G_LAM_FULL = 9,   // [2] Lambda landed (tx)
    G_U_FULL = 11,    // U^T in TMEM (and -W^T read)
    G_U_CONV = 12,    // U split into bf16 hi / lo in TMEM (256)
    G_U_RND = 13,     // U in TMEM rounded to tf32 (256)
    G_H_FULL = 14,    // h^T MMA done (and K~ read)
    G_H_READY = 15,   // bf16 h^T of the next chunk staged (256)
    G_HM_READY = 16,  // fp32 state re-scaled by the next chunk's decay (256)
    G_O_FULL = 17,    // [2] O^T MMAs of a chunk done (and Q', P read), per O buffer
    G_O_FREE = 19,    // [2] O^T buffer read by the output warps (128)
    G_DRAIN = 21,     // final commit of the MMA issuer
};

// TMEM columns.  The O^T accumulators are double-buffered by chunk parity: the next chunk's O^T MMAs do not wait
// for the output warps to read the previous chunk's.
constexpr uint32_t T2_U = 0, T2_UF = 64, T2_H = 256, T2_COLS = 512;
__device__ __forceinline__ uint32_t t2_o1(int c) { return (c & 1) ? 384u : 128u; }
__device__ __forceinline__ uint32_t t2_o2(int c) { return (c & 1) ? 448u : 192u; }

// One CTA per (sequence n, head h, block of 128 value columns).  Warp roles: 0 loads (TMA of V, bulk copies of
// the workspace units); 2 issues every MMA; 4-7 form w . V and store o; 8-15 (two state warpgroups) split U,
// refresh the bf16 copy of h^T, re-scale the fp32 state by the next chunk's per-channel decay and write hT;
// 1 and 3 idle.  All waits are bounded (time-out: error word, drain, exit).
template <bool O_F32>
__global__ void __launch_bounds__(kTcThreads, 1)
gdn2_tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w, const FwdParams p,
                   const uint8_t* ws, unsigned* err) {
    using namespace sm100;
    using L = G2Smem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 16);

    auto drain_wait = [&](uint64_t* bar, uint32_t parity) {
        const long long t0 = clock64();
        while (!mbar_try_wait(bar, parity))
            if (clock64() - t0 > kWaitLimitCycles) {
                atomicOr(err, kErrTimeout);
                break;
            }
    };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = p.dv / kTcDV;
    const int tile = blockIdx.x % n_tiles;
    const int h = (blockIdx.x / n_tiles) % p.H;
    const int n = blockIdx.x / (n_tiles * p.H);
    const int H = p.H, dv = p.dv, T = p.T;
    const int j0 = tile * kTcDV;

    int row, bos, eos;
    if (!tc_seq_bounds(p, n, row, bos, eos, err)) return;
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    const size_t state_base = ((size_t)n * H + h) * kTcDK * (size_t)dv + j0;
    const long long seq_start = (long long)row * T + bos;
    auto unit = [&](int c) { return ws + ((size_t)wy_slot(n, seq_start, c) * H + h) * G2Unit::BYTES; };

    if (nc == 0) {  // empty sequence: hT = h0
        if (p.hT)
            for (int e = tid; e < kTcDK * kTcDV; e += kTcThreads) {
                const int i = e / kTcDV, j = e % kTcDV;
                p.hT[state_base + (size_t)i * dv + j] = p.h0 ? p.h0[state_base + (size_t)i * dv + j] : 0.f;
            }
        return;
    }

    if (tid == 0) {
        for (int b = 0; b < (int)L::N_BARS; ++b) {
            uint32_t cnt = 1;
            if (b == G_U_CONV || b == G_U_RND || b == G_H_READY || b == G_HM_READY) cnt = 256;
            if (b == G_VW_FULL || b == G_O_FREE || b == G_O_FREE + 1) cnt = 128;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_v);
        if (!p.kda) prefetch_tensormap(&tm_w);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, T2_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sbase = smem_u32(sm);

    if (warp == 0) {
        // ================================================================ loads
        // iteration c issues the loads of chunk c + 1, each once the MMA of chunk c that read its buffer is done
        // (V and w once the U~ MMA has read w . V: it comes after the w . V of chunk c consumed them)
        int n_tw = 0, n_vr = 0, n_wt = 0, n_kt = 0, n_qp = 0, n_lam[2] = {0, 0};
        for (int c = -1; c < nc - 1; ++c) {
            const int c1 = c + 1;
            const uint8_t* u = unit(c1);
            const int tok = (int)(seq_start + (long long)c1 * kChunk);
            if (c >= 0 && !warp_wait(&bars[G_UT_DONE], c & 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_expect_tx(&bars[G_TW_FULL], 16384);
                bulk_load(sm + L::TW, u + G2Unit::TH, 16384, &bars[G_TW_FULL]);
                mbar_expect_tx(&bars[G_LAM_FULL + (c1 & 1)], 512);
                bulk_load(sm + L::LAM + (c1 & 1) * 512, u + G2Unit::LAM, 512, &bars[G_LAM_FULL + (c1 & 1)]);
            }
            n_tw++;
            n_lam[c1 & 1]++;
            if (lane == 0) {
                mbar_expect_tx(&bars[G_VR_FULL], p.kda ? 16384u : 49152u);
                tma_load_3d(sm + L::VH, &tm_v, &bars[G_VR_FULL], j0, h, tok);
                tma_load_3d(sm + L::VH + 8192, &tm_v, &bars[G_VR_FULL], j0 + 64, h, tok);
                if (!p.kda) tma_load_3d(sm + L::W32, &tm_w, &bars[G_VR_FULL], j0, h, tok);
            }
            n_vr++;
            if (c >= 0 && !warp_wait(&bars[G_U_FULL], c & 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_expect_tx(&bars[G_WT_FULL], 16384);
                bulk_load(sm + L::WT, u + G2Unit::WT, 16384, &bars[G_WT_FULL]);
            }
            n_wt++;
            if (c >= 0 && !warp_wait(&bars[G_H_FULL], c & 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_expect_tx(&bars[G_KT_FULL], 16384);
                bulk_load(sm + L::KT, u + G2Unit::KT, 16384, &bars[G_KT_FULL]);
            }
            n_kt++;
            if (c >= 0 && !warp_wait(&bars[G_O_FULL + (c & 1)], (c >> 1) & 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_expect_tx(&bars[G_QP_FULL], 16384);
                bulk_load(sm + L::QP, u + G2Unit::QP, 16384, &bars[G_QP_FULL]);
                mbar_expect_tx(&bars[G_P_FULL], 16384);
                bulk_load(sm + L::P, u + G2Unit::PH, 16384, &bars[G_P_FULL]);
                if (c1 + 1 < nc) {  // the next chunk's unit, V and w into L2
                    bulk_prefetch_l2(unit(c1 + 1), G2Unit::BYTES);
                    tma_prefetch_3d(&tm_v, j0, h, tok + kChunk);
                    tma_prefetch_3d(&tm_v, j0 + 64, h, tok + kChunk);
                    if (!p.kda) tma_prefetch_3d(&tm_w, j0, h, tok + kChunk);
                }
            }
            n_qp++;
        }
        // drain: every load this warp issued completes before the CTA may exit
        if (n_tw > 0) drain_wait(&bars[G_TW_FULL], (n_tw - 1) & 1);
        if (n_vr > 0) drain_wait(&bars[G_VR_FULL], (n_vr - 1) & 1);
        if (n_wt > 0) drain_wait(&bars[G_WT_FULL], (n_wt - 1) & 1);
        if (n_kt > 0) drain_wait(&bars[G_KT_FULL], (n_kt - 1) & 1);
        if (n_qp > 0) {
            drain_wait(&bars[G_QP_FULL], (n_qp - 1) & 1);
            drain_wait(&bars[G_P_FULL], (n_qp - 1) & 1);
        }
        for (int sl = 0; sl < 2; ++sl)
            if (n_lam[sl] > 0) drain_wait(&bars[G_LAM_FULL + sl], (n_lam[sl] - 1) & 1);
    } else if (warp == 2) {
        // ================================================================ every MMA, in chunk order
        if (lane == 0) {
            const uint32_t id_ut = idesc_bf16(128, 64, true, false);
            const uint32_t id_u2 = idesc_bf16(128, 64, false, true);
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_h = idesc_bf16(128, 128, false, true);
            const uint32_t id_o2 = idesc_tf32(128, 64, false, false);
            const uint32_t n16 = 2u << 17;  // N += 16 in an instruction descriptor
            const uint64_t d_vh = desc_mn_sw128(sbase + L::VH, 8192);
            const uint64_t d_vl = desc_mn_sw128(sbase + L::VL, 8192);
            const uint64_t d_t = desc_k_sw128(sbase + L::TW);
            const uint64_t d_wt = desc_mn_sw128(sbase + L::WT, 8192);
            const uint64_t d_kt = desc_mn_sw128(sbase + L::KT, 8192);
            const uint64_t d_qp = desc_k_sw128(sbase + L::QP);
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1;
                const uint64_t d_ht = desc_k_sw128(sbase + L::HT + st * L::HT_STAGE);
                if (!mbar_wait(&bars[G_VW_FULL], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[G_TW_FULL], c & 1, abort_flag, err)) break;
                tc_fence_after();
                // U~^T = (w.V)^T T^T as hi.hi + hi.lo + lo.hi; T is lower triangular, so k-step ks (tokens
                // s in [16 ks, 16 ks + 16)) updates only the columns r >= 16 ks
#pragma unroll
                for (int pass = 0; pass < 3; ++pass) {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma_bf16(tmem + T2_U + 16 * ks, (pass == 2 ? d_vl : d_vh) + ks * 128,
                                  d_t + (pass == 1 ? 512 : 0) + ks * 130, id_ut - ks * n16, (pass | ks) != 0);
                }
                umma_commit(&bars[G_UT_DONE]);
                // U^T -= h^T W^T
                if (!mbar_wait(&bars[G_WT_FULL], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[G_H_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + T2_U, d_ht + (kk >> 2) * 1024 + (kk & 3) * 2, d_wt + kk * 128, id_u2, 1);
                umma_commit(&bars[G_U_FULL]);
                // h^T += U^T K~  (U as bf16 hi and lo halves from TMEM)
                if (!mbar_wait(&bars[G_U_CONV], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[G_HM_READY], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[G_KT_FULL], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int ks = kk & 3;
                    const uint32_t a = tmem + T2_UF + (ks >> 1) * 32 + (kk >> 2) * 16 + (ks & 1) * 8;
                    umma_bf16_tmem_a(tmem + T2_H, a, d_kt + ks * 128, id_h, 1);
                }
                umma_commit(&bars[G_H_FULL]);
                // O1^T = h^T Q'^T, into the O buffer of this chunk's parity (read out two chunks ago)
                if (c >= 2 && !mbar_wait(&bars[G_O_FREE + st], ((c - 2) >> 1) & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[G_QP_FULL], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + t2_o1(c), d_ht + (kk >> 2) * 1024 + (kk & 3) * 2,
                              d_qp + (kk >> 2) * 512 + (kk & 3) * 2, id_o, kk > 0);
                // O2^T = U^T P^T on kind::tf32 (P lower triangular: k-step ks8 of 8 tokens reaches r >= 16 (ks8/2))
                if (!mbar_wait(&bars[G_P_FULL], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[G_U_RND], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int ks8 = 0; ks8 < 8; ++ks8) {
                    const int r0 = 16 * (ks8 >> 1);
                    const uint64_t b = desc_k_sw128(sbase + L::P + ((ks8 & 4) ? 8192 : 0)) +
                                       ((r0 * 128 + (ks8 & 3) * 32) >> 4);
                    umma_tf32_tmem_a(tmem + t2_o2(c) + r0, tmem + T2_U + 8 * ks8, b, id_o2 - (r0 >> 4) * n16, ks8 > 0);
                }
                umma_commit(&bars[G_O_FULL + st]);
            }
            umma_commit(&bars[G_DRAIN]);
            drain_wait(&bars[G_DRAIN], 0);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 3) {
        // idle
    } else if (warp < 8) {
        // ================================================================ w . V and the output
        // Iteration k: w . V of chunk k (from the V tile and w, as a bf16 hi + lo pair), then the output tile of
        // chunk k - 1 from TMEM, one token row per store.  A timed-out wait does not break out: the warp finishes
        // the iteration and leaves at the top of the next.
        const int t = tid - 128;
        const uint32_t lane_base = 32 * (warp & 3);
        const size_t ostride = (size_t)H * dv;
        for (int k = 0; k <= nc; ++k) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (k < nc) {
                const int c = k;
                const int Lc = min(kChunk, eos - bos - c * kChunk);
                const size_t tok0 = (size_t)(seq_start + (long long)c * kChunk);
                // thread: 16-byte chunk cc (8 value columns) of rows s = 8 it + t / 16
                const int cc = t & 15, panel = cc >> 3;
                float kda_beta[8];
                if (p.kda) {  // issued before the wait, so the loads overlap it
#pragma unroll
                    for (int it = 0; it < 8; ++it) {
                        const int s = 8 * it + (t >> 4);
                        kda_beta[it] = s < Lc ? p.beta[(tok0 + s) * H + h] : 0.f;
                    }
                }
                warp_wait(&bars[G_VR_FULL], c & 1, abort_flag, err);
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int s = 8 * it + (t >> 4);
                    const uint32_t off = panel * 8192u + sw128(s, cc & 7);
                    const uint4 vv = *reinterpret_cast<const uint4*>(sm + L::VH + off);
                    float wv[8];
                    if (s >= Lc) {  // rows of the next sequence, or TMA zero fill
#pragma unroll
                        for (int e = 0; e < 8; ++e) wv[e] = 0.f;
                    } else if (p.kda) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) wv[e] = kda_beta[it];
                    } else {
                        const float4* wp = reinterpret_cast<const float4*>(sm + L::W32 + s * 512 + 32 * cc);
                        const float4 w0 = wp[0], w1 = wp[1];
                        wv[0] = w0.x, wv[1] = w0.y, wv[2] = w0.z, wv[3] = w0.w;
                        wv[4] = w1.x, wv[5] = w1.y, wv[6] = w1.z, wv[7] = w1.w;
                    }
                    const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vw[e2]));
                        split_pack_bf16(x.x * wv[2 * e2], x.y * wv[2 * e2 + 1], hi[e2], lo[e2]);
                    }
                    *reinterpret_cast<uint4*>(sm + L::VH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4*>(sm + L::VL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
                fence_proxy_async();
                mbar_arrive(&bars[G_VW_FULL]);
            }
            if (k >= 1) {
                const int c = k - 1;
                const int Lc = min(kChunk, eos - bos - c * kChunk);
                warp_wait(&bars[G_O_FULL + (c & 1)], (c >> 1) & 1, abort_flag, err);
                tc_fence_after();
                const size_t tok0 = (size_t)(seq_start + (long long)c * kChunk);
                size_t off = (tok0 * H + h) * (size_t)dv + j0 + t;
#pragma unroll 1
                for (int r8 = 0; r8 < 64; r8 += 8) {
                    float v1[8], v2[8];
                    tmem_ld8(taddr(tmem, lane_base, t2_o1(c) + r8), v1);
                    tmem_ld8(taddr(tmem, lane_base, t2_o2(c) + r8), v2);
                    tmem_wait_ld();
                    if (r8 == 56) {
                        tc_fence_before();
                        mbar_arrive(&bars[G_O_FREE + (c & 1)]);
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float val = p.scale * (v1[q] + v2[q]);
                        if (r8 + q < Lc && p.o) {  // o is null when only the chunk states are wanted
                            if (O_F32) static_cast<float*>(p.o)[off] = val;
                            else static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(val);
                        }
                        off += ostride;
                    }
                }
            }
        }
    } else {
        // ================================================================ state warpgroups
        // Warpgroups 8-11 (half 0) and 12-15 (half 1): each splits half of U (tokens [32 half, 32 half + 32))
        // and refreshes half of the state (key channels [64 half, 64 half + 64)).
        const int half = (warp - 8) >> 2;
        const int j = tid & 127;
        const uint32_t lane_base = 32 * (warp & 3);
        const float* lam = reinterpret_cast<const float*>(sm + L::LAM);
        // backward pass only: the state at the start of chunk c, key channels [32 piece, 32 piece + 32)
        auto dump_state = [&](int c, int piece, const float(&v)[32]) {
            float* hp = p.h_chunks + ((size_t)wy_slot(n, seq_start, c) * H + h) * kTcDK * (size_t)dv + j0 +
                        (size_t)(32 * piece) * dv + j;
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                *hp = v[q];
                hp += dv;
            }
        };
        // initial state: bf16 copy and fp32 master pre-scaled by the first chunk's per-channel decay
        if (warp_wait(&bars[G_LAM_FULL + 0], 0, abort_flag, err)) {
#pragma unroll 1
            for (int piece = 2 * half; piece < 2 * half + 2; ++piece) {
                float v[32];
                const float* hp = p.h0 ? p.h0 + state_base + (size_t)(32 * piece) * dv + j : nullptr;
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    v[q] = hp ? *hp : 0.f;
                    hp += hp ? dv : 0;
                }
                if (p.h_chunks) dump_state(0, piece, v);
                st_half_line_bf16(sm + L::HT + (piece >> 1) * 16384, j, 4 * (piece & 1), v);
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] *= lam[32 * piece + q];
                tmem_st32(taddr(tmem, lane_base, T2_H + 32 * piece), v);
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bars[G_H_READY]);
            mbar_arrive(&bars[G_HM_READY]);
        }
        for (int c = 0; c < nc; ++c) {
            // ---- U as bf16 hi / lo pairs for the h^T MMA (to T2_UF: [hi | lo], 16 columns each per half), then
            // U itself rounded to tf32 in place for the kind::tf32 O2 MMA
            if (!warp_wait(&bars[G_U_FULL], c & 1, abort_flag, err)) break;
            tc_fence_after();
            {
                float u[32];
                tmem_ld32(taddr(tmem, lane_base, T2_U + 32 * half), u);
                tmem_wait_ld();
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) split_pack_bf16(u[2 * q], u[2 * q + 1], hi[q], lo[q]);
                tmem_st16u(taddr(tmem, lane_base, T2_UF + 32 * half), hi);
                tmem_st16u(taddr(tmem, lane_base, T2_UF + 32 * half + 16), lo);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[G_U_CONV]);
                uint32_t ur[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) ur[q] = f2tf32(u[q]);
                tmem_st32u(taddr(tmem, lane_base, T2_U + 32 * half), ur);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[G_U_RND]);
            // ---- state refresh (key channels of this half)
            if (!warp_wait(&bars[G_H_FULL], c & 1, abort_flag, err)) break;
            const bool last = c + 1 == nc;
            const int c1 = c + 1;
            if (!last && !warp_wait(&bars[G_LAM_FULL + (c1 & 1)], (c1 >> 1) & 1, abort_flag, err)) break;
            tc_fence_after();
#pragma unroll 1
            for (int piece = 2 * half; piece < 2 * half + 2; ++piece) {
                float v[32];
                tmem_ld32(taddr(tmem, lane_base, T2_H + 32 * piece), v);
                tmem_wait_ld();
                if (!last) {
                    st_half_line_bf16(sm + L::HT + (c1 & 1) * L::HT_STAGE + (piece >> 1) * 16384, j, 4 * (piece & 1),
                                      v);
                    if (p.h_chunks) dump_state(c1, piece, v);
                } else if (p.hT) {
                    float* hp = p.hT + state_base + (size_t)(32 * piece) * dv + j;
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        *hp = v[q];
                        hp += dv;
                    }
                }
            }
            if (!last) {
                fence_proxy_async();
                mbar_arrive(&bars[G_H_READY]);
                const float* lam_n = lam + (c1 & 1) * 128;
#pragma unroll 1
                for (int piece = 2 * half; piece < 2 * half + 2; ++piece) {
                    float v[32];
                    tmem_ld32(taddr(tmem, lane_base, T2_H + 32 * piece), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] *= lam_n[32 * piece + q];
                    tmem_st32(taddr(tmem, lane_base, T2_H + 32 * piece), v);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[G_HM_READY]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, T2_COLS);
    }
}

// ------------------------------------------------------------------------------------------ host side
// 3-D map over a [rows, H, d] fp32 tensor (d innermost), box box_d x 1 x 64, no swizzle (rows of box_d * 4 bytes).
inline bool make_map_f32(CUtensorMap* map, const void* base, int d, int H, long long rows, int box_d) {
    PFN_encodeTiled enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)d * H * 4};
    const cuuint32_t box[3] = {(cuuint32_t)box_d, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool tc2_supported(const FwdParams& p) { return p.dk == kTcDK && p.dv % kTcDV == 0 && p.T > 0; }

inline gdn_status launch_tc2(const FwdParams& p, bool o_f32, void* ws, size_t ws_bytes, unsigned* err,
                             cudaStream_t stream) {
    const size_t need = tc2_workspace_bytes(p.B, p.T, p.H, p.n_seq);
    if (!ws || ws_bytes < need) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "the tcgen05 GDN-2 path needs %zu bytes of workspace (got %zu)", need,
                 ws_bytes);
        return GDN_ERR_UNSUPPORTED;
    }
    CUtensorMap mq, mk, mv, mg, mb, mw;
    const long long rows = (long long)p.B * p.T;
    bool maps = make_map(&mq, p.q, p.dk, p.H, rows) && make_map(&mk, p.k, p.dk, p.H, rows) &&
                make_map(&mv, p.v, p.dv, p.H, rows) && make_map_f32(&mg, p.g, p.dk, p.H, rows, 128);
    // KDA reads its scalar beta directly; the maps of b and w are then unused (encoded over g as placeholders)
    maps = maps && make_map_f32(&mb, p.kda ? p.g : p.beta, p.dk, p.H, rows, 128) &&
           make_map_f32(&mw, p.kda ? p.g : p.w, p.kda ? p.dk : p.dv, p.H, rows, 128);
    if (!maps) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cuTensorMapEncodeTiled failed");
        return GDN_ERR_CUDA;
    }
    const long long prep_grid = (long long)wy_slots(p.B, p.T, p.n_seq) * p.H;
    if (prep_grid > 0x7fffffffLL) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "too many chunks for one launch");
        return GDN_ERR_UNSUPPORTED;
    }
    cudaError_t e = cudaFuncSetAttribute(gdn2_tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G2PrepSmem::ALLOC);
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    ProfScope prof_prep(PK_TC2_PREP, stream);
    gdn2_tc_prep_kernel<<<(unsigned)prep_grid, kG2Threads, G2PrepSmem::ALLOC, stream>>>(mq, mk, mg, mb, p,
                                                                                       static_cast<uint8_t*>(ws), err);
    prof_prep.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "GDN-2 prep kernel: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    auto kern = o_f32 ? gdn2_tc_fwd_kernel<true> : gdn2_tc_fwd_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G2Smem::ALLOC);
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    const unsigned grid = (unsigned)(p.dv / kTcDV) * p.H * p.n_seq;
    ProfScope prof_main(PK_TC2_MAIN, stream);
    kern<<<grid, kTcThreads, G2Smem::ALLOC, stream>>>(mv, mw, p, static_cast<const uint8_t*>(ws), err);
    prof_main.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "GDN-2 chunk kernel: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

}  // namespace gdn
