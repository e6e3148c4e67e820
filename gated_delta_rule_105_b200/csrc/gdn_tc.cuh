// tcgen05 (5th-generation tensor core) chunked forward of the gated delta rule, bf16 inputs: two kernels.
//
// Per chunk of C = 64 tokens (r, s = token rows; G = chunk-local cumulative gate in base 2;
// f_s = 2^(G_last - G_s)):
//   A   = strict_lower(beta_r 2^(G_r - G_s) k_r . k_s) ;  T = (I + A)^-1
//   T'  = T diag(beta 2^G) ;  T'' = T diag(beta)
//   W   = T' K ;  U = T'' V - W h                  (the corrected values)
//   P   = lower(2^(G_r - G_s) q_r . k_s)
//   O   = scale (diag(2^G) Q h + P U)              (read-out)
//   h  <- 2^(G_last) h + K^T diag(f) U
// This is the WY form of the intra-chunk dependency with one state handed from chunk to chunk
// (GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755, section "Chunked parallelism").
//
// The WY kernel (gdn_tc_wy_kernel) computes, for every (chunk, head) at once, A from K K^T, the inverse and
// T', T'' (T'' as a bf16 hi + lo pair), and P from Q K^T, and writes them to the workspace in the exact
// shared-memory form the MMAs read (40 KB per chunk and head).  Nothing in it depends on the state, so it runs
// fully parallel.
// The main kernel (gdn_tc_fwd_kernel) then walks each sequence's chunks: one CTA owns one (sequence n,
// head h, block of 128 value columns j); the state is kept transposed, h^T [j][i] (value column j on the 128
// TMEM lanes, key channel i on 128 columns), fp32 in TMEM for the whole sequence.  Every contraction is an
// M = 128 tcgen05.mma with bf16 operands in 128B-swizzled shared memory (or U in TMEM) and an fp32
// accumulator in TMEM.
// Precision: every bf16 operand whose rounding would reach the output at the bf16-ulp level is avoided or
// split.  U diag f (in TMEM, as the A operand of the h^T MMA) and T'' are bf16 hi + lo pairs; the read-out
// product U^T P^T runs on kind::tf32 with U rounded to tf32 in TMEM and P stored as tf32; 2^G_r is
// applied to the fp32 accumulator of h^T Q^T instead of to Q.  The remaining bf16 operands are h^T, W^T,
// T' and the inputs themselves.
// The operands T', T'' and P are lower triangular: the MMAs that read them skip the blocks above the
// diagonal (k-step ks of 16 tokens only reaches the output columns r >= 16 ks).
// All mbarrier waits are bounded: on time-out the CTA sets the error word and drains to the exit.
#pragma once

#include <cuda.h>

#include "gdn_sm100.cuh"

namespace gdn {

constexpr int kTcThreads = 512;  // main kernel: 16 warps
constexpr int kWyThreads = 128;  // WY kernel: one warpgroup
constexpr int kTcDV = 128;       // value columns per CTA
constexpr int kTcDK = 128;       // key dimension handled by these kernels
// workspace bytes per (chunk, head): T' | T''_hi | T''_lo (bf16 [r][s]) | P columns 0-31 | P columns 32-63
// (tf32 [r][s]), 8 KB each, every piece in the 128B-swizzled K-major form the chunk kernel's MMAs read
constexpr uint32_t kWyUnit = 40960;
constexpr uint32_t kWyP = 24576;  // offset of P in a unit

struct TcGate {  // one chunk's gate data
    float G[64];     // log2(e) * chunk-local cumulative g
    float beta[64];  // beta (0 past the end of the sequence)
    float f[64];     // 2^(G_last - G_s)
    float eG[64];    // 2^(G_r)
    float a[64];     // 2^(log2(e) g_r) = exp(g_r), the token's own decay (1 past the end of the sequence)
    float gamma;     // 2^(G_last)
    int L;           // valid rows in this chunk
    int pad[2];
};
static_assert(sizeof(TcGate) % 16 == 0, "gate stage size");


// One chunk's gates, by one warp (lane l: tokens 2l, 2l+1).  tok0 = global token index of row 0.
__device__ __forceinline__ void tc_make_gates(TcGate& gs, const FwdParams& p, size_t tok0, int Lc, int h, int lane) {
    using namespace sm100;
    float gv[2], bv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int r = 2 * lane + u;
        const size_t tok = (tok0 + r) * p.H + h;
        gv[u] = r < Lc ? p.g[tok] : 0.f;
        bv[u] = r < Lc ? p.beta[tok] : 0.f;
    }
    const float pair = gv[0] + gv[1];
    float incl = pair;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += y;
    }
    const float excl = incl - pair;
    const float G0 = (excl + gv[0]) * kLog2e, G1 = incl * kLog2e;
    const float Glast = __shfl_sync(0xffffffffu, G1, 31);
    gs.G[2 * lane] = G0;
    gs.G[2 * lane + 1] = G1;
    gs.beta[2 * lane] = bv[0];
    gs.beta[2 * lane + 1] = bv[1];
    gs.f[2 * lane] = ex2_approx(Glast - G0);
    gs.f[2 * lane + 1] = ex2_approx(Glast - G1);
    gs.eG[2 * lane] = ex2_approx(G0);
    gs.eG[2 * lane + 1] = ex2_approx(G1);
    gs.a[2 * lane] = ex2_approx(gv[0] * kLog2e);
    gs.a[2 * lane + 1] = ex2_approx(gv[1] * kLog2e);
    if (lane == 0) {
        gs.gamma = ex2_approx(Glast);
        gs.L = Lc;
    }
}

// fp32 -> tf32 (round to nearest, ties away), returned as the fp32 bit pattern with the low 13 bits clear.
__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// One row r of A (IS_A: beta_r Gamma_rs (k_r . k_s), s < r, fp32 into `arow`) or of P (Gamma_rs (q_r . k_s),
// s <= r, rounded to tf32 and stored as fp32 in the 128B-swizzled K-major layout of a kind::tf32 operand:
// columns 0-31 in `ph`, 32-63 in `pl`, in shared or global memory), columns [s_lo, s_hi], from the dot products
// in TMEM (`ta` = this warp's lanes, column of s = 0).  Gamma_rs = 2^(G_r - G_s) = a_r a_(r-1) ... a_(s+1) is a
// running product down from the highest column at or below r, started there with one exp2.
template <bool IS_A>
__device__ __forceinline__ void tc_row_pass(uint32_t ta, const TcGate& gs, int r, int s_lo, int s_hi, float* arow,
                                            uint8_t* ph, uint8_t* pl) {
    using namespace sm100;
    const int top = r < s_hi ? r : s_hi;
    float run = (top == r) ? 1.f : ex2_approx(gs.G[r] - gs.G[top]);
    const float br = IS_A ? gs.beta[r] : 1.f;
#pragma unroll 1
    for (int c8 = s_hi - 7; c8 >= s_lo; c8 -= 8) {
        float s8[8];
        tmem_ld8(ta + c8, s8);
        tmem_wait_ld();
        float x[8];
#pragma unroll
        for (int q = 7; q >= 0; --q) {
            const int s = c8 + q;
            x[q] = (IS_A ? (s < r) : (s <= r)) ? br * run * s8[q] : 0.f;
            if (s <= top && s > 0) run *= gs.a[s];
        }
        if (IS_A) {
            *reinterpret_cast<float4*>(arow + c8) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(arow + c8 + 4) = make_float4(x[4], x[5], x[6], x[7]);
        } else {
            uint8_t* panel = (c8 & 32) ? pl : ph;
            const uint32_t ch = (c8 & 31) >> 2;  // 16-byte chunk of 4 fp32
            *reinterpret_cast<uint4*>(panel + sw128(r, ch)) =
                make_uint4(f2tf32(x[0]), f2tf32(x[1]), f2tf32(x[2]), f2tf32(x[3]));
            *reinterpret_cast<uint4*>(panel + sw128(r, ch + 1)) =
                make_uint4(f2tf32(x[4]), f2tf32(x[5]), f2tf32(x[6]), f2tf32(x[7]));
        }
    }
}

// ------------------------------------------------------------------------------------------ the inverse
constexpr int kAsLd = 68;  // row stride (floats) of the [64][68] fp32 scratch holding A, then T

// D(16x8) += A(16x8) B(8x8), tf32 inputs, fp32 accumulate (legacy warp-level MMA, used only for the
// 16x16 blocks of the triangular inverse).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// 16x16 blocks of the scratch, as tf32 mma.sync fragments.  A block is named by its logical origin (r0, c0);
// `tr` = it is stored transposed in the mirrored position (element (r, c) of the logical block at scratch
// row c0 + c, column r0 + r).
struct Frag16 {
    uint32_t a[2][4];  // as the A operand: k-halves 0, 1
};
__device__ __forceinline__ float blk(const float* S, int r0, int c0, int r, int c, bool tr) {
    return tr ? S[(c0 + c) * kAsLd + r0 + r] : S[(r0 + r) * kAsLd + c0 + c];
}
__device__ __forceinline__ void load_a16(const float* S, int r0, int c0, bool tr, int lane, Frag16& f) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
        f.a[kh][0] = f2tf32(blk(S, r0, c0, g, 8 * kh + t, tr));
        f.a[kh][1] = f2tf32(blk(S, r0, c0, g + 8, 8 * kh + t, tr));
        f.a[kh][2] = f2tf32(blk(S, r0, c0, g, 8 * kh + t + 4, tr));
        f.a[kh][3] = f2tf32(blk(S, r0, c0, g + 8, 8 * kh + t + 4, tr));
    }
}
// acc (16x16 as two 16x8 n-halves) += A-frag(16x16) * B (16x16 block (r0, c0), transposed if tr).
__device__ __forceinline__ void mma16(float (&acc)[2][4], const Frag16& A, const float* S, int r0, int c0, bool tr,
                                      int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            uint32_t b[2];
            b[0] = f2tf32(blk(S, r0, c0, 8 * kh + t, 8 * nh + g, tr));
            b[1] = f2tf32(blk(S, r0, c0, 8 * kh + t + 4, 8 * nh + g, tr));
            mma_tf32(acc[nh], A.a[kh], b);
        }
    }
}
// Stores sgn * acc into the 16x16 block (r0, c0), transposed if tr.
__device__ __forceinline__ void store16(float* S, int r0, int c0, bool tr, int lane, const float (&acc)[2][4],
                                        float sgn) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int c = 8 * nh + 2 * t;
        float* p00 = tr ? &S[(c0 + c) * kAsLd + r0 + g] : &S[(r0 + g) * kAsLd + c0 + c];
        const int dc = tr ? kAsLd : 1, dr = tr ? 1 : kAsLd;
        p00[0] = sgn * acc[nh][0];
        p00[dc] = sgn * acc[nh][1];
        p00[8 * dr] = sgn * acc[nh][2];
        p00[8 * dr + dc] = sgn * acc[nh][3];
    }
}

// Where the blocks of T go once final.  An emitter receives elements of T itself: elem(r, s, x) one element,
// pair(r, s, x0, x1) the elements (r, s) and (r, s + 1), s even.  Every output is [r][s] K-major with 128-byte
// swizzle; only the blocks on and below the diagonal are written (the MMAs that read these operands skip the
// zero blocks above it).
// GDN: T' = T diag(beta 2^G) as bf16, and T'' = T diag(beta) as a bf16 hi + lo pair.
struct TEmit {
    uint8_t* tp;
    uint8_t* tpp;
    uint8_t* tppl;
    const float* beta;
    const float* eG;
    __device__ __forceinline__ void elem(int r, int s, float t) const {
        using namespace sm100;
        const float x = t * beta[s];
        const uint32_t off = sw128(r, s >> 3) + (s & 7) * 2;
        const __nv_bfloat16 xh = __float2bfloat16_rn(x);
        *reinterpret_cast<__nv_bfloat16*>(tp + off) = __float2bfloat16_rn(x * eG[s]);
        *reinterpret_cast<__nv_bfloat16*>(tpp + off) = xh;
        *reinterpret_cast<__nv_bfloat16*>(tppl + off) = __float2bfloat16_rn(x - __bfloat162float(xh));
    }
    __device__ __forceinline__ void pair(int r, int s, float t0, float t1) const {
        using namespace sm100;
        const float x0 = t0 * beta[s], x1 = t1 * beta[s + 1];
        const uint32_t off = sw128(r, s >> 3) + (s & 7) * 2;
        uint32_t hi, lo;
        split_pack_bf16(x0, x1, hi, lo);
        *reinterpret_cast<uint32_t*>(tp + off) = pack_bf16(x0 * eG[s], x1 * eG[s + 1]);
        *reinterpret_cast<uint32_t*>(tpp + off) = hi;
        *reinterpret_cast<uint32_t*>(tppl + off) = lo;
    }
};
// GDN-2: T itself as a bf16 hi + lo pair (the gates do not factor out of T).
struct TEmitPlain {
    uint8_t* th;
    uint8_t* tl;
    __device__ __forceinline__ void elem(int r, int s, float x) const {
        using namespace sm100;
        const uint32_t off = sw128(r, s >> 3) + (s & 7) * 2;
        const __nv_bfloat16 xh = __float2bfloat16_rn(x);
        *reinterpret_cast<__nv_bfloat16*>(th + off) = xh;
        *reinterpret_cast<__nv_bfloat16*>(tl + off) = __float2bfloat16_rn(x - __bfloat162float(xh));
    }
    __device__ __forceinline__ void pair(int r, int s, float x0, float x1) const {
        using namespace sm100;
        const uint32_t off = sw128(r, s >> 3) + (s & 7) * 2;
        uint32_t hi, lo;
        split_pack_bf16(x0, x1, hi, lo);
        *reinterpret_cast<uint32_t*>(th + off) = hi;
        *reinterpret_cast<uint32_t*>(tl + off) = lo;
    }
};
// Emits sgn * acc, the final 16x16 block (r0, c0) of T held as an mma.sync accumulator.
template <class Emit>
__device__ __forceinline__ void emit16(const Emit& em, int r0, int c0, int lane, const float (&acc)[2][4], float sgn) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int s = c0 + 8 * nh + 2 * t;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) em.pair(r0 + g + 8 * hr, s, sgn * acc[nh][2 * hr], sgn * acc[nh][2 * hr + 1]);
    }
}

// (I + A)^-1 for a strictly lower-triangular 64x64 A in the [64][68] fp32 scratch (upper triangle 0), by
// the 4 warps of one warpgroup; every block of T = (I + A)^-1 is emitted (TEmit) as soon as it is final.
// Steps: the four diagonal 16x16 blocks by forward substitution (one column per lane), left in place for
// the later steps; T_10 = -T_11 A_10 T_00 and T_32 = -T_33 A_32 T_22, stored transposed in the upper
// blocks (0, 1) and (2, 3); then the lower-left 32x32 quarter T_c = -T_b (A_c T_a), where T_a, T_b are
// the inverses of the two diagonal 32x32 quarters, with A_c T_a parked transposed in the upper blocks
// (q, p).  Each block product runs on tf32 MMAs, at most two per warp per step.  The lower off-diagonal
// blocks of A are left intact.  The code is unrolled: it is one chain of dependent shared-memory loads and
// MMAs, which only unrolling lets the compiler overlap.
template <class Emit>
__device__ __forceinline__ void invert_unit_lower64(float* S, int wid, int lane, uint32_t bar_id, const Emit& em) {
    using namespace sm100;
    {
        const int b0 = 16 * wid, c = lane & 15;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == c) ? 1.f : 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s) acc = fmaf(-S[(b0 + r) * kAsLd + b0 + s], t[s], acc);
            t[r] = (r < c) ? 0.f : acc;
        }
        __syncwarp();
        if (lane < 16) {
#pragma unroll
            for (int r = 0; r < 16; ++r) S[(b0 + r) * kAsLd + b0 + c] = t[r];
        }
        // emit column c of T_ii: lanes 0-15 rows 0-7, lanes 16-31 rows 8-15
        const int s = b0 + c, hr = lane >> 4;
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) em.elem(b0 + 8 * hr + rr, s, hr ? t[8 + rr] : t[rr]);
    }
    named_bar_sync(bar_id, 128);
    // T_10 (warp 0) and T_32 (warp 1): X = A_ij T_jj, then T_ij = -T_ii X
    if (wid < 2) {
        const int i = 1 + 2 * wid, j = 2 * wid;
        Frag16 f;
        load_a16(S, 16 * i, 16 * j, false, lane, f);
        float x[2][4] = {};
        mma16(x, f, S, 16 * j, 16 * j, false, lane);
        store16(S, 16 * i, 16 * j, true, lane, x, 1.f);
        __syncwarp();
        load_a16(S, 16 * i, 16 * i, false, lane, f);
        float y[2][4] = {};
        mma16(y, f, S, 16 * i, 16 * j, true, lane);
        __syncwarp();
        store16(S, 16 * i, 16 * j, true, lane, y, -1.f);
        emit16(em, 16 * i, 16 * j, lane, y, -1.f);
    }
    named_bar_sync(bar_id, 128);
    // X = A_c T_a for the blocks (p, q), p in {2, 3}, q in {0, 1}; one block per warp, parked in (p, q)
    const int p = 2 + (wid >> 1), q = wid & 1;
    {
        Frag16 f;
        float x[2][4] = {};
        load_a16(S, 16 * p, 16 * q, false, lane, f);  // A_pq T_qq
        mma16(x, f, S, 16 * q, 16 * q, false, lane);
        if (q == 0) {  // + A_p1 T_10
            load_a16(S, 16 * p, 16, false, lane, f);
            mma16(x, f, S, 16, 0, true, lane);
        }
        store16(S, 16 * p, 16 * q, true, lane, x, 1.f);
    }
    named_bar_sync(bar_id, 128);
    // T_c = -T_b X: T_2q = -T_22 X_2q ; T_3q = -(T_32 X_2q + T_33 X_3q); emitted only (not needed in S)
    {
        Frag16 f;
        float y[2][4] = {};
        if (p == 2) {
            load_a16(S, 32, 32, false, lane, f);
            mma16(y, f, S, 32, 16 * q, true, lane);
        } else {
            load_a16(S, 48, 32, true, lane, f);
            mma16(y, f, S, 32, 16 * q, true, lane);
            load_a16(S, 48, 48, false, lane, f);
            mma16(y, f, S, 48, 16 * q, true, lane);
        }
        emit16(em, 16 * p, 16 * q, lane, y, -1.f);
    }
}

// Validated sequence bounds of sequence n: row in q/k/v, first token bos and end eos within the row.
// Returns false (and sets the error word) for a malformed cu_seqlens entry.
__device__ __forceinline__ bool tc_seq_bounds(const FwdParams& p, int n, int& row, int& bos, int& eos, unsigned* err) {
    if (p.cu_seqlens) {
        row = 0;
        bos = p.cu_seqlens[n];
        eos = p.cu_seqlens[n + 1];
        if (bos < 0 || eos < bos || eos > p.T) {
            atomicOr(err, kErrSeqlens);
            return false;
        }
    } else {
        row = n;
        bos = 0;
        eos = p.T;
    }
    return true;
}

// The (sequence, chunk) that workspace slot `slot` belongs to: the unit's first global token index
// (row * T + bos + 64 c) goes to *tok0 and its valid rows to *Lc, which stays 0 for a slot no chunk uses.
__device__ __forceinline__ void wy_unit_of_slot(const FwdParams& p, long long slot, int* tok0, int* Lc,
                                                unsigned* err) {
    // the sequence n whose slot range holds `slot`: largest n with wy_slot(n, start_n, 0) <= slot
    int lo = 0, hi = p.n_seq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const long long st0 = p.cu_seqlens ? (long long)p.cu_seqlens[mid] : (long long)mid * p.T;
        if (wy_slot(mid, st0, 0) <= slot) lo = mid;
        else hi = mid - 1;
    }
    int row, bos, eos, c = 0;
    *Lc = 0;
    if (tc_seq_bounds(p, lo, row, bos, eos, err)) {
        const long long start = (long long)row * p.T + bos;
        const long long cc = slot - wy_slot(lo, start, 0);
        if (cc >= 0 && cc * kChunk < eos - bos) {
            c = (int)cc;
            *Lc = min(kChunk, eos - bos - c * kChunk);
        }
        *tok0 = (int)(start + (long long)c * kChunk);
    }
}

// ------------------------------------------------------------------------------------------ the WY kernel
// Shared-memory map (bytes from a 1024-aligned base).  The S1 MMA reads a 128-row A operand per 64-channel
// panel, rows 0-63 the K tile and rows 64-127 the Q tile ([K0 | Q0 | K1 | Q1], as in the chunk kernel), and K
// as its B operand.  Once S1 is in TMEM the four panels are free: the inverse writes T''_lo over K0, T''_hi over
// Q0 and T' over K1 (the P rows go straight to the workspace).
struct WySmem {
    static constexpr uint32_t K0 = 0, Q0 = 8192, K1 = 16384, Q1 = 24576;  // [64 tokens][128 B] swizzled each
    static constexpr uint32_t TPPL = K0, TPP = Q0, TP = K1;
    static constexpr uint32_t AS = 32768;  // A, then (I+A)^-1, fp32 [64][68]
    static constexpr uint32_t GATE = AS + 64 * kAsLd * 4;
    static constexpr uint32_t BARS = GATE + sizeof(TcGate);  // [0] K, Q landed, [1] S1 done
    static constexpr uint32_t MISC = BARS + 16;              // tmem base, abort flag, unit info
    static constexpr uint32_t END = MISC + 64;
    static constexpr uint32_t ALLOC = END + 1024;  // 4 CTAs per SM
};

// One CTA per (workspace slot, head): finds the (sequence, chunk) of its slot, builds A and P from S1 = [K; Q] K^T,
// inverts I + A and writes T', T''_hi, T''_lo and P of that chunk to the workspace.
__global__ void __launch_bounds__(kWyThreads) gdn_tc_wy_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const FwdParams p, uint8_t* ws, unsigned* err) {
    using namespace sm100;
    using L = WySmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 16);
    int* info = reinterpret_cast<int*>(sm + L::MISC + 32);  // row, start token, chunk, valid rows
    TcGate& gs = *reinterpret_cast<TcGate*>(sm + L::GATE);
    float* sA = reinterpret_cast<float*>(sm + L::AS);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long slot = blockIdx.x / p.H;
    const int h = blockIdx.x % p.H;

    if (tid == 0) {
        int Lc = 0;
        wy_unit_of_slot(p, slot, &info[1], &Lc, err);
        info[2] = Lc;
        if (Lc > 0) {
            mbar_init(&bars[0], 1);
            mbar_init(&bars[1], 1);
            *abort_flag = 0;
            fence_barrier_init();
            mbar_expect_tx(&bars[0], 32768);
            tma_load_3d(sm + L::K0, &tm_k, &bars[0], 0, h, info[1]);
            tma_load_3d(sm + L::Q0, &tm_q, &bars[0], 0, h, info[1]);
            tma_load_3d(sm + L::K1, &tm_k, &bars[0], 64, h, info[1]);
            tma_load_3d(sm + L::Q1, &tm_q, &bars[0], 64, h, info[1]);
        }
    }
    __syncthreads();
    const int tok0 = info[1], Lc = info[2];
    if (Lc == 0) return;  // unused slot
    if (warp == 0) {
        tmem_alloc(tmem_slot, 64);
        tmem_relinquish();
    }
    if (warp == 1) tc_make_gates(gs, p, (size_t)tok0, Lc, h, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        // S1 = [K; Q] K^T: k-steps 0-3 read channel panels K0 | Q0, 4-7 panels K1 | Q1, 16 KB further
        if (mbar_wait(&bars[0], 0, abort_flag, err)) {
            tc_fence_after();
            const uint64_t d = desc_k_sw128(smem_u32(sm));
            const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll 1
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t a = d + (kk >> 2) * 1024 + (kk & 3) * 2;
                umma_bf16(tmem, a, a, id, kk > 0);
            }
            umma_commit(&bars[1]);
        }
    }
    __syncwarp();
    const bool ok = warp_wait(&bars[1], 0, abort_flag, err);
    tc_fence_after();
    // rows of A (warps 0-1, TMEM lanes 0-63) and of P (warps 2-3, lanes 64-127, written straight to the unit in the
    // workspace); P rows 0-31 need columns 0-31 only, the chunk kernel's MMA never reads the blocks above the
    // diagonal
    uint8_t* dst = ws + ((size_t)slot * p.H + h) * kWyUnit;
    if (ok) {
        if (warp < 2) tc_row_pass<true>(taddr(tmem, 32 * warp, 0), gs, tid, 0, 63, sA + tid * kAsLd, nullptr, nullptr);
        else tc_row_pass<false>(taddr(tmem, 32 * warp, 0), gs, tid - 64, 0, warp == 2 ? 31 : 63, nullptr,
                                dst + kWyP, dst + kWyP + 8192);
    }
    tc_fence_before();
    const bool all_ok = __syncthreads_and(ok) != 0;  // one outcome for the CTA: the inverse has barriers
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
    if (!all_ok) return;
    const TEmit em{sm + L::TP, sm + L::TPP, sm + L::TPPL, gs.beta, gs.eG};
    invert_unit_lower64(sA, warp, lane, 1, em);
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
        bulk_store(dst, sm + L::TP, 8192);
        bulk_store(dst + 8192, sm + L::TPP, 8192);
        bulk_store(dst + 16384, sm + L::TPPL, 8192);
        bulk_commit();
        bulk_wait_read();  // the CTA may exit once the stores have read shared memory
    }
}

// ------------------------------------------------------------------------------------------ the main kernel
// Shared-memory map (bytes from a 1024-aligned base).
struct TcSmem {
    static constexpr uint32_t KQ = 0;  // 2 stages x [K ch0-63 | Q ch0-63 | K ch64-127 | Q ch64-127], 8 KB each
    static constexpr uint32_t KQ_STAGE = 32768;
    static constexpr uint32_t V = KQ + 2 * KQ_STAGE;  // V tile: j 0-63 | j 64-127, 8 KB each (MN-major A)
    static constexpr uint32_t TW = V + 16384;         // [T''_hi | T''_lo], [r][s] K-major, 8 KB each
    static constexpr uint32_t TP = TW + 16384;        // T': [r][s] K-major, 8 KB
    static constexpr uint32_t PH = TP + 8192;         // P, columns 0-31 [2]: [r][s] K-major tf32, 8 KB each
    static constexpr uint32_t PL = PH + 16384;        // P, columns 32-63 [2] (both loaded with the K/Q stage)
    static constexpr uint32_t WT = PL + 16384;        // -W^T: lines i (128) x 64 r, MN-major B, 16 KB
    static constexpr uint32_t HT = WT + 16384;        // h^T bf16 [2]: [j][i] K-major, panels i 0-63 | 64-127
    static constexpr uint32_t HT_STAGE = 32768;
    static constexpr uint32_t GATE = HT + 2 * HT_STAGE;  // 4 x TcGate
    static constexpr uint32_t BARS = GATE + 4 * sizeof(TcGate);
    static constexpr uint32_t N_BARS = 25;
    static constexpr uint32_t MISC = BARS + 8 * N_BARS;  // tmem base, abort flag
    static constexpr uint32_t END = MISC + 64;
    static constexpr uint32_t ALLOC = END + 1024;  // slack for the 1024-byte alignment of the base
};
static_assert(TcSmem::ALLOC <= 232448, "shared memory budget");

// Barrier indices.
enum TcBar : int {
    B_KQ_FULL = 0,     // [2] TMA K/Q and the bulk copy of P landed (tx)
    B_KQ_EMPTY = 2,    // [2] serial MMAs of the stage's chunk done
    B_VT_FULL = 4,     // V, T''_hi, T''_lo landed (tx)
    B_VT_EMPTY = 5,    // U^T MMA reading V and T'' done
    B_GATE = 6,        // [4] gate stage written
    B_TP_FULL = 10,    // T' landed (tx)
    B_W_FULL = 11,     // W^T in TMEM (and T' read)
    B_PREP = 12,       // [2] -W^T written (128)
    B_U_FULL = 14,     // U^T in TMEM (and -W^T no longer read)
    B_U_CONV = 15,     // U, U.f split into bf16 hi/lo in TMEM (256)
    B_H_FULL = 16,     // h^T MMA done
    B_H_READY = 17,    // bf16 h^T of the next chunk staged in shared memory (256)
    B_O_FULL = 18,     // O^T MMAs done
    B_O_FREE = 19,     // O^T TMEM read (128)
    B_DRAIN = 20,      // [2] final commit of each MMA issuer
    B_HM_READY = 22,   // fp32 state in TMEM re-scaled by the next chunk's decay (256)
    B_U_RND = 23,      // U in TMEM rounded to tf32 in place, for the O2 MMA (256)
    B_STALL = 24,      // diagnostic only: nothing ever arrives on it (gdn_debug_stall)
};

// Limit of the diagnostic wait on B_STALL (~1 ms): short, so the time-out path runs quickly.
constexpr long long kStallLimitCycles = 2000000LL;

// TMEM columns.  U^T is accumulated in fp32 at TM_U and read there, as tf32, by the O2 MMA; the state
// warpgroups write U diag f as bf16 hi/lo pairs (two values per column) to TM_UF for the h^T MMA.  Columns
// 0-63 are not used.
constexpr uint32_t TM_W = 64, TM_U = 128, TM_UF = 192, TM_O1 = 256, TM_O2 = 320, TM_H = 384, TM_COLS = 512;

// Warp roles (16 warps): 0 TMA producer (K, Q, V; bulk copies of T', T'' and P) and gates; 1 issues W^T; 2
// issues the serial MMAs (U^T, h^T, O^T); 3 idle; 4-7 (prep / output warpgroup) write -W^T and store o; 8-11
// and 12-15 (state warpgroups, one per half of U and of the key channels) split U into bf16 operands, refresh
// the bf16 copy of h^T (double-buffered), re-scale the fp32 state by the next chunk's decay and write hT.
template <bool O_F32>
__global__ void __launch_bounds__(kTcThreads, 1)
gdn_tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p,
                  const uint8_t* ws, unsigned* err) {
    using namespace sm100;
    using L = TcSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 16);
    TcGate* gates = reinterpret_cast<TcGate*>(sm + L::GATE);

    // Waits for in-flight copies or MMAs before exit even after an abort (bounded, error word only).
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
    // workspace unit of chunk c: T' at +0, T''_hi | T''_lo at +8 KB
    auto wy_unit = [&](int c) { return ws + ((size_t)wy_slot(n, seq_start, c) * H + h) * kWyUnit; };

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
            if (b == B_U_CONV || b == B_U_RND || b == B_H_READY || b == B_HM_READY) cnt = 256;
            if (b == B_PREP || b == B_PREP + 1 || b == B_O_FREE) cnt = 128;
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sbase = smem_u32(sm);

    if (warp == 0) {
        // ================================================================ producer: TMA, bulk copies, gates
        auto prefetch = [&](int c) {  // L2 prefetch of a later chunk, so the load issued later hits L2
            if (lane == 0 && c < nc) {
                const int tok = (int)(seq_start + c * kChunk);
                tma_prefetch_3d(&tm_k, 0, h, tok);
                tma_prefetch_3d(&tm_k, 64, h, tok);
                tma_prefetch_3d(&tm_q, 0, h, tok);
                tma_prefetch_3d(&tm_q, 64, h, tok);
                tma_prefetch_3d(&tm_v, j0, h, tok);
                tma_prefetch_3d(&tm_v, j0 + 64, h, tok);
                bulk_prefetch_l2(wy_unit(c), kWyUnit);
            }
        };
        // iteration c: T' of chunk c + 1 (once W^T of chunk c is done with it), V and T'' of chunk c + 1 (once
        // the U^T MMA of chunk c is), K/Q (+ gates) of chunk c + 2; the iterations before 0 fill the stages
        int kq_issued[2] = {0, 0}, vt_issued = 0, tp_issued = 0;
        for (int c = -2; c < nc; ++c) {
            const int c1 = c + 1, c2 = c + 2;
            if (c1 >= 0 && c1 < nc) {
                if (c >= 0 && !warp_wait(&bars[B_W_FULL], c & 1, abort_flag, err)) break;
                if (lane == 0) {
                    mbar_expect_tx(&bars[B_TP_FULL], 8192);
                    bulk_load(sm + L::TP, wy_unit(c1), 8192, &bars[B_TP_FULL]);
                }
                tp_issued++;
                if (c >= 0 && !warp_wait(&bars[B_VT_EMPTY], c & 1, abort_flag, err)) break;
                if (lane == 0) {
                    const int tok = (int)(seq_start + c1 * kChunk);
                    mbar_expect_tx(&bars[B_VT_FULL], 32768);
                    tma_load_3d(sm + L::V, &tm_v, &bars[B_VT_FULL], j0, h, tok);
                    tma_load_3d(sm + L::V + 8192, &tm_v, &bars[B_VT_FULL], j0 + 64, h, tok);
                    bulk_load(sm + L::TW, wy_unit(c1) + 8192, 16384, &bars[B_VT_FULL]);
                }
                vt_issued++;
            }
            if (c2 < nc) {
                const int st = c2 & 1;
                if (c >= 0 && !warp_wait(&bars[B_KQ_EMPTY + st], (c >> 1) & 1, abort_flag, err)) break;
                if (lane == 0) {
                    uint8_t* dst = sm + L::KQ + st * L::KQ_STAGE;
                    const int tok = (int)(seq_start + c2 * kChunk);
                    mbar_expect_tx(&bars[B_KQ_FULL + st], 32768 + 16384);
                    tma_load_3d(dst + 0, &tm_k, &bars[B_KQ_FULL + st], 0, h, tok);
                    tma_load_3d(dst + 8192, &tm_q, &bars[B_KQ_FULL + st], 0, h, tok);
                    tma_load_3d(dst + 16384, &tm_k, &bars[B_KQ_FULL + st], 64, h, tok);
                    tma_load_3d(dst + 24576, &tm_q, &bars[B_KQ_FULL + st], 64, h, tok);
                    bulk_load(sm + L::PH + st * 8192, wy_unit(c2) + kWyP, 8192, &bars[B_KQ_FULL + st]);
                    bulk_load(sm + L::PL + st * 8192, wy_unit(c2) + kWyP + 8192, 8192, &bars[B_KQ_FULL + st]);
                }
                kq_issued[st]++;
                tc_make_gates(gates[c2 & 3], p, (size_t)(seq_start + c2 * kChunk), min(kChunk, eos - bos - c2 * kChunk),
                              h, lane);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_GATE + (c2 & 3)]);
                prefetch(c2 + 1);
            }
        }
        // drain: wait for every load this warp issued before the CTA may exit
        for (int st = 0; st < 2; ++st)
            if (kq_issued[st] > 0) drain_wait(&bars[B_KQ_FULL + st], (kq_issued[st] - 1) & 1);
        if (vt_issued > 0) drain_wait(&bars[B_VT_FULL], (vt_issued - 1) & 1);
        if (tp_issued > 0) drain_wait(&bars[B_TP_FULL], (tp_issued - 1) & 1);
    } else if (warp == 1) {
        // ================================================================ W^T = K^T T'^T
        if (lane == 0) {
            const uint32_t id_w = idesc_bf16(128, 64, true, false);
            const uint32_t n16 = 2u << 17;  // N += 16 in an instruction descriptor (N / 8 at bit 17)
            const uint64_t d_tp = desc_k_sw128(sbase + L::TP);
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1;
                if (!mbar_wait(&bars[B_KQ_FULL + st], (c >> 1) & 1, abort_flag, err)) break;
                // W^T: K and T' of this chunk have landed and -W^T of the previous one has been read out of TMEM
                if (!mbar_wait(&bars[B_TP_FULL], c & 1, abort_flag, err)) break;
                if (c >= 1 && !mbar_wait(&bars[B_PREP + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag, err)) break;
                tc_fence_after();
                const uint64_t da = desc_mn_sw128(sbase + L::KQ + st * L::KQ_STAGE, 16384);
                // k-step kk (tokens s in [16 kk, 16 kk + 16)) reaches only the rows r >= 16 kk of T'
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_W + 16 * kk, da + kk * 128, d_tp + kk * 130, id_w - kk * n16, kk > 0);
                umma_commit(&bars[B_W_FULL]);
            }
            umma_commit(&bars[B_DRAIN]);
            drain_wait(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================================================================ serial MMAs (U^T, h^T, O^T)
        // The k-step loops are unrolled: issuing a tcgen05.mma from a rolled loop with run-time descriptor
        // arithmetic measured ~2x slower, and these issues are on the chunk loop's critical path.  Per chunk
        // the order is U^T (state-free half), U^T (state half), h^T, then the two O^T products: the h^T MMA
        // goes as soon as U diag f is split, and the O^T products (which read the bf16 h^T of this chunk
        // from its own buffer) fill the time the state warpgroups take to stage the next h^T.
        if (lane == 0) {
            const uint32_t id_u1 = idesc_bf16(128, 64, true, false);
            const uint32_t id_u2 = idesc_bf16(128, 64, false, true);
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_h = idesc_bf16(128, 128, false, true);
            const uint32_t id_o2 = idesc_tf32(128, 64, false, false);
            const uint32_t n16 = 2u << 17;
            const uint64_t d_v = desc_mn_sw128(sbase + L::V, 8192);
            const uint64_t d_t = desc_k_sw128(sbase + L::TW);
            const uint64_t d_wt = desc_mn_sw128(sbase + L::WT, 8192);
            int nc_run = nc;
            // Diagnostic: a wait on a barrier that nothing arrives on, with a short limit.  It runs out, sets
            // the error word and the abort flag, and this warp issues no MMA; every other warp then leaves
            // through its own bounded waits and drains what it issued.
            if (p.debug_stall && !mbar_wait_slow(&bars[B_STALL], 0, abort_flag, err, kStallLimitCycles)) nc_run = 0;
            for (int c = 0; c < nc_run; ++c) {
                const int st = c & 1;
                const uint32_t kq = sbase + L::KQ + st * L::KQ_STAGE;
                const uint64_t d_ht = desc_k_sw128(sbase + L::HT + st * L::HT_STAGE);
                if (!mbar_wait(&bars[B_VT_FULL], c & 1, abort_flag, err)) break;
                tc_fence_after();
                // U^T = V^T (T''_hi + T''_lo)^T - h^T W^T ; the first half does not need the state.  As T'' is
                // lower triangular, k-step ks (tokens s in [16 ks, 16 ks + 16)) updates only columns r >= 16 ks.
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const int ks = kk & 3;
                    umma_bf16(tmem + TM_U + 16 * ks, d_v + ks * 128, d_t + (kk >> 2) * 512 + ks * 130,
                              id_u1 - ks * n16, kk > 0);
                }
                umma_commit(&bars[B_VT_EMPTY]);
                if (!mbar_wait(&bars[B_PREP + st], (c >> 1) & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[B_H_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + TM_U, d_ht + (kk >> 2) * 1024 + (kk & 3) * 2, d_wt + kk * 128, id_u2, 1);
                umma_commit(&bars[B_U_FULL]);
                // h^T += (U diag f)^T K  (hi and lo halves)
                if (!mbar_wait(&bars[B_U_CONV], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[B_HM_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
                const uint64_t d_k = desc_mn_sw128(kq, 16384);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // kk < 4: hi, else lo; s-step ks covers values 16 ks .. 16 ks + 15
                    const int ks = kk & 3;
                    const uint32_t a = tmem + TM_UF + (ks >> 1) * 32 + (kk >> 2) * 16 + (ks & 1) * 8;
                    umma_bf16_tmem_a(tmem + TM_H, a, d_k + ks * 128, id_h, 1);
                }
                umma_commit(&bars[B_H_FULL]);
                // O1^T = h^T Q^T (scaled by 2^G_r in the epilogue)
                if (c >= 1 && !mbar_wait(&bars[B_O_FREE], (c - 1) & 1, abort_flag, err)) break;
                tc_fence_after();
                const uint64_t d_q = desc_k_sw128(kq + 8192);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t o = (kk >> 2) * 1024 + (kk & 3) * 2;
                    umma_bf16(tmem + TM_O1, d_ht + o, d_q + o, id_o, kk > 0);
                }
                if (!mbar_wait(&bars[B_U_RND], c & 1, abort_flag, err)) break;
                tc_fence_after();
                // O2^T = U^T P^T on kind::tf32: U fp32 straight from TM_U, P (columns 0-31 in PH, 32-63 in PL,
                // from the workspace with this chunk's K/Q stage); k-step ks8 covers 8 tokens and, P being lower
                // triangular, only columns r >= 16 (ks8 / 2)
#pragma unroll
                for (int ks8 = 0; ks8 < 8; ++ks8) {
                    const int r0 = 16 * (ks8 >> 1);
                    const uint64_t b = desc_k_sw128(sbase + ((ks8 & 4) ? L::PL : L::PH) + st * 8192) +
                                       ((r0 * 128 + (ks8 & 3) * 32) >> 4);
                    umma_tf32_tmem_a(tmem + TM_O2 + r0, tmem + TM_U + 8 * ks8, b, id_o2 - (r0 >> 4) * n16, ks8 > 0);
                }
                umma_commit(&bars[B_O_FULL]);
                umma_commit(&bars[B_KQ_EMPTY + st]);
            }
            umma_commit(&bars[B_DRAIN + 1]);
            drain_wait(&bars[B_DRAIN + 1], 0);
        }
        __syncwarp();
    } else if (warp == 3) {
        // idle: its TMEM lane quadrant is served by warps 7, 11 and 15
    } else if (warp < 8) {
        // ================================================================ prep / output warpgroup
        // Iteration k: (1) -W^T of chunk k, line i = t, from TMEM into shared memory.  (2) The output tile of
        // chunk k - 1: O1^T and O2^T read from TMEM (then released for the next chunk's O^T MMAs), combined and
        // stored to global memory, one token row per store (a warp writes 32 consecutive values of the row).
        // The warps run independently; a timed-out wait does not break out, the warp finishes the iteration
        // and leaves at the top of the next.
        const int t = tid - 128;  // TMEM lane: value column j of O^T / line of W^T
        const int wid = warp & 3;
        const uint32_t lane_base = 32 * wid;
        for (int k = 0; k <= nc; ++k) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            if (k < nc) {
                const int c = k, st = c & 1;
                warp_wait(&bars[B_W_FULL], c & 1, abort_flag, err);
                if (c >= 1) warp_wait(&bars[B_U_FULL], (c - 1) & 1, abort_flag, err);
                tc_fence_after();
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(taddr(tmem, lane_base, TM_W + 32 * half), v);
                    tmem_wait_ld();
                    st_half_line_bf16(sm + L::WT, t, 4 * half, v, -1.f);
                }
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(&bars[B_PREP + st]);
            }
            if (k >= 1) {
                const int c = k - 1;
                warp_wait(&bars[B_O_FULL], c & 1, abort_flag, err);
                tc_fence_after();
                const TcGate& gs = gates[c & 3];
                const int Lc = gs.L;
                const size_t tok0 = (size_t)(seq_start + (long long)c * kChunk);
                const size_t ostride = (size_t)H * dv;
                size_t off = (tok0 * H + h) * (size_t)dv + j0 + t;
#pragma unroll 1
                for (int r8 = 0; r8 < 64; r8 += 8) {
                    float v1[8], v2[8];
                    tmem_ld8(taddr(tmem, lane_base, TM_O1 + r8), v1);
                    tmem_ld8(taddr(tmem, lane_base, TM_O2 + r8), v2);
                    tmem_wait_ld();
                    if (r8 == 56) {
                        tc_fence_before();
                        mbar_arrive(&bars[B_O_FREE]);
                    }
                    const float4 e0 = *reinterpret_cast<const float4*>(gs.eG + r8);
                    const float4 e1 = *reinterpret_cast<const float4*>(gs.eG + r8 + 4);
                    const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float val = p.scale * fmaf(ev[q], v1[q], v2[q]);
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
        // Warpgroups 8-11 (half 0) and 12-15 (half 1) share the serial-chain work: each splits half of U
        // into bf16 operands and refreshes half of the state (key channels [64 half, 64 half + 64)).
        const int half = (warp - 8) >> 2;
        const int j = tid & 127;  // value column (TMEM lane)
        const uint32_t lane_base = 32 * (warp & 3);
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
        // initial state: bf16 copy and fp32 master pre-scaled by the first chunk's decay
        if (warp_wait(&bars[B_GATE + 0], 0, abort_flag, err)) {
            const float g0 = gates[0].gamma;
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
                for (int q = 0; q < 32; ++q) v[q] *= g0;
                tmem_st32(taddr(tmem, lane_base, TM_H + 32 * piece), v);
            }
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bars[B_H_READY]);
            mbar_arrive(&bars[B_HM_READY]);
        }
        for (int c = 0; c < nc; ++c) {
            const TcGate& gs = gates[c & 3];
            // ---- U diag f (values [32 half, 32 half + 32)) as bf16 hi/lo pairs for the h^T MMA, to TM_UF
            // ([hi | lo], 16 columns each per half); then U itself, rounded to tf32, back into TM_U for the
            // kind::tf32 O2 MMA.
            if (!warp_wait(&bars[B_U_FULL], c & 1, abort_flag, err)) break;
            if (!warp_wait(&bars[B_GATE + (c & 3)], (c >> 2) & 1, abort_flag, err)) break;
            tc_fence_after();
            {
                float u[32];
                tmem_ld32(taddr(tmem, lane_base, TM_U + 32 * half), u);
                tmem_wait_ld();
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int s0 = 32 * half + 2 * q;
                    split_pack_bf16(u[2 * q] * gs.f[s0], u[2 * q + 1] * gs.f[s0 + 1], hi[q], lo[q]);
                }
                tmem_st16u(taddr(tmem, lane_base, TM_UF + 32 * half), hi);
                tmem_st16u(taddr(tmem, lane_base, TM_UF + 32 * half + 16), lo);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[B_U_CONV]);
                // U back in place rounded to tf32: the tensor core would otherwise truncate the fp32 value
                uint32_t ur[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) ur[q] = f2tf32(u[q]);
                tmem_st32u(taddr(tmem, lane_base, TM_U + 32 * half), ur);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_U_RND]);
            // ---- state refresh (key channels of this half)
            if (!warp_wait(&bars[B_H_FULL], c & 1, abort_flag, err)) break;
            const bool last = c + 1 == nc;
            if (!last && !warp_wait(&bars[B_GATE + ((c + 1) & 3)], ((c + 1) >> 2) & 1, abort_flag, err)) break;
            tc_fence_after();
            const float gn = last ? 1.f : gates[(c + 1) & 3].gamma;
            // pass 1: the bf16 copy (what the next chunk's first MMAs wait for), or hT after the last chunk
#pragma unroll 1
            for (int piece = 2 * half; piece < 2 * half + 2; ++piece) {
                float v[32];
                tmem_ld32(taddr(tmem, lane_base, TM_H + 32 * piece), v);
                tmem_wait_ld();
                if (!last) {
                    st_half_line_bf16(sm + L::HT + ((c + 1) & 1) * L::HT_STAGE + (piece >> 1) * 16384, j,
                                      4 * (piece & 1), v);
                    if (p.h_chunks) dump_state(c + 1, piece, v);
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
                mbar_arrive(&bars[B_H_READY]);
                // pass 2: the fp32 master times the next chunk's decay (needed only by the next h^T MMA)
#pragma unroll 1
                for (int piece = 2 * half; piece < 2 * half + 2; ++piece) {
                    float v[32];
                    tmem_ld32(taddr(tmem, lane_base, TM_H + 32 * piece), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] *= gn;
                    tmem_st32(taddr(tmem, lane_base, TM_H + 32 * piece), v);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[B_HM_READY]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ------------------------------------------------------------------------------------------ host side
inline bool tc_supported(const FwdParams& p) { return p.dk == kTcDK && p.dv % kTcDV == 0 && p.T > 0; }
// Workspace bytes the tcgen05 path needs (the WY kernel's output).
inline size_t tc_workspace_bytes(int B, int T, int H, int n_seqs) {
    return (size_t)wy_slots(B, T, n_seqs) * (size_t)H * kWyUnit;
}

static thread_local char t_tc_msg[256];
inline const char* tc_last_error() { return t_tc_msg; }

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_encodeTiled get_encode_fn() {
    static PFN_encodeTiled fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(ptr);
    }
    return fn;
}

// 3-D map over a [rows, H, d] bf16 tensor (d innermost), box 64 x 1 x 64, 128-byte swizzle.
inline bool make_map(CUtensorMap* map, const void* base, int d, int H, long long rows) {
    PFN_encodeTiled enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * H * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline gdn_status launch_tc(const FwdParams& p, bool o_f32, void* ws, size_t ws_bytes, unsigned* err,
                            cudaStream_t stream) {
    const size_t need = tc_workspace_bytes(p.B, p.T, p.H, p.n_seq);
    if (!ws || ws_bytes < need) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "the tcgen05 path needs %zu bytes of workspace (got %zu)", need, ws_bytes);
        return GDN_ERR_UNSUPPORTED;
    }
    CUtensorMap mq, mk, mv;
    const long long rows = (long long)p.B * p.T;
    if (!make_map(&mq, p.q, p.dk, p.H, rows) || !make_map(&mk, p.k, p.dk, p.H, rows) ||
        !make_map(&mv, p.v, p.dv, p.H, rows)) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cuTensorMapEncodeTiled failed");
        return GDN_ERR_CUDA;
    }
    cudaError_t e = cudaFuncSetAttribute(gdn_tc_wy_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)WySmem::ALLOC);
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    const long long wy_grid = (long long)(wy_slots(p.B, p.T, p.n_seq)) * p.H;
    if (wy_grid > 0x7fffffffLL) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "too many chunks for one launch");
        return GDN_ERR_UNSUPPORTED;
    }
    ProfScope prof_wy(PK_TC_WY, stream);
    gdn_tc_wy_kernel<<<(unsigned)wy_grid, kWyThreads, WySmem::ALLOC, stream>>>(mq, mk, p, static_cast<uint8_t*>(ws),
                                                                                err);
    prof_wy.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "WY kernel: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    auto kern = o_f32 ? gdn_tc_fwd_kernel<true> : gdn_tc_fwd_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcSmem::ALLOC);
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    const unsigned grid = (unsigned)(p.dv / kTcDV) * p.H * p.n_seq;
    ProfScope prof_main(PK_TC_MAIN, stream);
    kern<<<grid, kTcThreads, TcSmem::ALLOC, stream>>>(mq, mk, mv, p, static_cast<const uint8_t*>(ws), err);
    prof_main.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "%s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

}  // namespace gdn
