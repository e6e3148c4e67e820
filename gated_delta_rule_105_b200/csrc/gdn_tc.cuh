// tcgen05 (5th-generation tensor core) chunked forward kernel for the gated delta rule, bf16 inputs.
//
// One CTA owns one (sequence n, head h, block of 128 value columns j) and walks the sequence's chunks of
// C = 64 tokens.  Every contraction is an M = 128 tcgen05.mma with bf16 operands in 128B-swizzled shared
// memory and an fp32 accumulator in tensor memory.  The state is kept transposed, h^T [j][i] (value column
// j on the 128 TMEM lanes, key channel i on 128 columns), fp32 in TMEM for the whole sequence.
//
// Per chunk (r, s = token rows; G = chunk-local cumulative gate in base 2; f_s = 2^(G_last - G_s)):
//   S1  = [K; Q] K^T                          (rows 0-63: K K^T, rows 64-127: Q K^T)
//   A   = strict_lower(beta_r 2^(G_r - G_s) S1_K) ;  P = lower(2^(G_r - G_s) S1_Q)
//   T   = (I + A)^-1 ; T' = T diag(beta 2^G) ; T'' = T diag(beta)
//   W^T = K^T T'^T
//   U^T = V^T T''^T - h^T W^T                 (= (T'' V - W h)^T, the corrected values)
//   O^T = diag(2^G) applied to h^T Q^T, + U^T P^T   (read-out, scaled by `scale` on the way out)
//   h^T <- 2^(G_last) h^T + (U diag f)^T K
// Precision: every bf16 operand whose rounding would reach the output at the bf16-ulp level is avoided or
// split.  U and U diag f are kept as bf16 hi + lo pairs (in TMEM, as the A operand), P and T'' likewise
// (in shared memory); 2^G_r is applied to the fp32 accumulator of h^T Q^T instead of to Q.  The remaining
// bf16 operands are h^T, W^T, T' and the inputs themselves.
// This is the WY form of the intra-chunk dependency with one state handed from chunk to chunk
// (GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755, section "Chunked parallelism").
//
// Warp roles (20 warps): 0 TMA producer and gate prep; 1 issues the h-independent MMAs (S1, W^T) one chunk
// ahead; 2 issues the serial MMAs (U^T, O^T, h^T); 3 stores the output tiles by TMA; 4-7 and 8-11 (two prep
// warpgroups) build A, P, (I+A)^-1, T', T'' and -W^T; 12-15 and 16-19 (state warpgroups, one per half of U,
// of the key channels and of the chunk's rows) split U into bf16 operands, refresh the bf16 copy of h^T,
// re-scale the fp32 state by the next chunk's decay, write hT and stage o.
// The operands T', T'' and P are lower triangular: the MMAs that read them skip the blocks above the
// diagonal (k-step ks of 16 tokens only reaches the output columns r >= 16 ks).
// All mbarrier waits are bounded: on time-out the CTA sets the error word and drains to the exit.
#pragma once

#include <cuda.h>

#include "gdn_sm100.cuh"

namespace gdn {

constexpr int kTcThreads = 640;

constexpr int kTcDV = 128;  // value columns per CTA
constexpr int kTcDK = 128;  // key dimension handled by this kernel

struct TcGate {  // one chunk's gate data, written by the producer warp
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

// Shared-memory map (bytes from a 1024-aligned base).
struct TcSmem {
    static constexpr uint32_t KQ = 0;  // 2 stages x [K ch0-63 | Q ch0-63 | K ch64-127 | Q ch64-127], 8 KB each
    static constexpr uint32_t KQ_STAGE = 32768;
    static constexpr uint32_t V = KQ + 2 * KQ_STAGE;  // V tile: j 0-63 | j 64-127, 8 KB each (MN-major A)
    static constexpr uint32_t TPP = V + 16384;        // T'' hi [2]: [r][s] K-major, 8 KB each
    static constexpr uint32_t TPPL = TPP + 16384;     // T'' lo [2]
    static constexpr uint32_t TP = TPPL + 16384;      // T': [r][s] K-major, 8 KB
    static constexpr uint32_t PH = TP + 8192;         // P hi [2]: [r][s] K-major, 8 KB each
    static constexpr uint32_t PL = PH + 16384;        // P lo [2]
    static constexpr uint32_t WT = PL + 16384;        // -W^T: lines i (128) x 64 r, MN-major B, 16 KB
    static constexpr uint32_t HT = WT + 16384;        // h^T bf16: [j][i] K-major, panels i 0-63 | 64-127, 16 KB each
    static constexpr uint32_t AS = HT + 32768;        // A, then (I+A)^-1, fp32 [64][68]
    static constexpr uint32_t AS_LD = 68;
    static constexpr uint32_t GATE = AS + 64 * AS_LD * 4;  // 4 x TcGate
    static constexpr uint32_t BARS = GATE + 4 * sizeof(TcGate);
    static constexpr uint32_t N_BARS = 32;
    static constexpr uint32_t MISC = BARS + 8 * N_BARS;  // tmem base, abort flag
    static constexpr uint32_t END = MISC + 64;
    static constexpr uint32_t ALLOC = END + 1024;  // slack for the 1024-byte alignment of the base
};
static_assert(TcSmem::ALLOC <= 232448, "shared memory budget");

// Barrier indices.
enum TcBar : int {
    B_KQ_FULL = 0,    // [2] TMA K/Q landed (tx)
    B_KQ_EMPTY = 2,   // [2] serial MMAs of the stage's chunk done
    B_V_FULL = 4,     // V landed (tx)
    B_V_EMPTY = 5,    // U^T MMA reading V done
    B_GATE = 6,       // [4] gate stage written
    B_S1_FULL = 10,   // S1 in TMEM
    B_S1_FREE = 11,   // prep read S1 (256 arrivals)
    B_TP_READY = 12,  // T' written (128)
    B_W_FULL = 13,    // W^T in TMEM
    B_PREP = 14,      // [2] T'', -W^T, P ready for the serial step (256)
    B_P_FREE = 16,    // [2] P, T'' stage free: O^T MMA done and the output staged there stored
    B_U_FULL = 18,    // U^T in TMEM (and -W^T, T'' no longer read)
    B_U_CONV = 19,    // U, U.f split into bf16 hi/lo in TMEM (256)
    B_H_FULL = 20,    // h^T MMA done
    B_H_READY = 21,   // bf16 h^T staged in shared memory (256)
    B_O_FULL = 22,    // O^T MMAs done
    B_O_FREE = 23,    // O^T TMEM read (256)
    B_DRAIN = 24,     // [2] final commit of each MMA issuer
    B_HM_READY = 26,  // fp32 state in TMEM re-scaled by the next chunk's decay (256)
    B_O_STAGED = 27,  // output tile staged in shared memory (256)
};

// TMEM columns.  U^T is accumulated in fp32 at TM_U; the state warpgroup then writes U as bf16 hi/lo pairs
// (two values per column) to TM_UF and U diag f, also as hi/lo pairs, in place over TM_U.
constexpr uint32_t TM_S1 = 0, TM_W = 64, TM_U = 128, TM_UF = 192, TM_O1 = 256, TM_O2 = 320, TM_H = 384,
                   TM_COLS = 512;

// ------------------------------------------------------------------------------------------ small helpers
__device__ __forceinline__ uint32_t f2tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D(16x8) += A(16x8) B(8x8), tf32 inputs, fp32 accumulate (legacy warp-level MMA, used only for the
// 16x16 blocks of the triangular inverse).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// 16x16 blocks of the [64][68] fp32 scratch, as tf32 mma.sync fragments.  A block is named by its logical
// origin (r0, c0); `tr` = it is stored transposed in the mirrored position (element (r, c) of the logical
// block at scratch row c0 + c, column r0 + r).
struct Frag16 {
    uint32_t a[2][4];  // as the A operand: k-halves 0, 1
};
__device__ __forceinline__ float blk(const float* S, int r0, int c0, int r, int c, bool tr) {
    return tr ? S[(c0 + c) * TcSmem::AS_LD + r0 + r] : S[(r0 + r) * TcSmem::AS_LD + c0 + c];
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
        float* p00 = tr ? &S[(c0 + c) * TcSmem::AS_LD + r0 + g] : &S[(r0 + g) * TcSmem::AS_LD + c0 + c];
        const int dc = tr ? TcSmem::AS_LD : 1, dr = tr ? 1 : TcSmem::AS_LD;
        p00[0] = sgn * acc[nh][0];
        p00[dc] = sgn * acc[nh][1];
        p00[8 * dr] = sgn * acc[nh][2];
        p00[8 * dr + dc] = sgn * acc[nh][3];
    }
}

// Where the blocks of T go once final: T' = T diag(beta 2^G) as bf16, and T'' = T diag(beta) as a bf16 hi + lo
// pair, each [r][s] K-major with 128-byte swizzle.  Only the blocks on and below the diagonal are written;
// the MMAs that read these operands skip the zero blocks above it.
struct TEmit {
    uint8_t* tp;
    uint8_t* tpp;
    uint8_t* tppl;
    const float* beta;
    const float* eG;
};
// Emits sgn * acc, the final 16x16 block (r0, c0) of T held as an mma.sync accumulator.
__device__ __forceinline__ void emit16(const TEmit& em, int r0, int c0, int lane, const float (&acc)[2][4], float sgn) {
    using namespace sm100;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int s = c0 + 8 * nh + 2 * t;
        const float b0 = sgn * em.beta[s], b1 = sgn * em.beta[s + 1];
        const float e0 = em.eG[s], e1 = em.eG[s + 1];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const float x0 = acc[nh][2 * hr] * b0, x1 = acc[nh][2 * hr + 1] * b1;
            const uint32_t off = sw128(r0 + g + 8 * hr, s >> 3) + (s & 7) * 2;
            uint32_t hi, lo;
            split_pack_bf16(x0, x1, hi, lo);
            *reinterpret_cast<uint32_t*>(em.tp + off) = pack_bf16(x0 * e0, x1 * e1);
            *reinterpret_cast<uint32_t*>(em.tpp + off) = hi;
            *reinterpret_cast<uint32_t*>(em.tppl + off) = lo;
        }
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
__device__ __forceinline__ void invert_unit_lower64(float* S, int wid, int lane, uint32_t bar_id, const TEmit& em) {
    using namespace sm100;
    {
        const int b0 = 16 * wid, c = lane & 15;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = (r == c) ? 1.f : 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s) acc = fmaf(-S[(b0 + r) * TcSmem::AS_LD + b0 + s], t[s], acc);
            t[r] = (r < c) ? 0.f : acc;
        }
        __syncwarp();
        if (lane < 16) {
#pragma unroll
            for (int r = 0; r < 16; ++r) S[(b0 + r) * TcSmem::AS_LD + b0 + c] = t[r];
        }
        // emit column c of T_ii: lanes 0-15 rows 0-7, lanes 16-31 rows 8-15
        const int s = b0 + c, hr = lane >> 4;
        const float bs = em.beta[s], es = em.eG[s];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const float x = (hr ? t[8 + rr] : t[rr]) * bs;
            const uint32_t off = sw128(b0 + 8 * hr + rr, s >> 3) + (s & 7) * 2;
            const __nv_bfloat16 xh = __float2bfloat16_rn(x);
            *reinterpret_cast<__nv_bfloat16*>(em.tp + off) = __float2bfloat16_rn(x * es);
            *reinterpret_cast<__nv_bfloat16*>(em.tpp + off) = xh;
            *reinterpret_cast<__nv_bfloat16*>(em.tppl + off) = __float2bfloat16_rn(x - __bfloat162float(xh));
        }
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

// ------------------------------------------------------------------------------------------ the kernel
template <bool O_F32>
__global__ void __launch_bounds__(kTcThreads, 1)
gdn_tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const FwdParams p,
                  unsigned* err) {
    using namespace sm100;
    using L = TcSmem;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC + 16);
    TcGate* gates = reinterpret_cast<TcGate*>(sm + L::GATE);
    float* sA = reinterpret_cast<float*>(sm + L::AS);

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
    const int nc = (eos - bos + kChunk - 1) / kChunk;
    const size_t state_base = ((size_t)n * H + h) * kTcDK * (size_t)dv + j0;

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
            const uint32_t cnt = (b == B_S1_FREE || b == B_PREP || b == B_PREP + 1 || b == B_U_CONV ||
                                  b == B_H_READY || b == B_HM_READY || b == B_O_FREE || b == B_O_STAGED)
                                     ? 256u
                                     : (b == B_TP_READY ? 128u : 1u);
            mbar_init(&bars[b], cnt);
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_o);
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
        // ================================================================ producer: TMA + gates
        int kq_issued[2] = {0, 0}, v_issued = 0;
        auto load_kq = [&](int c) {
            const int st = c & 1;
            if (lane == 0) {
                uint8_t* dst = sm + L::KQ + st * L::KQ_STAGE;
                const int tok = row * T + bos + c * kChunk;
                mbar_expect_tx(&bars[B_KQ_FULL + st], 32768);
                tma_load_3d(dst + 0, &tm_k, &bars[B_KQ_FULL + st], 0, h, tok);
                tma_load_3d(dst + 8192, &tm_q, &bars[B_KQ_FULL + st], 0, h, tok);
                tma_load_3d(dst + 16384, &tm_k, &bars[B_KQ_FULL + st], 64, h, tok);
                tma_load_3d(dst + 24576, &tm_q, &bars[B_KQ_FULL + st], 64, h, tok);
            }
            kq_issued[st]++;
        };
        auto load_v = [&](int c) {
            if (lane == 0) {
                const int tok = row * T + bos + c * kChunk;
                mbar_expect_tx(&bars[B_V_FULL], 16384);
                tma_load_3d(sm + L::V, &tm_v, &bars[B_V_FULL], j0, h, tok);
                tma_load_3d(sm + L::V + 8192, &tm_v, &bars[B_V_FULL], j0 + 64, h, tok);
            }
            v_issued++;
        };
        // L2 prefetch of a later chunk's tiles, so that the load issued once a stage frees up hits L2
        auto prefetch = [&](int c) {
            if (lane == 0 && c < nc) {
                const int tok = row * T + bos + c * kChunk;
                tma_prefetch_3d(&tm_k, 0, h, tok);
                tma_prefetch_3d(&tm_k, 64, h, tok);
                tma_prefetch_3d(&tm_q, 0, h, tok);
                tma_prefetch_3d(&tm_q, 64, h, tok);
                tma_prefetch_3d(&tm_v, j0, h, tok);
                tma_prefetch_3d(&tm_v, j0 + 64, h, tok);
            }
        };
        auto make_gates = [&](int c) {
            TcGate& gs = gates[c & 3];
            const int c0 = bos + c * kChunk;
            const int Lc = min(kChunk, eos - c0);
            float gv[2], bv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = 2 * lane + u;
                const size_t tok = ((size_t)row * T + c0 + r) * H + h;
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
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_GATE + (c & 3)]);
        };
        // iteration c loads V of chunk c + 1 and K/Q (+ gates) of chunk c + 2; the first two fill both stages
        for (int c = -2; c < nc; ++c) {
            if (c + 1 >= 0 && c + 1 < nc) {
                if (c >= 0 && !warp_wait(&bars[B_V_EMPTY], c & 1, abort_flag, err)) break;
                load_v(c + 1);
            }
            if (c + 2 < nc) {
                if (c >= 0 && !warp_wait(&bars[B_KQ_EMPTY + (c & 1)], (c >> 1) & 1, abort_flag, err)) break;
                load_kq(c + 2);
                make_gates(c + 2);
                prefetch(c + 3);
            }
        }
        // drain: wait for every load this warp issued before the CTA may exit
        for (int st = 0; st < 2; ++st)
            if (kq_issued[st] > 0) drain_wait(&bars[B_KQ_FULL + st], (kq_issued[st] - 1) & 1);
        if (v_issued > 0) drain_wait(&bars[B_V_FULL], (v_issued - 1) & 1);
    } else if (warp == 1) {
        // ================================================================ h-independent MMAs (S1, W^T)
        // Issued in readiness order.  S1 of chunk c + 1 needs its K/Q and the prep to have read S1 of chunk c,
        // which it normally has before chunk c's T' is ready; W^T of chunk c needs T'.  While both are
        // pending the thread sleeps on T' and checks the S1 conditions whenever it wakes.
        if (lane == 0) {
            const uint32_t id_s1 = idesc_bf16(128, 64, false, false);
            const uint32_t id_w = idesc_bf16(128, 64, true, false);
            const uint32_t n16 = 2u << 17;  // N += 16 in an instruction descriptor (N / 8 at bit 17)
            int ns = 0, nw = 0;  // next chunk for S1, for W^T
            long long last = clock64();
            auto s1_ready = [&]() {
                return mbar_test(&bars[B_KQ_FULL + (ns & 1)], (ns >> 1) & 1) &&
                       (ns == 0 || mbar_test(&bars[B_S1_FREE], (ns - 1) & 1));
            };
            while (nw < nc) {
                bool did = false;
                // S1 may run ahead of W^T by one chunk; W^T(nw) needs S1(nw) first
                const bool s1_due = ns < nc && ns <= nw + 1;
                if (s1_due && s1_ready()) {
                    tc_fence_after();
                    const uint64_t d = desc_k_sw128(sbase + L::KQ + (ns & 1) * L::KQ_STAGE);
#pragma unroll 1
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t a = d + (kk >> 2) * 1024 + (kk & 3) * 2;
                        umma_bf16(tmem + TM_S1, a, a, id_s1, kk > 0);
                    }
                    umma_commit(&bars[B_S1_FULL]);
                    ++ns;
                    did = true;
                } else if (nw < ns && mbar_try_wait_ns(&bars[B_TP_READY], nw & 1, s1_due ? 200u : kSuspendHintNs)) {
                    tc_fence_after();
                    const uint64_t da = desc_mn_sw128(sbase + L::KQ + (nw & 1) * L::KQ_STAGE, 16384);
                    const uint64_t db = desc_k_sw128(sbase + L::TP);
                    // k-step kk (tokens s in [16 kk, 16 kk + 16)) reaches only the rows r >= 16 kk of T'
#pragma unroll 1
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + TM_W + 16 * kk, da + kk * 128, db + kk * 130, id_w - kk * n16, kk > 0);
                    umma_commit(&bars[B_W_FULL]);
                    ++nw;
                    did = true;
                } else if (nw == ns) {  // only S1 can make progress: sleep on its K/Q, then on S1_FREE
                    mbar_try_wait(&bars[B_KQ_FULL + (ns & 1)], (ns >> 1) & 1);
                    if (ns > 0) mbar_try_wait(&bars[B_S1_FREE], (ns - 1) & 1);
                }
                if (did) {
                    last = clock64();
                } else {
                    if (*abort_flag) break;
                    if (clock64() - last > kWaitLimitCycles) {
                        *abort_flag = 1;
                        atomicOr(err, kErrTimeout);
                        break;
                    }
                }
            }
            umma_commit(&bars[B_DRAIN]);
            drain_wait(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================================================================ serial MMAs (U^T, O^T, h^T)
        // The k-step loops stay rolled (short code); descriptors advance by byte offset >> 4.
        if (lane == 0) {
            const uint32_t id_u1 = idesc_bf16(128, 64, true, false);
            const uint32_t id_u2 = idesc_bf16(128, 64, false, true);
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_h = idesc_bf16(128, 128, false, true);
            const uint32_t n16 = 2u << 17;  // N += 16 in an instruction descriptor (N / 8 at bit 17)
            const uint64_t d_v = desc_mn_sw128(sbase + L::V, 8192);
            const uint64_t d_ht = desc_k_sw128(sbase + L::HT);
            const uint64_t d_wt = desc_mn_sw128(sbase + L::WT, 8192);
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1;
                const uint32_t kq = sbase + L::KQ + st * L::KQ_STAGE;
                if (!mbar_wait(&bars[B_PREP + st], (c >> 1) & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[B_V_FULL], c & 1, abort_flag, err)) break;
                tc_fence_after();
                // U^T = V^T (T''_hi + T''_lo)^T - h^T W^T ; the first half does not need the state.  As T'' is
                // lower triangular, k-step ks (tokens s in [16 ks, 16 ks + 16)) updates only columns r >= 16 ks.
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const int ks = kk & 3;
                    const uint64_t b = desc_k_sw128(sbase + (kk < 4 ? L::TPP : L::TPPL) + st * 8192) + ks * 130;
                    umma_bf16(tmem + TM_U + 16 * ks, d_v + ks * 128, b, id_u1 - ks * n16, kk > 0);
                }
                if (!mbar_wait(&bars[B_H_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + TM_U, d_ht + (kk >> 2) * 1024 + (kk & 3) * 2, d_wt + kk * 128, id_u2, 1);
                umma_commit(&bars[B_U_FULL]);
                umma_commit(&bars[B_V_EMPTY]);
                // O1^T = h^T Q^T (scaled by 2^G_r in the epilogue)
                if (c >= 1 && !mbar_wait(&bars[B_O_FREE], (c - 1) & 1, abort_flag, err)) break;
                tc_fence_after();
                const uint64_t d_q = desc_k_sw128(kq + 8192);
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t o = (kk >> 2) * 1024 + (kk & 3) * 2;
                    umma_bf16(tmem + TM_O1, d_ht + o, d_q + o, id_o, kk > 0);
                }
                // h^T += (U diag f)^T K  (hi and lo halves) ;  O2^T = U^T P^T  (hi*hi + hi*lo + lo*hi)
                if (!mbar_wait(&bars[B_U_CONV], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[B_HM_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
                const uint64_t d_k = desc_mn_sw128(kq, 16384);
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {  // kk < 4: hi, else lo; s-step ks covers values 16 ks .. 16 ks + 15
                    const int ks = kk & 3;
                    const uint32_t a = tmem + TM_U + (ks >> 1) * 32 + (kk >> 2) * 16 + (ks & 1) * 8;
                    umma_bf16_tmem_a(tmem + TM_H, a, d_k + ks * 128, id_h, 1);
                }
                umma_commit(&bars[B_H_FULL]);
#pragma unroll 1
                for (int kk = 0; kk < 12; ++kk) {  // P lower triangular: k-step ks reaches columns r >= 16 ks
                    const int part = kk >> 2, ks = kk & 3;  // 0: Uhi Phi, 1: Uhi Plo, 2: Ulo Phi
                    const uint32_t a = tmem + TM_UF + (part == 2 ? 32 : 0) + ks * 8;
                    const uint64_t b = desc_k_sw128(sbase + (part == 1 ? L::PL : L::PH) + st * 8192) + ks * 130;
                    umma_bf16_tmem_a(tmem + TM_O2 + 16 * ks, a, b, id_o - ks * n16, kk > 0);
                }
                umma_commit(&bars[B_O_FULL]);
                umma_commit(&bars[B_KQ_EMPTY + st]);
            }
            umma_commit(&bars[B_DRAIN + 1]);
            drain_wait(&bars[B_DRAIN + 1], 0);
        }
        __syncwarp();
    } else if (warp == 3) {
        // ================================================================ output stores
        // A full chunk's o tile is staged by the state warpgroups in the P and T'' buffers of its stage (free
        // once its O^T MMAs are done) and leaves by TMA; a partial chunk is written directly by them.
        if (lane == 0) {
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1;
                if (!mbar_wait(&bars[B_O_STAGED], c & 1, abort_flag, err)) break;
                if (eos - bos - c * kChunk >= kChunk) {
                    const int tok0 = row * T + bos + c * kChunk;
                    const uint32_t rg[4] = {L::PH, L::PL, L::TPP, L::TPPL};
#pragma unroll
                    for (int b = 0; b < 4; ++b) tma_store_3d(&tm_o, sm + rg[b] + st * 8192, j0, h, tok0 + 16 * b);
                    bulk_commit();
                    bulk_wait_read_all();
                }
                mbar_arrive(&bars[B_P_FREE + st]);
            }
            bulk_wait_all();
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 12) {
        // ================================================================ prep warpgroups
        // Per chunk: (1) A rows, split by column halves over the quadrant-0/1 warps of both warpgroups;
        // (2) the first warpgroup inverts (I + A), writing T' (what the W^T MMA needs) and T'' as it goes,
        // while the quadrant-2/3 warps of the second build P; (3) -W^T.  A timed-out wait does not break out
        // here: the warpgroups finish the iteration and leave together at the top of the next.
        const int wsel = (warp - 4) >> 2;      // warpgroup 0 or 1
        const int t = (tid - 128) & 127;       // TMEM lane: row of S1 / line of W^T
        const int wid = warp & 3;
        for (int c = 0; c < nc; ++c) {
            if (named_bar_or(2, 256, *abort_flag != 0)) break;
            const int st = c & 1;
            warp_wait(&bars[B_S1_FULL], c & 1, abort_flag, err);
            warp_wait(&bars[B_GATE + (c & 3)], (c >> 2) & 1, abort_flag, err);
            tc_fence_after();
            const TcGate& gs = gates[c & 3];
            // Gamma_rs = 2^(G_r - G_s) = a_r a_(r-1) ... a_(s+1): a running product down from the highest
            // column at or below r of the columns handled, started there with one exp2; 8 columns at a time
            auto row_pass = [&](int r, int s_lo, int s_hi, bool is_a) {
                const int top = r < s_hi ? r : s_hi;
                float run = (top == r) ? 1.f : ex2_approx(gs.G[r] - gs.G[top]);
                const float br = is_a ? gs.beta[r] : 1.f;
#pragma unroll 1
                for (int c8 = s_hi - 7; c8 >= s_lo; c8 -= 8) {
                    float s8[8];
                    tmem_ld8(taddr(tmem, 32 * wid, TM_S1 + c8), s8);
                    tmem_wait_ld();
                    float x[8];
#pragma unroll
                    for (int q = 7; q >= 0; --q) {
                        const int s = c8 + q;
                        x[q] = (is_a ? (s < r) : (s <= r)) ? br * run * s8[q] : 0.f;
                        if (s <= top && s > 0) run *= gs.a[s];
                    }
                    if (is_a) {  // A row r: beta_r Gamma_rs (k_r . k_s), s < r
                        float* dst = &sA[r * L::AS_LD + c8];
                        *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
                        *reinterpret_cast<float4*>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
                    } else {  // P row r: Gamma_rs (q_r . k_s), s <= r, bf16 hi + lo
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) split_pack_bf16(x[2 * q], x[2 * q + 1], hi[q], lo[q]);
                        const uint32_t off = sw128(r, c8 >> 3);
                        *reinterpret_cast<uint4*>(sm + L::PH + st * 8192 + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4*>(sm + L::PL + st * 8192 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                }
            };
            // (1) A rows (lanes 0-63), columns [32 wsel, 32 wsel + 32); S1 is then read only by the P rows
            if (wid < 2) row_pass(t, 32 * wsel, 32 * wsel + 31, true);
            if (wsel == 0 || wid < 2) {
                tc_fence_before();
                mbar_arrive(&bars[B_S1_FREE]);
            }
            named_bar_sync(1, 256);
            // (2) the inverse (first warpgroup), emitting T' and T''; P rows (lanes 64-127 of the second).
            // T'' and P of chunk c go into the stage buffers of chunk c - 2, free once its output has left.
            if (c >= 2 && (wsel == 0 || wid >= 2))
                warp_wait(&bars[B_P_FREE + st], ((c - 2) >> 1) & 1, abort_flag, err);
            if (wsel == 0) {
                const TEmit em{sm + L::TP, sm + L::TPP + st * 8192, sm + L::TPPL + st * 8192, gs.beta, gs.eG};
                invert_unit_lower64(sA, wid, lane, 3, em);
                fence_proxy_async();
                mbar_arrive(&bars[B_TP_READY]);
            } else if (wid >= 2) {
                row_pass(t - 64, 0, 63, false);
                tc_fence_before();
                mbar_arrive(&bars[B_S1_FREE]);
            }
            // (3) -W^T line i = t, columns r of this warpgroup's half
            warp_wait(&bars[B_W_FULL], c & 1, abort_flag, err);
            if (c >= 1) warp_wait(&bars[B_U_FULL], (c - 1) & 1, abort_flag, err);
            tc_fence_after();
            {
                float v[32];
                tmem_ld32(taddr(tmem, 32 * wid, TM_W + 32 * wsel), v);
                tmem_wait_ld();
                st_half_line_bf16(sm + L::WT, t, 4 * wsel, v, -1.f);
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bars[B_PREP + st]);
        }
    } else if (warp >= 12) {
        // ================================================================ state / output warpgroups
        // Warpgroups 12-15 (half 0) and 16-19 (half 1) share the serial-chain work: each splits half of U
        // into bf16 operands, refreshes half of the state (key channels [64 half, 64 half + 64)) and then
        // stages half of the chunk's output rows for the TMA store.
        const int half = (warp - 12) >> 2;
        const int j = tid & 127;  // value column (TMEM lane)
        const uint32_t lane_base = 32 * (warp & 3);
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
            // ---- U (values [32 half, 32 half + 32)): fp32 accumulator -> bf16 hi/lo pairs.
            // U (for O2) goes to TM_UF (hi of values 0-63 in columns 0-31, lo in 32-63); U diag f (for h^T)
            // in place over its own fp32 columns of TM_U as [hi | lo], 16 columns each.
            if (!warp_wait(&bars[B_U_FULL], c & 1, abort_flag, err)) break;
            if (!warp_wait(&bars[B_GATE + (c & 3)], (c >> 2) & 1, abort_flag, err)) break;
            tc_fence_after();
            {
                float u[32];
                tmem_ld32(taddr(tmem, lane_base, TM_U + 32 * half), u);
                tmem_wait_ld();
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) split_pack_bf16(u[2 * q], u[2 * q + 1], hi[q], lo[q]);
                tmem_st16u(taddr(tmem, lane_base, TM_UF + 16 * half), hi);
                tmem_st16u(taddr(tmem, lane_base, TM_UF + 32 + 16 * half), lo);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int s0 = 32 * half + 2 * q;
                    split_pack_bf16(u[2 * q] * gs.f[s0], u[2 * q + 1] * gs.f[s0 + 1], hi[q], lo[q]);
                }
                tmem_st16u(taddr(tmem, lane_base, TM_U + 32 * half), hi);
                tmem_st16u(taddr(tmem, lane_base, TM_U + 32 * half + 16), lo);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[B_U_CONV]);
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
                    st_half_line_bf16(sm + L::HT + (piece >> 1) * 16384, j, 4 * (piece & 1), v);
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
            // ---- output rows [32 half, 32 half + 32): o_r = scale (2^G_r O1_r + O2_r), 8 rows at a time
            if (!warp_wait(&bars[B_O_FULL], c & 1, abort_flag, err)) break;
            tc_fence_after();
            const int Lc = gs.L;
            const int st = c & 1;
            const size_t tok0 = (size_t)row * T + bos + (size_t)c * kChunk;
            const size_t ostride = (size_t)H * dv;
            size_t off = ((tok0 + 32 * half) * H + h) * (size_t)dv + j0 + j;
            const uint32_t rg0 = half ? L::TPP : L::PH, rg1 = half ? L::TPPL : L::PL;
#pragma unroll 1
            for (int r8 = 32 * half; r8 < 32 * half + 32; r8 += 8) {
                float v1[8], v2[8];
                tmem_ld8(taddr(tmem, lane_base, TM_O1 + r8), v1);
                tmem_ld8(taddr(tmem, lane_base, TM_O2 + r8), v2);
                tmem_wait_ld();
                if (r8 == 32 * half + 24) {
                    tc_fence_before();
                    mbar_arrive(&bars[B_O_FREE]);
                }
                uint8_t* stg = sm + ((r8 & 16) ? rg1 : rg0) + st * 8192;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int r = r8 + q;
                    const float val = p.scale * fmaf(gs.eG[r], v1[q], v2[q]);
                    if (Lc == kChunk) {  // staged for the TMA store: row r & 15 of a [16][128] box
                        if (O_F32) reinterpret_cast<float*>(stg)[(r & 15) * kTcDV + j] = val;
                        else reinterpret_cast<__nv_bfloat16*>(stg)[(r & 15) * kTcDV + j] = __float2bfloat16_rn(val);
                    } else if (r < Lc) {
                        if (O_F32) static_cast<float*>(p.o)[off] = val;
                        else static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(val);
                    }
                    off += ostride;
                }
            }
            fence_proxy_async();
            mbar_arrive(&bars[B_O_STAGED]);
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
inline bool tc_supported(const FwdParams& p, bool gdn2, bool /*o_f32*/) {
    return !gdn2 && p.dk == kTcDK && p.dv % kTcDV == 0 && p.T > 0;
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

// 3-D map over the [rows, H, dv] output (fp32 or bf16), box 128 x 1 x 16 (one CTA's columns, 16 tokens),
// no swizzle: the store source is a row-major [16][128] tile.
inline bool make_out_map(CUtensorMap* map, void* base, int dv, int H, long long rows, bool f32) {
    PFN_encodeTiled enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t es = f32 ? 4 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)dv, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)dv * es, (cuuint64_t)dv * H * es};
    const cuuint32_t box[3] = {(cuuint32_t)kTcDV, 1, 16};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline gdn_status launch_tc(const FwdParams& p, bool gdn2, bool o_f32, unsigned* err, cudaStream_t stream) {
    if (gdn2) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "GDN-2 has no tcgen05 kernel yet");
        return GDN_ERR_UNSUPPORTED;
    }
    CUtensorMap mq, mk, mv, mo;
    const long long rows = (long long)p.B * p.T;
    if (!make_map(&mq, p.q, p.dk, p.H, rows) || !make_map(&mk, p.k, p.dk, p.H, rows) ||
        !make_map(&mv, p.v, p.dv, p.H, rows) || !make_out_map(&mo, p.o, p.dv, p.H, rows, o_f32)) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cuTensorMapEncodeTiled failed");
        return GDN_ERR_CUDA;
    }
    auto kern = o_f32 ? gdn_tc_fwd_kernel<true> : gdn_tc_fwd_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcSmem::ALLOC);
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    const unsigned grid = (unsigned)(p.dv / kTcDV) * p.H * p.n_seq;
    kern<<<grid, kTcThreads, TcSmem::ALLOC, stream>>>(mq, mk, mv, mo, p, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "%s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

}  // namespace gdn
