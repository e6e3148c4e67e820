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
// ahead; 2 issues the serial MMAs (U^T, O^T, h^T); 3 idle; 4-7 and 8-11 (two prep warpgroups, one per half
// of the 64 chunk columns) build A, P, T', T'' and -W^T, the first of them also (I+A)^-1; 12-15 (state
// warpgroup) split U into bf16 operands, refresh the bf16 copy of h^T, re-scale the fp32 state by the next
// chunk's decay and write hT; 16-19 (output warpgroup) write o.
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
    B_TP_READY = 12,  // T' written (256)
    B_W_FULL = 13,    // W^T in TMEM
    B_PREP = 14,      // [2] T'', -W^T, P ready for the serial step (256)
    B_P_FREE = 16,    // [2] O^T MMA reading P done
    B_U_FULL = 18,    // U^T in TMEM (and -W^T, T'' no longer read)
    B_U_CONV = 19,    // U, U.f split into bf16 hi/lo in TMEM (128)
    B_H_FULL = 20,    // h^T MMA done
    B_H_READY = 21,   // bf16 h^T staged in shared memory (128)
    B_O_FULL = 22,    // O^T MMAs done
    B_O_FREE = 23,    // O^T TMEM read (128)
    B_DRAIN = 24,     // [2] final commit of each MMA issuer
    B_HM_READY = 26,  // fp32 state in TMEM re-scaled by the next chunk's decay (128)
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

// (I + A)^-1 for a strictly lower-triangular 64x64 A in the [64][68] fp32 scratch (upper triangle 0), by
// the 4 warps of one warpgroup.  On return the diagonal 16x16 blocks hold T_ii in place, each
// off-diagonal block T_ij (i > j) is stored transposed in the upper-triangle block (j, i), and the lower
// off-diagonal blocks of A are left intact.  Steps: the four diagonal blocks by forward substitution (one
// column per lane); T_10 = -T_11 A_10 T_00 and T_32 = -T_33 A_32 T_22; then the lower-left 32x32 quarter
// T_c = -T_b (A_c T_a), where T_a, T_b are the inverses of the two diagonal 32x32 quarters -- each block
// product on tf32 MMAs, at most two per warp per step.
__device__ __forceinline__ void invert_unit_lower64(float* S, int wid, int lane, uint32_t bar_id) {
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
    // T_c = -T_b X: T_2q = -T_22 X_2q ; T_3q = -(T_32 X_2q + T_33 X_3q)
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
        named_bar_sync(bar_id, 128);  // every X block has been read
        store16(S, 16 * p, 16 * q, true, lane, y, -1.f);
    }
    named_bar_sync(bar_id, 128);
}
// Element (r, s) of T = (I + A)^-1 as left by invert_unit_lower64.
__device__ __forceinline__ float t_elem(const float* S, int r, int s) {
    if (s > r) return 0.f;
    return ((r >> 4) == (s >> 4)) ? S[r * TcSmem::AS_LD + s] : S[s * TcSmem::AS_LD + r];
}

// ------------------------------------------------------------------------------------------ the kernel
template <bool O_F32>
__global__ void __launch_bounds__(kTcThreads, 1)
gdn_tc_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p, unsigned* err) {
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
            const uint32_t cnt =
                (b == B_S1_FREE || b == B_TP_READY || b == B_PREP || b == B_PREP + 1)
                    ? 256u
                    : ((b == B_U_CONV || b == B_O_FREE || b == B_H_READY || b == B_HM_READY) ? 128u : 1u);
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
        load_kq(0);
        make_gates(0);
        if (nc > 1) {
            load_kq(1);
            make_gates(1);
        }
        load_v(0);
        for (int c = 0; c < nc; ++c) {
            if (c + 1 < nc) {
                if (!warp_wait(&bars[B_V_EMPTY], c & 1, abort_flag, err)) break;
                load_v(c + 1);
            }
            if (c + 2 < nc) {
                if (!warp_wait(&bars[B_KQ_EMPTY + (c & 1)], (c >> 1) & 1, abort_flag, err)) break;
                load_kq(c + 2);
                make_gates(c + 2);
            }
        }
        // drain: wait for every load this warp issued before the CTA may exit
        for (int st = 0; st < 2; ++st)
            if (kq_issued[st] > 0) drain_wait(&bars[B_KQ_FULL + st], (kq_issued[st] - 1) & 1);
        if (v_issued > 0) drain_wait(&bars[B_V_FULL], (v_issued - 1) & 1);
    } else if (warp == 1) {
        // ================================================================ h-independent MMAs (S1, W^T)
        if (lane == 0) {
            const uint32_t id_s1 = idesc_bf16(128, 64, false, false);
            const uint32_t id_w = idesc_bf16(128, 64, true, false);
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1;
                const uint32_t kq = sbase + L::KQ + st * L::KQ_STAGE;
                if (!mbar_wait(&bars[B_KQ_FULL + st], (c >> 1) & 1, abort_flag, err)) break;
                if (c >= 1 && !mbar_wait(&bars[B_S1_FREE], (c - 1) & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_bf16(tmem + TM_S1, desc_k_sw128(a), desc_k_sw128(a), id_s1, kk > 0);
                }
                umma_commit(&bars[B_S1_FULL]);
                if (!mbar_wait(&bars[B_TP_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_W, desc_mn_sw128(kq + kk * 2048, 16384),
                              desc_k_sw128(sbase + L::TP + kk * 32), id_w, kk > 0);
                umma_commit(&bars[B_W_FULL]);
            }
            umma_commit(&bars[B_DRAIN]);
            drain_wait(&bars[B_DRAIN], 0);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================================================================ serial MMAs (U^T, O^T, h^T)
        if (lane == 0) {
            const uint32_t id_u1 = idesc_bf16(128, 64, true, false);
            const uint32_t id_u2 = idesc_bf16(128, 64, false, true);
            const uint32_t id_o = idesc_bf16(128, 64, false, false);
            const uint32_t id_h = idesc_bf16(128, 128, false, true);
            for (int c = 0; c < nc; ++c) {
                const int st = c & 1;
                const uint32_t kq = sbase + L::KQ + st * L::KQ_STAGE;
                if (!mbar_wait(&bars[B_PREP + st], (c >> 1) & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[B_V_FULL], c & 1, abort_flag, err)) break;
                tc_fence_after();
                // U^T = V^T (T''_hi + T''_lo)^T - h^T W^T ; the first half does not need the state
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + TM_U, desc_mn_sw128(sbase + L::V + (kk & 3) * 2048, 8192),
                              desc_k_sw128(sbase + (kk < 4 ? L::TPP : L::TPPL) + st * 8192 + (kk & 3) * 32), id_u1,
                              kk > 0);
                if (!mbar_wait(&bars[B_H_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + TM_U, desc_k_sw128(sbase + L::HT + (kk >> 2) * 16384 + (kk & 3) * 32),
                              desc_mn_sw128(sbase + L::WT + kk * 2048, 8192), id_u2, 1);
                umma_commit(&bars[B_U_FULL]);
                umma_commit(&bars[B_V_EMPTY]);
                // O1^T = h^T Q^T (scaled by 2^G_r in the epilogue)
                if (c >= 1 && !mbar_wait(&bars[B_O_FREE], (c - 1) & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + TM_O1, desc_k_sw128(sbase + L::HT + (kk >> 2) * 16384 + (kk & 3) * 32),
                              desc_k_sw128(kq + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32), id_o, kk > 0);
                // h^T += (U diag f)^T K  (hi and lo halves) ;  O2^T = U^T P^T  (hi*hi + hi*lo + lo*hi)
                if (!mbar_wait(&bars[B_U_CONV], c & 1, abort_flag, err)) break;
                if (!mbar_wait(&bars[B_HM_READY], c & 1, abort_flag, err)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // kk < 4: hi, else lo; s-step ks covers values 16 ks .. 16 ks + 15
                    const int ks = kk & 3;
                    const uint32_t a = tmem + TM_U + (ks >> 1) * 32 + (kk >> 2) * 16 + (ks & 1) * 8;
                    umma_bf16_tmem_a(tmem + TM_H, a, desc_mn_sw128(kq + ks * 2048, 16384), id_h, 1);
                }
                umma_commit(&bars[B_H_FULL]);
#pragma unroll
                for (int kk = 0; kk < 12; ++kk) {
                    const int part = kk >> 2, ks = kk & 3;  // 0: Uhi Phi, 1: Uhi Plo, 2: Ulo Phi
                    const uint32_t a = tmem + TM_UF + (part == 2 ? 32 : 0) + ks * 8;
                    const uint32_t b = sbase + (part == 1 ? L::PL : L::PH) + st * 8192 + ks * 32;
                    umma_bf16_tmem_a(tmem + TM_O2, a, desc_k_sw128(b), id_o, kk > 0);
                }
                umma_commit(&bars[B_O_FULL]);
                umma_commit(&bars[B_KQ_EMPTY + st]);
                umma_commit(&bars[B_P_FREE + st]);
            }
            umma_commit(&bars[B_DRAIN + 1]);
            drain_wait(&bars[B_DRAIN + 1], 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 12) {
        // ================================================================ prep warpgroups
        // A timed-out wait does not break out here: the warpgroups finish the iteration (with whatever data)
        // and leave together at the top of the next one, so no thread is left waiting at a named barrier.
        const int wsel = (warp - 4) >> 2;      // 0: chunk columns 0-31, 1: columns 32-63
        const int t = (tid - 128) & 127;       // row of S1 / line of W^T (TMEM lane)
        const int wid = warp & 3;
        const int tp = tid - 128;              // 0..255 across both warpgroups
        for (int c = 0; c < nc; ++c) {
            if (named_bar_or(2, 256, *abort_flag != 0)) break;
            const int st = c & 1;
            warp_wait(&bars[B_S1_FULL], c & 1, abort_flag, err);
            tc_fence_after();
            warp_wait(&bars[B_GATE + (c & 3)], (c >> 2) & 1, abort_flag, err);
            const TcGate& gs = gates[c & 3];
            if (t >= 64 && c >= 2) warp_wait(&bars[B_P_FREE + st], ((c - 2) >> 1) & 1, abort_flag, err);
            // Gamma_rs = 2^(G_r - G_s) = a_r a_(r-1) ... a_(s+1): a running product from the highest column of
            // this half at or below r, started there with one exp2; 8 columns at a time, highest first
            {
                const int r = t & 63;
                const int s_hi = 32 * wsel + 31;
                const int top = r < s_hi ? r : s_hi;
                float run = (top == r) ? 1.f : ex2_approx(gs.G[r] - gs.G[top]);
                const float br = (t < 64) ? gs.beta[r] : 1.f;
#pragma unroll 1
                for (int ch = 3; ch >= 0; --ch) {
                    float s8[8];
                    tmem_ld8(taddr(tmem, 32 * wid, TM_S1 + 32 * wsel + 8 * ch), s8);
                    tmem_wait_ld();
                    float x[8];
#pragma unroll
                    for (int q = 7; q >= 0; --q) {
                        const int s = 32 * wsel + 8 * ch + q;
                        x[q] = (t < 64 ? (s < r) : (s <= r)) ? br * run * s8[q] : 0.f;
                        if (s <= top && s > 0) run *= gs.a[s];
                    }
                    if (t < 64) {  // A row r: beta_r Gamma_rs (k_r . k_s), s < r
                        float* dst = &sA[r * L::AS_LD + 32 * wsel + 8 * ch];
                        *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
                        *reinterpret_cast<float4*>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
                    } else {  // P row r: Gamma_rs (q_r . k_s), s <= r, bf16 hi + lo
                        float xh[8], xl[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) split_bf16(x[q], xh[q], xl[q]);
                        const uint32_t off = sw128(r, 4 * wsel + ch);
                        *reinterpret_cast<uint4*>(sm + L::PH + st * 8192 + off) =
                            make_uint4(pack_bf16(xh[0], xh[1]), pack_bf16(xh[2], xh[3]), pack_bf16(xh[4], xh[5]),
                                       pack_bf16(xh[6], xh[7]));
                        *reinterpret_cast<uint4*>(sm + L::PL + st * 8192 + off) =
                            make_uint4(pack_bf16(xl[0], xl[1]), pack_bf16(xl[2], xl[3]), pack_bf16(xl[4], xl[5]),
                                       pack_bf16(xl[6], xl[7]));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[B_S1_FREE]);
            named_bar_sync(1, 256);
            if (wsel == 0) invert_unit_lower64(sA, wid, lane, 3);
            named_bar_sync(1, 256);
            {  // T' = T diag(beta 2^G) (bf16) and T'' = T diag(beta) (bf16 hi + lo), [r][s] K-major
                const int r = tp >> 2, qd = tp & 3;  // 16 columns [16 qd, 16 qd + 16) of row r
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    float x1[8], xh[8], xl[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int s = 16 * qd + 8 * ch + q;
                        const float tb = t_elem(sA, r, s) * gs.beta[s];
                        x1[q] = tb * gs.eG[s];
                        split_bf16(tb, xh[q], xl[q]);
                    }
                    const uint32_t off = sw128(r, 2 * qd + ch);
                    *reinterpret_cast<uint4*>(sm + L::TP + off) =
                        make_uint4(pack_bf16(x1[0], x1[1]), pack_bf16(x1[2], x1[3]), pack_bf16(x1[4], x1[5]),
                                   pack_bf16(x1[6], x1[7]));
                    *reinterpret_cast<uint4*>(sm + L::TPP + st * 8192 + off) =
                        make_uint4(pack_bf16(xh[0], xh[1]), pack_bf16(xh[2], xh[3]), pack_bf16(xh[4], xh[5]),
                                   pack_bf16(xh[6], xh[7]));
                    *reinterpret_cast<uint4*>(sm + L::TPPL + st * 8192 + off) =
                        make_uint4(pack_bf16(xl[0], xl[1]), pack_bf16(xl[2], xl[3]), pack_bf16(xl[4], xl[5]),
                                   pack_bf16(xl[6], xl[7]));
                }
            }
            fence_proxy_async();
            mbar_arrive(&bars[B_TP_READY]);
            warp_wait(&bars[B_W_FULL], c & 1, abort_flag, err);
            if (c >= 1) warp_wait(&bars[B_U_FULL], (c - 1) & 1, abort_flag, err);
            tc_fence_after();
            {  // -W^T line i = t, columns r of this half
                float v[32];
                tmem_ld32(taddr(tmem, 32 * wid, TM_W + 32 * wsel), v);
                tmem_wait_ld();
                st_half_line_bf16(sm + L::WT, t, 4 * wsel, v, -1.f);
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&bars[B_PREP + st]);
        }
    } else if (warp >= 12 && warp < 16) {
        // ================================================================ state warpgroup
        const int j = tid & 127;  // value column (TMEM lane)
        const uint32_t lane_base = 32 * (warp & 3);
        // initial state: bf16 copy and fp32 master pre-scaled by the first chunk's decay
        if (warp_wait(&bars[B_GATE + 0], 0, abort_flag, err)) {
            const float g0 = gates[0].gamma;
#pragma unroll 1
            for (int piece = 0; piece < 4; ++piece) {
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
            // ---- U: fp32 accumulator -> bf16 hi/lo pairs for U and U diag f
            if (!warp_wait(&bars[B_U_FULL], c & 1, abort_flag, err)) break;
            if (!warp_wait(&bars[B_GATE + (c & 3)], (c >> 2) & 1, abort_flag, err)) break;
            tc_fence_after();
            // U (for O2) as bf16 hi/lo pairs in TM_UF: hi of values 0-63 in columns 0-31, lo in 32-63.
            // U diag f (for h^T) in place in TM_U, per 32 values: [hi 0-31 | lo 0-31 | hi 32-63 | lo 32-63],
            // 16 columns each -- every column is read (as fp32) before it is overwritten.
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
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
            // ---- state refresh: bf16 copy for the next chunk's MMAs, fp32 master times the next decay
            if (!warp_wait(&bars[B_H_FULL], c & 1, abort_flag, err)) break;
            const bool last = c + 1 == nc;
            if (!last && !warp_wait(&bars[B_GATE + ((c + 1) & 3)], ((c + 1) >> 2) & 1, abort_flag, err)) break;
            tc_fence_after();
            const float gn = last ? 1.f : gates[(c + 1) & 3].gamma;
            // pass 1: the bf16 copy (what the next chunk's first MMAs wait for), or hT after the last chunk
#pragma unroll 1
            for (int piece = 0; piece < 4; ++piece) {
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
                for (int piece = 0; piece < 4; ++piece) {
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
    } else if (warp >= 16) {
        // ================================================================ output warpgroup
        // o_r = scale (2^G_r O1_r + O2_r), read from TMEM 8 rows at a time
        const int j = tid & 127;  // value column (TMEM lane)
        const uint32_t lane_base = 32 * (warp & 3);
        for (int c = 0; c < nc; ++c) {
            const TcGate& gs = gates[c & 3];
            if (!warp_wait(&bars[B_GATE + (c & 3)], (c >> 2) & 1, abort_flag, err)) break;
            if (!warp_wait(&bars[B_O_FULL], c & 1, abort_flag, err)) break;
            tc_fence_after();
            const int Lc = gs.L;
            const size_t tok0 = (size_t)row * T + bos + (size_t)c * kChunk;
            const size_t ostride = (size_t)H * dv;
            size_t off = (tok0 * H + h) * (size_t)dv + j0 + j;
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
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int r = r8 + q;
                    if (r < Lc) {
                        const float val = p.scale * fmaf(gs.eG[r], v1[q], v2[q]);
                        if (O_F32) static_cast<float*>(p.o)[off] = val;
                        else static_cast<__nv_bfloat16*>(p.o)[off] = __float2bfloat16_rn(val);
                    }
                    off += ostride;
                }
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

inline gdn_status launch_tc(const FwdParams& p, bool gdn2, bool o_f32, unsigned* err, cudaStream_t stream) {
    if (gdn2) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "GDN-2 has no tcgen05 kernel yet");
        return GDN_ERR_UNSUPPORTED;
    }
    CUtensorMap mq, mk, mv;
    const long long rows = (long long)p.B * p.T;
    if (!make_map(&mq, p.q, p.dk, p.H, rows) || !make_map(&mk, p.k, p.dk, p.H, rows) ||
        !make_map(&mv, p.v, p.dv, p.H, rows)) {
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
    kern<<<grid, kTcThreads, TcSmem::ALLOC, stream>>>(mq, mk, mv, p, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(t_tc_msg, sizeof(t_tc_msg), "%s", cudaGetErrorString(e));
        return GDN_ERR_CUDA;
    }
    return GDN_OK;
}

}  // namespace gdn
