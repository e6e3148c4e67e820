// Register-blocked chunk products of the backward's walks along a sequence (256 threads, 32 value columns).
//
// The state-cotangent walk (and the GDN-2 forward state walk) repeats, chunk after chunk, a handful of small
// products between [64][dk], [64][64] and [dk][32] operands held in shared memory (Gated DeltaNet-2 article,
// section "Entrenamiento fragmentado y reconocimiento de puertas hacia atrás"; the walkthrough, section "分块并行").
// Each thread owns a 2 x 4 tile of a [64][32] result or an (dk/32) x 4 tile of a [dk][32] one and reads its
// operands as float2/float4 vectors, so one shared-memory wavefront feeds 8 to 16 FMAs instead of half of one.
//
// Layout: value tiles [rows][kTileLdv] (32 columns + 4 of padding, 16-byte rows); the [64][ld] row operands have
// ld a multiple of 4 and ld / 4 odd in its low bits so that the rows a warp reads fall in distinct banks.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

constexpr int kTileThreads = 256;       // the walks' block size
constexpr int kTileDv = 32;             // value columns per CTA
constexpr int kTileLdv = kTileDv + 4;   // row stride of a value tile (floats)

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float2 lds2(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ void sts4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void fma4(float (&acc)[4], float a, const float4& x) {
    acc[0] = fmaf(a, x.x, acc[0]);
    acc[1] = fmaf(a, x.y, acc[1]);
    acc[2] = fmaf(a, x.z, acc[2]);
    acc[3] = fmaf(a, x.w, acc[3]);
}

// The thread's tile of a [64][32] result: rows s0, s0 + 1, columns j0 .. j0 + 3.  A warp covers rows 8w .. 8w + 7.
__device__ __forceinline__ int tile_s0() { return 2 * (threadIdx.x >> 3); }
__device__ __forceinline__ int tile_j0() { return 4 * (threadIdx.x & 7); }
__device__ __forceinline__ int tile_warp_row() { return 8 * (threadIdx.x >> 5); }

// acc[u][c] += sum_{r = r0}^{63} A[r][s0 + u] X[r][j0 + c]   (A^T X; for a lower-triangular A the rows above the
// warp's first row 8w are zero in every column the warp owns, so r0 = 8w is exact)
template <int LDA>
__device__ __forceinline__ void tile_acc_AtX(const float* A, const float* X, int r0, float (&acc)[2][4]) {
    const int s0 = tile_s0(), j0 = tile_j0();
#pragma unroll 4
    for (int r = r0; r < kChunk; ++r) {
        const float2 a = lds2(A + r * LDA + s0);
        const float4 x = lds4(X + r * kTileLdv + j0);
        fma4(acc[0], a.x, x);
        fma4(acc[1], a.y, x);
    }
}

// acc[u][c] += sum_{i < kend} A[s0 + u][i] D[i][j0 + c]   (A D; kend a multiple of 4)
template <int LDA>
__device__ __forceinline__ void tile_acc_AD(const float* A, const float* D, int kend, float (&acc)[2][4]) {
    const int s0 = tile_s0(), j0 = tile_j0();
#pragma unroll 2
    for (int i = 0; i < kend; i += 4) {
        const float4 a0 = lds4(A + s0 * LDA + i), a1 = lds4(A + (s0 + 1) * LDA + i);
        const float4 d0 = lds4(D + (i + 0) * kTileLdv + j0), d1 = lds4(D + (i + 1) * kTileLdv + j0);
        const float4 d2 = lds4(D + (i + 2) * kTileLdv + j0), d3 = lds4(D + (i + 3) * kTileLdv + j0);
        fma4(acc[0], a0.x, d0);
        fma4(acc[0], a0.y, d1);
        fma4(acc[0], a0.z, d2);
        fma4(acc[0], a0.w, d3);
        fma4(acc[1], a1.x, d0);
        fma4(acc[1], a1.y, d1);
        fma4(acc[1], a1.z, d2);
        fma4(acc[1], a1.w, d3);
    }
}

// The same product over the full key width DK, as 4 x 4 blocks (rows 4 (tid / 16) .. + 3, the thread's columns) whose
// sum over i is split between the two lanes 8 apart (each sums half of DK); a shuffle combines the halves and
// each lane adds its own two rows s0, s0 + 1 to acc.  One 16-byte load feeds 16 FMAs instead of 8.  Called by
// every thread of the warp.
template <int DK, int LDA>
__device__ __forceinline__ void tile_acc_AD_split(const float* A, const float* D, float (&acc)[2][4]) {
    const int j0 = tile_j0(), pb = 4 * (threadIdx.x >> 4), kq = (threadIdx.x >> 3) & 1;
    float b[4][4] = {};
#pragma unroll 2
    for (int i = kq * (DK / 2); i < (kq + 1) * (DK / 2); i += 4) {
        float4 d[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) d[q] = lds4(D + (i + q) * kTileLdv + j0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 a = lds4(A + (pb + u) * LDA + i);
            fma4(b[u], a.x, d[0]);
            fma4(b[u], a.y, d[1]);
            fma4(b[u], a.z, d[2]);
            fma4(b[u], a.w, d[3]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q) b[u][q] += __shfl_xor_sync(0xffffffffu, b[u][q], 8);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        acc[0][q] += kq == 0 ? b[0][q] : b[2][q];
        acc[1][q] += kq == 0 ? b[1][q] : b[3][q];
    }
}

// The thread's tile of a [DK][32] result: rows i0 .. i0 + DK/32 - 1, columns j0 .. j0 + 3.
template <int DK>
__device__ __forceinline__ int tile_i0() { return (DK / 32) * (threadIdx.x >> 3); }

// acc[u][c] += sum_{r < 64} A[r][i0 + u] X[r][j0 + c]   (A^T X with A a [64][DK] row operand)
template <int DK, int LDA>
__device__ __forceinline__ void tile_acc_KtX(const float* A, const float* X, float (&acc)[DK / 32][4]) {
    static_assert(DK == 64 || DK == 128, "key width");
    const int i0 = tile_i0<DK>(), j0 = tile_j0();
#pragma unroll 4
    for (int r = 0; r < kChunk; ++r) {
        const float4 x = lds4(X + r * kTileLdv + j0);
        if constexpr (DK == 128) {
            const float4 a = lds4(A + r * LDA + i0);
            fma4(acc[0], a.x, x);
            fma4(acc[1], a.y, x);
            fma4(acc[2], a.z, x);
            fma4(acc[3], a.w, x);
        } else {
            const float2 a = lds2(A + r * LDA + i0);
            fma4(acc[0], a.x, x);
            fma4(acc[1], a.y, x);
        }
    }
}

// acc += A1^T X1 (+ A2^T X2 when A2 is given) on the thread's [DK][32] tile, for DK = 128 as 8 x 4 blocks (channels
// 8 (tid / 16) .. + 7, the thread's columns) whose sum over the 64 rows is split between the two lanes 8 apart; one
// shuffle combines the halves of both products and each lane adds its own four channels.  12 wavefronts feed 32
// FMAs per lane instead of 8 feeding 16.  Other widths use tile_acc_KtX.  Called by every thread of the warp.
template <int DK, int LDA>
__device__ __forceinline__ void tile_acc_KtX_split(const float* A1, const float* X1, const float* A2, const float* X2,
                                                   float (&acc)[DK / 32][4]) {
    if constexpr (DK != 128) {
        tile_acc_KtX<DK, LDA>(A1, X1, acc);
        if (A2) tile_acc_KtX<DK, LDA>(A2, X2, acc);
    } else {
        const int j0 = tile_j0(), cb = 8 * (threadIdx.x >> 4), kq = (threadIdx.x >> 3) & 1;
        float b[8][4] = {};
        for (int pass = 0; pass < (A2 ? 2 : 1); ++pass) {
            const float* A = pass ? A2 : A1;
            const float* X = pass ? X2 : X1;
#pragma unroll 4
            for (int r = 32 * kq; r < 32 * kq + 32; ++r) {
                const float4 x = lds4(X + r * kTileLdv + j0);
                const float4 a0 = lds4(A + r * LDA + cb), a1 = lds4(A + r * LDA + cb + 4);
                fma4(b[0], a0.x, x);
                fma4(b[1], a0.y, x);
                fma4(b[2], a0.z, x);
                fma4(b[3], a0.w, x);
                fma4(b[4], a1.x, x);
                fma4(b[5], a1.y, x);
                fma4(b[6], a1.z, x);
                fma4(b[7], a1.w, x);
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int q = 0; q < 4; ++q) b[u][q] += __shfl_xor_sync(0xffffffffu, b[u][q], 8);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[u][q] += kq == 0 ? b[u][q] : b[u + 4][q];
    }
}

// Eight consecutive inputs (bf16 or fp32, 16-byte aligned) as floats.
__device__ __forceinline__ void ldg8(const float* src, float (&o)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(src)), b = __ldg(reinterpret_cast<const float4*>(src) + 1);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void ldg8(const __nv_bfloat16* src, float (&o)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
    const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        o[2 * m] = __uint_as_float(w[m] << 16);
        o[2 * m + 1] = __uint_as_float(w[m] & 0xffff0000u);
    }
}
// Four consecutive inputs (8-byte aligned for bf16, 16-byte for fp32) as a float4.
__device__ __forceinline__ float4 ldg4(const float* src) { return __ldg(reinterpret_cast<const float4*>(src)); }
__device__ __forceinline__ float4 ldg4(const __nv_bfloat16* src) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}

// [64][DK] rows of a [tokens][H][DK] input into shared memory ([64][ld], rows past Lc zero), 8 values a load.
template <typename TIn, int DK>
__device__ __forceinline__ void tile_load_rows(float* dst, int ld, const TIn* src, size_t tok0, int H, int h, int Lc) {
    constexpr int G8 = DK / 8;
    for (int e = threadIdx.x; e < kChunk * G8; e += kTileThreads) {
        const int r = e / G8, c = 8 * (e % G8);
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (r < Lc) ldg8(src + ((tok0 + r) * H + h) * DK + c, v);
        sts4(dst + r * ld + c, v[0], v[1], v[2], v[3]);
        sts4(dst + r * ld + c + 4, v[4], v[5], v[6], v[7]);
    }
}

// A dense fp32 [64][64] matrix (16-byte aligned) into shared memory [64][ld].
__device__ __forceinline__ void tile_load_64x64(float* dst, int ld, const float* src) {
    for (int e = threadIdx.x; e < kChunk * kChunk / 4; e += kTileThreads) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src) + e);
        *reinterpret_cast<float4*>(dst + (e >> 4) * ld + 4 * (e & 15)) = v;
    }
}

// The CTA's 32 columns of a [rows][dv] fp32 state slice (row stride dv) to and from a [rows][kTileLdv] tile.
__device__ __forceinline__ void tile_store_state(float* g, int dv, const float* s, int rows) {
    for (int e = threadIdx.x; e < rows * (kTileDv / 4); e += kTileThreads) {
        const int i = e >> 3, c = 4 * (e & 7);
        *reinterpret_cast<float4*>(g + (size_t)i * dv + c) = lds4(s + i * kTileLdv + c);
    }
}
__device__ __forceinline__ void tile_load_state(float* s, const float* g, int dv, int rows) {
    for (int e = threadIdx.x; e < rows * (kTileDv / 4); e += kTileThreads) {
        const int i = e >> 3, c = 4 * (e & 7);
        *reinterpret_cast<float4*>(s + i * kTileLdv + c) =
            g ? *reinterpret_cast<const float4*>(g + (size_t)i * dv + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// The CTA's 32 value columns of 64 token rows of a [tokens][H][dv] input (rows past Lc zero).
template <typename TIn>
__device__ __forceinline__ void tile_load_values(float* s, const TIn* src, size_t tok0, int H, int h, int dv, int j0,
                                                 int Lc) {
    for (int e = threadIdx.x; e < kChunk * (kTileDv / 4); e += kTileThreads) {
        const int r = e >> 3, c = 4 * (e & 7);
        const float4 v = r < Lc ? ldg4(src + ((tok0 + r) * H + h) * dv + j0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(s + r * kTileLdv + c) = v;
    }
}

}  // namespace gdn

namespace gdn {

// Split-sum 4 x 4 blocks of the gradient kernels' [64][16] value tiles (row stride LDV): a block covers rows
// pb .. pb + 3 and columns tc .. tc + 3, its four adjacent lanes (kq = lane % 4) each sum a quarter of the
// inner index, shuffles combine the quarters and every lane keeps row pb + kq of the block.  All 32 lanes of
// the warp must call them together.
__device__ __forceinline__ void blk_keep_row(float (&b)[4][4], int kq, float (&out)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            b[u][q] += __shfl_xor_sync(0xffffffffu, b[u][q], 1);
            b[u][q] += __shfl_xor_sync(0xffffffffu, b[u][q], 2);
        }
#pragma unroll
    for (int q = 0; q < 4; ++q) out[q] = kq == 0 ? b[0][q] : kq == 1 ? b[1][q] : kq == 2 ? b[2][q] : b[3][q];
}

// out = sum_{s <= r} T[r][s] X[s][tc ..]  for r = pb + kq (T lower triangular, zero above its diagonal)
template <int LDT, int LDV>
__device__ __forceinline__ void blk_tri_TX(const float* T, const float* X, int pb, int kq, int tc, float (&out)[4]) {
    float b[4][4] = {};
    for (int s2 = kq; s2 < pb + 4; s2 += 4) {
        const float4 x = lds4(X + s2 * LDV + tc);
#pragma unroll
        for (int u = 0; u < 4; ++u) fma4(b[u], T[(pb + u) * LDT + s2], x);
    }
    blk_keep_row(b, kq, out);
}

// out = sum_{t >= r} T[t][r] X[t][tc ..]  for r = pb + kq (T^T X; T zero above its diagonal)
template <int LDT, int LDV>
__device__ __forceinline__ void blk_tri_TtX(const float* T, const float* X, int pb, int kq, int tc,
                                            float (&out)[4]) {
    float b[4][4] = {};
    for (int t = pb + kq; t < kChunk; t += 4) {
        const float4 x = lds4(X + t * LDV + tc);
#pragma unroll
        for (int u = 0; u < 4; ++u) fma4(b[u], T[t * LDT + pb + u], x);
    }
    blk_keep_row(b, kq, out);
}

// T = (I + A)^-1 for a strictly lower-triangular 64 x 64 A (row stride ldt), 256 threads, W a [64][ldt] scratch.
// The four diagonal 16 x 16 blocks by forward substitution, one warp each (16 columns x 2 lanes splitting each
// row's sum); then the blocks below the diagonal, one block-diagonal at a time (distance d = i - j = 1, 2, 3):
// W_ij = sum_{k=j}^{i-1} A_ik T_kj, then T_ij = -T_ii W_ij.  Seven block-wide barriers instead of one per row.
// Every entry of T is written (zero above the diagonal).  Called by every thread of the block.
__device__ __forceinline__ void inv_unit_lower64(const float* A, float* T, int ldt, float* W) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp < 4) {  // diagonal block `warp`
        const int R = 16 * warp, c = lane & 15, part = lane >> 4;
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
            for (int s2 = c + part; s2 < r; s2 += 2) acc = fmaf(A[(R + r) * ldt + R + s2], T[(R + s2) * ldt + R + c], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 16);
            if (part == 0) T[(R + r) * ldt + R + c] = r < c ? 0.f : (r == c ? 1.f : -acc);
            __syncwarp();
        }
    } else {  // the six blocks above the diagonal are zero
        for (int e = tid - 128; e < 6 * 256; e += 128) {
            const int b = e >> 8, r = (e >> 4) & 15, c = e & 15;
            const int bi = b < 3 ? 0 : (b < 5 ? 1 : 2), bj = b < 3 ? b + 1 : (b < 5 ? b - 1 : 3);
            T[(16 * bi + r) * ldt + 16 * bj + c] = 0.f;
        }
    }
    __syncthreads();
    const int r = tid >> 4, c = tid & 15;
    for (int d = 1; d < 4; ++d) {
        for (int j = 0; j + d < 4; ++j) {  // W_ij = sum_k A_ik T_kj over the blocks k = j .. i - 1
            const int i = j + d;
            float acc = 0.f;
            for (int kk = 16 * j; kk < 16 * i; ++kk) acc = fmaf(A[(16 * i + r) * ldt + kk], T[kk * ldt + 16 * j + c], acc);
            W[(16 * i + r) * ldt + 16 * j + c] = acc;
        }
        __syncthreads();
        for (int j = 0; j + d < 4; ++j) {  // T_ij = -T_ii W_ij (T_ii unit lower triangular)
            const int i = j + d;
            float acc = 0.f;
            for (int t = 0; t <= r; ++t) acc = fmaf(T[(16 * i + r) * ldt + 16 * i + t], W[(16 * i + t) * ldt + 16 * j + c], acc);
            T[(16 * i + r) * ldt + 16 * j + c] = -acc;
        }
        __syncthreads();
    }
}

// A [64][W] block of rows of a bf16 or fp32 tensor (row r at src + r * row_stride elements), held as raw 16-byte
// vectors in the loading thread's registers: loaded while the previous chunk computes, stored (as fp32) into
// shared memory once its buffers are free.  Rows at or past Lc are zero.
template <typename TIn, int W>
struct RowBlock {
    static constexpr int EPV = 16 / (int)sizeof(TIn);             // elements per vector
    static constexpr int VPR = W / EPV;                           // vectors per row
    static constexpr int N = kChunk * VPR / kTileThreads;         // vectors per thread
    static_assert(W % EPV == 0 && (kChunk * VPR) % kTileThreads == 0, "block shape");
    uint4 v[N];
    __device__ __forceinline__ void load(const TIn* src, size_t row_stride, int Lc) {
#pragma unroll
        for (int m = 0; m < N; ++m) {
            const int e = threadIdx.x + m * kTileThreads, r = e / VPR, c = e % VPR;
            v[m] = r < Lc ? __ldg(reinterpret_cast<const uint4*>(src + r * row_stride + c * EPV))
                          : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    // One element at a time, for a row stride that is not a multiple of 4 (v[m] holds EPV consecutive elements).
    __device__ __forceinline__ void store_scalar(float* dst, int ld) const {
#pragma unroll
        for (int m = 0; m < N; ++m) {
            const int e = threadIdx.x + m * kTileThreads, r = e / VPR, c = e % VPR;
            float* d = dst + r * ld + c * EPV;
            const unsigned w[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if constexpr (sizeof(TIn) == 2) {
                    d[2 * q] = __uint_as_float(w[q] << 16);
                    d[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
                } else {
                    d[q] = __uint_as_float(w[q]);
                }
            }
        }
    }
    __device__ __forceinline__ void store(float* dst, int ld) const {
#pragma unroll
        for (int m = 0; m < N; ++m) {
            const int e = threadIdx.x + m * kTileThreads, r = e / VPR, c = e % VPR;
            float* d = dst + r * ld + c * EPV;
            if constexpr (sizeof(TIn) == 2) {  // bf16: the upper 16 bits of an fp32
                sts4(d, __uint_as_float(v[m].x << 16), __uint_as_float(v[m].x & 0xffff0000u),
                     __uint_as_float(v[m].y << 16), __uint_as_float(v[m].y & 0xffff0000u));
                sts4(d + 4, __uint_as_float(v[m].z << 16), __uint_as_float(v[m].z & 0xffff0000u),
                     __uint_as_float(v[m].w << 16), __uint_as_float(v[m].w & 0xffff0000u));
            } else {
                sts4(d, __uint_as_float(v[m].x), __uint_as_float(v[m].y), __uint_as_float(v[m].z),
                     __uint_as_float(v[m].w));
            }
        }
    }
};

}  // namespace gdn
