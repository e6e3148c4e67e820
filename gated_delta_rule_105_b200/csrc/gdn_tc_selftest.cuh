// Self-test of the tcgen05 operand layouts used by the tensor-core kernel: a single CTA stages A and B in
// shared memory in one of the canonical 128B-swizzled layouts, runs the MMA k-step loop the kernel uses,
// and copies the fp32 accumulator out of tensor memory.  The host compares with A * B.
//
// mode 0: A K-major  [128 x 128] (two 64-column panels, 16 KB apart), B K-major  [N=64  x K=128] (panels 8 KB apart)
// mode 1: A MN-major [M=128 x K=64] (M blocks 8 KB apart),           B K-major  [N=64  x K=64]
// mode 2: A K-major  [128 x 64],                                     B MN-major [K=64  x N=128] (N blocks 8 KB apart)
// mode 3: A K-major  [128 x 128] (two panels),                       B MN-major [K=128 x N=64]
// mode 4: A in tensor memory [128 x 64] (bf16 pairs per column),      B K-major  [N=64  x K=64]
// mode 5: kind::tf32, A in tensor memory [128 x 32] (fp32, one per column), B K-major fp32  [N=64 x K=32]
#pragma once

#include "gdn_sm100.cuh"

namespace gdn {

struct SelftestShape {
    int M, N, K;
};
__host__ __device__ inline SelftestShape selftest_shape(int mode) {
    switch (mode) {
        case 0: return {128, 64, 128};
        case 1: return {128, 64, 64};
        case 2: return {128, 128, 64};
        case 4: return {128, 64, 64};
        case 5: return {128, 64, 32};
        default: return {128, 64, 128};
    }
}

// A: row-major [M][K] fp32, B: row-major [K][N] fp32, D: row-major [M][N] fp32.
__global__ void __launch_bounds__(128) gdn_umma_selftest_kernel(const float* A, const float* B, float* D, int mode,
                                                               unsigned* err) {
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;            // 32 KB
    uint8_t* sB = base + 32768;    // 32 KB
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    const SelftestShape s = selftest_shape(mode);
    const int tid = threadIdx.x, warp = tid / 32;

    // ---- stage A
    if (mode == 1) {
        // MN-major: line = k (0..63), 64 M elements per line, M block b at b * 8192
        for (int e = tid; e < s.M * s.K; e += 128) {
            const int m = e % s.M, k = e / s.M;
            const int blk = m / 64, mm = m % 64;
            uint8_t* p = sA + blk * 8192 + sw128(k, mm / 8) + (mm % 8) * 2;
            *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(A[m * s.K + k]);
        }
    } else if (mode < 4) {
        // K-major: line = m, 64 K per line, K panel p at p * 16384
        for (int e = tid; e < s.M * s.K; e += 128) {
            const int m = e / s.K, k = e % s.K;
            const int pnl = k / 64, kk = k % 64;
            uint8_t* p = sA + pnl * 16384 + sw128(m, kk / 8) + (kk % 8) * 2;
            *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(A[m * s.K + k]);
        }
    }
    // ---- stage B
    if (mode == 5) {  // K-major fp32: line = n, 32 K per 128-byte line
        for (int e = tid; e < s.K * s.N; e += 128) {
            const int k = e / s.N, n = e % s.N;
            *reinterpret_cast<float*>(sB + sw128(n, k / 4) + (k % 4) * 4) = B[k * s.N + n];
        }
    } else if (mode == 2 || mode == 3) {
        // MN-major: line = k, 64 N per line, N block b at b * 8192 (mode 2); mode 3 has one N block of 128 lines
        for (int e = tid; e < s.K * s.N; e += 128) {
            const int k = e / s.N, n = e % s.N;
            const int blk = n / 64, nn = n % 64;
            uint8_t* p = sB + blk * 8192 + sw128(k, nn / 8) + (nn % 8) * 2;
            *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(B[k * s.N + n]);
        }
    } else {
        // K-major: line = n, 64 K per line, K panel p at p * 8192
        for (int e = tid; e < s.K * s.N; e += 128) {
            const int k = e / s.N, n = e % s.N;
            const int pnl = k / 64, kk = k % 64;
            uint8_t* p = sB + pnl * 8192 + sw128(n, kk / 8) + (kk % 8) * 2;
            *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(B[k * s.N + n]);
        }
    }
    fence_proxy_async();
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base;
    if (mode == 4) {  // A rows into tensor memory columns 64..95, two bf16 per column
        const int m = warp * 32 + (tid % 32);
        uint32_t packed[32];
        for (int c = 0; c < 32; ++c) packed[c] = pack_bf16(A[m * s.K + 2 * c], A[m * s.K + 2 * c + 1]);
        tmem_st32u(taddr(tb, warp * 32, 64), packed);
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (mode == 5) {  // A rows into tensor memory columns 64..95, one fp32 per column
        const int m = warp * 32 + (tid % 32);
        float row[32];
        for (int c = 0; c < 32; ++c) row[c] = A[m * s.K + c];
        tmem_st32(taddr(tb, warp * 32, 64), row);
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (tid == 0 && mode == 5) {
        const uint32_t b0 = smem_u32(sB);
        for (int kk = 0; kk < s.K / 8; ++kk)
            umma_tf32_tmem_a(tb, tb + 64 + kk * 8, desc_k_sw128(b0 + kk * 32), idesc_tf32(s.M, s.N, false, false),
                             kk > 0 ? 1u : 0u);
        umma_commit(&bar);
    } else if (tid == 0) {
        const uint32_t idesc = idesc_bf16(s.M, s.N, mode == 1, mode == 2 || mode == 3);
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        for (int kk = 0; kk < s.K / 16; ++kk) {
            uint64_t ad, bd;
            if (mode == 1) ad = desc_mn_sw128(a0 + kk * 2048, 8192);
            else ad = desc_k_sw128(a0 + (kk / 4) * 16384 + (kk % 4) * 32);
            if (mode == 2) bd = desc_mn_sw128(b0 + kk * 2048, 8192);
            else if (mode == 3) bd = desc_mn_sw128(b0 + kk * 2048, 16384);
            else bd = desc_k_sw128(b0 + (kk / 4) * 8192 + (kk % 4) * 32);
            if (mode == 4) umma_bf16_tmem_a(tb, tb + 64 + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
            else umma_bf16(tb, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bar);
    }
    __syncwarp();
    const bool ok = mbar_wait(&bar, 0, &abort_flag, err);
    tc_fence_after();
    if (ok) {
        const int row = warp * 32 + (tid % 32);
        for (int c0 = 0; c0 < s.N; c0 += 32) {
            float v[32];
            tmem_ld32(taddr(tb, warp * 32, c0), v);
            tmem_wait_ld();
            for (int j = 0; j < 32; ++j) D[row * s.N + c0 + j] = v[j];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 128);
}

}  // namespace gdn
