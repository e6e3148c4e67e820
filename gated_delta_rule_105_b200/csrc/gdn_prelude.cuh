// The token mixer's prelude and epilogue: elementwise, HBM-bound kernels around the chunked recurrence.
//
// Prelude (one launch): q, k and v each pass a depthwise causal convolution with 4 taps and a SiLU, q and k are
// then L2-normalised over each head's channels, and the gates are formed: g = -exp(A_log) softplus(a + dt_bias),
// beta = sigmoid(b), and for GDN-2 a second sigmoid gate.  (GatedDeltaNet data-flow walkthrough, yfxerp.com/news/
// 367755: sections "Short convolution" -- kernel size 4, SiLU, the 3 previous inputs cached at inference --,
// "Gating" -- the two gate formulas and the L2 norm of q and k; Gated DeltaNet-2 article, 7minutos.es, section
// "Diseno de bloques y modelo hibrido".)  Per channel c with taps w[c][0..3]:
//     y[t][c] = silu(w[c][0] x[t-3][c] + w[c][1] x[t-2][c] + w[c][2] x[t-1][c] + w[c][3] x[t][c])
// where inputs before a sequence start come from the conv cache (oldest first) or are 0.
// Epilogue: y = o / sqrt(mean(o^2) + eps) * weight * silu(z) over each (token, head) row of dv channels (the
// walkthrough's fused RMSNorm with a Swish gate, data-flow step 5).
#pragma once

#include "gdn_common.cuh"

namespace gdn {

constexpr int kPreTokens = 64;   // tokens per prelude CTA
constexpr int kPreThreads = 256;  // 8 warps: warp w takes the tile's rows w, w + 8, ...

struct PreludeParams {
    const void* x[3];         // xq, xk [rows, H, dk]; xv [rows, H, dv]   (rows = B T)
    const float* w[3];        // taps [H d][4] of each path
    const float* conv_in;     // [N][2 H dk + H dv][3] or null (zeros)
    float* conv_out;          // same layout, or null
    void* y[3];               // q, k [rows, H, dk]; v [rows, H, dv]
    const float* a;           // [rows, H, ga]  -> g
    const float* A_log;       // [H]
    const float* dt_bias;     // [H]
    float* g;
    const float* b;           // [rows, H, gb]  -> beta = sigmoid(b)
    float* beta;
    const float* c;           // [rows, H, gc]  -> sigmoid(c), or null
    float* wgate;
    const int32_t* cu_seqlens;
    float l2_eps;
    int B, T, H, dk, dv, ga, gb, gc, n_seq;
};

// SiLU and sigmoid with the fast exponential and divide intrinsics (relative error ~2^-21, far below the fp32
// allowance); for x below about -87 the divide returns 0, which is the limit of both functions.
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.f + __expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

// Sequence of global token row tau: its index n and first row start.
__device__ __forceinline__ void pre_seq_of(const PreludeParams& p, long long tau, int& n, long long& start) {
    if (!p.cu_seqlens) {
        n = (int)(tau / p.T);
        start = (long long)n * p.T;
        return;
    }
    int lo = 0, hi = p.n_seq - 1;  // last n with cu[n] <= tau (and cu[n + 1] > tau: skips empty sequences)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cu_seqlens[mid] <= tau) lo = mid;
        else hi = mid - 1;
    }
    n = lo;
    start = p.cu_seqlens[lo];
}

// Shared memory of one prelude CTA: the tile's input rows tau0 - 3 .. tau0 + 63 of one head (fp32), then the
// sequence index and start of each of its 64 rows.
inline size_t prelude_smem_bytes(int d) { return (size_t)(kPreTokens + 3) * d * 4 + kPreTokens * (8 + 4); }

// grid: (64-token tiles, H, 3 paths: q, k, v); the q-path CTAs also form the gates of their tokens and head.
// Each lane keeps the taps of its channels in registers; one warp per token row computes the convolution, the
// SiLU and (q, k) the row's L2 norm.
template <typename TIO>
__global__ void __launch_bounds__(kPreThreads, 3) gdn_prelude_kernel(const PreludeParams p) {
    constexpr int TT = kPreTokens;
    extern __shared__ __align__(16) float pre_sm[];
    const int path = blockIdx.z, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long rows = (long long)p.B * p.T;
    const long long tau0 = (long long)blockIdx.x * TT;
    const int H = p.H;
    const int d = path == 2 ? p.dv : p.dk;
    float* xs = pre_sm;  // [TT + 3][d]
    long long* s_start = reinterpret_cast<long long*>(pre_sm + (TT + 3) * d);
    int* s_n = reinterpret_cast<int*>(s_start + TT);

    if (path == 0) {  // ---- gates of this tile's tokens and head
        const float A = expf(p.A_log[h]), bias = p.dt_bias[h];
        for (int e = tid; e < TT * p.ga; e += kPreThreads) {
            const long long tau = tau0 + e / p.ga;
            if (tau >= rows) break;
            const size_t idx = ((size_t)tau * H + h) * p.ga + e % p.ga;
            p.g[idx] = -A * softplus_f(p.a[idx] + bias);
        }
        for (int e = tid; e < TT * p.gb; e += kPreThreads) {
            const long long tau = tau0 + e / p.gb;
            if (tau >= rows) break;
            const size_t idx = ((size_t)tau * H + h) * p.gb + e % p.gb;
            p.beta[idx] = sigmoid_f(p.b[idx]);
        }
        if (p.c)
            for (int e = tid; e < TT * p.gc; e += kPreThreads) {
                const long long tau = tau0 + e / p.gc;
                if (tau >= rows) break;
                const size_t idx = ((size_t)tau * H + h) * p.gc + e % p.gc;
                p.wgate[idx] = sigmoid_f(p.c[idx]);
            }
    }

    const int c_all = 2 * H * p.dk + H * p.dv;
    const int c_base = (path == 0 ? 0 : path == 1 ? H * p.dk : 2 * H * p.dk) + h * d;  // this head's first channel
    const TIO* x = static_cast<const TIO*>(p.x[path]);
    if (tid < TT) {
        const long long tau = tau0 + tid;
        int n = 0;
        long long st = 0;
        if (tau < rows) pre_seq_of(p, tau, n, st);
        s_n[tid] = n;
        s_start[tid] = st;
    }
    // the tile's input rows, 16 bytes of the input per load
    constexpr int VEC = 16 / sizeof(TIO);
    const int vpr = d / VEC;  // vectors per row
    for (int e = tid; e < (TT + 3) * vpr; e += kPreThreads) {
        const int r = e / vpr, c0 = (e % vpr) * VEC;
        const long long src = tau0 - 3 + r;
        float* dst = xs + r * d + c0;
        float vals[VEC];
        if (src >= 0 && src < rows) {
            const uint4 u = *reinterpret_cast<const uint4*>(x + ((size_t)src * H + h) * d + c0);
            const TIO* vv = reinterpret_cast<const TIO*>(&u);
#pragma unroll
            for (int m = 0; m < VEC; ++m) vals[m] = to_f32(vv[m]);
        } else {
#pragma unroll
            for (int m = 0; m < VEC; ++m) vals[m] = 0.f;
        }
#pragma unroll
        for (int m = 0; m < VEC; m += 4)
            *reinterpret_cast<float4*>(dst + m) = make_float4(vals[m], vals[m + 1], vals[m + 2], vals[m + 3]);
    }
    // lane l owns the channel pairs (2 l + 64 c, 2 l + 64 c + 1), c < d / 64: a warp's shared-memory reads are
    // consecutive 8-byte words (no bank conflicts) and its stores are contiguous
    const int npair = d / 64;
    float tap[8][4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
        if (c < npair)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float4 w4 = *reinterpret_cast<const float4*>(p.w[path] + ((size_t)h * d + 2 * lane + 64 * c + u) * 4);
                tap[2 * c + u][0] = w4.x, tap[2 * c + u][1] = w4.y, tap[2 * c + u][2] = w4.z, tap[2 * c + u][3] = w4.w;
            }
    __syncthreads();
    // tap j (0: oldest) of output row r for channel i of the head
    auto input = [&](int r, int j, int i) -> float {
        const long long src = tau0 + r - 3 + j, st = s_start[r];
        if (src >= st) return xs[(r + j) * d + i];
        if (!p.conv_in) return 0.f;
        return p.conv_in[((size_t)s_n[r] * c_all + c_base + i) * 3 + (int)(src - st + 3)];
    };
    TIO* y = static_cast<TIO*>(p.y[path]);
    for (int r = warp; r < TT; r += kPreThreads / 32) {
        const long long tau = tau0 + r;
        if (tau >= rows) break;
        const bool near_start = tau - s_start[r] < 3;  // a tap may reach before the sequence start
        float yv[8];
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c < npair) {
                const int i = 2 * lane + 64 * c;
                float2 acc;
                if (near_start) {
                    acc.x = tap[2 * c][0] * input(r, 0, i);
                    acc.y = tap[2 * c + 1][0] * input(r, 0, i + 1);
#pragma unroll
                    for (int j = 1; j < 4; ++j) {
                        acc.x = fmaf(tap[2 * c][j], input(r, j, i), acc.x);
                        acc.y = fmaf(tap[2 * c + 1][j], input(r, j, i + 1), acc.y);
                    }
                } else {
                    const float2 x0 = *reinterpret_cast<const float2*>(xs + r * d + i);
                    acc.x = tap[2 * c][0] * x0.x;
                    acc.y = tap[2 * c + 1][0] * x0.y;
#pragma unroll
                    for (int j = 1; j < 4; ++j) {
                        const float2 xj = *reinterpret_cast<const float2*>(xs + (r + j) * d + i);
                        acc.x = fmaf(tap[2 * c][j], xj.x, acc.x);
                        acc.y = fmaf(tap[2 * c + 1][j], xj.y, acc.y);
                    }
                }
                yv[2 * c] = silu_f(acc.x);
                yv[2 * c + 1] = silu_f(acc.y);
                ss = fmaf(yv[2 * c], yv[2 * c], fmaf(yv[2 * c + 1], yv[2 * c + 1], ss));
            }
        float inv = 1.f;
        if (path < 2) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            inv = 1.f / sqrtf(ss + p.l2_eps);
        }
        TIO* dst = y + ((size_t)tau * H + h) * d + 2 * lane;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c < npair) {
                if (sizeof(TIO) == 2) {
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(yv[2 * c] * inv, yv[2 * c + 1] * inv);
                    *reinterpret_cast<__nv_bfloat162*>(dst + 64 * c) = b2;
                } else {
                    *reinterpret_cast<float2*>(dst + 64 * c) = make_float2(yv[2 * c] * inv, yv[2 * c + 1] * inv);
                }
            }
        // the cache of a sequence that ends at this row: its last three inputs, oldest first (each lane reads its
        // channels' values before writing them, so the cache may be updated in place for T == 1)
        if (p.conv_out) {
            const int n = s_n[r];
            const long long end = p.cu_seqlens ? (long long)p.cu_seqlens[n + 1] : s_start[r] + p.T;
            if (tau == end - 1)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    if (c < 2 * npair) {
                        const int i = 2 * lane + 64 * (c >> 1) + (c & 1);
                        const float v0 = input(r, 1, i), v1 = input(r, 2, i), v2 = input(r, 3, i);
                        float* cs = p.conv_out + ((size_t)n * c_all + c_base + i) * 3;
                        cs[0] = v0;
                        cs[1] = v1;
                        cs[2] = v2;
                    }
        }
    }
    // sequences without tokens keep their cache (copied, or zeros); tile 0 takes them
    if (p.conv_out && blockIdx.x == 0)
        for (int n = 0; n < p.n_seq; ++n) {
            const bool empty = p.cu_seqlens ? p.cu_seqlens[n] == p.cu_seqlens[n + 1] : p.T == 0;
            if (empty)
                for (int e = tid; e < 3 * d; e += kPreThreads) {
                    const size_t idx = ((size_t)n * c_all + c_base + e / 3) * 3 + e % 3;
                    p.conv_out[idx] = p.conv_in ? p.conv_in[idx] : 0.f;
                }
        }
}

// ---- epilogue: one warp per (token, head) row
struct OutGateParams {
    const void* o;
    const void* z;
    const float* weight;  // [dv]
    void* y;
    long long rows;       // B T H
    int dv;
    float eps;
};

template <typename TIO>
__global__ void __launch_bounds__(256) gdn_output_gate_kernel(const OutGateParams p) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    const int per = p.dv / 32;  // 2, 4, 6 or 8 consecutive channels per lane
    const TIO* o = static_cast<const TIO*>(p.o);
    const TIO* z = static_cast<const TIO*>(p.z);
    TIO* y = static_cast<TIO*>(p.y);
    float wt[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wt[e] = e < per ? p.weight[lane * per + e] : 0.f;
    for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < p.rows; row += warps) {
        const size_t base = (size_t)row * p.dv + lane * per;
        float ov[8], zv[8];
        if (per == 8 && sizeof(TIO) == 2) {  // one 16-byte load of each operand
            const uint4 uo = *reinterpret_cast<const uint4*>(o + base), uz = *reinterpret_cast<const uint4*>(z + base);
            const TIO* po = reinterpret_cast<const TIO*>(&uo);
            const TIO* pz = reinterpret_cast<const TIO*>(&uz);
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[e] = to_f32(po[e]), zv[e] = to_f32(pz[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ov[e] = e < per ? to_f32(o[base + e]) : 0.f;
                zv[e] = e < per ? to_f32(z[base + e]) : 0.f;
            }
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(ov[e], ov[e], ss);
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, s);
        const float inv = 1.f / sqrtf(ss / p.dv + p.eps);
        float yv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) yv[e] = ov[e] * inv * wt[e] * silu_f(zv[e]);
        if (per == 8 && sizeof(TIO) == 2) {
            uint4 u;
            TIO* pu = reinterpret_cast<TIO*>(&u);
#pragma unroll
            for (int e = 0; e < 8; ++e) pu[e] = from_f32<TIO>(yv[e]);
            *reinterpret_cast<uint4*>(y + base) = u;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (e < per) y[base + e] = from_f32<TIO>(yv[e]);
        }
    }
}

}  // namespace gdn
