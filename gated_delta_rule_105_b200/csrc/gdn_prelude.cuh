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

constexpr int kPreTokens = 16;   // tokens per prelude CTA
constexpr int kPreThreads = 256;

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

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }
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

// grid: (token tiles, H, 4 paths: q, k, v, gates)
template <typename TIO>
__global__ void __launch_bounds__(kPreThreads) gdn_prelude_kernel(const PreludeParams p) {
    constexpr int TT = kPreTokens;
    __shared__ float xs[TT + 3][256];  // inputs of rows tau0 - 3 .. tau0 + TT - 1 (one head's channels)
    __shared__ float ys[TT][256];
    __shared__ int s_n[TT];
    __shared__ long long s_start[TT];
    const int path = blockIdx.z, h = blockIdx.y, tid = threadIdx.x;
    const long long rows = (long long)p.B * p.T;
    const long long tau0 = (long long)blockIdx.x * TT;
    const int H = p.H;

    if (path == 3) {  // ---- gates of this tile's tokens and head
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
        return;
    }

    const int d = path == 2 ? p.dv : p.dk;
    const int c_all = 2 * H * p.dk + H * p.dv;
    const int c_base = (path == 0 ? 0 : path == 1 ? H * p.dk : 2 * H * p.dk) + h * d;  // this head's first channel
    const TIO* x = static_cast<const TIO*>(p.x[path]);
    const float* taps = p.w[path] + (size_t)h * d * 4;
    if (tid < TT) {
        const long long tau = tau0 + tid;
        int n = 0;
        long long st = 0;
        if (tau < rows) pre_seq_of(p, tau, n, st);
        s_n[tid] = n;
        s_start[tid] = st;
    }
    for (int e = tid; e < (TT + 3) * d; e += kPreThreads) {
        const int r = e / d, i = e % d;
        const long long src = tau0 - 3 + r;
        xs[r][i] = (src >= 0 && src < rows) ? to_f32(x[((size_t)src * H + h) * d + i]) : 0.f;
    }
    __syncthreads();
    // the convolution of output row r, channel i
    auto input = [&](int r, int j, int i) -> float {  // tap j (0: oldest) of output row r
        const long long src = tau0 + r - 3 + j, st = s_start[r];
        if (src >= st) return xs[r + j][i];
        if (!p.conv_in) return 0.f;
        return p.conv_in[((size_t)s_n[r] * c_all + c_base + i) * 3 + (int)(src - st + 3)];
    };
    for (int e = tid; e < TT * d; e += kPreThreads) {
        const int r = e / d, i = e % d;
        if (tau0 + r >= rows) continue;
        const float4 w4 = *reinterpret_cast<const float4*>(taps + i * 4);
        float acc = w4.x * input(r, 0, i);
        acc = fmaf(w4.y, input(r, 1, i), acc);
        acc = fmaf(w4.z, input(r, 2, i), acc);
        acc = fmaf(w4.w, input(r, 3, i), acc);
        ys[r][i] = silu_f(acc);
    }
    __syncthreads();
    // store, with the L2 norm of q and k: one warp per row
    TIO* y = static_cast<TIO*>(p.y[path]);
    const int warp = tid >> 5, lane = tid & 31;
    for (int r = warp; r < TT; r += kPreThreads / 32) {
        const long long tau = tau0 + r;
        if (tau >= rows) break;
        float inv = 1.f;
        if (path < 2) {
            float ss = 0.f;
            for (int i = lane; i < d; i += 32) ss = fmaf(ys[r][i], ys[r][i], ss);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            inv = 1.f / sqrtf(ss + p.l2_eps);
        }
        for (int i = lane; i < d; i += 32) y[((size_t)tau * H + h) * d + i] = from_f32<TIO>(ys[r][i] * inv);
    }
    // the cache of every sequence that ends in this tile: its last three inputs, oldest first.  One thread per
    // channel reads the three values before writing them, so the cache may be updated in place (T == 1).
    if (p.conv_out) {
        for (int r = 0; r < TT; ++r) {
            const long long tau = tau0 + r;
            if (tau >= rows) break;
            const int n = s_n[r];
            const long long end = p.cu_seqlens ? (long long)p.cu_seqlens[n + 1] : s_start[r] + p.T;
            if (tau != end - 1) continue;
            for (int i = tid; i < d; i += kPreThreads) {
                const float v0 = input(r, 1, i), v1 = input(r, 2, i), v2 = input(r, 3, i);
                float* dst = p.conv_out + ((size_t)n * c_all + c_base + i) * 3;
                dst[0] = v0;
                dst[1] = v1;
                dst[2] = v2;
            }
        }
        // sequences without tokens keep their cache (copied, or zeros); tile 0 takes them
        if (blockIdx.x == 0)
            for (int n = 0; n < p.n_seq; ++n) {
                const bool empty = p.cu_seqlens ? p.cu_seqlens[n] == p.cu_seqlens[n + 1] : p.T == 0;
                if (empty)
                    for (int e = tid; e < 3 * d; e += kPreThreads) {
                        const size_t idx = ((size_t)n * c_all + c_base + e / 3) * 3 + e % 3;
                        p.conv_out[idx] = p.conv_in ? p.conv_in[idx] : 0.f;
                    }
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
    const TIO* o = static_cast<const TIO*>(p.o);
    const TIO* z = static_cast<const TIO*>(p.z);
    TIO* y = static_cast<TIO*>(p.y);
    for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < p.rows; row += warps) {
        const size_t base = (size_t)row * p.dv;
        float ov[8], zv[8];
        const int per = p.dv / 32;  // 2, 4, 6 or 8 consecutive channels per lane
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            ov[e] = e < per ? to_f32(o[base + lane * per + e]) : 0.f;
            zv[e] = e < per ? to_f32(z[base + lane * per + e]) : 0.f;
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(ov[e], ov[e], ss);
#pragma unroll
        for (int s = 16; s > 0; s >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, s);
        const float inv = 1.f / sqrtf(ss / p.dv + p.eps);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (e < per) {
                const int j = lane * per + e;
                y[base + j] = from_f32<TIO>(ov[e] * inv * p.weight[j] * silu_f(zv[e]));
            }
    }
}

}  // namespace gdn
