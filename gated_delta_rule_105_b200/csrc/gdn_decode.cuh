// Recurrent decode step: one new token per sequence, the state updated in place.
//
// Per (sequence n, head h), with the state S (dk x dv, fp32) read and written once:
//   S <- Diag(a) S                       a = exp(g): one scalar (GDN) or one value per key channel (GDN-2, KDA)
//   u_j = z_j - sum_i e_i S_ij           e = beta k (GDN, KDA) or b . k (GDN-2); z = beta v (GDN, KDA) or w . v
//   S_ij <- S_ij + k_i u_j
//   o_j = scale sum_i q_i S_ij           (read after the write)
// This is one step of the token recurrence (GatedDeltaNet data-flow walkthrough, yfxerp.com/news/367755,
// section "Delta Rule: predict first, then correct"; Gated DeltaNet-2 article, 7minutos.es, section "Regla-2 del
// Delta cerrado", whose opening paragraph names decoding with constant memory as the point of the fixed-size
// state).  It is bound by the state's bytes: 8 dk dv bytes per (sequence, head), moved once.
//
// One CTA per (sequence, head, tile of 128 value columns, or 64 when dv is not a multiple of 128), one thread
// per value column of the tile: thread t owns 4 consecutive value columns (float4) of one quarter of the key
// rows, kept in registers between the read and the write; the two sums over i meet in shared memory.  The value
// columns of the state never mix, so the tiles are independent (128-column tiles keep 128 threads and their
// 128 state registers each at 3 CTAs per SM).
#pragma once

#include "gdn_common.cuh"

namespace gdn {

enum DecodeGates : int { DEC_GDN = 0, DEC_GDN2 = 1, DEC_KDA = 2 };

struct DecodeParams {
    const void* q;       // [N, H, dk]
    const void* k;       // [N, H, dk]
    const void* v;       // [N, H, dv]
    const float* g;      // GDN: [N, H]; GDN-2, KDA: [N, H, dk] (natural-log decay)
    const float* beta;   // GDN, KDA: [N, H]; GDN-2: erase gate b [N, H, dk]
    const float* w;      // GDN-2: write gate [N, H, dv]
    float* state;        // [N, H, dk, dv], in place
    void* o;             // [N, H, dv]
    float scale;
    int N, H, dk, dv, gates;
};

constexpr int kDecRowGroups = 4;

template <typename TIn, typename TOut, int DK>
__global__ void __launch_bounds__(256) gdn_decode_kernel(const DecodeParams p) {
    constexpr int RPT = DK / kDecRowGroups;  // key rows per thread
    __shared__ float sq[DK], sk[DK], se[DK], sa[DK];
    __shared__ float sz[256];
    __shared__ __align__(16) float red[2][kDecRowGroups][256];  // 16 KB
    const int dv = p.dv, tw = blockDim.x, cg_n = tw / 4, j0 = blockIdx.y * tw;
    const int tid = threadIdx.x, cgp = tid % cg_n, rg = tid / cg_n;
    const size_t nh = blockIdx.x;  // n * H + h
    const TIn* q = static_cast<const TIn*>(p.q) + nh * DK;
    const TIn* k = static_cast<const TIn*>(p.k) + nh * DK;
    const TIn* v = static_cast<const TIn*>(p.v) + nh * dv + j0;
    const bool per_channel = p.gates != DEC_GDN;
    const float a0 = per_channel ? 0.f : expf(p.g[nh]);
    const float b0 = p.gates == DEC_GDN2 ? 0.f : p.beta[nh];
    for (int i = tid; i < DK; i += blockDim.x) {
        const float kv = to_f32(k[i]);
        sq[i] = to_f32(q[i]);
        sk[i] = kv;
        sa[i] = per_channel ? expf(p.g[nh * DK + i]) : a0;
        se[i] = (p.gates == DEC_GDN2 ? p.beta[nh * DK + i] : b0) * kv;
    }
    for (int j = tid; j < tw; j += blockDim.x)
        sz[j] = (p.gates == DEC_GDN2 ? p.w[nh * dv + j0 + j] : b0) * to_f32(v[j]);
    __syncthreads();

    float4* st = reinterpret_cast<float4*>(p.state + nh * (size_t)DK * dv + j0) + cgp;
    const int row4 = dv / 4;  // float4s per state row
    const int r0 = rg * RPT;
    float4 S[RPT];
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) {
        const int i = r0 + rr;
        float4 x = st[(size_t)i * row4];
        const float a = sa[i], e = se[i];
        x.x *= a, x.y *= a, x.z *= a, x.w *= a;
        r.x = fmaf(e, x.x, r.x), r.y = fmaf(e, x.y, r.y), r.z = fmaf(e, x.z, r.z), r.w = fmaf(e, x.w, r.w);
        S[rr] = x;
    }
    *reinterpret_cast<float4*>(&red[0][rg][4 * cgp]) = r;
    __syncthreads();
    float4 u;
    {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g2 = 0; g2 < kDecRowGroups; ++g2) {
            const float4 x = *reinterpret_cast<const float4*>(&red[0][g2][4 * cgp]);
            t.x += x.x, t.y += x.y, t.z += x.z, t.w += x.w;
        }
        u = make_float4(sz[4 * cgp] - t.x, sz[4 * cgp + 1] - t.y, sz[4 * cgp + 2] - t.z, sz[4 * cgp + 3] - t.w);
    }
    float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) {
        const int i = r0 + rr;
        const float ki = sk[i], qi = sq[i];
        float4 x = S[rr];
        x.x = fmaf(ki, u.x, x.x), x.y = fmaf(ki, u.y, x.y), x.z = fmaf(ki, u.z, x.z), x.w = fmaf(ki, u.w, x.w);
        st[(size_t)i * row4] = x;
        ov.x = fmaf(qi, x.x, ov.x), ov.y = fmaf(qi, x.y, ov.y), ov.z = fmaf(qi, x.z, ov.z), ov.w = fmaf(qi, x.w, ov.w);
    }
    *reinterpret_cast<float4*>(&red[1][rg][4 * cgp]) = ov;
    __syncthreads();
    if (rg == 0) {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int g2 = 0; g2 < kDecRowGroups; ++g2) {
            const float4 x = *reinterpret_cast<const float4*>(&red[1][g2][4 * cgp]);
            t.x += x.x, t.y += x.y, t.z += x.z, t.w += x.w;
        }
        TOut* o = static_cast<TOut*>(p.o) + nh * dv + j0 + 4 * cgp;
        o[0] = from_f32<TOut>(p.scale * t.x);
        o[1] = from_f32<TOut>(p.scale * t.y);
        o[2] = from_f32<TOut>(p.scale * t.z);
        o[3] = from_f32<TOut>(p.scale * t.w);
    }
}

}  // namespace gdn
