// Shared device-side definitions of libgdn (one translation unit: gdn_api.cu includes every kernel).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// log2(e): the chunk-local cumulative gate is kept in base 2 so the kernels can use exp2
// (GatedDeltaNet data-flow walkthrough, section "Chunked parallelism": cumsum of g times 1.44269504).
constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLog2eD = 1.4426950408889634;
constexpr int kChunk = 64;  // BT = C = 64 tokens per chunk

// Bits of the device error word (read and cleared by gdn_check_error).
constexpr unsigned kErrTimeout = 1u;  // a bounded wait gave up
constexpr unsigned kErrSeqlens = 2u;  // cu_seqlens entry out of order or out of [0, T]

struct FwdParams {
    const void* q;
    const void* k;
    const void* v;
    const float* g;     // GDN [B,T,H]; GDN-2 [B,T,H,dk]
    const float* beta;  // GDN beta [B,T,H]; GDN-2 erase gate b [B,T,H,dk]
    const float* w;     // GDN-2 write gate [B,T,H,dv]; unused for GDN
    const float* h0;    // [N,H,dk,dv] or null
    void* o;
    float* hT;          // [N,H,dk,dv] or null
    const int32_t* cu_seqlens;  // [N+1] or null
    float scale;
    int B, T, H, dk, dv, n_seq;
    int debug_stall;  // diagnostic (gdn_debug_stall): 0 in every ordinary call
    int kda;          // GDN-2 entry as KDA: beta [B,T,H] is both the erase and the write gate; w unused
    float* h_chunks;  // SIMT kernel, backward pass only: the state at every chunk start [slot][H][dk][dv], or null
};

// Chunk slot of chunk c of sequence n that starts at global token offset `start` (row * T + bos):
// n + floor((start + 64 c) / 64).  Slots of different chunks never coincide, and all are below
// ceil(B T / 64) + (number of sequences).
__host__ __device__ inline long long wy_slot(int n, long long start, int c) { return n + (start >> 6) + c; }
inline long long wy_slots(int B, int T, int n_seqs) {
    return ((long long)B * T + kChunk - 1) / kChunk + (n_seqs > B ? n_seqs : B);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

}  // namespace gdn
