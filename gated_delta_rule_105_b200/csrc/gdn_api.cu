// libgdn C ABI: host-side argument checks, kernel selection and launches.  Every kernel of the library
// is included here so that they share one device error word without relocatable device code.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <type_traits>

#include "gdn.h"
#include "gdn_common.cuh"
#include "gdn_prof.cuh"
#include "gdn_simt.cuh"
#include "gdn_tc.cuh"
#include "gdn2_tc.cuh"
#include "gdn_decode.cuh"
#include "gdn_prelude.cuh"
#include "gdn_bwd.cuh"
#include "gdn2_bwd.cuh"
#include "gdn_tc_selftest.cuh"

namespace gdn {

__device__ unsigned int g_err_word;

static thread_local char t_msg[512];

// Scratch of gdn_chunk_fwd_noalloc, for callers that must not allocate device memory.  It is part of the
// library's device image: the CUDA runtime reserves it on a device when it loads this module there (with lazy
// module loading, at the first launch or symbol lookup of any entry point on that device) and keeps it until
// the process exits.  Its size is GDN_STATIC_WS_BYTES (gdn.h).
static __device__ __align__(256) uint8_t g_static_ws[GDN_STATIC_WS_BYTES];
static thread_local gdn_kernel t_last_kernel = GDN_KERNEL_AUTO;
static std::atomic<int> g_kernel_choice{GDN_KERNEL_AUTO};
static std::atomic<int> g_debug_stall{0};

// Device address of g_static_ws on each device.  In host code the array's name is only a host-side handle, so
// the address is looked up once per device, with that device current, by the first no-workspace call there.
constexpr int kMaxDevices = 64;
static std::atomic<void*> g_static_ws_addr[kMaxDevices];
static std::mutex g_static_ws_mu;

static gdn_status fail(gdn_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
    va_end(ap);
    return st;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static unsigned* err_word_ptr(gdn_status* st) {
    unsigned* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_err_word);
    if (e != cudaSuccess) {
        *st = fail(GDN_ERR_CUDA, "cudaGetSymbolAddress(error word): %s", cudaGetErrorString(e));
        return nullptr;
    }
    *st = GDN_OK;
    return ptr;
}

// Host checks shared by both operations.  Nothing touches the device before these pass.
static gdn_status check_common(const void* q, const void* k, const void* v, const float* g, const float* gate,
                               const float* w, bool gdn2, float scale, const float* h0, const void* o,
                               const float* hT, int B, int T, int H, int dk, int dv, int BT, gdn_dtype dt,
                               gdn_dtype o_dt, const int32_t* cu, int n_seqs, void* ws, size_t ws_bytes, int* n_seq_out) {
    t_msg[0] = 0;
    if (T > 0 && (!q || !k || !v || !g || !gate || !o || (gdn2 && !w)))
        return fail(GDN_ERR_INVALID_ARG, "a required pointer (q, k, v, g, %s, o%s) is NULL",
                    gdn2 ? "b" : "beta", gdn2 ? ", w" : "");
    const void* ptrs[] = {q, k, v, g, gate, w, h0, o, hT, cu, ws};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return fail(GDN_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", ptr);
    if (B < 1 || H < 1 || T < 0) return fail(GDN_ERR_INVALID_ARG, "need B >= 1, H >= 1, T >= 0 (got %d, %d, %d)", B, H, T);
    if (BT != kChunk) return fail(GDN_ERR_UNSUPPORTED, "BT must be %d (got %d)", kChunk, BT);
    if (dk != 64 && dk != 128) return fail(GDN_ERR_UNSUPPORTED, "dk must be 64 or 128 (got %d)", dk);
    if (dv < 64 || dv > 256 || dv % 64 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "dv must be a multiple of 64 in [64, 256] (got %d)", dv);
    if (dt != GDN_F32 && dt != GDN_BF16) return fail(GDN_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    if (o_dt != GDN_F32 && o_dt != dt)
        return fail(GDN_ERR_UNSUPPORTED, "o_dt must be GDN_F32 or the input dtype (got %d)", (int)o_dt);
    if (!std::isfinite(scale)) return fail(GDN_ERR_INVALID_ARG, "scale is not finite");
    if (ws_bytes > 0 && !ws) return fail(GDN_ERR_INVALID_ARG, "ws_bytes > 0 with a NULL workspace");
    if (cu) {
        if (B != 1) return fail(GDN_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (got %d)", B);
        if (n_seqs < 1 || n_seqs > 65535) return fail(GDN_ERR_INVALID_ARG, "n_seqs must be in [1, 65535] (got %d)", n_seqs);
        *n_seq_out = n_seqs;
    } else {
        if (n_seqs != 0 && n_seqs != B)
            return fail(GDN_ERR_INVALID_ARG, "without cu_seqlens n_seqs must be 0 or B (got %d)", n_seqs);
        if (B > 65535) return fail(GDN_ERR_INVALID_ARG, "B must be <= 65535 (got %d)", B);
        *n_seq_out = B;
    }
    if (H > 65535) return fail(GDN_ERR_INVALID_ARG, "H must be <= 65535 (got %d)", H);
    const double elems = (double)B * T * H * (dk > dv ? dk : dv);
    if (elems > 9.0e15) return fail(GDN_ERR_INVALID_ARG, "tensor too large");
    return GDN_OK;
}

template <typename TIn, typename TOut, int DK, bool GDN2>
static gdn_status launch_simt_dk(const FwdParams& p, unsigned* err, cudaStream_t stream) {
    constexpr int DVT = SimtDVT<GDN2>::value;
    using L = SimtSmem<DK, DVT, GDN2, sizeof(typename SimtGate<TIn>::type) / 4>;
    auto kern = gdn_simt_fwd_kernel<TIn, TOut, DK, DVT, GDN2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    dim3 grid(p.dv / DVT, p.H, p.n_seq);
    ProfScope prof(PK_SIMT, stream);
    kern<<<grid, kSimtThreads, L::bytes, stream>>>(p, err);
    prof.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "SIMT kernel launch: %s", cudaGetErrorString(e));
    return GDN_OK;
}

template <typename TIn, typename TOut, bool GDN2>
static gdn_status launch_simt_io(const FwdParams& p, unsigned* err, cudaStream_t stream) {
    return p.dk == 64 ? launch_simt_dk<TIn, TOut, 64, GDN2>(p, err, stream)
                      : launch_simt_dk<TIn, TOut, 128, GDN2>(p, err, stream);
}

template <bool GDN2>
static gdn_status launch_simt(const FwdParams& p, gdn_dtype dt, gdn_dtype o_dt, unsigned* err, cudaStream_t stream) {
    if (dt == GDN_F32) return launch_simt_io<float, float, GDN2>(p, err, stream);
    if (o_dt == GDN_F32) return launch_simt_io<__nv_bfloat16, float, GDN2>(p, err, stream);
    return launch_simt_io<__nv_bfloat16, __nv_bfloat16, GDN2>(p, err, stream);
}

static gdn_status run(const FwdParams& p, bool gdn2, gdn_dtype dt, gdn_dtype o_dt, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
    const int choice = g_kernel_choice.load();
    const bool tc_ok = dt == GDN_BF16 && (gdn2 ? tc2_supported(p) : tc_supported(p));
    if (choice == GDN_KERNEL_TC && !tc_ok)
        return fail(GDN_ERR_UNSUPPORTED, "the tcgen05 kernel needs bf16 inputs and a supported shape");
    gdn_status st;
    unsigned* err = err_word_ptr(&st);
    if (!err) return st;
    if (p.n_seq == 0 || p.H == 0) return GDN_OK;
    const bool use_tc = tc_ok && choice != GDN_KERNEL_SIMT;
    if (use_tc) {
        st = gdn2 ? launch_tc2(p, o_dt == GDN_F32, ws, ws_bytes, err, stream)
                  : launch_tc(p, o_dt == GDN_F32, ws, ws_bytes, err, stream);
        if (st == GDN_OK) {
            t_last_kernel = GDN_KERNEL_TC;
            return st;
        }
        fail(st, "tcgen05 kernel: %s", tc_last_error());
        if (st != GDN_ERR_UNSUPPORTED || choice == GDN_KERNEL_TC) return st;
        // AUTO: a configuration the tcgen05 build cannot take runs on the SIMT kernel
    }
    st = gdn2 ? launch_simt<true>(p, dt, o_dt, err, stream) : launch_simt<false>(p, dt, o_dt, err, stream);
    if (st == GDN_OK) {
        t_last_kernel = GDN_KERNEL_SIMT;
        t_msg[0] = 0;  // the refused tensor-core attempt is not a failure of this call
    }
    return st;
}

// The device address of the no-workspace scratch on the current device (see g_static_ws_addr).
static gdn_status static_scratch(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(GDN_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
    void* ptr = g_static_ws_addr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        std::lock_guard<std::mutex> lock(g_static_ws_mu);
        ptr = g_static_ws_addr[dev].load(std::memory_order_relaxed);
        if (!ptr) {
            e = cudaGetSymbolAddress(&ptr, g_static_ws);
            if (e != cudaSuccess || !ptr)
                return fail(GDN_ERR_CUDA, "static scratch address: %s", cudaGetErrorString(e));
            g_static_ws_addr[dev].store(ptr, std::memory_order_release);
        }
    }
    *out = ptr;
    return GDN_OK;
}

// ---- decode step
static gdn_status check_decode(const void* q, const void* k, const void* v, const float* g, const float* gate,
                               const float* w, int gates, float scale, const float* state, const void* o, int N, int H,
                               int dk, int dv, gdn_dtype dt, gdn_dtype o_dt) {
    t_msg[0] = 0;
    if (N < 1 || H < 1) return fail(GDN_ERR_INVALID_ARG, "need N >= 1, H >= 1 (got %d, %d)", N, H);
    if (!q || !k || !v || !g || !gate || !state || !o || (gates == DEC_GDN2 && !w))
        return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL");
    const void* ptrs[] = {q, k, v, g, gate, w, state, o};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return fail(GDN_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", ptr);
    if (dk != 64 && dk != 128) return fail(GDN_ERR_UNSUPPORTED, "dk must be 64 or 128 (got %d)", dk);
    if (dv < 64 || dv > 256 || dv % 64 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "dv must be a multiple of 64 in [64, 256] (got %d)", dv);
    if (dt != GDN_F32 && dt != GDN_BF16) return fail(GDN_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    if (o_dt != GDN_F32 && o_dt != dt)
        return fail(GDN_ERR_UNSUPPORTED, "o_dt must be GDN_F32 or the input dtype (got %d)", (int)o_dt);
    if (!std::isfinite(scale)) return fail(GDN_ERR_INVALID_ARG, "scale is not finite");
    if ((long long)N * H > 0x7fffffffLL) return fail(GDN_ERR_INVALID_ARG, "N * H too large");
    return GDN_OK;
}

template <typename TIn, typename TOut>
static gdn_status launch_decode_io(const DecodeParams& p, cudaStream_t stream) {
    auto kern = p.dk == 64 ? gdn_decode_kernel<TIn, TOut, 64> : gdn_decode_kernel<TIn, TOut, 128>;
    ProfScope prof(PK_DECODE, stream);
    const int tw = p.dv % 128 == 0 ? 128 : 64;  // value columns per CTA
    kern<<<dim3((unsigned)((long long)p.N * p.H), (unsigned)(p.dv / tw)), tw / 4 * kDecRowGroups, 0, stream>>>(p);
    prof.done();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "decode kernel launch: %s", cudaGetErrorString(e));
    return GDN_OK;
}

static gdn_status decode(const DecodeParams& p, gdn_dtype dt, gdn_dtype o_dt, cudaStream_t stream) {
    if (dt == GDN_F32) return launch_decode_io<float, float>(p, stream);
    if (o_dt == GDN_F32) return launch_decode_io<__nv_bfloat16, float>(p, stream);
    return launch_decode_io<__nv_bfloat16, __nv_bfloat16>(p, stream);
}

template <typename TIO>
static gdn_status launch_prelude(const PreludeParams& p, cudaStream_t stream) {
    const long long rows = (long long)p.B * p.T;
    const long long tiles = rows > 0 ? (rows + kPreTokens - 1) / kPreTokens : 1;
    if (tiles > 0x7fffffffLL) return fail(GDN_ERR_INVALID_ARG, "too many tokens for one launch");
    const size_t smem = prelude_smem_bytes(std::max(p.dk, p.dv));
    cudaError_t e0 = cudaFuncSetAttribute(gdn_prelude_kernel<TIO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem);
    if (e0 != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e0));
    ProfScope prof(PK_PRELUDE, stream);
    gdn_prelude_kernel<TIO><<<dim3((unsigned)tiles, p.H, 3), kPreThreads, smem, stream>>>(p);
    prof.done();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "prelude kernel launch: %s", cudaGetErrorString(e));
    return GDN_OK;
}

template <typename TIO>
static gdn_status launch_out_gate(const OutGateParams& p, cudaStream_t stream) {
    const long long blocks = std::min<long long>((p.rows + 7) / 8, 148LL * 16);
    ProfScope prof(PK_OUT_GATE, stream);
    gdn_output_gate_kernel<TIO><<<(unsigned)std::max<long long>(blocks, 1), 256, 0, stream>>>(p);
    prof.done();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "output gate kernel launch: %s", cudaGetErrorString(e));
    return GDN_OK;
}

// ---- backward
// Two fp32 states per chunk slot and head (the chunk-start states, the end-state cotangents), then T and P.
inline size_t bwd_state_bytes(int B, int T, int H, int dk, int dv, int n_seqs) {
    return 2 * (size_t)wy_slots(B, T, n_seqs) * H * (size_t)dk * dv * sizeof(float);
}
inline size_t bwd_tp_bytes(int B, int T, int H, int n_seqs) {
    return (size_t)wy_slots(B, T, n_seqs) * H * 2 * kChunk * kChunk * sizeof(float);
}
inline size_t bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int n_seqs) {
    return bwd_state_bytes(B, T, H, dk, dv, n_seqs) + bwd_tp_bytes(B, T, H, n_seqs);
}

// The state at every chunk start, for the backward pass (o not written).  GDN with bf16 inputs of a shape the
// tensor-core forward takes runs that forward, with the part of the backward workspace that the later kernels
// fill (`tc_ws`) as its scratch; everything else runs the SIMT forward.  (GDN-2 keeps the SIMT states: its
// gate gradient sums terms much larger than itself, and the bf16 operands of the tensor-core GDN-2 state,
// ~3e-3 of its RMS, came out at 3-10e-2 of dg's RMS against a 2e-2 bound.)
template <typename TIn, int DK, bool GDN2>
static gdn_status bwd_chunk_states(const FwdParams& fp, void* tc_ws, size_t tc_ws_bytes, unsigned* err,
                                   cudaStream_t stream) {
    if (!GDN2 && std::is_same<TIn, __nv_bfloat16>::value && g_kernel_choice.load() != GDN_KERNEL_SIMT &&
        tc_supported(fp)) {
        const gdn_status st = launch_tc(fp, false, tc_ws, tc_ws_bytes, err, stream);
        if (st == GDN_OK) return st;
        if (st != GDN_ERR_UNSUPPORTED) return fail(st, "tcgen05 forward of the backward pass: %s", tc_last_error());
    }
    return launch_simt_dk<TIn, float, DK, GDN2>(fp, err, stream);
}

template <typename TIn, int DK>
static gdn_status launch_bwd_dk(const FwdParams& fp, const BwdParams& bp, unsigned* err, cudaStream_t stream) {
    // (1) the state at every chunk start; the state-cotangent array serves as the tensor-core forward's scratch
    const size_t state_bytes = wy_slots(bp.B, bp.T, bp.n_seq) * (size_t)bp.H * DK * (size_t)bp.vdim * sizeof(float);
    gdn_status st = bwd_chunk_states<TIn, DK, false>(fp, bp.dh_chunks, state_bytes + bwd_tp_bytes(bp.B, bp.T, bp.H,
                                                                                                 bp.n_seq), err, stream);
    if (st != GDN_OK) return st;
    const long long grid = wy_slots(bp.B, bp.T, bp.n_seq) * bp.H;
    if (grid > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many chunks for one launch");
    ProfScope prof(PK_BWD, stream);
    // (2) T and P of every chunk
    auto kp = gdn_bwd_prep_kernel<TIn, DK>;
    cudaError_t e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BwPrepSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (grid > 0) kp<<<(unsigned)grid, kBwThreads, BwPrepSmem<DK>::bytes, stream>>>(bp, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward prep kernel: %s", cudaGetErrorString(e));
    // (3) the state cotangent, chunk by chunk backwards
    auto kdh = gdn_bwd_dh_kernel<TIn, DK>;
    e = cudaFuncSetAttribute(kdh, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BwDhSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    kdh<<<dim3(bp.vdim / BwDhSmem<DK>::DVT, bp.H, bp.n_seq), kBwThreads, BwDhSmem<DK>::bytes, stream>>>(bp, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward state kernel: %s", cudaGetErrorString(e));
    // (4) every input gradient, all chunks at once
    auto kc = gdn_bwd_chunk_kernel<TIn, DK>;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BwChunkSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (grid > 0) kc<<<(unsigned)grid, kBwThreads, BwChunkSmem<DK>::bytes, stream>>>(bp, err);
    prof.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward chunk kernel: %s", cudaGetErrorString(e));
    return GDN_OK;
}

// ---- backward of GDN-2 and KDA
inline size_t bwd2_tp_bytes(int B, int T, int H, int n_seqs) {
    return (size_t)wy_slots(B, T, n_seqs) * H * 2 * kChunk * kChunk * sizeof(float);
}
inline size_t bwd2_workspace_bytes(int B, int T, int H, int dk, int dv, int n_seqs) {
    return bwd_state_bytes(B, T, H, dk, dv, n_seqs) + bwd2_tp_bytes(B, T, H, n_seqs);
}

template <typename TIn, int DK>
static gdn_status launch_bwd2_dk(const FwdParams& fp, const Bwd2Params& bp, unsigned* err, cudaStream_t stream) {
    (void)fp;
    const long long grid = wy_slots(bp.B, bp.T, bp.n_seq) * bp.H;
    if (grid > 0x7fffffffLL) return fail(GDN_ERR_UNSUPPORTED, "too many chunks for one launch");
    ProfScope prof(PK_BWD, stream);
    // (0) T and P of every chunk
    auto kp = gdn2_bwd_prep_kernel<TIn, DK>;
    cudaError_t e = cudaFuncSetAttribute(kp, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Bw2PrepSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (grid > 0) kp<<<(unsigned)grid, kBw2Threads, Bw2PrepSmem<DK>::bytes, stream>>>(bp, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward prep kernel: %s", cudaGetErrorString(e));
    // (1) the state at every chunk start, walked forward with T
    auto kst = gdn2_bwd_states_kernel<TIn, DK>;
    e = cudaFuncSetAttribute(kst, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Bw2StSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    kst<<<dim3(bp.vdim / Bw2StSmem<DK>::DVT, bp.H, bp.n_seq), kBw2Threads, Bw2StSmem<DK>::bytes, stream>>>(bp, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward state kernel: %s", cudaGetErrorString(e));
    // (3) the state cotangent, chunk by chunk backwards
    auto kdh = gdn2_bwd_dh_kernel<TIn, DK>;
    e = cudaFuncSetAttribute(kdh, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Bw2DhSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    kdh<<<dim3(bp.vdim / Bw2DhSmem<DK>::DVT, bp.H, bp.n_seq), kBw2Threads, Bw2DhSmem<DK>::bytes, stream>>>(bp, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward state kernel: %s", cudaGetErrorString(e));
    // (4) every input gradient, all chunks at once
    auto kc = gdn2_bwd_chunk_kernel<TIn, DK>;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Bw2ChunkSmem<DK>::bytes);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (grid > 0) kc<<<(unsigned)grid, kBw2Threads, Bw2ChunkSmem<DK>::bytes, stream>>>(bp, err);
    prof.done();
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward chunk kernel: %s", cudaGetErrorString(e));
    return GDN_OK;
}

// Shared body of gdn2_chunk_bwd and gdn_kda_chunk_bwd (kda: b is beta [B,T,H], w and dw unused).
static gdn_status chunk_bwd2(const void* q, const void* k, const void* v, const float* g, const float* b,
                             const float* w, bool kda, float scale, const float* h0, const void* d_o, const float* dhT,
                             float* dq, float* dk, float* dv, float* dg, float* db, float* dw, float* dh0, int B, int T,
                             int H, int dk_, int dv_, int BT, gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
    int n_seq = 0;
    gdn_status st = check_common(q, k, v, g, b, w, !kda, scale, h0, d_o, dhT, B, T, H, dk_, dv_, BT, dt, dt,
                                 cu_seqlens, n_seqs, workspace, ws_bytes, &n_seq);
    if (st != GDN_OK) return st;
    if (T > 0 && (!dq || !dk || !dv || !dg || !db || (!kda && !dw)))
        return fail(GDN_ERR_INVALID_ARG, "a gradient output (dq, dk, dv, dg, %s) is NULL", kda ? "dbeta" : "db, dw");
    const void* outs[] = {dq, dk, dv, dg, db, dw, dh0};
    for (const void* ptr : outs)
        if (ptr && !aligned16(ptr)) return fail(GDN_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", ptr);
    const int ns = cu_seqlens ? n_seq : 0;
    const size_t need = bwd2_workspace_bytes(B, T, H, dk_, dv_, ns);
    if (!workspace || ws_bytes < need)
        return fail(GDN_ERR_INVALID_ARG, "the backward pass needs %zu bytes of workspace (got %zu)", need, ws_bytes);
    gdn_status es;
    unsigned* err = err_word_ptr(&es);
    if (!err) return es;
    const size_t states = bwd_state_bytes(B, T, H, dk_, dv_, ns) / sizeof(float);
    float* hc = static_cast<float*>(workspace);
    float* dhc = hc + states / 2;
    float* tp = hc + states;
    FwdParams fp{q, k, v, g, b, kda ? nullptr : w, h0, nullptr, nullptr, cu_seqlens, scale, B, T, H, dk_, dv_, n_seq};
    fp.kda = kda ? 1 : 0;
    fp.h_chunks = hc;
    Bwd2Params bp{q, k, v, g, b, kda ? nullptr : w, d_o, dhT, hc, dhc, tp, dq, dk, dv, dg, db, kda ? nullptr : dw,
                  dh0, cu_seqlens, scale, B, T, H, dk_, dv_, n_seq, kda ? 1 : 0, h0};
    if (dt == GDN_F32)
        return dk_ == 64 ? launch_bwd2_dk<float, 64>(fp, bp, err, stream) : launch_bwd2_dk<float, 128>(fp, bp, err, stream);
    return dk_ == 64 ? launch_bwd2_dk<__nv_bfloat16, 64>(fp, bp, err, stream)
                     : launch_bwd2_dk<__nv_bfloat16, 128>(fp, bp, err, stream);
}

}  // namespace gdn

using namespace gdn;

extern "C" {

size_t gdn_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs) {
    // the tcgen05 path (bf16 inputs) keeps T' and T'' of every chunk and head; the SIMT path needs nothing
    if (B < 1 || T < 1 || H < 1 || BT != kChunk || dk != kTcDK || dv < kTcDV || dv % kTcDV != 0 || n_seqs < 0)
        return 0;
    return tc_workspace_bytes(B, T, H, n_seqs);
}

size_t gdn2_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs) {
    // the tcgen05 GDN-2 / KDA path keeps one 80.5 KB unit per chunk and head; the SIMT path needs nothing
    if (B < 1 || T < 1 || H < 1 || BT != kChunk || dk != kTcDK || dv < kTcDV || dv % kTcDV != 0 || n_seqs < 0)
        return 0;
    return tc2_workspace_bytes(B, T, H, n_seqs);
}

gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float scale, const float* h0, void* o, float* hT, int B, int T, int H, int dk, int dv,
                         int BT, gdn_dtype dt, gdn_dtype o_dt, const int32_t* cu_seqlens, int n_seqs,
                         void* workspace, size_t ws_bytes, cudaStream_t stream) {
    int n_seq = 0;
    gdn_status st = check_common(q, k, v, g, beta, nullptr, false, scale, h0, o, hT, B, T, H, dk, dv, BT, dt,
                                 o_dt, cu_seqlens, n_seqs, workspace, ws_bytes, &n_seq);
    if (st != GDN_OK) return st;
    FwdParams p{q, k, v, g, beta, nullptr, h0, o, hT, cu_seqlens, scale, B, T, H, dk, dv, n_seq};
    p.debug_stall = g_debug_stall.load();
    return run(p, false, dt, o_dt, workspace, ws_bytes, stream);
}

gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                 float scale, const float* h0, void* o, float* hT, int B, int T, int H, int dk,
                                 int dv, int BT, gdn_dtype dt, gdn_dtype o_dt, const int32_t* cu_seqlens,
                                 int n_seqs, cudaStream_t stream) {
    int n_seq = 0;
    gdn_status st = check_common(q, k, v, g, beta, nullptr, false, scale, h0, o, hT, B, T, H, dk, dv, BT, dt,
                                 o_dt, cu_seqlens, n_seqs, nullptr, 0, &n_seq);
    if (st != GDN_OK) return st;
    FwdParams p{q, k, v, g, beta, nullptr, h0, o, hT, cu_seqlens, scale, B, T, H, dk, dv, n_seq};
    p.debug_stall = g_debug_stall.load();
    // The tensor-core path needs tc_workspace_bytes() of scratch; beyond the static array's size the call is
    // refused (callers that can allocate use gdn_chunk_fwd with their own workspace).
    const bool tc_path = dt == GDN_BF16 && tc_supported(p) &&
                         g_kernel_choice.load() != GDN_KERNEL_SIMT && n_seq > 0;
    if (tc_path) {
        const size_t need = tc_workspace_bytes(B, T, H, n_seq);
        if (need > (size_t)GDN_STATIC_WS_BYTES)
            return fail(GDN_ERR_UNSUPPORTED,
                        "gdn_chunk_fwd_noalloc: these sizes need %zu bytes of scratch, the static scratch holds %zu "
                        "(GDN_STATIC_WS_BYTES); use gdn_chunk_fwd with a caller workspace",
                        need, (size_t)GDN_STATIC_WS_BYTES);
    }
    void* ws = nullptr;
    st = static_scratch(&ws);
    if (st != GDN_OK) return st;
    return run(p, false, dt, o_dt, ws, (size_t)GDN_STATIC_WS_BYTES, stream);
}

gdn_status gdn2_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* b,
                          const float* w, float scale, const float* h0, void* o, float* hT, int B, int T, int H,
                          int dk, int dv, int BT, gdn_dtype dt, gdn_dtype o_dt, const int32_t* cu_seqlens,
                          int n_seqs, void* workspace, size_t ws_bytes, cudaStream_t stream) {
    int n_seq = 0;
    gdn_status st = check_common(q, k, v, g, b, w, true, scale, h0, o, hT, B, T, H, dk, dv, BT, dt, o_dt,
                                 cu_seqlens, n_seqs, workspace, ws_bytes, &n_seq);
    if (st != GDN_OK) return st;
    FwdParams p{q, k, v, g, b, w, h0, o, hT, cu_seqlens, scale, B, T, H, dk, dv, n_seq};
    return run(p, true, dt, o_dt, workspace, ws_bytes, stream);
}

gdn_status gdn_kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             float scale, const float* h0, void* o, float* hT, int B, int T, int H, int dk, int dv,
                             int BT, gdn_dtype dt, gdn_dtype o_dt, const int32_t* cu_seqlens, int n_seqs,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
    int n_seq = 0;
    gdn_status st = check_common(q, k, v, g, beta, nullptr, false, scale, h0, o, hT, B, T, H, dk, dv, BT, dt, o_dt,
                                 cu_seqlens, n_seqs, workspace, ws_bytes, &n_seq);
    if (st != GDN_OK) return st;
    FwdParams p{q, k, v, g, beta, nullptr, h0, o, hT, cu_seqlens, scale, B, T, H, dk, dv, n_seq};
    p.kda = 1;
    return run(p, true, dt, o_dt, workspace, ws_bytes, stream);
}

gdn_status gdn_decode_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta, float scale,
                          float* state, void* o, int N, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                          cudaStream_t stream) {
    gdn_status st = check_decode(q, k, v, g, beta, nullptr, DEC_GDN, scale, state, o, N, H, dk, dv, dt, o_dt);
    if (st != GDN_OK) return st;
    return decode(DecodeParams{q, k, v, g, beta, nullptr, state, o, scale, N, H, dk, dv, DEC_GDN}, dt, o_dt, stream);
}

gdn_status gdn2_decode_fwd(const void* q, const void* k, const void* v, const float* g, const float* b, const float* w,
                           float scale, float* state, void* o, int N, int H, int dk, int dv, gdn_dtype dt,
                           gdn_dtype o_dt, cudaStream_t stream) {
    gdn_status st = check_decode(q, k, v, g, b, w, DEC_GDN2, scale, state, o, N, H, dk, dv, dt, o_dt);
    if (st != GDN_OK) return st;
    return decode(DecodeParams{q, k, v, g, b, w, state, o, scale, N, H, dk, dv, DEC_GDN2}, dt, o_dt, stream);
}

gdn_status gdn_kda_decode_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                              float scale, float* state, void* o, int N, int H, int dk, int dv, gdn_dtype dt,
                              gdn_dtype o_dt, cudaStream_t stream) {
    gdn_status st = check_decode(q, k, v, g, beta, nullptr, DEC_KDA, scale, state, o, N, H, dk, dv, dt, o_dt);
    if (st != GDN_OK) return st;
    return decode(DecodeParams{q, k, v, g, beta, nullptr, state, o, scale, N, H, dk, dv, DEC_KDA}, dt, o_dt, stream);
}

gdn_status gdn_prelude_fwd(const void* xq, const void* xk, const void* xv, const float* wq, const float* wk,
                           const float* wv, const float* conv_in, float* conv_out, const float* a, const float* A_log,
                           const float* dt_bias, float* g, int g_width, const float* b, float* beta, int b_width,
                           const float* c, float* w_gate, int c_width, void* q, void* k, void* v, int B, int T, int H,
                           int dk, int dv, gdn_dtype dt, float l2_eps, const int32_t* cu_seqlens, int n_seqs,
                           cudaStream_t stream) {
    t_msg[0] = 0;
    if (B < 1 || H < 1 || T < 0) return fail(GDN_ERR_INVALID_ARG, "need B >= 1, H >= 1, T >= 0 (got %d, %d, %d)", B, H, T);
    if (T > 0 && (!xq || !xk || !xv || !wq || !wk || !wv || !a || !A_log || !dt_bias || !g || !b || !beta || !q ||
                  !k || !v))
        return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL");
    if ((c == nullptr) != (w_gate == nullptr)) return fail(GDN_ERR_INVALID_ARG, "c and w_gate go together");
    const void* ptrs[] = {xq, xk, xv, wq, wk, wv, conv_in, conv_out, a, g, b, beta, c, w_gate, q, k, v, cu_seqlens};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return fail(GDN_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", ptr);
    if (dk != 64 && dk != 128) return fail(GDN_ERR_UNSUPPORTED, "dk must be 64 or 128 (got %d)", dk);
    if (dv < 64 || dv > 256 || dv % 64 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "dv must be a multiple of 64 in [64, 256] (got %d)", dv);
    if (g_width < 1 || b_width < 1 || (c && c_width < 1) || g_width > 256 || b_width > 256 || c_width > 256)
        return fail(GDN_ERR_INVALID_ARG, "gate widths must be in [1, 256]");
    if (dt != GDN_F32 && dt != GDN_BF16) return fail(GDN_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    if (!(l2_eps >= 0.f) || !std::isfinite(l2_eps)) return fail(GDN_ERR_INVALID_ARG, "l2_eps must be >= 0");
    int n_seq = B;
    if (cu_seqlens) {
        if (B != 1) return fail(GDN_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (got %d)", B);
        if (n_seqs < 1 || n_seqs > 65535) return fail(GDN_ERR_INVALID_ARG, "n_seqs must be in [1, 65535]");
        n_seq = n_seqs;
    } else if (n_seqs != 0 && n_seqs != B) {
        return fail(GDN_ERR_INVALID_ARG, "without cu_seqlens n_seqs must be 0 or B (got %d)", n_seqs);
    }
    if (conv_in && conv_in == conv_out && (cu_seqlens || T != 1))
        return fail(GDN_ERR_INVALID_ARG, "conv_in and conv_out may be one buffer only for single-token steps (T == 1)");
    PreludeParams p{{xq, xk, xv}, {wq, wk, wv}, conv_in, conv_out, {q, k, v}, a, A_log, dt_bias, g, b, beta, c,
                    w_gate, cu_seqlens, l2_eps, B, T, H, dk, dv, g_width, b_width, c ? c_width : 0, n_seq};
    return dt == GDN_F32 ? launch_prelude<float>(p, stream) : launch_prelude<__nv_bfloat16>(p, stream);
}

gdn_status gdn_output_gate_fwd(const void* o, const void* z, const float* weight, void* y, long long rows, int dv,
                               gdn_dtype dt, float eps, cudaStream_t stream) {
    t_msg[0] = 0;
    if (rows < 0) return fail(GDN_ERR_INVALID_ARG, "rows must be >= 0");
    if (rows == 0) return GDN_OK;
    if (!o || !z || !weight || !y) return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL");
    const void* ptrs[] = {o, z, weight, y};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return fail(GDN_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", ptr);
    if (dv < 64 || dv > 256 || dv % 64 != 0)
        return fail(GDN_ERR_UNSUPPORTED, "dv must be a multiple of 64 in [64, 256] (got %d)", dv);
    if (dt != GDN_F32 && dt != GDN_BF16) return fail(GDN_ERR_UNSUPPORTED, "unknown dtype %d", (int)dt);
    if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(GDN_ERR_INVALID_ARG, "eps must be >= 0");
    OutGateParams p{o, z, weight, y, rows, dv, eps};
    return dt == GDN_F32 ? launch_out_gate<float>(p, stream) : launch_out_gate<__nv_bfloat16>(p, stream);
}

size_t gdn_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs) {
    if (B < 1 || T < 0 || H < 1 || BT != kChunk || (dk != 64 && dk != 128) || dv < 64 || dv > 256 || dv % 64 != 0 ||
        n_seqs < 0)
        return 0;
    return bwd_workspace_bytes(B, T, H, dk, dv, n_seqs);
}

gdn_status gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta, float scale,
                         const float* h0, const void* d_o, const float* dhT, float* dq, float* dk, float* dv,
                         float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_, int dv_, int BT,
                         gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs, void* workspace, size_t ws_bytes,
                         cudaStream_t stream) {
    int n_seq = 0;
    gdn_status st = check_common(q, k, v, g, beta, nullptr, false, scale, h0, d_o, dhT, B, T, H, dk_, dv_, BT, dt, dt,
                                 cu_seqlens, n_seqs, workspace, ws_bytes, &n_seq);
    if (st != GDN_OK) return st;
    if (T > 0 && (!dq || !dk || !dv || !dg || !dbeta))
        return fail(GDN_ERR_INVALID_ARG, "a gradient output (dq, dk, dv, dg, dbeta) is NULL");
    const void* outs[] = {dq, dk, dv, dg, dbeta, dh0};
    for (const void* ptr : outs)
        if (ptr && !aligned16(ptr)) return fail(GDN_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", ptr);
    const size_t need = bwd_workspace_bytes(B, T, H, dk_, dv_, cu_seqlens ? n_seq : 0);
    if (!workspace || ws_bytes < need)
        return fail(GDN_ERR_INVALID_ARG, "the backward pass needs %zu bytes of workspace (got %zu)", need, ws_bytes);
    gdn_status es;
    unsigned* err = err_word_ptr(&es);
    if (!err) return es;
    const size_t states = bwd_state_bytes(B, T, H, dk_, dv_, cu_seqlens ? n_seq : 0) / sizeof(float);
    float* hc = static_cast<float*>(workspace);
    float* dhc = hc + states / 2;
    float* tp = hc + states;
    FwdParams fp{q, k, v, g, beta, nullptr, h0, nullptr, nullptr, cu_seqlens, scale, B, T, H, dk_, dv_, n_seq};
    fp.h_chunks = hc;
    BwdParams bp{q, k, v, g, beta, d_o, dhT, hc, dhc, tp, dq, dk, dv, dg, dbeta, dh0, cu_seqlens, scale,
                 B, T, H, dk_, dv_, n_seq};
    if (dt == GDN_F32)
        return dk_ == 64 ? launch_bwd_dk<float, 64>(fp, bp, err, stream) : launch_bwd_dk<float, 128>(fp, bp, err, stream);
    return dk_ == 64 ? launch_bwd_dk<__nv_bfloat16, 64>(fp, bp, err, stream)
                     : launch_bwd_dk<__nv_bfloat16, 128>(fp, bp, err, stream);
}

size_t gdn2_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs) {
    if (B < 1 || T < 0 || H < 1 || BT != kChunk || (dk != 64 && dk != 128) || dv < 64 || dv > 256 || dv % 64 != 0 ||
        n_seqs < 0)
        return 0;
    return bwd2_workspace_bytes(B, T, H, dk, dv, n_seqs);
}

gdn_status gdn2_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* b, const float* w,
                          float scale, const float* h0, const void* d_o, const float* dhT, float* dq, float* dk,
                          float* dv, float* dg, float* db, float* dw, float* dh0, int B, int T, int H, int dk_, int dv_,
                          int BT, gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs, void* workspace,
                          size_t ws_bytes, cudaStream_t stream) {
    return chunk_bwd2(q, k, v, g, b, w, false, scale, h0, d_o, dhT, dq, dk, dv, dg, db, dw, dh0, B, T, H, dk_, dv_, BT,
                      dt, cu_seqlens, n_seqs, workspace, ws_bytes, stream);
}

gdn_status gdn_kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             float scale, const float* h0, const void* d_o, const float* dhT, float* dq, float* dk,
                             float* dv, float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_, int dv_,
                             int BT, gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs, void* workspace,
                             size_t ws_bytes, cudaStream_t stream) {
    return chunk_bwd2(q, k, v, g, beta, nullptr, true, scale, h0, d_o, dhT, dq, dk, dv, dg, dbeta, nullptr, dh0, B, T,
                      H, dk_, dv_, BT, dt, cu_seqlens, n_seqs, workspace, ws_bytes, stream);
}

gdn_status gdn_set_kernel(gdn_kernel kernel) {
    if (kernel != GDN_KERNEL_AUTO && kernel != GDN_KERNEL_SIMT && kernel != GDN_KERNEL_TC)
        return fail(GDN_ERR_INVALID_ARG, "unknown kernel family %d", (int)kernel);
    g_kernel_choice.store(kernel);
    return GDN_OK;
}

gdn_kernel gdn_last_kernel(void) { return t_last_kernel; }

gdn_status gdn_debug_stall(int on) {
    g_debug_stall.store(on != 0);
    return GDN_OK;
}

gdn_status gdn_check_error(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    unsigned word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, g_err_word, sizeof(word));
    if (e == cudaSuccess && word) e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
    if (word & kErrTimeout) return fail(GDN_ERR_TIMEOUT, "a bounded device wait ran out (word 0x%x)", word);
    if (word & kErrSeqlens) return fail(GDN_ERR_DEVICE_ARG, "cu_seqlens out of order or out of range (word 0x%x)", word);
    return GDN_OK;
}

const char* gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "ok";
        case GDN_ERR_INVALID_ARG: return "invalid argument";
        case GDN_ERR_UNSUPPORTED: return "unsupported shape or option";
        case GDN_ERR_CUDA: return "CUDA error";
        case GDN_ERR_TIMEOUT: return "device wait timed out";
        case GDN_ERR_DEVICE_ARG: return "invalid cu_seqlens seen on the device";
    }
    return "unknown status";
}

const char* gdn_last_error(void) { return t_msg; }

gdn_status gdn_profile_enable(int on) {
    prof_state().on.store(on != 0);
    return GDN_OK;
}

gdn_status gdn_profile_take(int kernel, int* launches, double* total_ms) {
    t_msg[0] = 0;
    if (kernel < 0 || kernel >= PK_COUNT) return fail(GDN_ERR_INVALID_ARG, "kernel id must be 0..%d", PK_COUNT - 1);
    if (!launches || !total_ms) return fail(GDN_ERR_INVALID_ARG, "NULL output pointer");
    if (!prof_take(kernel, launches, total_ms)) return fail(GDN_ERR_CUDA, "a recorded launch event failed");
    return GDN_OK;
}

gdn_status gdn_debug_umma_selftest(const float* A, const float* B, float* D, int mode, cudaStream_t stream) {
    t_msg[0] = 0;
    if (!A || !B || !D) return fail(GDN_ERR_INVALID_ARG, "NULL pointer");
    if (mode < 0 || mode > 5) return fail(GDN_ERR_INVALID_ARG, "mode must be 0..5 (got %d)", mode);
    gdn_status st;
    unsigned* err = err_word_ptr(&st);
    if (!err) return st;
    const int smem = 65536 + 1024;
    cudaError_t e = cudaFuncSetAttribute(gdn_umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    gdn_umma_selftest_kernel<<<1, 128, smem, stream>>>(A, B, D, mode, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "selftest launch: %s", cudaGetErrorString(e));
    return GDN_OK;
}

}  // extern "C"
