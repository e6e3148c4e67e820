/*
 * libgdn -- chunked gated delta rule forward pass on NVIDIA B200 (sm_100a).  C ABI.
 *
 * Operations
 *   gdn_chunk_fwd   Gated delta rule (GDN): per (sequence, head), with state S (dk x dv, fp32),
 *                     S_t = exp(g_t) S_{t-1} + k_t u_t^T,   u_t = beta_t v_t - beta_t exp(g_t) S_{t-1}^T k_t,
 *                     o_t = scale * S_t^T q_t   (read after the write at t).
 *                   Definition: GatedDeltaNet data-flow walkthrough (yfxerp.com/news/367755), section
 *                   "Delta Rule: predict first, then correct" (the token-by-token reference loop); the
 *                   chunked evaluation (BT = 64 tokens per chunk, one state handed between chunks, WY form
 *                   of the intra-chunk dependency, gate cumsum times log2(e) so exp2 can be used) follows
 *                   section "Chunked parallelism: how the Triton kernels turn serial into parallel".
 *   gdn2_chunk_fwd  Gated Delta Rule-2 (GDN-2): per-channel decay alpha_t = exp(g_t) on the key axis,
 *                   erase gate b_t on the key axis, write gate w_t on the value axis,
 *                     S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,  o_t = scale S_t^T q_t.
 *                   Definition: NVIDIA Gated DeltaNet-2 article (7minutos.es), section "Regla-2 del Delta
 *                   cerrado: dos puertas en lugar de una"; chunk size C = 64 from section "Entrenamiento
 *                   fragmentado".
 *   gdn_kda_chunk_fwd  KDA (Kimi Delta Attention): GDN-2 with a per-channel decay and one scalar write strength
 *                   beta_t used as both the erase gate (b_t = beta_t on every key channel) and the write gate
 *                   (w_t = beta_t on every value column):
 *                     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = scale S_t^T q_t.
 *                   Definition: the Gated DeltaNet-2 article, section "Regla-2 del Delta cerrado" (when the two
 *                   gates collapse to the same scalar the rule is KDA exactly).
 *   The read-out o_t and scale = dk^-1/2 are not printed on the pages; o_t = scale S_t^T q_t is the adopted
 *   reading (the same for every operation).
 *
 * Layouts (row-major, contiguous, all device pointers):
 *   q, k        [B, T, H, dk]   dtype `dt` (GDN_F32 or GDN_BF16)
 *   v           [B, T, H, dv]   dtype `dt`
 *   o           [B, T, H, dv]   dtype `o_dt`: GDN_F32, or `dt` itself.  A bf16 o carries the format's own
 *                               rounding (half an ulp, 2^-9 relative, per element) on top of the kernel's error.
 *   GDN:   g, beta  [B, T, H]        fp32; g is the natural-log decay (g <= 0 expected), beta the write strength
 *   GDN-2: g, b     [B, T, H, dk]    fp32 per-channel log-decay and erase gate;  w [B, T, H, dv] fp32 write gate
 *   KDA:   g [B, T, H, dk] fp32 per-channel log-decay;  beta [B, T, H] fp32
 *   h0, hT      [N, H, dk, dv]  fp32, N = B, or n_seqs with cu_seqlens.  h0 == NULL means zeros;
 *                               hT == NULL means the final state is not written.
 *   cu_seqlens  int32 [n_seqs + 1] or NULL.  With cu_seqlens, B must be 1 and the T tokens of the single
 *               row are n_seqs packed sequences [cu[n], cu[n+1]); the state starts from h0[n] at each
 *               sequence start and chunks are aligned to the sequence start (the last may be partial).
 *               cu[0] = 0, non-decreasing, cu[n_seqs] = T; a zero-length sequence gives hT[n] = h0[n].
 *
 * Supported shapes: BT == 64; dk in {64, 128}; dv a multiple of 64 in [64, 256]; B >= 1, H >= 1, T >= 0.
 * Every pointer must be 16-byte aligned.  The library never allocates, frees or synchronises inside a
 * *_fwd call: the caller owns every buffer, and work is enqueued on `stream` (asynchronous).
 *
 * Workspace: the tensor-core path (bf16 inputs, dk == 128, dv a multiple of 128) first computes the WY
 * factors of every (chunk, head) -- T' = T diag(beta e^G) and T'' = T diag(beta) with T = (I + A)^-1 -- and
 * the gated read-out matrix P of every chunk into `workspace`, then runs the chunk recurrence that reads them;
 * it needs gdn_workspace_bytes() bytes (40 KB per chunk slot and head; slots = ceil(B T / 64) + number of
 * sequences).  The workspace is scratch:
 * its contents are undefined before and after a call, and it must not be shared by calls in flight at the
 * same time.  With a smaller (or NULL) workspace, AUTO runs the SIMT kernel and TC returns
 * GDN_ERR_UNSUPPORTED.  The GDN-2 and KDA tensor-core path (same shape rule) keeps, per chunk slot and head, an
 * 80.5 KB unit of state-independent operands (T, W, P and the gate-scaled q and k of the chunk) and needs
 * gdn2_workspace_bytes() instead.
 *
 * Errors
 *   Arguments are checked on the host before anything is enqueued; a failed check returns
 *   GDN_ERR_INVALID_ARG (bad pointer, size, alignment) or GDN_ERR_UNSUPPORTED (a shape or option outside
 *   the supported set) and has no side effects.  A failed launch returns GDN_ERR_CUDA.  Conditions only the
 *   device can see (a cu_seqlens entry out of order or out of range; a bounded wait that ran out) set a
 *   device error word instead of faulting; gdn_check_error() synchronises the stream and reports it.
 *   gdn_last_error() returns a short description of the most recent failure on the calling thread.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,
    GDN_ERR_UNSUPPORTED = 2,
    GDN_ERR_CUDA = 3,
    GDN_ERR_TIMEOUT = 4,
    GDN_ERR_DEVICE_ARG = 5 /* reported by gdn_check_error: cu_seqlens out of order or out of range */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype; /* dtype of q, k, v (dt) and of o (o_dt) */

/* Kernel family used for a call.  AUTO picks the tensor-core (tcgen05) kernel for bf16 inputs when the
 * shape allows it and the SIMT fp32 kernel otherwise.  SIMT forces the fp32-FMA kernel (any dtype); TC
 * forces the tcgen05 kernel (bf16 only; GDN_ERR_UNSUPPORTED otherwise). */
typedef enum { GDN_KERNEL_AUTO = 0, GDN_KERNEL_SIMT = 1, GDN_KERNEL_TC = 2 } gdn_kernel;

/* Bytes of caller-provided device workspace the tensor-core path needs for these sizes (see Workspace
 * above); 0 when only the SIMT kernel can take them (then pass NULL, 0).  n_seqs as for the *_fwd calls. */
size_t gdn_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs);

/* Bytes of workspace the GDN-2 / KDA tensor-core path needs (see Workspace above); 0 when only the SIMT kernel can
 * take these sizes. */
size_t gdn2_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs);

/* Gated delta rule forward; see the header comment for the definition, layouts and errors. */
gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float scale, const float* h0, void* o, float* hT,
                         int B, int T, int H, int dk, int dv, int BT, gdn_dtype dt, gdn_dtype o_dt,
                         const int32_t* cu_seqlens, int n_seqs,
                         void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Size of the scratch array compiled into the library for gdn_chunk_fwd_noalloc: 256 MiB of device memory.  It is
 * part of the library's device code, so the CUDA runtime reserves it on each device where it loads that code and
 * keeps it until the process exits.  With lazy module loading (the CUDA default) that happens during the first
 * call of ANY libgdn entry point on a device -- also in processes that never call gdn_chunk_fwd_noalloc -- and
 * that first call can therefore fail with GDN_ERR_CUDA (out of memory) on a nearly full device. */
#define GDN_STATIC_WS_BYTES (256u * 1024u * 1024u)

/* gdn_chunk_fwd for callers that cannot allocate device memory.  (The pages have no counterpart to this entry
 * point: it exists for the library's users.)  Some callers may not call cudaMalloc at all: serving engines that
 * hand all free device memory to their own pool at start-up and forbid any later allocation; plug-ins running
 * inside a host framework that owns the device allocator; and latency-critical loops, where cudaMalloc and
 * cudaFree may synchronise the device and take unbounded time.  This entry point takes no workspace and
 * allocates nothing -- no cudaMalloc, cudaFree or allocating library routine: the tensor-core path keeps its
 * per-chunk WY factors in the library's static scratch array (GDN_STATIC_WS_BYTES, see above).  The caller still
 * passes every input and output buffer.
 *   Set-up: the first call on a device, with that device current, looks the scratch array's device address up
 *   (cudaGetSymbolAddress) and caches it for later calls on that device.  Make that first call before any stream
 *   capture, since the look-up may load the library's device code.
 *   Limit: when the call would run the tensor-core path (bf16 inputs, dk == 128, dv a multiple of 128, kernel not
 *   forced to SIMT) and gdn_workspace_bytes() for these sizes exceeds GDN_STATIC_WS_BYTES, the call is refused
 *   with GDN_ERR_UNSUPPORTED (gdn_last_error() says how much it needed) and nothing is enqueued.  Calls that run
 *   the SIMT kernel use no scratch and have no such limit.
 *   Sharing: every call in the process uses the same array on a device, and a call leaves its contents behind
 *   (nothing in it has to start at zero: each call writes every byte it later reads).  Calls that overlap on the
 *   device -- issued on different streams without ordering between them -- race on the array and give undefined
 *   results: issue them on one stream, or order them with events; concurrent callers use gdn_chunk_fwd with their
 *   own workspaces.
 * Arguments, layouts, results and errors are otherwise those of gdn_chunk_fwd. */
gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                 float scale, const float* h0, void* o, float* hT,
                                 int B, int T, int H, int dk, int dv, int BT, gdn_dtype dt, gdn_dtype o_dt,
                                 const int32_t* cu_seqlens, int n_seqs, cudaStream_t stream);

/* Gated Delta Rule-2 forward; g, b are [B,T,H,dk] and w is [B,T,H,dv], all fp32. */
gdn_status gdn2_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* b,
                          const float* w, float scale, const float* h0, void* o, float* hT,
                          int B, int T, int H, int dk, int dv, int BT, gdn_dtype dt, gdn_dtype o_dt,
                          const int32_t* cu_seqlens, int n_seqs,
                          void* workspace, size_t ws_bytes, cudaStream_t stream);

/* KDA forward (GDN-2 with b = w = beta); g is [B,T,H,dk] and beta [B,T,H], both fp32.  Workspace as for
 * gdn2_chunk_fwd (gdn2_workspace_bytes); arguments, layouts and errors otherwise those of gdn_chunk_fwd. */
gdn_status gdn_kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             float scale, const float* h0, void* o, float* hT,
                             int B, int T, int H, int dk, int dv, int BT, gdn_dtype dt, gdn_dtype o_dt,
                             const int32_t* cu_seqlens, int n_seqs,
                             void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Recurrent decode step: one new token for each of N sequences, the state updated in place.  Per (sequence n,
 * head h) it is one step of the token recurrence (the GatedDeltaNet walkthrough's reference loop, section "Delta
 * Rule: predict first, then correct"; GDN-2 and KDA as in the Gated DeltaNet-2 article, section "Regla-2 del Delta
 * cerrado"; decoding with constant memory is the point of the fixed-size state, the article's opening paragraph):
 *   S <- Diag(exp(g)) S;  u = z - S^T e;  S <- S + k u^T;  o = scale S^T q
 * with e = beta k, z = beta v (GDN; KDA with a per-channel g), or e = b . k, z = w . v (GDN-2).
 * Layouts (device, row-major): q, k [N, H, dk] and v [N, H, dv] in `dt`; o [N, H, dv] in `o_dt` (fp32 or `dt`);
 * state [N, H, dk, dv] fp32, read and overwritten (it is h0 on entry and hT on return).  GDN: g, beta [N, H];
 * GDN-2: g, b [N, H, dk] and w [N, H, dv]; KDA: g [N, H, dk] and beta [N, H]; all gates fp32.  dk in {64, 128},
 * dv a multiple of 64 in [64, 256], N >= 1, H >= 1, pointers 16-byte aligned.  Asynchronous on `stream`; the
 * caller owns every buffer; nothing is allocated.  Errors as for gdn_chunk_fwd (host checks before any launch). */
gdn_status gdn_decode_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta, float scale,
                          float* state, void* o, int N, int H, int dk, int dv, gdn_dtype dt, gdn_dtype o_dt,
                          cudaStream_t stream);
gdn_status gdn2_decode_fwd(const void* q, const void* k, const void* v, const float* g, const float* b, const float* w,
                           float scale, float* state, void* o, int N, int H, int dk, int dv, gdn_dtype dt,
                           gdn_dtype o_dt, cudaStream_t stream);
gdn_status gdn_kda_decode_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                              float scale, float* state, void* o, int N, int H, int dk, int dv, gdn_dtype dt,
                              gdn_dtype o_dt, cudaStream_t stream);

/* The mixer's prelude, one launch (GatedDeltaNet walkthrough, sections "Short convolution" and "Gating"; Gated
 * DeltaNet-2 article, section "Diseno de bloques y modelo hibrido"):
 *   q = l2norm(silu(conv4(xq))), k = l2norm(silu(conv4(xk))), v = silu(conv4(xv)),
 *   g = -exp(A_log[h]) * softplus(a + dt_bias[h]),  beta = sigmoid(b),  w_gate = sigmoid(c) (optional),
 * where conv4 is a depthwise causal convolution per channel, y[t] = w[0] x[t-3] + w[1] x[t-2] + w[2] x[t-1] + w[3] x[t]
 * (no bias), inputs before a sequence start taken from conv_in (or 0), and l2norm(x) = x / sqrt(sum x^2 + l2_eps) over
 * each head's channels.  Layouts (device, row-major): xq, xk, q, k [B, T, H, dk] and xv, v [B, T, H, dv] in `dt`;
 * taps wq, wk [H*dk][4], wv [H*dv][4] fp32; conv_in / conv_out [N][2*H*dk + H*dv][3] fp32 (channels of q, then k, then
 * v; the three inputs before / at the end of each sequence, oldest first; NULL conv_in means zeros, NULL conv_out
 * means not written; one buffer for both only when T == 1 and cu_seqlens is NULL, the decode step); a, g [B, T, H,
 * g_width], b, beta [B, T, H, b_width], c, w_gate [B, T, H, c_width] (c and w_gate both NULL or both given), A_log,
 * dt_bias [H], all fp32.  cu_seqlens as for gdn_chunk_fwd (sequence starts also restart the convolution).  dk in
 * {64, 128}, dv a multiple of 64 in [64, 256], widths in [1, 256].  Asynchronous, no allocation; host checks as for
 * gdn_chunk_fwd. */
gdn_status gdn_prelude_fwd(const void* xq, const void* xk, const void* xv, const float* wq, const float* wk,
                           const float* wv, const float* conv_in, float* conv_out, const float* a, const float* A_log,
                           const float* dt_bias, float* g, int g_width, const float* b, float* beta, int b_width,
                           const float* c, float* w_gate, int c_width, void* q, void* k, void* v, int B, int T, int H,
                           int dk, int dv, gdn_dtype dt, float l2_eps, const int32_t* cu_seqlens, int n_seqs,
                           cudaStream_t stream);

/* The mixer's epilogue (the walkthrough's fused RMSNorm with a Swish gate, data-flow step 5): over each of `rows`
 * rows of dv channels, y = o / sqrt(mean(o^2) + eps) * weight * silu(z).  o, z, y [rows][dv] in `dt` (device);
 * weight [dv] fp32, shared by every row.  dv a multiple of 64 in [64, 256].  Asynchronous, no allocation. */
gdn_status gdn_output_gate_fwd(const void* o, const void* z, const float* weight, void* y, long long rows, int dv,
                               gdn_dtype dt, float eps, cudaStream_t stream);

/* Backward pass (reverse mode) of gdn_chunk_fwd: given the cotangents d_o of o and dhT of the final state, the
 * gradients of <d_o, o> + <dhT, hT> with respect to q, k, v, g, beta and h0.  (The walkthrough's section "Chunked
 * parallelism" names this full backward for q, k, v, beta and g.)  It runs the chunk recurrence backwards through
 * the WY form: the forward states at every chunk start are recomputed into the workspace, the state cotangent is
 * carried from the last chunk to the first, and every chunk's input gradients are then formed in parallel.
 * Arithmetic is fp32 on CUDA cores for both input dtypes.
 * Layouts: q, k, v, d_o as for gdn_chunk_fwd (d_o [B,T,H,dv] in `dt`); g, beta [B,T,H] fp32; h0, dhT
 * [N,H,dk,dv] fp32 or NULL (zeros); outputs dq, dk [B,T,H,dk], dv [B,T,H,dv], dg, dbeta [B,T,H] and dh0
 * [N,H,dk,dv] (NULL: not written), all fp32, overwritten.  Workspace: gdn_bwd_workspace_bytes() bytes (two fp32
 * states and the fp32 T and P of every chunk slot and head), required.  bf16 inputs of a tensor-core shape
 * recompute the chunk-start states with the tensor-core forward, everything else with the SIMT forward.
 * Shapes, cu_seqlens and errors as for gdn_chunk_fwd. */
size_t gdn_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs);
gdn_status gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta, float scale,
                         const float* h0, const void* d_o, const float* dhT, float* dq, float* dk, float* dv,
                         float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_, int dv_, int BT,
                         gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs, void* workspace, size_t ws_bytes,
                         cudaStream_t stream);

/* Backward pass of gdn2_chunk_fwd (GDN-2) and of gdn_kda_chunk_fwd (KDA): the gradients of <d_o, o> + <dhT, hT>
 * with respect to q, k, v, the per-channel decay g, the gates and h0.  (Gated DeltaNet-2 article, section
 * "Entrenamiento fragmentado y reconocimiento de puertas hacia atras": the gate factors sit inside the gradient's
 * dot products; the walkthrough's section "Chunked parallelism" names the full backward.)  Same structure as
 * gdn_chunk_bwd, with the decay of every key channel inside A and P: the states at every chunk start are
 * recomputed, T = (I + A)^-1 and P of every chunk are formed into the workspace, the state cotangent is carried
 * from the last chunk to the first, and the input gradients of every chunk are formed in parallel.  The gate
 * gradient of channel i at row r comes out of the identity dGn_ri = q_ri dq_ri + e_ri de_ri - k_ri dk_ri (every
 * q and erase key carries exp(+G), every key exp(-G)) plus the chunk-end terms, then a reverse cumulative sum.
 * Arithmetic is fp32 on CUDA cores for both input dtypes.
 * GDN-2: g, b [B,T,H,dk], w [B,T,H,dv] fp32; outputs dq, dk, dg, db [B,T,H,dk], dv, dw [B,T,H,dv].
 * KDA: g [B,T,H,dk], beta [B,T,H] fp32; outputs dq, dk, dg [B,T,H,dk], dv [B,T,H,dv], dbeta [B,T,H] (beta is
 * both the erase and the write strength, so dbeta sums both shares).
 * Both: d_o [B,T,H,dv] in `dt`; h0, dhT [N,H,dk,dv] fp32 or NULL (zeros); dh0 [N,H,dk,dv] or NULL (not
 * written); every output fp32, overwritten.  Workspace: gdn2_bwd_workspace_bytes() bytes (two fp32 states and
 * the fp32 T and P of every chunk slot and head), required.  Shapes, cu_seqlens and errors as for
 * gdn_chunk_fwd. */
size_t gdn2_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, int BT, int n_seqs);
gdn_status gdn2_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* b, const float* w,
                          float scale, const float* h0, const void* d_o, const float* dhT, float* dq, float* dk,
                          float* dv, float* dg, float* db, float* dw, float* dh0, int B, int T, int H, int dk_, int dv_,
                          int BT, gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs, void* workspace,
                          size_t ws_bytes, cudaStream_t stream);
gdn_status gdn_kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             float scale, const float* h0, const void* d_o, const float* dhT, float* dq, float* dk,
                             float* dv, float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_, int dv_,
                             int BT, gdn_dtype dt, const int32_t* cu_seqlens, int n_seqs, void* workspace,
                             size_t ws_bytes, cudaStream_t stream);

/* Selects the kernel family for later calls from any thread (process-wide; default AUTO). */
gdn_status gdn_set_kernel(gdn_kernel kernel);

/* Kernel family that the most recent successful *_fwd call on this thread launched. */
gdn_kernel gdn_last_kernel(void);

/* Diagnostic of the device time-out path (no counterpart on the pages; off by default; process-wide).  While
 * on, every later tensor-core GDN call makes one of its chunk kernel's pipeline waits wait on a barrier that
 * nothing ever arrives on, with a ~1 ms limit.  The wait runs out, the kernel sets the device error word, its
 * warps leave through their own bounded waits after draining every copy and tensor-core operation they issued,
 * and the call's outputs are undefined; the call itself returns GDN_OK and gdn_check_error() then reports
 * GDN_ERR_TIMEOUT.  Calls on the SIMT kernel are not affected.  Returns GDN_OK. */
gdn_status gdn_debug_stall(int on);

/* Synchronises `stream`, then reads and clears the device error word of the current device:
 * GDN_OK, GDN_ERR_TIMEOUT, GDN_ERR_DEVICE_ARG, or GDN_ERR_CUDA if the stream reports a CUDA error. */
gdn_status gdn_check_error(cudaStream_t stream);

/* Static description of a status code. */
const char* gdn_status_string(gdn_status status);

/* Description of the most recent failure on the calling thread ("" if none). */
const char* gdn_last_error(void);

/* Diagnostic (no counterpart on the pages): checks the tensor-core operand layouts the tcgen05 kernels use.
 * One CTA stages A (row-major [M][K] fp32, device) and B (row-major [K][N] fp32, device) in shared or tensor
 * memory in the layout selected by `mode` -- bf16 operands: 0: A K-major 128x128, B K-major, N=64; 1: A
 * MN-major 128x64, B K-major, N=64; 2: A K-major 128x64, B MN-major, N=128; 3: A K-major 128x128, B
 * MN-major, N=64; 4: A 128x64 in tensor memory, B K-major, N=64; tf32 operands (fp32 storage): 5: A 128x32
 * in tensor memory, B K-major, N=64 -- runs the MMA k-step loop, and writes D = A B (fp32, row-major
 * [M][N], device).  Mode outside 0..5: GDN_ERR_INVALID_ARG.
 * Asynchronous on `stream`. */
gdn_status gdn_debug_umma_selftest(const float* A, const float* B, float* D, int mode, cudaStream_t stream);

/* Per-kernel device timing, a measurement aid (off by default; process-wide).  While enabled, every kernel
 * launch made by the *_fwd calls is bracketed by two CUDA events recorded on its stream.
 * gdn_profile_take(kernel, &launches, &total_ms) waits for the recorded events of one kernel -- 0: SIMT
 * kernel, 1: tensor-core WY kernel, 2: tensor-core chunk kernel, 3: GDN-2 / KDA prep kernel, 4: GDN-2 / KDA
 * chunk kernel, 5: decode kernel, 6: prelude kernel, 7: output gate kernel, 8: the backward's two kernels
 * (its forward recompute counts as 0) -- returns how many launches they cover and
 * their summed device time in milliseconds, and forgets them.  Errors: GDN_ERR_INVALID_ARG for an unknown
 * kernel id or NULL outputs, GDN_ERR_CUDA if an event failed. */
gdn_status gdn_profile_enable(int on);
gdn_status gdn_profile_take(int kernel, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
