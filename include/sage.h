/*
 * sage.h -- C ABI of the B200 (sm_100a) quantized-attention library (libsage.so).
 *
 * The library computes the forward pass of SageAttention-style quantized
 * attention:  out = softmax(Q K^T * sm_scale) V  with
 *   - K smoothed by subtracting its per-(batch, head, channel) mean over tokens,
 *   - Q in INT8 per 128-token block and K in INT8 per 64-token block
 *     (symmetric, one fp32 scale per block),
 *   - S = Q K^T on the INT8 tensor cores with int32 accumulation, dequantized
 *     by the block scales,
 *   - an online softmax in base 2 whose running row max stays on the integer
 *     grid (rescale factors are exact powers of two),
 *   - P (scaled by 448) and V (per-channel scale) in FP8 e4m3, P V on the FP8
 *     tensor cores with fp32 accumulation, bf16 output.
 *
 * Sources (web pages, by title and section):
 *   [H3]   "MiniMax H3 接入 SageAttention 实测加速", section 一 "SageAttention 加速了什么":
 *          Attention(Q,K,V) = Softmax(Q K^T / sqrt(d)) V; low-bit quantization and
 *          outlier smoothing of Q K^T; INT8 for QK and FP8 for PV.
 *   [SDPA] "SDPA稠密注意力模式：大模型推理加速的优化方案", section 三.1 "数学基础":
 *          the dense formula with the 1/sqrt(d_k) scale (the dense reference).
 *   [BLOG] "GitHub榜单静默期：Attention优化从架构转向推理加速", section 2.2:
 *          block-wise computation that never writes the attention matrix out.
 *   [SOL]  "ComfyUI-sol-attn" page, "核心亮点" items 1, 2 and 4: K-residual
 *          quantization with the block-mean term kept at bf16; zero-copy reads of a
 *          fused-qkv strided view; explicit, logged rejection of unsupported
 *          inputs instead of a silent fallback; scheduled sparsity, a value
 *          tau that may ramp over the sampling steps (sparse early, dense late).
 * Numeric points the pages leave open follow the readings C1..C9 of the
 * project's design notes (block sizes, rounding modes, integer-grid row max,
 * 448 P scale, per-channel V scale, fp32 accumulation, bf16 RNE output).
 *
 * Conventions for every entry point
 *   - Tensors are described by a base pointer plus four int64 ELEMENT strides in
 *     (b, h, n, c) order; the channel stride must be 1.  A fused [B,N,3,H,d]
 *     qkv buffer is passed as three views with strides (N*3*H*d, d, 3*H*d, 1)
 *     and read in place (no copy).
 *   - Inputs and output are bf16.  d must be 64 or 128; N >= 1; B, H >= 1;
 *     B*H <= 65535 and N <= 2^24.  Base pointers must be 16-byte aligned and
 *     the b, h, n strides multiples of 8 elements (16-byte vectors).
 *     Otherwise SAGE_ERR_INVALID_ARG (bad pointer/stride/shape/scale) or
 *     SAGE_ERR_UNSUPPORTED (d, B*H, N) is returned before anything is
 *     launched, and every size query below answers 0 for such a shape.
 *   - Input values are finite.  With an infinity or NaN in a block the codes of
 *     that block (and every output that uses them) are unspecified; nothing
 *     checks for it.
 *   - A forward launches its kernels back to back on `stream`; all but the
 *     first may begin while their predecessor finishes (programmatic dependent
 *     launch) and wait on the device for its results, so the call's ordering
 *     with respect to other work on `stream` is the ordinary stream order.
 *   - N_pad = ceil(N/128)*128.  Padded rows of every code buffer are written
 *     as zeros; padded blocks get scale 0.
 *   - Device tensors must live on the current device (checked on the first
 *     input and the output: SAGE_ERR_INVALID_ARG otherwise); kernels launch on
 *     the current device.
 *   - Every device buffer is owned by the caller; the library keeps no pointer
 *     after a call returns.  Calls are asynchronous on `stream` and return
 *     after the launches.  A kernel that gives up waiting on an internal
 *     barrier (a bounded wait) records it in a device error word that
 *     sage_check() reports as SAGE_ERR_TIMEOUT.
 *   - There is no fallback of any kind: an unsupported input is an error.
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle types as cudaStream_t / cudaEvent_t (the runtime's opaque pointers). */
typedef struct CUstream_st *sage_stream_t;
typedef struct CUevent_st *sage_event_t;

typedef enum {
    SAGE_OK = 0,
    SAGE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad stride, shape or scale   */
    SAGE_ERR_UNSUPPORTED = 2,  /* head dim not in {64,128}                             */
    SAGE_ERR_WORKSPACE = 3,    /* workspace given but smaller than required             */
    SAGE_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (message has it)    */
    SAGE_ERR_TIMEOUT = 5       /* a device-side bounded wait expired (see sage_check)   */
} sage_status_t;

/* Human-readable name of a status code (static string). */
const char *sage_status_string(sage_status_t status);

/* Detail of the last error raised on the calling host thread ("" if none). */
const char *sage_last_error_message(void);

/* Synchronize `stream`, then read and clear the device error word.  Returns
 * SAGE_ERR_TIMEOUT if any kernel of this library gave up on a bounded wait
 * since the last check, SAGE_ERR_CUDA on a failed synchronize, else SAGE_OK. */
sage_status_t sage_check(sage_stream_t stream);

/* Bytes of scratch sage_attn_fwd needs for this shape (codes, scales, stats).
 * 0 for an invalid shape.  Layout inside it is private. */
size_t sage_attn_workspace_bytes(int B, int H, int N, int d);

/* Bytes of scratch sage_quant_qk / sage_quant_v need (the partial statistics
 * of the smoothing mean and of the V channel maxima, one per pair of a head
 * and a CTA of the quantize kernel that covers part of it): with
 * S = B*H + min(512, B*H*ceil(N/128)) slots and up(x) = x rounded up to 1024,
 *   up(8*S*d) + up(4*S*d) + up(8*S)
 * (fp64 K sums, fp32 V maxima and a 64-bit publication flag per slot); 0 for
 * an invalid shape.  Nothing in it needs to start at zero. */
size_t sage_quant_workspace_bytes(int B, int H, int N, int d);

/*
 * sage_quant_qk -- smoothing plus block quantization of Q and K ([H3] section 一;
 * readings C1-C3).
 *   k_mean[b,h,c] = fp32( (sum_n K[b,h,n,c]) / N )   (the sum in fp64, exact
 *       whenever a column's values span fewer than 53 bits; one fp64 division)
 *   Q, per 128-token block:  amax = max|Q| over the block's valid tokens and all
 *       channels; q_scale = amax/127; q_i8 = rne(Q * (127/amax)) in [-127,127]
 *   K, the same per 64-token block on (K - k_mean).
 * Outputs (device, caller-allocated, contiguous):
 *   q_i8    int8  [B,H,N_pad,d]      q_scale float [B,H,N_pad/128]
 *   k_i8    int8  [B,H,N_pad,d]      k_scale float [B,H,N_pad/64]
 *   k_mean  float [B,H,d]  (may be NULL)
 * workspace: >= sage_quant_workspace_bytes() device bytes, or NULL to let the
 * library take it from the stream-ordered allocator for the duration of the call.
 */
sage_status_t sage_quant_qk(const void *q_bf16, const int64_t q_stride[4],
                            const void *k_bf16, const int64_t k_stride[4],
                            int B, int H, int N, int d,
                            int8_t *q_i8, float *q_scale,
                            int8_t *k_i8, float *k_scale, float *k_mean,
                            void *workspace, size_t workspace_bytes,
                            sage_stream_t stream);

/*
 * sage_quant_qk_noalloc -- sage_quant_qk for callers that cannot allocate device
 * memory while they run: an engine or server plugin whose device memory is
 * budgeted up front and whose execution path forbids cudaMalloc /
 * cudaMallocAsync, or code whose allocator belongs to a host framework.  The
 * pages have no counterpart of this entry point; it changes only where the
 * pass's scratch lives.
 *   Same arguments, outputs and results as sage_quant_qk, without the
 *   workspace.  The statistics scratch is a fixed array of
 *   SAGE_NOALLOC_SCRATCH_BYTES (4 MiB) inside the library's device memory;
 *   every GPU that loads the library holds it until the process exits.  A shape
 *   whose scratch (sage_quant_workspace_bytes, about 12*d*(B*H + 512) bytes)
 *   exceeds it is rejected with SAGE_ERR_WORKSPACE before anything is
 *   launched: e.g. (1,24,4608,128) and (1,24,65536,128) need 0.83 MB and
 *   (1,40,34020,128) 0.85 MB and fit; with d = 128 up to about 2200 heads
 *   (B*H) fit, with d = 64 about 4900.  The inputs must be on the current
 *   device (SAGE_ERR_INVALID_ARG otherwise).  The call allocates nothing.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and keeps it; make that first call before any stream
 *   capture, and do not go on using the library after cudaDeviceReset.
 *   All calls on a device share the array: calls that may overlap on the GPU
 *   (different streams without ordering) race and must be serialized by the
 *   caller.  The array keeps the last call's contents; nothing in it needs to
 *   start at zero.
 */
#define SAGE_NOALLOC_SCRATCH_BYTES (4u << 20)
sage_status_t sage_quant_qk_noalloc(const void *q_bf16, const int64_t q_stride[4],
                                    const void *k_bf16, const int64_t k_stride[4],
                                    int B, int H, int N, int d,
                                    int8_t *q_i8, float *q_scale,
                                    int8_t *k_i8, float *k_scale, float *k_mean,
                                    sage_stream_t stream);

/*
 * sage_quant_v -- V to FP8 e4m3 with one scale per (b,h,channel) ([H3] "FP8 for
 * PV"; reading C7):  amax_c = max_n |V|;  v_scale = amax_c/448;
 * v_e4m3[b,h,n,c] = e4m3_rn_satfinite(V * (448/amax_c)).
 * Outputs: v_e4m3 uint8 (e4m3 bits) [B,H,N_pad,d], token-major like the int8
 * codes; v_scale float [B,H,d].  workspace as for sage_quant_qk.
 */
sage_status_t sage_quant_v(const void *v_bf16, const int64_t v_stride[4],
                           int B, int H, int N, int d,
                           uint8_t *v_e4m3, float *v_scale,
                           void *workspace, size_t workspace_bytes,
                           sage_stream_t stream);

/*
 * sage_attn_quantized -- the fused attention kernel alone, on codes produced by
 * sage_quant_qk / sage_quant_v (or any producer of the same layouts):
 *   x = S_int * (q_scale * sm_scale * log2(e) * k_scale)   (int32 S on tcgen05 kind::i8)
 *   running max m on the integer grid; p = 2^(x - m); l = sum p (fp32)
 *   P = e4m3(448 p) in tensor memory; O += P V on tcgen05 kind::f8f6f4 (fp32)
 *   out = O * v_scale / (448 l) -> bf16 (round to nearest even)
 * [BLOG] section 2.2 (block-wise, no N x N matrix); readings C4-C8.
 * out: bf16, strides as described above.  sm_scale finite and > 0.
 */
sage_status_t sage_attn_quantized(const int8_t *q_i8, const float *q_scale,
                                  const int8_t *k_i8, const float *k_scale,
                                  const uint8_t *v_e4m3, const float *v_scale,
                                  void *out, const int64_t o_stride[4],
                                  int B, int H, int N, int d, float sm_scale,
                                  sage_stream_t stream);

/*
 * sage_attn_fwd -- the whole quantized attention forward: sage_quant_qk,
 * sage_quant_v and sage_attn_quantized on scratch taken from `workspace`
 * (>= sage_attn_workspace_bytes(B,H,N,d) bytes, or NULL: stream-ordered
 * allocation for the duration of the call).  q, k, v may be strided views of
 * one fused qkv buffer ([SOL] item 2).  sm_scale is usually 1/sqrt(d).
 */
sage_status_t sage_attn_fwd(const void *q, const int64_t q_stride[4],
                            const void *k, const int64_t k_stride[4],
                            const void *v, const int64_t v_stride[4],
                            void *out, const int64_t o_stride[4],
                            int B, int H, int N, int d, float sm_scale,
                            void *workspace, size_t workspace_bytes,
                            sage_stream_t stream);

/*
 * sage_attn_fwd_ev -- sage_attn_fwd that also records `attn_begin` / `attn_end`
 * (CUDA events created by the caller; either may be NULL) on `stream` right
 * before and right after the fused attention kernel, so a caller can time that
 * kernel inside the whole forward.  Same arguments, layouts and errors as
 * sage_attn_fwd, which is this call with two NULL events.
 */
sage_status_t sage_attn_fwd_ev(const void *q, const int64_t q_stride[4],
                               const void *k, const int64_t k_stride[4],
                               const void *v, const int64_t v_stride[4],
                               void *out, const int64_t o_stride[4],
                               int B, int H, int N, int d, float sm_scale,
                               void *workspace, size_t workspace_bytes,
                               sage_stream_t stream,
                               sage_event_t attn_begin, sage_event_t attn_end);

/* Layouts of the one host buffer that holds q, k and v for sage_attn_fwd_host. */
#define SAGE_LAYOUT_FUSED 0      /* [B,N,3,H,d]: per token, the q, k and v rows of every head */
#define SAGE_LAYOUT_CONTIGUOUS 1 /* [3,B,H,N,d]: q, then k, then v, each [B,H,N,d] */

/* Bytes of device scratch sage_attn_fwd_host needs (0 for a shape it rejects):
 * the input and output on the device plus two chunk workspaces. */
size_t sage_attn_fwd_host_scratch_bytes(int B, int H, int N, int d);

/*
 * sage_attn_fwd_host -- sage_attn_fwd on HOST memory, the end-to-end call:
 * `qkv_host` (bf16, `layout` as above) goes to the device, the forward runs,
 * and the bf16 result lands in `out_host` ([B,H,N,d] contiguous).  The heads
 * are processed in chunks on three internal streams so that host<->device
 * copies overlap the kernels of other chunks; each chunk's result is the
 * whole call's result for its heads, bit for bit (every statistic is per
 * head).  Host buffers should be page-locked (cudaHostAlloc / pinned) for the
 * copies to be asynchronous; pageable buffers work but serialise.
 *   scratch: device buffer of >= sage_attn_fwd_host_scratch_bytes(B,H,N,d)
 *            bytes, 256-byte aligned, or NULL (allocated and freed on `stream`).
 * Enqueued after the work already on `stream`; `stream` continues after the
 * whole call (out_host is complete once `stream` reaches that point).
 * Errors: SAGE_ERR_INVALID_ARG (null buffer, layout, shape, sm_scale),
 * SAGE_ERR_UNSUPPORTED (d; B*H > 65535 or N > 2^24, the limits of every
 * entry point), SAGE_ERR_WORKSPACE (scratch too small), SAGE_ERR_CUDA.  The pages have no counterpart; this is the call a serving
 * path with host-resident tensors makes.
 */
sage_status_t sage_attn_fwd_host(const void *qkv_host, int layout, void *out_host,
                                 int B, int H, int N, int d, float sm_scale,
                                 void *scratch, size_t scratch_bytes, sage_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Block-sparse skipping ([SOL] item 4).  The page names only the control     */
/* (tau, ramped over the sampling steps); the steps are this library's        */
/* readings S1-S4:                                                           */
/*   S1 query and key tiles of 128 tokens;                                    */
/*   S2 tile-pair score = mean dequantized score of the pair in log2 units,   */
/*      (sum_i q).(sum_j k) * fp32(sm_scale*log2 e) / (n_i n_j), from the    */
/*      codes of sage_quant_qk, in fp32 in a fixed order;                     */
/*   S3 query tile i keeps the shortest prefix of its key tiles, ranked by    */
/*      score (ties: lower index first), whose estimated mass                 */
/*      n_j 2^(score - top score) reaches tau of the row's total; tau >= 1    */
/*      keeps every tile, and a row never keeps fewer than one;               */
/*   S4 sage_tau_schedule: tau moves linearly over the sampling steps.        */
/* Mask layout: uint32 words [B*H][T][W], T = ceil(N/128) tiles,              */
/* W = ceil(T/32); bit j of row (b*H+h, i) set = query tile i attends to key  */
/* tile j.  A query tile whose row is empty gets output 0.  Sparse calls      */
/* accept N up to 4096*128 tokens (T <= 4096); larger is SAGE_ERR_UNSUPPORTED.*/
/* ------------------------------------------------------------------------ */

/* Bytes of one mask (0 for a shape rejected): B*H*T*W*4. */
size_t sage_block_mask_bytes(int B, int H, int N);

/* Bytes of scratch sage_block_select needs (0 for a shape rejected). */
size_t sage_block_select_workspace_bytes(int B, int H, int N, int d);

/*
 * sage_block_select -- readings S2 and S3 on the codes of sage_quant_qk
 * (q_i8/k_i8 [B,H,N_pad,d], q_scale [B,H,N_pad/128], k_scale [B,H,N_pad/64]):
 * writes `mask` (device, 4-byte aligned, sage_block_mask_bytes) and, if
 * `scores` is not NULL, the tile-pair scores as fp32 [B*H][T][T].
 * tau must be finite and > 0.  workspace: >= sage_block_select_workspace_bytes
 * bytes, 256-byte aligned, or NULL (stream-ordered allocation).
 */
sage_status_t sage_block_select(const int8_t *q_i8, const float *q_scale,
                                const int8_t *k_i8, const float *k_scale,
                                int B, int H, int N, int d, float sm_scale, float tau,
                                uint32_t *mask, float *scores,
                                void *workspace, size_t workspace_bytes,
                                sage_stream_t stream);

/* Bytes of scratch sage_attn_fwd_sparse needs: the forward's plus the
 * selection's plus one mask. */
size_t sage_attn_sparse_workspace_bytes(int B, int H, int N, int d);

/*
 * sage_attn_fwd_sparse -- sage_attn_fwd with block-sparse skipping: the
 * quantize pass, then the key-tile mask (mask_in if not NULL, else
 * sage_block_select with `tau`, copied to mask_out if that is not NULL), then
 * the fused attention kernel visiting only each query tile's kept key tiles.
 * With every bit set the result equals sage_attn_fwd's bit for bit; with
 * tau >= 1 and no mask_in the dense kernel runs (the same result).
 * attn_begin / attn_end: optional events recorded around the attention kernel
 * (as in sage_attn_fwd_ev).  Errors as sage_attn_fwd, plus SAGE_ERR_INVALID_ARG
 * for tau (when no mask_in is given) and misaligned masks, and
 * SAGE_ERR_UNSUPPORTED for T > 4096.
 */
sage_status_t sage_attn_fwd_sparse(const void *q, const int64_t q_stride[4],
                                   const void *k, const int64_t k_stride[4],
                                   const void *v, const int64_t v_stride[4],
                                   void *out, const int64_t o_stride[4],
                                   int B, int H, int N, int d, float sm_scale, float tau,
                                   const uint32_t *mask_in, uint32_t *mask_out,
                                   void *workspace, size_t workspace_bytes,
                                   sage_stream_t stream,
                                   sage_event_t attn_begin, sage_event_t attn_end);

/*
 * sage_tau_schedule -- reading S4: tau at sampling step `step` of `n_steps`,
 * tau_start at the first step moving linearly to tau_end at the last (steps
 * outside the range clamp to it; one step gives tau_end).  [SOL] item 4 ramps
 * from sparse (small tau) early to dense (tau = 1) late.  Host function.
 */
float sage_tau_schedule(int step, int n_steps, float tau_start, float tau_end);

/*
 * sage_attn_fwd_fused_q -- sage_attn_fwd with Q quantized inside the fused
 * attention kernel: the quantize pass codes K and V only; each attention CTA
 * loads its two tiles' bf16 Q rows, takes each tile's |max| and writes the
 * INT8 codes into shared memory with the same arithmetic, so the result equals
 * sage_attn_fwd's bit for bit.  Same arguments, scratch size
 * (sage_attn_workspace_bytes), events and errors as sage_attn_fwd_ev.
 */
sage_status_t sage_attn_fwd_fused_q(const void *q, const int64_t q_stride[4],
                                    const void *k, const int64_t k_stride[4],
                                    const void *v, const int64_t v_stride[4],
                                    void *out, const int64_t o_stride[4],
                                    int B, int H, int N, int d, float sm_scale,
                                    void *workspace, size_t workspace_bytes,
                                    sage_stream_t stream,
                                    sage_event_t attn_begin, sage_event_t attn_end);

/* ------------------------------------------------------------------------ */
/* K-residual quantization ([SOL] item 1: quantize only the residual of K     */
/* inside each block; keep the block-mean term at bf16 precision).  Readings  */
/* where the page is silent: the blocks are the 64-token K blocks; the block  */
/* mean is the mean of the block's valid tokens (summed exactly), rounded to  */
/* bf16; the residual fp32(k) - fp32(mean) is coded as the other INT8 codes;  */
/* every score of row r against a key of block b gains                        */
/* e[r][b] = (q_r . mean_b) * fp32(sm_scale * log2 e), from the bf16 inputs   */
/* with fp32 accumulation.  No smoothing by the global mean in this mode.     */
/* ------------------------------------------------------------------------ */

/*
 * sage_quant_k_residual -- the residual codes of K: k_i8 [B,H,N_pad,d] int8
 * (padded rows 0), k_scale [B,H,N_pad/64] fp32, k_bmean [B,H,N_pad/64,d] bf16
 * bit patterns (blocks past N: 0), all device buffers (k_bmean 16-byte aligned).
 */
sage_status_t sage_quant_k_residual(const void *k_bf16, const int64_t k_stride[4],
                                    int B, int H, int N, int d,
                                    int8_t *k_i8, float *k_scale, uint16_t *k_bmean,
                                    sage_stream_t stream);

/* Bytes of scratch sage_attn_fwd_kres needs on the current device (0 for a
 * shape rejected, or when the device cannot be queried): the codes, the V
 * statistics, the bf16 block means and the attention kernel's per-SM scratch
 * slots for the mean term ([SMs][N_pad/64][256] fp32: 1 KiB per SM and
 * 64-token block, linear in N). */
size_t sage_attn_kres_workspace_bytes(int B, int H, int N, int d);

/*
 * sage_attn_fwd_kres -- the forward with K-residual quantization instead of
 * the smoothing: Q and V coded as in sage_attn_fwd, K as in
 * sage_quant_k_residual, and the fused attention kernel adding the mean term
 * to each score's exponent.  Each attention CTA computes the mean term of its
 * 256 query rows against every 64-token block first, on the tensor cores
 * (tcgen05 kind::f16: bf16 Q rows times bf16 block means, fp32 accumulation,
 * times fp32(sm_scale * log2 e)), and keeps it in the scratch slot of the SM
 * it runs on.  Arguments, layouts, events and errors as sage_attn_fwd_ev;
 * the workspace is sage_attn_kres_workspace_bytes for the device the call
 * runs on.
 */
sage_status_t sage_attn_fwd_kres(const void *q, const int64_t q_stride[4],
                                 const void *k, const int64_t k_stride[4],
                                 const void *v, const int64_t v_stride[4],
                                 void *out, const int64_t o_stride[4],
                                 int B, int H, int N, int d, float sm_scale,
                                 void *workspace, size_t workspace_bytes,
                                 sage_stream_t stream,
                                 sage_event_t attn_begin, sage_event_t attn_end);

/*
 * sage_attn_dense_ref_gpu -- plain dense attention on the CUDA cores in fp32
 * ([SDPA] section 三.1, [H3] section 一): no quantization, no tensor cores,
 * exact softmax with a running max (fp32 expf).  For A/B checks only.
 */
sage_status_t sage_attn_dense_ref_gpu(const void *q, const int64_t q_stride[4],
                                      const void *k, const int64_t k_stride[4],
                                      const void *v, const int64_t v_stride[4],
                                      void *out, const int64_t o_stride[4],
                                      int B, int H, int N, int d, float sm_scale,
                                      sage_stream_t stream);

/*
 * sage_debug_qk_tile -- export one int32 S tile (128 queries x 128 keys) of
 * slab (b,h): rows q_tile*128.., keys kv_tile*128.., computed by the same
 * TMA + tcgen05 kind::i8 path the attention kernel uses.  q_i8/k_i8 as
 * written by sage_quant_qk.  s_out: device int32 [128][128], row-major.
 * Entries for keys or queries beyond N_pad are what the zero padding gives (0).
 */
sage_status_t sage_debug_qk_tile(const int8_t *q_i8, const int8_t *k_i8,
                                 int B, int H, int N, int d,
                                 int b, int h, int q_tile, int kv_tile,
                                 int32_t *s_out, sage_stream_t stream);

/*
 * sage_debug_wait_timeout -- a probe of the failure path every kernel uses:
 * one warp waits, bounded to `microseconds` (1..1000000) of SM clocks, on a
 * barrier that nothing arrives on, gives up, records the timeout in the
 * device error word (bit 0 and bit 8 + site 0) and returns normally.  The
 * next sage_check on the stream reports SAGE_ERR_TIMEOUT and clears the word;
 * the context stays usable.  Nothing faults, traps or hangs.
 */
sage_status_t sage_debug_wait_timeout(int microseconds, sage_stream_t stream);

/*
 * sage_debug_ex2_probe -- a throughput probe of the exponential unit, for
 * stating the softmax's ceiling next to the attention kernel's time: `blocks`
 * CTAs of 256 threads, each thread running eight independent chains of
 * `iters` base-2 exponentials (the ex2.approx.ftz instruction the softmax
 * issues), i.e. blocks * 256 * iters * 8 exponentials; the caller times the
 * launch on `stream`.  sink: device float[blocks * 256] on the current device
 * (4-byte aligned), written with the chains' sums.  blocks 1..65535, iters
 * 1..2^20 (SAGE_ERR_INVALID_ARG otherwise).  Asynchronous; not part of any
 * forward.
 */
sage_status_t sage_debug_ex2_probe(float *sink, int blocks, int iters, sage_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_H_ */
