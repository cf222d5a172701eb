// sage_internal.h -- host-side plumbing shared by the library's translation
// units (not installed; the public interface is include/sage.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

#include "sage.h"

namespace sage {

constexpr int kQBlock = 128;       // Q tokens per quantization block == attention query tile
constexpr int kKBlock = 64;        // K tokens per quantization block
constexpr int kKvTile = 128;       // keys per attention KV tile (two K blocks)
constexpr int kStatsMaxGrid = 512;  // quantize pass: at most this many CTAs (bounds its statistics slots)
constexpr unsigned kErrTimeoutBit = 1u;  // device error word: a bounded wait gave up
constexpr int kMaxSelectTiles = 4096;    // block-sparse selection: key tiles one row ranks in shared memory

// A bf16 [B,H,N,d] tensor given by base pointer and element strides (c stride 1).
struct Src {
    const uint16_t *p;
    int64_t sb, sh, sn;
};
struct Dst {
    uint16_t *p;
    int64_t sb, sh, sn;
};

struct Shape {
    int B, H, N, d;
    int BH() const { return B * H; }
    int n_pad() const { return ((N + kQBlock - 1) / kQBlock) * kQBlock; }
    int n_qblocks() const { return n_pad() / kQBlock; }
    int n_kblocks() const { return n_pad() / kKBlock; }
    // Quantize pass: one statistics partial per (CTA, head) it covers, kept in
    // slot CTA + head: at most BH + min(kStatsMaxGrid, 128-token blocks) slots.
    long long stats_slots() const {
        const long long blocks = (long long)BH() * n_qblocks();
        return BH() + (blocks < kStatsMaxGrid ? blocks : kStatsMaxGrid);
    }
    // Block-sparse masks: one row of mask_words() 32-bit words per (b,h, query
    // tile), bit j = key tile j (tiles of kKvTile tokens for both).
    int n_tiles() const { return (N + kKvTile - 1) / kKvTile; }
    int mask_words() const { return (n_tiles() + 31) / 32; }
};

// Scratch of the quantize pass: the statistics partials and their flags.
// The K column sums are fp64: a sum of bf16 values is exact there whenever the
// column's values span fewer than 53 bits (every workload here), so the mean
// does not depend on the order of the additions.
struct StatsWs {
    double *ksum_part;          // [slots][d]
    float *vmax_part;           // [slots][d]
    unsigned long long *flags;  // [slots]
};

// Codes and scales consumed by the attention kernel.
struct Codes {
    int8_t *q_i8;      // [BH][N_pad][d]
    float *q_scale;    // [BH][N_pad/128]
    int8_t *k_i8;      // [BH][N_pad][d]
    float *k_scale;    // [BH][N_pad/64]
    uint8_t *v_e4m3;   // [BH][N_pad][d]  e4m3 bits, token-major like the int8 codes
    float *v_scale;    // [BH][d]
};

// Record the calling thread's error message (what sage_last_error_message returns).
void set_last_error(const char *fmt, ...);

// Argument checks shared by the entry points (each records the message):
// the shape limits every kernel assumes, and that `p` is device memory of the
// current device (kernels launch on the current device; a pointer of another
// device would be read across the interconnect or fault).
sage_status_t check_shape(int B, int H, int N, int d);
// The shapes check_shape accepts, without recording an error (for the size
// queries, which answer 0 for every other shape).
bool shape_supported(int B, int H, int N, int d);
sage_status_t check_on_current_device(const void *p, const char *name);

size_t stats_ws_bytes(const Shape &s);
StatsWs carve_stats_ws(void *base, const Shape &s);
size_t codes_bytes(const Shape &s);
Codes carve_codes(void *base, const Shape &s);

// The quantize pass (sage_quant.cu) in one cooperatively launched kernel:
// statistics of k and/or v, then the codes of the tensors given (null ones are
// skipped; the combinations q+k+v, q+k, k+v, v and q+v).  `user_k_mean` may be
// null; the V scales go to c.v_scale.  With `k_bmean` (bf16 [BH][N_pad/64][d])
// K is coded in K-residual mode instead (combinations q+k+v and k only): the
// residual of each 64-token block's mean, whose bf16 value goes to k_bmean.
// With pool_qv / pool_kvT (q+k+v, smoothing) it also writes the pooled tile
// vectors of the block selection (select_pool_ptrs), so that launch_select
// can skip its pooling kernel.
cudaError_t launch_qpass(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                         float *user_k_mean, const Codes &c, cudaStream_t st, uint16_t *k_bmean = nullptr,
                         float *pool_qv = nullptr, float *pool_kvT = nullptr);
// 4-D tiled TMA map of a bf16 [B,H,N,d] view: box = 64 channels x `rows` tokens
// of one (b,h).  The N and H dimensions are handed to the hardware in stride
// order; *hn_swapped tells the kernel which coordinate comes second.
cudaError_t make_bf16_token_map(CUtensorMap *m, const Src &src, const Shape &s, uint32_t rows, int *hn_swapped,
                                bool swizzle128 = false);
// 3-D tiled TMA map of a contiguous bf16 [d2][d1][d0] array: box 64 x rows x 1,
// 128-byte swizzle, zeros outside the array.
cudaError_t make_bf16_map3(CUtensorMap *m, const uint16_t *base, uint64_t d0, uint64_t d1, uint64_t d2,
                           uint32_t rows);
// Device error word (bounded waits that gave up) of the current device.
unsigned *device_error_ptr();

// Launch `kern` with programmatic stream serialization: its CTAs may start
// while the previous kernel of `st` is still running (once every CTA of that
// kernel has signalled griddepcontrol.launch_dependents or exited).  The kernel
// executes griddepcontrol.wait before it reads or writes anything an earlier
// kernel of the stream writes or reads; the first kernel of a forward is
// launched the plain way, so each forward starts after the previous one ended.
template <typename... P, typename... A>
cudaError_t launch_dependent(void (*kern)(P...), dim3 grid, dim3 block, int smem, cudaStream_t st, A &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// Attention launchers (sage_attn.cu).
cudaError_t launch_attention(const Shape &s, const Codes &c, const Dst &out, float sm_scale, cudaStream_t st);
cudaError_t launch_attention_sparse(const Shape &s, const Codes &c, const Dst &out, float sm_scale,
                                    const uint32_t *kv_mask, cudaStream_t st);
// Q quantized in the attention kernel's prologue from the bf16 view q_bf16
// (c.q_i8 / c.q_scale are not used).
cudaError_t launch_attention_fused_q(const Shape &s, const Codes &c, const Src &q_bf16, const Dst &out,
                                     float sm_scale, cudaStream_t st);
// K-residual mode: the attention kernel that computes the mean term
// (q . mean_b) in its prologue on the tensor cores from the bf16 Q rows and
// the block means, keeping it in per-SM scratch slots of kres_slots() x nkb x
// 256 floats (sage_attn.cu).  kres_slots() is the current device's SM count
// (0 on error).  The residual codes and block means come from launch_qpass.
int kres_slots();
cudaError_t launch_attention_kres(const Shape &s, const Codes &c, const Src &q_bf16, const uint16_t *k_bmean,
                                  const Dst &out, float sm_scale, float *eslot, int n_slots, cudaStream_t st);
cudaError_t launch_debug_qk_tile(const Shape &s, const int8_t *q_i8, const int8_t *k_i8, int bh, int q_tile,
                                 int kv_tile, int32_t *s_out, cudaStream_t st);
cudaError_t read_and_clear_device_error(unsigned *value, cudaStream_t st);

// Block-sparse selection (sage_sparse.cu): scratch for the pooled tile
// vectors, the mask size, and the launcher (pooling, scores, ranking, kept
// prefix).  select_pool_ptrs gives the pooled vectors' places in that
// scratch; with `pooled` the launcher takes them as already written there
// (by the quantize pass) and skips its pooling kernel.
size_t select_ws_bytes(const Shape &s);
size_t mask_bytes(const Shape &s);
void select_pool_ptrs(void *ws, const Shape &s, float **qv, float **kvT);
cudaError_t launch_select(const Shape &s, const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                          const float *k_scale, float sm_scale, float tau, void *ws, uint32_t *mask, float *sbar_out,
                          cudaStream_t st, bool pooled = false);

// Dense fp32 reference (sage_dense_ref.cu).
cudaError_t launch_dense_ref(const Shape &s, const Src &q, const Src &k, const Src &v, const Dst &out,
                             float sm_scale, cudaStream_t st);

}  // namespace sage
