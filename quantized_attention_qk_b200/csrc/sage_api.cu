// sage_api.cu -- the extern "C" entry points declared in include/sage.h:
// argument validation (before any launch), scratch sizing and carving,
// stream-ordered launches, status codes and the per-thread error message.
// Unsupported inputs are rejected with an explicit status, never routed
// elsewhere (the "strict" behaviour the ComfyUI-sol-attn page describes in
// its 核心亮点 item 4).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "sage.h"
#include "sage_internal.h"

namespace sage {
namespace {

thread_local std::string g_last_error;

sage_status_t fail(sage_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

sage_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(SAGE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

constexpr size_t kAlign = 1024;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// bf16 tensor view: 16-byte aligned base, channel stride 1, other strides
// multiples of 8 elements (so every row starts on a 16-byte boundary).
sage_status_t check_view(const void *p, const int64_t *st, const char *name) {
    if (!p) return fail(SAGE_ERR_INVALID_ARG, "%s is null", name);
    if (!st) return fail(SAGE_ERR_INVALID_ARG, "%s strides are null", name);
    if (reinterpret_cast<uintptr_t>(p) % 16) return fail(SAGE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    if (st[3] != 1) return fail(SAGE_ERR_INVALID_ARG, "%s channel stride is %lld, must be 1", name, (long long)st[3]);
    for (int i = 0; i < 3; ++i)
        if (st[i] % 8 != 0)
            return fail(SAGE_ERR_INVALID_ARG, "%s stride[%d]=%lld is not a multiple of 8 elements", name, i,
                        (long long)st[i]);
    return SAGE_OK;
}

sage_status_t check_dev(const void *p, const char *name, size_t align = 16) {
    if (!p) return fail(SAGE_ERR_INVALID_ARG, "%s is null", name);
    if (reinterpret_cast<uintptr_t>(p) % align)
        return fail(SAGE_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
    return SAGE_OK;
}

Src src(const void *p, const int64_t *st) { return Src{static_cast<const uint16_t *>(p), st[0], st[1], st[2]}; }
Dst dst(void *p, const int64_t *st) { return Dst{static_cast<uint16_t *>(p), st[0], st[1], st[2]}; }

// Scratch obtained for one call: the caller's buffer or a stream-ordered allocation.
struct Scratch {
    void *ptr = nullptr;
    bool owned = false;
    cudaStream_t st = nullptr;
    ~Scratch() {
        if (owned && ptr) cudaFreeAsync(ptr, st);
    }
};

sage_status_t get_scratch(Scratch &s, void *ws, size_t ws_bytes, size_t need, cudaStream_t st) {
    s.st = st;
    if (ws) {
        if (ws_bytes < need)
            return fail(SAGE_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", ws_bytes, need);
        if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(SAGE_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
        s.ptr = ws;
        return SAGE_OK;
    }
    cudaError_t e = cudaMallocAsync(&s.ptr, need, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
    s.owned = true;
    return SAGE_OK;
}

}  // namespace

constexpr int64_t kMaxHeads = 65535;   // B*H: the attention grid's second dimension
constexpr int kMaxTokens = 1 << 24;

sage_status_t check_shape(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1) return fail(SAGE_ERR_INVALID_ARG, "shape B=%d H=%d N=%d must be positive", B, H, N);
    if (d != 64 && d != 128) return fail(SAGE_ERR_UNSUPPORTED, "head dim d=%d is not supported (64 or 128)", d);
    if ((int64_t)B * H > kMaxHeads) return fail(SAGE_ERR_UNSUPPORTED, "B*H=%lld exceeds 65535", (long long)B * H);
    if (N > kMaxTokens) return fail(SAGE_ERR_UNSUPPORTED, "N=%d exceeds 2^24 tokens", N);
    return SAGE_OK;
}

bool shape_supported(int B, int H, int N, int d) {
    return B >= 1 && H >= 1 && N >= 1 && (d == 64 || d == 128) && (int64_t)B * H <= kMaxHeads && N <= kMaxTokens;
}

sage_status_t check_on_current_device(const void *p, const char *name) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaPointerAttributes a{};
    if ((e = cudaPointerGetAttributes(&a, p)) != cudaSuccess) {
        cudaGetLastError();  // the query's error is not sticky; clear it
        return fail(SAGE_ERR_INVALID_ARG, "%s: %s", name, cudaGetErrorString(e));
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
        return fail(SAGE_ERR_INVALID_ARG, "%s is not device memory", name);
    if (a.device != dev)
        return fail(SAGE_ERR_INVALID_ARG, "%s is on device %d but device %d is current", name, a.device, dev);
    return SAGE_OK;
}

void set_last_error(const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
}

// Statistics scratch: per slot the fp64 K column sums, the fp32 V column
// maxima and a 64-bit flag.
size_t stats_ws_bytes(const Shape &s) {
    const size_t slots = static_cast<size_t>(s.stats_slots());
    return up(slots * s.d * sizeof(double)) + up(slots * s.d * sizeof(float)) + up(slots * 8);
}

StatsWs carve_stats_ws(void *base, const Shape &s) {
    char *p = static_cast<char *>(base);
    const size_t slots = static_cast<size_t>(s.stats_slots());
    const size_t kpart = up(slots * s.d * sizeof(double)), vpart = up(slots * s.d * sizeof(float));
    StatsWs w;
    w.ksum_part = reinterpret_cast<double *>(p);
    w.vmax_part = reinterpret_cast<float *>(p + kpart);
    w.flags = reinterpret_cast<unsigned long long *>(p + kpart + vpart);
    return w;
}

size_t codes_bytes(const Shape &s) {
    const size_t codes = up((size_t)s.BH() * s.n_pad() * s.d);
    return 3 * codes + up((size_t)s.BH() * s.n_qblocks() * 4) + up((size_t)s.BH() * s.n_kblocks() * 4) +
           up((size_t)s.BH() * s.d * 4);
}

Codes carve_codes(void *base, const Shape &s) {
    char *p = static_cast<char *>(base);
    const size_t codes = up((size_t)s.BH() * s.n_pad() * s.d);
    Codes c;
    c.q_i8 = reinterpret_cast<int8_t *>(p);
    c.k_i8 = reinterpret_cast<int8_t *>(p + codes);
    c.v_e4m3 = reinterpret_cast<uint8_t *>(p + 2 * codes);
    p += 3 * codes;
    c.q_scale = reinterpret_cast<float *>(p);
    p += up((size_t)s.BH() * s.n_qblocks() * 4);
    c.k_scale = reinterpret_cast<float *>(p);
    p += up((size_t)s.BH() * s.n_kblocks() * 4);
    c.v_scale = reinterpret_cast<float *>(p);
    return c;
}

}  // namespace sage

using namespace sage;

extern "C" {

const char *sage_status_string(sage_status_t status) {
    switch (status) {
        case SAGE_OK: return "SAGE_OK";
        case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
        case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
        case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
        case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
        case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    }
    return "SAGE_ERR_UNKNOWN";
}

const char *sage_last_error_message(void) { return g_last_error.c_str(); }

sage_status_t sage_check(sage_stream_t stream) {
    unsigned v = 0;
    cudaError_t e = read_and_clear_device_error(&v, stream);
    if (e != cudaSuccess) return cuda_fail(e, "sage_check");
    if (v & kErrTimeoutBit)
        return fail(SAGE_ERR_TIMEOUT, "a kernel gave up on a bounded wait (error word 0x%x: bit 8+k marks wait site k)",
                    v);
    return SAGE_OK;
}

size_t sage_quant_workspace_bytes(int B, int H, int N, int d) {
    if (!shape_supported(B, H, N, d)) return 0;
    return stats_ws_bytes(Shape{B, H, N, d});
}

size_t sage_attn_workspace_bytes(int B, int H, int N, int d) {
    if (!shape_supported(B, H, N, d)) return 0;
    const Shape s{B, H, N, d};
    return up(codes_bytes(s)) + stats_ws_bytes(s);
}

sage_status_t sage_quant_qk(const void *q_bf16, const int64_t q_stride[4], const void *k_bf16,
                            const int64_t k_stride[4], int B, int H, int N, int d, int8_t *q_i8, float *q_scale,
                            int8_t *k_i8, float *k_scale, float *k_mean, void *workspace, size_t workspace_bytes,
                            sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_view(q_bf16, q_stride, "q")) ||
        (r = check_view(k_bf16, k_stride, "k")) || (r = check_dev(q_i8, "q_i8", 16)) ||
        (r = check_dev(k_i8, "k_i8", 16)) || (r = check_dev(q_scale, "q_scale", 4)) ||
        (r = check_dev(k_scale, "k_scale", 4)) || (r = check_on_current_device(q_bf16, "q")) ||
        (r = check_on_current_device(q_i8, "q_i8")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Scratch scr;
    if ((r = get_scratch(scr, workspace, workspace_bytes, stats_ws_bytes(s), st))) return r;
    const StatsWs ws = carve_stats_ws(scr.ptr, s);
    const Src qs = src(q_bf16, q_stride), ks = src(k_bf16, k_stride);
    Codes c{};
    c.q_i8 = q_i8;
    c.q_scale = q_scale;
    c.k_i8 = k_i8;
    c.k_scale = k_scale;
    cudaError_t e = launch_qpass(s, &qs, &ks, nullptr, ws, k_mean, c, st);
    if (e != cudaSuccess) return cuda_fail(e, "quantize pass");
    return SAGE_OK;
}

sage_status_t sage_quant_v(const void *v_bf16, const int64_t v_stride[4], int B, int H, int N, int d,
                           uint8_t *v_e4m3, float *v_scale, void *workspace, size_t workspace_bytes,
                           sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_view(v_bf16, v_stride, "v")) ||
        (r = check_dev(v_e4m3, "v_e4m3", 16)) || (r = check_dev(v_scale, "v_scale", 4)) ||
        (r = check_on_current_device(v_bf16, "v")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Scratch scr;
    if ((r = get_scratch(scr, workspace, workspace_bytes, stats_ws_bytes(s), st))) return r;
    const StatsWs ws = carve_stats_ws(scr.ptr, s);
    const Src vs = src(v_bf16, v_stride);
    Codes c{};
    c.v_e4m3 = v_e4m3;
    c.v_scale = v_scale;
    cudaError_t e = launch_qpass(s, nullptr, nullptr, &vs, ws, nullptr, c, st);
    if (e != cudaSuccess) return cuda_fail(e, "quantize pass");
    return SAGE_OK;
}

static sage_status_t check_scale(float sm_scale) {
    if (!std::isfinite(sm_scale) || !(sm_scale > 0.f))
        return fail(SAGE_ERR_INVALID_ARG, "sm_scale=%g must be finite and > 0", (double)sm_scale);
    return SAGE_OK;
}

sage_status_t sage_attn_quantized(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8, const float *k_scale,
                                  const uint8_t *v_e4m3, const float *v_scale, void *out, const int64_t o_stride[4],
                                  int B, int H, int N, int d, float sm_scale, sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_dev(q_i8, "q_i8", 16)) ||
        (r = check_dev(k_i8, "k_i8", 16)) || (r = check_dev(v_e4m3, "v_e4m3", 16)) ||
        (r = check_dev(q_scale, "q_scale", 4)) || (r = check_dev(k_scale, "k_scale", 4)) ||
        (r = check_dev(v_scale, "v_scale", 4)) || (r = check_view(out, o_stride, "out")) ||
        (r = check_on_current_device(q_i8, "q_i8")) || (r = check_on_current_device(out, "out")))
        return r;
    const Shape s{B, H, N, d};
    Codes c;
    c.q_i8 = const_cast<int8_t *>(q_i8);
    c.q_scale = const_cast<float *>(q_scale);
    c.k_i8 = const_cast<int8_t *>(k_i8);
    c.k_scale = const_cast<float *>(k_scale);
    c.v_e4m3 = const_cast<uint8_t *>(v_e4m3);
    c.v_scale = const_cast<float *>(v_scale);
    cudaError_t e = launch_attention(s, c, dst(out, o_stride), sm_scale, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
    return SAGE_OK;
}

sage_status_t sage_attn_fwd_ev(const void *q, const int64_t q_stride[4], const void *k, const int64_t k_stride[4],
                               const void *v, const int64_t v_stride[4], void *out, const int64_t o_stride[4], int B,
                               int H, int N, int d, float sm_scale, void *workspace, size_t workspace_bytes,
                               sage_stream_t stream, sage_event_t attn_begin, sage_event_t attn_end) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_view(q, q_stride, "q")) ||
        (r = check_view(k, k_stride, "k")) || (r = check_view(v, v_stride, "v")) ||
        (r = check_view(out, o_stride, "out")) || (r = check_on_current_device(q, "q")) ||
        (r = check_on_current_device(out, "out")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Scratch scr;
    const size_t cb = up(codes_bytes(s));
    if ((r = get_scratch(scr, workspace, workspace_bytes, cb + stats_ws_bytes(s), st))) return r;
    const Codes c = carve_codes(scr.ptr, s);
    const StatsWs ws = carve_stats_ws(static_cast<char *>(scr.ptr) + cb, s);
    const Src qs = src(q, q_stride), ks = src(k, k_stride), vs = src(v, v_stride);
    cudaError_t e = launch_qpass(s, &qs, &ks, &vs, ws, nullptr, c, st);
    if (e != cudaSuccess) return cuda_fail(e, "quantize pass");
    if (attn_begin && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_begin), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_attention(s, c, dst(out, o_stride), sm_scale, st)) != cudaSuccess)
        return cuda_fail(e, "attention kernel");
    if (attn_end && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_end), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    return SAGE_OK;
}

sage_status_t sage_attn_fwd(const void *q, const int64_t q_stride[4], const void *k, const int64_t k_stride[4],
                            const void *v, const int64_t v_stride[4], void *out, const int64_t o_stride[4], int B,
                            int H, int N, int d, float sm_scale, void *workspace, size_t workspace_bytes,
                            sage_stream_t stream) {
    return sage_attn_fwd_ev(q, q_stride, k, k_stride, v, v_stride, out, o_stride, B, H, N, d, sm_scale, workspace,
                            workspace_bytes, stream, nullptr, nullptr);
}

static sage_status_t check_sparse_shape(int B, int H, int N, int d) {
    sage_status_t r = check_shape(B, H, N, d);
    if (r) return r;
    const Shape s{B, H, N, d};
    if (s.n_tiles() > kMaxSelectTiles)
        return fail(SAGE_ERR_UNSUPPORTED, "block-sparse calls take at most %d tiles of 128 tokens (N=%d gives %d)",
                    kMaxSelectTiles, N, s.n_tiles());
    return SAGE_OK;
}

static sage_status_t check_tau(float tau) {
    if (!std::isfinite(tau) || !(tau > 0.f))
        return fail(SAGE_ERR_INVALID_ARG, "tau=%g must be finite and > 0", (double)tau);
    return SAGE_OK;
}

size_t sage_block_mask_bytes(int B, int H, int N) {
    if (!shape_supported(B, H, N, 128)) return 0;
    const Shape s{B, H, N, 128};
    if (s.n_tiles() > kMaxSelectTiles) return 0;
    return mask_bytes(s);
}

size_t sage_block_select_workspace_bytes(int B, int H, int N, int d) {
    if (!shape_supported(B, H, N, d)) return 0;
    const Shape s{B, H, N, d};
    if (s.n_tiles() > kMaxSelectTiles) return 0;
    return select_ws_bytes(s);
}

sage_status_t sage_block_select(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8, const float *k_scale,
                                int B, int H, int N, int d, float sm_scale, float tau, uint32_t *mask, float *scores,
                                void *workspace, size_t workspace_bytes, sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_sparse_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_tau(tau)) ||
        (r = check_dev(q_i8, "q_i8", 16)) || (r = check_dev(k_i8, "k_i8", 16)) ||
        (r = check_dev(q_scale, "q_scale", 4)) || (r = check_dev(k_scale, "k_scale", 4)) ||
        (r = check_dev(mask, "mask", 4)) || (scores && (r = check_dev(scores, "scores", 4))) ||
        (r = check_on_current_device(q_i8, "q_i8")) || (r = check_on_current_device(mask, "mask")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Scratch scr;
    if ((r = get_scratch(scr, workspace, workspace_bytes, select_ws_bytes(s), st))) return r;
    cudaError_t e = launch_select(s, q_i8, q_scale, k_i8, k_scale, sm_scale, tau, scr.ptr, mask, scores, st);
    if (e != cudaSuccess) return cuda_fail(e, "block selection");
    return SAGE_OK;
}

size_t sage_attn_sparse_workspace_bytes(int B, int H, int N, int d) {
    if (!shape_supported(B, H, N, d)) return 0;
    const Shape s{B, H, N, d};
    if (s.n_tiles() > kMaxSelectTiles) return 0;
    return up(codes_bytes(s)) + up(stats_ws_bytes(s)) + up(select_ws_bytes(s)) + up(mask_bytes(s));
}

sage_status_t sage_attn_fwd_sparse(const void *q, const int64_t q_stride[4], const void *k, const int64_t k_stride[4],
                                   const void *v, const int64_t v_stride[4], void *out, const int64_t o_stride[4],
                                   int B, int H, int N, int d, float sm_scale, float tau, const uint32_t *mask_in,
                                   uint32_t *mask_out, void *workspace, size_t workspace_bytes, sage_stream_t stream,
                                   sage_event_t attn_begin, sage_event_t attn_end) {
    sage_status_t r;
    if ((r = check_sparse_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_view(q, q_stride, "q")) ||
        (r = check_view(k, k_stride, "k")) || (r = check_view(v, v_stride, "v")) ||
        (r = check_view(out, o_stride, "out")) || (!mask_in && (r = check_tau(tau))) ||
        (mask_in && (r = check_dev(mask_in, "mask_in", 4))) || (mask_out && (r = check_dev(mask_out, "mask_out", 4))) ||
        (r = check_on_current_device(q, "q")) || (r = check_on_current_device(out, "out")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Scratch scr;
    const size_t cb = up(codes_bytes(s)), sb = up(stats_ws_bytes(s)), selb = up(select_ws_bytes(s));
    if ((r = get_scratch(scr, workspace, workspace_bytes, cb + sb + selb + up(mask_bytes(s)), st))) return r;
    char *base = static_cast<char *>(scr.ptr);
    const Codes c = carve_codes(base, s);
    const StatsWs ws = carve_stats_ws(base + cb, s);
    const Src qs = src(q, q_stride), ks = src(k, k_stride), vs = src(v, v_stride);
    // tau >= 1 keeps every key tile (reading S3): the dense kernel computes the
    // same result bit for bit without walking step lists
    const bool dense = !mask_in && tau >= 1.f;
    const bool select = !mask_in && (!dense || mask_out);
    // with a selection to run, the quantize pass also pools the tiles' codes
    float *pool_qv = nullptr, *pool_kvT = nullptr;
    if (select) select_pool_ptrs(base + cb + sb, s, &pool_qv, &pool_kvT);
    cudaError_t e = launch_qpass(s, &qs, &ks, &vs, ws, nullptr, c, st, nullptr, pool_qv, pool_kvT);
    if (e != cudaSuccess) return cuda_fail(e, "quantize pass");
    const uint32_t *mask = mask_in;
    if (select) {
        uint32_t *m = mask_out ? mask_out : reinterpret_cast<uint32_t *>(base + cb + sb + selb);
        if ((e = launch_select(s, c.q_i8, c.q_scale, c.k_i8, c.k_scale, sm_scale, tau, base + cb + sb, m, nullptr,
                               st, true)) != cudaSuccess)
            return cuda_fail(e, "block selection");
        mask = m;
    } else if (mask_out) {
        if ((e = cudaMemcpyAsync(mask_out, mask_in, mask_bytes(s), cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
            return cuda_fail(e, "mask copy");
    }
    if (attn_begin && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_begin), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    e = dense ? launch_attention(s, c, dst(out, o_stride), sm_scale, st)
              : launch_attention_sparse(s, c, dst(out, o_stride), sm_scale, mask, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel");
    if (attn_end && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_end), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    return SAGE_OK;
}

sage_status_t sage_attn_fwd_fused_q(const void *q, const int64_t q_stride[4], const void *k,
                                   const int64_t k_stride[4], const void *v, const int64_t v_stride[4], void *out,
                                   const int64_t o_stride[4], int B, int H, int N, int d, float sm_scale,
                                   void *workspace, size_t workspace_bytes, sage_stream_t stream,
                                   sage_event_t attn_begin, sage_event_t attn_end) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_view(q, q_stride, "q")) ||
        (r = check_view(k, k_stride, "k")) || (r = check_view(v, v_stride, "v")) ||
        (r = check_view(out, o_stride, "out")) || (r = check_on_current_device(q, "q")) ||
        (r = check_on_current_device(out, "out")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    Scratch scr;
    const size_t cb = up(codes_bytes(s));
    if ((r = get_scratch(scr, workspace, workspace_bytes, cb + stats_ws_bytes(s), st))) return r;
    const Codes c = carve_codes(scr.ptr, s);
    const StatsWs ws = carve_stats_ws(static_cast<char *>(scr.ptr) + cb, s);
    const Src qs = src(q, q_stride), ks = src(k, k_stride), vs = src(v, v_stride);
    cudaError_t e = launch_qpass(s, nullptr, &ks, &vs, ws, nullptr, c, st);
    if (e != cudaSuccess) return cuda_fail(e, "quantize pass");
    if (attn_begin && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_begin), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_attention_fused_q(s, c, qs, dst(out, o_stride), sm_scale, st)) != cudaSuccess)
        return cuda_fail(e, "attention kernel");
    if (attn_end && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_end), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    return SAGE_OK;
}

static size_t kres_bmean_bytes(const Shape &s) { return up((size_t)s.BH() * s.n_kblocks() * s.d * 2); }
// per-SM scratch slots of the attention kernel's mean term: [SMs][nkb][256] fp32
static size_t kres_slot_bytes(const Shape &s) { return up((size_t)kres_slots() * s.n_kblocks() * 256 * 4); }

size_t sage_attn_kres_workspace_bytes(int B, int H, int N, int d) {
    if (!shape_supported(B, H, N, d)) return 0;
    const Shape s{B, H, N, d};
    if (kres_slots() <= 0) return 0;
    return up(codes_bytes(s)) + up(stats_ws_bytes(s)) + kres_bmean_bytes(s) + kres_slot_bytes(s);
}

sage_status_t sage_quant_k_residual(const void *k_bf16, const int64_t k_stride[4], int B, int H, int N, int d,
                                    int8_t *k_i8, float *k_scale, uint16_t *k_bmean, sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_view(k_bf16, k_stride, "k")) ||
        (r = check_dev(k_i8, "k_i8", 16)) || (r = check_dev(k_scale, "k_scale", 4)) ||
        (r = check_dev(k_bmean, "k_bmean", 16)) || (r = check_on_current_device(k_bf16, "k")) ||
        (r = check_on_current_device(k_i8, "k_i8")))
        return r;
    const Shape s{B, H, N, d};
    // K alone needs no statistics (each block's mean is its own), so no scratch
    const Src ks = src(k_bf16, k_stride);
    const StatsWs none{};
    Codes c{};
    c.k_i8 = k_i8;
    c.k_scale = k_scale;
    cudaError_t e = launch_qpass(s, nullptr, &ks, nullptr, none, nullptr, c, reinterpret_cast<cudaStream_t>(stream),
                                 k_bmean);
    if (e != cudaSuccess) return cuda_fail(e, "K-residual quantization");
    return SAGE_OK;
}

sage_status_t sage_attn_fwd_kres(const void *q, const int64_t q_stride[4], const void *k, const int64_t k_stride[4],
                                 const void *v, const int64_t v_stride[4], void *out, const int64_t o_stride[4], int B,
                                 int H, int N, int d, float sm_scale, void *workspace, size_t workspace_bytes,
                                 sage_stream_t stream, sage_event_t attn_begin, sage_event_t attn_end) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_view(q, q_stride, "q")) ||
        (r = check_view(k, k_stride, "k")) || (r = check_view(v, v_stride, "v")) ||
        (r = check_view(out, o_stride, "out")) || (r = check_on_current_device(q, "q")) ||
        (r = check_on_current_device(out, "out")))
        return r;
    const Shape s{B, H, N, d};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int n_slots = kres_slots();
    if (n_slots <= 0) return fail(SAGE_ERR_CUDA, "could not read the device's SM count");
    Scratch scr;
    const size_t cb = up(codes_bytes(s)), sb = up(stats_ws_bytes(s)), mb = kres_bmean_bytes(s);
    if ((r = get_scratch(scr, workspace, workspace_bytes, cb + sb + mb + kres_slot_bytes(s), st))) return r;
    char *base = static_cast<char *>(scr.ptr);
    const Codes c = carve_codes(base, s);
    const StatsWs ws = carve_stats_ws(base + cb, s);
    uint16_t *bmean = reinterpret_cast<uint16_t *>(base + cb + sb);
    float *eslot = reinterpret_cast<float *>(base + cb + sb + mb);
    const Src qs = src(q, q_stride), ks = src(k, k_stride), vs = src(v, v_stride);
    cudaError_t e = launch_qpass(s, &qs, &ks, &vs, ws, nullptr, c, st, bmean);
    if (e != cudaSuccess) return cuda_fail(e, "quantize pass (K-residual mode)");
    if (attn_begin && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_begin), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_attention_kres(s, c, qs, bmean, dst(out, o_stride), sm_scale, eslot, n_slots, st)) != cudaSuccess)
        return cuda_fail(e, "attention kernel");
    if (attn_end && (e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(attn_end), st)) != cudaSuccess)
        return cuda_fail(e, "cudaEventRecord");
    return SAGE_OK;
}

sage_status_t sage_attn_dense_ref_gpu(const void *q, const int64_t q_stride[4], const void *k,
                                      const int64_t k_stride[4], const void *v, const int64_t v_stride[4], void *out,
                                      const int64_t o_stride[4], int B, int H, int N, int d, float sm_scale,
                                      sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_scale(sm_scale)) || (r = check_view(q, q_stride, "q")) ||
        (r = check_view(k, k_stride, "k")) || (r = check_view(v, v_stride, "v")) ||
        (r = check_view(out, o_stride, "out")) || (r = check_on_current_device(q, "q")) ||
        (r = check_on_current_device(out, "out")))
        return r;
    const Shape s{B, H, N, d};
    cudaError_t e = launch_dense_ref(s, src(q, q_stride), src(k, k_stride), src(v, v_stride), dst(out, o_stride),
                                     sm_scale, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dense reference kernel");
    return SAGE_OK;
}

sage_status_t sage_debug_qk_tile(const int8_t *q_i8, const int8_t *k_i8, int B, int H, int N, int d, int b, int h,
                                 int q_tile, int kv_tile, int32_t *s_out, sage_stream_t stream) {
    sage_status_t r;
    if ((r = check_shape(B, H, N, d)) || (r = check_dev(q_i8, "q_i8", 16)) || (r = check_dev(k_i8, "k_i8", 16)) ||
        (r = check_dev(s_out, "s_out", 16)))
        return r;
    const Shape s{B, H, N, d};
    if (b < 0 || b >= B || h < 0 || h >= H || q_tile < 0 || q_tile >= s.n_qblocks() || kv_tile < 0 ||
        kv_tile >= s.n_qblocks())
        return fail(SAGE_ERR_INVALID_ARG, "tile (b=%d h=%d q_tile=%d kv_tile=%d) outside the tensor", b, h, q_tile,
                    kv_tile);
    if ((r = check_on_current_device(q_i8, "q_i8")) || (r = check_on_current_device(s_out, "s_out"))) return r;
    cudaError_t e = launch_debug_qk_tile(s, q_i8, k_i8, b * H + h, q_tile, kv_tile, s_out,
                                         reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "debug S tile");
    return SAGE_OK;
}

}  // extern "C"
