// sage_host.cu -- the forward on host memory.  The heads are cut into chunks
// that flow through host->device copies, the quantize and attention kernels
// and the device->host copy of their output on a few internal streams, so the
// copies of one chunk overlap the kernels of another (copies in both
// directions use their own copy engines).  Every chunk computes exactly what
// the whole call would for its heads: all statistics are per head.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>
#include <vector>

#include "sage.h"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr size_t kAlign = 1024;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

constexpr int kStreams = 3;  // internal streams (and chunk workspaces)
constexpr int kTailSplits = 2;  // the call's last chunk is cut into up to 3 halving pieces

// Heads per chunk: about 64 MiB of input per chunk, between 4 and 16 chunks
// per call (small chunks make the strided copies of a fused layout slow; few
// chunks leave the first copy and the last kernels unoverlapped).
int chunk_heads(int B, int H, int N, int d) {
    const double in_bytes = 6.0 * B * H * N * d;
    int chunks = static_cast<int>(in_bytes / (64.0 * 1024 * 1024)) + 1;
    chunks = chunks < 4 ? 4 : (chunks > 16 ? 16 : chunks);
    const int per_row = (chunks + B - 1) / B;  // chunks of each batch row
    return (H + per_row - 1) / per_row;
}

size_t chunk_ws_bytes(int hc, int N, int d) {
    const Shape cs{1, hc, N, d};
    return up(codes_bytes(cs)) + up(stats_ws_bytes(cs));
}

// kStreams non-blocking streams per device, created on first use and kept for
// the life of the process.
struct DeviceStreams {
    cudaStream_t s[kStreams] = {};
    bool ready = false;
};

cudaError_t device_streams(cudaStream_t (&out)[kStreams]) {
    static std::mutex mu;
    static DeviceStreams per_dev[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    DeviceStreams &ds = per_dev[dev];
    if (!ds.ready) {
        for (int i = 0; i < kStreams; ++i)
            if ((e = cudaStreamCreateWithFlags(&ds.s[i], cudaStreamNonBlocking)) != cudaSuccess) return e;
        ds.ready = true;
    }
    for (int i = 0; i < kStreams; ++i) out[i] = ds.s[i];
    return cudaSuccess;
}

// Events of one call, released when the call's work is enqueued (an event
// may be destroyed while work waiting on it is still pending).
struct Events {
    cudaEvent_t ev[1 + kStreams] = {};
    ~Events() {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
    }
};

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" {

size_t sage_attn_fwd_host_scratch_bytes(int B, int H, int N, int d) {
    if (!shape_supported(B, H, N, d)) return 0;
    const size_t elems = (size_t)B * H * N * d;
    return up(3 * elems * 2) + up(elems * 2) + kStreams * chunk_ws_bytes(chunk_heads(B, H, N, d), N, d);
}

sage_status_t sage_attn_fwd_host(const void *qkv_host, int layout, void *out_host, int B, int H, int N, int d,
                                 float sm_scale, void *scratch, size_t scratch_bytes, sage_stream_t stream) {
    if (!qkv_host || !out_host) {
        set_last_error("qkv_host and out_host must not be null");
        return SAGE_ERR_INVALID_ARG;
    }
    if (layout != SAGE_LAYOUT_FUSED && layout != SAGE_LAYOUT_CONTIGUOUS) {
        set_last_error("layout %d is neither SAGE_LAYOUT_FUSED nor SAGE_LAYOUT_CONTIGUOUS", layout);
        return SAGE_ERR_INVALID_ARG;
    }
    if (sage_status_t r = check_shape(B, H, N, d)) return r;
    if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) {
        set_last_error("sm_scale must be finite and positive");
        return SAGE_ERR_INVALID_ARG;
    }
    const size_t need = sage_attn_fwd_host_scratch_bytes(B, H, N, d);
    cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
    if (scratch && scratch_bytes < need) {
        set_last_error("scratch of %zu bytes is smaller than the %zu required", scratch_bytes, need);
        return SAGE_ERR_WORKSPACE;
    }
    if (scratch && reinterpret_cast<uintptr_t>(scratch) % 256) {
        set_last_error("scratch is not 256-byte aligned");
        return SAGE_ERR_INVALID_ARG;
    }
    auto cuda_fail = [](cudaError_t e, const char *what) {
        set_last_error("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
        return SAGE_ERR_CUDA;
    };
    cudaStream_t st[kStreams];
    cudaError_t e = device_streams(st);
    if (e != cudaSuccess) return cuda_fail(e, "internal streams");
    bool owned = false;
    if (!scratch) {
        if ((e = cudaMallocAsync(&scratch, need, user)) != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(scratch)");
        owned = true;
    }
    Events ev;
    bool forked = false;  // the internal streams wait on the caller's stream
    // Every return from here on goes through finish(): once the internal
    // streams took work, the caller's stream is made to wait for all of them
    // (also after an error, so that no copy into out_host or read of scratch
    // is still pending when the caller's stream moves on), and an owned
    // scratch is freed in stream order.  The first error is the one reported.
    auto finish = [&](sage_status_t status, cudaError_t err, const char *what) -> sage_status_t {
        if (status != SAGE_OK) cuda_fail(err, what);
        if (forked) {
            for (int i = 0; i < kStreams; ++i) {
                cudaError_t x = cudaEventRecord(ev.ev[1 + i], st[i]);
                if (x == cudaSuccess) x = cudaStreamWaitEvent(user, ev.ev[1 + i], 0);
                if (x != cudaSuccess && status == SAGE_OK) status = cuda_fail(x, "joining the internal streams");
            }
        }
        if (owned) {
            cudaError_t x = cudaFreeAsync(scratch, user);
            if (x != cudaSuccess && status == SAGE_OK) status = cuda_fail(x, "cudaFreeAsync(scratch)");
        }
        return status;
    };
    for (cudaEvent_t &x : ev.ev)
        if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess)
            return finish(SAGE_ERR_CUDA, e, "event");
    // the internal streams start after everything already on the caller's stream
    if ((e = cudaEventRecord(ev.ev[0], user)) != cudaSuccess) return finish(SAGE_ERR_CUDA, e, "cudaEventRecord");
    for (int i = 0; i < kStreams; ++i) {
        if ((e = cudaStreamWaitEvent(st[i], ev.ev[0], 0)) != cudaSuccess)
            return finish(SAGE_ERR_CUDA, e, "cudaStreamWaitEvent");
        forked = true;
    }

    const size_t elems = (size_t)B * H * N * d;
    char *base = static_cast<char *>(scratch);
    uint16_t *d_in = reinterpret_cast<uint16_t *>(base);
    uint16_t *d_out = reinterpret_cast<uint16_t *>(base + up(3 * elems * 2));
    const int hc_max = chunk_heads(B, H, N, d);
    char *ws0 = base + up(3 * elems * 2) + up(elems * 2);
    const size_t ws_step = chunk_ws_bytes(hc_max, N, d);
    const uint16_t *h_in = static_cast<const uint16_t *>(qkv_host);
    uint16_t *h_out = static_cast<uint16_t *>(out_host);
    const int64_t hd = (int64_t)H * d, nd = (int64_t)N * d;

    // the chunks: hc_max heads each, the last one of the call cut into
    // halving pieces (e.g. 6 heads -> 3, 2, 1), so that what cannot overlap
    // anything -- the last chunk's kernels and copy back -- is short
    struct Chunk { int b, h0, hc; };
    std::vector<Chunk> plan;
    for (int b = 0; b < B; ++b)
        for (int h0 = 0; h0 < H; h0 += hc_max) plan.push_back({b, h0, H - h0 < hc_max ? H - h0 : hc_max});
    {
        const Chunk last = plan.back();
        plan.pop_back();
        int h0 = last.h0, rem = last.hc;
        for (int i = 0; i < kTailSplits && rem > 1; ++i) {
            const int half = (rem + 1) / 2;
            plan.push_back({last.b, h0, half});
            h0 += half;
            rem -= half;
        }
        if (rem > 0) plan.push_back({last.b, h0, rem});
    }
    for (int c = 0; c < static_cast<int>(plan.size()); ++c) {
            const int b = plan[c].b, h0 = plan[c].h0, hc = plan[c].hc;
            cudaStream_t s = st[c % kStreams];
            char *ws = ws0 + (c % kStreams) * ws_step;
            const Shape cs{1, hc, N, d};
            Src q, k, v;
            if (layout == SAGE_LAYOUT_FUSED) {
                // [B,N,3,H,d]: each tensor's heads h0.. are a strided block of N rows
                const int64_t row = 3 * hd, boff = (int64_t)b * N * row;
                for (int x = 0; x < 3; ++x) {
                    const int64_t off = boff + x * hd + (int64_t)h0 * d;
                    e = cudaMemcpy2DAsync(d_in + off, row * 2, h_in + off, row * 2, (size_t)hc * d * 2, N,
                                          cudaMemcpyHostToDevice, s);
                    if (e != cudaSuccess) return finish(SAGE_ERR_CUDA, e, "host-to-device copy");
                }
                const uint16_t *p0 = d_in + boff + (int64_t)h0 * d;
                q = Src{p0, (int64_t)N * row, d, row};
                k = Src{p0 + hd, (int64_t)N * row, d, row};
                v = Src{p0 + 2 * hd, (int64_t)N * row, d, row};
            } else {
                // [3,B,H,N,d]: each tensor's heads h0.. of batch b are contiguous
                const int64_t off = ((int64_t)b * H + h0) * nd;
                for (int x = 0; x < 3; ++x) {
                    e = cudaMemcpyAsync(d_in + x * elems + off, h_in + x * elems + off, (size_t)hc * nd * 2,
                                        cudaMemcpyHostToDevice, s);
                    if (e != cudaSuccess) return finish(SAGE_ERR_CUDA, e, "host-to-device copy");
                }
                q = Src{d_in + off, (int64_t)H * nd, nd, d};
                k = Src{d_in + elems + off, (int64_t)H * nd, nd, d};
                v = Src{d_in + 2 * elems + off, (int64_t)H * nd, nd, d};
            }
            const int64_t ooff = ((int64_t)b * H + h0) * nd;
            const Dst o{d_out + ooff, (int64_t)H * nd, nd, d};
            const Codes codes = carve_codes(ws, cs);
            const StatsWs sw = carve_stats_ws(ws + up(codes_bytes(cs)), cs);
            if ((e = launch_qpass(cs, &q, &k, &v, sw, nullptr, codes, s)) != cudaSuccess)
                return finish(SAGE_ERR_CUDA, e, "quantize pass");
            if ((e = launch_attention(cs, codes, o, sm_scale, s)) != cudaSuccess)
                return finish(SAGE_ERR_CUDA, e, "attention kernel");
            if ((e = cudaMemcpyAsync(h_out + ooff, d_out + ooff, (size_t)hc * nd * 2, cudaMemcpyDeviceToHost, s)) !=
                cudaSuccess)
                return finish(SAGE_ERR_CUDA, e, "device-to-host copy");
        }
    // the caller's stream continues after all internal streams
    return finish(SAGE_OK, cudaSuccess, nullptr);
}

}  // extern "C"
