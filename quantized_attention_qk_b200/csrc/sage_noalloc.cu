// sage_noalloc.cu -- sage_quant_qk_noalloc: the smoothing + Q/K quantization
// pass for callers that may not allocate device memory while they run (an
// engine or server plugin whose device memory is budgeted up front and whose
// execution path forbids cudaMalloc / cudaMallocAsync, or code whose allocator
// belongs to a host framework).  The pass needs scratch for its per-chunk
// statistics; here that scratch is a fixed array in the library's own device
// memory instead of a caller buffer or a stream-ordered allocation.
//
// The array is loaded with the module, so every GPU that loads the library
// holds it (kNoAllocScratchBytes) until the process exits.  All calls on one
// device share it: calls that overlap on the GPU (e.g. on two streams without
// ordering between them) race on it and must be serialized by the caller.
// It keeps the last call's contents; every entry a call reads is written
// earlier in the same call, so nothing has to start at zero.  Its device
// address is looked up once per device and kept: a process that calls
// cudaDeviceReset and goes on using the library is not supported.
#include <cuda_runtime.h>

#include <mutex>

#include "sage.h"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr size_t kNoAllocScratchBytes = SAGE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current).  Host code cannot use the symbol
// itself: on the host it only names a stand-in, not device memory.
cudaError_t scratch_for_current_device(void **out) {
    static std::mutex mu;
    static void *ptrs[kMaxDevices] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace sage

extern "C" sage_status_t sage_quant_qk_noalloc(const void *q_bf16, const int64_t q_stride[4], const void *k_bf16,
                                               const int64_t k_stride[4], int B, int H, int N, int d, int8_t *q_i8,
                                               float *q_scale, int8_t *k_i8, float *k_scale, float *k_mean,
                                               sage_stream_t stream) {
    using namespace sage;
    sage_status_t r = check_shape(B, H, N, d);  // before the size arithmetic below
    if (r != SAGE_OK) return r;
    const Shape s{B, H, N, d};
    const size_t need = stats_ws_bytes(s);
    if (need > kNoAllocScratchBytes) {
        set_last_error("sage_quant_qk_noalloc: this shape needs %zu bytes of scratch "
                       "(sage_quant_workspace_bytes); the built-in scratch holds %zu",
                       need, kNoAllocScratchBytes);
        return SAGE_ERR_WORKSPACE;
    }
    // The array below belongs to the current device: the inputs must live there
    // too, or the kernels (launched on the current device) would write another
    // device's array.
    if (q_bf16 && (r = check_on_current_device(q_bf16, "q")) != SAGE_OK) return r;
    void *scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) {
        set_last_error("sage_quant_qk_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return SAGE_ERR_CUDA;
    }
    return sage_quant_qk(q_bf16, q_stride, k_bf16, k_stride, B, H, N, d, q_i8, q_scale, k_i8, k_scale, k_mean,
                         scratch, kNoAllocScratchBytes, stream);
}
