// sage_diag.cu -- diagnostics.
//   * A probe of the bounded-wait path: one warp waits on a shared-memory
//     barrier that nothing arrives on, with a short limit, through the same
//     helper every kernel of the library uses.  The wait gives up, records the
//     timeout (bit 0 and bit 8 + site of the device error word) and the kernel
//     returns normally, so the context stays usable and sage_check reports
//     SAGE_ERR_TIMEOUT.  Nothing faults, traps or hangs.
//   * A throughput probe of the exponential unit: the same `ex2.approx.ftz`
//     instruction the attention kernel's softmax issues, in eight independent
//     chains per thread over enough warps to keep the unit busy, so that the
//     caller can time it and state the softmax's exponential ceiling.
#include <cuda_runtime.h>

#include "sage.h"
#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kProbeSite = 0;

__global__ void __launch_bounds__(32) k_wait_probe(unsigned *err, long long limit_clocks) {
    __shared__ uint64_t bar;
    __shared__ AbortState abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival would complete phase 0; none comes
        abort.flag = 0;
        fence_barrier_init();
    }
    __syncwarp();
    wait_warp(&bar, 0, err, &abort, kProbeSite, limit_clocks);
}

// Eight chains x <- 2^x - 1.5 per thread (x stays in [-1.25, -0.5]), so every
// exponential depends only on its own chain's previous one; the sums are
// stored so that nothing is optimised away.
__global__ void __launch_bounds__(256) k_ex2_probe(float *sink, int iters) {
    float x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = -0.5f - 0.0625f * static_cast<float>((threadIdx.x + j) & 7);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = ex2_approx(x[j]) - 1.5f;
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += x[j];
    sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace
}  // namespace sage

using namespace sage;

extern "C" sage_status_t sage_debug_ex2_probe(float *sink, int blocks, int iters, sage_stream_t stream) {
    if (!sink || blocks < 1 || blocks > 65535 || iters < 1 || iters > (1 << 20)) {
        set_last_error("sink must be non-null, blocks in 1..65535, iters in 1..2^20");
        return SAGE_ERR_INVALID_ARG;
    }
    if (reinterpret_cast<uintptr_t>(sink) % 4) {
        set_last_error("sink is not 4-byte aligned");
        return SAGE_ERR_INVALID_ARG;
    }
    sage_status_t r = check_on_current_device(sink, "sink");
    if (r != SAGE_OK) return r;
    k_ex2_probe<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(sink, iters);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_last_error("ex2 probe launch: %s", cudaGetErrorString(e));
        return SAGE_ERR_CUDA;
    }
    return SAGE_OK;
}

extern "C" sage_status_t sage_debug_wait_timeout(int microseconds, sage_stream_t stream) {
    if (microseconds < 1 || microseconds > 1000000) {
        set_last_error("microseconds=%d must be in 1..1000000", microseconds);
        return SAGE_ERR_INVALID_ARG;
    }
    int dev = 0, khz = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev)) != cudaSuccess) {
        set_last_error("device query: %s", cudaGetErrorString(e));
        return SAGE_ERR_CUDA;
    }
    unsigned *err = device_error_ptr();
    if (!err) {
        set_last_error("device error word not found");
        return SAGE_ERR_CUDA;
    }
    const long long limit = (long long)microseconds * (khz > 0 ? khz : 2000000) / 1000;
    k_wait_probe<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(err, limit);
    if ((e = cudaGetLastError()) != cudaSuccess) {
        set_last_error("wait probe launch: %s", cudaGetErrorString(e));
        return SAGE_ERR_CUDA;
    }
    return SAGE_OK;
}
