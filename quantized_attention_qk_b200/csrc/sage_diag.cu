// sage_diag.cu -- a probe of the bounded-wait path: one warp waits on a
// shared-memory barrier that nothing arrives on, with a short limit, through
// the same helper every kernel of the library uses.  The wait gives up,
// records the timeout (bit 0 and bit 8 + site of the device error word) and
// the kernel returns normally, so the context stays usable and sage_check
// reports SAGE_ERR_TIMEOUT.  Nothing faults, traps or hangs.
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

}  // namespace
}  // namespace sage

using namespace sage;

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
