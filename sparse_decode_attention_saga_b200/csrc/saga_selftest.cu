// saga_selftest_wait_timeout: exercises the bounded-wait failure path of the
// kernels on purpose, without faulting or hanging the GPU.
//
// One CTA arms an mbarrier that nothing will ever complete and waits on it
// with the same bounded wait the pipelined kernels use (mbar_wait), but with
// a caller-chosen short limit.  When the wait gives up, the CTA raises the
// workspace's sticky timeout flag and returns; the host reads the flag with
// saga_workspace_error and the context stays usable.
#include <cuda_runtime.h>

#include "saga.h"
#include "saga_device.cuh"
#include "saga_kernels.h"

namespace saga {
namespace {

__global__ void wait_timeout_kernel(uint32_t* err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none ever comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (!mbar_wait(&bar, 0, &abort_flag, limit_ns) && threadIdx.x == 0)
        raise_device_error(err, kErrTimeout);
}

}  // namespace
}  // namespace saga

extern "C" int saga_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us,
                                          saga_stream_t stream) {
    if (!ws || ws_bytes < 256 || limit_us == 0 || limit_us > 1000000u) return SAGA_ERR_INVALID_ARG;
    saga::note_launches(1);
    saga::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint32_t*>(ws), static_cast<uint64_t>(limit_us) * 1000u);
    return cudaGetLastError() == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}
