// diag.cu -- exercise of the kernels' failure path: a bounded wait that can
// never be satisfied must give up, record SPOT_ERR_DEVICE_TIMEOUT in the
// status word and return, leaving the context usable.
#include "spot_device.cuh"
#include "spot_internal.h"

namespace spot {
namespace {

__global__ void unsatisfied_wait_kernel(uint32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);                  // expects one arrival that never comes
    fence_mbar_init();
    if (!mbar_wait_bounded(&bar, 0)) flag_status(status, kStatusTimeout);
}

}  // namespace
}  // namespace spot

extern "C" spot_status_t spot_check_wait_timeout(void* status_ws, void* stream) {
    if (!status_ws || (reinterpret_cast<uintptr_t>(status_ws) % 256) != 0)
        return SPOT_ERR_INVALID_ARG;
    spot::unsatisfied_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint32_t*>(status_ws));
    return cudaGetLastError() == cudaSuccess ? SPOT_OK : SPOT_ERR_CUDA;
}
