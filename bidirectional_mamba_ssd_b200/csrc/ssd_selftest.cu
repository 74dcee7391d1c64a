// Self-test of the library's bounded device waits: one CTA waits on an
// mbarrier that nothing arrives on, with the given time limit, through the
// same wait routine every kernel uses. The wait must give up, record a
// timeout in the workspace's status header and let the kernel exit, leaving
// the context usable; ssd_get_device_status then reports SSD_ERR_TIMEOUT.
#include "sm100.cuh"
#include "ssd_bidir.h"
#include "ssd_common.cuh"

namespace ssd {
namespace {

__global__ void selftest_wait_kernel(DeviceStatus *status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        sm100::mbar_init(sm100::smem_u32(&bar), 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)   // phase 0 never completes: no thread arrives
        sm100::mbar_wait(sm100::smem_u32(&bar), 0, &abort_flag, status, 999, limit_ns);
    __syncthreads();
}

}  // namespace
}  // namespace ssd

extern "C" int ssd_selftest_wait_timeout(void *workspace, size_t ws_bytes, int limit_us, void *stream) {
    if (!workspace || ws_bytes < ssd::kStatusBytes) return SSD_ERR_WORKSPACE;
    if (limit_us <= 0 || limit_us > 2000000) return SSD_ERR_INVALID_ARG;
    ssd::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<ssd::DeviceStatus *>(workspace), 1000ull * (unsigned long long)limit_us);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
