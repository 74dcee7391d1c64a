// Shared device helpers of the sm_100a SSD kernels: element loads/stores for
// the two I/O dtypes, the workspace status header and launch bookkeeping.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Status header at the start of every workspace. Kernels only ever OR flags
// into `flags`; ssd_get_device_status reads and clears it.
constexpr size_t kStatusBytes = 256;
struct DeviceStatus {
    unsigned int flags;       // kFlag* bits
    unsigned int where;       // id of the wait that expired first (diagnostic)
    unsigned int block;       // blockIdx.x of that wait
    unsigned int pad[61];
};
static_assert(sizeof(DeviceStatus) == kStatusBytes, "status header size");
enum : unsigned int { kFlagTimeout = 1u };

__device__ __forceinline__ void report_timeout(DeviceStatus *st, unsigned int where) {
    if (st) {
        unsigned int old = atomicOr(&st->flags, kFlagTimeout);
        if (!(old & kFlagTimeout)) {
            st->where = where;
            st->block = blockIdx.x;
        }
    }
}

template <typename T> struct IO;
template <> struct IO<float> {
    static __device__ __forceinline__ float load(const float *p) { return __ldg(p); }
    static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};
template <> struct IO<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
        return __bfloat162float(__ldg(p));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) {
        *p = __float2bfloat16_rn(v);
    }
};

}  // namespace ssd
