// Device helpers shared by the fused tensor-core kernels: L2 cache policies,
// TMA copies with cache hints, named barriers of the 128-thread epilogue
// groups, and a prefix scan over such a group.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "sm100.cuh"

namespace ssd {
namespace fused {

using namespace sm100;

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_4d_hint(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0,
                                                 int c1, int c2, int c3, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tma_load_5d_hint(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0,
                                                 int c1, int c2, int c3, int c4, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0,
                                                 int c1, int c2, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void st_global_v4_hint(void *p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before the kernel ahead of it in the stream has
// finished; it must wait before touching global memory. Without the launch
// attribute both are no-ops.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel (if launched that way) start its own prologue.
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// named barriers of the three epilogue groups (128 threads each)
__device__ __forceinline__ void sync_c() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void sync_a() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
__device__ __forceinline__ void sync_b() { asm volatile("bar.sync 3, 128;" ::: "memory"); }

__device__ __forceinline__ float bf2f(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Inclusive prefix sum of `a` over the 128 rows of an epilogue group and the
// group's total, with `sync` the group's named barrier and `red` 4 floats of
// the group's own scratch.
template <typename Sync>
__device__ __forceinline__ void scan1(float &a, float &ta, int row, float *red, Sync sync) {
    const int lane = row & 31, wq = row >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float na = __shfl_up_sync(0xffffffffu, a, o);
        if (lane >= o) a += na;
    }
    if (lane == 31) red[wq] = a;
    sync();
    float pa = 0.f;
    for (int k = 0; k < wq; ++k) pa += red[k];
    ta = (red[0] + red[1]) + (red[2] + red[3]);
    sync();
    a += pa;
}

}  // namespace fused
}  // namespace ssd
