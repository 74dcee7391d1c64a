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

// mbar_wait with its polling loop out of line: the call site holds one
// try_wait and a call, which keeps kernels with many wait sites small enough
// for the instruction cache. Same bound and abort rules as mbar_wait.
static __device__ __noinline__ bool mbar_wait_loop(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                            DeviceStatus *st, uint32_t where) {
    WaitClock clock;
    while (true) {
        if (*abort_flag) return false;
        if (mbar_try_wait(bar, parity)) return true;
        if (clock.expired(1000000000ull)) {
            *abort_flag = 1;
            report_timeout(st, where);
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait_ool(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                              DeviceStatus *st, uint32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_loop(bar, parity, abort_flag, st, where);
}

// ------------------------------------------------------------ global flags
// A flag store that publishes the writes before it (of this thread, and of
// the threads that passed a barrier with it) at GPU scope.
__device__ __forceinline__ void flag_release(unsigned int *f, unsigned int v) {
    asm volatile("fence.acq_rel.gpu;\n\tst.relaxed.gpu.global.u32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned int flag_acquire(const unsigned int *f) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}
// Poll a flag until it holds `v`, for at most `limit_ns` of waiting (the same
// clock rules as mbar_wait). On expiry: timeout in the status header, the
// CTA's abort flag up, false.
__device__ __forceinline__ bool flag_wait(const unsigned int *f, unsigned int v, volatile int *abort_flag,
                                          DeviceStatus *st, uint32_t where, uint64_t limit_ns = 1000000000ull) {
    if (flag_acquire(f) == v) return true;
    WaitClock clock;
    while (true) {
        if (*abort_flag) return false;
        if (flag_acquire(f) == v) return true;
        if (clock.expired(limit_ns)) {
            *abort_flag = 1;
            report_timeout(st, where);
            return false;
        }
        __nanosleep(64);
    }
}
// 16-byte global load that bypasses L1 (data another SM wrote), and store.
__device__ __forceinline__ float4 ld_cg_f4(const float *p) {
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ void st_f4(float *p, float a, float b, float c, float d) {
    asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
// Drop a 128-byte line from L2 without writing it back (its data is dead).
__device__ __forceinline__ void discard_l2_line(const void *p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}
// All threads of both CTAs of a cluster meet; global writes before it are
// visible to the other CTA after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
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
