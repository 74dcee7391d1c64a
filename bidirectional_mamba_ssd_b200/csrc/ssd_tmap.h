// Host-side TMA tensor maps of the SSD kernels (bf16, 128-byte swizzle, zero
// fill outside the tensor). The driver entry point is fetched through the
// runtime, so the library does not link libcuda.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {
namespace tmap {

constexpr int kTile = 128;   // tokens per tile
constexpr int kP = 64;       // headdim

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// dims/box innermost first; strides = byte strides of dims 1..rank-1.
inline bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims,
                     const uint64_t *strides, const uint32_t *box) {
    auto fn = encode_fn();
    if (!fn) return false;
    uint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// x or out: (batch, L, H, 64) -> box of 128 tokens x 64 for one (batch, head)
inline bool map_x(CUtensorMap *m, const void *p, int batch, int L, int H) {
    uint64_t dims[4] = {kP, (uint64_t)H, (uint64_t)L, (uint64_t)batch};
    uint64_t str[3] = {kP * 2, (uint64_t)H * kP * 2, (uint64_t)L * H * kP * 2};
    uint32_t box[4] = {64, 1, kTile, 1};
    return make_map(m, p, 4, dims, str, box);
}
// B or C: (ndir, batch, L, G, N) -> box of 128 tokens x 64 states
inline bool map_bc(CUtensorMap *m, const void *p, int ndir, int batch, int L, int G, int N) {
    uint64_t dims[5] = {(uint64_t)N, (uint64_t)G, (uint64_t)L, (uint64_t)batch, (uint64_t)ndir};
    uint64_t str[4] = {(uint64_t)N * 2, (uint64_t)G * N * 2, (uint64_t)L * G * N * 2,
                       (uint64_t)batch * L * G * N * 2};
    uint32_t box[5] = {64, 1, kTile, 1, 1};
    return make_map(m, p, 5, dims, str, box);
}
// tile states, bf16 (entries, N, 64) -> box of N x 64
inline bool map_h(CUtensorMap *m, const void *p, long long entries, int N) {
    uint64_t dims[3] = {kP, (uint64_t)N, (uint64_t)entries};
    uint64_t str[2] = {kP * 2, (uint64_t)N * kP * 2};
    uint32_t box[3] = {64, (uint32_t)N, 1};
    return make_map(m, p, 3, dims, str, box);
}

}  // namespace tmap
}  // namespace ssd
