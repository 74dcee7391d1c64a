// Row pieces of the decay-masked matrix of one 128-token tile, shared by the
// tensor-core kernels.
//
// For tile rows t and columns s (both 0..127), with a_t = A_f * (prefix sum of
// dt_f up to t) and a'_t = A_b * (suffix sum of dt_b from t):
//   M[t][s] = G_f[t][s] exp(a_t - a_s) dt_f[s]     for s <= t   (forward scan)
//           + G_b[t][s] exp(a'_t - a'_s) dt_b[s]   for s >= t   (reverse scan)
// with G = C.B^T of each direction. Columns are handled in blocks of 32. A warp
// owns 32 consecutive rows, i.e. exactly one block of rows, so relative to a
// column block J it is uniformly below it (forward terms only, every s <= t),
// above it (reverse terms only) or on it (both, masked). Off the diagonal the
// decay factorises through the block's edge, with both factors <= 1:
//   forward:  exp(a_t - a_s)   = exp(a_t - a_e) * exp(a_e - a_s),    e = last column of J
//   reverse:  exp(a'_t - a'_s) = exp(a'_t - a'_b) * exp(a'_b - a'_s), b = first column of J
// so a row needs one exp per block and the per-column factors
//   colf[s] = exp(a_e - a_s) dt_f[s],  colb[s] = exp(a'_b - a'_s) dt_b[s]
// are shared by all rows. On the diagonal block each entry takes its own exp.
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace ssd {

struct MaskVectors {
    const float *af, *ab;       // a_s and a'_s, 128 each
    const float *dtf, *dtb;     // dt_f[s], dt_b[s]
    const float *colf, *colb;   // per-column factors (see above)
};

// Columns [32 J + c0, 32 J + c0 + W) of row `row` (W = 16 or 32, c0 = 0 or
// 16 with W = 16), packed as W/2 bf16 pairs.
template <int W>
__device__ __forceinline__ void mask_cols(int J, int c0, int row, float my_af, float my_ab,
                                          const uint32_t (&gf)[W], const uint32_t (&gb)[W],
                                          const MaskVectors &v, uint32_t (&packed)[W / 2]) {
    const int wq = row >> 5;
    const int s0 = J * 32;
    const int s1 = s0 + c0;
    float m[W];
    if (J < wq) {
        const float rf = __expf(my_af - v.af[s0 + 31]);
#pragma unroll
        for (int q = 0; q < W; q += 4) {
            const float4 c = *reinterpret_cast<const float4 *>(v.colf + s1 + q);
            m[q + 0] = __uint_as_float(gf[q + 0]) * (rf * c.x);
            m[q + 1] = __uint_as_float(gf[q + 1]) * (rf * c.y);
            m[q + 2] = __uint_as_float(gf[q + 2]) * (rf * c.z);
            m[q + 3] = __uint_as_float(gf[q + 3]) * (rf * c.w);
        }
    } else if (J > wq) {
        const float rb = __expf(my_ab - v.ab[s0]);
#pragma unroll
        for (int q = 0; q < W; q += 4) {
            const float4 c = *reinterpret_cast<const float4 *>(v.colb + s1 + q);
            m[q + 0] = __uint_as_float(gb[q + 0]) * (rb * c.x);
            m[q + 1] = __uint_as_float(gb[q + 1]) * (rb * c.y);
            m[q + 2] = __uint_as_float(gb[q + 2]) * (rb * c.z);
            m[q + 3] = __uint_as_float(gb[q + 3]) * (rb * c.w);
        }
    } else {
        // diagonal block: column s is either left of the row (forward term
        // only), right of it (reverse term only) or the row's own token (both,
        // decay 1), so one exp per entry
        const int rr = row - s1;   // this row's position relative to the first column
#pragma unroll
        for (int q = 0; q < W; q += 4) {
            const float4 af4 = *reinterpret_cast<const float4 *>(v.af + s1 + q);
            const float4 ab4 = *reinterpret_cast<const float4 *>(v.ab + s1 + q);
            const float4 df4 = *reinterpret_cast<const float4 *>(v.dtf + s1 + q);
            const float4 db4 = *reinterpret_cast<const float4 *>(v.dtb + s1 + q);
            const float afs[4] = {af4.x, af4.y, af4.z, af4.w};
            const float abs_[4] = {ab4.x, ab4.y, ab4.z, ab4.w};
            const float dfs[4] = {df4.x, df4.y, df4.z, df4.w};
            const float dbs[4] = {db4.x, db4.y, db4.z, db4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = q + e;
                const bool fwd = c < rr, rev = c > rr;
                const float gfv = __uint_as_float(gf[c]), gbv = __uint_as_float(gb[c]);
                // the exponent of the selected side is <= 0; the other side is
                // never used, so its possible overflow is harmless
                const float x = __expf(fwd ? my_af - afs[e] : my_ab - abs_[e]);
                const float wv = fwd ? gfv * dfs[e] : gbv * dbs[e];
                m[c] = (fwd || rev) ? wv * x : gfv * dfs[e] + gbv * dbs[e];
            }
        }
    }
#pragma unroll
    for (int q = 0; q < W / 2; ++q) packed[q] = sm100::pack_bf16x2(m[2 * q], m[2 * q + 1]);
}

// Columns [32 J, 32 J + 32) of row `row`, packed as 16 bf16 pairs.
__device__ __forceinline__ void mask_block(int J, int row, float my_af, float my_ab,
                                           const uint32_t (&gf)[32], const uint32_t (&gb)[32],
                                           const MaskVectors &v, uint32_t (&packed)[16]) {
    mask_cols<32>(J, 0, row, my_af, my_ab, gf, gb, v, packed);
}

// Per-column factors of column s (call once per column, before mask_block).
__device__ __forceinline__ void mask_column_factors(int s, float a_s, float ab_s, float dtf_s,
                                                    float dtb_s, const float *af, const float *ab,
                                                    float *colf, float *colb) {
    colf[s] = __expf(af[s | 31] - a_s) * dtf_s;
    colb[s] = __expf(ab[s & ~31] - ab_s) * dtb_s;
}

// Scale row `row` of a 128 x 128-byte bf16 tile by w into dst (row-local: the
// 128-byte swizzle permutes 16-byte chunks within a row only). Each thread
// starts at a different chunk so the 32 rows of a warp hit distinct banks.
__device__ __forceinline__ void scale_row(const uint8_t *src_tile, uint8_t *dst_tile, int row, float w) {
    const uint4 *src = reinterpret_cast<const uint4 *>(src_tile + row * 128);
    uint4 *d = reinterpret_cast<uint4 *>(dst_tile + row * 128);
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = src[(k + row) & 7];   // all loads first (src may equal dst)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint32_t *q = reinterpret_cast<uint32_t *>(&v[k]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(q[j] << 16) * w, hi = __uint_as_float(q[j] & 0xffff0000u) * w;
            q[j] = sm100::pack_bf16x2(lo, hi);
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) d[(k + row) & 7] = v[k];
}

}  // namespace ssd
