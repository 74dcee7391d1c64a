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
// are shared by all rows. The diagonal block factorises the same way while its
// decay span is moderate (mask_diag).
#pragma once

#include <stdint.h>

#include "sm100.cuh"

namespace ssd {

struct MaskVectors {
    const float *af, *ab;       // a_s and a'_s, 128 each
    const float *dtf, *dtb;     // dt_f[s], dt_b[s]
    const float *colf, *colb;   // per-column factors (see above)
};

// Largest decay span, within one 32-column block, for which the diagonal
// block is evaluated in factorised form: the row factor is then at most
// e^kMaxSpan and the column factor at least e^-kMaxSpan dt, both far inside
// fp32's range.
constexpr float kMaxSpan = 60.f;

// Off the diagonal: columns [32 J + c0, 32 J + c0 + W) of row `row` (W = 16 or
// 32, c0 = 0 or 16 with W = 16) for a column block J other than the row's own,
// packed as W/2 bf16 pairs. `g` holds the one G these columns need: the
// forward G_f when J is left of the row (J < row / 32), else the reverse G_b.
// Both directions share one code path (row factor and column factors picked
// by direction), so it stays in the instruction cache.
template <int W>
__device__ __forceinline__ void mask_offdiag(int J, int c0, int row, float my_af, float my_ab,
                                             const uint32_t (&g)[W], const MaskVectors &v,
                                             uint32_t (&packed)[W / 2]) {
    const bool fwd = J < (row >> 5);
    const int s0 = J * 32;
    const float r = __expf(fwd ? my_af - v.af[s0 + 31] : my_ab - v.ab[s0]);
    const float *col = (fwd ? v.colf : v.colb) + s0 + c0;
    float m[W];
#pragma unroll
    for (int q = 0; q < W; q += 4) {
        const float4 c = *reinterpret_cast<const float4 *>(col + q);
        m[q + 0] = __uint_as_float(g[q + 0]) * (r * c.x);
        m[q + 1] = __uint_as_float(g[q + 1]) * (r * c.y);
        m[q + 2] = __uint_as_float(g[q + 2]) * (r * c.z);
        m[q + 3] = __uint_as_float(g[q + 3]) * (r * c.w);
    }
#pragma unroll
    for (int q = 0; q < W / 2; ++q) packed[q] = sm100::pack_bf16x2(m[2 * q], m[2 * q + 1]);
}

// The diagonal block (J = row / 32): columns [32 J + c0, 32 J + c0 + W) of
// row `row`. Column s is left of the row (forward term only), right of it
// (reverse term only) or the row's own token (both, decay 1). The decay
// factorises through the block's edges as off the diagonal, now with a row
// factor >= 1 and a column factor <= 1:
//   exp(a_t - a_s)   = exp(a_t - a_e)   * exp(a_e - a_s),     e = last column
//   exp(a'_t - a'_s) = exp(a'_t - a'_b) * exp(a'_b - a'_s),   b = first column
// which is exact in fp32 while the block's decay span stays below kMaxSpan;
// past that (a warp-uniform test) each entry takes its own exponential.
template <int W>
__device__ __forceinline__ void mask_diag(int J, int c0, int row, float my_af, float my_ab,
                                          const uint32_t (&gf)[W], const uint32_t (&gb)[W],
                                          const MaskVectors &v, uint32_t (&packed)[W / 2]) {
    const int s0 = J * 32;
    const int s1 = s0 + c0;
    const int rr = row - s1;   // this row's position relative to the first column
    float m[W];
    const float span_f = v.af[s0] - v.af[s0 + 31], span_b = v.ab[s0 + 31] - v.ab[s0];
    if (span_f < kMaxSpan && span_b < kMaxSpan) {
        const float rf = __expf(my_af - v.af[s0 + 31]), rb = __expf(my_ab - v.ab[s0]);
#pragma unroll
        for (int q = 0; q < W; q += 4) {
            const float4 cf4 = *reinterpret_cast<const float4 *>(v.colf + s1 + q);
            const float4 cb4 = *reinterpret_cast<const float4 *>(v.colb + s1 + q);
            const float4 df4 = *reinterpret_cast<const float4 *>(v.dtf + s1 + q);
            const float4 db4 = *reinterpret_cast<const float4 *>(v.dtb + s1 + q);
            const float cfs[4] = {cf4.x, cf4.y, cf4.z, cf4.w}, cbs[4] = {cb4.x, cb4.y, cb4.z, cb4.w};
            const float dfs[4] = {df4.x, df4.y, df4.z, df4.w}, dbs[4] = {db4.x, db4.y, db4.z, db4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = q + e;
                const float gfv = __uint_as_float(gf[c]), gbv = __uint_as_float(gb[c]);
                m[c] = c < rr ? gfv * (rf * cfs[e]) : c > rr ? gbv * (rb * cbs[e]) : gfv * dfs[e] + gbv * dbs[e];
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < W; ++c) {
            const int s = s1 + c;
            const float gfv = __uint_as_float(gf[c]), gbv = __uint_as_float(gb[c]);
            // the exponent of the selected side is <= 0
            m[c] = c < rr ? gfv * v.dtf[s] * __expf(my_af - v.af[s])
                 : c > rr ? gbv * v.dtb[s] * __expf(my_ab - v.ab[s])
                          : gfv * v.dtf[s] + gbv * v.dtb[s];
        }
    }
#pragma unroll
    for (int q = 0; q < W / 2; ++q) packed[q] = sm100::pack_bf16x2(m[2 * q], m[2 * q + 1]);
}

// The diagonal block for one direction only (a kernel that runs each scan in
// its own CTA): forward (FWD) keeps columns s <= t, reverse s >= t, the row's
// own token with decay 1; `a`, `dt`, `col` are that direction's a_s, dt_s and
// column factors. Factorised through the block's edge as mask_diag while the
// block's decay span stays below kMaxSpan, else one exponential per entry;
// dropped entries are selected as 0, never multiplied.
template <bool FWD, int W>
__device__ __forceinline__ void mask_diag1(int J, int c0, int row, float my_a, const uint32_t (&g)[W],
                                           const float *a, const float *dt, const float *col,
                                           uint32_t (&packed)[W / 2]) {
    const int s0 = J * 32;
    const int s1 = s0 + c0;
    const int rr = row - s1;
    float m[W];
    const float span = FWD ? a[s0] - a[s0 + 31] : a[s0 + 31] - a[s0];
    if (span < kMaxSpan) {
        const float r = __expf(my_a - (FWD ? a[s0 + 31] : a[s0]));
#pragma unroll
        for (int q = 0; q < W; q += 4) {
            const float4 c4 = *reinterpret_cast<const float4 *>(col + s1 + q);
            const float4 d4 = *reinterpret_cast<const float4 *>(dt + s1 + q);
            const float cs[4] = {c4.x, c4.y, c4.z, c4.w}, ds[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = q + e;
                const float gv = __uint_as_float(g[c]);
                const bool keep = FWD ? c < rr : c > rr;
                m[c] = keep ? gv * (r * cs[e]) : c == rr ? gv * ds[e] : 0.f;
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < W; ++c) {
            const int s = s1 + c;
            const float gv = __uint_as_float(g[c]);
            const bool keep = FWD ? c < rr : c > rr;
            // the exponent of a kept entry is <= 0
            m[c] = keep ? gv * dt[s] * __expf(my_a - a[s]) : c == rr ? gv * dt[s] : 0.f;
        }
    }
#pragma unroll
    for (int q = 0; q < W / 2; ++q) packed[q] = sm100::pack_bf16x2(m[2 * q], m[2 * q + 1]);
}

// Columns [32 J, 32 J + 32) of row `row` given both G blocks, packed as 16 bf16 pairs.
__device__ __forceinline__ void mask_block(int J, int row, float my_af, float my_ab,
                                           const uint32_t (&gf)[32], const uint32_t (&gb)[32],
                                           const MaskVectors &v, uint32_t (&packed)[16]) {
    const int wq = row >> 5;
    if (J < wq) mask_offdiag<32>(J, 0, row, my_af, my_ab, gf, v, packed);
    else if (J > wq) mask_offdiag<32>(J, 0, row, my_af, my_ab, gb, v, packed);
    else mask_diag<32>(J, 0, row, my_af, my_ab, gf, gb, v, packed);
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

// scale_row for distinct source and destination tiles, one 16-byte chunk at a
// time in a rolled loop (less code where instruction fetch is the limit).
__device__ __forceinline__ void scale_row_rolled(const uint8_t *src_tile, uint8_t *dst_tile, int row, float w) {
    const uint4 *src = reinterpret_cast<const uint4 *>(src_tile + row * 128);
    uint4 *d = reinterpret_cast<uint4 *>(dst_tile + row * 128);
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
        uint4 v = src[(k + row) & 7];
        uint32_t *q = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(q[j] << 16) * w, hi = __uint_as_float(q[j] & 0xffff0000u) * w;
            q[j] = sm100::pack_bf16x2(lo, hi);
        }
        d[(k + row) & 7] = v;
    }
}

// Row `row` of diag(w) X kept as two bf16 terms: the rounded product into
// hi_tile (in place over the x tile is fine) and the remainder into lo_tile,
// so the pair carries ~16 mantissa bits of w x instead of 8.
__device__ __forceinline__ void scale_row_split(uint8_t *hi_tile, uint8_t *lo_tile, int row, float w) {
    uint4 *hi = reinterpret_cast<uint4 *>(hi_tile + row * 128);
    uint4 *lo = reinterpret_cast<uint4 *>(lo_tile + row * 128);
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = hi[(k + row) & 7];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        uint32_t *q = reinterpret_cast<uint32_t *>(&v[k]);
        uint4 l;
        uint32_t *ql = reinterpret_cast<uint32_t *>(&l);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float a0 = __uint_as_float(q[j] << 16) * w, a1 = __uint_as_float(q[j] & 0xffff0000u) * w;
            const uint32_t h = sm100::pack_bf16x2(a0, a1);
            ql[j] = sm100::pack_bf16x2(a0 - __uint_as_float(h << 16), a1 - __uint_as_float(h & 0xffff0000u));
            q[j] = h;
        }
        lo[(k + row) & 7] = l;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) hi[(k + row) & 7] = v[k];
}

}  // namespace ssd
