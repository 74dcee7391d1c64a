// One-tile bidirectional SSD kernel for sm_100a: sequences of at most 128
// tokens, where both scans of a (batch, head) fit in one tensor-core tile and
// there is no state to carry.
//
// For a sequence that short the whole mixer is one masked product,
//   y = (M_f + M_b) X + (D_f + D_b) x,
//   M_f[t][s] = G_f[t][s] exp(a_t - a_s) dt_f[s] (s <= t),
//   M_b[t][s] = G_b[t][s] exp(a'_t - a'_s) dt_b[s] (s >= t),
// with G = C B^T of each direction. G depends only on the batch element and
// the B/C group, not on the head. Each CTA takes a contiguous run of (batch,
// head) units; for each B/C group in its run it forms G_f and G_b once on the
// tensor cores (TMEM, fp32), and then, for each head of the group, builds the
// head's mask from G and its own decays (bf16, in TMEM), runs Y = M X and
// writes y. With B/C shared by all heads (Mamba-2's ngroups = 1) the 24
// heads of a batch element share two G tiles.
// The two scans, added: "DiffuMamba: High-Throughput Diffusion LMs with Mamba
// Backbone", Technical Summary, 2. Methodology, Core Architecture. The
// packed 128-token, batch-512 shape: the "Waspr/mdlm-lm1b-gpt2-packed"
// model page (LM1B packed to 128 tokens, batch 512).
//
// Per CTA: 512 threads in four roles that hand work over through mbarriers,
// persistent over a contiguous run of (batch, head) units:
//  - warps 0..7 build the masked matrix of each head (warp w: TMEM lanes
//    32 (w % 4) .. + 31, the 16-column half w / 4 of each 32-column block)
//    into one of two bf16 M buffers in TMEM;
//  - warps 8..11 run each head's epilogue: y = Y + (D_f + D_b) x in fp32,
//    rounded to bf16 over the head's x in shared memory, then a TMA store;
//    their first thread issues the x loads, four heads ahead, and the stores;
//  - warp 12 (one thread) issues the C/B loads and the MMAs: G once per
//    group, Y = M X per head;
//  - warps 13..15 compute the decay vectors, each a whole head at a time,
//    heads j = 0, 1, 2 (mod 3) respectively, up to three heads ahead.
// The next group's C and B load while the current group's heads run. Every
// wait is bounded in time; an expired wait sets the workspace's timeout flag
// and the CTA stops storing.
#include <cuda.h>
#include <stdint.h>

#include "sm100.cuh"
#include "ssd_kernels.h"
#include "ssd_mask.cuh"
#include "ssd_tmap.h"
#include "ssd_fused_util.cuh"

namespace ssd {
namespace {

using namespace sm100;
using namespace fused;

constexpr int kT = 128;          // tokens of a sequence (at most)
constexpr int kThreads = 512;    // 8 mask warps, 4 epilogue warps, 1 MMA warp, 3 vector warps
constexpr uint32_t kSlab = 16384;   // 128 rows x 128 bytes

struct OneParams {
    const __nv_bfloat16 *dt;    // (2, batch, L, H)
    const float *A;             // (2, H)
    const float *D;             // (2, H)
    DeviceStatus *status;
    long long total;            // batch * H heads, taken in (batch, head) order
    int batch, L, H, G, hpg;    // hpg = H / G heads per B/C group
};

constexpr int kXS = 5;    // x slots (x of a head in, then its y out)
constexpr int kVS = 3;    // decay-vector buffers
// mbarriers: C and B of a group loaded; G of a group computed; x of a head
// loaded; Y of a head computed and read out (two buffers each); a head's
// vectors written; a head's masked matrix built (two buffers, one arrival per
// mask warp); a vector buffer read by every mask warp; all MMAs done
enum {
    B_CB = 0, B_G, B_X, B_Y = B_X + kXS, B_YE = B_Y + 2, B_V = B_YE + 2, B_MF = B_V + kVS, B_VE = B_MF + 2,
    B_END = B_VE + kVS, B_COUNT
};

template <int N>
struct OSmem {
    static constexpr uint32_t kTile = (N / 64) * kSlab;    // one 128 x N bf16 operand
    static constexpr uint32_t cb = 0;                      // C_f, B_f, C_b, B_b
    static constexpr uint32_t x = 4 * kTile;               // kXS x slots
    // kVS buffers of af, ab, dtf, dtb, colf, colb (128 floats each)
    static constexpr uint32_t kVecBytes = 6 * 512;
    static constexpr uint32_t vec = x + kXS * kSlab;
    static constexpr uint32_t small = vec + kVS * kVecBytes;
    static constexpr uint32_t bytes = small + 256;
};

// A (batch, head) unit and the step to the next one in (batch, head) order.
struct HeadPos {
    int b, h;
    __device__ __forceinline__ void next(int H) {
        if (++h == H) {
            h = 0;
            ++b;
        }
    }
};

// ---- packed fp32 pairs (sm_100a f32x2 arithmetic): two IEEE products per
// instruction, bit-identical to two scalar multiplies
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ uint64_t f2u(uint32_t lo, uint32_t hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// a * b + c on each element of the pairs, one rounding each (as fmaf)
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float lo_of(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_of(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
// a pair of fp32 values rounded to a bf16 pair (low element in the low half)
__device__ __forceinline__ uint32_t bf16x2_of(uint64_t v) {
    uint32_t d;
    asm("{\n\t.reg .f32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tcvt.rn.bf16x2.f32 %0, hi, lo;\n\t}" : "=r"(d) : "l"(v));
    return d;
}

// Off the diagonal: 16 columns [s1, s1 + 16) of one row of the masked matrix,
// g * (r * col[s]) with r the row's factor for the column block (forward or
// reverse, as in mask_offdiag) and col the direction's column factors.
__device__ __forceinline__ void offdiag16(const uint32_t (&g)[16], float r, const float *col,
                                          uint32_t (&packed)[8]) {
    const uint64_t rr = f2(r, r);
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
        const float4 c = *reinterpret_cast<const float4 *>(col + k);
        packed[k / 2] = bf16x2_of(mul2(f2u(g[k], g[k + 1]), mul2(rr, f2(c.x, c.y))));
        packed[k / 2 + 1] = bf16x2_of(mul2(f2u(g[k + 2], g[k + 3]), mul2(rr, f2(c.z, c.w))));
    }
}

// The diagonal block: columns [s1, s1 + 16) of row `row` (s1 = 32 J + c0, J =
// row / 32). The forward term g_f (r_f colf) is kept for s <= t and the reverse
// term g_b (r_b colb) for s >= t; on the row's own token both are kept, each
// equal to G dt there (the two factors of exp(a_t - a_e) exp(a_e - a_t)).
// Factorised while the block's decay span is below kMaxSpan, else one
// exponential per entry (as mask_diag).
__device__ __forceinline__ void diag16(int J, int c0, int row, float my_af, float my_ab,
                                       const uint32_t (&gf)[16], const uint32_t (&gb)[16], const MaskVectors &v,
                                       uint32_t (&packed)[8]) {
    const int s0 = J * 32, s1 = s0 + c0;
    const int rr = row - s1;   // the row's token relative to the first column
    const float span_f = v.af[s0] - v.af[s0 + 31], span_b = v.ab[s0 + 31] - v.ab[s0];
    if (span_f < kMaxSpan && span_b < kMaxSpan) {
        const uint64_t rf = f2(__expf(my_af - v.af[s0 + 31]), __expf(my_af - v.af[s0 + 31]));
        const uint64_t rb = f2(__expf(my_ab - v.ab[s0]), __expf(my_ab - v.ab[s0]));
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
            const float2 cf = *reinterpret_cast<const float2 *>(v.colf + s1 + k);
            const float2 cb = *reinterpret_cast<const float2 *>(v.colb + s1 + k);
            const uint64_t pf = mul2(f2u(gf[k], gf[k + 1]), mul2(rf, f2(cf.x, cf.y)));
            const uint64_t pb = mul2(f2u(gb[k], gb[k + 1]), mul2(rb, f2(cb.x, cb.y)));
            const float m0 = (k <= rr ? lo_of(pf) : 0.f) + (k >= rr ? lo_of(pb) : 0.f);
            const float m1 = (k + 1 <= rr ? hi_of(pf) : 0.f) + (k + 1 >= rr ? hi_of(pb) : 0.f);
            packed[k / 2] = pack_bf16x2(m0, m1);
        }
    } else {
        float m[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const int s = s1 + c;
            const float gfv = __uint_as_float(gf[c]), gbv = __uint_as_float(gb[c]);
            // the exponent of the selected side is <= 0
            m[c] = c < rr ? gfv * v.dtf[s] * __expf(my_af - v.af[s])
                 : c > rr ? gbv * v.dtb[s] * __expf(my_ab - v.ab[s])
                          : gfv * v.dtf[s] + gbv * v.dtb[s];
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) packed[k] = pack_bf16x2(m[2 * k], m[2 * k + 1]);
    }
}

// Named barrier over `count` threads that also ORs `pred` across them.
__device__ __forceinline__ bool bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void bar_named(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Wait until the shared-memory sources of all but the newest committed bulk
// store may be reused.
__device__ __forceinline__ void tma_store_wait_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
onetile_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_out,
               const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
               const OneParams p) {
    using S = OSmem<N>;
    constexpr int NSLAB = N / 64;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - smem_u32(smem_raw));
    uint64_t *bars = reinterpret_cast<uint64_t *>(g + S::small);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(g + S::small + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(g + S::small + 8 * B_COUNT + 4);
    static_assert(8 * B_COUNT + 8 <= 192, "barrier area");

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3;                   // TMEM lane quarter of the warp
    const int row = (q << 5) | lane;          // tile row (token t): TMEM lane
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    // this CTA's heads: [h0, h0 + n) of the (batch, head) list
    const long long h0 = (long long)blockIdx.x * p.total / gridDim.x;
    const int n = (int)((long long)(blockIdx.x + 1) * p.total / gridDim.x - h0);
    // (batch, head) of the CTA's head j; the loops step these incrementally
    auto head_at = [&](int j) { return HeadPos{(int)((h0 + j) / p.H), (int)((h0 + j) % p.H)}; };

    grid_launch_dependents();
    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), (i >= B_MF && i < B_VE + kVS) ? 8 : 1);
        fence_mbar_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_out);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_c);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: G_f [0,128), G_b [128,256); the masked matrix of even
    // heads [256,320), of odd heads [320,384) (bf16, two per column: matrix
    // columns [16 k, 16 k + 16) in TMEM columns [8 k, 8 k + 8)); Y of even
    // heads [384,448), of odd heads [448,512)
    const uint32_t tGf = tmem, tGb = tmem + 128;
    auto tM = [&](int j) { return tmem + 256 + 64 * (j & 1); };
    auto tY = [&](int j) { return tmem + 384 + 64 * (j & 1); };
    const uint32_t lane_off = (uint32_t)(q << 5) << 16;
    auto xslot = [&](int j) { return S::x + (uint32_t)(j % kXS) * kSlab; };
    auto vbuf = [&](int j) { return reinterpret_cast<float *>(g + S::vec + (j % kVS) * S::kVecBytes); };
    // the kernel ahead in the stream has finished before any global access
    grid_dependency_wait();

    if (warp < 8) {
        // ================= mask builders
        const int half = warp >> 2, c0 = 16 * half;
        HeadPos pos = head_at(0);
        int hg = pos.h % p.hpg;     // head j's place in its B/C group
        bool ok = true;             // warp-uniform: every wait of this warp so far succeeded
        int gk = 0;                 // groups begun
#pragma unroll 1
        for (int j = 0; j < n; ++j) {
            if (j > 0 && ++hg == p.hpg) hg = 0;
            if (j == 0 || hg == 0) {
                ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_G), (uint32_t)gk & 1u, abort_flag, p.status,
                                                                 1002));
                ++gk;
            }
            ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_V + j % kVS), (uint32_t)(j / kVS) & 1u,
                                                             abort_flag, p.status, 1003));
            // M of head j - 2 has been read by its MMA
            if (j >= 2)
                ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_Y + (j & 1)), (uint32_t)((j - 2) >> 1) & 1u,
                                                                 abort_flag, p.status, 1004));
            tc_fence_after();
            if (ok) {
                // row `row`, columns [32 J + c0, 32 J + c0 + 16) of every block J:
                // all G loads first, then the diagonal block and the three others
                const float *V = vbuf(j);
                const MaskVectors mv{V, V + 128, V + 256, V + 384, V + 512, V + 640};
                const float my_af = V[row], my_ab = V[128 + row];
                uint32_t gdf[16], gdb[16], go[3][16];
                tmem_ld16(tGf + lane_off + q * 32 + c0, gdf);
                tmem_ld16(tGb + lane_off + q * 32 + c0, gdb);
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int J = (q + 1 + k) & 3;
                    tmem_ld16((J < q ? tGf : tGb) + lane_off + J * 32 + c0, go[k]);
                }
                tmem_wait_ld();
                const uint32_t mrow = tM(j) + lane_off + 8 * half;
                uint32_t packed[8];
                diag16(q, c0, row, my_af, my_ab, gdf, gdb, mv, packed);
                tmem_st8(mrow + 16 * q, packed);
#pragma unroll
                for (int k = 0; k < 3; ++k) {
                    const int J = (q + 1 + k) & 3;
                    // forward blocks (left of the row's own) scale by exp(a_t - a_e), e
                    // the block's last token; reverse ones by exp(a'_t - a'_b), b its first
                    const float r = J < q ? __expf(my_af - V[J * 32 + 31]) : __expf(my_ab - V[128 + J * 32]);
                    offdiag16(go[k], r, (J < q ? V + 512 : V + 640) + J * 32 + c0, packed);
                    tmem_st8(mrow + 16 * J, packed);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (!ok) break;
            if (lane == 0) {
                mbar_arrive(bar(B_MF + (j & 1)));    // this warp's rows of M_j are built
                mbar_arrive(bar(B_VE + j % kVS));    // and it is done with head j's vectors
            }
        }
    } else if (warp >= 13) {
        // ================= decay vectors: warp 13 + k takes heads j = k (mod 3),
        // the whole head in one warp (lane l: tokens 4 l .. 4 l + 3, both
        // directions), into buffer j % 3 once the mask warps are done with head
        // j - 3. Per head: the decay sums (forward: A_f times the sum of dt_f
        // over tokens <= t; reverse: A_b times the sum of dt_b over tokens >=
        // t), dt, and the column factors exp(a_e - a_s) dt_s (e the last
        // (forward) or first (reverse) token of the 32-token block of s)
        const int vw = warp - 13;
        const int t0 = 4 * lane;
        bool ok = true;
        HeadPos pos = head_at(vw);
        float vf[4], vb[4], Af = 0.f, Ab = 0.f;
        auto load = [&](int j) {
#pragma unroll
            for (int k = 0; k < 4; ++k) vf[k] = vb[k] = 0.f;
            if (j < n) {
                Af = __ldg(p.A + pos.h);
                Ab = __ldg(p.A + p.H + pos.h);
                const __nv_bfloat16 *df = p.dt + (size_t)pos.b * p.L * p.H + pos.h;
                const __nv_bfloat16 *db = df + (size_t)p.batch * p.L * p.H;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (t0 + k < p.L) {
                        vf[k] = __bfloat162float(df[(size_t)(t0 + k) * p.H]);
                        vb[k] = __bfloat162float(db[(size_t)(t0 + k) * p.H]);
                    }
                pos.next(p.H);
                pos.next(p.H);
                pos.next(p.H);
            }
        };
        load(vw);
#pragma unroll 1
        for (int j = vw; j < n; j += kVS) {
            const float cf[4] = {vf[0], vf[1], vf[2], vf[3]}, cb[4] = {vb[0], vb[1], vb[2], vb[3]};
            const float A_f = Af, A_b = Ab;
            load(j + kVS);     // this warp's next head, in flight while this one is computed
            // inclusive sums over the lane's four tokens, then across the warp
            float sf[4], sb[4];
            sf[0] = cf[0];
            sb[0] = cb[0];
#pragma unroll
            for (int k = 1; k < 4; ++k) {
                sf[k] = sf[k - 1] + cf[k];
                sb[k] = sb[k - 1] + cb[k];
            }
            float xf = sf[3], xb = sb[3];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float nf = __shfl_up_sync(0xffffffffu, xf, o), nb = __shfl_up_sync(0xffffffffu, xb, o);
                if (lane >= o) {
                    xf += nf;
                    xb += nb;
                }
            }
            const float tot_b = __shfl_sync(0xffffffffu, xb, 31);
            const float pre_f = xf - sf[3], pre_b = xb - sb[3];     // sums over the lanes before this one
            float af[4], ab[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                af[k] = A_f * (pre_f + sf[k]);
                ab[k] = A_b * (tot_b - (pre_b + sb[k]) + cb[k]);
            }
            // block edges: the last token of the lane's 32-token block (forward),
            // its first (reverse)
            const float ef = __shfl_sync(0xffffffffu, af[3], lane | 7), eb = __shfl_sync(0xffffffffu, ab[0], lane & ~7);
            if (j >= kVS)
                ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_VE + j % kVS), (uint32_t)(j / kVS - 1) & 1u,
                                                                 abort_flag, p.status, 1011));
            if (!ok) break;
            float *V = vbuf(j);
            *reinterpret_cast<float4 *>(V + t0) = make_float4(af[0], af[1], af[2], af[3]);
            *reinterpret_cast<float4 *>(V + 128 + t0) = make_float4(ab[0], ab[1], ab[2], ab[3]);
            *reinterpret_cast<float4 *>(V + 256 + t0) = make_float4(cf[0], cf[1], cf[2], cf[3]);
            *reinterpret_cast<float4 *>(V + 384 + t0) = make_float4(cb[0], cb[1], cb[2], cb[3]);
            *reinterpret_cast<float4 *>(V + 512 + t0) =
                make_float4(__expf(ef - af[0]) * cf[0], __expf(ef - af[1]) * cf[1], __expf(ef - af[2]) * cf[2],
                            __expf(ef - af[3]) * cf[3]);
            *reinterpret_cast<float4 *>(V + 640 + t0) =
                make_float4(__expf(eb - ab[0]) * cb[0], __expf(eb - ab[1]) * cb[1], __expf(eb - ab[2]) * cb[2],
                            __expf(eb - ab[3]) * cb[3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_V + j % kVS));
        }
    } else if (warp == 12) {
        // ================= C/B loads and the MMAs (one thread)
        if (lane == 0) {
            constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, false);   // C (K) x B (K)
            constexpr uint32_t id_o = idesc_bf16_f32(128, 64, false, true);     // M (K) x X (MN)
            // C/B loads in flight: groups [cb_waited, cb_issued)
            int cb_issued = 0, cb_waited = 0;
            auto load_cb = [&](long long key) {
                const int b = (int)(key / p.G), gg = (int)(key % p.G);
                mbar_arrive_expect_tx(bar(B_CB), 4 * NSLAB * kSlab);
                for (int d = 0; d < 2; ++d)
                    for (int sl = 0; sl < NSLAB; ++sl) {
                        tma_load_5d(base + S::cb + (2 * d) * S::kTile + sl * kSlab, &tm_c, bar(B_CB), 64 * sl, gg,
                                    0, b, d);
                        tma_load_5d(base + S::cb + (2 * d + 1) * S::kTile + sl * kSlab, &tm_b, bar(B_CB), 64 * sl,
                                    gg, 0, b, d);
                    }
                ++cb_issued;
            };
            // G_f = C_f B_f^T and G_b = C_b B_b^T of the group in shared memory
            auto issue_g = [&]() {
                const bool okc = mbar_wait_ool(bar(B_CB), (uint32_t)cb_waited & 1u, abort_flag, p.status, 1001);
                ++cb_waited;
                tc_fence_after();
                if (okc) {
                    for (int d = 0; d < 2; ++d) {
                        const uint32_t ca = base + S::cb + (2 * d) * S::kTile, ba = ca + S::kTile;
#pragma unroll 1
                        for (int k = 0; k < N / 16; ++k) {
                            const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                            mma_bf16_ss(d ? tGb : tGf, sdesc_sw128(ca + ko, 0, 1024), sdesc_sw128(ba + ko, 0, 1024),
                                        id_g, k > 0);
                        }
                    }
                }
                mma_commit(bar(B_G));
            };
            // head j: its batch element, its group `gg` and its place `hg` in the group
            HeadPos pos = head_at(0);
            int gg = pos.h / p.hpg, hg = pos.h - gg * p.hpg;
            load_cb((long long)pos.b * p.G + gg);
            issue_g();
            int gk = 0;
#pragma unroll 1
            for (int j = 0; j < n; ++j) {
                if (j > 0) {
                    pos.next(p.H);
                    if (++hg == p.hpg) {
                        hg = 0;
                        gg = pos.h == 0 ? 0 : gg + 1;
                    }
                }
                bool okm = true;
                if (j == 0 || hg == 0) {
                    // G of this group is in TMEM: C and B of the next group, if this
                    // CTA has one, may load
                    okm = mbar_wait_ool(bar(B_G), (uint32_t)gk & 1u, abort_flag, p.status, 1009);
                    ++gk;
                    if (okm && j + (p.hpg - hg) < n) load_cb((long long)pos.b * p.G + gg + 1);
                }
                // Y_j = M_j X_j, once M_j is built, x_j is in and Y of head j - 2 has been read out
                okm = okm && mbar_wait_ool(bar(B_MF + (j & 1)), (uint32_t)(j >> 1) & 1u, abort_flag, p.status, 1010);
                okm = okm && mbar_wait_ool(bar(B_X + j % kXS), (uint32_t)(j / kXS) & 1u, abort_flag, p.status, 1005);
                if (j >= 2)
                    okm = okm && mbar_wait_ool(bar(B_YE + (j & 1)), (uint32_t)((j - 2) >> 1) & 1u, abort_flag,
                                               p.status, 1006);
                tc_fence_after();
                if (!okm) break;
                const uint32_t xa = base + xslot(j);
#pragma unroll
                for (int k = 0; k < 128 / 16; ++k)
                    mma_bf16_ts(tY(j), tM(j) + 8 * k, sdesc_sw128(xa + k * 2048, kSlab, 1024), id_o, k > 0);
                mma_commit(bar(B_Y + (j & 1)));
                // the next head starts a new group: its G, now that every row of M_j is built
                if (j + 1 < n && hg + 1 == p.hpg) issue_g();
            }
            // teardown: every MMA and C/B load of this thread has finished
            mma_commit(bar(B_END));
            mbar_drain(bar(B_END), 0);
            for (int k = cb_waited; k < cb_issued; ++k) mbar_drain(bar(B_CB), (uint32_t)k & 1u);
        }
        __syncwarp();
    } else {
        // ================= epilogue, x loads and y stores (warps 8..11)
        const int r = tid - 256;                  // tile row of the epilogue
        const bool leader = r == 0;
        int x_issued = 0, x_seen = 0;             // the leader's x loads: heads [x_seen, x_issued) in flight
        HeadPos pos_x = head_at(0);               // the leader's next x load
        auto load_x = [&](int j) {
            mbar_arrive_expect_tx(bar(B_X + j % kXS), kSlab);
            tma_load_4d(base + xslot(j), &tm_x, bar(B_X + j % kXS), 0, pos_x.h, 0, pos_x.b);
            pos_x.next(p.H);
            ++x_issued;
        };
        if (leader)
            for (int j = 0; j < kXS - 1 && j < n; ++j) load_x(j);
        bool ok = true;
        HeadPos pos_e = head_at(0);               // head i of the epilogue
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            if (i > 0) pos_e.next(p.H);
            const int hi = pos_e.h;
            const float ds = __ldg(p.D + hi) + __ldg(p.D + p.H + hi);
            // ---------------- epilogue of head i: y = Y + (D_f + D_b) x, written over x
            ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_Y + (i & 1)), (uint32_t)(i >> 1) & 1u, abort_flag,
                                                             p.status, 1007) &&
                                             mbar_wait_ool(bar(B_X + i % kXS), (uint32_t)(i / kXS) & 1u, abort_flag,
                                                           p.status, 1008));
            if (leader) x_seen = i + 1;
            tc_fence_after();
            uint32_t ya[32], yb[32];
            if (ok) {
                tmem_ld32(tY(i) + lane_off, ya);
                tmem_ld32(tY(i) + lane_off + 32, yb);
                tmem_wait_ld();
            }
            tc_fence_before();
            __syncwarp();    // the named barriers are warp-collective: reconverge after the leader's steps
            if (bar_or(2, 128, !ok)) break;
            if (leader) mbar_arrive(bar(B_YE + (i & 1)));    // Y_i read out: the MMA of head i + 2 may write it
            // y = Y + (D_f + D_b) x in fp32 (fused, two at a time), rounded once to
            // bf16 over x (whose MMA has completed) for the TMA store
            uint8_t *xs = g + xslot(i);
            const uint64_t dd = f2(ds, ds);
            // every x chunk of the row first (the stores below would otherwise
            // hold each load back: the swizzled addresses are not known apart)
            uint4 xv[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) xv[cc] = *reinterpret_cast<const uint4 *>(xs + sw128_offset(r, cc));
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
                const uint32_t xu[4] = {xv[cc].x, xv[cc].y, xv[cc].z, xv[cc].w};
                uint32_t o[4];
#pragma unroll
                for (int j2 = 0; j2 < 4; ++j2) {
                    const int c = (cc & 3) * 8 + 2 * j2;
                    const uint32_t y0 = cc < 4 ? ya[c] : yb[c], y1 = cc < 4 ? ya[c + 1] : yb[c + 1];
                    o[j2] = bf16x2_of(fma2(dd, f2u(xu[j2] << 16, xu[j2] & 0xffff0000u), f2u(y0, y1)));
                }
                *reinterpret_cast<uint4 *>(xs + sw128_offset(r, cc)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            bar_named(2, 128);
            if (leader) {
                tma_store_4d(&tm_out, base + xslot(i), 0, hi, 0, pos_e.b);
                tma_store_commit();
                // x of head i + 4 into the slot of head i - 1, once its y has left
                if (i + kXS - 1 < n) {
                    tma_store_wait_read1();
                    load_x(i + kXS - 1);
                }
            }
        }
        if (leader) {
            // teardown: this thread's x loads and y stores have finished
            for (int k = x_seen; k < x_issued; ++k) mbar_drain(bar(B_X + k % kXS), (uint32_t)(k / kXS) & 1u);
            tma_store_wait_all();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int N>
cudaError_t run_onetile(const TcArgs &a, cudaStream_t stream) {
    using S = OSmem<N>;
    if (a.ws_bytes < kStatusBytes) return cudaErrorInvalidValue;
    OneParams p{};
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.A = a.A;
    p.D = a.D;
    p.status = static_cast<DeviceStatus *>(a.workspace);
    p.total = (long long)a.batch * a.H;
    p.batch = a.batch; p.L = a.L; p.H = a.H; p.G = a.G; p.hpg = a.H / a.G;
    CUtensorMap tm_x, tm_out, tm_b, tm_c;
    if (!tmap::map_x(&tm_x, a.x, a.batch, a.L, a.H) || !tmap::map_x(&tm_out, a.out, a.batch, a.L, a.H) ||
        !tmap::map_bc(&tm_b, a.B, 2, a.batch, a.L, a.G, N) || !tmap::map_bc(&tm_c, a.C, 2, a.batch, a.L, a.G, N))
        return cudaErrorInvalidValue;
    auto k = onetile_kernel<N>;
    const size_t smem = S::bytes + 1024;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    const int sms = device_sms();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.total < (sms > 0 ? sms : 1) ? p.total : (sms > 0 ? sms : 1)));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // programmatic stream serialization: the prologue overlaps the end of the
    // kernel ahead; the kernel waits for it before any global access
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, tm_x, tm_out, tm_b, tm_c, p);
}

}  // namespace

bool tc_onetile_supported(int batch, int L, int H, int G, int N) {
    if (batch <= 0 || L <= 0 || L > kT || H <= 0 || G <= 0 || H % G != 0) return false;
    if (N != 64 && N != 128) return false;
    return (long long)batch * H < (1ll << 31);
}

cudaError_t launch_tc_onetile(const TcArgs &a, cudaStream_t s) {
    if (a.ndir != 2 || a.init || a.rinit || !a.C) return cudaErrorNotSupported;
    if (!tc_onetile_supported(a.batch, a.L, a.H, a.G, a.N)) return cudaErrorNotSupported;
    return a.N == 64 ? run_onetile<64>(a, s) : run_onetile<128>(a, s);
}

}  // namespace ssd
