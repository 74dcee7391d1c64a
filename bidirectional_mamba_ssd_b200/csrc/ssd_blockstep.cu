// One-tile block-diffusion step for sm_100a: both scans over a block of at
// most 64 tokens, the forward one from the cached prefix state, the reverse
// one confined to the block, one CTA per (batch, head) unit.
//
// A denoising step re-reads the whole active block: x, both directions' dt,
// B and C, and the cached forward state (P x N, fp32), and writes y. With 64
// tokens there is no recurrence across tiles, so the kernel stacks the two
// directions as the 128 rows of one tensor-core tile instead of running two
// scans:
//   rows 0..63   the forward direction (C_f, B_f, token t = row),
//   rows 64..127 the reverse direction (C_b, B_b, token t = row - 64).
// One MMA gives G = [C_f; C_b] [B_f; B_b]^T (128 x 128, fp32 in TMEM); its two
// diagonal 64 x 64 blocks are C_f B_f^T and C_b B_b^T. The threads replace G
// in TMEM by the bf16 masked matrix M: row t of the forward half keeps
// exp(a_t - a_s) dt_s G_ts for s <= t in its own block and zero elsewhere, the
// reverse half the same for s >= t with the reverse decay sums. A second MMA
// Y = M [X; X] (x stacked twice along K) gives the forward output in rows
// 0..63 and the reverse output in rows 64..127, and a third, Yo = [C_f; C_b] H
// (H the cached state as a bf16 N x P operand), the state term of the forward
// rows. The epilogue adds y_f + exp(a_t) Yo_t + y_b + (D_f + D_b) x, the
// reverse rows passing theirs through shared memory.
// Forward scan from the cached state and reverse scan confined to the block:
// "Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality", Abstract and Technical Contribution; the two scans added:
// "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone", Technical
// Summary, 2. Methodology, Core Architecture.
//
// Per CTA: 288 threads. Warp 8 (its lane 0) issues the TMA loads and the
// MMAs, each as soon as its operands are ready: G = C B^T while warps 0..3
// compute the decay vectors and every mask warp converts its part of the
// cached state; C H once the state is in shared memory; Y once the mask is
// built. Warps 0..7 own TMEM lanes 32 (w % 4) .. + 31 (tile rows) and column
// half w / 4 of every per-row step (the mask's 64-column halves, the output's
// 32-column halves). Every wait is bounded in time; an expired wait sets the
// workspace's timeout flag and the CTA stores nothing.
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

constexpr int kT = 64;          // tokens of a block (at most)
constexpr int kP = 64;          // headdim
constexpr int kThreads = 288;       // 8 mask and epilogue warps, 1 issuing warp
constexpr int kIssueWarp = 8;       // lane 0: the TMA loads and the MMAs
constexpr uint32_t kSlab = 16384;   // 128 rows x 128 bytes

struct BlockParams {
    const __nv_bfloat16 *x;     // (batch, T, H, 64)
    const __nv_bfloat16 *dt;    // (2, batch, T, H)
    const float *A;             // (2, H)
    const float *D;             // (2, H)
    const float *prefix;        // (batch, H, 64, N) or nullptr (zero state)
    __nv_bfloat16 *out;         // (batch, T, H, 64)
    DeviceStatus *status;
    int batch, T, H, G;
};

// mbarriers: C and B loaded; x loaded; G computed; the cached state in shared
// memory (one arrival per mask warp); the masked matrix built (one arrival per
// mask warp); Y and C H computed
enum { B_LOAD = 0, B_X, B_G, B_H, B_M, B_Y, B_COUNT };

template <int N>
struct BSmem {
    static constexpr uint32_t c = 0;                        // [C_f; C_b], N / 64 slabs
    static constexpr uint32_t b = c + (N / 64) * kSlab;     // [B_f; B_b]; later the reverse rows' y (fp32)
    static constexpr uint32_t x = b + (N / 64) * kSlab;     // [X; X]
    static constexpr uint32_t h = x + kSlab;                // H as N rows of 64 bf16
    static constexpr uint32_t vec = h + N * 128;            // a, dt, col: 128 floats each
    static constexpr uint32_t small = vec + 3 * 128 * 4;    // barriers, TMEM address, abort flag, scan partials
    static constexpr uint32_t bytes = small + 128;
    static_assert(2 * kSlab >= 64 * 64 * 4, "reverse rows' y fits over B");
};

// Inclusive prefix sum of v over the 64 rows of one direction (two warps,
// `part` two floats of shared memory for that direction), and the total.
__device__ __forceinline__ float scan64(float v, int lane, int wi, float *part, float &total) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) part[wi] = v;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    total = part[0] + part[1];
    return wi ? v + part[0] : v;
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
blockstep_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_c, const BlockParams p) {
    using S = BSmem<N>;
    constexpr int NSLAB = N / 64;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - smem_u32(smem_raw));
    uint64_t *bars = reinterpret_cast<uint64_t *>(g + S::small);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(g + S::small + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(g + S::small + 8 * B_COUNT + 4);
    float *part = reinterpret_cast<float *>(g + S::small + 64);     // scan partials, two per direction
    float *Va = reinterpret_cast<float *>(g + S::vec), *Vdt = Va + 128, *Vcol = Va + 256;
    static_assert(8 * B_COUNT + 8 <= 64, "barrier area");

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, ch = warp >> 2;
    const int row = (q << 5) | lane;          // tile row: TMEM lane
    const bool fwd = row < 64;
    const int t = fwd ? row : row - 64;       // the row's token in the block
    const int u = (int)blockIdx.x, b = u / p.H, h = u % p.H, gg = h / (p.H / p.G);
    const bool has_h = p.prefix != nullptr;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    grid_launch_dependents();
    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), i == B_H || i == B_M ? 8 : 1);
        fence_mbar_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_c);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: G, then the masked matrix, [0,128); Y [128,192); Yo [192,256)
    const uint32_t tG = tmem, tY = tmem + 128, tYo = tmem + 192;
    const uint32_t lane_off = (uint32_t)(q << 5) << 16;
    // the kernel ahead in the stream has finished before any global access
    grid_dependency_wait();

    constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, false);   // [C_f; C_b] (K) x [B_f; B_b] (K)
    constexpr uint32_t id_o = idesc_bf16_f32(128, 64, false, true);     // C (K) x H (MN); M (K) x [X; X] (MN)
    if (warp == kIssueWarp) {
        // ================= the issuing thread: loads, then each MMA as soon as
        // its operands are ready (G while the vectors and the state are prepared)
        if (lane == 0) {
            // [C_f; C_b] and [B_f; B_b]: a 64-row box per direction and 64-column slab
            mbar_arrive_expect_tx(bar(B_LOAD), 4 * NSLAB * 8192);
            for (int d = 0; d < 2; ++d)
                for (int sl = 0; sl < NSLAB; ++sl) {
                    tma_load_5d(base + S::c + sl * kSlab + d * 8192, &tm_c, bar(B_LOAD), 64 * sl, gg, 0, b, d);
                    tma_load_5d(base + S::b + sl * kSlab + d * 8192, &tm_b, bar(B_LOAD), 64 * sl, gg, 0, b, d);
                }
            // x twice: the K rows of both halves of M
            mbar_arrive_expect_tx(bar(B_X), 2 * 8192);
            tma_load_4d(base + S::x, &tm_x, bar(B_X), 0, h, 0, b);
            tma_load_4d(base + S::x + 8192, &tm_x, bar(B_X), 0, h, 0, b);
            bool ok = mbar_wait_ool(bar(B_LOAD), 0, abort_flag, p.status, 901);
            tc_fence_after();
            if (ok) {
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                    mma_bf16_ss(tG, sdesc_sw128(base + S::c + ko, 0, 1024), sdesc_sw128(base + S::b + ko, 0, 1024),
                                id_g, k > 0);
                }
                mma_commit(bar(B_G));
            }
            // C H once the cached state is in shared memory
            if (ok && has_h) {
                ok = mbar_wait_ool(bar(B_H), 0, abort_flag, p.status, 906);
                tc_fence_after();
                if (ok) {
#pragma unroll 1
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                        mma_bf16_ss(tYo, sdesc_sw128(base + S::c + ko, 0, 1024),
                                    sdesc_sw128(base + S::h + k * 2048, kSlab, 1024), id_o, k > 0);
                    }
                }
            }
            // Y = M [X; X] once every row of M is built and x is in: rows 0..63
            // the forward output, rows 64..127 the reverse one
            ok = ok && mbar_wait_ool(bar(B_M), 0, abort_flag, p.status, 907) &&
                 mbar_wait_ool(bar(B_X), 0, abort_flag, p.status, 903);
            tc_fence_after();
            if (ok && !*abort_flag) {
#pragma unroll 1
                for (int k = 0; k < 128 / 16; ++k)
                    mma_bf16_ts(tY, tG + 16 * k, sdesc_sw128(base + S::x + k * 2048, kSlab, 1024), id_o, k > 0);
            }
            mma_commit(bar(B_Y));
        }
        __syncwarp();
    } else {
        // ================= warps 0..7: the decay vectors (warps 0..3), the
        // cached state's bf16 copy, then the mask. Every global load in flight
        // at once: dt of the row (warps 0..3: forward rows in warps 0, 1,
        // reverse rows in warps 2, 3; tokens past the block's end have dt = 0)
        // and this thread's 32 values of the cached state, row n of H^T (H[p][n]
        // for p in its half of the 64)
        const float A = p.A[(fwd ? 0 : p.H) + h];
        float v = 0.f;
        if (ch == 0 && t < p.T) v = __bfloat162float(p.dt[(((size_t)(fwd ? 0 : 1) * p.batch + b) * p.T + t) * p.H + h]);
        const int n = tid & 127, half = tid >> 7;
        float hv[32];
        if (has_h && n < N) {
            const float *ip = p.prefix + (size_t)u * kP * N + n + (size_t)half * 32 * N;
#pragma unroll
            for (int j = 0; j < 32; ++j) hv[j] = __ldg(ip + (size_t)j * N);
        }
        // decay sums and mask vectors
        if (ch == 0) {
            float tot;
            const float pf = scan64(v, lane, q & 1, part + (fwd ? 0 : 2), tot);
            // a_t: decay sum from the block's start (forward) or end (reverse) through t
            const float a = fwd ? A * pf : A * (tot - pf + v);
            Va[row] = a;
            Vdt[row] = v;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // column factor exp(a_e - a_s) dt_s, e the 32-column block's last
            // (forward) or first (reverse) column
            Vcol[row] = __expf(Va[fwd ? (row | 31) : (row & ~31)] - a) * v;
        }
        // the cached state as the bf16 N x 64 operand of C H
        if (has_h) {
            if (n < N) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4 *>(g + S::h + sw128_offset(n, half * 4 + c)) =
                        make_uint4(pack_bf16x2(hv[8 * c], hv[8 * c + 1]), pack_bf16x2(hv[8 * c + 2], hv[8 * c + 3]),
                                   pack_bf16x2(hv[8 * c + 4], hv[8 * c + 5]), pack_bf16x2(hv[8 * c + 6], hv[8 * c + 7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_H));
        }
        __syncwarp();
        asm volatile("bar.sync 3, 256;" ::: "memory");    // the vectors, to every mask warp

        // ---------------- the masked matrix, in place of G: this thread's row, the
        // direction's 32-column block `ch` of its 64 columns, and zero over the
        // other direction's block `ch`
        const int lq = q & 1;                       // the row's 32-row block within its direction
        const int vo = fwd ? 0 : 64;                // the direction's vectors
        const float my_a = Va[row];
        const int Jm = fwd ? ch : ch + 2, Jz = fwd ? ch + 2 : ch;
        uint32_t packed[16];
        const bool zero = fwd ? ch > lq : ch < lq;
        // tcgen05.ld/st are warp-wide: every branch around them is uniform in the warp
        if (__all_sync(0xffffffffu, mbar_wait_ool(bar(B_G), 0, abort_flag, p.status, 902))) {
            tc_fence_after();
            if (zero) {
#pragma unroll
                for (int c = 0; c < 16; ++c) packed[c] = 0u;
            } else {
                uint32_t gv[32];
                tmem_ld32(tG + lane_off + Jm * 32, gv);
                tmem_wait_ld();
                const MaskVectors mv{Va + vo, Va + vo, Vdt + vo, Vdt + vo, Vcol + vo, Vcol + vo};
                if (ch != lq) mask_offdiag<32>(ch, 0, t, my_a, my_a, gv, mv, packed);
                else if (fwd) mask_diag1<true, 32>(ch, 0, t, my_a, gv, Va, Vdt, Vcol, packed);
                else mask_diag1<false, 32>(ch, 0, t, my_a, gv, Va + 64, Vdt + 64, Vcol + 64, packed);
            }
            // matrix columns [16 k, 16 k + 16) go to TMEM columns [16 k, 16 k + 8)
            tmem_st8(tG + lane_off + Jm * 32, *reinterpret_cast<const uint32_t (*)[8]>(&packed[0]));
            tmem_st8(tG + lane_off + Jm * 32 + 16, *reinterpret_cast<const uint32_t (*)[8]>(&packed[8]));
            const uint32_t zz[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            tmem_st8(tG + lane_off + Jz * 32, zz);
            tmem_st8(tG + lane_off + Jz * 32 + 16, zz);
            tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_M));      // this warp's part of M is built
    }

    // ---------------- the epilogue (warps 0..7)
    const bool mine = warp < kIssueWarp;
    bool ok = true;
    uint8_t *yb = g + S::b;
    if (mine) {
        ok = __all_sync(0xffffffffu, mbar_wait_ool(bar(B_Y), 0, abort_flag, p.status, 904) &&
                                         mbar_wait_ool(bar(B_X), 0, abort_flag, p.status, 905));
        tc_fence_after();
        // the reverse rows' y into shared memory over B (fp32, 64 floats a row,
        // 16-byte chunks permuted by the row so a warp's stores spread over banks)
        if (ok && !fwd) {
            uint32_t v[32];
            tmem_ld32(tY + lane_off + ch * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4)
                *reinterpret_cast<uint4 *>(yb + t * 256 + (((ch * 8 + c4) ^ (t & 15)) << 4)) =
                    make_uint4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
        }
    }
    __syncthreads();
    // ---------------- out = y_f + exp(a_t) Yo + y_b + (D_f + D_b) x: the forward
    // rows, 32 columns a thread (rows past the block's end load but do not store)
    if (mine && fwd && __all_sync(0xffffffffu, ok && !*abort_flag)) {
        const float my_a = Va[row];
        uint32_t yv[32], ov[32];
        tmem_ld32(tY + lane_off + ch * 32, yv);
        if (has_h) tmem_ld32(tYo + lane_off + ch * 32, ov);
        tmem_wait_ld();
        const float e = has_h ? __expf(my_a) : 0.f;
        const float dsum = p.D[h] + p.D[p.H + h];
        uint4 *dst = reinterpret_cast<uint4 *>(p.out + (((size_t)b * p.T + t) * p.H + h) * kP + ch * 32);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(g + S::x + sw128_offset(t, ch * 4 + cc));
            const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
            const uint4 b0 = *reinterpret_cast<const uint4 *>(yb + t * 256 + (((ch * 8 + 2 * cc) ^ (t & 15)) << 4));
            const uint4 b1 = *reinterpret_cast<const uint4 *>(yb + t * 256 + (((ch * 8 + 2 * cc + 1) ^ (t & 15)) << 4));
            const uint32_t bu[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            uint32_t o[4];
#pragma unroll
            for (int j2 = 0; j2 < 4; ++j2) {
                float r[2];
#pragma unroll
                for (int e2 = 0; e2 < 2; ++e2) {
                    const int c = cc * 8 + 2 * j2 + e2;
                    const float xe = bf2f(e2 ? (xu[j2] >> 16) : (xu[j2] & 0xffffu));
                    const float yo = has_h ? e * __uint_as_float(ov[c]) : 0.f;
                    r[e2] = __uint_as_float(yv[c]) + yo + __uint_as_float(bu[2 * j2 + e2]) + dsum * xe;
                }
                o[j2] = pack_bf16x2(r[0], r[1]);
            }
            if (t < p.T) dst[cc] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    // ---------------- teardown: the MMAs are complete (B_Y) before TMEM is released
    if (warp == kIssueWarp && lane == 0) mbar_drain(bar(B_Y), 0);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// x or out: (batch, T, H, 64) -> box of 64 tokens x 64 for one (batch, head)
bool map_x64(CUtensorMap *m, const void *ptr, int batch, int T, int H) {
    uint64_t dims[4] = {kP, (uint64_t)H, (uint64_t)T, (uint64_t)batch};
    uint64_t str[3] = {kP * 2, (uint64_t)H * kP * 2, (uint64_t)T * H * kP * 2};
    uint32_t box[4] = {64, 1, kT, 1};
    return tmap::make_map(m, ptr, 4, dims, str, box);
}
// B or C: (2, batch, T, G, N) -> box of 64 tokens x 64 states
bool map_bc64(CUtensorMap *m, const void *ptr, int batch, int T, int G, int N) {
    uint64_t dims[5] = {(uint64_t)N, (uint64_t)G, (uint64_t)T, (uint64_t)batch, 2};
    uint64_t str[4] = {(uint64_t)N * 2, (uint64_t)G * N * 2, (uint64_t)T * G * N * 2,
                       (uint64_t)batch * T * G * N * 2};
    uint32_t box[5] = {64, 1, kT, 1, 1};
    return tmap::make_map(m, ptr, 5, dims, str, box);
}

template <int N>
cudaError_t run_blockstep(const TcArgs &a, cudaStream_t stream) {
    using S = BSmem<N>;
    if (a.ws_bytes < kStatusBytes) return cudaErrorInvalidValue;
    BlockParams p{};
    p.x = static_cast<const __nv_bfloat16 *>(a.x);
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.A = a.A;
    p.D = a.D;
    p.prefix = a.init;
    p.out = static_cast<__nv_bfloat16 *>(a.out);
    p.status = static_cast<DeviceStatus *>(a.workspace);
    p.batch = a.batch; p.T = a.L; p.H = a.H; p.G = a.G;
    CUtensorMap tm_x, tm_b, tm_c;
    if (!map_x64(&tm_x, a.x, a.batch, a.L, a.H) || !map_bc64(&tm_b, a.B, a.batch, a.L, a.G, N) ||
        !map_bc64(&tm_c, a.C, a.batch, a.L, a.G, N))
        return cudaErrorInvalidValue;
    auto k = blockstep_kernel<N>;
    const size_t smem = S::bytes + 1024;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.batch * a.H));
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
    return cudaLaunchKernelEx(&cfg, k, tm_x, tm_b, tm_c, p);
}

}  // namespace

bool tc_blockstep_supported(int batch, int T, int H, int G, int N) {
    if (batch <= 0 || T <= 0 || T > kT || H <= 0 || G <= 0 || H % G != 0) return false;
    if (N != 64 && N != 128) return false;
    return (long long)batch * H < (1ll << 31);
}

cudaError_t launch_tc_blockstep(const TcArgs &a, cudaStream_t s) {
    if (!tc_blockstep_supported(a.batch, a.L, a.H, a.G, a.N)) return cudaErrorNotSupported;
    return a.N == 64 ? run_blockstep<64>(a, s) : run_blockstep<128>(a, s);
}

}  // namespace ssd
