// Tensor-core (tcgen05) kernels of the bidirectional SSD mixer, sm_100a.
//
// The sequence is cut into 128-token tiles. Within a tile the mixer is a
// dense contraction (the chunked form of the Mamba-2 SSD scan): with
// a_t = A * (sum of dt over the tile up to and including t),
//   forward  y_t  = sum_{s<=t} (C_t . B_s) exp(a_t - a_s) dt_s x_s + exp(a_t) C_t . H_in
// and, with a'_t = A' * (sum of dt' over the tile from t to its right end),
//   reverse  y'_t = sum_{s>=t} (C'_t . B'_s) exp(a'_t - a'_s) dt'_s x_s + exp(a'_t) C'_t . H'_in
// where H_in is the forward state entering the tile from the left and H'_in
// the reverse state entering it from the right. Tiles pass states through
//   H_next = exp(a_end) H + B^T diag(exp(a_end - a_s) dt_s) X.
// Because x is shared by both directions, the two masked 128x128 matrices
// are added before the single product with X.
//
// The forward + reverse sum follows "DiffuMamba: High-Throughput Diffusion
// LMs with Mamba Backbone", Technical Summary, 2. Methodology, Core
// Architecture (two Mamba-2 scans, added); the reverse scan is the forward
// one on the flipped sequence ("DiffMamba - Checkpoints" model card, Model
// details), evaluated here in natural order from the right end.
//
// Chunked path, three kernels:
//   tc_state_kernel  per (batch, head, direction, tile): S = B^T diag(w) X on
//                    the tensor cores, plus the tile's total decay;
//   tc_pass_kernel   per (batch, head, direction): the sequential state
//                    passing over tiles in fp32; writes every tile's incoming
//                    state (bf16, an MMA operand) and, for the prefix-state
//                    call, the final fp32 state;
//   tc_out_kernel    per (batch, head, tile): C.B^T of both directions, the
//                    decay mask, (M_f + M_b) X, C.H of both directions, the D
//                    term, and one bf16 TMA store of the output tile.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "sm100.cuh"
#include "ssd_kernels.h"
#include "ssd_mask.cuh"
#include "ssd_tmap.h"

namespace ssd {
namespace {

using namespace sm100;
using tmap::encode_fn;
using tmap::map_bc;
using tmap::map_h;
using tmap::map_x;

constexpr int kTile = 128;   // tokens per tile (MMA M)
constexpr int kP = 64;       // headdim
constexpr uint32_t kSlab = 16384;  // one 128-row x 128-byte swizzled slab

// ------------------------------------------------------------ device helpers
struct ChunkedParams {
    const __nv_bfloat16 *dt;   // (ndir, batch, L, H)
    const float *A;            // (ndir, H)
    const float *D;            // (2, H)
    float *S;                  // (batch, H, ndir, nt, N, 64) fp32 tile states
    float *g;                  // (batch, H, ndir, nt) tile decays
    __nv_bfloat16 *Hin;        // (batch, H, 2, nt, N, 64) incoming states, bf16
    const float *init;         // (batch, H, 64, N) or nullptr
    float *state_out;          // (batch, H, 64, N) or nullptr
    DeviceStatus *status;
    int batch, L, H, G, N, nt, ndir;
};

// Inclusive scan of one float per thread over a 128-thread block, in index
// order (prefix) or reverse order (suffix).
__device__ __forceinline__ float scan128(float v, bool suffix, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (!suffix) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        if (lane == 31) red[warp] = v;
    } else {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float n = __shfl_down_sync(0xffffffffu, v, o);
            if (lane + o < 32) v += n;
        }
        if (lane == 0) red[warp] = v;
    }
    __syncthreads();
    float add = 0.f;
    if (!suffix) {
        for (int k = 0; k < warp; ++k) add += red[k];
    } else {
        for (int k = warp + 1; k < 4; ++k) add += red[k];
    }
    __syncthreads();
    return v + add;
}

__device__ __forceinline__ float bf2f(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// ------------------------------------------------------------ kernel 1: tile states
// grid (nt, H, batch * ndir), 128 threads. S[n][p] = sum_s B[s][n] w_s X[s][p].
template <int N>
__global__ void __launch_bounds__(128) tc_state_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                       const __grid_constant__ CUtensorMap tm_b,
                                                       const ChunkedParams p) {
    constexpr int NSLAB = N / 64;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t sB = base;                      // NSLAB slabs
    const uint32_t sX = sB + NSLAB * kSlab;         // x tile
    const uint32_t sW = sX + kSlab;                 // diag(w) x, bf16 high part
    const uint32_t sWl = sW + kSlab;                // diag(w) x - high part, bf16
    uint8_t *small = gbase + (NSLAB + 3) * kSlab;
    uint64_t *bars = reinterpret_cast<uint64_t *>(small);        // [0] load, [1] mma
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(small + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(small + 20);
    float *red = reinterpret_cast<float *>(small + 32);

    const int tile = blockIdx.x, h = blockIdx.y;
    const int b = blockIdx.z / p.ndir, dir = blockIdx.z % p.ndir;
    const int g = h / (p.H / p.G);
    const int t0 = tile * kTile;
    const int tid = threadIdx.x;
    const uint32_t bar_load = smem_u32(&bars[0]), bar_mma = smem_u32(&bars[1]);

    if (tid == 0) {
        *abort_flag = 0;
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (tid < 32) {
        tmem_alloc(smem_u32(tmem_slot), 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == 0) {
        mbar_arrive_expect_tx(bar_load, (NSLAB + 1) * kSlab);
        tma_load_4d(sX, &tm_x, bar_load, 0, h, t0, b);
#pragma unroll
        for (int k = 0; k < NSLAB; ++k) tma_load_5d(sB + k * kSlab, &tm_b, bar_load, 64 * k, g, t0, b, dir);
    }

    // decay weights of this tile
    const int t = t0 + tid;
    const float dtv = t < p.L ? __bfloat162float(p.dt[((size_t)(dir * p.batch + b) * p.L + t) * p.H + h]) : 0.f;
    const float A = p.A[dir * p.H + h];
    const bool reverse = dir == 1;
    const float cs = scan128(dtv, reverse, red);     // forward: prefix sum; reverse: suffix sum
    __shared__ float total_s;
    if (reverse ? tid == 0 : tid == kTile - 1) total_s = cs;
    __syncthreads();
    const float total = total_s;
    // forward: w_s = exp(A (sum_{r>s} dt)) dt_s ; reverse: w_s = exp(A (sum_{r<s} dt)) dt_s
    const float w = __expf(A * (total - cs)) * dtv;

    const bool ok = mbar_wait(bar_load, 0, abort_flag, p.status, 1);
    if (ok) {
        // diag(w) X: row tid of the x tile, scaled; the swizzle permutes chunks
        // within a row only, so the row's 128 bytes are scaled in place order.
        // The product is kept as two bf16 terms (high part + remainder), so the
        // state carries ~16 mantissa bits of w x instead of 8.
        const uint4 *src = reinterpret_cast<const uint4 *>(gbase + (sX - base) + tid * 128);
        uint4 *dst = reinterpret_cast<uint4 *>(gbase + (sW - base) + tid * 128);
        uint4 *dstl = reinterpret_cast<uint4 *>(gbase + (sWl - base) + tid * 128);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = (k + tid) & 7;   // rows start at different chunks: no bank conflicts
            uint4 v = src[c], lo;
            uint32_t *u = reinterpret_cast<uint32_t *>(&v);
            uint32_t *ul = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float a0 = bf2f(u[j] & 0xffffu) * w, a1 = bf2f(u[j] >> 16) * w;
                const uint32_t hi = pack_bf16x2(a0, a1);
                ul[j] = pack_bf16x2(a0 - bf2f(hi & 0xffffu), a1 - bf2f(hi >> 16));
                u[j] = hi;
            }
            dst[c] = v;
            dstl[c] = lo;
        }
    }
    fence_proxy_async_smem();
    __syncthreads();

    bool issued = false;   // thread 0: whether the MMAs were issued
    if (tid == 0 && !*abort_flag) {
        issued = true;
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, 64, true, true);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
            // A = B^T (M = state index n, K = token s): MN-major, slabs of 64 n.
            // With N = 64 the second slab (rows 64..127 of D) reads the x tile
            // and the result rows are ignored.
            const uint64_t ad = sdesc_sw128(sB + k * 2048, kSlab, 1024);
            mma_bf16_ss(tmem, ad, sdesc_sw128(sW + k * 2048, kSlab, 1024), idesc, k > 0);
            mma_bf16_ss(tmem, ad, sdesc_sw128(sWl + k * 2048, kSlab, 1024), idesc, 1);
        }
        mma_commit(bar_mma);
    }
    __syncwarp();
    mbar_wait(bar_mma, 0, abort_flag, p.status, 2);
    tc_fence_after();

    const int warp = tid >> 5, lane = tid & 31;
    const int n = warp * 32 + lane;
    const size_t entry = ((size_t)(b * p.H + h) * p.ndir + dir) * p.nt + tile;
    uint32_t v[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + half * 32, v);
        tmem_wait_ld();
        if (n < N) {
            float4 *dst = reinterpret_cast<float4 *>(p.S + (entry * N + n) * kP + half * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                     __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
    }
    if (tid == 0) {
        p.g[entry] = __expf(A * total);
        // after an expired wait: the copies and MMAs this CTA started finish first
        mbar_drain(bar_load, 0);
        if (issued) mbar_drain(bar_mma, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------ kernel 2: state passing
// grid (N*64/1024, H, batch * ndir), 256 threads, 4 consecutive (n, p) values each.
__global__ void __launch_bounds__(256) tc_pass_kernel(const ChunkedParams p) {
    const int h = blockIdx.y, b = blockIdx.z / p.ndir, dir = blockIdx.z % p.ndir;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;   // element of the (N, 64) state
    const int n = e / kP, pc = e % kP;
    const size_t unit = (size_t)(b * p.H + h);
    float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
    if (dir == 0 && p.init) {
        const float *ip = p.init + unit * kP * p.N;
        hs = make_float4(ip[(pc + 0) * p.N + n], ip[(pc + 1) * p.N + n], ip[(pc + 2) * p.N + n],
                         ip[(pc + 3) * p.N + n]);
    }
    const size_t ebase = (unit * p.ndir + dir) * p.nt;
    for (int i = 0; i < p.nt; ++i) {
        const int tile = dir == 1 ? p.nt - 1 - i : i;
        const size_t entry = ebase + tile;
        if (p.Hin) {
            uint2 o;
            o.x = pack_bf16x2(hs.x, hs.y);
            o.y = pack_bf16x2(hs.z, hs.w);
            *reinterpret_cast<uint2 *>(p.Hin + entry * p.N * kP + e) = o;
        }
        const float4 s = *reinterpret_cast<const float4 *>(p.S + entry * p.N * kP + e);
        const float gg = p.g[entry];
        hs.x = fmaf(gg, hs.x, s.x);
        hs.y = fmaf(gg, hs.y, s.y);
        hs.z = fmaf(gg, hs.z, s.z);
        hs.w = fmaf(gg, hs.w, s.w);
    }
    if (dir == 0 && p.state_out) {
        float *op = p.state_out + unit * kP * p.N;
        op[(pc + 0) * p.N + n] = hs.x;
        op[(pc + 1) * p.N + n] = hs.y;
        op[(pc + 2) * p.N + n] = hs.z;
        op[(pc + 3) * p.N + n] = hs.w;
    }
}

// ------------------------------------------------------------ kernel 3: output tiles
// grid (nt, H, batch), 128 threads; thread t owns output row t of the tile.
template <int N>
__global__ void __launch_bounds__(128) tc_out_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                     const __grid_constant__ CUtensorMap tm_b,
                                                     const __grid_constant__ CUtensorMap tm_c,
                                                     const __grid_constant__ CUtensorMap tm_h,
                                                     const __grid_constant__ CUtensorMap tm_out,
                                                     const ChunkedParams p) {
    constexpr int NSLAB = N / 64;
    constexpr uint32_t kHBytes = N * 128;   // one bf16 (N, 64) state
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *gbase = smem_raw + (base - smem_u32(smem_raw));
    const uint32_t sX = base;
    const uint32_t sBf = sX + kSlab;
    const uint32_t sCf = sBf + NSLAB * kSlab;
    const uint32_t sBb = sCf + NSLAB * kSlab;
    const uint32_t sCb = sBb + NSLAB * kSlab;
    const uint32_t sHf = sCb + NSLAB * kSlab;
    const uint32_t sHb = sHf + kHBytes;
    const uint32_t sM = sHb + kHBytes;             // 2 slabs: masked matrix, K-major
    uint8_t *small = gbase + (sM - base) + 2 * kSlab;
    uint64_t *bars = reinterpret_cast<uint64_t *>(small);    // load, mma1, mma2
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(small + 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(small + 36);
    float *red = reinterpret_cast<float *>(small + 64);
    float *af = red + 8;            // A_f * prefix sum of dt_f
    float *ab = af + kTile;         // A_b * suffix sum of dt_b
    float *dtf = ab + kTile;
    float *dtb = dtf + kTile;
    float *colf = dtb + kTile;      // per-column mask factors
    float *colb = colf + kTile;

    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / (p.H / p.G);
    const int t0 = tile * kTile;
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t bar_load = smem_u32(&bars[0]), bar_mma1 = smem_u32(&bars[1]),
                   bar_mma2 = smem_u32(&bars[2]);

    if (tid == 0) {
        *abort_flag = 0;
        mbar_init(bar_load, 1);
        mbar_init(bar_mma1, 1);
        mbar_init(bar_mma2, 1);
        fence_mbar_init();
    }
    if (tid < 32) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: G_f [0,128) G_b [128,256) Yo_f [256,320) Yo_b [320,384) Yd [384,448)
    const uint32_t tG_f = tmem, tG_b = tmem + 128, tYo_f = tmem + 256, tYo_b = tmem + 320,
                   tYd = tmem + 384;

    if (tid == 0) {
        const long long ef = (((long long)b * p.H + h) * 2 + 0) * p.nt + tile;
        const long long eb = (((long long)b * p.H + h) * 2 + 1) * p.nt + tile;
        mbar_arrive_expect_tx(bar_load, (1 + 4 * NSLAB) * kSlab + 2 * kHBytes);
        tma_load_4d(sX, &tm_x, bar_load, 0, h, t0, b);
#pragma unroll
        for (int k = 0; k < NSLAB; ++k) {
            tma_load_5d(sBf + k * kSlab, &tm_b, bar_load, 64 * k, g, t0, b, 0);
            tma_load_5d(sCf + k * kSlab, &tm_c, bar_load, 64 * k, g, t0, b, 0);
            tma_load_5d(sBb + k * kSlab, &tm_b, bar_load, 64 * k, g, t0, b, 1);
            tma_load_5d(sCb + k * kSlab, &tm_c, bar_load, 64 * k, g, t0, b, 1);
        }
        // 3-d map over (64, N, entries): coordinate order innermost first
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(sHf),
            "l"(reinterpret_cast<uint64_t>(&tm_h)), "r"(bar_load), "r"(0), "r"(0), "r"((int)ef)
            : "memory");
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(sHb),
            "l"(reinterpret_cast<uint64_t>(&tm_h)), "r"(bar_load), "r"(0), "r"(0), "r"((int)eb)
            : "memory");
    }

    // decay sums of both directions for this tile
    const int t = t0 + tid;
    const size_t dt_dir = (size_t)p.batch * p.L * p.H;
    const float vf = t < p.L ? __bfloat162float(p.dt[((size_t)b * p.L + t) * p.H + h]) : 0.f;
    const float vb = t < p.L ? __bfloat162float(p.dt[dt_dir + ((size_t)b * p.L + t) * p.H + h]) : 0.f;
    const float Af = p.A[h], Ab = p.A[p.H + h];
    const float csf = scan128(vf, false, red);
    const float csb = scan128(vb, true, red);
    af[tid] = Af * csf;
    ab[tid] = Ab * csb;
    dtf[tid] = vf;
    dtb[tid] = vb;
    __syncthreads();
    const float my_af = af[tid], my_ab = ab[tid];
    mask_column_factors(tid, my_af, my_ab, vf, vb, af, ab, colf, colb);

    mbar_wait(bar_load, 0, abort_flag, p.status, 11);
    __syncthreads();
    bool issued1 = false, issued2 = false;   // thread 0: which MMA groups were issued
    if (tid == 0 && !*abort_flag) {
        issued1 = true;
        tc_fence_after();
        constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t id_o = idesc_bf16_f32(128, 64, false, true);
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;   // K-major step
            const uint64_t dCf = sdesc_sw128(sCf + ko, 0, 1024), dBf = sdesc_sw128(sBf + ko, 0, 1024);
            const uint64_t dCb = sdesc_sw128(sCb + ko, 0, 1024), dBb = sdesc_sw128(sBb + ko, 0, 1024);
            mma_bf16_ss(tG_f, dCf, dBf, id_g, k > 0);
            mma_bf16_ss(tG_b, dCb, dBb, id_g, k > 0);
            // C . H: B operand = state (rows n = K, 64 p = N), MN-major
            const uint64_t dHf = sdesc_sw128(sHf + k * 2048, kSlab, 1024);
            const uint64_t dHb = sdesc_sw128(sHb + k * 2048, kSlab, 1024);
            mma_bf16_ss(tYo_f, dCf, dHf, id_o, k > 0);
            mma_bf16_ss(tYo_b, dCb, dHb, id_o, k > 0);
        }
        mma_commit(bar_mma1);
    }
    __syncwarp();
    mbar_wait(bar_mma1, 0, abort_flag, p.status, 12);
    tc_fence_after();

    // masked matrix M = M_f + M_b, bf16, K-major into sM (column factors ready:
    // the load wait above is preceded by a block barrier)
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint8_t *mrow = gbase + (sM - base);
    const MaskVectors mv{af, ab, dtf, dtb, colf, colb};
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
        uint32_t gf[32], gb[32], packed[16];
        tmem_ld32(tG_f + lane_base + j * 32, gf);
        tmem_ld32(tG_b + lane_base + j * 32, gb);
        tmem_wait_ld();
        mask_block(j, tid, my_af, my_ab, gf, gb, mv, packed);
        // columns j*32 .. j*32+31 = slab j/2, chunks (j%2)*4 .. +3
        uint8_t *slab = mrow + (j >> 1) * kSlab;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int chunk = (j & 1) * 4 + c;
            *reinterpret_cast<uint4 *>(slab + sw128_offset(tid, chunk)) =
                make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && !*abort_flag) {
        issued2 = true;
        tc_fence_after();
        constexpr uint32_t id_y = idesc_bf16_f32(128, 64, false, true);
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
            const uint64_t dM = sdesc_sw128(sM + (k >> 2) * kSlab + (k & 3) * 32, 0, 1024);
            const uint64_t dX = sdesc_sw128(sX + k * 2048, kSlab, 1024);
            mma_bf16_ss(tYd, dM, dX, id_y, k > 0);
        }
        mma_commit(bar_mma2);
    }
    __syncwarp();
    mbar_wait(bar_mma2, 0, abort_flag, p.status, 13);
    tc_fence_after();

    // y = Yd + exp(a_t) Yo_f + exp(a'_t) Yo_b + (D_f + D_b) x, written over the x tile
    const float ef = __expf(my_af), eb = __expf(my_ab);
    const float dsum = p.D[h] + p.D[p.H + h];
    uint8_t *xrow = gbase + (sX - base);
#pragma unroll 1
    for (int j = 0; j < 2; ++j) {
        uint32_t yd[32], yf[32], yb[32];
        tmem_ld32(tYd + lane_base + j * 32, yd);
        tmem_ld32(tYo_f + lane_base + j * 32, yf);
        tmem_ld32(tYo_b + lane_base + j * 32, yb);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint4 *q = reinterpret_cast<uint4 *>(xrow + sw128_offset(tid, j * 4 + c));
            uint4 xv = *q;
            uint32_t *xu = reinterpret_cast<uint32_t *>(&xv);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i0 = c * 8 + 2 * u;
                float y0 = __uint_as_float(yd[i0]) + ef * __uint_as_float(yf[i0]) +
                           eb * __uint_as_float(yb[i0]) + dsum * bf2f(xu[u] & 0xffffu);
                float y1 = __uint_as_float(yd[i0 + 1]) + ef * __uint_as_float(yf[i0 + 1]) +
                           eb * __uint_as_float(yb[i0 + 1]) + dsum * bf2f(xu[u] >> 16);
                xu[u] = pack_bf16x2(y0, y1);
            }
            *q = xv;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        if (!*abort_flag) {
            tma_store_4d(&tm_out, sX, 0, h, t0, b);
            tma_store_commit();
        }
        tma_store_wait_all();
        // after an expired wait: the copies and MMAs this CTA started finish first
        mbar_drain(bar_load, 0);
        if (issued1) mbar_drain(bar_mma1, 0);
        if (issued2) mbar_drain(bar_mma2, 0);
    }
    __syncthreads();
    if (tid < 32) tmem_dealloc(tmem, 512);
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct ChunkedLayout {
    size_t s_off, g_off, h_off, total;
};

ChunkedLayout chunked_layout(int batch, int L, int H, int N, int ndir) {
    const size_t nt = (size_t)(L + kTile - 1) / kTile;
    const size_t entries = (size_t)batch * H * ndir * nt;
    ChunkedLayout c;
    c.s_off = 0;
    c.g_off = align256(c.s_off + entries * N * kP * sizeof(float));
    c.h_off = align256(c.g_off + entries * sizeof(float));
    c.total = c.h_off + (ndir == 2 ? align256(entries * N * kP * 2) : 0);
    return c;
}

constexpr size_t state_smem(int N) { return (N / 64 + 3) * kSlab + 1024 + 256; }
constexpr size_t out_smem(int N) {
    return kSlab + 4 * (N / 64) * kSlab + 2 * (size_t)N * 128 + 2 * kSlab + 1024 + 64 + 32 + 6 * kTile * 4 + 64;
}

template <int N>
cudaError_t run_chunked(const TcArgs &a, cudaStream_t stream) {
    const int nt = (a.L + kTile - 1) / kTile;
    const ChunkedLayout lay = chunked_layout(a.batch, a.L, a.H, N, a.ndir);
    if (a.ws_bytes < kStatusBytes + lay.total) return cudaErrorInvalidValue;
    char *scratch = static_cast<char *>(a.workspace) + kStatusBytes;
    ChunkedParams p{};
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.A = a.A;
    p.D = a.D;
    p.S = reinterpret_cast<float *>(scratch + lay.s_off);
    p.g = reinterpret_cast<float *>(scratch + lay.g_off);
    p.Hin = a.ndir == 2 ? reinterpret_cast<__nv_bfloat16 *>(scratch + lay.h_off) : nullptr;
    p.init = a.init;
    p.state_out = a.state_out;
    p.status = static_cast<DeviceStatus *>(a.workspace);
    p.batch = a.batch; p.L = a.L; p.H = a.H; p.G = a.G; p.N = N; p.nt = nt; p.ndir = a.ndir;

    CUtensorMap tm_x, tm_b;
    if (!map_x(&tm_x, a.x, a.batch, a.L, a.H) || !map_bc(&tm_b, a.B, a.ndir, a.batch, a.L, a.G, N))
        return cudaErrorInvalidValue;

    cudaError_t e;
    {
        auto k = tc_state_kernel<N>;
        const size_t sm = state_smem(N);
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
            return e;
        k<<<dim3(nt, a.H, a.batch * a.ndir), 128, sm, stream>>>(tm_x, tm_b, p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    tc_pass_kernel<<<dim3(N * kP / 1024, a.H, a.batch * a.ndir), 256, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.ndir == 1) return cudaSuccess;

    CUtensorMap tm_c, tm_h, tm_out;
    if (!map_bc(&tm_c, a.C, 2, a.batch, a.L, a.G, N) ||
        !map_h(&tm_h, p.Hin, (long long)a.batch * a.H * 2 * nt, N) ||
        !map_x(&tm_out, a.out, a.batch, a.L, a.H))
        return cudaErrorInvalidValue;
    auto k3 = tc_out_kernel<N>;
    const size_t sm3 = out_smem(N);
    if ((e = cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm3)) != cudaSuccess)
        return e;
    k3<<<dim3(nt, a.H, a.batch), 128, sm3, stream>>>(tm_x, tm_b, tm_c, tm_h, tm_out, p);
    return cudaGetLastError();
}

}  // namespace

size_t tc_chunked_scratch_bytes(int batch, int L, int H, int N, int ndir) {
    return chunked_layout(batch, L, H, N, ndir).total;
}

cudaError_t launch_tc_chunked(const TcArgs &a, cudaStream_t stream) {
    if (a.L == 0 || a.batch == 0) return cudaErrorNotSupported;
    if (!encode_fn()) return cudaErrorNotSupported;
    // TMA coordinates are 32-bit: entries of the state map must fit
    if ((long long)a.batch * a.H * 2 * ((a.L + kTile - 1) / kTile) >= (1ll << 31)) return cudaErrorNotSupported;
    return a.N == 64 ? run_chunked<64>(a, stream) : run_chunked<128>(a, stream);
}

}  // namespace ssd
