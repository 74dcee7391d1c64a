// Two-CTA bidirectional SSD kernel for sm_100a: each (batch, head) unit is
// taken by a cluster of two CTAs, one per scan direction, that run their scan
// in its own order and meet once per tile.
//
// The forward CTA walks the unit's 128-token tiles left to right and the
// reverse CTA right to left. Each carries its direction's state across tiles
// in fp32 registers, so neither needs a separate state pass: per tile it
// computes G = C.B^T, the one-direction decay mask, Y = M X, Yo = C.H (the
// state entering the tile) and the tile state S = B^T diag(w) X, on the
// tensor cores with TMA-staged operands. The two directions' outputs for a
// tile are added in fp32: the direction that reaches the tile first (the
// forward one on the left half of the sequence, the reverse one on the right
// half) stores Y + e Yo as an fp32 partial in global memory, which stays in
// L2, and signals it by arriving on a barrier in the other CTA's shared
// memory (one barrier per unit parity and tile); the other direction waits on
// that barrier in its own shared memory, adds the partial to its own
// Y + e Yo, adds (D_f + D_b) x, rounds once to bf16, stores the tile with TMA,
// and drops the partial's lines from L2 without a write-back. Addition in
// fp32 commutes, so the sum does not depend on which direction came first.
// Forward and reverse scans, added: "DiffuMamba: High-Throughput Diffusion
// LMs with Mamba Backbone", Technical Summary, 2. Methodology, Core
// Architecture; reverse = forward on the flipped sequence: "DiffMamba -
// Checkpoints" model card, Model details.
//
// Per CTA (448 threads):
//   warp 0       TMA producer: C and B tiles (4-slot ring, two tiles deep),
//                x tiles (3 slots)
//   warp 1       TMEM owner and MMA issuer (one thread). Per step n: G(n)
//                into one of two TMEM buffers, then Y(n-1) = M(n-1) X (the
//                mask of step n-1 was built meanwhile), Yo(n) into one of
//                two buffers, S(n)
//   warps 2..5   group C: the step's decay sums and mask vectors, the state
//                chain H <- exp(A sum dt) H + S (fp32 registers, bf16 copy for
//                the C.H MMA) and diag(w) X
//   warps 6..9   group A and warps 10..13 group B: the masked matrix (A the
//                32-column blocks 0 and 2, B blocks 1 and 3, written back into
//                the G buffer as bf16, the A operand of Y = M X from TMEM),
//                then the previous step's output (half of the columns each)
// In every group thread r owns tile row r = 32 * (warp % 4) + lane.
//
// Partial slots and their barriers are indexed by (cluster, unit parity,
// tile): a direction writes a slot for unit j + 2 only after reading the
// other direction's partials of unit j + 1, which the other direction wrote
// after it had read every partial of unit j, so a barrier is never arrived on
// twice before its waiters saw the first phase. The barrier protocol is modelled on
// the CPU (tests/test_pair_protocol.py). Every wait is bounded in time; an
// expired wait sets the workspace's timeout flag and the CTA runs to its end
// without storing. Both CTAs meet at a cluster barrier before either exits,
// so no arrival targets the shared memory of a CTA that has left.
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

constexpr int kTile = 128;
constexpr int kP = 64;
constexpr uint32_t kSlab = 16384;           // 128 rows x 128 bytes
constexpr int kRing = 4;                    // C/B slots of 32 KB: two tiles
constexpr int kXS = 3;                      // x slots
constexpr int kThreads = 448;
constexpr int kMaxNt = 256;                 // tiles per sequence (one partial barrier per tile and unit parity)
constexpr size_t kPartFloats = (size_t)kTile * kP;   // one fp32 partial tile (32 KB)

struct PairParams {
    const __nv_bfloat16 *dt;   // (2, batch, L, H)
    const float *A;            // (2, H)
    const float *D;            // (2, H)
    const float *init;         // (batch, H, 64, N) forward start state or nullptr
    const float *rinit;        // (batch, H, 64, N) reverse start state (at the sequence end) or nullptr
    float *part;               // (clusters, 2, nt) fp32 partial tiles, 16 column chunks x 128 rows x 4
    DeviceStatus *status;
    int batch, L, H, G, nt, units;
    int x2;                    // each direction scans its own x (tm_xr holds the reverse one's)
};

enum {
    B_RING_FULL = 0,                  // kRing
    B_RING_EMPTY = B_RING_FULL + kRing,
    B_X_FULL = B_RING_EMPTY + kRing,  // kXS
    B_X_EMPTY = B_X_FULL + kXS,
    B_G_READY = B_X_EMPTY + kXS,      // 2: MMA -> groups A and B, per G buffer
    B_M_READY = B_G_READY + 2,        // 2: groups A and B -> MMA (count 2), per G buffer
    B_Y_READY = B_M_READY + 2,        // MMA -> groups A and B
    B_Y_FREE,                         // group B -> MMA: Y and that step's Yo buffer are read
    B_H_READY,                        // group C -> MMA: H of the step is in shared memory
    B_XW_READY,                       // group C -> MMA: diag(w) X of the step
    B_S_READY,                        // MMA -> group C: S of the step (every MMA of the step done)
    B_VEC_READY,                      // 2: group C -> groups A and B
    B_VEC_FREE = B_VEC_READY + 2,     // 2: groups A and B -> group C (count 2)
    B_MMA_DONE = B_VEC_FREE + 2,
    B_COUNT
};

// Per-step vectors of one direction, from group C to groups A and B.
struct StepVec {
    float a[kTile];     // a_t: A times the sum of dt from the tile's start (forward) or end (reverse) through t
    float dt[kTile];
    float col[kTile];   // per-column mask factors
};

template <int N>
struct PSmem {
    static constexpr uint32_t kBC = N * 256;               // one B or C tile
    static constexpr uint32_t ring = 0;                    // kRing slots of 32 KB
    static constexpr uint32_t x0 = ring + kRing * 2 * kSlab;
    static constexpr uint32_t h = x0 + kXS * kSlab;        // bf16 (N, 64) state
    static constexpr uint32_t xw = h + N * 128;            // diag(w) X
    static constexpr uint32_t small = xw + kSlab;
    static constexpr uint32_t pbar = small + 512 + 2 * sizeof(StepVec);   // (unit parity, tile) barriers
    static constexpr uint32_t bytes = pbar + 8 * 2 * kMaxNt;
    static __device__ __forceinline__ uint32_t xslot(uint32_t j) { return x0 + j * kSlab; }
};


// ---- partial-ready barriers: a release arrival on the other CTA's barrier
// (distributed shared memory) after this CTA's partial stores, and an acquire
// wait at cluster scope on the own barrier before loading the other's partial
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_peer(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
static __device__ __noinline__ bool mbar_wait_cl_loop(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                      DeviceStatus *st, uint32_t where) {
    WaitClock clock;
    while (true) {
        if (*abort_flag) return false;
        if (mbar_try_wait_cl(bar, parity)) return true;
        if (clock.expired(1000000000ull)) {
            *abort_flag = 1;
            report_timeout(st, where);
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             DeviceStatus *st, uint32_t where) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    return mbar_wait_cl_loop(bar, parity, abort_flag, st, where);
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
tc_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_xr,
               const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
               const __grid_constant__ CUtensorMap tm_out, const PairParams p) {
    using S = PSmem<N>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - smem_u32(smem_raw));
    uint64_t *bars = reinterpret_cast<uint64_t *>(g + S::small);
    static_assert(8 * B_COUNT + 8 <= 256, "barrier area");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(g + S::small + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(g + S::small + 8 * B_COUNT + 4);
    float *red = reinterpret_cast<float *>(g + S::small + 256);          // 4 floats: group C scans
    StepVec *vec = reinterpret_cast<StepVec *>(g + S::small + 512);      // 2 buffers

    const int tid = threadIdx.x, warp = tid >> 5;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    // the cluster's two CTAs: rank 0 forward, rank 1 reverse
    const int dir = (int)(blockIdx.x & 1u), cl = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
    const int nt = p.nt;

    grid_launch_dependents();
    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < B_COUNT; ++i) {
            const bool two = i == B_M_READY || i == B_M_READY + 1 || i == B_VEC_FREE || i == B_VEC_FREE + 1;
            mbar_init(bar(i), two ? 2 : 1);
        }
    }
    // the partial-ready barriers: one per (unit parity, tile), completed by the
    // other CTA's arrival once it has stored its partial of that tile
    for (int q = tid; q < 2 * p.nt; q += kThreads) mbar_init(base + S::pbar + 8 * q, 1);
    fence_mbar_init();
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    // the kernel ahead in the stream has finished before any global access
    grid_dependency_wait();
    // both CTAs' barriers are initialised before either arrives on the other's
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr int NSLAB = N / 64;
    const bool fwd = dir == 0;
    const int lane = tid & 31;
    // TMEM columns: G/M buffers [0,128) and [128,256), Y [256,320), Yo buffers
    // [320,384) and [384,448), S [448,512)
    const uint32_t tY = tmem + 256, tS = tmem + 448;
    auto tG = [&](uint32_t n) { return tmem + 128 * (n & 1); };
    auto tYo = [&](uint32_t n) { return tmem + 320 + 64 * (n & 1); };
    const int hpg = p.H / p.G;
    const float *given = fwd ? p.init : p.rinit;
    auto tile_of = [&](int k) { return fwd ? k : nt - 1 - k; };
    // this direction reaches tile_of(k) before the other one (ties: forward)
    auto first_at = [&](int k) { return 2 * k < nt - 1 || (2 * k == nt - 1 && fwd); };
    // the state entering the unit's first tile is zero: no C.H term
    auto hzero = [&](int k) { return k == 0 && given == nullptr; };
    const size_t dt_off = (size_t)dir * p.batch * p.L * p.H;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(fwd ? &tm_x : &tm_xr);
            prefetch_tmap(&tm_b);
            prefetch_tmap(&tm_c);
            prefetch_tmap(&tm_out);
            const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
            uint32_t kr = 0, kx = 0;
            bool ok = true;
            for (int u = cl; ok && u < p.units; u += ncl) {
                const int b = u / p.H, h = u % p.H, gg = h / hpg;
                for (int k = 0; ok && k < nt; ++k) {
                    const int t0 = tile_of(k) * kTile;
                    const CUtensorMap *maps[2] = {&tm_c, &tm_b};
                    for (int q = 0; q < 2; ++q) {
                        const uint32_t s = kr % kRing;
                        if (kr >= kRing &&
                            !(ok = mbar_wait_ool(bar(B_RING_EMPTY + s), ((kr / kRing) - 1) & 1, abort_flag, p.status, 501)))
                            break;
                        ++kr;
                        mbar_arrive_expect_tx(bar(B_RING_FULL + s), S::kBC);
                        for (int sl = 0; sl < NSLAB; ++sl)
                            tma_load_5d_hint(base + S::ring + s * 2 * kSlab + sl * kSlab, maps[q],
                                             bar(B_RING_FULL + s), 64 * sl, gg, t0, b, dir, stream);
                    }
                    if (!ok) break;
                    const uint32_t xs = kx % kXS;
                    if (kx >= kXS &&
                        !(ok = mbar_wait_ool(bar(B_X_EMPTY + xs), ((kx / kXS) - 1) & 1, abort_flag, p.status, 502)))
                        break;
                    ++kx;
                    // the first reader of an x tile keeps it in L2 for the other direction
                    mbar_arrive_expect_tx(bar(B_X_FULL + xs), kSlab);
                    tma_load_4d_hint(base + S::xslot(xs), fwd ? &tm_x : &tm_xr, bar(B_X_FULL + xs), 0, h, t0, b,
                                     first_at(k) ? keep : stream);
                }
            }
            // every load issued has landed before the CTA may exit
            for (uint32_t k = kr > kRing ? kr - kRing : 0; k < kr; ++k)
                mbar_drain(bar(B_RING_FULL + k % kRing), (k / kRing) & 1);
            for (uint32_t k = kx > kXS ? kx - kXS : 0; k < kx; ++k) mbar_drain(bar(B_X_FULL + k % kXS), (k / kXS) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_state = idesc_bf16_f32(128, 64, true, true);   // B^T (MN) x diag(w) X (MN)
            constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, false);    // C (K) x B (K)
            constexpr uint32_t id_o = idesc_bf16_f32(128, 64, false, true);      // C (K) x H (MN); M (K) x X (MN)
            uint32_t kr = 0, nxw = 0, n = 0;
            auto slot_addr = [&](uint32_t s) { return base + S::ring + s * 2 * kSlab; };
            // Y(m) = M(m) X(m): the mask is in G buffer m & 1, X in x slot m % kXS
            auto issue_y = [&](uint32_t m) {
                mbar_wait_ool(bar(B_M_READY + (m & 1)), (m >> 1) & 1, abort_flag, p.status, 601);
                const uint32_t xs = m % kXS;
                mbar_wait_ool(bar(B_X_FULL + xs), (m / kXS) & 1, abort_flag, p.status, 602);
                if (m >= 1) mbar_wait_ool(bar(B_Y_FREE), (m - 1) & 1, abort_flag, p.status, 603);
                tc_fence_after();
                const uint32_t sX = base + S::xslot(xs);
#pragma unroll 1
                for (int k = 0; k < kTile / 16; ++k)
                    mma_bf16_ts(tY, tG(m) + 16 * k, sdesc_sw128(sX + k * 2048, kSlab, 1024), id_o, k > 0);
                mma_commit(bar(B_Y_READY));
            };
            const uint32_t nsteps = (uint32_t)((p.units - cl + ncl - 1) / ncl) * (uint32_t)nt;
#pragma unroll 1
            for (n = 0; n <= nsteps && !*abort_flag; ++n) {
                const int k = (int)(n % nt);
                uint32_t rC = 0, rB = 0, sC = 0, sB = 0;
                if (n < nsteps) {
                    rC = kr % kRing;
                    mbar_wait_ool(bar(B_RING_FULL + rC), (kr / kRing) & 1, abort_flag, p.status, 604);
                    ++kr;
                    rB = kr % kRing;
                    mbar_wait_ool(bar(B_RING_FULL + rB), (kr / kRing) & 1, abort_flag, p.status, 605);
                    ++kr;
                    tc_fence_after();
                    sC = slot_addr(rC);
                    sB = slot_addr(rB);
                    // G(n) = C B^T; buffer n & 1 was last read by Y(n - 2), issued before
#pragma unroll 1
                    for (int q = 0; q < N / 16; ++q) {
                        const uint32_t ko = (q >> 2) * kSlab + (q & 3) * 32;
                        mma_bf16_ss(tG(n), sdesc_sw128(sC + ko, 0, 1024), sdesc_sw128(sB + ko, 0, 1024), id_g,
                                    q > 0);
                    }
                    mma_commit(bar(B_G_READY + (n & 1)));
                }
                if (n >= 1) issue_y(n - 1);
                if (n == nsteps) break;   // that was the last step's Y
                // Yo(n) = C H: H is the state entering the tile; buffer n & 1 was read
                // by the output of step n - 2, done before Y(n - 1) was issued
                mbar_wait_ool(bar(B_H_READY), n & 1, abort_flag, p.status, 606);
                tc_fence_after();
                if (!hzero(k)) {
#pragma unroll 1
                    for (int q = 0; q < N / 16; ++q) {
                        const uint32_t ko = (q >> 2) * kSlab + (q & 3) * 32;
                        mma_bf16_ss(tYo(n), sdesc_sw128(sC + ko, 0, 1024),
                                    sdesc_sw128(base + S::h + q * 2048, kSlab, 1024), id_o, q > 0);
                    }
                }
                mma_commit(bar(B_RING_EMPTY + rC));
                // S(n) = B^T diag(w) X, the tile's own state (none after the unit's last tile)
                if (k < nt - 1) {
                    mbar_wait_ool(bar(B_XW_READY), nxw & 1, abort_flag, p.status, 607);
                    ++nxw;
                    tc_fence_after();
#pragma unroll 1
                    for (int q = 0; q < kTile / 16; ++q)
                        mma_bf16_ss(tS, sdesc_sw128(sB + q * 2048, kSlab, 1024),
                                    sdesc_sw128(base + S::xw + q * 2048, kSlab, 1024), id_state, q > 0);
                }
                mma_commit(bar(B_S_READY));
                mma_commit(bar(B_RING_EMPTY + rB));
            }
            // all MMAs complete before TMEM is released
            mma_commit(bar(B_MMA_DONE));
            mbar_drain(bar(B_MMA_DONE), 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ group C
        const int row = ((warp & 3) << 5) | lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
        float hreg[kP];
        // dt of the next step, fetched a step ahead (volatile loads, so the
        // compiler keeps them early)
        uint32_t raw = 0;
        auto load_dt = [&](int u, int k) {
            raw = 0;
            if (u >= p.units) return;
            const int b = u / p.H, h = u % p.H, t = tile_of(k) * kTile + row;
            if (t < p.L) {
                const __nv_bfloat16 *q = p.dt + dt_off + ((size_t)b * p.L + t) * p.H + h;
                asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(raw) : "l"(q));
            }
        };
        int cu = cl, ck = 0;
        load_dt(cu, ck);
        uint32_t n = 0;
        float gprev = 0.f;   // exp(A * sum of dt) of the previous tile
        for (int u = cl; u < p.units; u += ncl) {
            const int h = u % p.H;
            const float A = p.A[dir * p.H + h];
            for (int k = 0; k < nt; ++k, ++n) {
                const float v = bf2f(raw);
                if (++ck == nt) {
                    ck = 0;
                    cu += ncl;
                }
                load_dt(cu, ck);
                float pf = v, tot;
                scan1(pf, tot, row, red, sync_c);           // inclusive prefix sum in token order
                // decay sums from the tile's start (forward) or end (reverse) through t
                const float my_a = fwd ? A * pf : A * (tot - pf + v);
                const uint32_t vb = n & 1;
                if (n >= 2) mbar_wait_ool(bar(B_VEC_FREE + vb), ((n >> 1) - 1) & 1, abort_flag, p.status, 701);
                StepVec &V = vec[vb];
                V.a[row] = my_a;
                V.dt[row] = v;
                sync_c();
                // column factor exp(a_e - a_s) dt_s, e the column block's last (forward)
                // or first (reverse) column
                V.col[row] = __expf(V.a[fwd ? (row | 31) : (row & ~31)] - my_a) * v;
                sync_c();
                if (row == 0) mbar_arrive(bar(B_VEC_READY + vb));
                // every MMA of the previous step is done: S is in TMEM, H and
                // diag(w) X may be overwritten
                if (n >= 1) mbar_wait_ool(bar(B_S_READY), (n - 1) & 1, abort_flag, p.status, 702);
                tc_fence_after();
                if (k == 0) {
                    // the unit's start state (row n of the transposed (64, N) state) or zero
                    if (given && row < N) {
                        const float *ip = given + (size_t)u * kP * N + row;
#pragma unroll
                        for (int j = 0; j < kP; ++j) hreg[j] = ip[(size_t)j * N];
                    } else {
#pragma unroll
                        for (int j = 0; j < kP; ++j) hreg[j] = 0.f;
                    }
                } else {
                    // H <- exp(A sum dt) H + S of the previous tile
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t sv[32];
                        tmem_ld32(tS + lane_off + half * 32, sv);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            hreg[half * 32 + j] = fmaf(gprev, hreg[half * 32 + j], __uint_as_float(sv[j]));
                    }
                }
                if (!hzero(k) && row < N) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(g + S::h + sw128_offset(row, c)) =
                            make_uint4(pack_bf16x2(hreg[8 * c], hreg[8 * c + 1]),
                                       pack_bf16x2(hreg[8 * c + 2], hreg[8 * c + 3]),
                                       pack_bf16x2(hreg[8 * c + 4], hreg[8 * c + 5]),
                                       pack_bf16x2(hreg[8 * c + 6], hreg[8 * c + 7]));
                }
                fence_proxy_async_smem();
                tc_fence_before();
                sync_c();
                if (row == 0) mbar_arrive(bar(B_H_READY));
                if (k < nt - 1) {
                    // diag(w) X with w_s = exp(A * sum of dt over the rest of the tile
                    // in the scan's direction) dt_s
                    const float w = __expf(A * (fwd ? tot - pf : pf - v)) * v;
                    const uint32_t xs = n % kXS;
                    mbar_wait_ool(bar(B_X_FULL + xs), (n / kXS) & 1, abort_flag, p.status, 703);
                    scale_row_rolled(g + S::xslot(xs), g + S::xw, row, w);
                    fence_proxy_async_smem();
                    sync_c();
                    if (row == 0) mbar_arrive(bar(B_XW_READY));
                }
                gprev = __expf(A * tot);
            }
        }
    } else {
        // ------------------------------------------------------------ groups A and B
        const bool is_b = warp >= 10;
        const int row = ((warp & 3) << 5) | lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
        const int c0 = is_b ? 16 : 0;       // which half of each 32-column block, and of the output
        const int wq = warp & 3;            // this warp's row block
        auto sync_g = [&]() { if (is_b) sync_b(); else sync_a(); };
        auto sync_ab = [&]() { asm volatile("bar.sync 4, 256;" ::: "memory"); };

        // the output of step m (unit u, step k of it) from Y, Yo and, for the
        // direction that comes second, the other direction's partial
        auto out = [&](uint32_t m, int u, int k, float my_a) {
            const int i = tile_of(k), b = u / p.H, h = u % p.H;
            const uint32_t xs = m % kXS;
            const bool second = !first_at(k);
            const int j = (u - cl) / ncl;
            const size_t slot = ((size_t)cl * 2 + (j & 1)) * nt + i;
            const uint32_t pb = base + S::pbar + 8 * ((uint32_t)(j & 1) * nt + i);
            float *part = p.part + slot * kPartFloats;
            if (second) mbar_wait_cl(pb, (uint32_t)(j >> 1) & 1u, abort_flag, p.status, 801);
            // the other direction's partial for this thread's 32 columns, loaded
            // before the wait for Y so its L2 latency overlaps it
            float4 pv[8];
            if (second) {
#pragma unroll
                for (int e8 = 0; e8 < 8; ++e8) pv[e8] = ld_cg_f4(part + ((size_t)((c0 >> 1) + e8) * kTile + row) * 4);
            }
            mbar_wait_ool(bar(B_Y_READY), m & 1, abort_flag, p.status, 802);
            tc_fence_after();
            const float e = __expf(my_a);
            const bool yz = hzero(k);
            // D terms: with one x for both directions the second adds (D_f + D_b) x
            // after the partial; with one x per direction each adds its own D x
            // before (so the sum is the same whichever comes first)
            const float d_own = p.x2 ? p.D[dir * p.H + h] : 0.f;
            const float dsum = p.x2 ? 0.f : p.D[h] + p.D[p.H + h];
            const bool need_x = second || p.x2;
            uint8_t *xt = g + S::xslot(xs);
            const int q0 = c0 >> 3;              // first 16-column quarter: 0 or 2
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const int q = q0 + qq;
                uint32_t yv[16], ov[16];
                tmem_ld16(tY + lane_off + q * 16, yv);
                if (yz) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) ov[c] = 0u;
                } else {
                    tmem_ld16(tYo(m) + lane_off + q * 16, ov);
                }
                uint4 xv[2];
                if (need_x) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) xv[cc] = *reinterpret_cast<const uint4 *>(xt + sw128_offset(row, q * 2 + cc));
                }
                tmem_wait_ld();
                const uint32_t *xu = reinterpret_cast<const uint32_t *>(xv);
                auto xval = [&](int c) { return bf2f((c & 1) ? (xu[c >> 1] >> 16) : (xu[c >> 1] & 0xffffu)); };
                float y[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) y[c] = __uint_as_float(yv[c]) + e * __uint_as_float(ov[c]);
                if (p.x2) {
#pragma unroll
                    for (int c = 0; c < 16; ++c) y[c] += d_own * xval(c);
                }
                if (!second) {
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4)
                        st_f4(part + ((size_t)(q * 4 + e4) * kTile + row) * 4, y[4 * e4], y[4 * e4 + 1],
                              y[4 * e4 + 2], y[4 * e4 + 3]);
                } else {
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        y[4 * e4] += pv[4 * qq + e4].x;
                        y[4 * e4 + 1] += pv[4 * qq + e4].y;
                        y[4 * e4 + 2] += pv[4 * qq + e4].z;
                        y[4 * e4 + 3] += pv[4 * qq + e4].w;
                    }
                    uint4 ov4[2];
                    uint32_t *ou = reinterpret_cast<uint32_t *>(ov4);
#pragma unroll
                    for (int c2 = 0; c2 < 8; ++c2)
                        ou[c2] = pack_bf16x2(y[2 * c2] + dsum * xval(2 * c2), y[2 * c2 + 1] + dsum * xval(2 * c2 + 1));
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) *reinterpret_cast<uint4 *>(xt + sw128_offset(row, q * 2 + cc)) = ov4[cc];
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            sync_ab();
            // the partial is consumed: its 256 lines of 128 bytes leave L2 unwritten
            if (second) discard_l2_line(part + (size_t)((is_b ? 128 : 0) + row) * 32);
            if (is_b && row == 0) {
                mbar_arrive(bar(B_Y_FREE));
                if (!second) {
                    if (!*abort_flag) mbar_arrive_peer(peer_addr(pb, cluster_rank() ^ 1u));
                } else {
                    if (!*abort_flag) {
                        tma_store_4d(&tm_out, base + S::xslot(xs), 0, h, i * kTile, b);
                        tma_store_commit();
                    }
                    tma_store_wait_read();      // the store has read the slot
                }
                mbar_arrive(bar(B_X_EMPTY + xs));
            }
        };

        // steps of this CTA: its units (every ncl-th from cl) times nt tiles
        const uint32_t nsteps = (uint32_t)((p.units - cl + ncl - 1) / ncl) * (uint32_t)nt;
        float pa = 0.f;          // a_t of the previous step's row, for its output
#pragma unroll 1
        for (uint32_t n = 0; n <= nsteps; ++n) {
            float my_a = 0.f;
            if (n < nsteps) {
                // ---------------- mask of step n into G buffer n & 1
                const uint32_t vb = n & 1;
                mbar_wait_ool(bar(B_VEC_READY + vb), (n >> 1) & 1, abort_flag, p.status, 803);
                const StepVec &V = vec[vb];
                my_a = V.a[row];
                mbar_wait_ool(bar(B_G_READY + (n & 1)), (n >> 1) & 1, abort_flag, p.status, 804);
                tc_fence_after();
                const MaskVectors mv{V.a, V.a, V.dt, V.dt, V.col, V.col};
                const uint32_t tg = tG(n);
#pragma unroll 1
                for (int J = is_b ? 1 : 0; J < 4; J += 2) {
                    uint32_t packed[16];
                    if (fwd ? J > wq : J < wq) {      // entirely on the other direction's side
#pragma unroll
                        for (int c = 0; c < 16; ++c) packed[c] = 0u;
                    } else {
                        uint32_t gv[32];
                        tmem_ld32(tg + lane_off + J * 32, gv);
                        tmem_wait_ld();
                        if (J != wq) {
                            mask_offdiag<32>(J, 0, row, my_a, my_a, gv, mv, packed);
                        } else {
                            if (fwd) mask_diag1<true, 32>(J, 0, row, my_a, gv, V.a, V.dt, V.col, packed);
                            else mask_diag1<false, 32>(J, 0, row, my_a, gv, V.a, V.dt, V.col, packed);
                        }
                    }
                    // matrix columns [16 k, 16 k + 16) go to TMEM columns [16 k, 16 k + 8)
                    tmem_st8(tg + lane_off + J * 32, *reinterpret_cast<const uint32_t (*)[8]>(&packed[0]));
                    tmem_st8(tg + lane_off + J * 32 + 16, *reinterpret_cast<const uint32_t (*)[8]>(&packed[8]));
                }
                tmem_wait_st();
                tc_fence_before();
                sync_g();
                if (row == 0) {
                    mbar_arrive(bar(B_M_READY + (n & 1)));
                    mbar_arrive(bar(B_VEC_FREE + vb));
                }
            }
            // ---------------- output of the previous step
            if (n >= 1) {
                const uint32_t m = n - 1;
                out(m, cl + (int)(m / nt) * ncl, (int)(m % nt), pa);
            }
            pa = my_a;
        }
        if (is_b && row == 0) tma_store_wait_all();
    }


    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    // neither CTA leaves while the other may still arrive on its barriers
    cluster_sync_all();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// Clusters a call uses at most: one per two SMs, no more than there are units.
int pair_clusters_max(int units) {
    const int sms = device_sms();
    const int c = sms > 1 ? sms / 2 : 1;
    return units < c ? units : c;
}


template <int N>
cudaError_t run_pair(const TcArgs &a, cudaStream_t stream) {
    using S = PSmem<N>;
    const int nt = (a.L + kTile - 1) / kTile;
    const int units = a.batch * a.H;
    const int cmax = pair_clusters_max(units);
    if (a.ws_bytes < kStatusBytes + tc_pair_scratch_bytes(a.batch, a.L, a.H, N)) return cudaErrorInvalidValue;
    PairParams p{};
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.A = a.A;
    p.D = a.D;
    p.init = a.init;
    p.rinit = a.rinit;
    char *ws = static_cast<char *>(a.workspace);
    p.status = reinterpret_cast<DeviceStatus *>(ws);
    // partial tiles start on a 256-byte boundary whatever the workspace's own
    // alignment (the L2 discard works on whole 128-byte lines)
    const uintptr_t pa = reinterpret_cast<uintptr_t>(ws + kStatusBytes);
    p.part = reinterpret_cast<float *>((pa + 255) & ~(uintptr_t)255);
    p.batch = a.batch; p.L = a.L; p.H = a.H; p.G = a.G; p.nt = nt; p.units = units;

    p.x2 = a.x_dir_stride != 0;
    CUtensorMap tm_x, tm_xr, tm_b, tm_c, tm_out;
    const void *xr = p.x2 ? static_cast<const void *>(static_cast<const __nv_bfloat16 *>(a.x) + a.x_dir_stride) : a.x;
    if (!tmap::map_x(&tm_x, a.x, a.batch, a.L, a.H) || !tmap::map_x(&tm_xr, xr, a.batch, a.L, a.H) ||
        !tmap::map_bc(&tm_b, a.B, 2, a.batch, a.L, a.G, N) ||
        !tmap::map_bc(&tm_c, a.C, 2, a.batch, a.L, a.G, N) || !tmap::map_x(&tm_out, a.out, a.batch, a.L, a.H))
        return cudaErrorInvalidValue;
    auto k = tc_pair_kernel<N>;
    const size_t smem = S::bytes + 1024;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic stream serialization: the prologue overlaps the end of the
    // kernel ahead; the kernel waits for it before any global access
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2 * cmax);
    // as many clusters as the GPU holds at once (the kernel is persistent)
    int active = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&active, k, &cfg)) != cudaSuccess) return e;
    if (active < 1) return cudaErrorNotSupported;
    const int ncl = active < cmax ? active : cmax;
    cfg.gridDim = dim3(2 * ncl);
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k, tm_x, tm_xr, tm_b, tm_c, tm_out, p);
}

}  // namespace

size_t tc_pair_scratch_bytes(int batch, int L, int H, int N) {
    (void)N;
    const int nt = (L + kTile - 1) / kTile;
    const int cmax = pair_clusters_max(batch * H);
    if (cmax < 1 || nt < 1) return 0;
    return 256 + (size_t)cmax * 2 * nt * kPartFloats * sizeof(float);
}

bool tc_pair_supported(int batch, int L, int H, int G, int N) {
    (void)G;
    if (L <= kTile || batch <= 0) return false;     // at least two tiles per sequence
    if ((L + kTile - 1) / kTile > kMaxNt) return false;
    if (N != 64 && N != 128) return false;
    return (long long)batch * H < (1ll << 31);
}

cudaError_t launch_tc_pair(const TcArgs &a, cudaStream_t stream) {
    if (!tc_pair_supported(a.batch, a.L, a.H, a.G, a.N)) return cudaErrorNotSupported;
    if (!tmap::encode_fn()) return cudaErrorNotSupported;
    return a.N == 64 ? run_pair<64>(a, stream) : run_pair<128>(a, stream);
}

}  // namespace ssd
