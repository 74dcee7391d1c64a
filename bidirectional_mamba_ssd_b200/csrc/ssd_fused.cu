// Fused bidirectional SSD kernel for sm_100a: one persistent CTA per SM walks
// (batch, head) units; for each unit it computes both scans and writes the
// summed output once.
//
// Per unit, in two phases over 128-token tiles (the tile algebra is the one
// described in ssd_tc.cu):
//   phase 1, tiles right to left: the reverse scan's tile states
//            S' = B'^T diag(w') X on the tensor cores, chained in fp32
//            registers into the reverse state entering each tile from the
//            right; those states (bf16, the MMA operand of phase 2) go to
//            the workspace and stay L2-resident until phase 2 reads them;
//   phase 2, tiles left to right: C.B^T of both directions, the decay mask,
//            (M_f + M_b) X, C_f.H_f and C_b.H_b, the forward state chained
//            in fp32 registers, y = Yd + e_f Yo_f + e_b Yo_b + (D_f + D_b) x,
//            one bf16 TMA store per tile.
// Forward and reverse scans, added: "DiffuMamba: High-Throughput Diffusion
// LMs with Mamba Backbone", Technical Summary, 2. Methodology, Core
// Architecture; reverse = forward on the flipped sequence: "DiffMamba -
// Checkpoints" model card, Model details.
//
// Warp roles (448 threads):
//   warp 0       TMA producer: x tiles (2 slots), B/C tiles (4-slot ring),
//                reverse states (1 slot)
//   warp 1       TMEM owner and MMA issuer (one thread)
//   warps 2..5   epilogue group C: decay sums (both directions in one scan),
//                diag(w) X, the per-tile vectors, the fp32 state chains of
//                both directions and the reverse states' store
//   warps 6..9   epilogue group A: the first 16 columns of each 32-column
//                block of the masked matrix, the first 32 output columns
//   warps 10..13 epilogue group B: the last 16 columns of each block, the
//                last 32 output columns and the tile's TMA store
// In every group thread r owns tile row r = 32 * (warp % 4) + lane (its TMEM
// lane). Group C prepares tile i + 1 while groups A and B build the masked
// matrix of tile i. The masked matrix is written as bf16 into TMEM over the
// consumed C_f.B_f^T columns and read there as the A operand of
// (M_f + M_b) X. In phase 1, diag(w') X overwrites its own x slot and the
// tile states alternate between two TMEM buffers (the C.B^T columns are idle
// then); group C chains each tile's state one step late, so its scans and
// scaling of the next tile overlap the MMA.
// Phase-1 inputs (x, B') are loaded with an L2 evict-last hint and re-read in
// phase 2 with evict-first, so the re-read mostly hits L2.
//
// Every wait is an mbarrier wait bounded in time (sm100.cuh); a lost arrival
// sets the workspace's timeout flag and the CTA runs to its end.
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
constexpr uint32_t kSlab = 16384;       // 128 rows x 128 bytes
constexpr int kRing = 4;                // B/C ring slots (32 KB each)
constexpr int kThreads = 448;
constexpr int kXMax = 2;                // most x slots of any mode
constexpr int kG1 = 8;                  // state-pass tile decays in flight (>= x slots + 2)

// What one launch computes (a template parameter: each mode is its own kernel)
enum : int {
    kModeBidir = 0,      // both scans, summed output
    kModeBidirInit = 1,  // the same with the forward scan started from a given state
    kModeState = 2,      // the forward scan's final state only (optionally from a given state)
    kModeStateRev = 3,   // the reverse scan's final state only (the state at the sequence start)
};

// x slots: two in every mode. The count must be even: groups A and B take
// alternate state-pass tiles, and with an even count each group always gets
// the same slots and waits on every phase of their barriers (with an odd
// count a group could wait on a slot's next phase before the phase another
// group used had completed, and the parity wait would pass at once). The
// state mode pairs each slot with a buffer for the low part of diag(w) X.
template <int N, int MODE>
constexpr int x_slots() { return 2; }

struct FusedParams {
    const __nv_bfloat16 *dt;   // (2, batch, L, H); state mode: (batch, L, H)
    const float *A;            // (2, H); state mode: (H)
    const float *D;            // (2, H)
    __nv_bfloat16 *hb;         // (units, nt, N, 64) reverse states entering each tile
    const float *init;         // (batch, H, 64, N) forward start state (init / state modes) or nullptr
    const float *rinit;        // (batch, H, 64, N) reverse start state at the sequence end (init mode) or nullptr
    float *state_out;          // (batch, H, 64, N) final state of the state modes
    float *decay_out;          // (batch, H) state modes: exp(A * sum of dt) over the sequence, or nullptr
    DeviceStatus *status;
    int batch, L, H, G, nt, units;
    const float *dt_bias;      // DTRAW: (2, H); dt holds the raw projection
    float dt_lo, dt_hi;        // DTRAW: the step-size range
    int layer_units, A_layer;  // layers stacked along the batch: A, D of unit u at + (u / layer_units) * A_layer
    // 0: the next kernel may start its prologue at once, and this one waits for
    // the kernel ahead before touching global memory; 1: the next kernel may
    // start only after this one's wait (so it need not wait itself); 2: no wait
    // (launched right after an order-1 kernel, whose wait covers its inputs)
    int launch_order;
};

// A and D of unit u: a layer's own when several layers are stacked along the batch
__device__ __forceinline__ const float *layer_ptr(const float *base, const FusedParams &p, int u) {
    return p.layer_units ? base + (size_t)(u / p.layer_units) * p.A_layer : base;
}

// The step size from the raw projection (DTRAW): softplus(raw + bias),
// clamped to [lo, hi]. softplus(u) = log(1 + e^u), equal to u in fp32 beyond 20.
__device__ __forceinline__ float dt_from_raw(float raw, float bias, float lo, float hi) {
    const float u = raw + bias;
    const float sp = u > 20.f ? u : log1pf(__expf(u));
    return fminf(fmaxf(sp, lo), hi);
}

// barrier indices
enum {
    B_RING_FULL = 0,                 // kRing
    B_RING_EMPTY = B_RING_FULL + kRing,
    B_X_FULL = B_RING_EMPTY + kRing, // kXMax (x_slots() used)
    B_X_EMPTY = B_X_FULL + kXMax,    // kXMax
    B_HB_FULL = B_X_EMPTY + kXMax,
    B_HB_EMPTY,
    B_HB_WRITTEN,                    // group C -> producer: phase-1 states are in global memory
    B_G_READY,                       // MMA -> groups A and B (phase 2)
    B_S_READY,                       // MMA -> group C (phase 2)
    B_Y_READY,                       // MMA -> groups A and B
    B_P1S_READY,                     // 2: MMA -> group C, phase-1 tile state per TMEM buffer
    B_P1S_FREE = B_P1S_READY + 2,    // 2: group C -> MMA
    // per x slot (kXMax): diag(w) X of the tile in that slot is ready. One
    // barrier per slot, not a single one: in the state pass the preparing
    // groups can release several tiles before the MMA issuer takes the first,
    // and a single barrier would complete two phases under the issuer's
    // parity wait; a slot is refilled only after the MMA that read it.
    B_XW_READY = B_P1S_FREE + 2,
    B_M_READY = B_XW_READY + kXMax,  // groups A and B -> MMA (count 2)
    B_S_FREE,                        // group C -> MMA (phase 2)
    B_Y_FREE,                        // group B -> MMA
    B_VEC_READY,                     // 2: group C -> groups A and B, per vector buffer
    B_VEC_FREE = B_VEC_READY + 2,    // 2: groups A and B -> group C (count 2)
    B_G1_READY = B_VEC_FREE + 2,     // kG1: groups A/B -> group C, state-pass tile decay per buffer
    B_MMA_DONE = B_G1_READY + kG1,   // MMA issuer, at teardown
    B_COUNT
};

// Per-tile vectors group C writes and groups A and B read.
struct TileVec {
    float af[kTile];    // A_f * prefix sums of dt_f
    float ab[kTile];    // A_b * suffix sums of dt_b
    float dtf[kTile], dtb[kTile];
    float colf[kTile], colb[kTile];   // per-column mask factors
    float totf, totb;   // tile sums of dt_f, dt_b
    float pad[2];
};

// Inclusive prefix sums of two values over the 128 rows of group C (row
// order), and both totals.
__device__ __forceinline__ void scan2(float &a, float &b, float &ta, float &tb, int row, float *red) {
    const int lane = row & 31, wq = row >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float na = __shfl_up_sync(0xffffffffu, a, o);
        const float nb = __shfl_up_sync(0xffffffffu, b, o);
        if (lane >= o) {
            a += na;
            b += nb;
        }
    }
    if (lane == 31) {
        red[wq] = a;
        red[4 + wq] = b;
    }
    sync_c();
    float pa = 0.f, pb = 0.f;
    for (int k = 0; k < wq; ++k) {
        pa += red[k];
        pb += red[4 + k];
    }
    ta = (red[0] + red[1]) + (red[2] + red[3]);
    tb = (red[4] + red[5]) + (red[6] + red[7]);
    sync_c();
    a += pa;
    b += pb;
}

template <int N>
struct Smem {
    static constexpr uint32_t kBC = N * 256;            // one B or C tile (N/64 slabs)
    static constexpr uint32_t kH = N * 128;             // one bf16 (N, 64) state
    static constexpr uint32_t x0 = 0;                   // 2 x slots
    static constexpr uint32_t ring = x0 + 2 * kSlab;    // kRing slots of 32 KB
    static constexpr uint32_t hb = ring + kRing * 2 * kSlab;
    static constexpr uint32_t hf = hb + kH;
    static constexpr uint32_t xw = hf + kH;             // diag(w) x
    static constexpr uint32_t small = xw + kSlab;
    static constexpr uint32_t bytes = small + 7168;     // barriers, scan scratch, 2 tile-vector buffers
    static __device__ __forceinline__ uint32_t xslot(uint32_t j) { return x0 + j * kSlab; }
    // state mode: the low part of diag(w) X of x slot j, in the diag(w) X
    // buffer or the 16 KB from H_b on (H_b alone for N = 128, with H_f for N = 64)
    static __device__ __forceinline__ uint32_t loslot(uint32_t j) { return j == 0 ? xw : hb; }
    static_assert(hb + kSlab <= xw, "low-part slot 1");
};

// REUSE (one-tile sequences whose B/C are shared by several heads): each CTA
// takes a contiguous range of units (else every gridDim-th), and an output
// tile whose C/B tiles are those of the unit before it on the same CTA (same
// batch element and B/C group) takes them from the ring in place. DTRAW: dt
// holds the raw projection, and every valid token's step size is
// dt_from_raw of it (tokens past the end keep 0). Template parameters, so that
// the other kernels carry none of their code.
template <int N, int MODE, bool REUSE, bool DTRAW>
__global__ void __launch_bounds__(kThreads, 1)
tc_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_h,
                const __grid_constant__ CUtensorMap tm_out, const FusedParams p) {
    using S = Smem<N>;
    constexpr int NSLAB = N / 64;
    constexpr uint32_t kXS = x_slots<N, MODE>();
    constexpr bool kOut = MODE == kModeBidir || MODE == kModeBidirInit;   // an output pass follows the state pass
    constexpr bool kFwd1 = MODE == kModeState;     // the state pass runs forward (else reverse)
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *g = smem_raw + (base - smem_u32(smem_raw));
    uint64_t *bars = reinterpret_cast<uint64_t *>(g + S::small);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(g + S::small + 8 * B_COUNT);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(g + S::small + 8 * B_COUNT + 4);
    static_assert(8 * B_COUNT + 8 <= 416, "barrier area");
    float *gdec1 = reinterpret_cast<float *>(g + S::small + 416);  // kG1 state-pass tile decays
    float *red_ab = reinterpret_cast<float *>(g + S::small + 448); // 2 x 4 floats, groups A and B scans
    float *red = reinterpret_cast<float *>(g + S::small + 480);    // 8 floats, group C scans
    TileVec *vec = reinterpret_cast<TileVec *>(g + S::small + 512);  // 2 buffers

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    // the next kernel in the stream may set itself up while this one runs
    if (p.launch_order != 1) grid_launch_dependents();
    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(bar(i), (i == B_M_READY || i == B_VEC_FREE || i == B_VEC_FREE + 1) ? 2 : 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    // the kernel ahead in the stream has finished and its writes are visible
    // before this one reads or writes global memory
    if (p.launch_order != 2) grid_dependency_wait();
    if (p.launch_order == 1) grid_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: G_f [0,128), G_b [128,256), Yo_f [256,320), Yo_b [320,384),
    // Yd [384,448), S [448,512). The masked matrix M (bf16 pairs) reuses G_f's
    // columns: matrix columns [16k, 16k + 16) go to TMEM columns [16k, 16k + 8),
    // written by the group that consumed G_f's columns [16k, 16k + 16) (group A
    // for even k, group B for odd k); phase-1 tile states alternate between
    // TMEM columns [0,64) and [64,128).
    const uint32_t tGf = tmem, tGb = tmem + 128, tYof = tmem + 256, tYob = tmem + 320,
                   tYd = tmem + 384, tS = tmem + 448;
    const int nt = p.nt;
    // tiles of the state pass: all of them in the state modes; before an output
    // pass all but tile 0, whose own tile state no tile to its left receives
    const int n1t = kOut ? nt - 1 : nt;
    const int hpg = p.H / p.G;
    // this CTA's units: [u_begin, u_end) with step u_step (every gridDim-th
    // unit, or with REUSE a contiguous range)
    const int per = REUSE ? p.units / (int)gridDim.x : 0, rem = REUSE ? p.units % (int)gridDim.x : 0;
    const int u_begin = REUSE ? (int)blockIdx.x * per + ((int)blockIdx.x < rem ? (int)blockIdx.x : rem)
                              : (int)blockIdx.x;
    const int u_end = REUSE ? u_begin + per + ((int)blockIdx.x < rem ? 1 : 0) : p.units;
    const int u_step = REUSE ? 1 : (int)gridDim.x;
    // the reverse state entering the last tile is zero (no given reverse start
    // state): it is neither stored nor loaded, C_b H_b is not formed and the
    // output leaves its term out
    const bool rzero = MODE == kModeBidir || p.rinit == nullptr;
    auto hb_zero = [&](int i) { return kOut && rzero && i == nt - 1; };
    // C/B reuse: unit u's output tile takes the previous unit's C/B tiles
    auto same_bc = [&](int u) {
        if constexpr (!REUSE || !kOut) return false;
        return u > u_begin && u < u_end && (u - 1) / p.H == u / p.H && ((u - 1) % p.H) / hpg == (u % p.H) / hpg;
    };
    const size_t dt_dir = (size_t)p.batch * p.L * p.H;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
            // kr, kx, kh count the loads issued; each is issued only once its
            // slot is free, so at most one load per barrier is ever in flight
            uint32_t kr = 0, kx = 0, kh = 0;
            uint32_t units_done = 0;
            auto ring_slot = [&](uint32_t &s) -> bool {
                s = kr % kRing;
                return kr < kRing ||
                       mbar_wait(bar(B_RING_EMPTY + s), ((kr / kRing) - 1) & 1, abort_flag, p.status, 101);
            };
            auto x_slot = [&](uint32_t &s) -> bool {
                s = kx % kXS;
                return kx < kXS || mbar_wait(bar(B_X_EMPTY + s), ((kx / kXS) - 1) & 1, abort_flag, p.status, 102);
            };
            // the state pass's x and B are read once in the state mode; otherwise
            // the output pass reads them again from L2
            const uint64_t pol1 = kOut ? keep : stream;
            // after an expired wait anywhere in the CTA, no further loads are issued
            bool ok = true;
            for (int u = u_begin; ok && u < u_end; u += u_step, ++units_done) {
                const int b = u / p.H, h = u % p.H, gg = h / hpg;
                for (int k1 = 0; ok && k1 < n1t; ++k1) {    // phase 1: x, B of the state pass
                    const int i = kFwd1 ? k1 : nt - 1 - k1;
                    uint32_t xs, rs;
                    if (!(ok = x_slot(xs))) break;
                    ++kx;
                    mbar_arrive_expect_tx(bar(B_X_FULL + xs), kSlab);
                    tma_load_4d_hint(base + S::xslot(xs), &tm_x, bar(B_X_FULL + xs), 0, h, i * kTile, b, pol1);
                    if (!(ok = ring_slot(rs))) break;
                    ++kr;
                    mbar_arrive_expect_tx(bar(B_RING_FULL + rs), S::kBC);
                    for (int k = 0; k < NSLAB; ++k)
                        tma_load_5d_hint(base + S::ring + rs * 2 * kSlab + k * kSlab, &tm_b, bar(B_RING_FULL + rs),
                                         64 * k, gg, i * kTile, b, kFwd1 ? 0 : 1, pol1);
                }
                if (!ok) break;
                for (int i = 0; kOut && ok && i < nt; ++i) {        // phase 2: x, C_f, B_f, C_b, B_b, H_b
                    const int t0 = i * kTile;
                    uint32_t xs;
                    if (!(ok = x_slot(xs))) break;
                    ++kx;
                    mbar_arrive_expect_tx(bar(B_X_FULL + xs), kSlab);
                    tma_load_4d_hint(base + S::xslot(xs), &tm_x, bar(B_X_FULL + xs), 0, h, t0, b, stream);
                    const CUtensorMap *maps[4] = {&tm_c, &tm_b, &tm_c, &tm_b};
                    const int dirs[4] = {0, 0, 1, 1};
                    for (int j = 0; ok && !same_bc(u) && j < 4; ++j) {
                        uint32_t rs;
                        if (!(ok = ring_slot(rs))) break;
                        ++kr;
                        mbar_arrive_expect_tx(bar(B_RING_FULL + rs), S::kBC);
                        for (int k = 0; k < NSLAB; ++k)
                            tma_load_5d_hint(base + S::ring + rs * 2 * kSlab + k * kSlab, maps[j],
                                             bar(B_RING_FULL + rs), 64 * k, gg, t0, b, dirs[j], stream);
                    }
                    if (!ok) break;
                    // the unit's reverse states are in global memory once group C is
                    // past its reverse chain; the x and B/C loads above go out before
                    if (i == 0 && !(ok = mbar_wait(bar(B_HB_WRITTEN), units_done & 1, abort_flag, p.status, 103)))
                        break;
                    if (kh >= 1 && !(ok = mbar_wait(bar(B_HB_EMPTY), (kh - 1) & 1, abort_flag, p.status, 104))) break;
                    ++kh;
                    if (hb_zero(i)) {
                        mbar_arrive(bar(B_HB_FULL));   // nothing to load: C_b H_b is not formed
                    } else {
                        mbar_arrive_expect_tx(bar(B_HB_FULL), S::kH);
                        tma_load_3d_hint(base + S::hb, &tm_h, bar(B_HB_FULL), 0, 0, u * nt + i, stream);
                    }
                }
            }
            // every load issued has landed before the CTA may exit (waited on only
            // after an expired wait, when consumers may have stopped waiting)
            for (uint32_t k = kr > kRing ? kr - kRing : 0; k < kr; ++k)
                mbar_drain(bar(B_RING_FULL + k % kRing), (k / kRing) & 1);
            for (uint32_t k = kx > kXS ? kx - kXS : 0; k < kx; ++k) mbar_drain(bar(B_X_FULL + k % kXS), (k / kXS) & 1);
            if (kh >= 1) mbar_drain(bar(B_HB_FULL), (kh - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_state = idesc_bf16_f32(128, 64, true, true);   // B^T (MN) x X' (MN)
            constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, false);    // C (K) x B (K)
            constexpr uint32_t id_o = idesc_bf16_f32(128, 64, false, true);      // C (K) x H (MN); M (K) x X (MN)
            uint32_t kr = 0, kx = 0, kh = 0, n1 = 0;
            uint32_t n_m = 0, n_sfree = 0, n_yfree = 0, n_hbw = 0;
            bool first2 = true;
            auto wait_ring = [&](uint32_t k) -> uint32_t {
                const uint32_t s = k % kRing;
                mbar_wait(bar(B_RING_FULL + s), (k / kRing) & 1, abort_flag, p.status, 201);
                return s;
            };
            auto slot_addr = [&](uint32_t s) { return base + S::ring + s * 2 * kSlab; };
            // after an expired wait anywhere in the CTA, no further tiles are issued
            uint32_t rCf = 0, rBf = 0, rCb = 0, rBb = 0;   // the output tile's ring slots
            for (int u = u_begin; u < u_end && !*abort_flag; u += u_step) {
                const bool reuse = same_bc(u), keep_bc = same_bc(u + u_step);
                for (int k1 = 0; k1 < n1t && !*abort_flag; ++k1, ++n1) {  // phase 1: S = B^T (diag(w) X in the x slot)
                    const uint32_t n = kx++, xs = n % kXS;
                    const uint32_t rs = wait_ring(kr++);
                    mbar_wait(bar(B_XW_READY + xs), (n / kXS) & 1, abort_flag, p.status, 202);
                    const uint32_t pb = n1 & 1;
                    if (n1 >= 2) mbar_wait(bar(B_P1S_FREE + pb), ((n1 >> 1) - 1) & 1, abort_flag, p.status, 203);
                    tc_fence_after();
                    const uint32_t sB = slot_addr(rs), sX = base + S::xslot(xs);
                    for (int k = 0; k < kTile / 16; ++k)
                        mma_bf16_ss(tGf + 64 * pb, sdesc_sw128(sB + k * 2048, kSlab, 1024),
                                    sdesc_sw128(sX + k * 2048, kSlab, 1024), id_state, k > 0);
                    if constexpr (!kOut) {   // state mode: plus B^T (low part of diag(w) X)
                        const uint32_t sL = base + S::loslot(xs);
                        for (int k = 0; k < kTile / 16; ++k)
                            mma_bf16_ss(tGf + 64 * pb, sdesc_sw128(sB + k * 2048, kSlab, 1024),
                                        sdesc_sw128(sL + k * 2048, kSlab, 1024), id_state, 1);
                    }
                    mma_commit(bar(B_P1S_READY + pb));
                    mma_commit(bar(B_RING_EMPTY + rs));
                    mma_commit(bar(B_X_EMPTY + xs));
                }
                for (int i = 0; kOut && i < nt && !*abort_flag; ++i) {   // phase 2
                    const uint32_t n = kx++, xs = n % kXS;
                    if (!reuse) {
                        rCf = wait_ring(kr++);
                        rBf = wait_ring(kr++);
                        rCb = wait_ring(kr++);
                        rBb = wait_ring(kr++);
                    }
                    const uint32_t sCf = slot_addr(rCf), sBf = slot_addr(rBf);
                    const uint32_t sCb = slot_addr(rCb), sBb = slot_addr(rBb);
                    // G_f overwrites the reverse pass's TMEM tile states and Y_o,f reads
                    // H_f: the unit's first output tile waits until group C is done with
                    // the former and has zeroed (or seeded) the latter
                    if (i == 0) mbar_wait(bar(B_HB_WRITTEN), n_hbw++ & 1, abort_flag, p.status, 210);
                    tc_fence_after();
                    // G_f = C_f B_f^T, G_b = C_b B_b^T (earlier readers of these TMEM
                    // columns are MMAs issued before, which complete in order)
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                        mma_bf16_ss(tGf, sdesc_sw128(sCf + ko, 0, 1024), sdesc_sw128(sBf + ko, 0, 1024), id_g, k > 0);
                    }
                    for (int k = 0; k < N / 16; ++k) {
                        const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                        mma_bf16_ss(tGb, sdesc_sw128(sCb + ko, 0, 1024), sdesc_sw128(sBb + ko, 0, 1024), id_g, k > 0);
                    }
                    mma_commit(bar(B_G_READY));
                    if (!keep_bc) mma_commit(bar(B_RING_EMPTY + rBb));
                    // the previous tile's outputs and state are consumed; H_f is this tile's
                    if (!first2) {
                        mbar_wait(bar(B_Y_FREE), n_yfree++ & 1, abort_flag, p.status, 205);
                        mbar_wait(bar(B_S_FREE), n_sfree++ & 1, abort_flag, p.status, 206);
                    }
                    first2 = false;
                    tc_fence_after();
                    for (int k = 0; k < N / 16; ++k) {      // Yo_f = C_f H_f
                        const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                        mma_bf16_ss(tYof, sdesc_sw128(sCf + ko, 0, 1024),
                                    sdesc_sw128(base + S::hf + k * 2048, kSlab, 1024), id_o, k > 0);
                    }
                    if (!keep_bc) mma_commit(bar(B_RING_EMPTY + rCf));
                    mbar_wait(bar(B_HB_FULL), kh++ & 1, abort_flag, p.status, 207);
                    tc_fence_after();
                    for (int k = 0; !hb_zero(i) && k < N / 16; ++k) {      // Yo_b = C_b H_b
                        const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                        mma_bf16_ss(tYob, sdesc_sw128(sCb + ko, 0, 1024),
                                    sdesc_sw128(base + S::hb + k * 2048, kSlab, 1024), id_o, k > 0);
                    }
                    if (!keep_bc) mma_commit(bar(B_RING_EMPTY + rCb));
                    mma_commit(bar(B_HB_EMPTY));
                    mbar_wait(bar(B_XW_READY + xs), (n / kXS) & 1, abort_flag, p.status, 208);
                    tc_fence_after();
                    for (int k = 0; k < kTile / 16; ++k)    // S_f = B_f^T diag(w_f) X
                        mma_bf16_ss(tS, sdesc_sw128(sBf + k * 2048, kSlab, 1024),
                                    sdesc_sw128(base + S::xw + k * 2048, kSlab, 1024), id_state, k > 0);
                    mma_commit(bar(B_S_READY));
                    if (!keep_bc) mma_commit(bar(B_RING_EMPTY + rBf));
                    mbar_wait(bar(B_M_READY), n_m++ & 1, abort_flag, p.status, 209);
                    mbar_wait(bar(B_X_FULL + xs), (n / kXS) & 1, abort_flag, p.status, 204);
                    tc_fence_after();
                    const uint32_t sX = base + S::xslot(xs);
                    for (int k = 0; k < kTile / 16; ++k)    // Yd = M X, M from TMEM
                        mma_bf16_ts(tYd, tGf + 16 * k, sdesc_sw128(sX + k * 2048, kSlab, 1024), id_o, k > 0);
                    mma_commit(bar(B_Y_READY));
                }
            }
            // all MMAs complete before TMEM is released
            mma_commit(bar(B_MMA_DONE));
            mbar_drain(bar(B_MMA_DONE), 0);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ group C
        const int row = ((warp & 3) << 5) | lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
        const uint64_t keep = policy_evict_last();
        uint32_t kx = 0, n_s = 0, nvec = 0, n1 = 0;
        float hreg[kP];
        // hreg <- a given start state of unit u (row n of the (64, N) state,
        // transposed: hreg[p] = state[p][n]) or zero
        auto start_state = [&](int u, const float *given) {
            if (given && row < N) {
                const float *ip = given + (size_t)u * kP * N + row;
#pragma unroll
                for (int j = 0; j < kP; ++j) hreg[j] = ip[(size_t)j * N];
            } else {
#pragma unroll
                for (int j = 0; j < kP; ++j) hreg[j] = 0.f;
            }
        };
        // dt of the next output-pass tile is fetched a tile ahead (volatile
        // loads, so the compiler keeps them a tile early)
        uint32_t rawf = 0, rawb = 0;
        bool dt_valid = false;          // DTRAW: the token of rawf / rawb lies in the sequence
        auto load_dt = [&](int u, int i) {
            rawf = 0;
            rawb = 0;
            dt_valid = false;
            if (u >= u_end) return;
            const int b = u / p.H, h = u % p.H, t = i * kTile + row;
            if (t < p.L) {
                dt_valid = true;
                const size_t o = ((size_t)b * p.L + t) * p.H + h;
                asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(rawb) : "l"(p.dt + dt_dir + o));
                asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(rawf) : "l"(p.dt + o));
            }
        };
        auto take_dt = [&](float &vf, float &vb, int h) {
            vf = __uint_as_float(rawf << 16);
            vb = __uint_as_float(rawb << 16);
            if constexpr (DTRAW) {
                vf = dt_valid ? dt_from_raw(vf, p.dt_bias[h], p.dt_lo, p.dt_hi) : 0.f;
                vb = dt_valid ? dt_from_raw(vb, p.dt_bias[p.H + h], p.dt_lo, p.dt_hi) : 0.f;
            }
        };
        int cu = u_begin, ci = 0;   // the output-pass tile whose dt is in flight
        if constexpr (kOut) load_dt(cu, ci);
        while (cu < u_end) {
            const int u = cu;
            const int h = u % p.H;
            const float *Au = layer_ptr(p.A, p, u);
            const float Af = Au[h], Ab = kOut ? Au[p.H + h] : 0.f;
            // ---------------- phase 1: the state chain (reverse, right to left; in
            // the state mode forward, from the given state). Groups A and B prepare
            // the tiles (diag(w) X, tile decay); this group stores the reverse
            // state entering each tile (output modes) and folds the tile's state in.
            start_state(u, kFwd1 ? p.init : (MODE == kModeBidirInit ? p.rinit : nullptr));
            float lsum = 0.f;               // state modes: log of the sequence's decay, from the tile decays
            for (int k1 = 0; k1 < nt; ++k1) {
                const int i = kFwd1 ? k1 : nt - 1 - k1;
                if (kOut && row < N && !hb_zero(i)) {
                    __nv_bfloat16 *dst = p.hb + (((size_t)u * nt + i) * N + row) * kP;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        uint4 v = make_uint4(pack_bf16x2(hreg[8 * c], hreg[8 * c + 1]),
                                             pack_bf16x2(hreg[8 * c + 2], hreg[8 * c + 3]),
                                             pack_bf16x2(hreg[8 * c + 4], hreg[8 * c + 5]),
                                             pack_bf16x2(hreg[8 * c + 6], hreg[8 * c + 7]));
                        st_global_v4_hint(dst + 8 * c, v, keep);
                    }
                }
                if (k1 == n1t) break;        // reverse: tile 0's own state is not needed
                const uint32_t pbuf = n1 & 1;
                mbar_wait(bar(B_G1_READY + n1 % kG1), (n1 / kG1) & 1, abort_flag, p.status, 303);
                const float gdec = gdec1[n1 % kG1];
                if (!kOut) lsum += __logf(gdec);   // -inf once a tile decays to 0: the product is 0 then
                mbar_wait(bar(B_P1S_READY + pbuf), (n1 >> 1) & 1, abort_flag, p.status, 301);
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t v[32];
                    tmem_ld32(tGf + 64 * pbuf + lane_off + half * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        hreg[half * 32 + j] = fmaf(gdec, hreg[half * 32 + j], __uint_as_float(v[j]));
                }
                tc_fence_before();
                sync_c();
                if (row == 0) mbar_arrive(bar(B_P1S_FREE + pbuf));
                ++n1;
            }
            if constexpr (!kOut) {
                // the state mode's result: the forward state after the last tile
                if (row < N) {
                    float *op = p.state_out + (size_t)u * kP * N + row;
#pragma unroll
                    for (int j = 0; j < kP; ++j) op[(size_t)j * N] = hreg[j];
                }
                if (row == 0 && p.decay_out) p.decay_out[u] = __expf(lsum);
                cu += u_step;
                continue;
            }
            kx += n1t;       // the reverse pass's x loads and diag(w') X releases belong to groups A and B
            // phase 2 starts from H_f = 0 (the init mode: from the given state); the
            // reverse states go to the TMA proxy
            start_state(u, MODE == kModeBidirInit ? p.init : nullptr);
            if (row < N) {
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(g + S::hf + sw128_offset(row, c)) =
                        make_uint4(pack_bf16x2(hreg[8 * c], hreg[8 * c + 1]), pack_bf16x2(hreg[8 * c + 2], hreg[8 * c + 3]),
                                   pack_bf16x2(hreg[8 * c + 4], hreg[8 * c + 5]), pack_bf16x2(hreg[8 * c + 6], hreg[8 * c + 7]));
            }
            fence_proxy_async_smem();
            fence_proxy_async_global();
            sync_c();
            if (row == 0) mbar_arrive(bar(B_HB_WRITTEN));
            // ---------------- phase 2: decay sums, vectors, diag(w_f) X, forward chain
            for (int i = 0; i < nt; ++i) {
                float vf, vb;
                take_dt(vf, vb, h);
                if (++ci == nt) { ci = 0; cu += u_step; }
                load_dt(cu, ci);
                float pf = vf, pb = vb, totf, totb;
                scan2(pf, pb, totf, totb, row, red);
                const float csb = totb - pb + vb;
                const float my_af = Af * pf, my_ab = Ab * csb;
                const uint32_t vb_i = nvec & 1;
                if (nvec >= 2) mbar_wait(bar(B_VEC_FREE + vb_i), ((nvec >> 1) - 1) & 1, abort_flag, p.status, 311);
                TileVec &V = vec[vb_i];
                V.af[row] = my_af;
                V.ab[row] = my_ab;
                V.dtf[row] = vf;
                V.dtb[row] = vb;
                if (row == 0) {
                    V.totf = totf;
                    V.totb = totb;
                }
                sync_c();
                mask_column_factors(row, my_af, my_ab, vf, vb, V.af, V.ab, V.colf, V.colb);
                sync_c();
                if (row == 0) mbar_arrive(bar(B_VEC_READY + vb_i));
                ++nvec;
                // diag(w_f) X into the X' buffer (the previous state MMA, which read
                // it, completed before this group's last state step)
                const float wf = __expf(Af * (totf - pf)) * vf;   // exp(A sum_{r>s} dt) dt_s
                const uint32_t nx = kx++, xs = nx % kXS;
                mbar_wait(bar(B_X_FULL + xs), (nx / kXS) & 1, abort_flag, p.status, 312);
                scale_row(g + S::xslot(xs), g + S::xw, row, wf);
                fence_proxy_async_smem();
                sync_c();
                if (row == 0) mbar_arrive(bar(B_XW_READY + xs));
                // forward chain: H_f <- exp(A sum dt) H_f + S_f; bf16 copy for C_f.H_f
                const float gdec = __expf(Af * totf);
                mbar_wait(bar(B_S_READY), n_s++ & 1, abort_flag, p.status, 313);
                tc_fence_after();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t v[32];
                    tmem_ld32(tS + lane_off + half * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        hreg[half * 32 + j] = fmaf(gdec, hreg[half * 32 + j], __uint_as_float(v[j]));
                }
                if (row < N) {
                    uint8_t *hrow = g + S::hf;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(hrow + sw128_offset(row, c)) =
                            make_uint4(pack_bf16x2(hreg[8 * c], hreg[8 * c + 1]),
                                       pack_bf16x2(hreg[8 * c + 2], hreg[8 * c + 3]),
                                       pack_bf16x2(hreg[8 * c + 4], hreg[8 * c + 5]),
                                       pack_bf16x2(hreg[8 * c + 6], hreg[8 * c + 7]));
                }
                fence_proxy_async_smem();
                tc_fence_before();
                sync_c();
                if (row == 0) mbar_arrive(bar(B_S_FREE));
            }
        }
    } else {
        // ------------------------------------------------------------ groups A and B
        const bool is_b = warp >= 10;
        const int row = ((warp & 3) << 5) | lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
        const int c0 = is_b ? 16 : 0;       // which half of each 32-column block, and of the output
        auto sync_g = [&]() { if (is_b) sync_b(); else sync_a(); };
        auto sync_ab = [&]() { asm volatile("bar.sync 4, 256;" ::: "memory"); };
        uint32_t kx = 0, n_g = 0, n_y = 0, nvec = 0, m1 = 0;
        float *red_g = red_ab + (is_b ? 4 : 0);
        for (int u = u_begin; u < u_end; u += u_step) {
            const int b = u / p.H, h = u % p.H;
            const float *Au = layer_ptr(p.A, p, u), *Du = layer_ptr(p.D, p, u);
            const float dsum = kOut ? Du[h] + Du[p.H + h] : 0.f;
            // the state pass's direction: reverse in the output modes, forward in the state mode
            const float A1 = kFwd1 ? Au[h] : Au[p.H + h];
            const size_t dt1 = kFwd1 ? 0 : dt_dir;
            // ---------------- phase 1: every other state-pass tile (by the CTA's
            // running tile count m1: group A the even ones, group B the odd ones):
            // w_s = exp(A sum dt_r) dt_s over the rest of the tile in the pass's
            // direction (reverse: r < s, forward: r > s), diag(w) X in place in
            // the x slot, and the tile decay exp(A sum dt) for group C's chain.
            uint32_t rawn = 0;               // dt of this group's next tile, fetched a tile ahead
            bool rawn_valid = false;         // its token lies in the sequence
            bool have = false;
            // DTRAW: the state pass's step size from the raw projection
            const float bias1 = DTRAW ? p.dt_bias[kFwd1 ? h : p.H + h] : 0.f;
            auto dt1_of = [&](float raw) { return DTRAW ? dt_from_raw(raw, bias1, p.dt_lo, p.dt_hi) : raw; };
            for (int k1 = 0; k1 < n1t; ++k1, ++m1, ++kx) {
                if ((m1 & 1) != (uint32_t)is_b) continue;
                const int i = kFwd1 ? k1 : nt - 1 - k1;
                float vb = 0.f;
                if (have) {
                    if (rawn_valid) vb = dt1_of(bf2f(rawn));
                } else {
                    const int t = i * kTile + row;
                    if (t < p.L) vb = dt1_of(__bfloat162float(p.dt[dt1 + ((size_t)b * p.L + t) * p.H + h]));
                }
                have = k1 + 2 < n1t;         // this group's next tile, two on in the pass's order
                rawn = 0;
                rawn_valid = false;
                if (have) {
                    const int t = (kFwd1 ? i + 2 : i - 2) * kTile + row;
                    if (t < p.L) {
                        rawn_valid = true;
                        const size_t o = dt1 + ((size_t)b * p.L + t) * p.H + h;
                        asm volatile("ld.global.nc.u16 %0, [%1];" : "=r"(rawn) : "l"(p.dt + o));
                    }
                }
                float pb = vb, tot;
                scan1(pb, tot, row, red_g, sync_g);          // pb: inclusive prefix sum
                const float w = __expf(A1 * (kFwd1 ? tot - pb : pb - vb)) * vb;
                const uint32_t xs = kx % kXS;
                mbar_wait(bar(B_X_FULL + xs), (kx / kXS) & 1, abort_flag, p.status, 404);
                uint8_t *xt = g + S::xslot(xs);
                if constexpr (kOut) scale_row(xt, xt, row, w);
                else scale_row_split(xt, g + S::loslot(xs), row, w);   // the state is a result: 16 bits of w x
                fence_proxy_async_smem();
                if (row == 0) gdec1[m1 % kG1] = __expf(A1 * tot);
                sync_g();
                if (row == 0) {
                    mbar_arrive(bar(B_XW_READY + xs));
                    mbar_arrive(bar(B_G1_READY + m1 % kG1));
                }
            }
            // ---------------- phase 2: masked matrix halves and output halves
            for (int i = 0; kOut && i < nt; ++i) {
                const int t0 = i * kTile;
                const uint32_t vb_i = nvec & 1;
                mbar_wait(bar(B_VEC_READY + vb_i), (nvec >> 1) & 1, abort_flag, p.status, 401);
                const TileVec &V = vec[vb_i];
                const float my_af = V.af[row], my_ab = V.ab[row];
                mbar_wait(bar(B_G_READY), n_g++ & 1, abort_flag, p.status, 402);
                tc_fence_after();
                {
                    const MaskVectors mv{V.af, V.ab, V.dtf, V.dtb, V.colf, V.colb};
                    const int wq = warp & 3;        // this warp's row block
#pragma unroll 1
                    for (int J = 0; J < 4; ++J) {
                        uint32_t packed[8];
                        if (J != wq) {              // one direction: only its G is read
                            uint32_t g[16];
                            tmem_ld16((J < wq ? tGf : tGb) + lane_off + J * 32 + c0, g);
                            tmem_wait_ld();
                            mask_offdiag<16>(J, c0, row, my_af, my_ab, g, mv, packed);
                        } else {
                            uint32_t gf[16], gb[16];
                            tmem_ld16(tGf + lane_off + J * 32 + c0, gf);
                            tmem_ld16(tGb + lane_off + J * 32 + c0, gb);
                            tmem_wait_ld();
                            mask_diag<16>(J, c0, row, my_af, my_ab, gf, gb, mv, packed);
                        }
                        tmem_st8(tGf + lane_off + J * 32 + c0, packed);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                sync_g();
                if (row == 0) {
                    mbar_arrive(bar(B_M_READY));
                    mbar_arrive(bar(B_VEC_FREE + vb_i));
                }
                ++nvec;
                const uint32_t xs = kx++ % kXS;
                // output columns [2 c0, 2 c0 + 32) of the tile over the x slot
                // (group A the first half, group B the second), then one TMA store
                mbar_wait(bar(B_Y_READY), n_y++ & 1, abort_flag, p.status, 403);
                tc_fence_after();
                const float ef = __expf(my_af), eb = __expf(my_ab);
                uint8_t *xt = g + S::xslot(xs);
                const int q0 = c0 >> 3;              // 0 or 2: first 16-column quarter
#pragma unroll 1
                for (int q = q0; q < q0 + 2; ++q) {
                    uint32_t yd[16], yf[16], yb[16];
                    tmem_ld16(tYd + lane_off + q * 16, yd);
                    tmem_ld16(tYof + lane_off + q * 16, yf);
                    if (hb_zero(i)) {   // warp-uniform: the tile has no C_b H_b term
#pragma unroll
                        for (int j = 0; j < 16; ++j) yb[j] = 0u;
                    } else {
                        tmem_ld16(tYob + lane_off + q * 16, yb);
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint4 *qp = reinterpret_cast<uint4 *>(xt + sw128_offset(row, q * 2 + c));
                        uint4 xv = *qp;
                        uint32_t *xu = reinterpret_cast<uint32_t *>(&xv);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i0 = c * 8 + 2 * e;
                            const float y0 = __uint_as_float(yd[i0]) + ef * __uint_as_float(yf[i0]) +
                                             eb * __uint_as_float(yb[i0]) + dsum * bf2f(xu[e] & 0xffffu);
                            const float y1 = __uint_as_float(yd[i0 + 1]) + ef * __uint_as_float(yf[i0 + 1]) +
                                             eb * __uint_as_float(yb[i0 + 1]) + dsum * bf2f(xu[e] >> 16);
                            xu[e] = pack_bf16x2(y0, y1);
                        }
                        *qp = xv;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                sync_ab();
                if (is_b && row == 0) {
                    mbar_arrive(bar(B_Y_FREE));
                    if (!*abort_flag) {
                        tma_store_4d(&tm_out, base + S::xslot(xs), 0, h, t0, b);
                        tma_store_commit();
                    }
                    tma_store_wait_read();      // the store has read the slot
                    mbar_arrive(bar(B_X_EMPTY + xs));
                }
            }
        }
        if (is_b && row == 0) tma_store_wait_all();
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

template <int N, int MODE, bool REUSE, bool DTRAW>
cudaError_t run_fused(const TcArgs &a, cudaStream_t stream) {
    using S = Smem<N>;
    constexpr bool kOut = MODE == kModeBidir || MODE == kModeBidirInit;
    const int nt = (a.L + kTile - 1) / kTile;
    const int units = a.batch * a.H;
    if (a.ws_bytes < kStatusBytes + (kOut ? tc_fused_scratch_bytes(a.batch, a.L, a.H, N) : 0))
        return cudaErrorInvalidValue;
    if (!kOut && !a.state_out) return cudaErrorInvalidValue;
    FusedParams p{};
    p.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    p.A = a.A;
    p.D = a.D;
    p.hb = kOut ? reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(a.workspace) + kStatusBytes) : nullptr;
    p.init = a.init;
    p.rinit = a.rinit;
    p.state_out = a.state_out;
    p.decay_out = a.decay_out;
    p.status = static_cast<DeviceStatus *>(a.workspace);
    p.batch = a.batch; p.L = a.L; p.H = a.H; p.G = a.G; p.nt = nt; p.units = units;
    p.dt_bias = a.dt_bias;
    p.dt_lo = a.dt_lo;
    p.dt_hi = a.dt_hi;
    p.layer_units = a.layer_units;
    p.A_layer = a.A_layer;
    p.launch_order = a.launch_order;

    CUtensorMap tm_x, tm_b, tm_c, tm_h, tm_out;
    // the forward state mode may be given single-direction B; every other mode reads both directions' layout
    if (!tmap::map_x(&tm_x, a.x, a.batch, a.L, a.H) ||
        !tmap::map_bc(&tm_b, a.B, MODE == kModeState ? 1 : 2, a.batch, a.L, a.G, N))
        return cudaErrorInvalidValue;
    if (kOut) {
        if (!tmap::map_bc(&tm_c, a.C, 2, a.batch, a.L, a.G, N) ||
            !tmap::map_h(&tm_h, p.hb, (long long)units * nt, N) || !tmap::map_x(&tm_out, a.out, a.batch, a.L, a.H))
            return cudaErrorInvalidValue;
    } else {
        tm_c = tm_h = tm_out = tm_x;   // not read in the state mode
    }
    int dev = 0, sms = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    auto k = tc_fused_kernel<N, MODE, REUSE, DTRAW>;
    const size_t smem = S::bytes + 1024;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    int grid = units < sms ? units : sms;
    if (a.grid_cap > 0 && grid > a.grid_cap) grid = a.grid_cap;
    // programmatic stream serialization: the prologue (barriers, TMEM) overlaps
    // the end of the kernel ahead; the kernel waits for it before any global access
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, tm_x, tm_b, tm_c, tm_h, tm_out, p);
}

template <int MODE, bool DTRAW = false>
cudaError_t launch_mode(const TcArgs &a, cudaStream_t stream) {
    if (a.L <= 0 || a.batch <= 0) return cudaErrorNotSupported;
    if (a.N != 64 && a.N != 128) return cudaErrorNotSupported;
    if (!tmap::encode_fn()) return cudaErrorNotSupported;
    const long long entries = (long long)a.batch * a.H * ((a.L + kTile - 1) / kTile);
    if (entries >= (1ll << 31)) return cudaErrorNotSupported;
    constexpr bool kOut = MODE == kModeBidir || MODE == kModeBidirInit;
    // one-tile sequences with B/C shared by several heads: consecutive heads on
    // one CTA, taking their C/B tiles from the ring in place
    if (kOut && a.L <= kTile && a.G < a.H)
        return a.N == 64 ? run_fused<64, MODE, kOut, DTRAW>(a, stream) : run_fused<128, MODE, kOut, DTRAW>(a, stream);
    return a.N == 64 ? run_fused<64, MODE, false, DTRAW>(a, stream) : run_fused<128, MODE, false, DTRAW>(a, stream);
}

}  // namespace

size_t tc_fused_scratch_bytes(int batch, int L, int H, int N) {
    const size_t nt = (size_t)(L + kTile - 1) / kTile;
    return align256((size_t)batch * H * nt * N * kP * 2);
}

bool tc_fused_supported(int batch, int L, int H, int G, int N) {
    (void)G;
    if (L <= 0 || batch <= 0) return false;
    if (N != 64 && N != 128) return false;
    // one unit per CTA at a time: worthwhile when the units fill the GPU
    if ((long long)batch * H < 148) return false;
    const long long entries = (long long)batch * H * ((L + kTile - 1) / kTile);
    return entries < (1ll << 31);
}

cudaError_t launch_tc_fused(const TcArgs &a, cudaStream_t stream) {
    return a.init || a.rinit ? launch_mode<kModeBidirInit>(a, stream) : launch_mode<kModeBidir>(a, stream);
}

cudaError_t launch_tc_fused_dtraw(const TcArgs &a, cudaStream_t stream) {
    if (!a.dt_bias || a.init || a.rinit) return cudaErrorNotSupported;
    return launch_mode<kModeBidir, true>(a, stream);
}

cudaError_t launch_tc_fused_state(const TcArgs &a, cudaStream_t stream) {
    return launch_mode<kModeState>(a, stream);
}

cudaError_t launch_tc_fused_state_rev(const TcArgs &a, cudaStream_t stream) {
    return launch_mode<kModeStateRev>(a, stream);
}

}  // namespace ssd
