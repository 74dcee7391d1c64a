// One-tile bidirectional SSD kernel for sm_100a: sequences of at most 128
// tokens, where both scans of a (batch, head) fit in one tensor-core tile and
// there is no state to carry.
//
// For a sequence that short the whole mixer is one masked product,
//   y = (M_f + M_b) X + (D_f + D_b) x,
//   M_f[t][s] = G_f[t][s] exp(a_t - a_s) dt_f[s] (s <= t),
//   M_b[t][s] = G_b[t][s] exp(a'_t - a'_s) dt_b[s] (s >= t),
// with G = C B^T of each direction. G depends only on the B/C group, not on
// the head, so the kernel takes one (batch, B/C group) at a time, forms G_f
// and G_b once on the tensor cores (TMEM, fp32), and then, for each head of
// the group, builds the head's mask from G and its own decays (bf16, in
// TMEM), runs Y = M X and writes y. With B/C shared by all heads (Mamba-2's
// ngroups = 1) the 24 heads of a batch element share two G tiles.
// The two scans, added: "DiffuMamba: High-Throughput Diffusion LMs with Mamba
// Backbone", Technical Summary, 2. Methodology, Core Architecture; the
// packed 128-token shape: "Diffusion Mamba ... (LM1B, packed sequences of
// 128)" as the pages' second workload.
//
// Per CTA: 256 threads, persistent over work units (a batch element, a B/C
// group and a run of its heads). Thread 0 issues the TMA loads and the MMAs;
// warp w owns TMEM lanes 32 (w % 4) .. + 31 (tile rows) and the 32-column
// blocks w / 4 and w / 4 + 2 of the mask, and 32 of the 64 output columns.
// The next unit's C and B load while the current unit's heads run; each
// head's x loads while the head before it runs. Every wait is bounded in
// time; an expired wait sets the workspace's timeout flag and the CTA stores
// nothing.
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
constexpr int kThreads = 256;
constexpr uint32_t kSlab = 16384;   // 128 rows x 128 bytes

struct OneParams {
    const __nv_bfloat16 *dt;    // (2, batch, L, H)
    const float *A;             // (2, H)
    const float *D;             // (2, H)
    DeviceStatus *status;
    long long total;            // batch * H heads, taken in (batch, head) order
    int batch, L, H, G, hpg;    // hpg = H / G heads per B/C group
};

// mbarriers: C and B of a group loaded; G of a group computed; x of a head
// loaded (kXS slots); Y of a head computed (two buffers); all MMAs done
constexpr int kXS = 5;
enum { B_CB = 0, B_G, B_X, B_Y = B_X + kXS, B_END = B_Y + 2, B_COUNT };

template <int N>
struct OSmem {
    static constexpr uint32_t kTile = (N / 64) * kSlab;    // one 128 x N bf16 operand
    static constexpr uint32_t cb = 0;                      // C_f, B_f, C_b, B_b
    static constexpr uint32_t x = 4 * kTile;               // kXS x slots (x in, then y out)
    static constexpr uint32_t vec = x + kXS * kSlab;       // two buffers of af, ab, dtf, dtb, colf, colb
    static constexpr uint32_t small = vec + 2 * 6 * 128 * 4;
    static constexpr uint32_t bytes = small + 128;
};

// Inclusive prefix sum of v over the 128 threads of one direction (four
// warps, named barrier `id`, `part` four floats of shared memory); `total`
// the sum over all of them.
__device__ __forceinline__ float scan128(float v, int lane, int wq, float *part, int id, float &total) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) part[wq] = v;
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
    float before = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (k < wq) before += part[k];
    total = part[0] + part[1] + part[2] + part[3];
    return v + before;
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
    float *part = reinterpret_cast<float *>(g + S::small + 96);     // scan partials, four per direction
    static_assert(8 * B_COUNT + 8 <= 96, "barrier area");

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, k2 = warp >> 2;
    const int row = (q << 5) | lane;          // tile row (token t): TMEM lane
    // the decay vectors: threads 0..127 the forward direction of token tid,
    // threads 128..255 the reverse direction of token tid - 128
    const int vdir = tid >> 7, vt = tid & 127;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    // this CTA's heads: [h0, h0 + n) of the (batch, head) list
    const long long h0 = (long long)blockIdx.x * p.total / gridDim.x;
    const int n = (int)((long long)(blockIdx.x + 1) * p.total / gridDim.x - h0);
    const long long key_last = (h0 + n - 1) / p.hpg;   // B/C group of the last head
    auto head_b = [&](int j) { return (int)((h0 + j) / p.H); };
    auto head_h = [&](int j) { return (int)((h0 + j) % p.H); };
    auto head_key = [&](int j) { return (h0 + j) / p.hpg; };   // batch * G + group

    grid_launch_dependents();
    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < B_COUNT; ++i) mbar_init(bar(i), 1);
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
    // TMEM columns: G_f [0,128), G_b [128,256), the masked matrix M [256,384)
    // (bf16: matrix columns [16 k, 16 k + 16) in TMEM columns [16 k, 16 k + 8)),
    // Y of even heads [384,448), of odd heads [448,512)
    const uint32_t tGf = tmem, tGb = tmem + 128, tM = tmem + 256;
    auto tY = [&](int j) { return tmem + 384 + 64 * (j & 1); };
    const uint32_t lane_off = (uint32_t)(q << 5) << 16;
    auto xslot = [&](int j) { return S::x + (uint32_t)(j % kXS) * kSlab; };
    auto vbuf = [&](int j) { return reinterpret_cast<float *>(g + S::vec + (j & 1) * 6 * 512); };
    // the kernel ahead in the stream has finished before any global access
    grid_dependency_wait();

    // thread 0's copies in flight: x loads of heads [x_waited, x_issued), C/B
    // loads of groups [cb_waited, cb_issued)
    int x_issued = 0, x_waited = 0, cb_issued = 0, cb_waited = 0;
    auto load_cb = [&](long long key) {
        const int b = (int)(key / p.G), gg = (int)(key % p.G);
        mbar_arrive_expect_tx(bar(B_CB), 4 * NSLAB * kSlab);
        for (int d = 0; d < 2; ++d)
            for (int sl = 0; sl < NSLAB; ++sl) {
                tma_load_5d(base + S::cb + (2 * d) * S::kTile + sl * kSlab, &tm_c, bar(B_CB), 64 * sl, gg, 0, b, d);
                tma_load_5d(base + S::cb + (2 * d + 1) * S::kTile + sl * kSlab, &tm_b, bar(B_CB), 64 * sl, gg, 0, b,
                            d);
            }
        ++cb_issued;
    };
    auto load_x = [&](int j) {
        mbar_arrive_expect_tx(bar(B_X + j % kXS), kSlab);
        tma_load_4d(base + xslot(j), &tm_x, bar(B_X + j % kXS), 0, head_h(j), 0, head_b(j));
        ++x_issued;
    };
    constexpr uint32_t id_g = idesc_bf16_f32(128, 128, false, false);   // C (K) x B (K)
    constexpr uint32_t id_o = idesc_bf16_f32(128, 64, false, true);     // M (K) x X (MN)
    // G_f = C_f B_f^T and G_b = C_b B_b^T of the group in shared memory
    auto issue_g = [&]() {
        const bool ok = mbar_wait_ool(bar(B_CB), (uint32_t)cb_waited & 1u, abort_flag, p.status, 1001);
        ++cb_waited;
        tc_fence_after();
        if (ok) {
            for (int d = 0; d < 2; ++d) {
                const uint32_t ca = base + S::cb + (2 * d) * S::kTile, ba = ca + S::kTile;
#pragma unroll 1
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t ko = (k >> 2) * kSlab + (k & 3) * 32;
                    mma_bf16_ss(d ? tGb : tGf, sdesc_sw128(ca + ko, 0, 1024), sdesc_sw128(ba + ko, 0, 1024), id_g,
                                k > 0);
                }
            }
        }
        mma_commit(bar(B_G));
    };

    // the per-head vectors of head j into buffer j & 1: the direction's decay
    // sums a (forward: A_f times the sum of dt_f over tokens <= t; reverse:
    // A_b times the sum of dt_b over tokens >= t), dt and the column factors
    // (exp(a_e - a_s) dt_s with e the last (forward) or first (reverse) token
    // of the 32-token block of s)
    auto vectors = [&](int j, float v, float A) {
        float tot;
        const float pf = scan128(v, lane, q, part + 4 * vdir, 1 + vdir, tot);
        const float a = vdir == 0 ? A * pf : A * (tot - pf + v);
        const float edge = __shfl_sync(0xffffffffu, a, vdir == 0 ? 31 : 0);
        float *V = vbuf(j);
        V[vdir * 128 + vt] = a;                          // af, ab
        V[256 + vdir * 128 + vt] = v;                    // dtf, dtb
        V[512 + vdir * 128 + vt] = __expf(edge - a) * v; // colf, colb
    };
    // dt and A of head j for this thread's direction and token
    auto load_dt = [&](int j, float &v, float &A) {
        const int b = head_b(j), h = head_h(j);
        A = __ldg(p.A + vdir * p.H + h);
        v = vt < p.L ? __bfloat162float(p.dt[(((size_t)vdir * p.batch + b) * p.L + vt) * p.H + h]) : 0.f;
    };

    if (tid == 0) {
        load_cb(head_key(0));
        load_x(0);
        if (n > 1) load_x(1);
    }
    {
        float v, A;
        load_dt(0, v, A);
        vectors(0, v, A);
    }
    if (tid == 0) issue_g();
    __syncthreads();

    bool ok = true;              // warp-uniform: every wait of this warp so far succeeded
    int gk = 0;                  // this CTA's group count before the current head
    float ds_prev = 0.f;         // D_f + D_b of head j - 1
    bool failed = false;
#pragma unroll 1
    for (int j = 0; j <= n; ++j) {
        float ds_cur = 0.f;
        if (j < n) {
            // prefetch the next head's dt and A; D of this head
            float v_next = 0.f, A_next = 0.f;
            if (j + 1 < n) load_dt(j + 1, v_next, A_next);
            const int hj = head_h(j);
            ds_cur = __ldg(p.D + hj) + __ldg(p.D + p.H + hj);
            const bool first = j == 0 || head_key(j) != head_key(j - 1);
            if (first) {
                ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_G), (uint32_t)gk & 1u, abort_flag, p.status,
                                                                 1002));
                ++gk;
                // G of this group is in TMEM: C and B of the next group load
                if (tid == 0 && ok && head_key(j) < key_last) load_cb(head_key(j) + 1);
            }
            // ---------------- the masked matrix of head j: row `row`, columns
            // [32 J + 16 k2, 32 J + 16 k2 + 16) of each 32-column block J
            // (M is free once head j - 1's MMA has completed)
            if (j > 0)
                ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_Y + ((j - 1) & 1)), (uint32_t)((j - 1) >> 1) & 1u,
                                                                 abort_flag, p.status, 1003));
            tc_fence_after();
            if (ok) {
                const float *V = vbuf(j);
                const MaskVectors mv{V, V + 128, V + 256, V + 384, V + 512, V + 640};
                const float my_af = V[row], my_ab = V[128 + row];
                const int c0 = 16 * k2;
#pragma unroll 1
                for (int J = 0; J < 4; ++J) {
                    uint32_t packed[8];
                    if (J == q) {
                        uint32_t gf[16], gb[16];
                        tmem_ld16(tGf + lane_off + J * 32 + c0, gf);
                        tmem_ld16(tGb + lane_off + J * 32 + c0, gb);
                        tmem_wait_ld();
                        mask_diag<16>(J, c0, row, my_af, my_ab, gf, gb, mv, packed);
                    } else {
                        uint32_t gv[16];
                        tmem_ld16((J < q ? tGf : tGb) + lane_off + J * 32 + c0, gv);
                        tmem_wait_ld();
                        mask_offdiag<16>(J, c0, row, my_af, my_ab, gv, mv, packed);
                    }
                    tmem_st8(tM + lane_off + J * 32 + c0, packed);
                }
                tmem_wait_st();
            }
            if (j + 1 < n) vectors(j + 1, v_next, A_next);
        }
        tc_fence_before();
        failed = __syncthreads_or(!ok);
        if (failed) break;
        if (tid == 0) {
            tc_fence_after();
            if (j < n) {
                // Y_j = M X_j
                const bool xok = mbar_wait_ool(bar(B_X + j % kXS), (uint32_t)(j / kXS) & 1u, abort_flag, p.status, 1004);
                ++x_waited;
                if (xok && !*abort_flag) {
                    const uint32_t xa = base + xslot(j);
#pragma unroll 1
                    for (int k = 0; k < 128 / 16; ++k)
                        mma_bf16_ts(tY(j), tM + 16 * k, sdesc_sw128(xa + k * 2048, kSlab, 1024), id_o, k > 0);
                }
                mma_commit(bar(B_Y + (j & 1)));
                // the next head starts a new group: its G, once all rows of M_j are built
                if (j + 1 < n && head_key(j + 1) != head_key(j)) issue_g();
            }
            // y of head j - 2 (written over its x in the epilogue of the last iteration)
            if (j >= 2) {
                tma_store_4d(&tm_out, base + xslot(j - 2), 0, head_h(j - 2), 0, head_b(j - 2));
                tma_store_commit();
            }
            // x of head j + 2 into the slot of head j - 3, once its y has left
            if (j + 2 < n) {
                tma_store_wait_read1();
                load_x(j + 2);
            }
        }
        // ---------------- epilogue of head j - 1: y = Y + (D_f + D_b) x, in
        // place of x (row `row`, columns [32 k2, 32 k2 + 32))
        if (j > 0) {
            const int e = j - 1;
            ok = __all_sync(0xffffffffu, ok && mbar_wait_ool(bar(B_Y + (e & 1)), (uint32_t)(e >> 1) & 1u, abort_flag,
                                                             p.status, 1005) &&
                                             mbar_wait_ool(bar(B_X + e % kXS), (uint32_t)(e / kXS) & 1u, abort_flag,
                                                           p.status, 1006));
            tc_fence_after();
            if (ok) {
                uint32_t yv[32];
                tmem_ld32(tY(e) + lane_off + k2 * 32, yv);
                tmem_wait_ld();
                uint8_t *xs = g + xslot(e);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint4 *ptr = reinterpret_cast<uint4 *>(xs + sw128_offset(row, k2 * 4 + cc));
                    const uint4 xv = *ptr;
                    const uint32_t xu[4] = {xv.x, xv.y, xv.z, xv.w};
                    uint32_t o[4];
#pragma unroll
                    for (int j2 = 0; j2 < 4; ++j2) {
                        const int c = cc * 8 + 2 * j2;
                        o[j2] = pack_bf16x2(__uint_as_float(yv[c]) + ds_prev * bf2f(xu[j2] & 0xffffu),
                                            __uint_as_float(yv[c + 1]) + ds_prev * bf2f(xu[j2] >> 16));
                    }
                    *ptr = make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_proxy_async_smem();
            }
        }
        ds_prev = ds_cur;
    }
    // y of the last head
    tc_fence_before();
    failed = __syncthreads_or(failed || !ok);
    if (tid == 0) {
        if (!failed && n >= 1) {
            tma_store_4d(&tm_out, base + xslot(n - 1), 0, head_h(n - 1), 0, head_b(n - 1));
            tma_store_commit();
        }
        // teardown: every MMA, load and store of this CTA has finished before
        // its shared memory and TMEM are released
        mma_commit(bar(B_END));
        mbar_drain(bar(B_END), 0);
        for (int k = x_waited; k < x_issued; ++k) mbar_drain(bar(B_X + k % kXS), (uint32_t)(k / kXS) & 1u);
        for (int k = cb_waited; k < cb_issued; ++k) mbar_drain(bar(B_CB), (uint32_t)k & 1u);
        tma_store_wait_all();
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
