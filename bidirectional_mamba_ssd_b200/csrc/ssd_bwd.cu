// Backward pass of the bidirectional SSD mixer on CUDA cores, fp32 state and
// arithmetic: the gradients of sum(dy * y) with respect to x, dt, A, B, C
// and D ("Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality", Key Results and Technical Contribution: the models are
// trained through the mixer with a full-block objective).
//
// Per (batch, head, direction) item, with a_t = exp(dt_t A), the scan's
// states h_t = a_t h_{t-1} + dt_t B_t x_t^T (N x P) and their adjoints
// g_t = C_t dy_t^T + a_{t'} g_{t'} (t' the token after t in the scan's
// order), one CTA runs
//   1. the scan in its own order, storing every kRun-th state h_t (fp32) to
//      its scratch as a checkpoint and forming dC_t = h_t dy_t on the way;
//   2. the adjoint scan in the opposite order, one run of kRun tokens at a
//      time: the run's states are recomputed from its checkpoint into a
//      kRun-slot buffer (small enough to stay in L2, and each thread reads
//      back only what it wrote), then the run's tokens form
//      dx_t += dt_t B_t^T g_t,  dB_t += dt_t g_t x_t,
//      ddt_t = B_t^T g_t x_t + A a_t <g_t, h_{t-1}>,  dA += dt_t a_t <g_t, h_{t-1}>.
// Each direction's scan may start from a given state (the forward one's
// prefix, the reverse one's suffix: (batch, H, P, N) fp32), which then also
// gets its gradient, the adjoint left after the direction's first token
// (a_first g_first); the block step is the forward scan from a prefix state
// and the reverse scan from zero.
// The skip term adds (D_f + D_b) dy_t to dx (folded into the forward item's
// own contribution, so each dx element receives exactly two fp32 additions,
// whose sum does not depend on their order) and sum_t <dy_t, x_t> to dD of
// both directions.
//
// Layout as the sequential forward scan (ssd_simt.cu): thread (p, q) of 256
// owns column p of the state for the N/4 values of n in quarter q.
// Reductions over n (dx) go through shared memory per staged chunk of
// tokens; reductions over p (dB, dC) use a transposing warp reduction that
// leaves each lane one finished n, then one add across the quarter's two
// warps. The grid is persistent (items loop over CTAs), so scratch is
// ceil(L / kRun) checkpoints plus kRun buffer slots of N x P fp32 per CTA.
#include "ssd_common.cuh"
#include "ssd_kernels.h"

namespace ssd {
namespace {

constexpr int kP = 64;
constexpr int kThreads = 256;
constexpr int kTB = 32;        // tokens staged per round
constexpr int kRun = 8;        // tokens per checkpoint (divides kTB)
static_assert(kTB % kRun == 0, "runs tile the staged rounds");

// Sum of v[j] over the 32 lanes of a warp for NQ values j, transposed: on
// return each lane holds the sum for one index j (transposed_index), and
// 32 / NQ lanes hold each sum. NQ is a power of two, at most 32.
template <int NQ>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[NQ], int lane) {
    // halve the vector each step: keep the half this lane is responsible for
    // and add the partner's copy of it
#pragma unroll
    for (int w = NQ / 2, m = 16; w >= 1; w >>= 1, m >>= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int j = 0; j < w; ++j) {
            const float send = upper ? v[j] : v[j + w];
            const float keep = upper ? v[j + w] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    // the lane bits below the last step's are unused: lanes that differ only
    // there share an index and hold partial sums of disjoint lane sets
    float s = v[0];
#pragma unroll
    for (int m = 1; m < 32 / NQ; m <<= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    return s;
}

// The lanes that write a transposed sum: one per index.
template <int NQ>
__device__ __forceinline__ bool transposed_writer(int lane) { return (lane & (32 / NQ - 1)) == 0; }

// The index j a lane holds after warp_transpose_sum<NQ>: the bits of the
// lane, from the top, pick the upper or lower half at each step.
template <int NQ>
__device__ __forceinline__ int transposed_index(int lane) {
    int j = 0;
#pragma unroll
    for (int w = NQ / 2, m = 16; w >= 1; w >>= 1, m >>= 1)
        if (lane & m) j += w;
    return j;
}

struct BwdArgs {
    const void *x, *dt, *B, *C, *dy;
    const float *A, *D;
    float *dx, *ddt, *dA, *dB, *dC, *dD;
    float *scratch;            // per CTA: (ceil(L / kRun) + kRun) * N * 64 floats
    const float *init[2];      // start state per direction (batch, H, 64, N), or nullptr (zero)
    float *dinit[2];           // its gradient per direction, or nullptr
    int batch, L, H, G;
};

template <typename T, int N>
__global__ void __launch_bounds__(kThreads)
bwd_scan_kernel(const BwdArgs a) {
    constexpr int NQ = N / 4;
    extern __shared__ float smem[];
    float *Bs = smem;                       // [kTB][N]
    float *Cs = Bs + kTB * N;               // [kTB][N]
    float *xs = Cs + kTB * N;               // [kTB][kP]
    float *dys = xs + kTB * kP;             // [kTB][kP]
    float *dts = dys + kTB * kP;            // [kTB]
    float *part = dts + kTB;                // [kTB][4][kP]   dx partials over quarters
    float *nsum = part + kTB * 4 * kP;      // [kTB][2][N]    dB / dC halves over the quarter's warps
    float *red = nsum + kTB * 2 * N;        // [kTB][8]       <g, h_{t-1}> per warp

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p = tid & (kP - 1), q = tid >> 6, half = (tid >> 5) & 1;
    const int L = a.L;
    const int items = a.batch * a.H * 2;
    const size_t dt_dir = (size_t)a.batch * L * a.H;
    const size_t bc_dir = (size_t)a.batch * L * a.G * N;
    const int nck = (L + kRun - 1) / kRun;
    float *ckpt = a.scratch + (size_t)blockIdx.x * (nck + kRun) * N * kP;   // h after tokens kRun j + kRun - 1
    float *runbuf = ckpt + (size_t)nck * N * kP;                            // h_{s0 - 1 + m}, m < kRun
    const int jt = transposed_index<NQ>(lane);

    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int d = item & 1, unit = item >> 1;
        const int b = unit / a.H, h = unit % a.H;
        const int g = h / (a.H / a.G);
        const bool reverse = d == 1;
        const float Ad = a.A[d * a.H + h];
        const T *dtp = static_cast<const T *>(a.dt) + d * dt_dir;
        const T *Bp = static_cast<const T *>(a.B) + d * bc_dir;
        const T *Cp = static_cast<const T *>(a.C) + d * bc_dir;
        const T *xp = static_cast<const T *>(a.x);
        const T *dyp = static_cast<const T *>(a.dy);
        const float dsum = a.D[h] + a.D[a.H + h];

        // stage tokens [k0, k0 + nt) of the scan's order
        auto stage = [&](int k0, int nt) {
            __syncthreads();
            for (int idx = tid; idx < nt * N; idx += kThreads) {
                const int i = idx / N, n = idx - i * N;
                const int t = reverse ? (L - 1 - (k0 + i)) : (k0 + i);
                const size_t off = ((size_t)(b * L + t) * a.G + g) * N + n;
                Bs[idx] = IO<T>::load(Bp + off);
                Cs[idx] = IO<T>::load(Cp + off);
            }
            for (int idx = tid; idx < nt * kP; idx += kThreads) {
                const int i = idx / kP, pp = idx - i * kP;
                const int t = reverse ? (L - 1 - (k0 + i)) : (k0 + i);
                const size_t o = ((size_t)(b * L + t) * a.H + h) * kP + pp;
                xs[idx] = IO<T>::load(xp + o);
                dys[idx] = IO<T>::load(dyp + o);
            }
            if (tid < nt) {
                const int t = reverse ? (L - 1 - (k0 + tid)) : (k0 + tid);
                dts[tid] = IO<T>::load(dtp + (size_t)(b * L + t) * a.H + h);
            }
            __syncthreads();
        };
        auto token_of = [&](int k) { return reverse ? (L - 1 - k) : k; };

        // ---------------- 1. the scan: states to scratch, dC on the way
        // the start state: element (n, p) of unit (b, h) sits at init[((b H + h) 64 + p) N + n]
        const float *init = a.init[d] ? a.init[d] + ((size_t)(b * a.H + h) * kP + p) * N + q * NQ : nullptr;
        float hs[NQ];
#pragma unroll
        for (int j = 0; j < NQ; ++j) hs[j] = init ? init[j] : 0.f;
        for (int k0 = 0; k0 < L; k0 += kTB) {
            const int nt = min(kTB, L - k0);
            stage(k0, nt);
            for (int i = 0; i < nt; ++i) {
                const float dtv = dts[i];
                const float decay = expf(dtv * Ad);
                const float coef = dtv * xs[i * kP + p];
                const float dyv = dys[i * kP + p];
                const float *Bi = Bs + i * N + q * NQ;
                float w[NQ];
#pragma unroll
                for (int j = 0; j < NQ; ++j) {
                    hs[j] = fmaf(decay, hs[j], coef * Bi[j]);
                    w[j] = hs[j] * dyv;
                }
                if ((k0 + i) % kRun == kRun - 1) {
                    float *hk = ckpt + (size_t)((k0 + i) / kRun) * N * kP;
#pragma unroll
                    for (int j = 0; j < NQ; ++j) hk[(size_t)(q * NQ + j) * kP + p] = hs[j];
                }
                // dC_t[n] = sum_p h_t[n][p] dy_t[p]
                const float s = warp_transpose_sum<NQ>(w, lane);
                if (transposed_writer<NQ>(lane)) nsum[(i * 2 + half) * N + q * NQ + jt] = s;
            }
            __syncthreads();
            for (int idx = tid; idx < nt * N; idx += kThreads) {
                const int i = idx / N, n = idx - i * N;
                const int t = token_of(k0 + i);
                const size_t off = d * bc_dir + ((size_t)(b * L + t) * a.G + g) * N + n;
                const float v = nsum[(i * 2) * N + n] + nsum[(i * 2 + 1) * N + n];
                if (a.H == a.G) a.dC[off] = v;
                else atomicAdd(a.dC + off, v);
            }
        }
        // (each thread reads back only the state elements it wrote: no barrier)

        // ---------------- 2. the adjoint scan, in the opposite order
        float gs[NQ];
#pragma unroll
        for (int j = 0; j < NQ; ++j) gs[j] = 0.f;
        float dA_acc = 0.f, xdy_acc = 0.f;
        for (int c = (L - 1) / kTB; c >= 0; --c) {
            // staged round of scan-order tokens [k0, k0 + nt), walked from the
            // top down; rounds start at multiples of kTB, so no run straddles two
            const int k0 = c * kTB, nt = min(kTB, L - k0);
            stage(k0, nt);
            for (int i = nt - 1; i >= 0; --i) {
                const int k = k0 + i;
                const int s0 = k & ~(kRun - 1);   // first token of k's run
                if (i == nt - 1 || k % kRun == kRun - 1) {
                    // the run's states h_{s0 - 1} .. h_{k - 1} into slots 0 .. k - s0,
                    // from the checkpoint before the run (zero before the first token)
                    float hr[NQ];
                    if (s0 > 0) {
                        const float *hc = ckpt + (size_t)(s0 / kRun - 1) * N * kP;
#pragma unroll
                        for (int j = 0; j < NQ; ++j) hr[j] = hc[(size_t)(q * NQ + j) * kP + p];
                    } else {
#pragma unroll
                        for (int j = 0; j < NQ; ++j) hr[j] = init ? init[j] : 0.f;
                    }
                    for (int m = 0; m <= k - s0; ++m) {
                        if (m > 0) {
                            const int ii = s0 - k0 + m - 1;   // token s0 + m - 1 in the staged round
                            const float dtm = dts[ii];
                            const float dec = expf(dtm * Ad);
                            const float cf = dtm * xs[ii * kP + p];
                            const float *Bm = Bs + ii * N + q * NQ;
#pragma unroll
                            for (int j = 0; j < NQ; ++j) hr[j] = fmaf(dec, hr[j], cf * Bm[j]);
                        }
                        float *hb = runbuf + (size_t)m * N * kP;
#pragma unroll
                        for (int j = 0; j < NQ; ++j) hb[(size_t)(q * NQ + j) * kP + p] = hr[j];
                    }
                }
                const float dtv = dts[i];
                const float decay = expf(dtv * Ad);
                const float xv = xs[i * kP + p], dyv = dys[i * kP + p];
                const float *Bi = Bs + i * N + q * NQ;
                const float *Ci = Cs + i * N + q * NQ;
                // h_{t-1}: the state before this token (slot k - s0 of the run's buffer)
                const float *hp = runbuf + (size_t)(k - s0) * N * kP;
                float u = 0.f, ghp = 0.f;
                float w[NQ];
#pragma unroll
                for (int j = 0; j < NQ; ++j) {
                    gs[j] = fmaf(Ci[j], dyv, gs[j]);
                    u = fmaf(Bi[j], gs[j], u);
                    const float hprev = hp[(size_t)(q * NQ + j) * kP + p];
                    ghp = fmaf(gs[j], hprev, ghp);
                    w[j] = gs[j] * xv;
                }
                part[(i * 4 + q) * kP + p] = u;
                // dB_t[n] = dt_t sum_p g_t[n][p] x_t[p]
                const float s = warp_transpose_sum<NQ>(w, lane);
                if (transposed_writer<NQ>(lane)) nsum[(i * 2 + half) * N + q * NQ + jt] = s;
                // <g_t, h_{t-1}> over the CTA, per warp here
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) ghp += __shfl_xor_sync(0xffffffffu, ghp, m);
                if (lane == 0) red[i * 8 + warp] = ghp;
#pragma unroll
                for (int j = 0; j < NQ; ++j) gs[j] *= decay;
                if (d == 0 && q == 0) xdy_acc = fmaf(xv, dyv, xdy_acc);   // each p once
            }
            __syncthreads();
            // dx (per token and p: the four quarters), dB, ddt, dA
            for (int idx = tid; idx < nt * kP; idx += kThreads) {
                const int i = idx / kP, pp = idx - i * kP;
                const int t = token_of(k0 + i);
                const float *pi = part + i * 4 * kP + pp;
                float v = dts[i] * ((pi[0] + pi[kP]) + (pi[2 * kP] + pi[3 * kP]));
                if (d == 0) v += dsum * dys[idx];
                atomicAdd(a.dx + ((size_t)(b * L + t) * a.H + h) * kP + pp, v);
            }
            for (int idx = tid; idx < nt * N; idx += kThreads) {
                const int i = idx / N, n = idx - i * N;
                const int t = token_of(k0 + i);
                const size_t off = d * bc_dir + ((size_t)(b * L + t) * a.G + g) * N + n;
                const float v = dts[i] * (nsum[(i * 2) * N + n] + nsum[(i * 2 + 1) * N + n]);
                if (a.H == a.G) a.dB[off] = v;
                else atomicAdd(a.dB + off, v);
            }
            if (tid < nt) {
                const int i = tid;
                const int t = token_of(k0 + i);
                const float dtv = dts[i];
                const float decay = expf(dtv * Ad);
                float ghp = 0.f;
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8) ghp += red[i * 8 + w8];
                // B_t^T g_t x_t = sum_p x_t[p] (sum_n B_t[n] g_t[n][p])
                float gbx = 0.f;
                for (int pp = 0; pp < kP; ++pp) {
                    const float *pi = part + i * 4 * kP + pp;
                    gbx = fmaf(xs[i * kP + pp], (pi[0] + pi[kP]) + (pi[2 * kP] + pi[3 * kP]), gbx);
                }
                a.ddt[d * dt_dir + (size_t)(b * L + t) * a.H + h] = gbx + Ad * decay * ghp;
                dA_acc += dtv * decay * ghp;
            }
        }
        // the start state's gradient: the adjoint left after the first token
        if (a.dinit[d]) {
            float *di = a.dinit[d] + ((size_t)(b * a.H + h) * kP + p) * N + q * NQ;
#pragma unroll
            for (int j = 0; j < NQ; ++j) di[j] = gs[j];
        }
        // dA over this item's tokens (held by threads 0..kTB-1), dD
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            dA_acc += __shfl_xor_sync(0xffffffffu, dA_acc, m);
            xdy_acc += __shfl_xor_sync(0xffffffffu, xdy_acc, m);
        }
        __syncthreads();
        if (lane == 0) red[warp] = xdy_acc;
        __syncthreads();
        if (tid == 0) {
            atomicAdd(a.dA + d * a.H + h, dA_acc);
            if (d == 0) {
                float s = 0.f;
                for (int w8 = 0; w8 < 8; ++w8) s += red[w8];
                atomicAdd(a.dD + h, s);
                atomicAdd(a.dD + a.H + h, s);
            }
        }
    }
}

template <int N>
size_t bwd_smem() {
    return sizeof(float) * (2 * kTB * N + 2 * kTB * kP + kTB + kTB * 4 * kP + kTB * 2 * N + kTB * 8);
}

template <typename T, int N>
cudaError_t run_bwd(const BwdArgs &a, int grid, cudaStream_t stream) {
    auto k = bwd_scan_kernel<T, N>;
    const size_t smem = bwd_smem<N>();
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Persistent grid: two CTAs per SM at most, and no more than there are items.
int bwd_grid(int batch, int H) {
    const int sms = device_sms();
    const long long items = 2LL * batch * H;
    const long long cap = 2LL * (sms > 0 ? sms : 1);
    return (int)(items < cap ? items : cap);
}

size_t bwd_scratch_bytes(int batch, int L, int H, int N) {
    const size_t nck = ((size_t)L + kRun - 1) / kRun;
    return (size_t)bwd_grid(batch, H) * (nck + kRun) * N * kP * sizeof(float);
}

cudaError_t launch_bwd(const BwdLaunch &l, cudaStream_t stream) {
    if (l.N != 64 && l.N != 128) return cudaErrorNotSupported;
    BwdArgs a{};
    a.x = l.x; a.dt = l.dt; a.B = l.B; a.C = l.C; a.dy = l.dy; a.A = l.A; a.D = l.D;
    a.dx = l.dx; a.ddt = l.ddt; a.dA = l.dA; a.dB = l.dB; a.dC = l.dC; a.dD = l.dD;
    a.scratch = l.scratch;
    a.init[0] = l.init_f; a.init[1] = l.init_b;
    a.dinit[0] = l.dinit_f; a.dinit[1] = l.dinit_b;
    a.batch = l.batch; a.L = l.L; a.H = l.H; a.G = l.G;
    const int grid = bwd_grid(l.batch, l.H);
    // outputs that receive atomic additions start at zero
    const size_t nx = (size_t)l.batch * l.L * l.H * kP, nbc = 2 * (size_t)l.batch * l.L * l.G * l.N;
    cudaError_t e;
    if ((e = cudaMemsetAsync(l.dx, 0, nx * sizeof(float), stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(l.dA, 0, 2 * (size_t)l.H * sizeof(float), stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(l.dD, 0, 2 * (size_t)l.H * sizeof(float), stream)) != cudaSuccess) return e;
    if (l.H != l.G) {
        if ((e = cudaMemsetAsync(l.dB, 0, nbc * sizeof(float), stream)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(l.dC, 0, nbc * sizeof(float), stream)) != cudaSuccess) return e;
    }
    if (l.bf16) return l.N == 64 ? run_bwd<__nv_bfloat16, 64>(a, grid, stream) : run_bwd<__nv_bfloat16, 128>(a, grid, stream);
    return l.N == 64 ? run_bwd<float, 64>(a, grid, stream) : run_bwd<float, 128>(a, grid, stream);
}

}  // namespace ssd
