// The steps either side of the bidirectional mixer in a Mamba-2 layer, on
// CUDA cores (each is a pass over memory: HBM-bound):
//  - conv_silu_kernel: both directions' depthwise conv1d + SiLU over the
//    projected xBC channels, causal for the forward scan and anti-causal (the
//    flipped sequence's causal conv) for the reverse scan, written straight
//    into the mixer's per-direction x, B and C layouts;
//  - dt_prep_kernel: the scans' step size from the raw projection,
//    dt = clamp(softplus(dt_raw + dt_bias));
//  - gated_rmsnorm_kernel: Mamba-2's gated RMS norm of the summed mixer output,
//    out = y SiLU(z) / sqrt(mean((y SiLU(z))^2) + eps) * w over the H * P
//    channels of a token.
// "DiffMamba - Checkpoints" model card, Model details: forward and flipped-
// reverse Mamba-2 layers with weight-tied projections and Mamba-2 defaults
// (depthwise conv of width 4 before the scan, gated RMS norm after it).
#include "ssd_common.cuh"
#include "ssd_kernels.h"

namespace ssd {
namespace {

constexpr int kConvThreads = 256;
constexpr int kConvTokens = 32;      // tokens per thread
constexpr int kMaxConv = 4;          // widest conv supported

__device__ __forceinline__ float silu(float v) { return v / (1.f + __expf(-v)); }

// One thread: channel c of one batch element over kConvTokens tokens. Tap k of
// the forward conv reads token t - (K - 1) + k, of the reverse conv token
// t + (K - 1) - k (zero outside the sequence). The inputs t - 3 .. t + 3 sit
// in a register window that moves one token per step, so every input is
// loaded once per thread (coalesced across the channels of a warp); the
// channel's 2 K weights and 2 biases stay in registers.
template <typename T>
__global__ void __launch_bounds__(kConvThreads)
conv_silu_kernel(const T *__restrict__ xbc, const float *__restrict__ w, const float *__restrict__ bias,
                 T *__restrict__ x2, T *__restrict__ B2, T *__restrict__ C2, int batch, int L, int HP, int GN,
                 int K) {
    constexpr int R = kMaxConv - 1;          // window radius
    const int cin = HP + 2 * GN;
    const int c = blockIdx.x * kConvThreads + threadIdx.x;
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * kConvTokens;
    if (c >= cin) return;
    // taps aligned to the window: forward weight of window slot j (token t - R + j)
    // and reverse weight of slot j (token t - R + j), zero where the conv has no tap
    float wf[2 * R + 1], wr[2 * R + 1];
#pragma unroll
    for (int j = 0; j < 2 * R + 1; ++j) {
        const int kf = j - R + (K - 1);      // forward tap reading token t - R + j
        const int kr = R + (K - 1) - j;      // reverse tap reading token t - R + j
        wf[j] = (kf >= 0 && kf < K && j <= R) ? w[(size_t)c * K + kf] : 0.f;
        wr[j] = (kr >= 0 && kr < K && j >= R) ? w[(size_t)cin * K + (size_t)c * K + kr] : 0.f;
    }
    const float bf = bias[c], bb = bias[cin + c];
    const T *in = xbc + (size_t)b * L * cin + c;
    auto load = [&](int t) { return (t >= 0 && t < L) ? IO<T>::load(in + (size_t)t * cin) : 0.f; };
    // destination of this channel in each direction
    T *dst;
    size_t ld, dir_stride;
    if (c < HP) {
        dst = x2 + (size_t)b * L * HP + c; ld = HP; dir_stride = (size_t)batch * L * HP;
    } else if (c < HP + GN) {
        dst = B2 + (size_t)b * L * GN + (c - HP); ld = GN; dir_stride = (size_t)batch * L * GN;
    } else {
        dst = C2 + (size_t)b * L * GN + (c - HP - GN); ld = GN; dir_stride = (size_t)batch * L * GN;
    }
    float win[2 * R + 1];
#pragma unroll
    for (int j = 0; j < 2 * R + 1; ++j) win[j] = load(t0 - R + j);
#pragma unroll
    for (int i = 0; i < kConvTokens; ++i) {
        const int t = t0 + i;
        const float next = load(t + R + 1);   // issued a step ahead
        if (t < L) {
            float f = bf, r = bb;
#pragma unroll
            for (int j = 0; j < 2 * R + 1; ++j) {
                f = fmaf(wf[j], win[j], f);
                r = fmaf(wr[j], win[j], r);
            }
            IO<T>::store(dst + (size_t)t * ld, silu(f));
            IO<T>::store(dst + dir_stride + (size_t)t * ld, silu(r));
        }
#pragma unroll
        for (int j = 0; j < 2 * R; ++j) win[j] = win[j + 1];
        win[2 * R] = next;
    }
}

// dt[d][b][t][h] = clamp(softplus(raw + bias[d][h]), lo, hi); softplus(u) =
// log(1 + e^u), taken as u beyond 20 (where the two agree in fp32).
template <typename T>
__global__ void dt_prep_kernel(const T *__restrict__ raw, const float *__restrict__ bias, T *__restrict__ dt,
                               long long per_dir, int H, float lo, float hi) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * per_dir) return;
    const int d = i >= per_dir ? 1 : 0;
    const int h = (int)((i - d * per_dir) % H);
    const float u = IO<T>::load(raw + i) + bias[d * H + h];
    const float sp = u > 20.f ? u : log1pf(__expf(u));
    IO<T>::store(dt + i, fminf(fmaxf(sp, lo), hi));
}

// One warp per token: v = y SiLU(z) over the token's C channels (fp32),
// r = 1 / sqrt(mean(v^2) + eps), out = v r w.
template <typename T>
__global__ void __launch_bounds__(256)
gated_rmsnorm_kernel(const T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w,
                     T *__restrict__ out, long long rows, int C, float eps) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const T *yr = y + row * C, *zr = z + row * C;
    T *orow = out + row * C;
    float ss = 0.f;
    for (int c = lane; c < C; c += 32) {
        const float v = IO<T>::load(yr + c) * silu(IO<T>::load(zr + c));
        ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float r = rsqrtf(ss / (float)C + eps);
    for (int c = lane; c < C; c += 32) {
        const float v = IO<T>::load(yr + c) * silu(IO<T>::load(zr + c));
        IO<T>::store(orow + c, v * r * w[c]);
    }
}

template <typename T>
cudaError_t run_conv(const BlockLaunch &l, cudaStream_t s) {
    const int cin = l.HP + 2 * l.GN;
    dim3 grid((cin + kConvThreads - 1) / kConvThreads, (l.L + kConvTokens - 1) / kConvTokens, l.batch);
    conv_silu_kernel<T><<<grid, kConvThreads, 0, s>>>(static_cast<const T *>(l.xbc), l.conv_w, l.conv_b,
                                                      static_cast<T *>(l.x2), static_cast<T *>(l.B2),
                                                      static_cast<T *>(l.C2), l.batch, l.L, l.HP, l.GN, l.K);
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_dt(const BlockLaunch &l, cudaStream_t s) {
    const long long per_dir = (long long)l.batch * l.L * l.H;
    const long long n = 2 * per_dir;
    dt_prep_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(static_cast<const T *>(l.dt_raw), l.dt_bias,
                                                                  static_cast<T *>(l.dt), per_dir, l.H, l.dt_lo,
                                                                  l.dt_hi);
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_norm(const BlockLaunch &l, cudaStream_t s) {
    const long long rows = (long long)l.batch * l.L;
    gated_rmsnorm_kernel<T><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
        static_cast<const T *>(l.y), static_cast<const T *>(l.z), l.norm_w, static_cast<T *>(l.out), rows, l.HP,
        l.eps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_conv_silu(const BlockLaunch &l, cudaStream_t s) {
    if (l.K < 1 || l.K > kMaxConv) return cudaErrorNotSupported;
    return l.bf16 ? run_conv<__nv_bfloat16>(l, s) : run_conv<float>(l, s);
}

cudaError_t launch_dt_prep(const BlockLaunch &l, cudaStream_t s) {
    return l.bf16 ? run_dt<__nv_bfloat16>(l, s) : run_dt<float>(l, s);
}

cudaError_t launch_gated_rmsnorm(const BlockLaunch &l, cudaStream_t s) {
    return l.bf16 ? run_norm<__nv_bfloat16>(l, s) : run_norm<float>(l, s);
}

}  // namespace ssd
