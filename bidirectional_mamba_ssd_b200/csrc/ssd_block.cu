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
constexpr int kConvTokens = 8;       // tokens per thread (its whole input window is loaded at once)
constexpr int kMaxConv = 4;          // widest conv supported

__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// Four consecutive channels of the I/O type as floats (8 bytes of bf16 or 16
// of fp32; the channel index is a multiple of 4).
template <typename T> struct Vec4;
template <> struct Vec4<float> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[4]) {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec4<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[4]) {
        const uint2 q = *reinterpret_cast<const uint2 *>(p);
        v[0] = __uint_as_float(q.x << 16); v[1] = __uint_as_float(q.x & 0xffff0000u);
        v[2] = __uint_as_float(q.y << 16); v[3] = __uint_as_float(q.y & 0xffff0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[4]) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
        *reinterpret_cast<uint2 *>(p) = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
    }
};

// One thread: channels [c, c + 4) of one batch element over kConvTokens
// tokens. Tap k of the forward conv reads token t - (K - 1) + k, of the
// reverse conv token t + (K - 1) - k (zero outside the sequence). The inputs
// its 8 tokens read (t0 - K + 1 .. t0 + 7 + K - 1) are loaded into registers
// at once, 4 channels per load (coalesced across the channels of a warp), so
// the thread waits for memory once; the channels' 2 K weights and 2 biases stay
// in registers. The x, B and C blocks of channels are multiples of 4 wide, so
// a thread's channels go to one of them.
template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads)
conv_silu_kernel(const T *__restrict__ xbc, const float *__restrict__ w, const float *__restrict__ bias,
                 T *__restrict__ x2, T *__restrict__ B2, T *__restrict__ C2, int batch, int L, int HP, int GN) {
    constexpr int R = K - 1;                 // window radius
    const int cin = HP + 2 * GN;
    const int c = 4 * (blockIdx.x * kConvThreads + threadIdx.x);
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * kConvTokens;
    if (c >= cin) return;
    // wf[e][k]: forward tap k of channel c + e (reads token t - R + k); wr[e][k]:
    // reverse tap k (reads token t + R - k)
    float wf[4][K], wr[4][K], bf[4], bb[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            wf[e][k] = w[(size_t)(c + e) * K + k];
            wr[e][k] = w[(size_t)cin * K + (size_t)(c + e) * K + k];
        }
        bf[e] = bias[c + e];
        bb[e] = bias[cin + c + e];
    }
    const T *in = xbc + (size_t)b * L * cin + c;
    // destination of these channels in each direction
    T *dst;
    size_t ld, dir_stride;
    if (c < HP) {
        dst = x2 + (size_t)b * L * HP + c; ld = HP; dir_stride = (size_t)batch * L * HP;
    } else if (c < HP + GN) {
        dst = B2 + (size_t)b * L * GN + (c - HP); ld = GN; dir_stride = (size_t)batch * L * GN;
    } else {
        dst = C2 + (size_t)b * L * GN + (c - HP - GN); ld = GN; dir_stride = (size_t)batch * L * GN;
    }
    // every input the thread's tokens read (slot j holds token t0 - R + j),
    // loaded before any is used
    float win[kConvTokens + 2 * R][4];
#pragma unroll
    for (int j = 0; j < kConvTokens + 2 * R; ++j) {
        const int t = t0 - R + j;
        if (t >= 0 && t < L) {
            Vec4<T>::load(in + (size_t)t * cin, win[j]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) win[j][e] = 0.f;
        }
    }
#pragma unroll
    for (int i = 0; i < kConvTokens; ++i) {
        const int t = t0 + i;
        if (t < L) {
            float f[4], r[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                f[e] = bf[e];
                r[e] = bb[e];
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    f[e] = fmaf(wf[e][k], win[i + k][e], f[e]);           // token t - R + k
                    r[e] = fmaf(wr[e][k], win[i + 2 * R - k][e], r[e]);   // token t + R - k
                }
                f[e] = silu(f[e]);
                r[e] = silu(r[e]);
            }
            Vec4<T>::store(dst + (size_t)t * ld, f);
            Vec4<T>::store(dst + dir_stride + (size_t)t * ld, r);
        }
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

// Eight consecutive channels of the I/O type as floats (16 bytes of bf16;
// two 16-byte loads of fp32).
template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[8]) {
        const uint4 q = *reinterpret_cast<const uint4 *>(p);
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(u[k] << 16);
            v[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint32_t u[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
            u[k] = *reinterpret_cast<uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(u[0], u[1], u[2], u[3]);
    }
};
template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[8]) {
        const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[8]) {
        reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
};

constexpr int kNormChunks = 8;   // 8-channel chunks per lane held in registers: C <= 32 * 8 * 8

// One warp per token: v = y SiLU(z) over the token's C channels (fp32, C a
// multiple of 8 and at most 2048), r = 1 / sqrt(mean(v^2) + eps), out = v r w.
// Each lane loads its chunks of 8 channels once (16-byte loads) and keeps v in
// registers between the sum and the scaling.
template <typename T>
__global__ void __launch_bounds__(256)
gated_rmsnorm_kernel(const T *__restrict__ y, const T *__restrict__ z, const float *__restrict__ w,
                     T *__restrict__ out, long long rows, int C, float eps) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const T *yr = y + row * C, *zr = z + row * C;
    T *orow = out + row * C;
    const int chunks = C / 8;
    float v[kNormChunks][8];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kNormChunks; ++k) {
        const int ch = lane + 32 * k;
        if (ch < chunks) {
            float yv[8], zv[8];
            Vec8<T>::load(yr + 8 * ch, yv);
            Vec8<T>::load(zr + 8 * ch, zv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[k][e] = yv[e] * silu(zv[e]);
                ss = fmaf(v[k][e], v[k][e], ss);
            }
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float r = rsqrtf(ss / (float)C + eps);
#pragma unroll
    for (int k = 0; k < kNormChunks; ++k) {
        const int ch = lane + 32 * k;
        if (ch < chunks) {
            float o[8], wv[8];
            Vec8<float>::load(w + 8 * ch, wv);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = v[k][e] * r * wv[e];
            Vec8<T>::store(orow + 8 * ch, o);
        }
    }
}

template <typename T, int K>
cudaError_t run_conv_k(const BlockLaunch &l, cudaStream_t s) {
    const int cin = l.HP + 2 * l.GN;
    dim3 grid((cin / 4 + kConvThreads - 1) / kConvThreads, (l.L + kConvTokens - 1) / kConvTokens, l.batch);
    conv_silu_kernel<T, K><<<grid, kConvThreads, 0, s>>>(static_cast<const T *>(l.xbc), l.conv_w, l.conv_b,
                                                         static_cast<T *>(l.x2), static_cast<T *>(l.B2),
                                                         static_cast<T *>(l.C2), l.batch, l.L, l.HP, l.GN);
    return cudaGetLastError();
}

template <typename T>
cudaError_t run_conv(const BlockLaunch &l, cudaStream_t s) {
    switch (l.K) {
        case 1: return run_conv_k<T, 1>(l, s);
        case 2: return run_conv_k<T, 2>(l, s);
        case 3: return run_conv_k<T, 3>(l, s);
        default: return run_conv_k<T, 4>(l, s);
    }
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
    if (l.HP % 4 || l.GN % 4) return cudaErrorNotSupported;   // 4 channels per thread
    return l.bf16 ? run_conv<__nv_bfloat16>(l, s) : run_conv<float>(l, s);
}

cudaError_t launch_dt_prep(const BlockLaunch &l, cudaStream_t s) {
    return l.bf16 ? run_dt<__nv_bfloat16>(l, s) : run_dt<float>(l, s);
}

cudaError_t launch_gated_rmsnorm(const BlockLaunch &l, cudaStream_t s) {
    if (l.HP % 8 || l.HP > 32 * 8 * kNormChunks) return cudaErrorNotSupported;
    return l.bf16 ? run_norm<__nv_bfloat16>(l, s) : run_norm<float>(l, s);
}

}  // namespace ssd
