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

constexpr int kMaxConv = 4;          // widest conv supported

__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }

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

// One direction's conv + SiLU for 8 consecutive channels (16 bytes of bf16)
// of one batch element over a run of kConvRun tokens: the forward conv's tap k
// reads token t - (K - 1) + k, the reverse conv's tap k token t + (K - 1) - k
// (zero outside the sequence). The thread keeps its direction's taps for its
// channels and the last K - 1 input rows in registers and, per group of 8
// tokens, issues the group's 8 row loads (16 bytes each, 512 contiguous bytes
// across a warp) before it uses any, so each group waits for memory once. The
// x, B and C blocks of channels are multiples of 8 wide, so a thread's
// channels go to one of them.
// 8 channels of the I/O type kept as loaded (4 registers of bf16 pairs, 8 of
// fp32) until used.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
    uint4 q;
    __device__ __forceinline__ void load(const __nv_bfloat16 *p) { q = *reinterpret_cast<const uint4 *>(p); }
    __device__ __forceinline__ void zero() { q = make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ void unpack(float (&v)[8]) const {
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(u[k] << 16);
            v[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
        }
    }
};
template <> struct Raw8<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float *p) {
        a = reinterpret_cast<const float4 *>(p)[0];
        b = reinterpret_cast<const float4 *>(p)[1];
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void unpack(float (&v)[8]) const {
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

constexpr int kConvRun = 64;     // tokens per thread
constexpr int kConvGroup = 8;    // rows loaded at once
constexpr int kConvBlock = 128;  // threads per CTA: 128 chunks of 8 channels

template <typename T, int K>
__global__ void __launch_bounds__(kConvBlock)
conv_silu_kernel(const T *__restrict__ xbc, const float *__restrict__ w, const float *__restrict__ bias,
                 T *__restrict__ x2, T *__restrict__ B2, T *__restrict__ C2, int batch, int L, int HP, int GN) {
    constexpr int R = K - 1;
    const int cin = HP + 2 * GN;
    const int c = 8 * (blockIdx.x * kConvBlock + threadIdx.x);
    const int dir = blockIdx.y & 1, t0 = (blockIdx.y >> 1) * kConvRun, b = blockIdx.z;
    if (c >= cin) return;
    // wk[e][m]: the tap that multiplies window slot m, slot m holding token
    // t - R + m (forward) or t + m (reverse) for output token t
    float wk[8][K], bk[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
#pragma unroll
        for (int m = 0; m < K; ++m)
            wk[e][m] = w[(size_t)dir * cin * K + (size_t)(c + e) * K + (dir ? R - m : m)];
        bk[e] = bias[(size_t)dir * cin + c + e];
    }
    T *dst;
    size_t ld;
    if (c < HP) {
        dst = x2 + (size_t)b * L * HP + c; ld = HP;
        if (dir) dst += (size_t)batch * L * HP;
    } else if (c < HP + GN) {
        dst = B2 + (size_t)b * L * GN + (c - HP); ld = GN;
        if (dir) dst += (size_t)batch * L * GN;
    } else {
        dst = C2 + (size_t)b * L * GN + (c - HP - GN); ld = GN;
        if (dir) dst += (size_t)batch * L * GN;
    }
    const T *in = xbc + (size_t)b * L * cin + c;
    // first input row of the window of token t0: t0 - R (forward) or t0 (reverse)
    const int first = t0 - (dir ? 0 : R);
    auto load = [&](int t, Raw8<T> &r) {
        if (t >= 0 && t < L) r.load(in + (size_t)t * cin);
        else r.zero();
    };
    float win[K][8];
#pragma unroll
    for (int m = 0; m < R; ++m) {
        Raw8<T> r;
        load(first + m, r);
        r.unpack(win[m]);
    }
    const int end = min(t0 + kConvRun, L);
    for (int g0 = t0; g0 < end; g0 += kConvGroup) {
        Raw8<T> rows[kConvGroup];
#pragma unroll
        for (int i = 0; i < kConvGroup; ++i) load(first + (g0 - t0) + i + R, rows[i]);
#pragma unroll
        for (int i = 0; i < kConvGroup; ++i) {
            rows[i].unpack(win[R]);
            float o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float a = bk[e];
#pragma unroll
                for (int m = 0; m < K; ++m) a = fmaf(wk[e][m], win[m][e], a);
                o[e] = silu(a);
            }
            const int t = g0 + i;
            if (t < end) Vec8<T>::store(dst + (size_t)t * ld, o);
#pragma unroll
            for (int m = 0; m < R; ++m)
#pragma unroll
                for (int e = 0; e < 8; ++e) win[m][e] = win[m + 1][e];
        }
    }
}

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
    dim3 grid((cin / 8 + kConvBlock - 1) / kConvBlock, 2 * ((l.L + kConvRun - 1) / kConvRun), l.batch);
    conv_silu_kernel<T, K><<<grid, kConvBlock, 0, s>>>(static_cast<const T *>(l.xbc), l.conv_w, l.conv_b,
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
    if (l.HP % 8 || l.GN % 8) return cudaErrorNotSupported;   // 8-channel chunks
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
