// Sequential SSD scan on CUDA cores, fp32 state and arithmetic.
//
// One CTA per (batch, head). The N x P state of a scan lives in registers of
// 256 threads: thread (p, q) owns h[n][p] for the N/4 values n in quarter q.
// Per token the threads apply h <- exp(dt A) h + dt B x^T and read
// y = C^T h, exactly the recurrence of the Mamba-2 SSD layer; the forward
// scan walks the sequence left to right, the reverse scan right to left
// ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
// Technical Summary, 2. Methodology, Core Architecture: forward and backward
// Mamba-2, added). Two kernels:
//  - scan_simt_seq_kernel (256 threads): the forward scan into an fp32
//    buffer, then the reverse scan, which adds the buffer and the D terms as
//    it writes out.
//  - scan_simt_pair_kernel (512 threads, both scans): for calls whose units
//    take a single round of CTAs, the two scans run side by side in two
//    256-thread halves (each with its own named barrier) into their own fp32
//    buffers, and once both are done the CTA adds them and the D terms; each
//    staged token's decay exp(dt A) is formed once, off the token chain.
//
// This path serves fp32 I/O, where its plain recurrence keeps relative error
// near 1e-6, and is the second, independent GPU path for bf16 I/O. Tokens are
// staged through shared memory 32 at a time so global reads are coalesced;
// the staging also forms each token's decay exp(dt A), which takes the
// exponential off the token-to-token chain.
#include "ssd_common.cuh"
#include "ssd_kernels.h"

namespace ssd {
namespace {

constexpr int kP = 64;        // headdim
constexpr int kThreads = 256; // 64 head-dim lanes x 4 state quarters
constexpr int kHalf = kThreads;  // threads per direction in the pair kernel
constexpr int kTB = 32;       // tokens staged per round

// shared-memory floats of one direction's staging area
template <int N>
constexpr int stage_floats() { return 2 * kTB * N + kTB * kP + 2 * kTB + kTB * 4 * kP; }

template <typename T, int N>
__global__ void __launch_bounds__(kThreads)
scan_simt_seq_kernel(const SimtArgs a) {
    constexpr int NQ = N / 4;
    extern __shared__ float smem[];
    float *Bs = smem;                       // [kTB][N]
    float *Cs = Bs + kTB * N;               // [kTB][N]
    float *xs = Cs + kTB * N;               // [kTB][kP]
    float *dts = xs + kTB * kP;             // [kTB]
    float *part = dts + kTB;                // [kTB][4][kP]

    const int unit = blockIdx.x;
    const int b = unit / a.H, h = unit % a.H;
    const int g = h / (a.H / a.G);
    const int tid = threadIdx.x;
    const int p = tid & (kP - 1), q = tid >> 6;
    const int L = a.L;
    const T *x = static_cast<const T *>(a.x);
    T *out = static_cast<T *>(a.out);

    const float dsum = a.has_output ? (a.D[h] + a.D[a.H + h]) : 0.f;
    // D terms: with one x both go on at the end; with one x per direction each
    // direction adds its own D x
    const bool x2 = a.x_dir_stride != 0;
    const float d_first = (a.has_output && x2) ? a.D[h] : 0.f;
    const float d_last = (a.has_output && x2) ? a.D[a.H + h] : dsum;
    float hs[NQ];

    for (int dir = 0; dir < a.ndir; ++dir) {
        const bool reverse = dir == 1;
        const T *xd = x + dir * a.x_dir_stride;
        // Starting state: the forward scan may start from a given state.
        if (dir == 0 && a.init) {
            const float *ip = a.init + ((size_t)unit * kP + p) * N + q * NQ;
#pragma unroll
            for (int j = 0; j < NQ; ++j) hs[j] = ip[j];
        } else {
#pragma unroll
            for (int j = 0; j < NQ; ++j) hs[j] = 0.f;
        }
        const float Ad = a.A[dir * a.A_dir_stride + h];
        const T *dtp = static_cast<const T *>(a.dt) + dir * a.dt_dir_stride;
        const T *Bp = static_cast<const T *>(a.B) + dir * a.bc_dir_stride;
        const T *Cp = a.C ? static_cast<const T *>(a.C) + dir * a.bc_dir_stride : nullptr;

        for (int t0 = 0; t0 < L; t0 += kTB) {
            const int nt = min(kTB, L - t0);
            __syncthreads();  // previous round's smem fully consumed
            for (int idx = tid; idx < nt * N; idx += kThreads) {
                const int i = idx / N, n = idx - i * N;
                const int t = reverse ? (L - 1 - (t0 + i)) : (t0 + i);
                const size_t off = ((size_t)(b * L + t) * a.G + g) * N + n;
                Bs[i * N + n] = IO<T>::load(Bp + off);
                if (Cp) Cs[i * N + n] = IO<T>::load(Cp + off);
            }
            for (int idx = tid; idx < nt * kP; idx += kThreads) {
                const int i = idx / kP, pp = idx - i * kP;
                const int t = reverse ? (L - 1 - (t0 + i)) : (t0 + i);
                xs[idx] = IO<T>::load(xd + ((size_t)(b * L + t) * a.H + h) * kP + pp);
            }
            if (tid < nt) {
                const int t = reverse ? (L - 1 - (t0 + tid)) : (t0 + tid);
                dts[tid] = IO<T>::load(dtp + (size_t)(b * L + t) * a.H + h);
            }
            __syncthreads();
            for (int i = 0; i < nt; ++i) {
                const float dtv = dts[i];
                const float decay = expf(dtv * Ad);
                const float coef = dtv * xs[i * kP + p];
                const float *Bi = Bs + i * N + q * NQ;
                const float *Ci = Cs + i * N + q * NQ;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < NQ; ++j) {
                    hs[j] = fmaf(decay, hs[j], coef * Bi[j]);
                    if (Cp) acc = fmaf(Ci[j], hs[j], acc);
                }
                if (Cp) part[(i * 4 + q) * kP + p] = acc;
            }
            if (a.has_output) {
                __syncthreads();
                for (int idx = tid; idx < nt * kP; idx += kThreads) {
                    const int i = idx / kP, pp = idx - i * kP;
                    const int t = reverse ? (L - 1 - (t0 + i)) : (t0 + i);
                    const float *pi = part + i * 4 * kP + pp;
                    const float y = (pi[0] + pi[kP]) + (pi[2 * kP] + pi[3 * kP]);
                    const size_t o = ((size_t)(b * L + t) * a.H + h) * kP + pp;
                    if (dir == 0 && a.ndir == 2) {
                        a.yacc[o] = x2 ? y + d_first * xs[idx] : y;
                    } else {
                        const float prev = (a.ndir == 2) ? a.yacc[o] : 0.f;
                        IO<T>::store(out + o, prev + y + d_last * xs[idx]);
                    }
                }
            }
        }
        __syncthreads();  // forward partials visible to the reverse pass
    }

    if (a.state_out) {
        float *sp = a.state_out + ((size_t)unit * kP + p) * N + q * NQ;
#pragma unroll
        for (int j = 0; j < NQ; ++j) sp[j] = hs[j];
    }
}

template <typename T, int N>
cudaError_t launch_seq(const SimtArgs &a, cudaStream_t stream) {
    const size_t smem = sizeof(float) * (2 * kTB * N + kTB * kP + kTB + kTB * 4 * kP);
    auto kern = scan_simt_seq_kernel<T, N>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<a.batch * a.H, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, int N>
__global__ void __launch_bounds__(2 * kHalf)
scan_simt_pair_kernel(const SimtArgs a) {
    constexpr int NQ = N / 4;
    extern __shared__ float smem[];
    const int half = threadIdx.x / kHalf, lt = threadIdx.x % kHalf;
    float *Bs = smem + half * stage_floats<N>();  // [kTB][N]
    float *Cs = Bs + kTB * N;                     // [kTB][N]
    float *xs = Cs + kTB * N;                     // [kTB][kP]
    float *dts = xs + kTB * kP;                   // [kTB]
    float *decs = dts + kTB;                      // [kTB]      exp(dt A)
    float *part = decs + kTB;                     // [kTB][4][kP]
    // this direction's named barrier (ids 1 and 2) over its 256 threads; the
    // ids are literals so that the kernel holds three barriers, not all sixteen
    auto sync_dir = [&]() {
        if (half == 0) asm volatile("bar.sync 1, 256;" ::: "memory");
        else asm volatile("bar.sync 2, 256;" ::: "memory");
    };

    const int unit = blockIdx.x;
    const int b = unit / a.H, h = unit % a.H;
    const int g = h / (a.H / a.G);
    const int p = lt & (kP - 1), q = lt >> 6;
    const int L = a.L;
    const T *x = static_cast<const T *>(a.x);
    T *out = static_cast<T *>(a.out);
    const size_t yplane = (size_t)a.batch * L * a.H * kP;   // one direction's output buffer
    const float dsum = a.D[h] + a.D[a.H + h];

    float hs[NQ];
    {
        const int dir = half;
        const bool reverse = dir == 1;
        float *yacc = a.yacc + dir * yplane;
        // Starting state: the forward scan may start from a given state.
        if (dir == 0 && a.init) {
            const float *ip = a.init + ((size_t)unit * kP + p) * N + q * NQ;
#pragma unroll
            for (int j = 0; j < NQ; ++j) hs[j] = ip[j];
        } else {
#pragma unroll
            for (int j = 0; j < NQ; ++j) hs[j] = 0.f;
        }
        const float Ad = a.A[dir * a.A_dir_stride + h];
        const T *dtp = static_cast<const T *>(a.dt) + dir * a.dt_dir_stride;
        const T *Bp = static_cast<const T *>(a.B) + dir * a.bc_dir_stride;
        const T *Cp = a.C ? static_cast<const T *>(a.C) + dir * a.bc_dir_stride : nullptr;

        for (int t0 = 0; t0 < L; t0 += kTB) {
            const int nt = min(kTB, L - t0);
            sync_dir();  // previous round's staging fully consumed
            for (int idx = lt; idx < nt * N; idx += kHalf) {
                const int i = idx / N, n = idx - i * N;
                const int t = reverse ? (L - 1 - (t0 + i)) : (t0 + i);
                const size_t off = ((size_t)(b * L + t) * a.G + g) * N + n;
                Bs[i * N + n] = IO<T>::load(Bp + off);
                if (Cp) Cs[i * N + n] = IO<T>::load(Cp + off);
            }
            if (lt < nt) {
                const int t = reverse ? (L - 1 - (t0 + lt)) : (t0 + lt);
                const float dtv = IO<T>::load(dtp + (size_t)(b * L + t) * a.H + h);
                dts[lt] = dtv;
                decs[lt] = expf(dtv * Ad);
            }
            for (int idx = lt; idx < nt * kP; idx += kHalf) {
                const int i = idx / kP, pp = idx - i * kP;
                const int t = reverse ? (L - 1 - (t0 + i)) : (t0 + i);
                xs[idx] = IO<T>::load(x + ((size_t)(b * L + t) * a.H + h) * kP + pp);
            }
            sync_dir();
#pragma unroll 4
            for (int i = 0; i < kTB; ++i) {
                if (i >= nt) break;
                const float decay = decs[i];
                const float coef = dts[i] * xs[i * kP + p];
                const float *Bi = Bs + i * N + q * NQ;
                const float *Ci = Cs + i * N + q * NQ;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < NQ; ++j) {
                    hs[j] = fmaf(decay, hs[j], coef * Bi[j]);
                    if (Cp) acc = fmaf(Ci[j], hs[j], acc);
                }
                if (Cp) part[(i * 4 + q) * kP + p] = acc;
            }
            if (a.has_output) {
                sync_dir();
                for (int idx = lt; idx < nt * kP; idx += kHalf) {
                    const int i = idx / kP, pp = idx - i * kP;
                    const int t = reverse ? (L - 1 - (t0 + i)) : (t0 + i);
                    const float *pi = part + i * 4 * kP + pp;
                    const float y = (pi[0] + pi[kP]) + (pi[2 * kP] + pi[3 * kP]);
                    const size_t o = ((size_t)(b * L + t) * a.H + h) * kP + pp;
                    yacc[o] = y;
                }
            }
        }

        if (dir == 0 && a.state_out) {
            float *sp = a.state_out + ((size_t)unit * kP + p) * N + q * NQ;
#pragma unroll
            for (int j = 0; j < NQ; ++j) sp[j] = hs[j];
        }
    }
    if (!a.has_output) return;
    // both scans' outputs are in their buffers: out = y_f + y_b + (D_f + D_b) x
    __syncthreads();
    for (long long idx = threadIdx.x; idx < (long long)L * kP; idx += blockDim.x) {
        const int t = (int)(idx / kP), pp = (int)(idx - (long long)t * kP);
        const size_t o = ((size_t)(b * L + t) * a.H + h) * kP + pp;
        const float yb = a.ndir == 2 ? a.yacc[yplane + o] : 0.f;
        IO<T>::store(out + o, a.yacc[o] + yb + dsum * IO<T>::load(x + o));
    }
}

template <typename T, int N>
cudaError_t launch_t(const SimtArgs &a, cudaStream_t stream) {
    // both scans side by side while the units take one round of CTAs
    const int sms = device_sms();
    if (a.ndir == 2 && a.has_output && a.x_dir_stride == 0 && a.batch * a.H <= (sms > 0 ? sms : 148)) {
        const size_t smem = sizeof(float) * 2 * (size_t)stage_floats<N>();
        auto kern = scan_simt_pair_kernel<T, N>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<a.batch * a.H, 2 * kHalf, smem, stream>>>(a);
        return cudaGetLastError();
    }
    return launch_seq<T, N>(a, stream);
}

}  // namespace

cudaError_t launch_scan_simt(const SimtArgs &a, bool bf16, int N, cudaStream_t stream) {
    if (a.batch * a.H == 0 || a.L == 0) {
        // Empty sequences still define a state: copy (or zero) it.
        if (a.state_out && a.batch * a.H > 0) {
            const size_t bytes = sizeof(float) * (size_t)a.batch * a.H * kP * N;
            if (a.init) {
                if (a.init == a.state_out) return cudaSuccess;
                return cudaMemcpyAsync(a.state_out, a.init, bytes, cudaMemcpyDeviceToDevice, stream);
            }
            return cudaMemsetAsync(a.state_out, 0, bytes, stream);
        }
        return cudaSuccess;
    }
    if (bf16) {
        return N == 64 ? launch_t<__nv_bfloat16, 64>(a, stream) : launch_t<__nv_bfloat16, 128>(a, stream);
    }
    return N == 64 ? launch_t<float, 64>(a, stream) : launch_t<float, 128>(a, stream);
}

}  // namespace ssd
