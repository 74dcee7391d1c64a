// Bidirectional scan of long sequences split into segments, for batches with
// fewer (batch, head) units than SMs: the fused kernel takes one unit per SM,
// so a few long sequences would leave most SMs idle. Each sequence is viewed
// as S consecutive segments (the row-major tensors reshape for free to
// batch*S sequences of L/S tokens) and:
//   1. the fused kernel's forward state mode gives each segment's forward
//      state at its end, from zero;
//   2. its reverse state mode gives each segment's reverse state at its
//      start, from zero;
//   3. seg_scan_kernel turns those into the state entering each segment from
//      the left (forward) and from the right (reverse):
//        Hf_in(s) = sum_{r<s} (prod_{r<q<s} g_f(q)) Sf(r),
//        Hb_in(s) = sum_{r>s} (prod_{s<q<r} g_b(q)) Sb(r),
//      with g(q) = exp(A sum of dt over segment q), which the state passes
//      also return (the product of their tile decays); given starting states
//      of the whole sequence (a segment of a longer one) enter as the term
//      from beyond its ends;
//   4. the two-CTA kernel (the fused kernel where the segments are too long
//      or too short for it) runs on the segments, its forward scan seeded
//      with Hf_in and its reverse scan with Hb_in.
// The recurrence is linear in the state, so this equals the scan over the
// whole sequence up to rounding. The pages describe no such split (they run
// 65K-token full-sequence denoising: "Training Hybrid Block Diffusion
// Language Models with Partial Bidirectionality", Key Results); it is the
// plain consequence of the recurrence, used here to spread a few long
// sequences over all SMs.
#include <cuda_bf16.h>
#include <stdint.h>

#include "ssd_common.cuh"
#include "ssd_kernels.h"

namespace ssd {
namespace {

constexpr int kP = 64;
constexpr int kMaxSeg = 64;
constexpr int kScanThreads = 256;

// grid (batch * H, 2 directions, N * 64 / 1024), 256 threads, one float4 of
// the state per thread; Gf, Gb: each segment's decay exp(A * sum of dt over
// the segment), from the state passes. H0f, H0b (batch, H, 64, N) or nullptr:
// the forward state before the sequence and the reverse state after it. The
// segments' states are loaded eight at a time before the chain over them, so
// a thread waits for one round trip per eight segments, not one per segment.
__global__ void __launch_bounds__(kScanThreads) seg_scan_kernel(const float *Sf, const float *Sb, const float *Gf,
                                                                const float *Gb, const float *H0f, const float *H0b,
                                                                float *Hf, float *Hb, int H, int S, int N) {
    const int u = blockIdx.x, dir = blockIdx.y;
    const int b = u / H, h = u % H;
    const int elems = kP * N;
    const int e = (blockIdx.z * kScanThreads + threadIdx.x) * 4;
    if (e >= elems) return;
    const float *sin = dir ? Sb : Sf;
    const float *gin = dir ? Gb : Gf;
    const float *h0 = dir ? H0b : H0f;
    float *hout = dir ? Hb : Hf;
    float4 acc = h0 ? *reinterpret_cast<const float4 *>(h0 + (size_t)u * elems + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int kBatch = 8;
    for (int k0 = 0; k0 < S; k0 += kBatch) {
        float4 v[kBatch];
        float g[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (k0 + j < S) {
                const int seg = dir ? S - 1 - (k0 + j) : k0 + j;
                const size_t su = (size_t)(b * S + seg) * H + h;   // segment unit of the reshaped batch
                v[j] = *reinterpret_cast<const float4 *>(sin + su * elems + e);
                g[j] = gin[su];
            }
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (k0 + j < S) {
                const int seg = dir ? S - 1 - (k0 + j) : k0 + j;
                const size_t su = (size_t)(b * S + seg) * H + h;
                *reinterpret_cast<float4 *>(hout + su * elems + e) = acc;
                acc = make_float4(fmaf(g[j], acc.x, v[j].x), fmaf(g[j], acc.y, v[j].y), fmaf(g[j], acc.z, v[j].z),
                                  fmaf(g[j], acc.w, v[j].w));
            }
        }
    }
}

// grid (batch * H, 2 directions, elems / 1024), 256 threads, one float4 of
// the state per thread. From the end states S and decays g of all nseg
// segments of a sequence, laid out segment-major (S (nseg, batch, H, P, N),
// g (nseg, batch, H)), the state entering segment `seg`: from the left,
// Hf = sum_{q<seg} (prod_{q<r<seg} g_f(r)) S_f(q); from the right,
// Hb = sum_{q>seg} (prod_{seg<r<q} g_b(r)) S_b(q). The same recurrence as
// seg_scan_kernel, for segments that sit on other GPUs.
__global__ void __launch_bounds__(kScanThreads) seg_carry_kernel(const float *Sf, const float *Gf, const float *Sb,
                                                                 const float *Gb, float *Hf, float *Hb, int units,
                                                                 int nseg, int seg, int elems) {
    const int u = blockIdx.x, dir = blockIdx.y;
    const int e = (blockIdx.z * kScanThreads + threadIdx.x) * 4;
    if (e >= elems) return;
    const float *sin = dir ? Sb : Sf;
    const float *gin = dir ? Gb : Gf;
    const int first = dir ? nseg - 1 : 0, last = seg, step = dir ? -1 : 1;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int q = first; q != last; q += step) {
        const size_t su = (size_t)q * units + u;
        const float4 v = *reinterpret_cast<const float4 *>(sin + su * elems + e);
        const float g = gin[su];
        acc = make_float4(fmaf(g, acc.x, v.x), fmaf(g, acc.y, v.y), fmaf(g, acc.z, v.z), fmaf(g, acc.w, v.w));
    }
    *reinterpret_cast<float4 *>((dir ? Hb : Hf) + (size_t)u * elems + e) = acc;
}

// grid (batch * H, 2 directions), 256 threads. From the S segments' own
// states and decays (reshaped-batch layout, as seg_scan_kernel), the whole
// sequence's: forward state after its last token, reverse state before its
// first, and the two decays (the products of the segments').
__global__ void __launch_bounds__(kScanThreads) seg_total_kernel(const float *Sf, const float *Sb, const float *Gf,
                                                                 const float *Gb, float *Tf, float *Tb, float *Df,
                                                                 float *Db, int H, int S, int N) {
    const int u = blockIdx.x, dir = blockIdx.y;
    const int b = u / H, h = u % H;
    const float *sin = dir ? Sb : Sf;
    const float *gin = dir ? Gb : Gf;
    float *tout = (dir ? Tb : Tf) + (size_t)u * kP * N;
    const int elems = kP * N;
    for (int e = threadIdx.x * 4; e < elems; e += kScanThreads * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < S; ++k) {
            const int seg = dir ? S - 1 - k : k;
            const size_t su = (size_t)(b * S + seg) * H + h;
            const float4 v = *reinterpret_cast<const float4 *>(sin + su * elems + e);
            const float g = gin[su];
            acc = make_float4(fmaf(g, acc.x, v.x), fmaf(g, acc.y, v.y), fmaf(g, acc.z, v.z), fmaf(g, acc.w, v.w));
        }
        *reinterpret_cast<float4 *>(tout + e) = acc;
    }
    if (threadIdx.x == 0) {
        float g = 1.f;
        for (int k = 0; k < S; ++k) g *= gin[(size_t)(b * S + k) * H + h];
        (dir ? Db : Df)[u] = g;
    }
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct SegLayout {
    size_t fused, states, decays, total;   // fused kernel scratch, then Sf, Sb, Hf, Hb, then Gf, Gb
};

// the segments' kernel for the last step: the two-CTA kernel when it takes
// segments of this length
bool seg_pair(int batch, int L, int H, int G, int N, int S) {
    return tc_pair_supported(batch * S, L / S, H, G, N);
}

SegLayout seg_layout(int batch, int L, int H, int N, int S) {
    SegLayout l;
    const size_t f = tc_fused_scratch_bytes(batch * S, L / S, H, N);
    const size_t q = tc_pair_supported(batch * S, L / S, H, 1, N) ? tc_pair_scratch_bytes(batch * S, L / S, H, N) : 0;
    l.fused = align256(f > q ? f : q);
    l.states = align256((size_t)batch * S * H * kP * N * sizeof(float));
    l.decays = align256((size_t)batch * S * H * sizeof(float));
    l.total = l.fused + 4 * l.states + 2 * l.decays;
    return l;
}

}  // namespace

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

int seg_count(long long units, int L, int sms) {
    if (sms <= 0 || units >= sms || L < 2 * 128) return 1;
    // segments of 2..256 tiles run on the two-CTA kernel, one cluster of two
    // SMs each: the S (dividing L) with the lowest estimated time, the fewest
    // segments on ties. The estimate: rounds of segments over the clusters
    // times (tiles per segment + 3, the pipeline's fill and drain per
    // segment), plus the two state passes (one CTA per segment and SM, a tile
    // there costing about 0.3 of a two-CTA step). Measured on 32 x 65536
    // tokens: S = 16 1.065 ms, 4 1.137, 8 1.143, 32 1.105, 64 1.266; on
    // 32 x 16384: S = 4 0.300 ms, 8 0.308, 16 0.315, 32 0.412
    {
        const long long ncl = sms / 2 > 0 ? sms / 2 : 1;
        int best = 0;
        long long best_cost = 0;
        for (int S = 2; S <= kMaxSeg; ++S) {
            if (L % S) continue;
            const long long nt = (L / S + 127) / 128;
            if (nt < 2 || nt > 256 || L / S <= 128) continue;
            const long long rp = (units * S + ncl - 1) / ncl, rf = (units * S + sms - 1) / sms;
            const long long cost = 5 * rp * (nt + 3) + 3 * rf * nt;
            if (!best || cost < best_cost) {
                best = S;
                best_cost = cost;
            }
        }
        if (best) return best;
    }
    // else the fewest segments that give one round of the fused kernel over
    // at least 4/5 of the SMs: every segment adds its own state passes and
    // pass boundaries, and measured on 32 x 65536 tokens, 4 segments (128
    // units) beat 8, 16, 32 and 64 (1.12 ms against 1.22 to 1.47 ms)
    int last = 1;
    for (int S = 2; S <= kMaxSeg && L / S >= 128; ++S) {
        if (L % S) continue;
        if (units * S * 5 >= 4LL * sms) return S;
        last = S;
    }
    return last;
}

size_t tc_segmented_scratch_bytes(int batch, int L, int H, int N) {
    size_t m = 0;
    for (int S = 2; S <= kMaxSeg && L / S >= 128; ++S) {
        if (L % S) continue;
        const size_t t = seg_layout(batch, L, H, N, S).total;
        m = t > m ? t : m;
    }
    return m;
}

// The forward and reverse state passes read the same x. With units enough
// for both halves of the GPU they run side by side, each on half the SMs: the
// reverse pass is released only once the forward pass's wait for the kernel
// ahead is over and does not wait itself, so the two CTAs on a unit run at the
// same time and the second read of each x tile comes from L2.
static void share_state_passes(TcArgs &f, TcArgs &r) {
    const int sms = device_sms();
    if (sms < 2 || (long long)f.batch * f.H < sms) return;
    f.grid_cap = sms / 2;
    f.launch_order = 1;
    r.grid_cap = sms - sms / 2;
    r.launch_order = 2;
}

cudaError_t launch_tc_segmented(const TcArgs &a, int S, cudaStream_t stream) {
    if (S < 2 || S > kMaxSeg || a.L % S || a.L / S < 1 || a.ndir != 2) return cudaErrorNotSupported;
    const SegLayout lay = seg_layout(a.batch, a.L, a.H, a.N, S);
    if (a.ws_bytes < kStatusBytes + lay.total) return cudaErrorInvalidValue;
    char *scratch = static_cast<char *>(a.workspace) + kStatusBytes;
    float *Sf = reinterpret_cast<float *>(scratch + lay.fused);
    float *Sb = reinterpret_cast<float *>(scratch + lay.fused + lay.states);
    float *Hf = reinterpret_cast<float *>(scratch + lay.fused + 2 * lay.states);
    float *Hb = reinterpret_cast<float *>(scratch + lay.fused + 3 * lay.states);
    float *Gf = reinterpret_cast<float *>(scratch + lay.fused + 4 * lay.states);
    float *Gb = reinterpret_cast<float *>(scratch + lay.fused + 4 * lay.states + lay.decays);
    TcArgs v = a;             // the segments as a batch of batch * S sequences of L / S tokens
    v.batch = a.batch * S;
    v.L = a.L / S;
    v.init = nullptr;
    v.rinit = nullptr;
    cudaError_t e;
    TcArgs f = v;
    f.state_out = Sf;
    f.decay_out = Gf;
    TcArgs r = v;
    r.state_out = Sb;
    r.decay_out = Gb;
    share_state_passes(f, r);
    if ((e = launch_tc_fused_state(f, stream)) != cudaSuccess) return e;
    if ((e = launch_tc_fused_state_rev(r, stream)) != cudaSuccess) return e;
    // launched without programmatic serialization: waits for both passes
    const int zb = (kP * a.N + kScanThreads * 4 - 1) / (kScanThreads * 4);
    seg_scan_kernel<<<dim3(a.batch * a.H, 2, zb), kScanThreads, 0, stream>>>(Sf, Sb, Gf, Gb, a.init, a.rinit, Hf, Hb,
                                                                            a.H, S, a.N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    TcArgs o = v;
    o.init = Hf;
    o.rinit = Hb;
    if (seg_pair(a.batch, a.L, a.H, a.G, a.N, S)) return launch_tc_pair(o, stream);
    return launch_tc_fused(o, stream);
}

}  // namespace ssd

namespace ssd {

cudaError_t launch_seg_carry(const float *Sf, const float *Gf, const float *Sb, const float *Gb, float *Hf, float *Hb,
                             int batch, int H, int N, int nseg, int seg, cudaStream_t stream) {
    const int units = batch * H;
    if (units <= 0) return cudaSuccess;
    const int elems = kP * N;
    const int zb = (elems + kScanThreads * 4 - 1) / (kScanThreads * 4);
    seg_carry_kernel<<<dim3(units, 2, zb), kScanThreads, 0, stream>>>(Sf, Gf, Sb, Gb, Hf, Hb, units, nseg, seg, elems);
    return cudaGetLastError();
}

cudaError_t launch_tc_segment_totals(const TcArgs &a, int S, float *fwd_state, float *fwd_decay, float *rev_state,
                                     float *rev_decay, cudaStream_t stream) {
    if (S < 2 || S > kMaxSeg || a.L % S || a.ndir != 2) return cudaErrorNotSupported;
    const SegLayout lay = seg_layout(a.batch, a.L, a.H, a.N, S);
    if (a.ws_bytes < kStatusBytes + lay.total) return cudaErrorInvalidValue;
    char *scratch = static_cast<char *>(a.workspace) + kStatusBytes;
    float *Sf = reinterpret_cast<float *>(scratch + lay.fused);
    float *Sb = reinterpret_cast<float *>(scratch + lay.fused + lay.states);
    float *Gf = reinterpret_cast<float *>(scratch + lay.fused + 4 * lay.states);
    float *Gb = reinterpret_cast<float *>(scratch + lay.fused + 4 * lay.states + lay.decays);
    TcArgs v = a;             // the segments as a batch of batch * S sequences of L / S tokens
    v.batch = a.batch * S;
    v.L = a.L / S;
    v.init = nullptr;
    v.rinit = nullptr;
    cudaError_t e;
    TcArgs f = v;
    f.state_out = Sf;
    f.decay_out = Gf;
    TcArgs r = v;
    r.state_out = Sb;
    r.decay_out = Gb;
    share_state_passes(f, r);
    if ((e = launch_tc_fused_state(f, stream)) != cudaSuccess) return e;
    if ((e = launch_tc_fused_state_rev(r, stream)) != cudaSuccess) return e;
    // launched without programmatic serialization: waits for both passes
    seg_total_kernel<<<dim3(a.batch * a.H, 2), kScanThreads, 0, stream>>>(Sf, Sb, Gf, Gb, fwd_state, rev_state,
                                                                         fwd_decay, rev_decay, a.H, S, a.N);
    return cudaGetLastError();
}

}  // namespace ssd
