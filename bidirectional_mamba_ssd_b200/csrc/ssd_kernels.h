// Internal launch interface between the C ABI (ssd_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "ssd_common.cuh"

namespace ssd {

// Arguments of the sequential CUDA-core scan (ssd_simt.cu).
struct SimtArgs {
    const void *x;            // (batch, L, H, 64) io
    const void *dt;           // direction 0 base; + dir * dt_dir_stride elements
    const float *A;           // A[dir * A_dir_stride + h]
    const void *B;            // direction 0 base; + dir * bc_dir_stride elements
    const void *C;            // as B; nullptr when no output is read
    const float *D;           // (2, H) when has_output
    const float *init;        // (batch, H, 64, N) start of the forward scan, or nullptr
    float *state_out;         // (batch, H, 64, N) final forward state, or nullptr
    void *out;                // (batch, L, H, 64) io when has_output
    float *yacc;              // (batch, L, H, 64) fp32 scratch for the forward partial
    long long dt_dir_stride, bc_dir_stride;
    int A_dir_stride;
    // elements between the two directions' x when each direction scans its own
    // x (x then holds (2, batch, L, H, 64)); 0 = one x for both directions
    long long x_dir_stride = 0;
    int batch, L, H, G;
    int ndir;                 // 1: forward only, 2: forward + reverse
    int has_output;
};

cudaError_t launch_scan_simt(const SimtArgs &a, bool bf16, int N, cudaStream_t stream);

// Arguments of the tensor-core kernels (ssd_tc.cu). bf16 I/O only.
struct TcArgs {
    const void *x;            // (batch, L, H, 64) bf16
    const void *dt;           // (2, batch, L, H) bf16 (forward only: (batch, L, H))
    const float *A;           // (2, H) (forward only: (H))
    const void *B;            // (2, batch, L, G, N) bf16
    const void *C;            // (2, batch, L, G, N) bf16 or nullptr
    const float *D;           // (2, H)
    const float *init;        // (batch, H, 64, N) forward start state or nullptr
    const float *rinit = nullptr;  // (batch, H, 64, N) reverse start state (at the sequence end) or nullptr
    float *decay_out = nullptr;    // (batch, H) fused state modes: exp(A * sum of dt) over the sequence
    const float *dt_bias = nullptr;  // (2, H) with launch_tc_fused_dtraw: dt holds the raw projection
    float dt_lo = 0.f, dt_hi = 0.f;  // with launch_tc_fused_dtraw: the step-size range
    // several layers stacked along the batch: units of layer l are
    // [l * layer_units, (l + 1) * layer_units) and read A (and D) from
    // A + l * A_layer (D + l * A_layer); 0 = one layer
    int layer_units = 0, A_layer = 0;
    // elements between the two directions' x when each scans its own x
    // (launch_tc_pair only; x then holds (2, batch, L, H, 64)); 0 = one x
    long long x_dir_stride = 0;
    // fused kernel only: at most this many CTAs (0 = one per SM), and the
    // launch order of its kernel (FusedParams::launch_order)
    int grid_cap = 0, launch_order = 0;
    float *state_out;         // (batch, H, 64, N) or nullptr
    void *out;                // (batch, L, H, 64) bf16
    void *workspace;          // status header + scratch
    size_t ws_bytes;
    int batch, L, H, G, N;
    int ndir;                 // 1 (prefix state) or 2
};

// Scratch bytes (after the status header) the tensor-core paths need.
size_t tc_chunked_scratch_bytes(int batch, int L, int H, int N, int ndir);
size_t tc_fused_scratch_bytes(int batch, int L, int H, int N);
bool tc_fused_supported(int batch, int L, int H, int G, int N);

cudaError_t launch_tc_chunked(const TcArgs &a, cudaStream_t stream);
// Fused kernel, both scans summed; with a.init the forward scan starts from
// that state (block step).
cudaError_t launch_tc_fused(const TcArgs &a, cudaStream_t stream);
// Fused kernel, both scans, with the step size prepared from the raw
// projection in the kernel: dt = clamp(softplus(dt_raw + a.dt_bias), a.dt_lo,
// a.dt_hi) for every token in the sequence (a.dt holds dt_raw).
cudaError_t launch_tc_fused_dtraw(const TcArgs &a, cudaStream_t stream);
// Fused kernel, forward scan only: the final state into a.state_out, from
// a.init or zero (prefix state); needs no scratch past the status header.
cudaError_t launch_tc_fused_state(const TcArgs &a, cudaStream_t stream);
// Fused kernel, reverse scan only (direction 1 of the direction-stacked
// inputs): the state at the sequence start into a.state_out, from zero.
cudaError_t launch_tc_fused_state_rev(const TcArgs &a, cudaStream_t stream);

// Input and output steps of the mixer block (ssd_block.cu).
struct BlockLaunch {
    const void *xbc;            // (batch, L, HP + 2 GN) io
    const float *conv_w;        // (2, HP + 2 GN, K)
    const float *conv_b;        // (2, HP + 2 GN)
    void *x2, *B2, *C2;         // (2, batch, L, HP), (2, batch, L, GN) io
    const void *dt_raw;         // (2, batch, L, H) io
    const float *dt_bias;       // (2, H)
    void *dt;                   // (2, batch, L, H) io
    const void *y, *z;          // (batch, L, HP) io
    const float *norm_w;        // (HP)
    void *out;                  // (batch, L, HP) io
    float dt_lo, dt_hi, eps;
    int batch, L, H, HP, GN, K;
    bool bf16;
};
cudaError_t launch_conv_silu(const BlockLaunch &l, cudaStream_t stream);
cudaError_t launch_dt_prep(const BlockLaunch &l, cudaStream_t stream);
cudaError_t launch_gated_rmsnorm(const BlockLaunch &l, cudaStream_t stream);

// Backward pass (ssd_bwd.cu): gradients of sum(dy * y) of the bidirectional
// mixer, fp32 outputs, any I/O dtype; persistent CTAs, each with L states of
// scratch.
struct BwdLaunch {
    const void *x, *dt, *B, *C, *dy;   // io dtype
    const float *A, *D;
    float *dx, *ddt, *dA, *dB, *dC, *dD;
    float *scratch;
    const float *init_f = nullptr, *init_b = nullptr;   // start states (batch, H, 64, N) or nullptr
    float *dinit_f = nullptr, *dinit_b = nullptr;        // their gradients, or nullptr
    int batch, L, H, G, N;
    bool bf16;
};
int bwd_grid(int batch, int H);
size_t bwd_scratch_bytes(int batch, int L, int H, int N);
cudaError_t launch_bwd(const BwdLaunch &l, cudaStream_t stream);

// Two-CTA kernel (ssd_pair.cu): each (batch, head) unit taken by a cluster of
// two CTAs, one per scan direction, meeting per tile through an fp32 partial
// in the workspace; both scans summed, a.init / a.rinit as launch_tc_fused.
// Sequences of at least two 128-token tiles.
size_t tc_pair_scratch_bytes(int batch, int L, int H, int N);
bool tc_pair_supported(int batch, int L, int H, int G, int N);
cudaError_t launch_tc_pair(const TcArgs &a, cudaStream_t stream);

// One-tile block step (ssd_blockstep.cu): both scans over a block of at most
// 64 tokens, forward from a.init (or zero), reverse from zero; bf16, ndir 2,
// one CTA per (batch, head). Needs only the workspace's status header.
bool tc_blockstep_supported(int batch, int T, int H, int G, int N);
cudaError_t launch_tc_blockstep(const TcArgs &a, cudaStream_t stream);

// One-tile sequences (ssd_onetile.cu): seqlen <= 128, both scans summed,
// bf16, ndir 2, no start states; persistent CTAs over runs of (batch, head)
// units, G = C B^T of each direction computed once per B/C group. Needs only
// the workspace's status header.
bool tc_onetile_supported(int batch, int L, int H, int G, int N);
cudaError_t launch_tc_onetile(const TcArgs &a, cudaStream_t stream);

// Long sequences with fewer (batch, head) units than SMs: each sequence split
// into S segments (seg_count: the fewest, S dividing L, that fill 4/5 of `sms`
// SMs in one round; 1 = none), states handed across segments,
// then the fused kernel on the segments.
int seg_count(long long units, int L, int sms);
size_t tc_segmented_scratch_bytes(int batch, int L, int H, int N);   // max over the S in use
cudaError_t launch_tc_segmented(const TcArgs &a, int S, cudaStream_t stream);
// The whole sequence's own end states and decays (as the fused state modes
// give them) from S segments' state passes and one combining kernel.
cudaError_t launch_tc_segment_totals(const TcArgs &a, int S, float *fwd_state, float *fwd_decay, float *rev_state,
                                     float *rev_decay, cudaStream_t stream);
int device_sms();   // SM count of the current device, 0 if it cannot be read
// The forward and reverse states entering segment `seg` of nseg, from every
// segment's own end states and decays (segment-major arrays; see
// seg_carry_kernel); Hf, Hb (batch, H, 64, N).
cudaError_t launch_seg_carry(const float *Sf, const float *Gf, const float *Sb, const float *Gb, float *Hf, float *Hb,
                             int batch, int H, int N, int nseg, int seg, cudaStream_t stream);

}  // namespace ssd
