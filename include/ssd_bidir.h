/*
 * ssd_bidir.h - C ABI of the bidirectional Mamba-2 SSD mixer for B200 (sm_100a).
 *
 * What the mixer computes, per batch element b, head h and direction
 * d in {forward, reverse} (head h reads B/C group g = h / (nheads/ngroups)):
 *
 *   forward,  t = 0 .. L-1:  h_t  = exp(dt_t A_h) h_{t-1}  + dt_t B_t x_t^T,  yf_t = C_t^T h_t
 *   reverse,  t = L-1 .. 0:  h'_t = exp(dt'_t A'_h) h'_{t+1} + dt'_t B'_t x_t^T, yb_t = C'_t^T h'_t
 *   out_t = yf_t + yb_t + (D_h + D'_h) x_t
 *
 * with an N x P state (N = dstate, P = headdim) starting at zero.
 *  - "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
 *    Technical Summary, 2. Methodology, Core Architecture: a forward and a
 *    backward Mamba-2 layer over the sequence, added.
 *  - "DiffMamba - Checkpoints" model card, Model details: the backward
 *    layer is Mamba-2 on the flipped sequence. The reverse scan here reads
 *    its inputs in natural token order from the right end, which is the
 *    same thing without materialising a flipped copy.
 *  - The pages name Mamba-2 without printing its recurrence; the scalar-
 *    decay selective SSM above is the standard Mamba-2 (SSD) definition.
 *  - "Training Hybrid Block Diffusion Language Models with Partial
 *    Bidirectionality", Abstract and Methodology: for block diffusion the
 *    reverse scan is confined to the active block, so the forward state of
 *    the prefix is a cache that is reused exactly (ssd_prefix_state,
 *    ssd_block_step).
 *
 * Conventions for every entry point
 *  - All tensor arguments are DEVICE pointers to dense row-major arrays in
 *    natural token order, 16-byte aligned. The caller allocates and owns
 *    every buffer, the workspace included; the library allocates nothing,
 *    keeps no global state and never synchronises (except
 *    ssd_get_device_status).
 *  - "io" = the I/O dtype chosen by `dtype` (SSD_F32 or SSD_BF16): x, dt,
 *    B, C and out use it. A, D and states are always fp32.
 *  - Direction-stacked tensors have a leading dimension of 2:
 *    [0] = forward, [1] = reverse.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *    enqueued on it; results are ready when the stream reaches that point.
 *  - Arguments are checked on the host before anything is launched; a bad
 *    argument returns an error code and launches nothing. Launch failures
 *    return SSD_ERR_CUDA. A device-side wait that ran out of its iteration
 *    bound sets a flag in the workspace header that ssd_get_device_status
 *    reports; the kernel then returns without finishing its output.
 *  - Supported in this version: headdim == 64, dstate in {64, 128},
 *    nheads % ngroups == 0, chunk in {64, 128, 256}, seqlen >= 0 (no
 *    multiple-of-chunk requirement). Other shapes return
 *    SSD_ERR_UNSUPPORTED.
 *  - chunk is the chunk length of the chunked evaluation. The result does
 *    not depend on it beyond floating-point rounding. The fp32 path runs a
 *    sequential scan and ignores it; the bf16 tensor-core path evaluates
 *    128-token tiles (see each function).
 *  - Calls that share a workspace must not overlap on the device.
 */
#ifndef SSD_BIDIR_H
#define SSD_BIDIR_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* I/O element type. */
enum {
    SSD_F32 = 0,  /* IEEE fp32 */
    SSD_BF16 = 1  /* bfloat16; outputs rounded to nearest-even once, at the final store */
};

/* Status codes. */
enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, negative size, ngroups not dividing nheads */
    SSD_ERR_UNSUPPORTED = -2,   /* valid but not implemented: headdim, dstate, chunk, dtype */
    SSD_ERR_CUDA = -3,          /* a CUDA launch or driver call failed (cudaGetLastError) */
    SSD_ERR_WORKSPACE = -4,     /* workspace NULL or smaller than ssd_workspace_bytes() */
    SSD_ERR_TIMEOUT = -5        /* a bounded device-side wait expired (from ssd_get_device_status) */
};

/* Operation ids for ssd_workspace_bytes. */
enum {
    SSD_OP_BIDIR_FWD = 0, SSD_OP_PREFIX_STATE = 1, SSD_OP_BLOCK_STEP = 2, SSD_OP_BIDIR_BWD = 3,
    SSD_OP_BIDIR_FWD_X2 = 4, SSD_OP_MIXER_BLOCK = 5
};

/* Kernel selection for ssd_bidir_fwd_path (tests and benchmarks). */
enum {
    SSD_PATH_AUTO = 0,     /* what ssd_bidir_fwd uses */
    SSD_PATH_SIMT = 1,     /* sequential fp32 scan on CUDA cores, any dtype */
    SSD_PATH_CHUNKED = 2,  /* tensor-core chunked path in three kernels (states through the workspace) */
    SSD_PATH_FUSED = 3,    /* tensor-core path, one kernel per (batch, head) */
    SSD_PATH_SEGMENTED = 4, /* long sequences, few (batch, head): each sequence split into S
                              segments (S divides seqlen); forward and reverse segment states
                              (fused kernel, state modes), a segment scan, then the fused
                              kernel on the segments seeded with the handed-over states */
    SSD_PATH_PAIR = 5,     /* tensor-core path, one cluster of two CTAs per (batch, head):
                              each CTA runs one scan direction over the tiles in that
                              direction's order, carrying its state on chip; a tile's two
                              directions meet through an fp32 partial in the workspace.
                              128 < seqlen <= 32768 (2 to 256 128-token tiles) */
    SSD_PATH_BLOCK = 6,    /* ssd_block_step only: one CTA per (batch, head) over a block of at
                              most 64 tokens, both directions stacked as the rows of one
                              tensor-core tile */
    SSD_PATH_ONETILE = 7   /* bf16, seqlen <= 128 (one tensor-core tile), dstate 64 or 128:
                              each CTA takes a run of (batch, head) units, computes both
                              directions' C B^T once per B/C group and reuses it for every
                              head of the group (mask and one MMA per head); what
                              SSD_PATH_AUTO runs for these sizes */
};

/* The SSD_PATH_* that ssd_bidir_fwd (SSD_PATH_AUTO) runs for these sizes, or
 * a negative status for arguments it rejects. Host only; launches nothing. */
int ssd_select_path(int batch, int seqlen, int nheads, int headdim, int dstate,
                    int ngroups, int chunk, int dtype);

/* Bytes of device workspace the operation needs for these sizes (always at
 * least the 256-byte status header). `seqlen` is the block length for
 * SSD_OP_BLOCK_STEP. Returns 0 for arguments the operation rejects. */
size_t ssd_workspace_bytes(int op, int batch, int seqlen, int nheads, int headdim,
                           int dstate, int ngroups, int chunk, int dtype);

/* Zero the workspace's status header (256 bytes) on `stream`. A workspace
 * must be initialised once before first use (zero-filled memory counts). */
int ssd_workspace_init(void *workspace, size_t ws_bytes, void *stream);

/* Full-sequence bidirectional mixer (both scans over the whole sequence).
 *   x    (batch, seqlen, nheads, headdim)           io
 *   dt   (2, batch, seqlen, nheads)                 io, > 0 (already softplus'ed; used as given)
 *   A    (2, nheads)                                fp32, <= 0
 *   B, C (2, batch, seqlen, ngroups, dstate)        io
 *   D    (2, nheads)                                fp32
 *   out  (batch, seqlen, nheads, headdim)           io, overwritten; must not alias an input
 * bf16 I/O runs the tensor-core path: state and accumulation fp32, the
 * decay-masked C.B^T tile and the chunk states rounded to bf16 as MMA
 * operands. fp32 I/O runs the sequential fp32 scan.
 * Source: "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
 * Technical Summary, 2. Methodology, Core Architecture. */
int ssd_bidir_fwd(const void *x, const void *dt, const float *A, const void *B,
                  const void *C, const float *D, void *out,
                  int batch, int seqlen, int nheads, int headdim, int dstate,
                  int ngroups, int chunk, int dtype,
                  void *workspace, size_t ws_bytes, void *stream);

/* ssd_bidir_fwd with an explicit kernel choice (SSD_PATH_*). A path that
 * cannot run these arguments returns SSD_ERR_UNSUPPORTED. The workspace
 * must be at least ssd_workspace_bytes(SSD_OP_BIDIR_FWD, ...). */
int ssd_bidir_fwd_path(const void *x, const void *dt, const float *A, const void *B,
                       const void *C, const float *D, void *out,
                       int batch, int seqlen, int nheads, int headdim, int dstate,
                       int ngroups, int chunk, int dtype, int path,
                       void *workspace, size_t ws_bytes, void *stream);

/* Forward-only state after the last token of each sequence: the cache that
 * block diffusion reuses ("Training Hybrid Block Diffusion Language Models
 * with Partial Bidirectionality", Abstract: prefix-only states reused
 * exactly; Technical Contribution: timestep-free prefix cache).
 *   x          (batch, seqlen, nheads, headdim)     io
 *   dt         (batch, seqlen, nheads)              io, forward direction only
 *   A          (nheads)                             fp32
 *   B          (batch, seqlen, ngroups, dstate)     io
 *   init_state (batch, nheads, headdim, dstate)     fp32, NULL = zero start
 *   state_out  (batch, nheads, headdim, dstate)     fp32; may equal init_state (in-place update,
 *                                                   e.g. committing a finished block)
 * The state is stored as headdim rows of dstate values: state[b][h][p][n] = h[n][p].
 * bf16 I/O runs on the tensor cores: with at least 64 (batch, head) units the
 * fused kernel (one unit per SM at a time, all its tiles in one launch, no
 * scratch past the status header), else the tile-parallel chunked kernels;
 * fp32 I/O and seqlen 0 run the sequential fp32 scan. */
int ssd_prefix_state(const void *x, const void *dt, const float *A, const void *B,
                     const float *init_state, float *state_out,
                     int batch, int seqlen, int nheads, int headdim, int dstate,
                     int ngroups, int chunk, int dtype,
                     void *workspace, size_t ws_bytes, void *stream);

/* ssd_prefix_state with an explicit kernel choice (tests and benchmarks):
 * SSD_PATH_AUTO, SSD_PATH_SIMT, SSD_PATH_CHUNKED or SSD_PATH_FUSED; the last
 * two take bf16 I/O only (else SSD_ERR_UNSUPPORTED). */
int ssd_prefix_state_path(const void *x, const void *dt, const float *A, const void *B,
                          const float *init_state, float *state_out,
                          int batch, int seqlen, int nheads, int headdim, int dstate,
                          int ngroups, int chunk, int dtype, int path,
                          void *workspace, size_t ws_bytes, void *stream);

/* One denoising step on the active block of blk_len tokens: the forward scan
 * starts from the cached prefix state, the reverse scan starts from zero at
 * the block's right end and sees only the block ("Training Hybrid Block
 * Diffusion Language Models with Partial Bidirectionality", Methodology and
 * Key Results: the reverse scan is restricted to the active block so states
 * stay prefix-only). prefix_state is only read.
 *   x            (batch, blk_len, nheads, headdim)        io
 *   dt           (2, batch, blk_len, nheads)              io
 *   A, D         (2, nheads)                              fp32
 *   B, C         (2, batch, blk_len, ngroups, dstate)     io
 *   prefix_state (batch, nheads, headdim, dstate)         fp32, NULL = zero prefix
 *   out          (batch, blk_len, nheads, headdim)        io, overwritten
 * bf16 I/O runs on the tensor cores (the prefix state enters the C.H product
 * as a bf16 operand): blocks of at most 64 tokens on the one-tile kernel
 * (SSD_PATH_BLOCK), longer blocks with at least 64 (batch, head) units on the
 * fused bidirectional kernel with its forward scan seeded from prefix_state,
 * else on the chunked kernels; fp32 I/O runs the sequential fp32 scan. */
int ssd_block_step(const void *x, const void *dt, const float *A, const void *B,
                   const void *C, const float *D, const float *prefix_state, void *out,
                   int batch, int blk_len, int nheads, int headdim, int dstate,
                   int ngroups, int dtype,
                   void *workspace, size_t ws_bytes, void *stream);

/* ssd_block_step with an explicit kernel choice, as ssd_prefix_state_path:
 * SSD_PATH_AUTO, SIMT, CHUNKED, FUSED or BLOCK (bf16, blk_len <= 64;
 * SSD_ERR_UNSUPPORTED otherwise). */
int ssd_block_step_path(const void *x, const void *dt, const float *A, const void *B,
                        const void *C, const float *D, const float *prefix_state, void *out,
                        int batch, int blk_len, int nheads, int headdim, int dstate,
                        int ngroups, int dtype, int path,
                        void *workspace, size_t ws_bytes, void *stream);

/* ssd_bidir_fwd with the step size prepared inside the kernel from the raw
 * dt projection of a Mamba-2 layer:
 *   dt = min(max(softplus(dt_raw + dt_bias[d][h]), dt_min), dt_max),
 *   softplus(u) = log(1 + exp(u)),
 * for every token of every sequence (the pages name Mamba-2 without printing
 * its parametrisation; this is the standard Mamba-2 one, the input side of
 * the mixer). It saves writing and reading back a prepared dt tensor.
 *   dt_raw   (2, batch, seqlen, nheads)  io (bf16), the raw projection
 *   dt_bias  (2, nheads)                 fp32
 *   dt_min, dt_max                       0 <= dt_min <= dt_max (INFINITY for no upper bound)
 * Other arguments as ssd_bidir_fwd. bf16 I/O only (the fused kernel, for any
 * number of (batch, head) units); fp32 returns SSD_ERR_UNSUPPORTED. Workspace:
 * at least ssd_workspace_bytes(SSD_OP_BIDIR_FWD, ..., chunk 64, SSD_BF16). */
int ssd_bidir_fwd_dtraw(const void *x, const void *dt_raw, const float *dt_bias, float dt_min, float dt_max,
                        const float *A, const void *B, const void *C, const float *D, void *out,
                        int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                        int dtype, void *workspace, size_t ws_bytes, void *stream);

/* Sequences split across GPUs (or any other split into segments): each
 * holder of one segment of every sequence computes its segment's own states,
 * the holders exchange them (one all-gather of nseg x (2 states + 2 decays)
 * per (batch, head)), and each then runs its segment seeded with the states
 * the rest of the sequence leaves. The recurrence is linear in the state, so
 * this is the whole-sequence mixer up to rounding: the state entering a
 * segment is the sum of the earlier segments' end states, each decayed over
 * the segments in between ("Training Hybrid Block Diffusion Language Models
 * with Partial Bidirectionality", Key Results: full-sequence denoising at
 * 65K and 262K tokens; the pages describe no split across GPUs, only the
 * lengths). bf16 I/O only (the fused kernel's state and seeded modes); fp32
 * returns SSD_ERR_UNSUPPORTED. With too few (batch, head) units to fill the
 * GPU, both calls split each local sequence further into segments, as
 * SSD_PATH_SEGMENTED does. Workspace: at least
 * ssd_workspace_bytes(SSD_OP_BIDIR_FWD, ..., chunk 64, SSD_BF16) for
 * ssd_segment_states and ssd_bidir_fwd_seeded. */

/* A segment's own states, each scan starting from zero at its own end:
 *   x, dt, A, B  as for ssd_bidir_fwd over the segment (seqlen >= 1)
 *   fwd_state    (batch, nheads, headdim, dstate) fp32: forward state after the segment's last token
 *   fwd_decay    (batch, nheads) fp32: exp(A_f[h] * sum of dt_f over the segment)
 *   rev_state    (batch, nheads, headdim, dstate) fp32: reverse state before its first token
 *   rev_decay    (batch, nheads) fp32: exp(A_b[h] * sum of dt_b over the segment)
 * States are stored as headdim rows of dstate values, as ssd_prefix_state's. */
int ssd_segment_states(const void *x, const void *dt, const float *A, const void *B,
                       float *fwd_state, float *fwd_decay, float *rev_state, float *rev_decay,
                       int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                       int dtype, void *workspace, size_t ws_bytes, void *stream);

/* The states entering segment `seg` (0 <= seg < nseg) from the gathered
 * states of all nseg segments, segment-major: fwd_states / rev_states
 * (nseg, batch, nheads, headdim, dstate), fwd_decays / rev_decays
 * (nseg, batch, nheads), all fp32 as ssd_segment_states writes them.
 *   fwd_in (batch, nheads, headdim, dstate): forward state before the segment
 *          (zero for seg 0)
 *   rev_in (batch, nheads, headdim, dstate): reverse state after the segment
 *          (zero for seg nseg - 1)
 * No workspace. */
int ssd_segment_carry(const float *fwd_states, const float *fwd_decays, const float *rev_states,
                      const float *rev_decays, int nseg, int seg, float *fwd_in, float *rev_in,
                      int batch, int nheads, int headdim, int dstate, void *stream);

/* Both scans over a segment with given starting states: the forward scan
 * from fwd_init (state before the first token), the reverse scan from
 * rev_init (reverse state after the last token); NULL = zero. Other
 * arguments as ssd_bidir_fwd; out (batch, seqlen, nheads, headdim) io. The
 * starting states enter the C.H products as bf16 operands. */
int ssd_bidir_fwd_seeded(const void *x, const void *dt, const float *A, const void *B,
                         const void *C, const float *D, const float *fwd_init, const float *rev_init,
                         void *out, int batch, int seqlen, int nheads, int headdim, int dstate,
                         int ngroups, int dtype, void *workspace, size_t ws_bytes, void *stream);

/* The bidirectional mixer with each direction scanning its own x (the mixer
 * of a layer whose two directions have their own input conv, see
 * ssd_mixer_block_fwd):
 *   out_t = yf_t(x2[0]) + yb_t(x2[1]) + D_f x2[0]_t + D_b x2[1]_t
 *   x2   (2, batch, seqlen, nheads, headdim)   io; other arguments as ssd_bidir_fwd
 * bf16 with 128 < seqlen <= 32768 runs the two-CTA tensor-core kernel, otherwise the
 * sequential scan. The two directions' fp32 results are added in an order
 * that does not depend on which direction finishes first. */
int ssd_bidir_fwd_x2(const void *x2, const void *dt, const float *A, const void *B, const void *C,
                     const float *D, void *out, int batch, int seqlen, int nheads, int headdim,
                     int dstate, int ngroups, int dtype, void *workspace, size_t ws_bytes, void *stream);

/* A bidirectional Mamba-2 mixer with its input and output steps ("DiffMamba
 * - Checkpoints" model card, Model details: forward and flipped-reverse
 * Mamba-2 layers with weight-tied projections, Mamba-2 defaults; the pages
 * print none of these steps, so they are the standard Mamba-2 ones, read for
 * two directions):
 *   1. u_d = SiLU(conv1d_d(xbc) + conv_b_d), depthwise over the channels, causal
 *      for d = forward, anti-causal (the flipped sequence's causal conv) for
 *      d = reverse; split into x_d (H*P), B_d (G*N), C_d (G*N);
 *   2. dt_d = clamp(softplus(dt_raw_d + dt_bias_d), dt_min, dt_max);
 *   3. y = ssd_bidir_fwd_x2(x_d, dt, A, B, C, D);
 *   4. out = y SiLU(z) / sqrt(mean_c((y SiLU(z))^2) + norm_eps) * norm_w over
 *      the H*P channels of each token.
 *   xbc     (batch, seqlen, nheads*headdim + 2*ngroups*dstate)   io
 *   z       (batch, seqlen, nheads, headdim)                     io
 *   dt_raw  (2, batch, seqlen, nheads)                           io
 *   conv_w  (2, nheads*headdim + 2*ngroups*dstate, conv_k)       fp32, conv_k in 1..4
 *   conv_b  (2, nheads*headdim + 2*ngroups*dstate)               fp32
 *   dt_bias, A, D (2, nheads) fp32;  norm_w (nheads*headdim) fp32
 *   out     (batch, seqlen, nheads, headdim)                     io
 * The intermediates (u, dt, y) are stored in the I/O dtype in the workspace
 * (ssd_workspace_bytes with SSD_OP_MIXER_BLOCK). Four launches: conv, dt,
 * mixer, norm. */
int ssd_mixer_block_fwd(const void *xbc, const void *z, const void *dt_raw, const float *conv_w,
                        const float *conv_b, int conv_k, const float *dt_bias, float dt_min, float dt_max,
                        const float *A, const float *D, const float *norm_w, float norm_eps, void *out,
                        int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups, int dtype,
                        void *workspace, size_t ws_bytes, void *stream);

/* ssd_prefix_state for several layers at once (block diffusion keeps one
 * cached forward state per layer; "Training Hybrid Block Diffusion Language
 * Models with Partial Bidirectionality", Methodology: the states of the
 * prefix are reused exactly, so committing a finished block updates every
 * layer's cache). The layers' tensors are stacked along a leading dimension:
 *   x          (layers, batch, seqlen, nheads, headdim)   io
 *   dt         (layers, batch, seqlen, nheads)            io (forward direction)
 *   A          (layers, nheads)                           fp32 (forward direction)
 *   B          (layers, batch, seqlen, ngroups, dstate)   io (forward direction)
 *   init_state (layers, batch, nheads, headdim, dstate)   fp32, nullable
 *   state_out  (layers, batch, nheads, headdim, dstate)   fp32, may alias init_state
 * With bf16 I/O and at least 64 (layer, batch, head) units this is one
 * launch of the fused kernel's forward-state mode over all layers (each unit
 * reads its own layer's A); otherwise one ssd_prefix_state per layer. The
 * workspace is ssd_workspace_bytes(SSD_OP_PREFIX_STATE, layers * batch, ...).
 * Returns as ssd_prefix_state. */
int ssd_prefix_state_layers(const void *x, const void *dt, const float *A, const void *B,
                            const float *init_state, float *state_out, int layers, int batch,
                            int seqlen, int nheads, int headdim, int dstate, int ngroups, int chunk,
                            int dtype, void *workspace, size_t ws_bytes, void *stream);

/* Backward pass of ssd_bidir_fwd: the gradients of the scalar sum(dy * out)
 * with respect to every input, for training through the mixer.
 *   dy   (batch, seqlen, nheads, headdim)           io, the gradient of out
 *   dx   (batch, seqlen, nheads, headdim)           fp32
 *   ddt  (2, batch, seqlen, nheads)                 fp32
 *   dA, dD (2, nheads)                              fp32
 *   dB, dC (2, batch, seqlen, ngroups, dstate)      fp32
 * Other arguments as for ssd_bidir_fwd (either I/O dtype). Every output is
 * overwritten. Each (batch, head, direction) runs its scan on CUDA cores in
 * fp32, keeping every 8th state in the workspace, then the adjoint scan in the
 * opposite order, recomputing each run of 8 states from its checkpoint; the
 * workspace (ssd_workspace_bytes with SSD_OP_BIDIR_BWD) holds
 * ceil(seqlen / 8) + 8 states of dstate x headdim fp32 per CTA of a
 * persistent grid (about 1.3 GB at batch 32, seqlen 1024, 24 heads, dstate
 * 128). dx gets
 * exactly two additions per element and is deterministic; with ngroups <
 * nheads the heads of a group add into dB and dC atomically, in no fixed
 * order. Source: "Training Hybrid Block Diffusion Language Models with
 * Partial Bidirectionality", Key Results and Technical Contribution (the
 * models are trained through the mixer with a full-block objective). */
int ssd_bidir_bwd(const void *x, const void *dt, const float *A, const void *B, const void *C,
                  const float *D, const void *dy, float *dx, float *ddt, float *dA, float *dB,
                  float *dC, float *dD, int batch, int seqlen, int nheads, int headdim, int dstate,
                  int ngroups, int dtype, void *workspace, size_t ws_bytes, void *stream);

/* Backward pass of ssd_bidir_fwd_seeded (and so of ssd_block_step: a forward
 * start state and no reverse one): ssd_bidir_bwd's gradients with each
 * direction's scan starting from its given state, plus the gradients of the
 * start states.
 *   fwd_init, rev_init     (batch, nheads, headdim, dstate)   fp32, read; NULL = zero
 *   d_fwd_init, d_rev_init (batch, nheads, headdim, dstate)   fp32, overwritten; NULL = not wanted
 * The start state's gradient is the adjoint of the state before the
 * direction's first token. Other arguments, workspace and determinism as for
 * ssd_bidir_bwd. Source: "Training Hybrid Block Diffusion Language Models
 * with Partial Bidirectionality", Methodology and Technical Contribution
 * (training through the block-confined scans with the prefix state). */
int ssd_bidir_bwd_seeded(const void *x, const void *dt, const float *A, const void *B,
                         const void *C, const float *D, const float *fwd_init,
                         const float *rev_init, const void *dy, float *dx, float *ddt, float *dA,
                         float *dB, float *dC, float *dD, float *d_fwd_init, float *d_rev_init,
                         int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                         int dtype, void *workspace, size_t ws_bytes, void *stream);

/* ssd_bidir_fwd for callers that cannot allocate device memory when they
 * call the mixer: code running under CUDA graph capture in the global mode,
 * where cudaMalloc is not allowed; plug-ins inside a runtime that has already
 * reserved the GPU's memory for its own pool; loops where an allocation would
 * synchronise the device. (The pages describe no such interface; it has no
 * counterpart there.) Arguments as for ssd_bidir_fwd, without the workspace.
 *  - bf16 I/O only (the fused tensor-core kernel); fp32 returns
 *    SSD_ERR_UNSUPPORTED.
 *  - Scratch is a fixed 32 MiB array (plus a 256-byte status header) inside
 *    the library. Under CUDA's default lazy module loading it is reserved on
 *    a device by the first call on that device, which may therefore allocate
 *    and synchronise (with CUDA_MODULE_LOADING=EAGER: when the context is
 *    created); it stays reserved until the process exits. Make the first call
 *    on each device before any stream capture. Problems needing more, i.e.
 *    batch * nheads * ceil(seqlen / 128) * dstate * 128 bytes > 32 MiB,
 *    return SSD_ERR_WORKSPACE and launch nothing.
 *  - Allocates nothing after that first call: no cudaMalloc, no cudaFree, no
 *    allocating library call. Every call looks the array's device address up
 *    with the calling device current (a cheap host-side query).
 *  - Every call shares the one array: calls that overlap on the GPU (other
 *    streams, other host threads) race and give wrong results. Each call
 *    clears the status header and overwrites the state area before reading it.
 *  - Device-side wait timeouts are recorded in the array's header and are not
 *    reported by this entry point: ssd_noalloc_get_status reads them, before
 *    the next call clears the header. */
int ssd_bidir_fwd_noalloc(const void *x, const void *dt, const float *A, const void *B,
                          const void *C, const float *D, void *out,
                          int batch, int seqlen, int nheads, int headdim, int dstate,
                          int ngroups, int chunk, int dtype, void *stream);

/* ssd_get_device_status for ssd_bidir_fwd_noalloc: synchronise `stream`, read
 * and clear the status header of the no-allocation entry point's own array
 * (on the current device). Returns as ssd_get_device_status; allocates
 * nothing. */
int ssd_noalloc_get_status(void *stream);

/* Synchronise `stream`, read and clear the workspace's status header.
 * Returns SSD_OK, SSD_ERR_TIMEOUT (a bounded device wait expired in a call
 * since the last check) or SSD_ERR_CUDA (the stream reported an error). */
int ssd_get_device_status(const void *workspace, void *stream);

/* Self-test of the bounded device waits: launches one CTA that waits on an
 * mbarrier nothing arrives on, for at most limit_us microseconds (1 ..
 * 2,000,000). The wait gives up, the kernel records SSD_ERR_TIMEOUT in the
 * workspace's status header and exits; nothing faults and the context stays
 * usable. Read the result with ssd_get_device_status. */
int ssd_selftest_wait_timeout(void *workspace, size_t ws_bytes, int limit_us, void *stream);

/* Static description of a status code. */
const char *ssd_error_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_BIDIR_H */
