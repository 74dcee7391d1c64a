// C ABI of the bidirectional SSD mixer: argument checks, workspace sizing and
// dispatch to the kernels. Declarations and documentation: include/ssd_bidir.h.
#include <stdint.h>
#include <string.h>

#include "ssd_bidir.h"
#include "ssd_kernels.h"

using ssd::SimtArgs;
using ssd::TcArgs;

namespace {

constexpr int kHeaddim = 64;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Shape checks shared by every entry point. Returns SSD_OK or an error code.
int check_shape(int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                int chunk, int dtype, bool check_chunk) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
        return SSD_ERR_INVALID_ARG;
    if (nheads % ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (headdim != kHeaddim) return SSD_ERR_UNSUPPORTED;
    if (dstate != 64 && dstate != 128) return SSD_ERR_UNSUPPORTED;
    if (check_chunk && chunk != 64 && chunk != 128 && chunk != 256) return SSD_ERR_UNSUPPORTED;
    // Index arithmetic uses 64-bit offsets, but token counts stay in int.
    if ((long long)batch * seqlen > (1ll << 31) - 1) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

int to_status(cudaError_t e) {
    if (e == cudaSuccess) return SSD_OK;
    if (e == cudaErrorNotSupported) return SSD_ERR_UNSUPPORTED;
    return SSD_ERR_CUDA;
}

size_t simt_scratch(int op, int batch, int seqlen, int nheads) {
    if (op == SSD_OP_PREFIX_STATE) return 0;
    // one fp32 output buffer per scan direction
    return 2 * sizeof(float) * (size_t)batch * seqlen * nheads * kHeaddim;
}

size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

float *scratch_ptr(void *ws) { return reinterpret_cast<float *>(static_cast<char *>(ws) + ssd::kStatusBytes); }

// Prefix states and block steps take the fused kernel (one (batch, head) per
// SM at a time, all tiles in one launch) from this many units, else the
// tile-parallel chunked kernels.
constexpr long long kFusedMinUnits = 64;

// Longest sequence, in 128-token tiles, that SSD_PATH_AUTO gives the two-CTA
// kernel: each cluster keeps up to half a sequence of 32 KB partial tiles live.
constexpr long long kPairMaxTiles = 16;

// Kernel choice of SSD_PATH_AUTO: bf16 runs on the tensor cores: the one-tile
// kernel for sequences of at most one 128-token tile; two CTAs per (batch,
// head), one per direction, for sequences of 2..16 tiles with a unit for
// every two SMs; one CTA per (batch, head) when there are enough of those to
// fill the GPU; else the segmented or tile-parallel chunked kernels; fp32
// runs the sequential scan.
int auto_path(int batch, int seqlen, int nheads, int ngroups, int dstate, int dtype) {
    if (dtype != SSD_BF16) return SSD_PATH_SIMT;
    if (ssd::tc_onetile_supported(batch, seqlen, nheads, ngroups, dstate)) return SSD_PATH_ONETILE;
    // two to 16 tiles and a (batch, head) unit for every two SMs: one cluster of
    // two CTAs per unit, each running one scan direction (the partial tiles the
    // directions exchange stay in L2 up to this length)
    {
        const long long units = (long long)batch * nheads, nt = (seqlen + 127) / 128;
        const int sms = ssd::device_sms();
        if (nt >= 2 && nt <= kPairMaxTiles && sms > 0 && units >= sms / 2 &&
            ssd::tc_pair_supported(batch, seqlen, nheads, ngroups, dstate))
            return SSD_PATH_PAIR;
    }
    if (ssd::tc_fused_supported(batch, seqlen, nheads, ngroups, dstate)) return SSD_PATH_FUSED;
    // a few long sequences: split them into segments when that leaves at
    // least 4 tiles per SM to work on
    const long long units = (long long)batch * nheads, nt = (seqlen + 127) / 128;
    const int sms = ssd::device_sms();
    if (units * nt >= 4LL * sms && ssd::seg_count(units, seqlen, sms) > 1) return SSD_PATH_SEGMENTED;
    return SSD_PATH_CHUNKED;
}

int bidir_impl(const void *x, const void *dt, const float *A, const void *B, const void *C,
               const float *D, void *out, int batch, int seqlen, int nheads, int headdim,
               int dstate, int ngroups, int chunk, int dtype, int path, void *workspace,
               size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype, true);
    if (rc != SSD_OK) return rc;
    if ((path < SSD_PATH_AUTO || path > SSD_PATH_PAIR) && path != SSD_PATH_ONETILE) return SSD_ERR_INVALID_ARG;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, seqlen, nheads, headdim, dstate,
                                       ngroups, chunk, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!x || !dt || !A || !B || !C || !D || !out) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(out) ||
        !aligned4(A) || !aligned4(D))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (path == SSD_PATH_AUTO) path = auto_path(batch, seqlen, nheads, ngroups, dstate, dtype);

    if (path == SSD_PATH_SIMT) {
        SimtArgs a{};
        a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D;
        a.out = out; a.yacc = scratch_ptr(workspace);
        a.dt_dir_stride = (long long)batch * seqlen * nheads;
        a.bc_dir_stride = (long long)batch * seqlen * ngroups * dstate;
        a.A_dir_stride = nheads;
        a.batch = batch; a.L = seqlen; a.H = nheads; a.G = ngroups;
        a.ndir = 2; a.has_output = 1;
        return to_status(ssd::launch_scan_simt(a, dtype == SSD_BF16, dstate, s));
    }
    if (dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    TcArgs t{};
    t.x = x; t.dt = dt; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
    t.workspace = workspace; t.ws_bytes = ws_bytes;
    t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
    if (path == SSD_PATH_FUSED) return to_status(ssd::launch_tc_fused(t, s));
    if (path == SSD_PATH_PAIR) return to_status(ssd::launch_tc_pair(t, s));
    if (path == SSD_PATH_ONETILE) return to_status(ssd::launch_tc_onetile(t, s));
    if (path == SSD_PATH_SEGMENTED) {
        // at least two segments, even where one would be chosen
        const int sms = ssd::device_sms();
        int S = ssd::seg_count((long long)batch * nheads, seqlen, sms > 0 ? sms : 1);
        for (int k = 2; S < 2 && k <= 64 && seqlen / k >= 128; ++k)
            if (seqlen % k == 0) S = k;
        if (S < 2) return SSD_ERR_UNSUPPORTED;
        return to_status(ssd::launch_tc_segmented(t, S, s));
    }
    return to_status(ssd::launch_tc_chunked(t, s));
}

// Scratch of ssd_bidir_fwd_x2: the two-CTA kernel's partial tiles (bf16,
// more than one tile) or the sequential scan's fp32 forward partial.
size_t x2_scratch(int batch, int seqlen, int nheads, int dstate, int dtype) {
    size_t s = simt_scratch(SSD_OP_BIDIR_FWD, batch, seqlen, nheads);
    if (dtype == SSD_BF16 && ssd::tc_pair_supported(batch, seqlen, nheads, 1, dstate)) {
        const size_t q = ssd::tc_pair_scratch_bytes(batch, seqlen, nheads, dstate);
        s = s > q ? s : q;
    }
    return s;
}

// Workspace of ssd_mixer_block_fwd after the status header: the mixer's own
// scratch first (it is passed the workspace as its own), then the
// intermediates, each 256-byte aligned.
struct BlockWs {
    size_t mixer, x2, b2, c2, dt, y, total;
};
BlockWs block_ws(int batch, int seqlen, int nheads, int dstate, int ngroups, int dtype) {
    BlockWs w{};
    const size_t io = dtype == SSD_BF16 ? 2 : 4;
    const size_t tok = (size_t)batch * seqlen;
    w.mixer = round256(x2_scratch(batch, seqlen, nheads, dstate, dtype));
    size_t o = 0;
    w.x2 = o; o += round256(2 * tok * nheads * kHeaddim * io);
    w.b2 = o; o += round256(2 * tok * ngroups * dstate * io);
    w.c2 = o; o += round256(2 * tok * ngroups * dstate * io);
    w.dt = o; o += round256(2 * tok * nheads * io);
    w.y = o; o += round256(tok * nheads * kHeaddim * io);
    w.total = o;
    return w;
}

}  // namespace

extern "C" {

size_t ssd_workspace_bytes(int op, int batch, int seqlen, int nheads, int headdim, int dstate,
                           int ngroups, int chunk, int dtype) {
    const bool use_chunk = op != SSD_OP_BLOCK_STEP;
    if (check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype, use_chunk) != SSD_OK)
        return 0;
    size_t scratch = simt_scratch(op, batch, seqlen, nheads);
    if (dtype == SSD_BF16) {
        if (op == SSD_OP_BIDIR_FWD) {
            size_t c = ssd::tc_chunked_scratch_bytes(batch, seqlen, nheads, dstate, 2);
            size_t f = ssd::tc_fused_scratch_bytes(batch, seqlen, nheads, dstate);
            size_t g = ssd::tc_segmented_scratch_bytes(batch, seqlen, nheads, dstate);
            size_t q = ssd::tc_pair_scratch_bytes(batch, seqlen, nheads, dstate);
            scratch = scratch > c ? scratch : c;
            scratch = scratch > f ? scratch : f;
            scratch = scratch > g ? scratch : g;
            scratch = scratch > q ? scratch : q;
        } else if (op == SSD_OP_PREFIX_STATE) {
            size_t c = ssd::tc_chunked_scratch_bytes(batch, seqlen, nheads, dstate, 1);
            scratch = scratch > c ? scratch : c;
        } else if (op == SSD_OP_BIDIR_BWD) {
            scratch = 0;
        } else if (op == SSD_OP_BLOCK_STEP) {
            size_t c = ssd::tc_chunked_scratch_bytes(batch, seqlen, nheads, dstate, 2);
            size_t f = ssd::tc_fused_scratch_bytes(batch, seqlen, nheads, dstate);
            scratch = scratch > c ? scratch : c;
            scratch = scratch > f ? scratch : f;
        }
    }
    if (op == SSD_OP_BIDIR_BWD) scratch = ssd::bwd_scratch_bytes(batch, seqlen, nheads, dstate);
    if (op == SSD_OP_BIDIR_FWD_X2) scratch = x2_scratch(batch, seqlen, nheads, dstate, dtype);
    if (op == SSD_OP_MIXER_BLOCK) {
        const BlockWs w = block_ws(batch, seqlen, nheads, dstate, ngroups, dtype);
        scratch = w.mixer + w.total;
    }
    return ssd::kStatusBytes + round256(scratch);
}

int ssd_select_path(int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                    int chunk, int dtype) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype, true);
    if (rc != SSD_OK) return rc;
    return auto_path(batch, seqlen, nheads, ngroups, dstate, dtype);
}

int ssd_workspace_init(void *workspace, size_t ws_bytes, void *stream) {
    if (!workspace || ws_bytes < ssd::kStatusBytes) return SSD_ERR_WORKSPACE;
    cudaError_t e = cudaMemsetAsync(workspace, 0, ssd::kStatusBytes, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

int ssd_bidir_fwd(const void *x, const void *dt, const float *A, const void *B, const void *C,
                  const float *D, void *out, int batch, int seqlen, int nheads, int headdim,
                  int dstate, int ngroups, int chunk, int dtype, void *workspace, size_t ws_bytes,
                  void *stream) {
    return bidir_impl(x, dt, A, B, C, D, out, batch, seqlen, nheads, headdim, dstate, ngroups,
                      chunk, dtype, SSD_PATH_AUTO, workspace, ws_bytes, stream);
}

int ssd_bidir_fwd_path(const void *x, const void *dt, const float *A, const void *B, const void *C,
                       const float *D, void *out, int batch, int seqlen, int nheads, int headdim,
                       int dstate, int ngroups, int chunk, int dtype, int path, void *workspace,
                       size_t ws_bytes, void *stream) {
    return bidir_impl(x, dt, A, B, C, D, out, batch, seqlen, nheads, headdim, dstate, ngroups,
                      chunk, dtype, path, workspace, ws_bytes, stream);
}

int ssd_prefix_state_path(const void *x, const void *dt, const float *A, const void *B,
                          const float *init_state, float *state_out, int batch, int seqlen, int nheads,
                          int headdim, int dstate, int ngroups, int chunk, int dtype, int path,
                          void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype, true);
    if (rc != SSD_OK) return rc;
    if (path < SSD_PATH_AUTO || path > SSD_PATH_FUSED) return SSD_ERR_INVALID_ARG;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_PREFIX_STATE, batch, seqlen, nheads, headdim, dstate,
                                       ngroups, chunk, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0) return SSD_OK;
    if (!state_out || !aligned16(state_out)) return SSD_ERR_INVALID_ARG;
    if (init_state && !aligned16(init_state)) return SSD_ERR_INVALID_ARG;
    if (seqlen > 0) {
        if (!x || !dt || !A || !B) return SSD_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned4(A)) return SSD_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (path == SSD_PATH_AUTO && dtype == SSD_BF16 && seqlen > 0)
        path = (long long)batch * nheads >= kFusedMinUnits ? SSD_PATH_FUSED : SSD_PATH_CHUNKED;
    if ((path == SSD_PATH_CHUNKED || path == SSD_PATH_FUSED) && dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    // an empty sequence (the state is the initial one) goes to the scan kernel below
    if ((path == SSD_PATH_CHUNKED || path == SSD_PATH_FUSED) && seqlen > 0) {
        TcArgs t{};
        t.x = x; t.dt = dt; t.A = A; t.B = B; t.init = init_state; t.state_out = state_out;
        t.workspace = workspace; t.ws_bytes = ws_bytes;
        t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 1;
        return to_status(path == SSD_PATH_FUSED ? ssd::launch_tc_fused_state(t, s) : ssd::launch_tc_chunked(t, s));
    }
    SimtArgs a{};
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = nullptr; a.D = nullptr;
    a.init = init_state; a.state_out = state_out;
    a.dt_dir_stride = 0; a.bc_dir_stride = 0; a.A_dir_stride = 0;
    a.batch = batch; a.L = seqlen; a.H = nheads; a.G = ngroups;
    a.ndir = 1; a.has_output = 0;
    return to_status(ssd::launch_scan_simt(a, dtype == SSD_BF16, dstate, s));
}

int ssd_prefix_state(const void *x, const void *dt, const float *A, const void *B,
                     const float *init_state, float *state_out, int batch, int seqlen, int nheads,
                     int headdim, int dstate, int ngroups, int chunk, int dtype, void *workspace,
                     size_t ws_bytes, void *stream) {
    return ssd_prefix_state_path(x, dt, A, B, init_state, state_out, batch, seqlen, nheads, headdim,
                                 dstate, ngroups, chunk, dtype, SSD_PATH_AUTO, workspace, ws_bytes, stream);
}

int ssd_prefix_state_layers(const void *x, const void *dt, const float *A, const void *B, const float *init_state,
                            float *state_out, int layers, int batch, int seqlen, int nheads, int headdim, int dstate,
                            int ngroups, int chunk, int dtype, void *workspace, size_t ws_bytes, void *stream) {
    if (layers <= 0) return SSD_ERR_INVALID_ARG;
    if ((long long)layers * batch > (1ll << 31) - 1) return SSD_ERR_UNSUPPORTED;
    const int lb = layers * batch;
    int rc = check_shape(lb, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype, true);
    if (rc != SSD_OK) return rc;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_PREFIX_STATE, lb, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype))
        return SSD_ERR_WORKSPACE;
    if (lb == 0) return SSD_OK;
    if (!state_out || !aligned16(state_out) || (init_state && !aligned16(init_state))) return SSD_ERR_INVALID_ARG;
    if (seqlen > 0 && (!x || !dt || !A || !B || !aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned4(A)))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SSD_BF16 && seqlen > 0 && (long long)lb * nheads >= kFusedMinUnits) {
        // one launch: the layers are batch elements that read their own layer's A
        TcArgs t{};
        t.x = x; t.dt = dt; t.A = A; t.B = B; t.init = init_state; t.state_out = state_out;
        t.workspace = workspace; t.ws_bytes = ws_bytes;
        t.batch = lb; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 1;
        t.layer_units = batch * nheads;
        t.A_layer = nheads;
        return to_status(ssd::launch_tc_fused_state(t, s));
    }
    // otherwise one call per layer on that layer's slices
    const size_t io = dtype == SSD_BF16 ? 2 : 4;
    const size_t xl = (size_t)batch * seqlen * nheads * headdim, dtl = (size_t)batch * seqlen * nheads;
    const size_t bl = (size_t)batch * seqlen * ngroups * dstate, sl = (size_t)batch * nheads * headdim * dstate;
    for (int l = 0; l < layers; ++l) {
        rc = ssd_prefix_state_path(x ? static_cast<const char *>(x) + l * xl * io : nullptr,
                                   dt ? static_cast<const char *>(dt) + l * dtl * io : nullptr, A ? A + (size_t)l * nheads : nullptr,
                                   B ? static_cast<const char *>(B) + l * bl * io : nullptr,
                                   init_state ? init_state + l * sl : nullptr, state_out + l * sl, batch, seqlen, nheads,
                                   headdim, dstate, ngroups, chunk, dtype, SSD_PATH_AUTO, workspace, ws_bytes, stream);
        if (rc != SSD_OK) return rc;
    }
    return SSD_OK;
}

int ssd_block_step_path(const void *x, const void *dt, const float *A, const void *B, const void *C,
                        const float *D, const float *prefix_state, void *out, int batch, int blk_len,
                        int nheads, int headdim, int dstate, int ngroups, int dtype, int path,
                        void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, blk_len, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if ((path < SSD_PATH_AUTO || path > SSD_PATH_FUSED) && path != SSD_PATH_BLOCK) return SSD_ERR_INVALID_ARG;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BLOCK_STEP, batch, blk_len, nheads, headdim, dstate,
                                       ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0 || blk_len == 0) return SSD_OK;
    if (!x || !dt || !A || !B || !C || !D || !out) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(out) ||
        !aligned4(A) || !aligned4(D))
        return SSD_ERR_INVALID_ARG;
    if (prefix_state && !aligned16(prefix_state)) return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (path == SSD_PATH_AUTO && dtype == SSD_BF16) {
        if (ssd::tc_blockstep_supported(batch, blk_len, nheads, ngroups, dstate))
            path = SSD_PATH_BLOCK;
        else
            path = (long long)batch * nheads >= kFusedMinUnits ? SSD_PATH_FUSED : SSD_PATH_CHUNKED;
    }
    if ((path == SSD_PATH_CHUNKED || path == SSD_PATH_FUSED || path == SSD_PATH_BLOCK) && dtype != SSD_BF16)
        return SSD_ERR_UNSUPPORTED;
    if (path == SSD_PATH_BLOCK) {
        if (!ssd::tc_blockstep_supported(batch, blk_len, nheads, ngroups, dstate)) return SSD_ERR_UNSUPPORTED;
        // the two directions stacked as one tile's rows, forward from the cached state
        TcArgs t{};
        t.x = x; t.dt = dt; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
        t.init = prefix_state;
        t.workspace = workspace; t.ws_bytes = ws_bytes;
        t.batch = batch; t.L = blk_len; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
        return to_status(ssd::launch_tc_blockstep(t, s));
    }
    if (path == SSD_PATH_CHUNKED || path == SSD_PATH_FUSED) {
        // both scans over the block, the forward one starting from the cached
        // state (zero if none) and the reverse one from zero
        TcArgs t{};
        t.x = x; t.dt = dt; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
        t.init = prefix_state;
        t.workspace = workspace; t.ws_bytes = ws_bytes;
        t.batch = batch; t.L = blk_len; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
        return to_status(path == SSD_PATH_FUSED ? ssd::launch_tc_fused(t, s) : ssd::launch_tc_chunked(t, s));
    }
    SimtArgs a{};
    a.x = x; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D;
    a.init = prefix_state; a.state_out = nullptr;
    a.out = out; a.yacc = scratch_ptr(workspace);
    a.dt_dir_stride = (long long)batch * blk_len * nheads;
    a.bc_dir_stride = (long long)batch * blk_len * ngroups * dstate;
    a.A_dir_stride = nheads;
    a.batch = batch; a.L = blk_len; a.H = nheads; a.G = ngroups;
    a.ndir = 2; a.has_output = 1;
    return to_status(ssd::launch_scan_simt(a, dtype == SSD_BF16, dstate, s));
}

int ssd_block_step(const void *x, const void *dt, const float *A, const void *B, const void *C,
                   const float *D, const float *prefix_state, void *out, int batch, int blk_len,
                   int nheads, int headdim, int dstate, int ngroups, int dtype, void *workspace,
                   size_t ws_bytes, void *stream) {
    return ssd_block_step_path(x, dt, A, B, C, D, prefix_state, out, batch, blk_len, nheads, headdim,
                               dstate, ngroups, dtype, SSD_PATH_AUTO, workspace, ws_bytes, stream);
}

int ssd_bidir_fwd_dtraw(const void *x, const void *dt_raw, const float *dt_bias, float dt_min, float dt_max,
                        const float *A, const void *B, const void *C, const float *D, void *out, int batch,
                        int seqlen, int nheads, int headdim, int dstate, int ngroups, int dtype, void *workspace,
                        size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if (dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    // NaN bounds fail both comparisons
    if (!(dt_min >= 0.f) || !(dt_max >= dt_min)) return SSD_ERR_INVALID_ARG;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!x || !dt_raw || !dt_bias || !A || !B || !C || !D || !out) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt_raw) || !aligned16(B) || !aligned16(C) || !aligned16(out) ||
        !aligned4(dt_bias) || !aligned4(A) || !aligned4(D))
        return SSD_ERR_INVALID_ARG;
    TcArgs t{};
    t.x = x; t.dt = dt_raw; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
    t.dt_bias = dt_bias; t.dt_lo = dt_min; t.dt_hi = dt_max;
    t.workspace = workspace; t.ws_bytes = ws_bytes;
    t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
    return to_status(ssd::launch_tc_fused_dtraw(t, static_cast<cudaStream_t>(stream)));
}

// Segments to split each sequence into when a call has too few (batch, head)
// units to fill the GPU (as SSD_PATH_AUTO chooses the segmented path); 1 = none.
int few_unit_segments(int batch, int seqlen, int nheads) {
    const long long units = (long long)batch * nheads, nt = (seqlen + 127) / 128;
    const int sms = ssd::device_sms();
    if (sms <= 0 || units >= sms || units * nt < 4LL * sms) return 1;
    return ssd::seg_count(units, seqlen, sms);
}

int ssd_segment_states(const void *x, const void *dt, const float *A, const void *B, float *fwd_state,
                       float *fwd_decay, float *rev_state, float *rev_decay, int batch, int seqlen, int nheads,
                       int headdim, int dstate, int ngroups, int dtype, void *workspace, size_t ws_bytes,
                       void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if (dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0) return SSD_OK;
    if (seqlen == 0) return SSD_ERR_UNSUPPORTED;
    if (!x || !dt || !A || !B || !fwd_state || !fwd_decay || !rev_state || !rev_decay) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned4(A) || !aligned16(fwd_state) ||
        !aligned16(rev_state) || !aligned4(fwd_decay) || !aligned4(rev_decay))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the fused kernel's forward and reverse state modes, from zero
    TcArgs t{};
    t.x = x; t.dt = dt; t.A = A; t.B = B;
    t.workspace = workspace; t.ws_bytes = ws_bytes;
    t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
    // few long sequences: state passes over segments of each, then their totals
    const int S = few_unit_segments(batch, seqlen, nheads);
    if (S > 1) return to_status(ssd::launch_tc_segment_totals(t, S, fwd_state, fwd_decay, rev_state, rev_decay, s));
    TcArgs f = t;
    f.state_out = fwd_state;
    f.decay_out = fwd_decay;
    cudaError_t e = ssd::launch_tc_fused_state(f, s);
    if (e != cudaSuccess) return to_status(e);
    TcArgs r = t;
    r.state_out = rev_state;
    r.decay_out = rev_decay;
    return to_status(ssd::launch_tc_fused_state_rev(r, s));
}

int ssd_segment_carry(const float *fwd_states, const float *fwd_decays, const float *rev_states,
                      const float *rev_decays, int nseg, int seg, float *fwd_in, float *rev_in, int batch,
                      int nheads, int headdim, int dstate, void *stream) {
    if (batch < 0 || nheads <= 0 || nseg <= 0 || seg < 0 || seg >= nseg) return SSD_ERR_INVALID_ARG;
    if (headdim != 64 || (dstate != 64 && dstate != 128)) return SSD_ERR_UNSUPPORTED;
    if ((long long)batch * nheads * nseg >= (1ll << 31)) return SSD_ERR_UNSUPPORTED;
    if (batch == 0) return SSD_OK;
    if (!fwd_states || !fwd_decays || !rev_states || !rev_decays || !fwd_in || !rev_in) return SSD_ERR_INVALID_ARG;
    if (!aligned16(fwd_states) || !aligned16(rev_states) || !aligned16(fwd_in) || !aligned16(rev_in) ||
        !aligned4(fwd_decays) || !aligned4(rev_decays))
        return SSD_ERR_INVALID_ARG;
    return to_status(ssd::launch_seg_carry(fwd_states, fwd_decays, rev_states, rev_decays, fwd_in, rev_in, batch,
                                           nheads, dstate, nseg, seg, static_cast<cudaStream_t>(stream)));
}

int ssd_bidir_fwd_seeded(const void *x, const void *dt, const float *A, const void *B, const void *C,
                         const float *D, const float *fwd_init, const float *rev_init, void *out, int batch,
                         int seqlen, int nheads, int headdim, int dstate, int ngroups, int dtype, void *workspace,
                         size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if (dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!x || !dt || !A || !B || !C || !D || !out) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(out) || !aligned4(A) ||
        !aligned4(D))
        return SSD_ERR_INVALID_ARG;
    if ((fwd_init && !aligned16(fwd_init)) || (rev_init && !aligned16(rev_init))) return SSD_ERR_INVALID_ARG;
    // the fused kernel's seeded mode: forward scan from fwd_init, reverse scan
    // from rev_init at the sequence end (zero where NULL)
    TcArgs t{};
    t.x = x; t.dt = dt; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
    t.init = fwd_init; t.rinit = rev_init;
    t.workspace = workspace; t.ws_bytes = ws_bytes;
    t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
    // few long sequences: the segmented path, its scan starting from the seeds
    const int S = few_unit_segments(batch, seqlen, nheads);
    if (S > 1) return to_status(ssd::launch_tc_segmented(t, S, static_cast<cudaStream_t>(stream)));
    return to_status(ssd::launch_tc_fused(t, static_cast<cudaStream_t>(stream)));
}

int ssd_bidir_bwd_seeded(const void *x, const void *dt, const float *A, const void *B, const void *C,
                         const float *D, const float *fwd_init, const float *rev_init, const void *dy, float *dx,
                         float *ddt, float *dA, float *dB, float *dC, float *dD, float *d_fwd_init,
                         float *d_rev_init, int batch, int seqlen, int nheads, int headdim, int dstate,
                         int ngroups, int dtype, void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BIDIR_BWD, batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (!dA || !dD || !aligned4(dA) || !aligned4(dD)) return SSD_ERR_INVALID_ARG;
    if ((fwd_init && !aligned4(fwd_init)) || (rev_init && !aligned4(rev_init)) ||
        (d_fwd_init && !aligned4(d_fwd_init)) || (d_rev_init && !aligned4(d_rev_init)))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = sizeof(float) * (size_t)batch * nheads * headdim * dstate;
    if (batch == 0 || seqlen == 0) {
        // no tokens: every gradient is zero (dA, dD and the start states' are the only non-empty ones)
        if (cudaMemsetAsync(dA, 0, 2 * sizeof(float) * nheads, s) != cudaSuccess ||
            cudaMemsetAsync(dD, 0, 2 * sizeof(float) * nheads, s) != cudaSuccess ||
            (d_fwd_init && state_bytes && cudaMemsetAsync(d_fwd_init, 0, state_bytes, s) != cudaSuccess) ||
            (d_rev_init && state_bytes && cudaMemsetAsync(d_rev_init, 0, state_bytes, s) != cudaSuccess))
            return SSD_ERR_CUDA;
        return SSD_OK;
    }
    if (!x || !dt || !A || !B || !C || !D || !dy || !dx || !ddt || !dB || !dC) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(dy) || !aligned16(dx) ||
        !aligned16(ddt) || !aligned16(dB) || !aligned16(dC) || !aligned4(A) || !aligned4(D))
        return SSD_ERR_INVALID_ARG;
    ssd::BwdLaunch l{};
    l.x = x; l.dt = dt; l.B = B; l.C = C; l.dy = dy; l.A = A; l.D = D;
    l.dx = dx; l.ddt = ddt; l.dA = dA; l.dB = dB; l.dC = dC; l.dD = dD;
    l.init_f = fwd_init; l.init_b = rev_init; l.dinit_f = d_fwd_init; l.dinit_b = d_rev_init;
    l.scratch = scratch_ptr(workspace);
    l.batch = batch; l.L = seqlen; l.H = nheads; l.G = ngroups; l.N = dstate;
    l.bf16 = dtype == SSD_BF16;
    return to_status(ssd::launch_bwd(l, s));
}

int ssd_bidir_bwd(const void *x, const void *dt, const float *A, const void *B, const void *C, const float *D,
                  const void *dy, float *dx, float *ddt, float *dA, float *dB, float *dC, float *dD, int batch,
                  int seqlen, int nheads, int headdim, int dstate, int ngroups, int dtype, void *workspace,
                  size_t ws_bytes, void *stream) {
    return ssd_bidir_bwd_seeded(x, dt, A, B, C, D, nullptr, nullptr, dy, dx, ddt, dA, dB, dC, dD, nullptr, nullptr,
                                batch, seqlen, nheads, headdim, dstate, ngroups, dtype, workspace, ws_bytes, stream);
}

int ssd_bidir_fwd_x2(const void *x2, const void *dt, const float *A, const void *B, const void *C, const float *D,
                     void *out, int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups, int dtype,
                     void *workspace, size_t ws_bytes, void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_BIDIR_FWD_X2, batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!x2 || !dt || !A || !B || !C || !D || !out) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x2) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(out) || !aligned4(A) ||
        !aligned4(D))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long xdir = (long long)batch * seqlen * nheads * headdim;
    if (dtype == SSD_BF16 && ssd::tc_pair_supported(batch, seqlen, nheads, ngroups, dstate)) {
        TcArgs t{};
        t.x = x2; t.dt = dt; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
        t.workspace = workspace; t.ws_bytes = ws_bytes;
        t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
        t.x_dir_stride = xdir;
        return to_status(ssd::launch_tc_pair(t, s));
    }
    SimtArgs a{};
    a.x = x2; a.dt = dt; a.A = A; a.B = B; a.C = C; a.D = D;
    a.out = out; a.yacc = scratch_ptr(workspace);
    a.dt_dir_stride = (long long)batch * seqlen * nheads;
    a.bc_dir_stride = (long long)batch * seqlen * ngroups * dstate;
    a.A_dir_stride = nheads;
    a.x_dir_stride = xdir;
    a.batch = batch; a.L = seqlen; a.H = nheads; a.G = ngroups;
    a.ndir = 2; a.has_output = 1;
    return to_status(ssd::launch_scan_simt(a, dtype == SSD_BF16, dstate, s));
}

int ssd_mixer_block_fwd(const void *xbc, const void *z, const void *dt_raw, const float *conv_w, const float *conv_b,
                        int conv_k, const float *dt_bias, float dt_min, float dt_max, const float *A, const float *D,
                        const float *norm_w, float norm_eps, void *out, int batch, int seqlen, int nheads,
                        int headdim, int dstate, int ngroups, int dtype, void *workspace, size_t ws_bytes,
                        void *stream) {
    int rc = check_shape(batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype, false);
    if (rc != SSD_OK) return rc;
    if (conv_k < 1 || conv_k > 4) return SSD_ERR_UNSUPPORTED;
    if (!(dt_min >= 0.f) || !(dt_max >= dt_min) || !(norm_eps >= 0.f)) return SSD_ERR_INVALID_ARG;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SSD_ERR_INVALID_ARG;
    if (ws_bytes < ssd_workspace_bytes(SSD_OP_MIXER_BLOCK, batch, seqlen, nheads, headdim, dstate, ngroups, 64, dtype))
        return SSD_ERR_WORKSPACE;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!xbc || !z || !dt_raw || !conv_w || !conv_b || !dt_bias || !A || !D || !norm_w || !out)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(xbc) || !aligned16(z) || !aligned16(dt_raw) || !aligned16(out) || !aligned4(conv_w) ||
        !aligned4(conv_b) || !aligned4(dt_bias) || !aligned4(A) || !aligned4(D) || !aligned4(norm_w))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const BlockWs w = block_ws(batch, seqlen, nheads, dstate, ngroups, dtype);
    char *inter = static_cast<char *>(workspace) + ssd::kStatusBytes + w.mixer;
    ssd::BlockLaunch l{};
    l.xbc = xbc; l.conv_w = conv_w; l.conv_b = conv_b;
    l.x2 = inter + w.x2; l.B2 = inter + w.b2; l.C2 = inter + w.c2;
    l.dt_raw = dt_raw; l.dt_bias = dt_bias; l.dt = inter + w.dt;
    l.y = inter + w.y; l.z = z; l.norm_w = norm_w; l.out = out;
    l.dt_lo = dt_min; l.dt_hi = dt_max; l.eps = norm_eps;
    l.batch = batch; l.L = seqlen; l.H = nheads; l.HP = nheads * headdim; l.GN = ngroups * dstate; l.K = conv_k;
    l.bf16 = dtype == SSD_BF16;
    if ((rc = to_status(ssd::launch_conv_silu(l, s))) != SSD_OK) return rc;
    if ((rc = to_status(ssd::launch_dt_prep(l, s))) != SSD_OK) return rc;
    // the mixer gets the workspace's header and its own scratch
    rc = ssd_bidir_fwd_x2(l.x2, l.dt, A, l.B2, l.C2, D, const_cast<void *>(l.y), batch, seqlen, nheads, headdim,
                          dstate, ngroups, dtype, workspace, ssd::kStatusBytes + w.mixer, stream);
    if (rc != SSD_OK) return rc;
    return to_status(ssd::launch_gated_rmsnorm(l, s));
}

int ssd_get_device_status(const void *workspace, void *stream) {
    if (!workspace) return SSD_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ssd::DeviceStatus st;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSD_ERR_CUDA;
    if (cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    if (st.flags == 0) return SSD_OK;
    if (cudaMemset(const_cast<void *>(workspace), 0, sizeof(st)) != cudaSuccess) return SSD_ERR_CUDA;
    return (st.flags & ssd::kFlagTimeout) ? SSD_ERR_TIMEOUT : SSD_ERR_CUDA;
}

const char *ssd_error_string(int status) {
    switch (status) {
        case SSD_OK: return "ok";
        case SSD_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size, ngroups does not divide nheads)";
        case SSD_ERR_UNSUPPORTED: return "unsupported shape, chunk, dtype or path";
        case SSD_ERR_CUDA: return "CUDA launch or runtime error";
        case SSD_ERR_WORKSPACE: return "workspace missing or too small";
        case SSD_ERR_TIMEOUT: return "a bounded device-side wait expired";
        default: return "unknown status";
    }
}

int ssd_version(void) { return 100; }

}  // extern "C"
