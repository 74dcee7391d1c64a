// ssd_bidir_fwd_noalloc: the bidirectional mixer for callers that cannot hand
// the library a workspace.
//
// Some callers cannot allocate device memory at the point where they call the
// mixer: code that runs while a CUDA graph is being captured in the global
// capture mode (cudaMalloc is illegal there), plug-ins living inside a
// serving runtime that has already reserved the GPU's memory for its own pool
// and hands out no allocator, and latency-critical loops where a cudaMalloc or
// cudaFree would synchronise the device. This entry point needs nothing from
// them but the inputs and the output: its scratch is a fixed array in the
// library's own device memory.
//
// When that array is reserved: under CUDA's default lazy module loading, the
// module holding it is loaded onto a device by the first call on that device
// (its cudaGetSymbolAddress), so the 32 MiB are reserved then and that first
// call may allocate and synchronise; with CUDA_MODULE_LOADING=EAGER they are
// reserved when the context is created. Either way they stay reserved until
// the process exits. Make the first call on each device before any stream
// capture begins.
//
// It runs the same fused tensor-core kernel as ssd_bidir_fwd (bf16 I/O), with
// that array as the kernel's workspace: a 256-byte status header, then the
// reverse scan's per-tile states (batch * nheads * ceil(seqlen/128) * dstate
// * 64 bf16 values), which is what limits the problem size.
#include "ssd_bidir.h"
#include "ssd_kernels.h"

namespace {

// Largest scratch the entry point accepts (after the status header).
constexpr size_t kNoAllocScratchMax = 32ull << 20;  // 32 MiB
constexpr size_t kNoAllocBytes = ssd::kStatusBytes + kNoAllocScratchMax;

// The scratch itself. Every GPU that loads the library holds it until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch on the current device. In host code the
// symbol is only a host-side stand-in, so the address is looked up on every
// call, with the calling device (and its context) current: a cached address
// could outlive a cudaDeviceReset or belong to another context of the same
// device. Once the module is loaded the lookup is a cheap host-side query.
int scratch_address(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
    *out = p;
    return SSD_OK;
}

}  // namespace

extern "C" int ssd_bidir_fwd_noalloc(const void *x, const void *dt, const float *A, const void *B,
                                     const void *C, const float *D, void *out, int batch, int seqlen,
                                     int nheads, int headdim, int dstate, int ngroups, int chunk,
                                     int dtype, void *stream) {
    const int sel = ssd_select_path(batch, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype);
    if (sel < 0) return sel;
    if (dtype != SSD_BF16) return SSD_ERR_UNSUPPORTED;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (ssd::tc_fused_scratch_bytes(batch, seqlen, nheads, dstate) > kNoAllocScratchMax)
        return SSD_ERR_WORKSPACE;
    if (!x || !dt || !A || !B || !C || !D || !out) return SSD_ERR_INVALID_ARG;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dt) |
                           reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(C) |
                           reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis || (reinterpret_cast<uintptr_t>(A) & 3u) || (reinterpret_cast<uintptr_t>(D) & 3u))
        return SSD_ERR_INVALID_ARG;

    void *scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != SSD_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents: the status header must
    // start clear; the state area is fully written before it is read.
    if (cudaMemsetAsync(scratch, 0, ssd::kStatusBytes, s) != cudaSuccess) return SSD_ERR_CUDA;

    ssd::TcArgs t{};
    t.x = x; t.dt = dt; t.A = A; t.B = B; t.C = C; t.D = D; t.out = out;
    t.workspace = scratch;
    t.ws_bytes = kNoAllocBytes;
    t.batch = batch; t.L = seqlen; t.H = nheads; t.G = ngroups; t.N = dstate; t.ndir = 2;
    cudaError_t e = ssd::launch_tc_fused(t, s);
    if (e == cudaSuccess) return SSD_OK;
    return e == cudaErrorNotSupported ? SSD_ERR_UNSUPPORTED : SSD_ERR_CUDA;
}

// The status of the calls made through ssd_bidir_fwd_noalloc: the array's own
// 256-byte header, read and cleared as ssd_get_device_status does for a
// workspace (it synchronises the stream; nothing is allocated).
extern "C" int ssd_noalloc_get_status(void *stream) {
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != SSD_OK) return rc;
    return ssd_get_device_status(scratch, stream);
}
