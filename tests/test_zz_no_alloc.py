"""ssd_bidir_fwd_noalloc: the entry point for callers that cannot allocate device
memory (graph capture in global mode, runtimes that own all of the GPU's
memory, loops where an allocation would synchronise the device). It takes no
workspace; its scratch is a fixed array inside the library.

Checked through the C ABI against ssd_bidir_fwd on two calls in a row (the
array keeps the previous call's contents, so the second call must not see
them). This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import ssd_inputs as si
from paritylib import TOL_BF16, half_ulp_bf16, rms
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

NAMES = ("x", "dt", "A", "B", "C", "D")


def _noalloc(lib, inp, out, chunk, stream):
    batch, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[-2:]
    ptrs = [ctypes.c_void_p(inp[n].data_ptr()) for n in NAMES] + [ctypes.c_void_p(out.data_ptr())]
    return lib.ssd_bidir_fwd_noalloc(*ptrs, batch, L, H, P, N, G, chunk, 1, ctypes.c_void_p(stream))


def test_noalloc_matches_bidir_fwd_on_two_calls():
    import bidirectional_mamba_ssd_b200 as ssd
    lib = ssd.lib
    lib.ssd_bidir_fwd_noalloc.restype = ctypes.c_int
    lib.ssd_bidir_fwd_noalloc.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    stream = torch.cuda.current_stream().cuda_stream
    shapes = [(2, 384, 8, 128, 8, 256), (3, 200, 6, 64, 2, 64)]
    for k, (batch, L, H, N, G, chunk) in enumerate(shapes):
        inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=40 + k, device="cuda")
        ref = ssd.ssd_bidir_fwd(*(inp[n] for n in NAMES), chunk=chunk)
        out = torch.full_like(inp["x"], float("nan"))
        assert _noalloc(lib, inp, out, chunk, stream) == 0
        torch.cuda.synchronize()
        y, o = to_f64(out), to_f64(ref)
        # both results are bf16-rounded: allow each its half ulp, then the bf16 bar
        d = np.abs(y - o) - 2 * half_ulp_bf16(np.maximum(np.abs(y), np.abs(o)))
        assert np.isfinite(y).all()
        assert np.max(d) <= TOL_BF16 * rms(o), f"call {k}: {np.max(d) / rms(o):.3e}"


def test_noalloc_rejects_oversized_problem():
    import bidirectional_mamba_ssd_b200 as ssd
    lib = ssd.lib
    lib.ssd_bidir_fwd_noalloc.restype = ctypes.c_int
    lib.ssd_bidir_fwd_noalloc.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    fake = [ctypes.c_void_p(1 << 20)] * 7
    # 32 x 24 heads x 8 tiles x 128 states x 64 x 2 bytes = 100 MB of states > 32 MiB
    rc = lib.ssd_bidir_fwd_noalloc(*fake, 32, 1024, 24, 64, 128, 24, 256, 1, None)
    assert rc == ssd.SSD_ERR_WORKSPACE
