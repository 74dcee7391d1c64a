"""ssd_bidir_fwd_noalloc: the entry point for callers that cannot allocate device
memory (graph capture in global mode, runtimes that own all of the GPU's
memory, loops where an allocation would synchronise the device). It takes no
workspace; its scratch is a fixed array inside the library.

Checked through the C ABI, on several calls in a row (the array keeps the
previous call's contents, so a later call must not see them):
  - against the fp64 oracle, element by element on sampled (batch, head)
    units, at the bf16 parity bar of every other GPU test;
  - against ssd_bidir_fwd forced onto the same fused kernel with a workspace
    of its own: same kernel, same inputs, so the outputs must be bit-identical;
  - its status header, read through ssd_noalloc_get_status after each call.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import ssd_inputs as si
from paritylib import check, oracle_units, sample_units
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu

NAMES = ("x", "dt", "A", "B", "C", "D")


def _lib():
    import bidirectional_mamba_ssd_b200 as ssd
    lib = ssd.lib
    lib.ssd_bidir_fwd_noalloc.restype = ctypes.c_int
    lib.ssd_bidir_fwd_noalloc.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    return ssd, lib


def _noalloc(lib, inp, out, chunk, stream):
    batch, L, H, P = inp["x"].shape
    G, N = inp["B"].shape[-2:]
    ptrs = [ctypes.c_void_p(inp[n].data_ptr()) for n in NAMES] + [ctypes.c_void_p(out.data_ptr())]
    return lib.ssd_bidir_fwd_noalloc(*ptrs, batch, L, H, P, N, G, chunk, 1, ctypes.c_void_p(stream))


# (batch, L, H, N, G, chunk): ragged tails, G < H, d_state 64 and 128, and a
# shape with more (batch, head) units than SMs; the first comes back last
SHAPES = [(2, 384, 8, 128, 8, 256), (3, 200, 6, 64, 2, 64), (8, 300, 24, 128, 24, 128),
          (2, 384, 8, 128, 8, 256)]


def test_noalloc_matches_oracle_and_fused_path_on_calls_in_a_row():
    ssd, lib = _lib()
    stream = torch.cuda.current_stream().cuda_stream
    for k, (batch, L, H, N, G, chunk) in enumerate(SHAPES):
        inp = si.bidir_inputs(batch, L, H, 64, N, G, "bf16", seed=40 + k, device="cuda")
        out = torch.full_like(inp["x"], float("nan"))
        assert _noalloc(lib, inp, out, chunk, stream) == 0
        ref = ssd.ssd_bidir_fwd(*(inp[n] for n in NAMES), chunk=chunk, path=ssd.SSD_PATH_FUSED)
        torch.cuda.synchronize()
        y = to_f64(out)
        assert np.isfinite(y).all(), f"call {k}: non-finite output"
        # the same kernel on the same inputs: bit-identical
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {k}: differs from the fused path"
        units = sample_units(batch, H, 6, seed=k)
        exp = oracle_units(inp, units)
        for (b, h), o in exp.items():
            check(y[b, :, h], o, torch.bfloat16, f"call {k} unit ({b},{h})")
        # the call's own status header: no bounded wait expired
        assert lib.ssd_noalloc_get_status(ctypes.c_void_p(stream)) == 0, f"call {k}: status"


def test_noalloc_rejects_oversized_problem():
    ssd, lib = _lib()
    fake = [ctypes.c_void_p(1 << 20)] * 7
    # 32 x 24 heads x 8 tiles x 128 states x 64 x 2 bytes = 100 MB of states > 32 MiB
    rc = lib.ssd_bidir_fwd_noalloc(*fake, 32, 1024, 24, 64, 128, 24, 256, 1, None)
    assert rc == ssd.SSD_ERR_WORKSPACE
