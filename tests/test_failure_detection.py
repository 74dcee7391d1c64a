"""Failure detection without a GPU fault: a device-side wait that nobody
satisfies runs out of its time bound, the kernel records a timeout in the
workspace header and exits; the host reads SSD_ERR_TIMEOUT and the context
keeps working. Nothing here faults, traps or hangs."""
import ctypes

import pytest
import torch

import ssd_inputs as si
from paritylib import check
from ssd_inputs import to_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import bidirectional_mamba_ssd_b200 as ssd
    import oracle
    ws = ssd.Workspace()
    buf = ws.get(1 << 12)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert ssd.lib.ssd_selftest_wait_timeout(ctypes.c_void_p(buf.data_ptr()), buf.numel(), 20000, stream) == 0
    assert ws.status() == ssd.SSD_ERR_TIMEOUT
    assert ws.status() == ssd.SSD_OK            # read-and-clear
    # the context is still usable: a normal call succeeds and is correct
    inp = si.bidir_inputs(1, 256, 4, 64, 128, 4, "bf16", seed=3, device="cuda")
    y = ssd.ssd_bidir_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], workspace=ws)
    torch.cuda.synchronize()
    assert ws.status() == ssd.SSD_OK
    o = oracle.bidir(*(to_f64(inp[k]) for k in ("x", "dt", "A", "B", "C", "D")))
    check(to_f64(y), o, torch.bfloat16, "after timeout")


def test_selftest_rejects_bad_limits():
    import bidirectional_mamba_ssd_b200 as ssd
    fake = ctypes.c_void_p(1 << 20)
    assert ssd.lib.ssd_selftest_wait_timeout(fake, 4096, 0, None) == ssd.SSD_ERR_INVALID_ARG
    assert ssd.lib.ssd_selftest_wait_timeout(None, 4096, 100, None) == ssd.SSD_ERR_WORKSPACE
