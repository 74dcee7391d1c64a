"""Host-only checks of the C ABI: the library loads, exports every function
include/ssd_bidir.h declares, sizes workspaces, and rejects bad arguments
before launching anything (so these calls never reach the GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd_bidir.h")


@pytest.fixture(scope="module")
def lib():
    from bidirectional_mamba_ssd_b200 import build as b
    b.build()
    from bidirectional_mamba_ssd_b200 import _lib
    return _lib.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(ssd_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["ssd_bidir_fwd", "ssd_prefix_state", "ssd_block_step", "ssd_workspace_bytes",
              "ssd_get_device_status", "ssd_error_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from bidirectional_mamba_ssd_b200 import _lib
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_no_torch_in_the_abi():
    src = open(HEADER).read()
    assert "torch" not in src.lower().replace("torch (", "")
    assert "at::" not in src and "c10" not in src


def test_version_and_errors(lib):
    assert lib.ssd_version() >= 100
    for code in [0, -1, -2, -3, -4, -5]:
        assert lib.ssd_error_string(code)
    assert b"unknown" in lib.ssd_error_string(42)


def ws_bytes(lib, op=0, batch=2, L=256, H=4, P=64, N=128, G=4, chunk=128, dtype=1):
    return lib.ssd_workspace_bytes(op, batch, L, H, P, N, G, chunk, dtype)


def test_workspace_sizes(lib):
    assert ws_bytes(lib) >= 256
    assert ws_bytes(lib) % 256 == 0
    # the sequential path's fp32 forward partial: batch*L*H*P*4 bytes at least
    assert ws_bytes(lib, dtype=0) >= 256 + 2 * 256 * 4 * 64 * 4
    assert ws_bytes(lib, op=1, dtype=0) == 256
    assert ws_bytes(lib, op=2, L=64) >= 256 + 2 * 64 * 4 * 64 * 4
    # rejected shapes size to 0
    assert ws_bytes(lib, P=32) == 0
    assert ws_bytes(lib, N=96) == 0
    assert ws_bytes(lib, G=3) == 0
    assert ws_bytes(lib, chunk=100) == 0
    assert ws_bytes(lib, dtype=7) == 0
    assert ws_bytes(lib, L=-1) == 0


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced on these paths


def bidir_call(lib, ptrs=None, ws=FAKE, wsb=1 << 40, batch=2, L=256, H=4, P=64, N=128, G=4,
               chunk=128, dtype=1, path=None):
    p = ptrs or [FAKE] * 7
    args = [ctypes.c_void_p(v) for v in p] + [batch, L, H, P, N, G, chunk, dtype]
    if path is None:
        return lib.ssd_bidir_fwd(*args, ctypes.c_void_p(ws), wsb, None)
    return lib.ssd_bidir_fwd_path(*args, path, ctypes.c_void_p(ws), wsb, None)


def test_bidir_rejects_bad_arguments(lib):
    assert bidir_call(lib, P=32) == -2
    assert bidir_call(lib, N=256) == -2
    assert bidir_call(lib, chunk=96) == -2
    assert bidir_call(lib, dtype=5) == -2
    assert bidir_call(lib, G=3) == -1
    assert bidir_call(lib, batch=-1) == -1
    assert bidir_call(lib, H=0) == -1
    assert bidir_call(lib, ws=0) == -4
    assert bidir_call(lib, wsb=255) == -4
    assert bidir_call(lib, wsb=ws_bytes(lib) - 1) == -4
    assert bidir_call(lib, path=9) == -1
    for i in range(7):
        p = [FAKE] * 7
        p[i] = 0
        assert bidir_call(lib, ptrs=p) == -1, i
        p[i] = FAKE + 2  # misaligned
        assert bidir_call(lib, ptrs=p) == -1, i
    assert bidir_call(lib, ws=FAKE + 8) == -1


def test_bidir_empty_problem_launches_nothing(lib):
    # zero tokens: nothing to compute, null tensor pointers are fine
    assert bidir_call(lib, ptrs=[0] * 7, batch=0) == 0
    assert bidir_call(lib, ptrs=[0] * 7, L=0) == 0


def test_prefix_and_block_reject_bad_arguments(lib):
    v = ctypes.c_void_p
    ps = lambda *ints, ws=FAKE, wsb=1 << 40, init=0, out=FAKE: lib.ssd_prefix_state(
        v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(init), v(out), *ints, v(ws), wsb, None)
    assert ps(2, 128, 4, 64, 128, 4, 128, 1, ws=0) == -4
    assert ps(2, 128, 4, 64, 128, 3, 128, 1) == -1
    assert ps(2, 128, 4, 32, 128, 4, 128, 1) == -2
    assert ps(2, 128, 4, 64, 128, 4, 128, 1, out=0) == -1
    assert ps(2, 128, 4, 64, 128, 4, 128, 1, init=FAKE + 4) == -1
    bs = lambda *ints, ws=FAKE, wsb=1 << 40, ptr=FAKE: lib.ssd_block_step(
        v(ptr), v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(0), v(FAKE), *ints, v(ws), wsb, None)
    assert bs(4, 64, 32, 64, 128, 32, 1, ws=0) == -4
    assert bs(4, 64, 32, 64, 128, 5, 1) == -1
    assert bs(4, 64, 32, 64, 64, 32, 9) == -2
    assert bs(4, 64, 32, 64, 128, 32, 1, ptr=0) == -1
    assert bs(0, 64, 32, 64, 128, 32, 1, ptr=0) == 0


def test_auto_path_takes_the_one_tile_kernel_for_short_bf16_sequences(lib):
    """ssd_select_path (host only): bf16 sequences of at most 128 tokens with
    d_state 64 or 128 run the one-tile kernel (SSD_PATH_ONETILE = 7) whatever
    the batch and grouping; longer ones, fp32 and other d_state do not."""
    sp = lambda *a: lib.ssd_select_path(*a)
    for batch, L, H, N, G in [(512, 128, 24, 128, 1), (1, 1, 2, 64, 1), (6, 100, 8, 128, 2), (3, 77, 8, 64, 8)]:
        assert sp(batch, L, H, 64, N, G, 64, 1) == 7, (batch, L, H, N, G)
    assert sp(512, 129, 24, 64, 128, 1, 64, 1) != 7
    assert sp(512, 128, 24, 64, 128, 1, 64, 0) == 1          # fp32: the sequential scan
    assert sp(4, 128, 24, 64, 32, 1, 64, 1) != 7             # d_state 32 is not a one-tile shape


def test_status_requires_workspace(lib):
    assert lib.ssd_get_device_status(None, None) == -4
    assert lib.ssd_workspace_init(None, 256, None) == -4


def test_segment_entry_points_reject_bad_arguments(lib):
    v = ctypes.c_void_p
    st = lambda *ints, ws=FAKE, wsb=1 << 40, x=FAKE, so=FAKE: lib.ssd_segment_states(
        v(x), v(FAKE), v(FAKE), v(FAKE), v(so), v(FAKE), v(FAKE), v(FAKE), *ints, v(ws), wsb, None)
    assert st(2, 256, 4, 64, 128, 4, 1, ws=0) == -4
    assert st(2, 256, 4, 64, 128, 3, 1) == -1            # ngroups does not divide nheads
    assert st(2, 256, 4, 64, 128, 4, 0) == -2            # fp32: not on this path
    assert st(2, 0, 4, 64, 128, 4, 1) == -2              # an empty segment has no states to compute
    assert st(2, 256, 4, 64, 128, 4, 1, x=0) == -1
    assert st(2, 256, 4, 64, 128, 4, 1, so=FAKE + 4) == -1
    assert st(0, 256, 4, 64, 128, 4, 1, x=0) == 0
    cy = lambda nseg, seg, *ints, fi=FAKE: lib.ssd_segment_carry(
        v(FAKE), v(FAKE), v(FAKE), v(FAKE), nseg, seg, v(fi), v(FAKE), *ints, None)
    assert cy(4, 4, 2, 4, 64, 128) == -1                 # seg out of range
    assert cy(4, -1, 2, 4, 64, 128) == -1
    assert cy(0, 0, 2, 4, 64, 128) == -1
    assert cy(4, 1, 2, 4, 64, 96) == -2
    assert cy(4, 1, 2, 4, 64, 128, fi=0) == -1
    assert cy(4, 1, 0, 4, 64, 128, fi=0) == 0
    sd = lambda *ints, ws=FAKE, wsb=1 << 40, out=FAKE, init=0: lib.ssd_bidir_fwd_seeded(
        v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(init), v(0), v(out), *ints, v(ws), wsb, None)
    assert sd(2, 256, 4, 64, 128, 4, 1, ws=0) == -4
    assert sd(2, 256, 4, 64, 128, 4, 0) == -2
    assert sd(2, 256, 4, 64, 128, 4, 1, out=0) == -1
    assert sd(2, 256, 4, 64, 128, 4, 1, init=FAKE + 8) == -1
    assert sd(2, 0, 4, 64, 128, 4, 1, out=0) == 0


def test_dtraw_rejects_bad_arguments(lib):
    v = ctypes.c_void_p
    f = ctypes.c_float
    call = lambda *ints, lo=0.0, hi=1.0, ws=FAKE, wsb=1 << 40, bias=FAKE, out=FAKE: lib.ssd_bidir_fwd_dtraw(
        v(FAKE), v(FAKE), v(bias), f(lo), f(hi), v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(out), *ints, v(ws), wsb, None)
    assert call(2, 256, 4, 64, 128, 4, 1, ws=0) == -4
    assert call(2, 256, 4, 64, 128, 4, 0) == -2                   # fp32: not on this path
    assert call(2, 256, 4, 64, 128, 4, 1, lo=-1.0) == -1          # negative lower bound
    assert call(2, 256, 4, 64, 128, 4, 1, lo=0.2, hi=0.1) == -1   # empty range
    assert call(2, 256, 4, 64, 128, 4, 1, lo=float("nan")) == -1
    assert call(2, 256, 4, 64, 128, 4, 1, bias=0) == -1
    assert call(2, 256, 4, 64, 128, 4, 1, bias=FAKE + 2) == -1
    assert call(2, 0, 4, 64, 128, 4, 1, out=0) == 0
