"""Bidirectional Mamba-2 SSD mixer for B200 (sm_100a): Python binding.

A thin layer over the C ABI of libssd_bidir.so (include/ssd_bidir.h): it
checks that the torch tensors it is handed are contiguous CUDA tensors of
the expected dtype, passes their device pointers, sizes and the current CUDA
stream to the library, and allocates outputs and the workspace with torch.
Every step of the computation runs in the library's kernels.

Functions carry the C names:
  ssd_bidir_fwd(x, dt, A, B, C, D, chunk=256)          -> out
  ssd_bidir_bwd(x, dt, A, B, C, D, dy)                 -> dict of fp32 gradients dx, ddt, dA, dB, dC, dD
  ssd_bidir_fwd_x2(x2, dt, A, B, C, D)                 -> out (each direction scans its own x, x2 (2,b,L,H,P))
  ssd_mixer_block_fwd(xbc, z, dt_raw, conv_w, conv_b, dt_bias, A, D, norm_w, H, G, N) -> out
  ssd_prefix_state(x, dt, A, B, init=None, chunk=256)  -> state (batch, H, P, N) fp32
  ssd_prefix_state_layers(x, dt, A, B, init=None)      -> states (layers, batch, H, P, N) fp32
  ssd_block_step(x, dt, A, B, C, D, prefix_state)      -> out
  ssd_segment_states(x, dt, A, B)                      -> (fwd_state, fwd_decay, rev_state, rev_decay)
  ssd_segment_carry(fwd_states, fwd_decays, rev_states, rev_decays, seg) -> (fwd_in, rev_in)
  ssd_bidir_fwd_seeded(x, dt, A, B, C, D, fwd_init, rev_init)           -> out
  ssd_bidir_fwd_dtraw(x, dt_raw, dt_bias, A, B, C, D, dt_min, dt_max)   -> out
The sequence-sharded mixer over a process group is in seqshard.py; the
block-diffusion cache of several layers and the CUDA-graph block loop are in
blockdiff.py.
Shapes (row-major, natural token order; [0] forward, [1] reverse):
  x (batch, L, H, P); dt (2, batch, L, H); A, D (2, H) fp32;
  B, C (2, batch, L, G, N); out like x.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib as _c
from ._lib import (SSD_PATH_AUTO, SSD_PATH_SIMT, SSD_PATH_CHUNKED, SSD_PATH_FUSED, SSD_PATH_SEGMENTED,  # noqa: F401
                   SSD_PATH_PAIR, SSD_PATH_BLOCK, SSD_PATH_ONETILE,
                   SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA,
                   SSD_ERR_WORKSPACE, SSD_ERR_TIMEOUT, SSD_OP_BIDIR_FWD, SSD_OP_PREFIX_STATE,
                   SSD_OP_BLOCK_STEP, SSD_OP_BIDIR_BWD, SSD_OP_BIDIR_FWD_X2, SSD_OP_MIXER_BLOCK)

__all__ = ["ssd_bidir_fwd", "ssd_bidir_bwd", "ssd_bidir_fwd_x2", "ssd_mixer_block_fwd", "ssd_prefix_state",
           "ssd_prefix_state_layers", "ssd_block_step",
           "ssd_segment_states",
           "ssd_segment_carry", "ssd_bidir_fwd_seeded", "ssd_bidir_fwd_dtraw", "ssd_workspace_bytes",
           "ssd_get_device_status", "SSDError", "Workspace", "lib"]

lib = _c.load()

_DT = {torch.float32: _c.SSD_F32, torch.bfloat16: _c.SSD_BF16}


class SSDError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.ssd_error_string(status).decode()} (status {status})")


def _check(rc: int, what: str):
    if rc != _c.SSD_OK:
        raise SSDError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(t, name, dtype=None, device=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims (got {tuple(t.shape)})")


def ssd_workspace_bytes(op, batch, seqlen, nheads, headdim, dstate, ngroups, chunk, dtype) -> int:
    code = _DT[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return int(lib.ssd_workspace_bytes(op, batch, seqlen, nheads, headdim, dstate, ngroups,
                                       chunk, code))


class Workspace:
    """A device buffer for the library's workspace, grown on demand.

    The first 256 bytes are the status header; the buffer is zero-filled on
    (re)allocation, which initialises it. One Workspace must not be shared by
    calls that overlap on the device (different streams)."""

    def __init__(self, device=None):
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf

    def status(self) -> int:
        """Synchronise the current stream and read (and clear) the status header."""
        if self.buf is None:
            return _c.SSD_OK
        return int(lib.ssd_get_device_status(_ptr(self.buf), ctypes.c_void_p(_stream(self.device))))


_default_ws: dict = {}


def _workspace(device, stream, ws):
    if ws is not None:
        return ws
    key = (device.index, stream)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def ssd_get_device_status(ws: Workspace | None = None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device())
    w = _workspace(dev, _stream(dev), ws)
    return w.status()


def _dims(x, B):
    batch, L, H, P = x.shape
    G, N = B.shape[-2], B.shape[-1]
    return batch, L, H, P, G, N


def ssd_bidir_fwd(x, dt, A, B, C, D, out=None, *, chunk: int = 256, path: int = SSD_PATH_AUTO,
                  workspace: Workspace | None = None):
    """Bidirectional SSD mixer over whole sequences (include/ssd_bidir.h: ssd_bidir_fwd)."""
    _need(x, "x", ndim=4)
    dev, io = x.device, x.dtype
    if io not in _DT:
        raise ValueError(f"x dtype {io} not supported (float32 or bfloat16)")
    _need(dt, "dt", io, dev, 4)
    _need(B, "B", io, dev, 5)
    _need(C, "C", io, dev, 5)
    _need(A, "A", torch.float32, dev, 2)
    _need(D, "D", torch.float32, dev, 2)
    batch, L, H, P, G, N = _dims(x, B)
    if tuple(dt.shape) != (2, batch, L, H) or tuple(B.shape) != (2, batch, L, G, N) \
            or tuple(C.shape) != tuple(B.shape) or tuple(A.shape) != (2, H) or tuple(D.shape) != (2, H):
        raise ValueError("shape mismatch: want x (b,L,H,P), dt (2,b,L,H), B/C (2,b,L,G,N), A/D (2,H)")
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", io, dev, 4)
        if out.shape != x.shape:
            raise ValueError("out must have x's shape")
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, L, H, P, N, G, chunk, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_bidir_fwd")
    buf = ws.get(nbytes)
    rc = lib.ssd_bidir_fwd_path(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(out),
                                batch, L, H, P, N, G, chunk, _DT[io], int(path),
                                _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_bidir_fwd")
    return out


def ssd_prefix_state(x, dt, A, B, init=None, out=None, *, chunk: int = 256, path: int = SSD_PATH_AUTO,
                     workspace: Workspace | None = None):
    """Forward-only state after the last token (include/ssd_bidir.h: ssd_prefix_state,
    ssd_prefix_state_path). dt (batch, L, H), A (H), B (batch, L, G, N): the forward
    direction's. `path`: as for ssd_bidir_fwd."""
    _need(x, "x", ndim=4)
    dev, io = x.device, x.dtype
    if io not in _DT:
        raise ValueError(f"x dtype {io} not supported (float32 or bfloat16)")
    _need(dt, "dt", io, dev, 3)
    _need(B, "B", io, dev, 4)
    _need(A, "A", torch.float32, dev, 1)
    batch, L, H, P = x.shape
    G, N = B.shape[-2], B.shape[-1]
    if tuple(dt.shape) != (batch, L, H) or tuple(B.shape) != (batch, L, G, N) or tuple(A.shape) != (H,):
        raise ValueError("shape mismatch: want x (b,L,H,P), dt (b,L,H), B (b,L,G,N), A (H)")
    if init is not None:
        _need(init, "init", torch.float32, dev, 4)
        if tuple(init.shape) != (batch, H, P, N):
            raise ValueError("init must be (batch, H, P, N)")
    if out is None:
        out = torch.empty(batch, H, P, N, dtype=torch.float32, device=dev)
    else:
        _need(out, "out", torch.float32, dev, 4)
        if tuple(out.shape) != (batch, H, P, N):
            raise ValueError("out must be (batch, H, P, N)")
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_PREFIX_STATE, batch, L, H, P, N, G, chunk, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_prefix_state")
    buf = ws.get(nbytes)
    rc = lib.ssd_prefix_state_path(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(init), _ptr(out),
                                   batch, L, H, P, N, G, chunk, _DT[io], int(path),
                                   _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_prefix_state")
    return out


def ssd_prefix_state_layers(x, dt, A, B, init=None, out=None, *, chunk: int = 256,
                            workspace: Workspace | None = None):
    """Forward-only states of several layers at once (include/ssd_bidir.h:
    ssd_prefix_state_layers): x (layers, batch, L, H, P), dt (layers, batch, L,
    H), A (layers, H), B (layers, batch, L, G, N), init / out (layers, batch, H,
    P, N) fp32; out may be init (in-place commit)."""
    _need(x, "x", ndim=5)
    dev, io = x.device, x.dtype
    if io not in _DT:
        raise ValueError(f"x dtype {io} not supported (float32 or bfloat16)")
    _need(dt, "dt", io, dev, 4)
    _need(B, "B", io, dev, 5)
    _need(A, "A", torch.float32, dev, 2)
    layers, batch, L, H, P = x.shape
    G, N = B.shape[-2], B.shape[-1]
    if tuple(dt.shape) != (layers, batch, L, H) or tuple(B.shape) != (layers, batch, L, G, N) \
            or tuple(A.shape) != (layers, H):
        raise ValueError("shape mismatch: want x (l,b,L,H,P), dt (l,b,L,H), B (l,b,L,G,N), A (l,H)")
    shape = (layers, batch, H, P, N)
    if init is not None:
        _need(init, "init", torch.float32, dev, 5)
        if tuple(init.shape) != shape:
            raise ValueError("init must be (layers, batch, H, P, N)")
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=dev)
    else:
        _need(out, "out", torch.float32, dev, 5)
        if tuple(out.shape) != shape:
            raise ValueError("out must be (layers, batch, H, P, N)")
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_PREFIX_STATE, layers * batch, L, H, P, N, G, chunk, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_prefix_state_layers")
    buf = ws.get(nbytes)
    rc = lib.ssd_prefix_state_layers(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(init), _ptr(out),
                                     layers, batch, L, H, P, N, G, chunk, _DT[io],
                                     _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_prefix_state_layers")
    return out


def ssd_block_step(x, dt, A, B, C, D, prefix_state, out=None, *, path: int = SSD_PATH_AUTO,
                   workspace: Workspace | None = None):
    """One block-diffusion step on the active block (include/ssd_bidir.h: ssd_block_step,
    ssd_block_step_path). `path`: SSD_PATH_AUTO, SIMT, CHUNKED, FUSED or BLOCK (the
    one-tile kernel, bf16 blocks of at most 64 tokens)."""
    _need(x, "x", ndim=4)
    dev, io = x.device, x.dtype
    if io not in _DT:
        raise ValueError(f"x dtype {io} not supported (float32 or bfloat16)")
    _need(dt, "dt", io, dev, 4)
    _need(B, "B", io, dev, 5)
    _need(C, "C", io, dev, 5)
    _need(A, "A", torch.float32, dev, 2)
    _need(D, "D", torch.float32, dev, 2)
    batch, T, H, P, G, N = _dims(x, B)
    if tuple(dt.shape) != (2, batch, T, H) or tuple(B.shape) != (2, batch, T, G, N) \
            or tuple(C.shape) != tuple(B.shape) or tuple(A.shape) != (2, H) or tuple(D.shape) != (2, H):
        raise ValueError("shape mismatch: want x (b,T,H,P), dt (2,b,T,H), B/C (2,b,T,G,N), A/D (2,H)")
    if prefix_state is not None:
        _need(prefix_state, "prefix_state", torch.float32, dev, 4)
        if tuple(prefix_state.shape) != (batch, H, P, N):
            raise ValueError("prefix_state must be (batch, H, P, N)")
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", io, dev, 4)
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_BLOCK_STEP, batch, T, H, P, N, G, 64, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_block_step")
    buf = ws.get(nbytes)
    rc = lib.ssd_block_step_path(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                 _ptr(prefix_state), _ptr(out), batch, T, H, P, N, G, _DT[io],
                                 int(path), _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_block_step")
    return out


def _bidir_args(x, dt, A, B, C, D, what):
    _need(x, "x", ndim=4)
    dev, io = x.device, x.dtype
    if io != torch.bfloat16:
        raise ValueError(f"{what}: bf16 I/O only (got {io})")
    _need(dt, "dt", io, dev, 4)
    _need(B, "B", io, dev, 5)
    _need(A, "A", torch.float32, dev, 2)
    batch, L, H, P, G, N = _dims(x, B)
    if tuple(dt.shape) != (2, batch, L, H) or tuple(B.shape) != (2, batch, L, G, N) or tuple(A.shape) != (2, H):
        raise ValueError("shape mismatch: want x (b,L,H,P), dt (2,b,L,H), B (2,b,L,G,N), A (2,H)")
    if C is not None:
        _need(C, "C", io, dev, 5)
        _need(D, "D", torch.float32, dev, 2)
        if tuple(C.shape) != tuple(B.shape) or tuple(D.shape) != (2, H):
            raise ValueError("shape mismatch: want C like B, D (2,H)")
    return dev, io, batch, L, H, P, G, N


def _state(t, name, dev, shape):
    if t is not None:
        _need(t, name, torch.float32, dev, len(shape))
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must be {tuple(shape)}")


def ssd_segment_states(x, dt, A, B, *, workspace: Workspace | None = None):
    """A segment's own states from zero (include/ssd_bidir.h: ssd_segment_states):
    returns (fwd_state, fwd_decay, rev_state, rev_decay), states (batch, H, P, N)
    and decays (batch, H), fp32."""
    dev, io, batch, L, H, P, G, N = _bidir_args(x, dt, A, B, None, None, "ssd_segment_states")
    fs = torch.empty(batch, H, P, N, dtype=torch.float32, device=dev)
    rs = torch.empty_like(fs)
    fd = torch.empty(batch, H, dtype=torch.float32, device=dev)
    rd = torch.empty_like(fd)
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    buf = ws.get(max(ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, L, H, P, N, G, 64, io), 256))
    rc = lib.ssd_segment_states(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(fs), _ptr(fd), _ptr(rs), _ptr(rd),
                                batch, L, H, P, N, G, _DT[io], _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_segment_states")
    return fs, fd, rs, rd


def ssd_segment_carry(fwd_states, fwd_decays, rev_states, rev_decays, seg: int):
    """The states entering segment `seg` from all segments' own states, gathered
    segment-major (include/ssd_bidir.h: ssd_segment_carry): states (nseg, batch,
    H, P, N), decays (nseg, batch, H). Returns (fwd_in, rev_in), (batch, H, P, N)."""
    _need(fwd_states, "fwd_states", torch.float32, None, 5)
    dev = fwd_states.device
    nseg, batch, H, P, N = fwd_states.shape
    _state(rev_states, "rev_states", dev, (nseg, batch, H, P, N))
    _state(fwd_decays, "fwd_decays", dev, (nseg, batch, H))
    _state(rev_decays, "rev_decays", dev, (nseg, batch, H))
    fi = torch.empty(batch, H, P, N, dtype=torch.float32, device=dev)
    ri = torch.empty_like(fi)
    rc = lib.ssd_segment_carry(_ptr(fwd_states), _ptr(fwd_decays), _ptr(rev_states), _ptr(rev_decays),
                               nseg, int(seg), _ptr(fi), _ptr(ri), batch, H, P, N,
                               ctypes.c_void_p(_stream(dev)))
    _check(rc, "ssd_segment_carry")
    return fi, ri


def ssd_bidir_fwd_seeded(x, dt, A, B, C, D, fwd_init=None, rev_init=None, out=None, *,
                         workspace: Workspace | None = None):
    """Both scans over a segment, the forward one from fwd_init and the reverse
    one from rev_init at its end (include/ssd_bidir.h: ssd_bidir_fwd_seeded)."""
    dev, io, batch, L, H, P, G, N = _bidir_args(x, dt, A, B, C, D, "ssd_bidir_fwd_seeded")
    _state(fwd_init, "fwd_init", dev, (batch, H, P, N))
    _state(rev_init, "rev_init", dev, (batch, H, P, N))
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", io, dev, 4)
        if out.shape != x.shape:
            raise ValueError("out must have x's shape")
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    buf = ws.get(max(ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, L, H, P, N, G, 64, io), 256))
    rc = lib.ssd_bidir_fwd_seeded(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(fwd_init),
                                  _ptr(rev_init), _ptr(out), batch, L, H, P, N, G, _DT[io],
                                  _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_bidir_fwd_seeded")
    return out


def ssd_bidir_fwd_dtraw(x, dt_raw, dt_bias, A, B, C, D, dt_min: float = 0.0, dt_max: float = float("inf"),
                        out=None, *, workspace: Workspace | None = None):
    """The mixer with the step size prepared in the kernel from the raw
    projection: dt = clamp(softplus(dt_raw + dt_bias), dt_min, dt_max)
    (include/ssd_bidir.h: ssd_bidir_fwd_dtraw). dt_raw like dt, dt_bias (2, H) fp32."""
    dev, io, batch, L, H, P, G, N = _bidir_args(x, dt_raw, A, B, C, D, "ssd_bidir_fwd_dtraw")
    _need(dt_bias, "dt_bias", torch.float32, dev, 2)
    if tuple(dt_bias.shape) != (2, H):
        raise ValueError("dt_bias must be (2, H)")
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", io, dev, 4)
        if out.shape != x.shape:
            raise ValueError("out must have x's shape")
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    buf = ws.get(max(ssd_workspace_bytes(SSD_OP_BIDIR_FWD, batch, L, H, P, N, G, 64, io), 256))
    rc = lib.ssd_bidir_fwd_dtraw(_ptr(x), _ptr(dt_raw), _ptr(dt_bias), float(dt_min), float(dt_max),
                                 _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(out), batch, L, H, P, N, G, _DT[io],
                                 _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_bidir_fwd_dtraw")
    return out


def ssd_bidir_bwd(x, dt, A, B, C, D, dy, *, fwd_init=None, rev_init=None,
                  workspace: Workspace | None = None) -> dict:
    """Gradients of sum(dy * ssd_bidir_fwd(x, dt, A, B, C, D)) with respect to
    every input (include/ssd_bidir.h: ssd_bidir_bwd), as fp32 tensors shaped
    like the inputs: dx, ddt, dA, dB, dC, dD. With fwd_init / rev_init
    (batch, H, P, N) fp32, the scans start from those states
    (ssd_bidir_fwd_seeded; ssd_bidir_bwd_seeded) and the dict also holds
    d_fwd_init / d_rev_init, their gradients."""
    _need(x, "x", ndim=4)
    dev, io = x.device, x.dtype
    if io not in _DT:
        raise ValueError(f"x dtype {io} not supported (float32 or bfloat16)")
    _need(dt, "dt", io, dev, 4)
    _need(B, "B", io, dev, 5)
    _need(C, "C", io, dev, 5)
    _need(dy, "dy", io, dev, 4)
    _need(A, "A", torch.float32, dev, 2)
    _need(D, "D", torch.float32, dev, 2)
    batch, L, H, P, G, N = _dims(x, B)
    if tuple(dt.shape) != (2, batch, L, H) or tuple(B.shape) != (2, batch, L, G, N) \
            or tuple(C.shape) != tuple(B.shape) or tuple(A.shape) != (2, H) or tuple(D.shape) != (2, H) \
            or dy.shape != x.shape:
        raise ValueError("shape mismatch: want x, dy (b,L,H,P), dt (2,b,L,H), B/C (2,b,L,G,N), A/D (2,H)")
    for name, st in (("fwd_init", fwd_init), ("rev_init", rev_init)):
        if st is not None:
            _need(st, name, torch.float32, dev, 4)
            if tuple(st.shape) != (batch, H, P, N):
                raise ValueError(f"{name} must be (batch, H, P, N)")
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"dx": torch.empty(x.shape, **f32), "ddt": torch.empty(dt.shape, **f32), "dA": torch.empty(A.shape, **f32),
         "dB": torch.empty(B.shape, **f32), "dC": torch.empty(C.shape, **f32), "dD": torch.empty(D.shape, **f32)}
    if fwd_init is not None:
        g["d_fwd_init"] = torch.empty((batch, H, P, N), **f32)
    if rev_init is not None:
        g["d_rev_init"] = torch.empty((batch, H, P, N), **f32)
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_BIDIR_BWD, batch, L, H, P, N, G, 64, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_bidir_bwd")
    buf = ws.get(nbytes)
    opt = lambda t: _ptr(t) if t is not None else None
    rc = lib.ssd_bidir_bwd_seeded(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), opt(fwd_init),
                                  opt(rev_init), _ptr(dy),
                                  *(_ptr(g[k]) for k in ("dx", "ddt", "dA", "dB", "dC", "dD")),
                                  opt(g.get("d_fwd_init")), opt(g.get("d_rev_init")),
                                  batch, L, H, P, N, G, _DT[io], _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_bidir_bwd")
    return g


def ssd_block_step_bwd(x, dt, A, B, C, D, prefix_state, dy, *, workspace: Workspace | None = None) -> dict:
    """Gradients of sum(dy * ssd_block_step(x, dt, A, B, C, D, prefix_state))
    with respect to the block's inputs and (as d_prefix_state, when one is
    given) the cached prefix state: the seeded backward with a forward start
    state and none for the reverse scan (include/ssd_bidir.h:
    ssd_bidir_bwd_seeded)."""
    g = ssd_bidir_bwd(x, dt, A, B, C, D, dy, fwd_init=prefix_state, workspace=workspace)
    if "d_fwd_init" in g:
        g["d_prefix_state"] = g.pop("d_fwd_init")
    return g


def ssd_bidir_fwd_x2(x2, dt, A, B, C, D, out=None, *, workspace: Workspace | None = None):
    """The bidirectional mixer with each direction scanning its own x
    (include/ssd_bidir.h: ssd_bidir_fwd_x2): x2 (2, batch, L, H, P)."""
    _need(x2, "x2", ndim=5)
    dev, io = x2.device, x2.dtype
    if io not in _DT:
        raise ValueError(f"x2 dtype {io} not supported (float32 or bfloat16)")
    _need(dt, "dt", io, dev, 4)
    _need(B, "B", io, dev, 5)
    _need(C, "C", io, dev, 5)
    _need(A, "A", torch.float32, dev, 2)
    _need(D, "D", torch.float32, dev, 2)
    two, batch, L, H, P = x2.shape
    G, N = B.shape[-2:]
    if two != 2 or tuple(dt.shape) != (2, batch, L, H) or tuple(B.shape) != (2, batch, L, G, N) \
            or tuple(C.shape) != tuple(B.shape) or tuple(A.shape) != (2, H) or tuple(D.shape) != (2, H):
        raise ValueError("shape mismatch: want x2 (2,b,L,H,P), dt (2,b,L,H), B/C (2,b,L,G,N), A/D (2,H)")
    if out is None:
        out = torch.empty(x2.shape[1:], dtype=io, device=dev)
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_BIDIR_FWD_X2, batch, L, H, P, N, G, 64, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_bidir_fwd_x2")
    buf = ws.get(nbytes)
    rc = lib.ssd_bidir_fwd_x2(_ptr(x2), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(out),
                              batch, L, H, P, N, G, _DT[io], _ptr(buf), buf.numel(), ctypes.c_void_p(stream))
    _check(rc, "ssd_bidir_fwd_x2")
    return out


def ssd_mixer_block_fwd(xbc, z, dt_raw, conv_w, conv_b, dt_bias, A, D, norm_w, nheads: int, ngroups: int,
                        dstate: int, *, dt_min: float = 0.0, dt_max: float = float("inf"), norm_eps: float = 1e-5,
                        out=None, workspace: Workspace | None = None):
    """The mixer with its input and output steps (include/ssd_bidir.h:
    ssd_mixer_block_fwd): xbc (batch, L, H*P + 2*G*N), z (batch, L, H, P),
    dt_raw (2, batch, L, H), conv_w (2, Cin, K), conv_b (2, Cin), dt_bias, A,
    D (2, H), norm_w (H*P,). Returns out (batch, L, H, P)."""
    _need(xbc, "xbc", ndim=3)
    dev, io = xbc.device, xbc.dtype
    if io not in _DT:
        raise ValueError(f"xbc dtype {io} not supported (float32 or bfloat16)")
    batch, L, cin = xbc.shape
    P = (cin - 2 * ngroups * dstate) // nheads
    if nheads * P + 2 * ngroups * dstate != cin:
        raise ValueError("xbc channels must be nheads*headdim + 2*ngroups*dstate")
    _need(z, "z", io, dev, 4)
    _need(dt_raw, "dt_raw", io, dev, 4)
    for name, t, nd in (("conv_w", conv_w, 3), ("conv_b", conv_b, 2), ("dt_bias", dt_bias, 2), ("A", A, 2),
                        ("D", D, 2), ("norm_w", norm_w, 1)):
        _need(t, name, torch.float32, dev, nd)
    K = conv_w.shape[2]
    if tuple(z.shape) != (batch, L, nheads, P) or tuple(dt_raw.shape) != (2, batch, L, nheads) \
            or tuple(conv_w.shape) != (2, cin, K) or tuple(conv_b.shape) != (2, cin) \
            or tuple(dt_bias.shape) != (2, nheads) or tuple(A.shape) != (2, nheads) or tuple(D.shape) != (2, nheads) \
            or tuple(norm_w.shape) != (nheads * P,):
        raise ValueError("shape mismatch in ssd_mixer_block_fwd")
    if out is None:
        out = torch.empty(batch, L, nheads, P, dtype=io, device=dev)
    stream = _stream(dev)
    ws = _workspace(dev, stream, workspace)
    nbytes = ssd_workspace_bytes(SSD_OP_MIXER_BLOCK, batch, L, nheads, P, dstate, ngroups, 64, io)
    if nbytes == 0:
        _check(_c.SSD_ERR_UNSUPPORTED, "ssd_mixer_block_fwd")
    buf = ws.get(nbytes)
    rc = lib.ssd_mixer_block_fwd(_ptr(xbc), _ptr(z), _ptr(dt_raw), _ptr(conv_w), _ptr(conv_b), K, _ptr(dt_bias),
                                 float(dt_min), float(dt_max), _ptr(A), _ptr(D), _ptr(norm_w), float(norm_eps),
                                 _ptr(out), batch, L, nheads, P, dstate, ngroups, _DT[io], _ptr(buf), buf.numel(),
                                 ctypes.c_void_p(stream))
    _check(rc, "ssd_mixer_block_fwd")
    return out
