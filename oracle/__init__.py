"""fp64 CPU oracle for the bidirectional Mamba-2 SSD mixer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the library and its binding never
do. It shares no code with the CUDA path (see ``ssd_oracle.c`` for the
definition it follows and the passages it cites).

Every function takes numpy arrays of any float dtype (they are widened to
float64, so bf16 inputs handed to the GPU are seen here exactly), in the
library's layouts:

    x      (batch, L, H, P)
    dt     (2, batch, L, H)      [0] forward, [1] reverse
    A      (2, H)
    B, C   (2, batch, L, G, N)
    D      (2, H)
    state  (batch, H, P, N)      forward state, P rows of N

Parity status: pinned. ``tests/test_oracle_pins.py`` checks this oracle
against the materialised quadratic form, closed forms (A -> -inf, A = 0, the
geometric series of a constant input), the flip identity, composability of
prefix states and a hand-worked golden example; none of those checks calls
the oracle's own loop to produce its expected value. ``bidir_seeded`` is
pinned to the other functions: with zero states it is ``block_step`` with no
prefix; its segments, seeded with the states the rest of the sequence leaves
(from ``prefix_state`` on either side, the reverse one through the flip
identity), put together give ``bidir`` over the whole sequence.
``bidir_bwd`` (gradients) is pinned by central finite differences of
``bidir``, by the exact adjoint identities of the maps that are linear (y in
x, in B and in C) and by the closed form of a memoryless scan (A -> -inf);
``tests/test_oracle_bwd_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libssd_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c with gcc (-O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def configure(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    i = ctypes.c_int
    lib.ssd_oracle_bidir.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, ip, i, i]
    lib.ssd_oracle_prefix_state.argtypes = [dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i]
    lib.ssd_oracle_block_step.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i]
    lib.ssd_oracle_bidir_seeded.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i]
    lib.ssd_oracle_bidir_bwd.argtypes = [dp] * 13 + [i] * 7
    lib.ssd_oracle_threads.argtypes = [i]
    for f in (lib.ssd_oracle_bidir, lib.ssd_oracle_prefix_state, lib.ssd_oracle_block_step,
              lib.ssd_oracle_bidir_seeded, lib.ssd_oracle_bidir_bwd, lib.ssd_oracle_threads):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _f64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def threads(n: int = 0) -> int:
    """Set (n > 0) and return the OpenMP thread count the oracle uses."""
    return _load().ssd_oracle_threads(int(n))


def bidir(x, dt, A, B, C, D, units=None, nthreads: int = 0) -> np.ndarray:
    """y = forward scan + reverse scan + (D_f + D_b) x over whole sequences.

    units: optional iterable of (b, h) pairs; only those outputs are computed
    (the rest of the returned array is NaN)."""
    x = np.asarray(x)
    batch, L, H, P = x.shape
    G, N = np.asarray(B).shape[-2:]
    out = np.full((batch, L, H, P), np.nan)
    keep = [_f64(a) for a in (x, dt, A, B, C, D)]
    po = out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    if units is None:
        uptr, nu = None, 0
    else:
        uarr = np.ascontiguousarray(np.array([b * H + h for b, h in units], dtype=np.int32))
        uptr, nu = uarr.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), len(uarr)
    rc = _load().ssd_oracle_bidir(*(p for _, p in keep), po, batch, L, H, P, N, G,
                                  uptr, nu, int(nthreads))
    if rc != 0:
        raise ValueError("oracle bidir: bad arguments")
    return out


def prefix_state(x, dt, A, B, init=None, nthreads: int = 0) -> np.ndarray:
    """Forward-only state after the last token; dt (batch, L, H), A (H),
    B (batch, L, G, N) are the forward direction's. Returns (batch, H, P, N)."""
    x = np.asarray(x)
    batch, L, H, P = x.shape
    G, N = np.asarray(B).shape[-2:]
    out = np.zeros((batch, H, P, N))
    keep = [_f64(a) for a in (x, dt, A, B)]
    if init is None:
        pinit = None
    else:
        init_a, pinit = _f64(init)
    po = out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    rc = _load().ssd_oracle_prefix_state(*(p for _, p in keep), pinit, po,
                                         batch, L, H, P, N, G, int(nthreads))
    if rc != 0:
        raise ValueError("oracle prefix_state: bad arguments")
    return out


def block_step(x, dt, A, B, C, D, prefix, nthreads: int = 0) -> np.ndarray:
    """One block-diffusion step over a block of T tokens: forward scan from
    the prefix state, reverse scan confined to the block, plus D terms."""
    x = np.asarray(x)
    batch, T, H, P = x.shape
    G, N = np.asarray(B).shape[-2:]
    out = np.zeros((batch, T, H, P))
    keep = [_f64(a) for a in (x, dt, A, B, C, D)]
    if prefix is None:
        pp = None
    else:
        pre_a, pp = _f64(prefix)
    po = out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    rc = _load().ssd_oracle_block_step(*(p for _, p in keep), pp, po,
                                       batch, T, H, P, N, G, int(nthreads))
    if rc != 0:
        raise ValueError("oracle block_step: bad arguments")
    return out


def bidir_seeded(x, dt, A, B, C, D, prefix=None, suffix=None, nthreads: int = 0) -> np.ndarray:
    """Both scans over a segment with given starting states: the forward scan
    from `prefix` (the state before the first token), the reverse scan from
    `suffix` (the reverse state after the last token), plus the D terms.
    prefix, suffix (batch, H, P, N) or None (zero)."""
    x = np.asarray(x)
    batch, L, H, P = x.shape
    G, N = np.asarray(B).shape[-2:]
    out = np.zeros((batch, L, H, P))
    keep = [_f64(a) for a in (x, dt, A, B, C, D)]
    ptrs = []
    for s in (prefix, suffix):
        if s is None:
            ptrs.append(None)
        else:
            a, pa = _f64(s)
            keep.append((a, pa))
            ptrs.append(pa)
    po = out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    rc = _load().ssd_oracle_bidir_seeded(*(p for _, p in keep[:6]), ptrs[0], ptrs[1], po,
                                         batch, L, H, P, N, G, int(nthreads))
    if rc != 0:
        raise ValueError("oracle bidir_seeded: bad arguments")
    return out


def dt_prep(dt_raw, dt_bias, dt_min=0.0, dt_max=np.inf) -> np.ndarray:
    """The step size a Mamba-2 layer feeds its scan, from the raw projection:
    dt = clamp(softplus(dt_raw + dt_bias[d, h]), dt_min, dt_max), with
    softplus(u) = log(1 + exp(u)), in fp64. dt_raw (2, batch, L, H), dt_bias
    (2, H). The pages name Mamba-2 without printing its parametrisation; this
    is the standard Mamba-2 one (a positive step from a biased softplus,
    limited to a range), the input side of the mixer (before the scan)."""
    u = np.asarray(dt_raw, dtype=np.float64) + np.asarray(dt_bias, dtype=np.float64)[:, None, None, :]
    sp = np.logaddexp(0.0, u)          # log(1 + exp(u)) without overflow
    return np.clip(sp, dt_min, dt_max)


def bidir_bwd(x, dt, A, B, C, D, dy, nthreads: int = 0) -> dict:
    """Gradients of sum(dy * bidir(x, dt, A, B, C, D)) with respect to every
    input, in fp64, from the adjoint of the recurrence token by token (see
    ssd_oracle.c). Returns a dict of arrays shaped like the inputs: dx, ddt,
    dA, dB, dC, dD."""
    x = np.asarray(x)
    batch, L, H, P = x.shape
    G, N = np.asarray(B).shape[-2:]
    keep = [_f64(a) for a in (x, dt, A, B, C, D, dy)]
    outs = {"dx": np.zeros((batch, L, H, P)), "ddt": np.zeros((2, batch, L, H)), "dA": np.zeros((2, H)),
            "dB": np.zeros((2, batch, L, G, N)), "dC": np.zeros((2, batch, L, G, N)), "dD": np.zeros((2, H))}
    po = [outs[k].ctypes.data_as(ctypes.POINTER(ctypes.c_double)) for k in ("dx", "ddt", "dA", "dB", "dC", "dD")]
    rc = _load().ssd_oracle_bidir_bwd(*(p for _, p in keep), *po, batch, L, H, P, N, G, int(nthreads))
    if rc != 0:
        raise ValueError("oracle bidir_bwd: bad arguments")
    return outs
