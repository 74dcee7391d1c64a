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
    lib.ssd_oracle_bidir_bwd_seeded.argtypes = [dp] * 17 + [i] * 7
    lib.ssd_oracle_threads.argtypes = [i]
    for f in (lib.ssd_oracle_bidir, lib.ssd_oracle_prefix_state, lib.ssd_oracle_block_step,
              lib.ssd_oracle_bidir_seeded, lib.ssd_oracle_bidir_bwd, lib.ssd_oracle_bidir_bwd_seeded,
              lib.ssd_oracle_threads):
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


def bidir_bwd(x, dt, A, B, C, D, dy, prefix=None, suffix=None, nthreads: int = 0) -> dict:
    """Gradients of sum(dy * bidir_seeded(x, dt, A, B, C, D, prefix, suffix))
    (bidir when both states are None) with respect to every input, in fp64,
    from the adjoint of the recurrence token by token (see ssd_oracle.c).
    Returns a dict of arrays shaped like the inputs: dx, ddt, dA, dB, dC, dD,
    and dprefix / dsuffix for the states that are given. With suffix None and
    a prefix, these are the gradients of the block step."""
    x = np.asarray(x)
    batch, L, H, P = x.shape
    G, N = np.asarray(B).shape[-2:]
    keep = [_f64(a) for a in (x, dt, A, B, C, D)]
    states = [None if s is None else _f64(s) for s in (prefix, suffix)]
    keep_dy = _f64(dy)
    outs = {"dx": np.zeros((batch, L, H, P)), "ddt": np.zeros((2, batch, L, H)), "dA": np.zeros((2, H)),
            "dB": np.zeros((2, batch, L, G, N)), "dC": np.zeros((2, batch, L, G, N)), "dD": np.zeros((2, H))}
    if prefix is not None:
        outs["dprefix"] = np.zeros((batch, H, P, N))
    if suffix is not None:
        outs["dsuffix"] = np.zeros((batch, H, P, N))
    dp = ctypes.POINTER(ctypes.c_double)
    po = [outs[k].ctypes.data_as(dp) for k in ("dx", "ddt", "dA", "dB", "dC", "dD")]
    pd = [outs[k].ctypes.data_as(dp) if k in outs else None for k in ("dprefix", "dsuffix")]
    rc = _load().ssd_oracle_bidir_bwd_seeded(*(p for _, p in keep), *(None if s is None else s[1] for s in states),
                                             keep_dy[1], *po, *pd, batch, L, H, P, N, G, int(nthreads))
    if rc != 0:
        raise ValueError("oracle bidir_bwd: bad arguments")
    return outs


# ------------------------------------------------------------------ mixer block
# The steps either side of the mixer in a Mamba-2 layer, for the bidirectional
# model ("DiffMamba - Checkpoints" model card, Model details: forward and
# flipped-reverse Mamba-2 layers with weight-tied projections, Mamba-2
# defaults). The pages print none of these steps; they are the standard
# Mamba-2 ones, read for two directions as follows (listed with the other
# readings): each direction has its own depthwise conv1d over the projected
# xBC channels, causal for the forward scan and, for the reverse scan, the
# flipped sequence's causal conv, i.e. anti-causal in natural order; SiLU
# after it; the channels split into x (H*P), B (G*N), C (G*N); each direction
# scans its own x and adds its own D x; the summed output is gated by SiLU(z)
# and RMS-normalised over its H*P channels with one weight vector.

def silu(v):
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def conv_silu(xbc, w, bias):
    """Both directions' depthwise conv1d + SiLU of xbc (batch, L, Cin): w (2,
    Cin, K), bias (2, Cin). Forward: out[t] = sum_k w[0][c][k] in[t - K + 1 + k];
    reverse: out[t] = sum_k w[1][c][k] in[t + K - 1 - k]; zero outside the
    sequence. Returns (2, batch, L, Cin) after SiLU."""
    xbc = np.asarray(xbc, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    bias = np.asarray(bias, dtype=np.float64)
    batch, L, cin = xbc.shape
    K = w.shape[2]
    out = np.zeros((2, batch, L, cin))
    for t in range(L):
        acc_f = np.array(bias[0], dtype=np.float64) * np.ones((batch, cin))
        acc_b = np.array(bias[1], dtype=np.float64) * np.ones((batch, cin))
        for k in range(K):
            s = t - (K - 1) + k            # forward tap k reads token s
            if 0 <= s < L:
                acc_f = acc_f + w[0][:, k] * xbc[:, s]
            r = t + (K - 1) - k            # reverse tap k reads token r
            if 0 <= r < L:
                acc_b = acc_b + w[1][:, k] * xbc[:, r]
        out[0, :, t] = acc_f
        out[1, :, t] = acc_b
    return silu(out)


def split_xbc(u, H, P, G, N):
    """(2, batch, L, H*P + 2*G*N) -> x2 (2, batch, L, H, P), B, C (2, batch, L, G, N)."""
    two, batch, L, _ = u.shape
    x2 = u[..., :H * P].reshape(two, batch, L, H, P)
    B = u[..., H * P:H * P + G * N].reshape(two, batch, L, G, N)
    C = u[..., H * P + G * N:].reshape(two, batch, L, G, N)
    return x2, B, C


def bidir_x2(x2, dt, A, B, C, D, nthreads: int = 0):
    """The bidirectional mixer with each direction scanning its own x:
    y = scan_f(x2[0]) + scan_b(x2[1]) + D_f x2[0] + D_b x2[1]. Each direction's
    part is the pinned bidir() with the other direction's C and D zeroed."""
    C = np.asarray(C, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    parts = []
    for d in range(2):
        Cd, Dd = C.copy(), D.copy()
        Cd[1 - d] = 0.0
        Dd[1 - d] = 0.0
        parts.append(bidir(x2[d], dt, A, B, Cd, Dd, nthreads=nthreads))
    return parts[0] + parts[1]


def gated_rmsnorm(y, z, w, eps=1e-5):
    """Mamba-2's gated RMS norm of the mixer output over its H*P channels:
    v = y * SiLU(z), out = v / sqrt(mean(v^2) + eps) * w. y, z (batch, L, H,
    P); w (H*P,)."""
    y = np.asarray(y, dtype=np.float64)
    batch, L, H, P = y.shape
    v = (y * silu(z)).reshape(batch, L, H * P)
    r = 1.0 / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return (v * r * np.asarray(w, dtype=np.float64)).reshape(batch, L, H, P)


def mixer_block(xbc, z, dt_raw, conv_w, conv_b, dt_bias, A, D, norm_w, H, P, G, N,
                dt_min=0.0, dt_max=np.inf, eps=1e-5):
    """The bidirectional mixer with its input and output steps: conv1d + SiLU
    per direction, the step size from the raw projection (dt_prep), the mixer
    with per-direction x, then the gated RMS norm of the sum."""
    u = conv_silu(xbc, conv_w, conv_b)
    x2, B, C = split_xbc(u, H, P, G, N)
    dt = dt_prep(dt_raw, dt_bias, dt_min, dt_max)
    y = bidir_x2(x2, dt, A, B, C, D)
    return gated_rmsnorm(y, z, norm_w, eps)
