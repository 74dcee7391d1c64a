"""Pins of the oracle's mixer-block steps (conv1d + SiLU per direction, the
mixer with per-direction x, the gated RMS norm), on the CPU. None of these
checks computes its expected value with the code it checks:
  * conv: a delta kernel is the identity, a one-hot tap is a shifted copy with
    zeros outside the sequence, a constant input gives the sum of the taps
    plus the bias, and the reverse conv is the forward conv of the flipped
    sequence, flipped back;
  * the mixer with per-direction x against the materialised quadratic form,
    written out here with each direction reading its own x, and against the
    shared-x mixer when both x are equal;
  * the norm: unit RMS with unit weights, invariance to a positive scale, a
    hand-worked two-channel case.
"""
import math

import numpy as np

import oracle


def _silu(v):
    return v / (1.0 + np.exp(-v))


def test_conv_delta_kernel_is_identity():
    rng = np.random.default_rng(0)
    xbc = rng.standard_normal((2, 11, 7))
    w = np.zeros((2, 7, 4))
    w[:, :, 3] = 1.0                      # the tap on the current token, both directions
    out = oracle.conv_silu(xbc, w, np.zeros((2, 7)))
    assert np.array_equal(out[0], _silu(xbc)) and np.array_equal(out[1], _silu(xbc))


def test_conv_one_hot_tap_is_a_shift():
    rng = np.random.default_rng(1)
    xbc = rng.standard_normal((1, 9, 3))
    for k in range(4):
        w = np.zeros((2, 3, 4))
        w[:, :, k] = 1.0
        out = oracle.conv_silu(xbc, w, np.zeros((2, 3)))
        lag = 3 - k                        # forward reads token t - lag, reverse t + lag
        fwd = np.zeros_like(xbc)
        rev = np.zeros_like(xbc)
        fwd[:, lag:] = xbc[:, :9 - lag]
        rev[:, :9 - lag] = xbc[:, lag:]
        assert np.allclose(out[0], _silu(fwd), atol=0, rtol=1e-15)
        assert np.allclose(out[1], _silu(rev), atol=0, rtol=1e-15)


def test_conv_constant_input_is_sum_of_taps():
    rng = np.random.default_rng(2)
    w = rng.standard_normal((2, 5, 4))
    bias = rng.standard_normal((2, 5))
    xbc = np.full((1, 10, 5), 0.7)
    out = oracle.conv_silu(xbc, w, bias)
    for d, inner in ((0, slice(3, 10)), (1, slice(0, 7))):   # tokens whose window lies inside
        pre = 0.7 * w[d].sum(axis=1) + bias[d]
        assert np.allclose(out[d, 0, inner], _silu(pre)[None, :], rtol=1e-14, atol=0)
    # at the sequence ends only the taps inside the sequence count
    pre0 = 0.7 * w[0][:, 3] + bias[0]
    assert np.allclose(out[0, 0, 0], _silu(pre0), rtol=1e-14)
    pre9 = 0.7 * w[1][:, 3] + bias[1]
    assert np.allclose(out[1, 0, 9], _silu(pre9), rtol=1e-14)


def test_conv_reverse_is_flipped_forward():
    rng = np.random.default_rng(3)
    xbc = rng.standard_normal((2, 12, 6))
    w = rng.standard_normal((2, 6, 4))
    bias = rng.standard_normal((2, 6))
    out = oracle.conv_silu(xbc, w, bias)
    # the reverse direction's weights used as a forward conv on the flipped sequence
    flipped = oracle.conv_silu(xbc[:, ::-1], np.stack([w[1], w[1]]), np.stack([bias[1], bias[1]]))[0][:, ::-1]
    assert np.allclose(out[1], flipped, rtol=1e-14, atol=1e-15)


def _quadratic_x2(x2, dt, A, B, C, D):
    """sum_d (Lmask_d o C_d B_d^T)(dt_d x_d) + D_d x_d, entry by entry."""
    _, batch, L, H, P = x2.shape
    G = B.shape[3]
    y = np.zeros((batch, L, H, P))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            for t in range(L):
                acc = D[0, h] * x2[0, b, t, h] + D[1, h] * x2[1, b, t, h]
                for s in range(L):
                    if s <= t:
                        w = (math.exp(A[0, h] * dt[0, b, s + 1:t + 1, h].sum())
                             * np.dot(C[0, b, t, g], B[0, b, s, g]) * dt[0, b, s, h])
                        acc = acc + w * x2[0, b, s, h]
                    if s >= t:
                        w = (math.exp(A[1, h] * dt[1, b, t:s, h].sum())
                             * np.dot(C[1, b, t, g], B[1, b, s, g]) * dt[1, b, s, h])
                        acc = acc + w * x2[1, b, s, h]
                y[b, t, h] = acc
    return y


def test_mixer_with_two_x_matches_quadratic_form():
    rng = np.random.default_rng(4)
    batch, L, H, P, N, G = 2, 9, 4, 3, 5, 2
    x2 = rng.standard_normal((2, batch, L, H, P))
    dt = rng.uniform(0.05, 0.6, (2, batch, L, H))
    A = -rng.uniform(0.2, 2.0, (2, H))
    B = rng.standard_normal((2, batch, L, G, N))
    C = rng.standard_normal((2, batch, L, G, N))
    D = rng.standard_normal((2, H))
    y = oracle.bidir_x2(x2, dt, A, B, C, D)
    q = _quadratic_x2(x2, dt, A, B, C, D)
    assert np.max(np.abs(y - q)) <= 1e-12 * np.max(np.abs(q))
    # equal x in both directions: the shared-x mixer
    same = np.stack([x2[0], x2[0]])
    assert np.allclose(oracle.bidir_x2(same, dt, A, B, C, D), oracle.bidir(x2[0], dt, A, B, C, D), rtol=1e-13,
                       atol=1e-13)


def test_gated_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((2, 5, 3, 4))
    z = rng.standard_normal((2, 5, 3, 4))
    out = oracle.gated_rmsnorm(y, z, np.ones(12), eps=0.0)
    assert np.allclose(np.mean(out.reshape(2, 5, 12) ** 2, axis=-1), 1.0, rtol=1e-13)
    assert np.allclose(oracle.gated_rmsnorm(3.5 * y, z, np.ones(12), eps=0.0), out, rtol=1e-13, atol=1e-14)
    w = rng.standard_normal(12)
    assert np.allclose(oracle.gated_rmsnorm(y, z, w, eps=0.0), out * w.reshape(3, 4), rtol=1e-13, atol=1e-14)


def test_gated_rmsnorm_two_channel_hand_worked():
    # y = (3, 4), z large enough that SiLU(z) = z to double precision, so
    # v = (3z, 4z), mean(v^2) = 12.5 z^2 and out = (3, 4) / sqrt(12.5) * w
    y = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    z = np.full((1, 1, 1, 2), 50.0)
    out = oracle.gated_rmsnorm(y, z, np.array([2.0, -1.0]), eps=0.0).ravel()
    want = np.array([3.0 * 2.0, 4.0 * -1.0]) / math.sqrt(12.5)
    assert np.allclose(out, want, rtol=1e-12)


# plausible mistakes in the block steps: each must fail at least one pin above
def _mut_reverse_conv_causal(xbc, w, bias):
    f = _REAL["conv_silu"](xbc, np.stack([w[0], w[1]]), bias)
    g = _REAL["conv_silu"](xbc, np.stack([w[1], w[1]]), np.stack([bias[1], bias[1]]))
    return np.stack([f[0], g[0]])        # reverse computed causally


def _mut_conv_no_bias(xbc, w, bias):
    return _REAL["conv_silu"](xbc, w, np.zeros_like(np.asarray(bias, dtype=np.float64)))


def _mut_conv_no_silu(xbc, w, bias):
    return _pre_activation(xbc, w, bias)


def _pre_activation(xbc, w, bias):
    batch, L, cin = np.asarray(xbc).shape
    K = np.asarray(w).shape[2]
    out = np.zeros((2, batch, L, cin))
    for t in range(L):
        for k in range(K):
            s, r = t - (K - 1) + k, t + (K - 1) - k
            if 0 <= s < L:
                out[0, :, t] += w[0][:, k] * xbc[:, s]
            if 0 <= r < L:
                out[1, :, t] += w[1][:, k] * xbc[:, r]
    return out + np.asarray(bias)[:, None, None, :]


def _mut_x2_shared_x(x2, dt, A, B, C, D, nthreads=0):
    return _REAL["bidir"](x2[0], dt, A, B, C, D)


def _mut_x2_one_d(x2, dt, A, B, C, D, nthreads=0):
    D1 = np.asarray(D, dtype=np.float64).copy()
    D1[1] = 0.0
    return _REAL["bidir_x2"](x2, dt, A, B, C, D1)


def _mut_norm_abs(y, z, w, eps=1e-5):
    y = np.asarray(y, dtype=np.float64)
    batch, L, H, P = y.shape
    v = (y * oracle.silu(z)).reshape(batch, L, H * P)
    return (v / (np.mean(np.abs(v), axis=-1, keepdims=True) + eps) * w).reshape(batch, L, H, P)


def _mut_norm_gate_after(y, z, w, eps=1e-5):
    y = np.asarray(y, dtype=np.float64)
    batch, L, H, P = y.shape
    v = y.reshape(batch, L, H * P)
    n = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return (n * np.asarray(w) * oracle.silu(z).reshape(batch, L, H * P)).reshape(batch, L, H, P)


_REAL = {"conv_silu": oracle.conv_silu, "bidir": oracle.bidir, "bidir_x2": oracle.bidir_x2,
         "gated_rmsnorm": oracle.gated_rmsnorm}
_BLOCK_MUTANTS = [("conv_silu", _mut_reverse_conv_causal), ("conv_silu", _mut_conv_no_bias),
                  ("conv_silu", _mut_conv_no_silu), ("bidir_x2", _mut_x2_shared_x), ("bidir_x2", _mut_x2_one_d),
                  ("gated_rmsnorm", _mut_norm_abs), ("gated_rmsnorm", _mut_norm_gate_after)]
_BLOCK_PINS = [test_conv_delta_kernel_is_identity, test_conv_one_hot_tap_is_a_shift,
               test_conv_constant_input_is_sum_of_taps, test_conv_reverse_is_flipped_forward,
               test_mixer_with_two_x_matches_quadratic_form, test_gated_rmsnorm_unit_rms_and_scale_invariance,
               test_gated_rmsnorm_two_channel_hand_worked]


def test_block_pins_catch_planted_mistakes(monkeypatch):
    for name, fn in _BLOCK_MUTANTS:
        with monkeypatch.context() as m:
            m.setattr(oracle, name, fn)
            failed = 0
            for pin in _BLOCK_PINS:
                try:
                    pin()
                except (AssertionError, ValueError):
                    failed += 1
            assert failed, f"no pin caught {fn.__name__}"
