"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each expected value here comes from a different computation than the oracle's
sequential loop: the materialised quadratic (attention-like) form of the scan,
closed forms of special cases, identities the method fixes, and a hand-worked
example. The definitions pinned:
  - forward + reverse Mamba-2 scans, added ("DiffuMamba: High-Throughput
    Diffusion LMs with Mamba Backbone", Technical Summary, 2. Methodology,
    Core Architecture);
  - the reverse scan is Mamba-2 on the flipped sequence ("DiffMamba -
    Checkpoints" model card, Model details);
  - the forward state of a prefix is exact and reusable, the reverse scan is
    confined to the active block ("Training Hybrid Block Diffusion Language
    Models with Partial Bidirectionality", Abstract, Methodology).
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(rng, batch=2, L=13, H=4, P=3, N=5, G=2, a_scale=1.0):
    x = rng.standard_normal((batch, L, H, P))
    dt = rng.uniform(0.05, 0.6, size=(2, batch, L, H))
    A = -rng.uniform(0.2, 2.0, size=(2, H)) * a_scale
    B = rng.standard_normal((2, batch, L, G, N))
    C = rng.standard_normal((2, batch, L, G, N))
    D = rng.standard_normal((2, H))
    return x, dt, A, B, C, D


def quadratic_form(x, dt, A, B, C, D):
    """y = sum_d (Lmask_d o C_d B_d^T)(dt_d x) + (D_f + D_b) x, built entry by entry.

    Lmask_f[t,s] = exp(A_f * sum_{r=s+1..t} dt_f[r]) for s <= t, else 0;
    Lmask_b[t,s] = exp(A_b * sum_{r=t..s-1} dt_b[r]) for s >= t, else 0.
    """
    batch, L, H, P = x.shape
    G = B.shape[3]
    y = np.zeros_like(x)
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            for t in range(L):
                acc = np.zeros(P)
                for s in range(L):
                    if s <= t:  # forward
                        seg = dt[0, b, s + 1:t + 1, h].sum()
                        w = math.exp(A[0, h] * seg) * np.dot(C[0, b, t, g], B[0, b, s, g]) * dt[0, b, s, h]
                        acc += w * x[b, s, h]
                    if s >= t:  # reverse
                        seg = dt[1, b, t:s, h].sum()
                        w = math.exp(A[1, h] * seg) * np.dot(C[1, b, t, g], B[1, b, s, g]) * dt[1, b, s, h]
                        acc += w * x[b, s, h]
                y[b, t, h] = acc + (D[0, h] + D[1, h]) * x[b, t, h]
    return y


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


def test_matches_quadratic_form():
    rng = np.random.default_rng(1)
    prob = rand_problem(rng)
    y = oracle.bidir(*prob)
    assert rel(y, quadratic_form(*prob)) < 1e-12


def test_quadratic_form_groups_and_shapes():
    # H/G = 3 heads per group, P != N, odd sizes: a wrong group index or a
    # transposed B/C/x operand cannot agree here.
    rng = np.random.default_rng(2)
    prob = rand_problem(rng, batch=1, L=9, H=6, P=2, N=7, G=2)
    assert rel(oracle.bidir(*prob), quadratic_form(*prob)) < 1e-12


def test_golden_hand_worked():
    vals = {}
    with open(os.path.join(GOLDEN, "hand_worked_L3.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, *v = line.split()
                vals[k] = np.array([float(t) for t in v])
    L = 3
    x = vals["x"].reshape(1, L, 1, 1)
    dt = np.stack([vals["dt_f"], vals["dt_b"]]).reshape(2, 1, L, 1)
    A = np.array([vals["A_f"], vals["A_b"]]).reshape(2, 1)
    B = np.stack([vals["B_f"], vals["B_b"]]).reshape(2, 1, L, 1, 1)
    C = np.stack([vals["C_f"], vals["C_b"]]).reshape(2, 1, L, 1, 1)
    D = np.array([vals["D_f"], vals["D_b"]]).reshape(2, 1)
    y = oracle.bidir(x, dt, A, B, C, D)
    np.testing.assert_allclose(y.reshape(L), vals["y"], rtol=1e-14, atol=1e-14)
    st = oracle.prefix_state(x, dt[0], A[0], B[0])
    np.testing.assert_allclose(st.reshape(-1), vals["state"], rtol=1e-14)


def test_flip_identity():
    """bidir(x; f, b) = fwd(x; f) + flip(fwd(flip x; flipped b))."""
    rng = np.random.default_rng(3)
    x, dt, A, B, C, D = rand_problem(rng, batch=2, L=21)
    y = oracle.bidir(x, dt, A, B, C, D)
    # forward direction alone: silence the reverse direction's output and D.
    Cz, Dz = C.copy(), D.copy()
    Cz[1] = 0.0
    Dz[1] = 0.0
    y_f = oracle.bidir(x, dt, A, B, Cz, Dz)
    # reverse direction as a forward scan over the flipped sequence.
    fl = lambda a, ax: np.flip(a, axis=ax).copy()
    dt2 = np.stack([fl(dt[1], 1), np.zeros_like(dt[1])])
    B2 = np.stack([fl(B[1], 1), np.zeros_like(B[1])])
    C2 = np.stack([fl(C[1], 1), np.zeros_like(C[1])])
    A2 = np.stack([A[1], A[1]])
    D2 = np.stack([D[1], np.zeros_like(D[1])])
    y_b = fl(oracle.bidir(fl(x, 1), dt2, A2, B2, C2, D2), 1)
    assert rel(y, y_f + y_b) < 1e-13


def test_closed_form_A_to_minus_infinity():
    """exp(dt*A) underflows to 0: each token only sees itself."""
    rng = np.random.default_rng(4)
    x, dt, A, B, C, D = rand_problem(rng, L=11)
    A = np.full_like(A, -1e6)
    y = oracle.bidir(x, dt, A, B, C, D)
    H, G = x.shape[2], B.shape[3]
    gidx = np.arange(H) // (H // G)
    cb_f = np.einsum("blhn,blhn->blh", C[0][:, :, gidx], B[0][:, :, gidx])
    cb_b = np.einsum("blhn,blhn->blh", C[1][:, :, gidx], B[1][:, :, gidx])
    coef = dt[0] * cb_f + dt[1] * cb_b + (D[0] + D[1])[None, None, :]
    assert rel(y, coef[..., None] * x) < 1e-13


def test_single_token():
    rng = np.random.default_rng(5)
    x, dt, A, B, C, D = rand_problem(rng, L=1)
    y = oracle.bidir(x, dt, A, B, C, D)
    H, G = x.shape[2], B.shape[3]
    gidx = np.arange(H) // (H // G)
    coef = sum(dt[d] * np.einsum("blhn,blhn->blh", C[d][:, :, gidx], B[d][:, :, gidx]) for d in range(2))
    coef = coef + (D[0] + D[1])[None, None, :]
    assert rel(y, coef[..., None] * x) < 1e-14


def test_closed_form_A_zero_is_cumulative_linear_attention():
    """A = 0: forward = causal prefix sums of dt_s B_s x_s^T read by C_t; reverse = suffix sums."""
    rng = np.random.default_rng(6)
    x, dt, A, B, C, D = rand_problem(rng, L=17)
    A = np.zeros_like(A)
    y = oracle.bidir(x, dt, A, B, C, D)
    H, G = x.shape[2], B.shape[3]
    gidx = np.arange(H) // (H // G)
    Bh = [B[d][:, :, gidx] for d in range(2)]  # (b, L, H, N)
    Ch = [C[d][:, :, gidx] for d in range(2)]
    outer_f = dt[0][..., None, None] * Bh[0][..., :, None] * x[..., None, :]  # (b,L,H,N,P)
    outer_b = dt[1][..., None, None] * Bh[1][..., :, None] * x[..., None, :]
    S_f = np.cumsum(outer_f, axis=1)
    S_b = np.flip(np.cumsum(np.flip(outer_b, 1), axis=1), 1)
    ref = (np.einsum("blhn,blhnp->blhp", Ch[0], S_f) + np.einsum("blhn,blhnp->blhp", Ch[1], S_b)
           + (D[0] + D[1])[None, None, :, None] * x)
    assert rel(y, ref) < 1e-12


def test_geometric_series_constant_input():
    """Scalar state, constant dt, A, B, C and x = 1: h_t is a geometric sum."""
    L, dtv, Av, bv, cv = 40, 0.3, -0.7, 1.3, -0.4
    a = math.exp(dtv * Av)
    x = np.ones((1, L, 1, 1))
    dt = np.full((2, 1, L, 1), dtv)
    A = np.full((2, 1), Av)
    B = np.full((2, 1, L, 1, 1), bv)
    C = np.full((2, 1, L, 1, 1), cv)
    D = np.zeros((2, 1))
    y = oracle.bidir(x, dt, A, B, C, D).reshape(L)
    t = np.arange(L)
    fwd = cv * dtv * bv * (1 - a ** (t + 1)) / (1 - a)
    rev = cv * dtv * bv * (1 - a ** (L - t)) / (1 - a)
    np.testing.assert_allclose(y, fwd + rev, rtol=1e-13)
    st = oracle.prefix_state(x, dt[0], A[0], B[0]).reshape(())
    np.testing.assert_allclose(st, dtv * bv * (1 - a ** L) / (1 - a), rtol=1e-13)


def test_linearity_in_x():
    rng = np.random.default_rng(7)
    x1, dt, A, B, C, D = rand_problem(rng, L=15)
    x2 = rng.standard_normal(x1.shape)
    y = oracle.bidir(2.5 * x1 - 0.75 * x2, dt, A, B, C, D)
    y12 = 2.5 * oracle.bidir(x1, dt, A, B, C, D) - 0.75 * oracle.bidir(x2, dt, A, B, C, D)
    assert rel(y, y12) < 1e-13


def test_prefix_state_closed_form():
    """h_L[p, n] = sum_s exp(A sum_{r=s+1..L-1} dt_r) dt_s B_s[n] x_s[p], stored (P, N)."""
    rng = np.random.default_rng(8)
    x, dt, A, B, C, D = rand_problem(rng, batch=2, L=12, H=4, P=3, N=5, G=2)
    st = oracle.prefix_state(x, dt[0], A[0], B[0])
    batch, L, H, P = x.shape
    N = B.shape[-1]
    ref = np.zeros((batch, H, P, N))
    for b in range(batch):
        for h in range(H):
            g = h // 2
            for s in range(L):
                w = math.exp(A[0, h] * dt[0, b, s + 1:, h].sum()) * dt[0, b, s, h]
                ref[b, h] += w * np.outer(x[b, s, h], B[0, b, s, g])
    assert rel(st, ref) < 1e-13


def test_prefix_state_composes():
    """state(prefix ++ block) = prefix_state(block, init = state(prefix))."""
    rng = np.random.default_rng(9)
    x, dt, A, B, C, D = rand_problem(rng, batch=2, L=30)
    k = 19
    full = oracle.prefix_state(x, dt[0], A[0], B[0])
    pre = oracle.prefix_state(x[:, :k], dt[0][:, :k], A[0], B[0][:, :k])
    cont = oracle.prefix_state(x[:, k:], dt[0][:, k:], A[0], B[0][:, k:], init=pre)
    assert rel(cont, full) < 1e-13


def test_block_step_equals_split_scans():
    """Forward part of a block step = last T forward outputs over prefix ++ block;
    reverse part = the reverse scan over the block alone (confined to the block)."""
    rng = np.random.default_rng(10)
    x, dt, A, B, C, D = rand_problem(rng, batch=2, L=26)
    k = 18
    T = x.shape[1] - k
    pre = oracle.prefix_state(x[:, :k], dt[0][:, :k], A[0], B[0][:, :k])
    xb = x[:, k:]
    dtb, Bb, Cb = dt[:, :, k:], B[:, :, k:], C[:, :, k:]
    y_step = oracle.block_step(xb, dtb, A, Bb, Cb, D, pre)
    # forward over the whole sequence (reverse silenced), last T tokens
    Cf, Df = C.copy(), D.copy()
    Cf[1] = 0.0
    Df[:] = 0.0
    y_fwd = oracle.bidir(x, dt, A, B, Cf, Df)[:, k:]
    # reverse over the block alone (forward silenced), plus both D terms
    Cr = Cb.copy()
    Cr[0] = 0.0
    y_rev = oracle.bidir(xb, dtb, A, Bb, Cr, D)
    assert rel(y_step, y_fwd + y_rev) < 1e-12
    assert T == 8


def test_block_step_depends_on_prefix_only_through_state():
    """A prefix whose state is wiped (decay exactly 0) by a token with x = 0 and a
    huge dt leaves the same state as the shorter prefix behind it."""
    rng = np.random.default_rng(11)
    x, dt, A, B, C, D = rand_problem(rng, batch=1, L=20)
    k = 12
    junk = 5
    xj = np.concatenate([rng.standard_normal((1, junk, 4, 3)), np.zeros((1, 1, 4, 3)), x[:, :k]], 1)
    dtj = np.concatenate([rng.uniform(0.1, 0.5, (1, junk, 4)), np.full((1, 1, 4), 1e6), dt[0][:, :k]], 1)
    Bj = np.concatenate([rng.standard_normal((1, junk, 2, 5)), np.ones((1, 1, 2, 5)), B[0][:, :k]], 1)
    s1 = oracle.prefix_state(x[:, :k], dt[0][:, :k], A[0], B[0][:, :k])
    s2 = oracle.prefix_state(xj, dtj, A[0], Bj)
    assert np.array_equal(s1, s2)
    args = (x[:, k:], dt[:, :, k:], A, B[:, :, k:], C[:, :, k:], D)
    assert np.array_equal(oracle.block_step(*args, s1), oracle.block_step(*args, s2))


def test_bidir_seeded_with_zero_states_is_the_plain_mixer():
    rng = np.random.default_rng(21)
    x, dt, A, B, C, D = rand_problem(rng, batch=2, L=17)
    y0 = oracle.bidir_seeded(x, dt, A, B, C, D)
    assert np.array_equal(y0, oracle.block_step(x, dt, A, B, C, D, None))
    assert rel(y0, oracle.bidir(x, dt, A, B, C, D)) < 1e-14


def _reverse_state_after(x, dt, A, B, k):
    """The reverse state entering token k - 1 from the right: the reverse scan
    over tokens k..L-1, written as a forward prefix state of the flipped tail
    (the flip identity), with the reverse direction's parameters."""
    fl = lambda a: np.flip(a, axis=1).copy()
    return oracle.prefix_state(fl(x[:, k:]), fl(dt[1][:, k:]), A[1], fl(B[1][:, k:]))


def test_bidir_seeded_segments_rebuild_the_whole_sequence():
    """A sequence cut into segments, each seeded with the forward state the
    tokens before it leave and the reverse state the tokens after it leave,
    gives the whole-sequence mixer, segment by segment."""
    rng = np.random.default_rng(22)
    x, dt, A, B, C, D = rand_problem(rng, batch=2, L=29)
    full = oracle.bidir(x, dt, A, B, C, D)
    cuts = [0, 9, 20, 29]
    parts = []
    for k0, k1 in zip(cuts[:-1], cuts[1:]):
        pre = oracle.prefix_state(x[:, :k0], dt[0][:, :k0], A[0], B[0][:, :k0]) if k0 > 0 else None
        suf = _reverse_state_after(x, dt, A, B, k1) if k1 < x.shape[1] else None
        parts.append(oracle.bidir_seeded(x[:, k0:k1], dt[:, :, k0:k1], A, B[:, :, k0:k1], C[:, :, k0:k1], D,
                                         pre, suf))
    assert rel(np.concatenate(parts, axis=1), full) < 1e-12


def test_bidir_seeded_reverse_start_mirrors_forward_start():
    """Seeding the reverse scan at the right end is seeding the forward scan of
    the flipped sequence with the directions swapped."""
    rng = np.random.default_rng(23)
    x, dt, A, B, C, D = rand_problem(rng, batch=1, L=11)
    s = rng.standard_normal((1, 4, 3, 5))
    y = oracle.bidir_seeded(x, dt, A, B, C, D, None, s)
    sw = lambda a: np.flip(a[::-1], axis=2).copy()   # swap directions, flip tokens
    y2 = oracle.bidir_seeded(np.flip(x, 1).copy(), sw(dt), A[::-1].copy(), sw(B), sw(C), D[::-1].copy(), s, None)
    assert rel(y, np.flip(y2, 1)) < 1e-13


def test_dt_prep_closed_forms():
    """softplus(0) = ln 2; softplus(u) - softplus(-u) = u; softplus(u) -> u for
    large u and -> e^u for very negative u; the clamp is applied after."""
    z = np.zeros((2, 1, 3, 2))
    assert np.allclose(oracle.dt_prep(z, np.zeros((2, 2))), math.log(2.0), rtol=0, atol=1e-15)
    u = np.linspace(-30, 30, 61).reshape(1, 1, 61, 1).repeat(2, axis=0)
    b = np.zeros((2, 1))
    assert np.allclose(oracle.dt_prep(u, b) - oracle.dt_prep(-u, b), u, rtol=0, atol=1e-12)
    assert abs(oracle.dt_prep(np.full((2, 1, 1, 1), 40.0), b)[0, 0, 0, 0] - 40.0) < 1e-15
    assert abs(oracle.dt_prep(np.full((2, 1, 1, 1), -40.0), b)[0, 0, 0, 0] / math.exp(-40.0) - 1) < 1e-15
    # the bias is per direction and head, added before the softplus
    bias = np.array([[0.5, -1.0], [2.0, 0.0]])
    got = oracle.dt_prep(np.zeros((2, 1, 1, 2)), bias)
    want = np.log1p(np.exp(bias))[:, None, None, :]
    assert np.allclose(got, want, rtol=1e-15, atol=0)
    clamped = oracle.dt_prep(np.full((2, 1, 2, 2), -10.0), np.zeros((2, 2)), dt_min=1e-3, dt_max=0.1)
    assert np.all(clamped == 1e-3)
    clamped = oracle.dt_prep(np.full((2, 1, 2, 2), 10.0), np.zeros((2, 2)), dt_min=1e-3, dt_max=0.1)
    assert np.all(clamped == 0.1)


def test_units_subset_matches_full():
    rng = np.random.default_rng(12)
    prob = rand_problem(rng, batch=3, L=10, H=4)
    full = oracle.bidir(*prob)
    units = [(0, 3), (2, 1), (1, 0)]
    part = oracle.bidir(*prob, units=units)
    for b, h in units:
        assert np.array_equal(part[b, :, h], full[b, :, h])
    assert np.isnan(part[0, :, 0]).all()


def test_threads_do_not_change_results():
    rng = np.random.default_rng(13)
    prob = rand_problem(rng, batch=3, L=25, H=4)
    assert np.array_equal(oracle.bidir(*prob, nthreads=1), oracle.bidir(*prob, nthreads=4))
