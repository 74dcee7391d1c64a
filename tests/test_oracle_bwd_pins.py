"""Pins of the oracle's gradients (oracle.bidir_bwd), on the CPU.

None of these checks computes its expected value with the backward code it
checks:
  * central finite differences of the forward oracle (oracle.bidir) along a
    random direction of each input, the derivative of sum(dy * y);
  * the exact adjoint identities of the maps that are linear: y is linear in
    x, and (with the other inputs fixed) in B, in C and in D, so for any v
    <dy, y(v) - y(0)> = <grad, v> up to rounding;
  * the closed form of a memoryless scan (A -> -inf, exp underflows to 0 in
    fp64): y_t = (sum_d dt_d,t C_d,t . B_d,t + D_f + D_b) x_t, whose
    gradients are written out by hand below;
  * with given start states (the seeded scans, and the block step: forward
    from a prefix state, reverse from zero): central differences of
    oracle.bidir_seeded and of oracle.block_step, including along the
    states, and the adjoint identity of the states (y is affine in them).
A planted mistake in the backward code must fail at least one of them
(test_bwd_pins_catch_planted_mistake).
"""
import ctypes
import subprocess

import numpy as np
import pytest

import oracle

NAMES = ("x", "dt", "A", "B", "C", "D")


def _problem(seed=0, batch=2, L=7, H=4, P=3, N=5, G=2):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((batch, L, H, P)),
                dt=rng.uniform(0.02, 0.3, (2, batch, L, H)),
                A=-rng.uniform(0.5, 4.0, (2, H)),
                B=rng.standard_normal((2, batch, L, G, N)) / 3,
                C=rng.standard_normal((2, batch, L, G, N)) / 3,
                D=rng.standard_normal((2, H))), rng.standard_normal((batch, L, H, P))


def _loss(inp, dy):
    return float(np.sum(dy * oracle.bidir(*(inp[k] for k in NAMES))))


@pytest.mark.parametrize("name", NAMES)
def test_bwd_matches_central_differences(name):
    inp, dy = _problem(seed=1)
    g = oracle.bidir_bwd(*(inp[k] for k in NAMES), dy)
    rng = np.random.default_rng(2)
    v = rng.standard_normal(inp[name].shape)
    eps = 1e-6 * max(1.0, float(np.max(np.abs(inp[name]))))
    plus, minus = dict(inp), dict(inp)
    plus[name] = inp[name] + eps * v
    minus[name] = inp[name] - eps * v
    fd = (_loss(plus, dy) - _loss(minus, dy)) / (2 * eps)
    an = float(np.sum(g["d" + name] * v))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"d{name}: finite difference {fd} vs adjoint {an}"


def _linear_part(inp, name, v):
    """y with input `name` set to v, minus y with it set to zero."""
    a, z = dict(inp), dict(inp)
    a[name] = v
    z[name] = np.zeros_like(v)
    return oracle.bidir(*(a[k] for k in NAMES)) - oracle.bidir(*(z[k] for k in NAMES))


@pytest.mark.parametrize("name", ["x", "B", "C", "D"])
def test_bwd_adjoint_identity_of_linear_inputs(name):
    inp, dy = _problem(seed=3, batch=1, L=9, H=2, P=4, N=3, G=1)
    g = oracle.bidir_bwd(*(inp[k] for k in NAMES), dy)
    v = np.random.default_rng(4).standard_normal(inp[name].shape)
    if name in ("B", "C"):
        # y is linear in B (C) for fixed C (B): the gradient at v is that of the map
        at_v = dict(inp)
        at_v[name] = v
        g = oracle.bidir_bwd(*(at_v[k] for k in NAMES), dy)
    lhs = float(np.sum(dy * _linear_part(inp, name, v)))
    rhs = float(np.sum(g["d" + name] * v))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), f"{name}: <dy, y(v)> {lhs} vs <grad, v> {rhs}"


def test_bwd_memoryless_closed_form():
    inp, dy = _problem(seed=5, batch=2, L=6, H=4, P=3, N=5, G=2)
    inp["A"] = np.full((2, 4), -1e6)          # exp(dt A) == 0 exactly in fp64
    g = oracle.bidir_bwd(*(inp[k] for k in NAMES), dy)
    x, dt, B, C, D = inp["x"], inp["dt"], inp["B"], inp["C"], inp["D"]
    batch, L, H, P = x.shape
    G = B.shape[3]
    hpg = H // G
    dx = np.zeros_like(x)
    ddt = np.zeros_like(dt)
    dB = np.zeros_like(B)
    dC = np.zeros_like(C)
    for b in range(batch):
        for t in range(L):
            for h in range(H):
                gg = h // hpg
                xdy = float(np.dot(x[b, t, h], dy[b, t, h]))
                s = D[0, h] + D[1, h]
                for d in range(2):
                    cb = float(np.dot(C[d, b, t, gg], B[d, b, t, gg]))
                    s += dt[d, b, t, h] * cb
                    ddt[d, b, t, h] = cb * xdy
                    dB[d, b, t, gg] += dt[d, b, t, h] * C[d, b, t, gg] * xdy
                    dC[d, b, t, gg] += dt[d, b, t, h] * B[d, b, t, gg] * xdy
                dx[b, t, h] = s * dy[b, t, h]
    dD = np.einsum("bthp,bthp->h", x, dy)
    for k, want in (("dx", dx), ("ddt", ddt), ("dB", dB), ("dC", dC)):
        assert np.allclose(g[k], want, rtol=1e-12, atol=1e-12), k
    assert np.allclose(g["dD"], np.stack([dD, dD]), rtol=1e-12)
    assert np.all(g["dA"] == 0.0)


def _seeded(seed=3, batch=2, L=6, H=4, P=3, N=5, G=2):
    inp, dy = _problem(seed, batch, L, H, P, N, G)
    rng = np.random.default_rng(seed + 100)
    inp["prefix"] = rng.standard_normal((batch, H, P, N))
    inp["suffix"] = rng.standard_normal((batch, H, P, N))
    return inp, dy


def _seeded_loss(inp, dy):
    return float(np.sum(dy * oracle.bidir_seeded(*(inp[k] for k in NAMES), prefix=inp["prefix"],
                                                  suffix=inp["suffix"])))


@pytest.mark.parametrize("name", NAMES + ("prefix", "suffix"))
def test_seeded_bwd_matches_central_differences(name):
    inp, dy = _seeded()
    g = oracle.bidir_bwd(*(inp[k] for k in NAMES), dy, prefix=inp["prefix"], suffix=inp["suffix"])
    v = np.random.default_rng(4).standard_normal(inp[name].shape)
    eps = 1e-6 * max(1.0, float(np.max(np.abs(inp[name]))))
    plus, minus = dict(inp), dict(inp)
    plus[name] = inp[name] + eps * v
    minus[name] = inp[name] - eps * v
    fd = (_seeded_loss(plus, dy) - _seeded_loss(minus, dy)) / (2 * eps)
    an = float(np.sum(g["d" + name] * v))
    assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"d{name}: finite difference {fd} vs adjoint {an}"


def test_state_gradients_adjoint_identity():
    """y is affine in each start state: <dy, y(s + v) - y(s)> = <ds, v>."""
    inp, dy = _seeded(seed=5)
    g = oracle.bidir_bwd(*(inp[k] for k in NAMES), dy, prefix=inp["prefix"], suffix=inp["suffix"])
    base = oracle.bidir_seeded(*(inp[k] for k in NAMES), prefix=inp["prefix"], suffix=inp["suffix"])
    rng = np.random.default_rng(6)
    for name in ("prefix", "suffix"):
        v = rng.standard_normal(inp[name].shape)
        moved = dict(inp)
        moved[name] = inp[name] + v
        y = oracle.bidir_seeded(*(moved[k] for k in NAMES), prefix=moved["prefix"], suffix=moved["suffix"])
        lhs, rhs = float(np.sum(dy * (y - base))), float(np.sum(g["d" + name] * v))
        assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)), f"d{name}: {lhs} vs {rhs}"


def test_block_step_gradients_match_central_differences():
    """The block step's gradients (prefix given, no suffix) against central
    differences of oracle.block_step, its own forward definition."""
    inp, dy = _seeded(seed=7, L=5)
    g = oracle.bidir_bwd(*(inp[k] for k in NAMES), dy, prefix=inp["prefix"])
    assert "dsuffix" not in g
    rng = np.random.default_rng(8)
    for name in ("prefix", "dt", "A", "x"):
        v = rng.standard_normal(inp[name].shape)
        eps = 1e-6 * max(1.0, float(np.max(np.abs(inp[name]))))
        f = lambda d: float(np.sum(dy * oracle.block_step(*((inp[k] + d * v) if k == name else inp[k]
                                                             for k in NAMES),
                                                           (inp["prefix"] + d * v) if name == "prefix"
                                                           else inp["prefix"])))
        fd = (f(eps) - f(-eps)) / (2 * eps)
        an = float(np.sum(g["d" + name] * v))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"block step d{name}: {fd} vs {an}"


# (name, text in ssd_oracle.c's backward code, replacement): plausible mistakes
BWD_MUTANTS = [
    ("ddt_without_decay_term", "ddtu[(ptrdiff_t)t * dt_ts] = gbx + Ad * a * ghp;", "ddtu[(ptrdiff_t)t * dt_ts] = gbx;"),
    ("dA_without_dt", "dA_acc += dtt * a * ghp;", "dA_acc += a * ghp;"),
    ("adjoint_decayed_before_input", "for (size_t q = 0; q < SN; ++q) gadj[q] *= a;   /* adjoint of h_{t-1}'s share */",
     "for (size_t q = 0; q < SN; ++q) gadj[q] *= 1.0;"),
    ("dx_without_skip", "dxu[(ptrdiff_t)t * x_ts + p] += dsum * dyu[(ptrdiff_t)t * x_ts + p];", "(void)dsum;"),
    ("dB_without_dt", "dBu[(ptrdiff_t)t * bc_ts + n] += dtt * s;", "dBu[(ptrdiff_t)t * bc_ts + n] += s;"),
    ("dC_from_previous_state", "s += ht[(size_t)n * P + p] * dyt[p];", "s += hp[(size_t)n * P + p] * dyt[p];"),
    ("reverse_adjoint_walks_forward", "const int t = d ? (L - 1 - k) : k;\n                    const double dtt = dtu[(ptrdiff_t)t * dt_ts];\n                    const double a = exp(dtt * Ad);\n                    const double *Bt = Bu + (ptrdiff_t)t * bc_ts;\n                    const double *Ct",
     "const int t = k;\n                    const double dtt = dtu[(ptrdiff_t)t * dt_ts];\n                    const double a = exp(dtt * Ad);\n                    const double *Bt = Bu + (ptrdiff_t)t * bc_ts;\n                    const double *Ct"),
    ("start_state_adjoint_without_first_decay",
     "du[(size_t)p * N + n] = L > 0 ? gadj[(size_t)n * P + p] : 0.0;",
     "du[(size_t)p * N + n] = L > 0 ? gadj[(size_t)n * P + p] / exp(dtu[(ptrdiff_t)(d ? L - 1 : 0) * dt_ts] * Ad) : 0.0;"),
    ("start_state_not_transposed", "hs[(size_t)n * P + p] = iu[(size_t)p * N + n];",
     "hs[(size_t)n * P + p] = iu[(size_t)n * P + p];"),
    ("start_state_ignored_in_scan", "for (int p = 0; p < P; ++p) hs[(size_t)n * P + p] = iu[(size_t)p * N + n];",
     "for (int p = 0; p < P; ++p) hs[(size_t)n * P + p] = 0.0 * iu[(size_t)p * N + n];"),
]

BWD_PINS = [
    lambda: [test_bwd_matches_central_differences(n) for n in NAMES],
    lambda: [test_bwd_adjoint_identity_of_linear_inputs(n) for n in ("x", "B", "C", "D")],
    test_bwd_memoryless_closed_form,
    lambda: [test_seeded_bwd_matches_central_differences(n) for n in NAMES + ("prefix", "suffix")],
    test_state_gradients_adjoint_identity,
    test_block_step_gradients_match_central_differences,
]


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_bwd_pins_catch_planted_mistake(tmp_path, monkeypatch, name, old, new):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {name}"
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(src.replace(old, new))
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(c), "-o", str(so), "-lm"],
                   check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(str(so))))
    failed = 0
    for pin in BWD_PINS:
        try:
            pin()
        except (AssertionError, ValueError):
            failed += 1
    assert failed, f"no pin caught mutant {name}"
