"""The oracle's pins are strong enough: plant a plausible mistake in a copy of
the oracle's C source, rebuild it, and check that at least one pin fails.

Mistakes are planted on the CPU only, in a temporary copy; the real oracle is
never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

PIN_CHECKS = [
    pins.test_matches_quadratic_form,
    pins.test_quadratic_form_groups_and_shapes,
    pins.test_golden_hand_worked,
    pins.test_flip_identity,
    pins.test_closed_form_A_to_minus_infinity,
    pins.test_closed_form_A_zero_is_cumulative_linear_attention,
    pins.test_geometric_series_constant_input,
    pins.test_prefix_state_closed_form,
    pins.test_prefix_state_composes,
    pins.test_block_step_equals_split_scans,
    pins.test_bidir_seeded_with_zero_states_is_the_plain_mixer,
    pins.test_bidir_seeded_segments_rebuild_the_whole_sequence,
    pins.test_bidir_seeded_reverse_start_mirrors_forward_start,
]

# (name, text in ssd_oracle.c, replacement)
MUTANTS = [
    ("decay_half", "const double decay = exp(dtt * A);", "const double decay = exp(0.5 * dtt * A);"),
    ("drop_dt_on_input", "const double bn = dtt * Bt[n];", "const double bn = Bt[n];"),
    ("decay_after_input", "hn[p] = decay * hn[p] + bn * xt[p];", "hn[p] = decay * (hn[p] + bn * xt[p]);"),
    ("reverse_walks_forward", "int t = reverse ? (L - 1 - step) : step;", "int t = step;"),
    ("D_forward_only", "const double dsum = D[hh] + D[H + hh];", "const double dsum = D[hh];"),
    ("group_index_modulo", "const int b = u / H, hh = u % H, g = hh / hpg;", "const int b = u / H, hh = u % H, g = hh % G;"),
    ("read_out_with_B", "const double *Ct = Cm + (ptrdiff_t)t * bc_ts;", "const double *Ct = Bm + (ptrdiff_t)t * bc_ts;"),
    ("state_not_transposed", "so[(size_t)p * N + n] = h[(size_t)n * P + p];", "so[(size_t)n * P + p] = h[(size_t)n * P + p];"),
    ("reverse_uses_forward_A", "A[d * H + hh], Bu, Cu", "A[hh], Bu, Cu"),
    ("block_reverse_from_prefix", "(d == 0 && prefix)", "(prefix)"),
    ("output_off_by_one_token", "double *yt = y + (size_t)t * P;", "double *yt = y + (size_t)((t + 1) % L) * P;"),
    ("seeded_reverse_start_ignored", "const double *start = d == 0 ? prefix : suffix;",
     "const double *start = d == 0 ? prefix : NULL;"),
    ("seeded_starts_swapped", "const double *start = d == 0 ? prefix : suffix;",
     "const double *start = d == 0 ? suffix : prefix;"),
]


def _build_mutant(tmp_path, old, new):
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old}"
    src = src.replace(old, new)
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(src)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", str(c), "-o", str(so), "-lm"],
                   check=True)
    return oracle.configure(ctypes.CDLL(str(so)))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, monkeypatch, name, old, new):
    lib = _build_mutant(tmp_path, old, new)
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for check in PIN_CHECKS:
        try:
            check()
        except (AssertionError, ValueError):
            failed.append(check.__name__)
    assert failed, f"no pin caught mutant {name}"


# (name, a mistaken dt_prep): the closed-form pin must reject each
def _dt_prep_mutants():
    import numpy as np

    def no_bias(dt_raw, dt_bias, dt_min=0.0, dt_max=np.inf):
        return np.clip(np.logaddexp(0.0, np.asarray(dt_raw, np.float64)), dt_min, dt_max)

    def exp_not_softplus(dt_raw, dt_bias, dt_min=0.0, dt_max=np.inf):
        u = np.asarray(dt_raw, np.float64) + np.asarray(dt_bias, np.float64)[:, None, None, :]
        return np.clip(np.exp(u), dt_min, dt_max)

    def bias_per_direction_swapped(dt_raw, dt_bias, dt_min=0.0, dt_max=np.inf):
        u = np.asarray(dt_raw, np.float64) + np.asarray(dt_bias, np.float64)[::-1, None, None, :]
        return np.clip(np.logaddexp(0.0, u), dt_min, dt_max)

    def clamp_before_softplus(dt_raw, dt_bias, dt_min=0.0, dt_max=np.inf):
        u = np.asarray(dt_raw, np.float64) + np.asarray(dt_bias, np.float64)[:, None, None, :]
        return np.logaddexp(0.0, np.clip(u, dt_min, dt_max))

    return [("no_bias", no_bias), ("exp_not_softplus", exp_not_softplus),
            ("bias_directions_swapped", bias_per_direction_swapped), ("clamp_before_softplus", clamp_before_softplus)]


@pytest.mark.parametrize("name,fn", _dt_prep_mutants(), ids=[m[0] for m in _dt_prep_mutants()])
def test_dt_prep_pin_catches_planted_mistake(monkeypatch, name, fn):
    monkeypatch.setattr(oracle, "dt_prep", fn)
    with pytest.raises(AssertionError):
        pins.test_dt_prep_closed_forms()
