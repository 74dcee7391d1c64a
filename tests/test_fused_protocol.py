"""Barrier protocol of the fused tensor-core kernel (ssd_fused.cu), checked
on the CPU.

A discrete-event model of one CTA: the TMA producer, the MMA issuer, the
state-chain group (C) and the two mask/output groups (A, B, which also prepare
the reverse pass's tiles, alternately), each taking the
same mbarrier waits and arrivals, named-barrier syncs, TMA loads, MMA commits
and TMA stores, in the same order, as the kernel. Asynchronous completions
(TMA loads, MMAs in issue order, the output store's read) land after random,
heavy-tailed delays, and runnable roles are stepped in random order.

Each schedule is checked for
  * phase overrun: a barrier completing two phases past the one a role waits
    for (the hardware parity wait would then miss both),
  * deadlock: every role blocked with nothing in flight,
  * data races: every buffer (x slots, the B/C ring, H_b, H_f, diag(w) X, the
    TMEM accumulators by 16-column block, the per-tile vectors) carries the
    version its last writer left, and each read names the version it needs.

The model must be kept in step with the kernel when its protocol changes.
A planted variant with a single diag(w) X barrier (the kernel's earlier
design, which did overrun on the GPU) must be caught.
"""
import random

from protocol_sim import Bug, Sched, run_roles


class Sim(Sched):
    """One CTA's schedule. mode: 'bidir' (both scans, output pass; the block
    step's seeded variant has the same protocol) or 'state' (the forward state
    pass alone); kxs: x slots; xw_per_slot False plants the earlier single
    diag(w) X barrier."""
    def __init__(self, nt, units, seed, kRing=4, mode='bidir', kxs=2, xw_per_slot=True, heavy=0.1, bc=None,
                 release_early=False, rzero=True):
        super().__init__(seed, heavy)
        self.nt, self.units, self.kRing = nt, units, kRing
        self.mode, self.kxs, self.xw_per_slot = mode, kxs, xw_per_slot
        self.kG1 = 8
        # bc[j]: the C/B tiles unit j reads (units of one batch element and B/C
        # group share them); one-tile units reuse the previous unit's in place
        self.bc = bc
        self.release_early = release_early   # planted: release reused slots after each unit
        # the reverse state entering the last tile is zero (no given reverse start
        # state): not stored, not loaded, no C_b H_b
        self.rzero = rzero
    def hb_zero(self, i):
        return self.rzero and i == self.nt - 1
    def bc_of(self, units_list, j):
        return self.bc[j] if self.bc is not None else units_list[j]
    def reuse(self, units_list, j):
        """unit j takes its C/B tiles from the previous unit's ring slots"""
        return (self.mode == 'bidir' and self.nt == 1 and self.bc is not None and 0 < j < len(units_list)
                and self.bc[j] == self.bc[j - 1])
    def n1t(self):
        """tiles of the state pass: all forward; in reverse all but the leftmost"""
        return self.nt if self.mode == 'state' else self.nt - 1
    def xw(self, n):
        """barrier and phase of diag(w) X for the tile with x load index n"""
        if self.xw_per_slot:
            return 'XW_READY%d' % (n % self.kxs), n // self.kxs
        return 'XW_READY', n

# ---------------------------------------------------------------- roles
# A role is a generator yielding commands:
#   ('wait', bar, k)      wait for completion of phase k (parity k & 1)
#   ('arrive', bar)
#   ('tma', bar, [(res, val)])          async load: writes then arrives
#   ('mma', [(res,val)] reads, [(res,val)] writes)   in-order async
#   ('commit', bar)                     arrives when all prior MMAs are done
#   ('read', res, val) / ('write', res, val)
#   ('sync', name, n)                   named barrier over n roles
#   ('store', [(res,val)]) then ('store_wait',)

def producer(S, units_list):
    nt, R, X = S.nt, S.kRing, S.kxs
    kr = kx = kh = 0
    units_done = 0
    for j, u in enumerate(units_list):
        for i in range(S.n1t()):                 # the state pass's tiles, in its order
            xs = kx % X
            if kx >= X:
                yield ('wait', 'X_EMPTY%d' % xs, kx // X - 1)
            kx += 1
            yield ('tma', 'X_FULL%d' % xs, [(('x', xs, 0), ('x', u, 1, i)), (('x', xs, 1), ('x', u, 1, i))])
            rs = kr % R
            if kr >= R:
                yield ('wait', 'RING_EMPTY%d' % rs, kr // R - 1)
            kr += 1
            yield ('tma', 'RING_FULL%d' % rs, [(('ring', rs), ('B1', u, i))])
        units_done += 1
        if S.mode == 'state':
            continue
        for i in range(nt):
            xs = kx % X
            if kx >= X:
                yield ('wait', 'X_EMPTY%d' % xs, kx // X - 1)
            kx += 1
            yield ('tma', 'X_FULL%d' % xs, [(('x', xs, 0), ('x', u, 2, i)), (('x', xs, 1), ('x', u, 2, i))])
            for name in ('Cf', 'Bf', 'Cb', 'Bb'):
                if S.reuse(units_list, j):
                    break
                rs = kr % R
                if kr >= R:
                    yield ('wait', 'RING_EMPTY%d' % rs, kr // R - 1)
                kr += 1
                yield ('tma', 'RING_FULL%d' % rs, [(('ring', rs), (name, S.bc_of(units_list, j), i))])
            if i == 0:
                yield ('wait', 'HB_WRITTEN', units_done - 1)
            if kh >= 1:
                yield ('wait', 'HB_EMPTY', kh - 1)
            kh += 1
            if S.hb_zero(i):
                # the reverse state entering the last tile is zero: nothing is loaded
                yield ('arrive', 'HB_FULL')
            else:
                yield ('tma_hb', 'HB_FULL', u, i)

def mma(S, units_list):
    nt, R, X = S.nt, S.kRing, S.kxs
    kr = kx = kh = n1 = 0
    n_m = n_sfree = n_yfree = n_hbw = 0
    first2 = True
    rCf = rBf = rCb = rBb = None
    for j, u in enumerate(units_list):
        bcu = S.bc_of(units_list, j)
        reuse = S.reuse(units_list, j)
        keep = S.reuse(units_list, j + 1) and not S.release_early
        for i in range(S.n1t()):
            n = kx; xs = n % X; kx += 1
            rs = kr % R
            yield ('wait', 'RING_FULL%d' % rs, kr // R); kr += 1
            yield ('wait',) + S.xw(n)
            pb = n1 % 2
            if n1 >= 2:
                yield ('wait', 'P1S_FREE%d' % pb, (n1 >> 1) - 1)
            yield ('mma', [(('ring', rs), ('B1', u, i)), (('x', xs, 0), ('xw1', u, i)), (('x', xs, 1), ('xw1', u, i))],
                   [(('tGf', b), ('S1', u, i)) for b in range(4 * pb, 4 * pb + 4)])
            yield ('commit', 'P1S_READY%d' % pb)
            yield ('commit', 'RING_EMPTY%d' % rs)
            yield ('commit', 'X_EMPTY%d' % xs)
            n1 += 1
        if S.mode == 'state':
            continue
        for i in range(nt):
            n = kx; xs = n % X; kx += 1
            if not reuse:
                slots = []
                for name in ('Cf', 'Bf', 'Cb', 'Bb'):
                    rs = kr % R
                    yield ('wait', 'RING_FULL%d' % rs, kr // R); kr += 1
                    slots.append(rs)
                rCf, rBf, rCb, rBb = slots
            if i == 0:
                yield ('wait', 'HB_WRITTEN', n_hbw); n_hbw += 1
            yield ('mma', [(('ring', rCf), ('Cf', bcu, i)), (('ring', rBf), ('Bf', bcu, i))],
                   [(('tGf', b), ('Gf', u, i)) for b in range(8)])
            yield ('mma', [(('ring', rCb), ('Cb', bcu, i)), (('ring', rBb), ('Bb', bcu, i))],
                   [(('tGb', b), ('Gb', u, i)) for b in range(8)])
            yield ('commit', 'G_READY')
            if not keep:
                yield ('commit', 'RING_EMPTY%d' % rBb)
            if not first2:
                yield ('wait', 'Y_FREE', n_yfree); n_yfree += 1
                yield ('wait', 'S_FREE', n_sfree); n_sfree += 1
            first2 = False
            yield ('mma', [(('ring', rCf), ('Cf', bcu, i)), ('hf', ('hf', u, i))], [(('Yof', 0), ('Yof', u, i)), (('Yof', 1), ('Yof', u, i))])
            if not keep:
                yield ('commit', 'RING_EMPTY%d' % rCf)
            yield ('wait', 'HB_FULL', kh); kh += 1
            if not S.hb_zero(i):   # a zero reverse state has no C_b H_b term
                yield ('mma', [(('ring', rCb), ('Cb', bcu, i)), ('hb', ('hb', u, i))], [(('Yob', 0), ('Yob', u, i)), (('Yob', 1), ('Yob', u, i))])
            if not keep:
                yield ('commit', 'RING_EMPTY%d' % rCb)
            yield ('commit', 'HB_EMPTY')
            yield ('wait',) + S.xw(n)
            yield ('mma', [(('ring', rBf), ('Bf', bcu, i)), ('xw', ('xw', u, i))], [('S', ('S', u, i))])
            yield ('commit', 'S_READY')
            if not keep:
                yield ('commit', 'RING_EMPTY%d' % rBf)
            yield ('wait', 'M_READY', n_m); n_m += 1
            yield ('wait', 'X_FULL%d' % xs, n // X)
            yield ('mma', [(('tGf', b), ('M', u, i)) for b in range(8)] + [(('x', xs, 0), ('x', u, 2, i)), (('x', xs, 1), ('x', u, 2, i))],
                   [(('Yd', 0), ('Yd', u, i)), (('Yd', 1), ('Yd', u, i))])
            yield ('commit', 'Y_READY')

def group_c(S, units_list):
    nt, X, K = S.nt, S.kxs, S.kG1
    kx = n_s = nvec = n1 = 0
    for u in units_list:
        # phase 1: the state chain only (groups A and B prepare the tiles); the
        # reverse chain stores nt states and folds all tiles but the last one
        for i in range(nt):
            if S.mode != 'state':
                if not S.hb_zero(i):   # a zero reverse state is not stored
                    yield ('write', ('hbg', u, i), ('hbg', u, i))
            if i == S.n1t():
                break
            pb = n1 % 2
            yield ('wait', 'G1_READY%d' % (n1 % K), n1 // K)
            yield ('read', ('gdec', n1 % K), ('g', u, i))
            yield ('wait', 'P1S_READY%d' % pb, n1 >> 1)
            for b in range(4 * pb, 4 * pb + 4):
                yield ('read', ('tGf', b), ('S1', u, i))
            yield ('sync', 'c', 1)
            yield ('arrive', 'P1S_FREE%d' % pb)
            n1 += 1
        if S.mode == 'state':
            continue
        kx += S.n1t()
        yield ('write', 'hf', ('hf', u, 0))
        yield ('arrive', 'HB_WRITTEN')
        for i in range(nt):
            vb = nvec % 2
            if nvec >= 2:
                yield ('wait', 'VEC_FREE%d' % vb, (nvec >> 1) - 1)
            yield ('write', ('vec', vb), ('V', u, i))
            yield ('arrive', 'VEC_READY%d' % vb)
            nvec += 1
            n = kx; xs = n % X; kx += 1
            yield ('wait', 'X_FULL%d' % xs, n // X)
            for hh in (0, 1):
                yield ('read', ('x', xs, hh), ('x', u, 2, i))
            yield ('write', 'xw', ('xw', u, i))
            yield ('arrive', S.xw(n)[0])
            yield ('wait', 'S_READY', n_s); n_s += 1
            yield ('read', 'S', ('S', u, i))
            yield ('write', 'hf', ('hf', u, i + 1))
            yield ('read', 'S', ('S', u, i))
            yield ('arrive', 'S_FREE')

def group_ab(S, units_list, is_b):
    nt, X, K = S.nt, S.kxs, S.kG1
    kx = n_g = n_y = nvec = m1 = 0
    half = 1 if is_b else 0
    blocks = range(half, 8, 2)
    for u in units_list:
        # phase 1: every other state-pass tile, by the running tile count
        for i in range(S.n1t()):
            if (m1 & 1) == half:
                xs = kx % X
                yield ('wait', 'X_FULL%d' % xs, kx // X)
                for hh in (0, 1):
                    yield ('read', ('x', xs, hh), ('x', u, 1, i))
                for hh in (0, 1):
                    yield ('write', ('x', xs, hh), ('xw1', u, i))
                yield ('write', ('gdec', m1 % K), ('g', u, i))
                yield ('sync', 'b' if is_b else 'a', 1)
                yield ('arrive', S.xw(kx)[0])
                yield ('arrive', 'G1_READY%d' % (m1 % K))
            m1 += 1
            kx += 1
        if S.mode == 'state':
            continue
        for i in range(nt):
            vb = nvec % 2
            yield ('wait', 'VEC_READY%d' % vb, nvec >> 1)
            yield ('read', ('vec', vb), ('V', u, i))
            yield ('wait', 'G_READY', n_g); n_g += 1
            for b in blocks:
                yield ('read', ('tGf', b), ('Gf', u, i))
                yield ('read', ('tGb', b), ('Gb', u, i))
            for b in blocks:
                yield ('write', ('tGf', b), ('M', u, i))
            yield ('read', ('vec', vb), ('V', u, i))
            yield ('sync', 'b' if is_b else 'a', 1)
            yield ('arrive', 'M_READY')
            yield ('arrive', 'VEC_FREE%d' % vb)
            nvec += 1
            xs = kx % X; kx += 1
            yield ('wait', 'Y_READY', n_y); n_y += 1
            outs = ('Yd', 'Yof') if S.hb_zero(i) else ('Yd', 'Yof', 'Yob')   # no C_b H_b for a zero state
            for nm in outs:
                yield ('read', (nm, half), (nm, u, i))
            yield ('read', ('x', xs, half), ('x', u, 2, i))
            yield ('write', ('x', xs, half), ('y', u, i))
            for nm in outs:
                yield ('read', (nm, half), (nm, u, i))
            yield ('sync', 'ab', 2)
            if is_b:
                yield ('arrive', 'Y_FREE')
                yield ('store', [(('x', xs, 0), ('y', u, i)), (('x', xs, 1), ('y', u, i))])
                yield ('store_wait',)
                yield ('arrive', 'X_EMPTY%d' % xs)

def run(S, units_list):
    counts = {'M_READY': 2, 'VEC_FREE0': 2, 'VEC_FREE1': 2}
    roles = {
        'prod': producer(S, units_list), 'mma': mma(S, units_list), 'C': group_c(S, units_list),
        'A': group_ab(S, units_list, False), 'B': group_ab(S, units_list, True),
    }
    run_roles(S, roles, counts)


def _schedules(n, mode='bidir', kxs=2, xw_per_slot=True, seed0=0, shared_bc=False, release_early=False,
               rzero=True):
    fails = []
    for seed in range(seed0, seed0 + n):
        r = random.Random(seed)
        nt = 1 if shared_bc else r.choice([1, 2, 3, 4, 5, 9])
        nunits = r.choice([3, 5, 8]) if shared_bc else r.choice([1, 2, 3])
        # runs of units on the same C/B tiles (consecutive heads of one batch element)
        bc = None
        if shared_bc:
            bc, g = [], 0
            for _ in range(nunits):
                if bc and r.random() < 0.4:
                    g += 1
                bc.append(g)
        S = Sim(nt, nunits, seed, mode=mode, kxs=kxs, xw_per_slot=xw_per_slot,
                heavy=r.choice([0.0, 0.05, 0.2, 0.5]), bc=bc, release_early=release_early, rzero=rzero)
        try:
            run(S, list(range(nunits)))
        except Bug as e:
            fails.append(f"seed {seed} nt {nt} units {nunits}: {e}")
    return fails


def test_fused_protocol_has_no_overrun_deadlock_or_race():
    fails = _schedules(2000)
    assert not fails, "\n".join(fails[:5])


def test_state_mode_protocol():
    """The forward state pass alone (its 2 x slots each paired with a low-part
    buffer that lives and dies with the slot)."""
    fails = _schedules(1500, mode='state', kxs=2)
    assert not fails, "\n".join(fails[:5])


def test_model_catches_odd_slot_count_in_state_mode():
    """With an odd number of x slots the alternating preparing groups do not
    see every phase of a slot: one of them can pass a slot's parity wait
    before the load another group waited for has landed."""
    fails = _schedules(200, mode='state', kxs=3)
    assert fails and any("read ('x'" in f for f in fails)


def test_model_catches_single_diag_w_x_barrier():
    fails = _schedules(100, xw_per_slot=False)
    assert fails and any("overrun on XW_READY" in f for f in fails)


def test_one_tile_units_reusing_shared_c_b_tiles():
    """One-tile sequences whose consecutive units (heads of one batch element
    and B/C group) take their C/B tiles from the ring in place: the slots are
    released only after the last unit of a run, and no load is issued for the
    others."""
    fails = _schedules(1500, shared_bc=True)
    assert not fails, "\n".join(fails[:5])


def test_model_catches_reused_slots_released_per_unit():
    fails = _schedules(300, shared_bc=True, release_early=True)
    assert fails and any("read ('ring'" in f or "overrun" in f for f in fails)


def test_seeded_reverse_start_loads_the_last_tile_state():
    """With a given reverse start state the last tile's reverse state is
    stored, loaded and multiplied like every other tile's."""
    fails = _schedules(1000, rzero=False)
    assert not fails, "\n".join(fails[:5])
