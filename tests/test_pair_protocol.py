"""Barrier protocol of the two-CTA bidirectional kernel (ssd_pair.cu), checked
on the CPU.

One cluster of two CTAs per (batch, head) unit: the forward CTA walks the
unit's 128-token tiles left to right, the reverse CTA right to left, each
with its own producer, MMA issuer, state-chain group (C) and mask/output
groups (A, B). A tile's two directions meet through global memory: the
direction that reaches the tile first stores its fp32 partial output and
then arrives on a barrier in the other CTA's shared memory (one barrier and
one partial slot per unit parity and tile); the other waits on that barrier,
adds the partial and stores the bf16 output. The model takes the kernel's
mbarrier waits and arrivals (those across the pair included), named-barrier
syncs, TMA loads, MMA commits (one in-order tensor pipe per CTA) and TMA
stores, in the kernel's order, with random heavy-tailed delays on every
asynchronous completion and random stepping order.

Each schedule is checked for phase overrun (a barrier moving two phases
past a waiter), deadlock (within a CTA or across the pair) and stale
reads of every buffer: the B/C ring, the x slots, H, diag(w) X, the TMEM
accumulators (G double-buffered, Y, Yo double-buffered, S), the per-tile
vectors and the partial slots in global memory.

Planted variants that the model must catch: partial slots not split by unit
parity (the forward CTA overwrites a partial before the reverse CTA has read
it), a partial barrier waited on with the unit's own phase instead of the
unit pair's, a single Yo accumulator (the next tile's C.H overwrites it before the
output epilogue has read it) and a single M_READY barrier (two mask phases
complete under one parity wait).
"""
import random

from protocol_sim import Bug, Sched, run_roles


class Pair(Sched):
    """One cluster's schedule: nt tiles per unit, units processed in order by
    both CTAs. init[d]: the direction starts from a given state (else zero,
    and the unit's first tile has no C.H term)."""
    def __init__(self, nt, units, seed, heavy=0.1, init=(False, False), par_slots=True, yo_double=True,
                 m_per_buf=True, phase_pairs=True):
        super().__init__(seed, heavy)
        self.nt, self.units = nt, units
        self.init = init
        self.par_slots = par_slots      # partial slots split by unit parity
        self.yo_double = yo_double      # two Yo accumulators
        self.m_per_buf = m_per_buf      # one M_READY barrier per G buffer
        self.phase_pairs = phase_pairs  # a partial barrier completes once per two units

    def steps(self, d):
        """(n, j, u, k, i) of every step of direction d (0 forward, 1 reverse)."""
        n = 0
        for j, u in enumerate(self.units):
            for k in range(self.nt):
                yield n, j, u, k, (k if d == 0 else self.nt - 1 - k)
                n += 1

    def first(self, d, k):
        """the direction reaches the tile before the other one (ties: forward)"""
        return 2 * k < self.nt - 1 or (2 * k == self.nt - 1 and d == 0)

    def hzero(self, d, k):
        return k == 0 and not self.init[d]

    def has_s(self, k):
        return k < self.nt - 1

    def slot(self, j, i):
        return ((j & 1) if self.par_slots else 0, i)

    def part_bar(self, d, j, i):
        """the partial barrier of tile i, unit j, in CTA d's shared memory, and
        the phase its waiters wait for (one completion per unit of the slot)"""
        par, t = self.slot(j, i)
        return 'fb'[d] + '.PART%d_%d' % (par, t), (j >> 1) if self.par_slots and self.phase_pairs else j

    def yo(self, n):
        return n & 1 if self.yo_double else 0

    def mready(self, n):
        """barrier and phase of the mask of step n"""
        if self.m_per_buf:
            return 'M_READY%d' % (n & 1), n >> 1
        return 'M_READY', n


def producer(S, d):
    p = 'fb'[d] + '.'
    kr = kx = 0
    for n, j, u, k, i in S.steps(d):
        for op in ('C', 'B'):
            rs = kr % 4
            if kr >= 4:
                yield ('wait', p + 'RING_EMPTY%d' % rs, kr // 4 - 1)
            kr += 1
            yield ('tma', p + 'RING_FULL%d' % rs, [((p + 'ring', rs), (op, d, u, i))])
        xs = kx % 3
        if kx >= 3:
            yield ('wait', p + 'X_EMPTY%d' % xs, kx // 3 - 1)
        kx += 1
        yield ('tma', p + 'X_FULL%d' % xs, [((p + 'x', xs, h), ('x', u, i)) for h in (0, 1)])


def mma(S, d):
    p = 'fb'[d] + '.'
    pipe = p + 'tc'
    kr = nxw = 0
    prev = None     # (n, u, i, xs) of the previous step: its Y = M X is issued one step late

    def y_of(m, um, im, xsm):
        bar, ph = S.mready(m)
        yield ('wait', p + bar, ph)
        yield ('wait', p + 'X_FULL%d' % xsm, m // 3)
        if m >= 1:
            yield ('wait', p + 'Y_FREE', m - 1)
        reads = [((p + 'G%d' % (m & 1), h), ('M', d, um, im)) for h in (0, 1)]
        reads += [((p + 'x', xsm, h), ('x', um, im)) for h in (0, 1)]
        yield ('mma', reads, [((p + 'Y', h), ('Y', d, um, im)) for h in (0, 1)], pipe)
        yield ('commit', p + 'Y_READY', pipe)

    for n, j, u, k, i in S.steps(d):
        rC = kr % 4
        yield ('wait', p + 'RING_FULL%d' % rC, kr // 4); kr += 1
        rB = kr % 4
        yield ('wait', p + 'RING_FULL%d' % rB, kr // 4); kr += 1
        b = n & 1
        yield ('mma', [((p + 'ring', rC), ('C', d, u, i)), ((p + 'ring', rB), ('B', d, u, i))],
               [((p + 'G%d' % b, h), ('G', d, u, i)) for h in (0, 1)], pipe)
        yield ('commit', p + 'G_READY%d' % b, pipe)
        if prev is not None:
            yield from y_of(*prev)
        yield ('wait', p + 'H_READY', n)
        if not S.hzero(d, k):
            yb = S.yo(n)
            yield ('mma', [((p + 'ring', rC), ('C', d, u, i)), (p + 'H', ('H', d, u, k))],
                   [((p + 'Yo%d' % yb, h), ('Yo', d, u, i)) for h in (0, 1)], pipe)
        yield ('commit', p + 'RING_EMPTY%d' % rC, pipe)
        if S.has_s(k):
            yield ('wait', p + 'XW_READY', nxw); nxw += 1
            yield ('mma', [((p + 'ring', rB), ('B', d, u, i)), (p + 'xw', ('xw', d, u, k))],
                   [(p + 'S', ('S', d, u, k))], pipe)
        yield ('commit', p + 'S_READY', pipe)
        yield ('commit', p + 'RING_EMPTY%d' % rB, pipe)
        prev = (n, u, i, n % 3)
    if prev is not None:
        yield from y_of(*prev)
    yield ('commit', p + 'MMA_DONE', pipe)
    yield ('wait', p + 'MMA_DONE', 0)


def group_c(S, d):
    p = 'fb'[d] + '.'
    for n, j, u, k, i in S.steps(d):
        vb = n & 1
        if n >= 2:
            yield ('wait', p + 'VEC_FREE%d' % vb, (n >> 1) - 1)
        yield ('write', (p + 'vec', vb), ('V', d, u, i))
        yield ('sync', p + 'c', 1)
        yield ('arrive', p + 'VEC_READY%d' % vb)
        if n >= 1:
            yield ('wait', p + 'S_READY', n - 1)
        if k > 0:
            yield ('read', p + 'S', ('S', d, u, k - 1))
        if not S.hzero(d, k):
            yield ('write', p + 'H', ('H', d, u, k))
        yield ('sync', p + 'c', 1)
        yield ('arrive', p + 'H_READY')
        if S.has_s(k):
            xs = n % 3
            yield ('wait', p + 'X_FULL%d' % xs, n // 3)
            for h in (0, 1):
                yield ('read', (p + 'x', xs, h), ('x', u, i))
            yield ('write', p + 'xw', ('xw', d, u, k))
            yield ('sync', p + 'c', 1)
            yield ('arrive', p + 'XW_READY')


def group_ab(S, d, is_b):
    p = 'fb'[d] + '.'
    half = 1 if is_b else 0
    g = p + ('b' if is_b else 'a')
    steps = list(S.steps(d))

    def mask(n, u, i):
        vb = n & 1
        yield ('wait', p + 'VEC_READY%d' % vb, n >> 1)
        yield ('read', (p + 'vec', vb), ('V', d, u, i))
        yield ('wait', p + 'G_READY%d' % (n & 1), n >> 1)
        yield ('read', (p + 'G%d' % (n & 1), half), ('G', d, u, i))
        yield ('write', (p + 'G%d' % (n & 1), half), ('M', d, u, i))
        yield ('sync', g, 1)
        yield ('arrive', p + S.mready(n)[0])
        yield ('arrive', p + 'VEC_FREE%d' % vb)

    def out(n, j, u, k, i):
        xs = n % 3
        second = not S.first(d, k)
        slot = S.slot(j, i)
        if second:
            # every thread waits on the barrier in its own CTA
            yield ('wait',) + S.part_bar(d, j, i)
        yield ('wait', p + 'Y_READY', n)
        yield ('read', (p + 'Y', half), ('Y', d, u, i))
        if not S.hzero(d, k):
            yield ('read', (p + 'Yo%d' % S.yo(n), half), ('Yo', d, u, i))
        if second:
            yield ('read', ('part',) + slot + (half,), ('P', 1 - d, u, i))
            yield ('read', (p + 'x', xs, half), ('x', u, i))
            yield ('write', (p + 'x', xs, half), ('y', u, i))
        else:
            yield ('write', ('part',) + slot + (half,), ('P', d, u, i))
        yield ('sync', p + 'ab', 2)
        if second:
            # the partial's lines are dropped from L2 after both groups read them
            yield ('write', ('part',) + slot + (half,), ('discarded',))
        if is_b:
            yield ('arrive', p + 'Y_FREE')
            if second:
                yield ('store_g', [((p + 'x', xs, 0), ('y', u, i)), ((p + 'x', xs, 1), ('y', u, i))],
                       [(('out', u, i), ('y', u, i))])
                yield ('store_wait',)
            else:
                # release arrival on the other CTA's barrier of this slot
                yield ('arrive', S.part_bar(1 - d, j, i)[0])
            yield ('arrive', p + 'X_EMPTY%d' % xs)

    prev = None
    for n, j, u, k, i in steps:
        yield from mask(n, u, i)
        if prev is not None:
            yield from out(*prev)
        prev = (n, j, u, k, i)
    if prev is not None:
        yield from out(*prev)
    if is_b:
        yield ('store_wait_all',)


def run(S):
    counts = {}
    for p in ('f.', 'b.'):
        for b in ('M_READY0', 'M_READY1', 'M_READY', 'VEC_FREE0', 'VEC_FREE1'):
            counts[p + b] = 2
    roles = {}
    for d in (0, 1):
        p = 'fb'[d]
        roles[p + 'prod'] = producer(S, d)
        roles[p + 'mma'] = mma(S, d)
        roles[p + 'C'] = group_c(S, d)
        roles[p + 'A'] = group_ab(S, d, False)
        roles[p + 'B'] = group_ab(S, d, True)
    run_roles(S, roles, counts)
    # every output tile of every unit was written once, by the second direction
    for u in S.units:
        for i in range(S.nt):
            S.read(('out', u, i), ('y', u, i), 'final output')


def _schedules(n, seed0=0, **kw):
    fails = []
    for seed in range(seed0, seed0 + n):
        r = random.Random(seed)
        nt = r.choice([2, 3, 4, 5, 8])
        nunits = r.choice([1, 2, 3, 5])
        init = (r.random() < 0.3, r.random() < 0.3)
        S = Pair(nt, [3 * q + 1 for q in range(nunits)], seed, heavy=r.choice([0.0, 0.05, 0.2, 0.5]), init=init,
                 **kw)
        try:
            run(S)
        except Bug as e:
            fails.append(f"seed {seed} nt {nt} units {nunits}: {e}")
    return fails


def test_pair_protocol_has_no_overrun_deadlock_or_race():
    fails = _schedules(1500)
    assert not fails, "\n".join(fails[:5])


def test_model_catches_partial_slots_without_unit_parity():
    fails = _schedules(400, par_slots=False)
    assert fails and any("read ('part'" in f or "overrun" in f for f in fails)


def test_model_catches_single_yo_accumulator():
    fails = _schedules(300, yo_double=False)
    assert fails and any("Yo" in f for f in fails)


def test_model_catches_single_mask_barrier():
    fails = _schedules(300, m_per_buf=False)
    assert fails and any("overrun on" in f and "M_READY" in f for f in fails)


def test_model_catches_partial_barrier_phase_per_unit():
    fails = _schedules(200, phase_pairs=False)
    assert fails and any("deadlock" in f or "overrun" in f for f in fails)
