"""Barrier protocol of the one-tile kernel (ssd_onetile.cu), checked on the CPU.

One CTA runs a contiguous run of (batch, head) units. Their B/C groups may
start and end anywhere in the run. The CTA has four roles that hand work
over through mbarriers:
  - the MMA thread loads each group's C and B (the next group's as soon as
    the current group's G is computed), computes G once per group, and
    computes Y = M X per head into one of two Y buffers;
  - the mask warps read G and a head's vectors and write the head's masked
    matrix into one of two M buffers;
  - the vector warps (three, heads j = 0, 1, 2 mod 3) write a head's vectors
    into one of three buffers;
  - the epilogue warps (a named barrier among them) read Y and the head's x
    slot, write y over it and store it. Their leader loads x four heads
    ahead, into the slot whose store has finished reading (five slots).
The model runs these steps in the kernel's order, with random heavy-tailed
delays on every TMA load, MMA and store, and random stepping order. Each
schedule is checked for phase overruns, deadlock and stale reads of every
buffer: C/B, G, the vectors, M, Y, the x slots and the outputs.

Planted variants that the model must catch: the x load issued without
waiting for the previous store's read of that slot; vector buffers rewritten
without the mask warps' release; M rewritten before the MMA that read it has
completed; Y rewritten before the epilogue has read it; a single Y buffer;
and the next group's G computed as soon as its C and B are in, before the
mask warps are done with the current group's.
"""
import random

from protocol_sim import Bug, Sched, run_roles

XS, VS = 5, 3


class OneTile(Sched):
    """One CTA: `groups[j]` is the B/C group of the run's head j (contiguous
    runs of equal ids)."""
    def __init__(self, groups, seed, heavy=0.1, x_wait=True, v_release=True, m_wait=True, y_wait=True,
                 y_double=True, g_after_masks=True, masks=2, epis=2):
        super().__init__(seed, heavy)
        self.groups = groups
        self.n = len(groups)
        self.x_wait, self.v_release, self.m_wait, self.y_wait = x_wait, v_release, m_wait, y_wait
        self.y_double, self.g_after_masks = y_double, g_after_masks
        self.masks, self.epis = masks, epis

    def first(self, j):
        return j == 0 or self.groups[j] != self.groups[j - 1]

    def gidx(self, j):
        """the group's index within the run"""
        return sum(1 for k in range(j + 1) if self.first(k)) - 1

    def yd(self, j):
        """the TMEM buffer Y_j is written to (the barriers stay per parity)"""
        return 'Y%d' % (j & 1 if self.y_double else 0)


def mma(S):
    n = S.n
    ngroups = S.gidx(n - 1) + 1
    cb_waited = 0

    def load_cb(g):
        return ('tma', 'CB', [('cb', ('CB', g))])

    def issue_g(g):
        nonlocal cb_waited
        yield ('wait', 'CB', cb_waited)
        cb_waited += 1
        yield ('mma', [('cb', ('CB', g))], [('G', ('G', g))])
        yield ('commit', 'G')

    yield load_cb(0)
    yield from issue_g(0)
    gk = 0
    for j in range(n):
        g = S.gidx(j)
        if S.first(j):
            yield ('wait', 'G', gk)
            gk += 1
            if g + 1 < ngroups:
                yield load_cb(g + 1)
                if not S.g_after_masks:
                    yield from issue_g(g + 1)
        yield ('wait', 'MF%d' % (j & 1), j >> 1)
        yield ('wait', 'X%d' % (j % XS), j // XS)
        if j >= 2 and S.y_wait:
            yield ('wait', 'YE%d' % (j & 1), (j - 2) >> 1)
        yield ('mma', [('M%d' % (j & 1), ('M', j)), (('x', j % XS), ('x', j))], [(S.yd(j), ('Y', j))])
        yield ('commit', 'YB%d' % (j & 1))
        if S.g_after_masks and j + 1 < n and S.first(j + 1):
            yield from issue_g(g + 1)


def mask(S, w):
    gk = 0
    for j in range(S.n):
        if S.first(j):
            yield ('wait', 'G', gk)
            gk += 1
        yield ('wait', 'V%d' % (j % VS), j // VS)
        if j >= 2 and S.m_wait:
            yield ('wait', 'YB%d' % (j & 1), (j - 2) >> 1)      # the MMA of head j - 2 has read M
        yield ('read', 'G', ('G', S.gidx(j)))
        yield ('read', ('V', j % VS), ('V', j))
        yield ('write', 'M%d' % (j & 1), ('M', j))
        yield ('arrive', 'MF%d' % (j & 1))
        yield ('arrive', 'VE%d' % (j % VS))


def vectors(S, v):
    for j in range(v, S.n, VS):
        if j >= VS and S.v_release:
            yield ('wait', 'VE%d' % (j % VS), j // VS - 1)
        yield ('write', ('V', j % VS), ('V', j))
        yield ('arrive', 'V%d' % (j % VS))


def epilogue(S, e):
    leader = e == 0
    n = S.n
    if leader:
        for j in range(min(XS - 1, n)):
            yield ('tma', 'X%d' % (j % XS), [(('x', j % XS), ('x', j))])
    for i in range(n):
        yield ('wait', 'YB%d' % (i & 1), i >> 1)
        yield ('wait', 'X%d' % (i % XS), i // XS)
        yield ('read', S.yd(i), ('Y', i))
        yield ('sync', 'epi_a', S.epis)
        if leader:
            yield ('arrive', 'YE%d' % (i & 1))
        yield ('read', ('x', i % XS), ('x', i))
        yield ('sync', 'epi_b', S.epis)
        if leader:
            yield ('write', ('x', i % XS), ('y', i))
        yield ('sync', 'epi_c', S.epis)
        if leader:
            yield ('store_g', [(('x', i % XS), ('y', i))], [(('out', i), ('y', i))])
            if i + XS - 1 < n:
                if S.x_wait:
                    yield ('store_wait1',)
                yield ('tma', 'X%d' % ((i + XS - 1) % XS), [(('x', (i + XS - 1) % XS), ('x', i + XS - 1))])
    if leader:
        yield ('store_wait_all',)


def run(S):
    counts = {'MF0': S.masks, 'MF1': S.masks, 'VE0': S.masks, 'VE1': S.masks, 'VE2': S.masks}
    roles = {'mma': mma(S)}
    for w in range(S.masks):
        roles['mask%d' % w] = mask(S, w)
    for v in range(VS):
        roles['vec%d' % v] = vectors(S, v)
    for e in range(S.epis):
        roles['epi%d' % e] = epilogue(S, e)
    run_roles(S, roles, counts)
    for i in range(S.n):
        S.read(('out', i), ('y', i), 'final output')


def _groups(r):
    hpg = r.choice([1, 2, 3, 5, 24])
    off = r.randrange(hpg)
    n = r.choice([1, 2, 3, 4, 6, 9, 13])
    return [(off + j) // hpg for j in range(n)]


def _schedules(count, seed0=0, **kw):
    fails = []
    for seed in range(seed0, seed0 + count):
        r = random.Random(seed)
        groups = _groups(r)
        S = OneTile(groups, seed, heavy=r.choice([0.0, 0.05, 0.2, 0.5]), **kw)
        try:
            run(S)
        except Bug as e:
            fails.append(f"seed {seed} groups {groups}: {e}")
    return fails


def test_onetile_protocol_has_no_overrun_deadlock_or_race():
    fails = _schedules(1500)
    assert not fails, "\n".join(fails[:5])


def test_model_catches_x_load_before_the_store_has_read_the_slot():
    fails = _schedules(600, x_wait=False)
    assert fails and any("('x'" in f or "store read" in f for f in fails)


def test_model_catches_vectors_rewritten_without_release():
    fails = _schedules(400, v_release=False)
    assert fails and any("'V'" in f for f in fails)


def test_model_catches_mask_written_before_its_mma_completed():
    fails = _schedules(400, m_wait=False)
    assert fails and any("'M'" in f for f in fails)


def test_model_catches_y_rewritten_before_the_epilogue_read_it():
    fails = _schedules(400, y_wait=False)
    assert fails and any("'Y'" in f for f in fails)


def test_model_catches_single_y_buffer():
    fails = _schedules(400, y_double=False)
    assert fails and any("'Y'" in f for f in fails)


def test_model_catches_next_g_before_the_masks_are_done():
    fails = _schedules(400, g_after_masks=False)
    assert fails and any("'G'" in f for f in fails)
