"""Barrier protocol of the block-step kernel (ssd_blockstep.cu), checked on
the CPU.

One CTA per (batch, head) unit, nine warps. The issuing warp's lane 0 loads
C, B and x with TMA. It computes G = [C_f; C_b][B_f; B_b]^T as soon as C and
B are in, then C H once every mask warp has put its part of the cached state
in shared memory ("state ready", one arrival per mask warp). It computes Y =
M [X; X] once every mask warp has written its part of M over G ("mask
built", one arrival per mask warp) and x is in, and commits both products.
The mask warps load dt and the state, compute the decay vectors (warps 0..3,
a named barrier), convert the state and arrive, pass a named barrier over all
eight, wait for G, build the mask and arrive. Then a CTA barrier, and the
epilogue reads Y, C H and x and stores the output.

The model runs these steps in the kernel's order, with random heavy-tailed
delays on every TMA load and MMA and random stepping order. Each schedule is
checked for phase overruns, deadlock and stale reads: C/B, x, the state, the
vectors, G, M, Y and C H.

Planted variants that the model must catch: C H issued without waiting for
the state, Y issued without waiting for the mask, the mask built without
waiting for G, and the epilogue reading before the MMAs' commit.
"""
import random

from protocol_sim import Bug, Sched, run_roles


class Step(Sched):
    def __init__(self, seed, heavy=0.1, has_h=True, wait_h=True, wait_m=True, wait_g=True, wait_y=True, masks=4):
        super().__init__(seed, heavy)
        self.has_h, self.wait_h, self.wait_m, self.wait_g, self.wait_y = has_h, wait_h, wait_m, wait_g, wait_y
        self.masks = masks


def issuer(S):
    yield ('tma', 'LOAD', [('C', 'C'), ('B', 'B')])
    yield ('tma', 'X', [('x', 'x')])
    yield ('wait', 'LOAD', 0)
    # G into TMEM: every mask warp's region (its 32 rows, its column block)
    yield ('mma', [('C', 'C'), ('B', 'B')], [(('G', w), 'G') for w in range(S.masks)])
    yield ('commit', 'G')
    if S.has_h:
        if S.wait_h:
            yield ('wait', 'H', 0)
        yield ('mma', [('C', 'C')] + [(('H', w), 'H') for w in range(S.masks)], [('Yo', 'Yo')])
    if S.wait_m:
        yield ('wait', 'M', 0)
    yield ('wait', 'X', 0)
    yield ('mma', [(('G', w), 'M') for w in range(S.masks)] + [('x', 'x')], [('Y', 'Y')])
    yield ('commit', 'Y')
    yield ('sync', 'cta', S.masks + 1)          # the epilogue's CTA barrier
    yield ('sync', 'cta2', S.masks + 1)         # teardown


def mask_warp(S, w):
    vec = w < S.masks // 2                      # warps 0..3 compute the vectors
    if vec:
        yield ('sync', 'scan', S.masks // 2)
        yield ('write', ('V', w), 'V')
        yield ('sync', 'scan2', S.masks // 2)
    if S.has_h:
        yield ('write', ('H', w), 'H')          # this warp's rows of the state's bf16 copy
        yield ('arrive', 'H')
    yield ('sync', 'vec', S.masks)             # the vectors, to every mask warp
    for v in range(S.masks // 2):
        yield ('read', ('V', v), 'V')
    if S.wait_g:
        yield ('wait', 'G', 0)
    yield ('read', ('G', w), 'G')
    yield ('write', ('G', w), 'M')              # this warp's part of M in place of G
    yield ('arrive', 'M')
    # the epilogue
    if S.wait_y:
        yield ('wait', 'Y', 0)
    yield ('wait', 'X', 0)
    yield ('read', 'Y', 'Y')
    if S.has_h:
        yield ('read', 'Yo', 'Yo')
    yield ('sync', 'cta', S.masks + 1)
    yield ('read', 'x', 'x')
    yield ('write', ('out', w), 'y')
    yield ('sync', 'cta2', S.masks + 1)


def run(S):
    counts = {'H': S.masks, 'M': S.masks}
    roles = {'issuer': issuer(S)}
    for w in range(S.masks):
        roles['mask%d' % w] = mask_warp(S, w)
    run_roles(S, roles, counts)
    for w in range(S.masks):
        S.read(('out', w), 'y', 'final output')


def _schedules(count, **kw):
    fails = []
    for seed in range(count):
        r = random.Random(seed)
        has_h = kw.get('has_h', r.random() < 0.8)
        S = Step(seed, heavy=r.choice([0.0, 0.05, 0.2, 0.5]), has_h=has_h,
                 **{k: v for k, v in kw.items() if k != 'has_h'})
        try:
            run(S)
        except Bug as e:
            fails.append(f"seed {seed}: {e}")
    return fails


def test_blockstep_protocol_has_no_overrun_deadlock_or_race():
    fails = _schedules(1500)
    assert not fails, "\n".join(fails[:5])


def test_model_catches_c_h_before_the_state_is_in():
    fails = _schedules(300, has_h=True, wait_h=False)
    assert fails and any("read ('H'" in f for f in fails)


def test_model_catches_y_before_the_mask_is_built():
    fails = _schedules(300, wait_m=False)
    assert fails and any("('G'" in f for f in fails)


def test_model_catches_mask_before_g():
    fails = _schedules(300, wait_g=False)
    assert fails and any("('G'" in f for f in fails)


def test_model_catches_epilogue_before_the_commit():
    fails = _schedules(300, wait_y=False)
    assert fails and any("read Y " in f or "read Yo " in f for f in fails)
