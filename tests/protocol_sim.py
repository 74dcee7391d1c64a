"""Discrete-event engine for the barrier-protocol models of the persistent
tensor-core kernels (test_fused_protocol.py, test_pair_protocol.py,
test_onetile_protocol.py, test_blockstep_protocol.py).

Roles are generators that yield the commands below; asynchronous completions
(TMA loads and stores, MMAs in issue order) land after random, heavy-tailed
delays, and runnable roles are stepped in random order. A schedule fails on a
phase overrun (a barrier completing two phases past the one a role waits for,
which the hardware parity wait would miss), on deadlock, and on a read that
does not see the version of a buffer it needs.

Commands:
  ('wait', bar, k)      wait for completion of phase k (parity k & 1)
  ('arrive', bar)
  ('tma', bar, [(res, val)])          async load: writes then arrives
  ('mma', [(res,val)] reads, [(res,val)] writes[, pipe])   in-order async
  ('commit', bar[, pipe])             arrives when all prior MMAs (of the pipe) are done
  ('read', res, val) / ('write', res, val)
  ('sync', name, n)                   named barrier over n roles
  ('store', [(res,val)]) then ('store_wait',)      store's shared-memory read
  ('store_wait1',)                    the shared-memory reads of all but the
                                      role's newest store (bulk wait_group.read 1)
  ('store_g', [(res,val)] smem reads, [(res,val)] global writes)
  ('store_wait_all',)                 all of the role's stores complete
  ('gset', flag, value)               a release store of a flag in global memory
  ('gwait', flag, value)              an acquire poll until the flag holds value;
                                      seeing a later value is an overrun
"""
import heapq
import itertools
import random


class Bug(Exception):
    pass

class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.c = name, count, count, 0
    def arrive(self):
        self.pending -= 1
        if self.pending < 0:
            raise Bug(f"{self.name}: too many arrivals")
        if self.pending == 0:
            self.c += 1
            self.pending = self.count

class Sched:
    """The state of one schedule: barriers, buffer versions, the event queue."""
    def __init__(self, seed, heavy=0.1):
        self.r = random.Random(seed)
        self.heavy = heavy
        self.bars = {}
        self.res = {}
        self.t = 0.0
        self.ev = []          # (time, seq, fn)
        self.seq = itertools.count()
        self.mma_done = {}    # per tensor pipe: completion time of its last MMA
        self.flags = {}       # global-memory flags (gset / gwait), start at 0
    def bar(self, name, count=1):
        if name not in self.bars:
            self.bars[name] = Bar(name, count)
        return self.bars[name]
    def delay(self):
        d = self.r.expovariate(1.0)
        if self.r.random() < self.heavy:
            d *= self.r.choice([10, 50, 200])
        return d
    def at(self, t, fn):
        heapq.heappush(self.ev, (t, next(self.seq), fn))
    def write(self, k, v):
        self.res[k] = v
    def read(self, k, v, who):
        got = self.res.get(k)
        if got != v:
            raise Bug(f"{who}: read {k} expected {v} got {got} at t={self.t:.2f}")


def run_roles(S, roles, counts):
    """Step the role generators `roles` (name -> generator) to completion on
    the schedule `S`; `counts` gives the arrival count of barriers other than 1."""
    cur = {k: None for k in roles}        # pending command per role
    ready = {k: 0.0 for k in roles}
    done = set()
    syncs = {}                            # name -> set of roles arrived
    store_pending = {}
    store_reads = {}                      # role -> shared-memory read times of its stores, in order
    store_done = {}                       # role -> completion time of its last global store
    def bar(n):
        return S.bar(n, counts.get(n, 1))
    def step_role(name):
        """Try to make progress on role `name`; return True if it advanced."""
        if cur[name] is None:
            try:
                cur[name] = next(roles[name])
            except StopIteration:
                done.add(name)
                return True
        c = cur[name]
        op = c[0]
        if op == 'wait':
            b = bar(c[1]); k = c[2]
            if b.c >= k + 2:
                raise Bug(f"{name}: overrun on {c[1]}: waiting for phase {k}, completed {b.c}")
            if (b.c & 1) != (k & 1):     # the phase with parity k&1 completed (c == k+1)
                cur[name] = None
                return True
            return False
        if op == 'arrive':
            bar(c[1]).arrive()
        elif op == 'tma':
            bn, writes = c[1], c[2]
            def land(writes=writes, bn=bn):
                for k, v in writes:
                    S.write(k, v)
                bar(bn).arrive()
            S.at(S.t + S.delay(), land)
        elif op == 'tma_hb':
            bn, u, i = c[1], c[2], c[3]
            S.read(('hbg', u, i), ('hbg', u, i), name + ' hb load issue')
            def land(bn=bn, u=u, i=i):
                S.write('hb', ('hb', u, i))
                bar(bn).arrive()
            S.at(S.t + S.delay(), land)
        elif op == 'mma':
            reads, writes = c[1], c[2]
            pipe = c[3] if len(c) > 3 else None     # one in-order tensor pipe per CTA
            tdone = max(S.mma_done.get(pipe, 0.0), S.t) + S.delay()
            S.mma_done[pipe] = tdone
            def ex(reads=reads, writes=writes):
                for k, v in reads:
                    S.read(k, v, 'mma exec')
                for k, v in writes:
                    S.write(k, v)
            S.at(tdone, ex)
        elif op == 'commit':
            bn = c[1]
            pipe = c[2] if len(c) > 2 else None
            S.at(max(S.mma_done.get(pipe, 0.0), S.t) + 1e-6, lambda bn=bn: bar(bn).arrive())
        elif op == 'read':
            S.read(c[1], c[2], name)
        elif op == 'write':
            S.write(c[1], c[2])
        elif op == 'sync':
            nm, n = c[1], c[2]
            if n == 1:
                pass
            else:
                s = syncs.setdefault(nm, set())
                s.add(name)
                if len(s) < n:
                    return False
                # all arrived: release the others lazily
                for other in list(s):
                    if other != name and cur[other] == c:
                        cur[other] = None
                syncs[nm] = set()
        elif op == 'store':
            for k, v in c[1]:
                S.read(k, v, 'store issue')
            tr = S.t + S.delay()
            store_pending[name] = (tr, c[1])
            def rd(items=c[1]):
                for k, v in items:
                    S.read(k, v, 'store read')
            S.at(tr, rd)
        elif op == 'store_g':
            # a TMA store: reads shared memory by tr, writes global memory at tc
            for k, v in c[1]:
                S.read(k, v, 'store issue')
            tr = S.t + S.delay()
            tc = tr + S.delay()
            store_pending[name] = (tr, c[1])
            store_reads.setdefault(name, []).append(tr)
            store_done[name] = max(store_done.get(name, 0.0), tc)
            def rd(items=c[1]):
                for k, v in items:
                    S.read(k, v, 'store read')
            def wr(items=c[2]):
                for k, v in items:
                    S.write(k, v)
            S.at(tr, rd)
            S.at(tc, wr)
        elif op == 'store_wait':
            tr, _ = store_pending[name]
            if S.t < tr:
                return False
        elif op == 'store_wait1':
            if S.t < max(store_reads.get(name, [0.0])[:-1], default=0.0):
                return False
        elif op == 'store_wait_all':
            if S.t < store_done.get(name, 0.0):
                return False
        elif op == 'gset':
            S.flags[c[1]] = c[2]
        elif op == 'gwait':
            got = S.flags.get(c[1], 0)
            if got != c[2]:
                if got > c[2]:
                    raise Bug(f"{name}: flag {c[1]} overrun: waiting for {c[2]}, holds {got}")
                return False
        cur[name] = None
        return True
    while len(done) < len(roles):
        progressed = True
        while progressed:
            progressed = False
            order = [r for r in roles if r not in done]
            S.r.shuffle(order)
            for r in order:
                if r in done or ready[r] > S.t:
                    continue
                # a sync waiter whose partner already released it
                if step_role(r):
                    ready[r] = S.t + (S.r.expovariate(4.0) if S.r.random() < 0.5 else 0.0)
                    progressed = True
        if len(done) == len(roles):
            break
        nxt = [ready[r] for r in roles if r not in done and ready[r] > S.t]
        tnext = min(nxt) if nxt else None
        if S.ev and (tnext is None or S.ev[0][0] <= tnext):
            t, _, fn = heapq.heappop(S.ev)
            S.t = max(S.t, t)
            fn()
        elif tnext is not None:
            S.t = tnext
        else:
            state = {r: cur[r] for r in roles if r not in done}
            raise Bug(f"deadlock at t={S.t:.2f}: {state}")
    while S.ev:
        t, _, fn = heapq.heappop(S.ev)
        S.t = t
        fn()
