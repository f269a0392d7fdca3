"""Model check of the persistent prefill attention kernels' barrier protocols
(attention_tc.cu: attn_prefill_tc_persistent_kernel, one head per item, and
attn_prefill_tc_dual_kernel, two heads of a GQA group per item), run on the
CPU.

Five actors are simulated under random interleavings: the TMA producer, the
MMA issuer, the softmax warps (which also read O out at the end of every
item), and the two asynchronous engines (TMA copies and tensor-core
operations, each completing in issue order). mbarriers follow their parity
semantics: a wait for parity p returns once the phase with that parity has
completed, so a waiter two phases behind would pass wrongly. The model
checks, at every wait, that the completed phase is exactly the one meant,
and at every buffer access that the data is the intended version (Q per
item, K/V per tile, S per tile, P per tile, O per item). The waits mirror
the kernel's; the kernel and this model are kept in step by hand. Dropping
any of the protocol's cross-item waits must make the model fail."""
import random

import pytest


class ProtocolError(Exception):
    pass


class Bar:
    def __init__(self, expected=1):
        self.exp, self.arr, self.done = expected, 0, 0

    def arrive(self):
        self.arr += 1
        if self.arr == self.exp:
            self.arr, self.done = 0, self.done + 1

    def passes(self, parity):
        return (self.done & 1) != parity


def simulate(nkts, seed, drop=()):
    """Run one random schedule over items with nkts[i] key tiles each."""
    rng = random.Random(seed)
    bars = {}
    for i in range(2):
        for n in ('q_full', 'q_empty', 'k_full', 'k_empty', 'v_full', 'v_empty', 's_full'):
            bars[f'{n}{i}'] = Bar()
    for n in ('p_full', 'o_done'):
        bars[n] = Bar()
    st = dict(Q=[None, None], K=[None, None], V=[None, None], S=[None, None], P=None, O_item=None, O_tiles=set(),
              s_read=set(), o_read=set(), pv_done=set(), s_done=set())
    tma, tc = [], []
    first = [sum(nkts[:i]) for i in range(len(nkts))]

    def wait(name, n):  # wait for completion number n of barrier `name`
        b = bars[name]
        while not b.passes(n & 1):
            yield 'blocked'
        if b.done != n + 1:
            raise ProtocolError(f'{name}: passed for completion {n} with {b.done} completed')

    def producer():
        t = 0
        for i, n in enumerate(nkts):
            qs = i & 1
            if i >= 2:
                yield from wait(f'q_empty{qs}', (i >> 1) - 1)
                if not set(range(first[i - 2], first[i - 2] + nkts[i - 2])) <= st['s_done']:
                    raise ProtocolError('Q buffer reloaded while still read')
            tma.append(('Q', qs, i))
            for _ in range(n):
                s = t & 1
                if t >= 2:
                    yield from wait(f'k_empty{s}', (t >> 1) - 1)
                    if t - 2 not in st['s_done']:
                        raise ProtocolError('K stage reloaded while still read')
                tma.append(('K', s, t))
                if t >= 2:
                    yield from wait(f'v_empty{s}', (t >> 1) - 1)
                    if t - 2 not in st['pv_done']:
                        raise ProtocolError('V stage reloaded while still read')
                tma.append(('V', s, t))
                t += 1
                yield 'step'

    def mma():
        t = 0
        for i, n in enumerate(nkts):
            qs = i & 1
            yield from wait(f'q_full{qs}', i >> 1)

            def issue_s(tt):
                yield from wait(f'k_full{tt & 1}', tt >> 1)
                tc.extend([('S', tt, qs, i), ('commit', f's_full{tt & 1}'), ('commit', f'k_empty{tt & 1}')])

            yield from issue_s(t)
            for j in range(n):
                tj = t + j
                if j + 1 < n:
                    yield from issue_s(tj + 1)
                elif 'q_empty' not in drop:
                    tc.append(('commit', f'q_empty{qs}'))
                yield from wait('p_full', tj)
                yield from wait(f'v_full{tj & 1}', tj >> 1)
                tc.extend([('PV', tj, i, j), ('commit', f'v_empty{tj & 1}'), ('commit', 'o_done')])
                yield 'step'
            t += n

    def softmax():
        t = 0
        for i, n in enumerate(nkts):
            for j in range(n):
                yield from wait(f's_full{t & 1}', t >> 1)
                if st['S'][t & 1] != t:
                    raise ProtocolError('softmax read a stale S')
                st['s_read'].add(t)
                yield 'step'
                if t > 0 and 'softmax_o_done' not in drop:
                    yield from wait('o_done', t - 1)
                if t > 0 and t - 1 not in st['pv_done']:
                    raise ProtocolError('P overwritten before its product ran')
                if j > 0 and st['O_item'] != i:
                    raise ProtocolError('rescaled another item\'s O')
                st['P'] = t
                bars['p_full'].arrive()
                t += 1
            # O / l of item i out of TMEM
            if 'softmax_o_final' not in drop:
                yield from wait('o_done', t - 1)
            want = set(range(t - n, t))
            if st['O_item'] != i or st['O_tiles'] != want:
                raise ProtocolError('read the wrong O')
            yield 'step'
            if st['O_item'] != i or st['O_tiles'] != want:
                raise ProtocolError('O changed while being read')
            st['o_read'].add(i)

    def run_tma():
        kind, s, x = tma.pop(0)
        st[kind][s] = x
        bars[f'{kind.lower()}_full{s}'].arrive()

    def run_tc():
        op = tc.pop(0)
        if op[0] == 'S':
            _, tt, qs, i = op
            if st['Q'][qs] != i or st['K'][tt & 1] != tt:
                raise ProtocolError('S product read a stale Q or K')
            if tt >= 2 and tt - 2 not in st['s_read']:
                raise ProtocolError('S buffer overwritten before it was read')
            st['S'][tt & 1] = tt
            st['s_done'].add(tt)
        elif op[0] == 'PV':
            _, tt, i, j = op
            if st['P'] != tt or st['V'][tt & 1] != tt:
                raise ProtocolError('P V product read a stale P or V')
            if j == 0:
                if i > 0 and i - 1 not in st['o_read']:
                    raise ProtocolError('O overwritten before it was read')
                st['O_item'], st['O_tiles'] = i, set()
            st['O_tiles'].add(tt)
            st['pv_done'].add(tt)
        else:
            bars[op[1]].arrive()

    actors = {'producer': producer(), 'mma': mma(), 'softmax': softmax()}
    # each actor and engine runs at its own random rate, so some schedules
    # starve one of them for long stretches
    rate = {a: rng.choice([0.05, 0.3, 1.0]) for a in list(actors) + ['tma', 'tc']}
    finished, idle = set(), 0
    while len(finished) < len(actors):
        moved = False
        names = [a for a in actors if a not in finished]
        rng.shuffle(names)
        for a in names:
            if rng.random() >= rate[a]:
                continue
            try:
                moved |= next(actors[a]) != 'blocked'
            except StopIteration:
                finished.add(a)
                moved = True
        if tma and rng.random() < rate['tma']:
            run_tma()
            moved = True
        if tc and rng.random() < rate['tc']:
            run_tc()
            moved = True
        idle = 0 if moved else idle + 1
        if idle > 2000:
            raise ProtocolError(f'deadlock; finished: {sorted(finished)}')
    while tc:
        run_tc()
    if len(st['o_read']) != len(nkts):
        raise ProtocolError('an item was never written out')


def _cases(n):
    for seed in range(n):
        rng = random.Random(seed * 7 + 1)
        yield [rng.choice([1, 1, 2, 3, 5, 16]) for _ in range(rng.randint(1, 7))], seed


def test_protocol_holds_under_random_schedules():
    for nkts, seed in _cases(400):
        simulate(nkts, seed)


@pytest.mark.parametrize('drop', ['softmax_o_final', 'softmax_o_done', 'q_empty'])
def test_dropping_a_wait_is_caught(drop):
    with pytest.raises(ProtocolError):
        for nkts, seed in _cases(400):
            simulate(nkts, seed, drop=(drop,))


# ------------------------------------------------ two heads of a group per item
def simulate_dual(nkts, seed, drop=()):
    """The barrier protocol of attn_prefill_tc_dual_kernel: items of two query
    tiles (A, B) that share every K and V tile; one Q buffer per tile; S_X
    single-buffered per tile with P_X written over it; per key tile the
    products run P_A V, S_A(t+1), P_B V, S_B(t+1). Products writing different
    accumulators need not run in issue order on the hardware, so the model
    checks at issue time that S_X(t+1) follows the completion of P_X(t) V(t)
    (the wait on o_done[X]) instead of relying on the in-order queue."""
    rng = random.Random(seed)
    bars = {}
    for i in range(2):
        for n in ('q_full', 'q_empty', 'k_full', 'k_empty', 'v_full', 'v_empty', 's_full', 'o_done'):
            bars[f'{n}{i}'] = Bar()
        bars[f'p_full{i}'] = Bar()
    st = dict(Q=[None, None], K=[None, None], V=[None, None], S=[None, None], P=[None, None],
              O=[None, None], O_tiles=[set(), set()], o_read=[set(), set()], pv_done=set(), s_done=set(),
              s_read=[set(), set()])
    tma, tc = [], []
    first = [sum(nkts[:i]) for i in range(len(nkts))]

    def wait(name, n):
        b = bars[name]
        while not b.passes(n & 1):
            yield 'blocked'
        if b.done != n + 1:
            raise ProtocolError(f'{name}: passed for completion {n} with {b.done} completed')

    def producer():
        t = 0
        for i, n in enumerate(nkts):
            for j in range(n):
                s = t & 1
                if t >= 2 and 'k_empty' not in drop:
                    yield from wait(f'k_empty{s}', (t >> 1) - 1)
                if t >= 2 and not {(0, t - 2), (1, t - 2)} <= st['s_done']:
                    raise ProtocolError('K stage reloaded while still read')
                tma.append(('K', s, t))
                if j == 0:
                    for x in range(2):
                        if i >= 1:
                            if 'q_empty' not in drop:
                                yield from wait(f'q_empty{x}', i - 1)
                            last = first[i - 1] + nkts[i - 1] - 1
                            if (x, last) not in st['s_done']:
                                raise ProtocolError('Q buffer reloaded while still read')
                        tma.append(('Q', x, i))
                if t >= 2:
                    yield from wait(f'v_empty{s}', (t >> 1) - 1)
                    if not {(0, t - 2), (1, t - 2)} <= st['pv_done']:
                        raise ProtocolError('V stage reloaded while still read')
                tma.append(('V', s, t))
                t += 1
                yield 'step'

    def mma():
        t = 0
        for i, n in enumerate(nkts):
            for x in range(2):
                yield from wait(f'q_full{x}', i)

            def issue_s(x, tt, last):
                if tt > 0 and 'o_done_before_s' not in drop:
                    yield from wait(f'o_done{x}', tt - 1)
                if tt > 0 and (x, tt - 1) not in st['pv_done']:
                    raise ProtocolError('S overwrites a P whose product has not run')
                if x == 0:
                    yield from wait(f'k_full{tt & 1}', tt >> 1)
                tc.append(('S', x, tt, i))
                tc.append(('commit', f's_full{x}'))
                if x == 1:
                    tc.append(('commit', f'k_empty{tt & 1}'))
                if last:
                    tc.append(('commit', f'q_empty{x}'))

            def issue_pv(x, tt, j):
                yield from wait(f'p_full{x}', tt)
                if x == 0:
                    yield from wait(f'v_full{tt & 1}', tt >> 1)
                tc.append(('PV', x, tt, i, j))
                if x == 1:
                    tc.append(('commit', f'v_empty{tt & 1}'))
                tc.append(('commit', f'o_done{x}'))

            yield from issue_s(0, t, n == 1)
            yield from issue_s(1, t, n == 1)
            for j in range(n):
                tj = t + j
                more, last_next = j + 1 < n, j + 2 == n
                yield from issue_pv(0, tj, j)
                if more:
                    yield from issue_s(0, tj + 1, last_next)
                yield from issue_pv(1, tj, j)
                if more:
                    yield from issue_s(1, tj + 1, last_next)
                yield 'step'
            t += n

    def softmax(x):
        t = 0
        for i, n in enumerate(nkts):
            for j in range(n):
                yield from wait(f's_full{x}', t)
                if st['S'][x] != t:
                    raise ProtocolError('softmax read a stale S')
                yield 'step'
                if rng.random() < 0.3 and j > 0:   # a rescale of O: no wait
                    if st['O'][x] != i or (x, t - 1) not in st['pv_done']:
                        raise ProtocolError('rescaled an O that is not up to date')
                if st['S'][x] != t:
                    raise ProtocolError('S overwritten before P was stored')
                st['P'][x] = t
                bars[f'p_full{x}'].arrive()
                t += 1
            if 'softmax_o_final' not in drop:
                yield from wait(f'o_done{x}', t - 1)
            want = set(range(t - n, t))
            if st['O'][x] != i or st['O_tiles'][x] != want:
                raise ProtocolError('read the wrong O')
            yield 'step'
            if st['O'][x] != i or st['O_tiles'][x] != want:
                raise ProtocolError('O changed while being read')
            st['o_read'][x].add(i)

    def run_tma():
        kind, s, v = tma.pop(0)
        st[kind][s] = v
        bars[f'{kind.lower()}_full{s}'].arrive()

    def run_tc():
        op = tc.pop(0)
        if op[0] == 'S':
            _, x, tt, i = op
            if st['Q'][x] != i or st['K'][tt & 1] != tt:
                raise ProtocolError('S product read a stale Q or K')
            st['S'][x] = tt
            st['P'][x] = None
            st['s_done'].add((x, tt))
        elif op[0] == 'PV':
            _, x, tt, i, j = op
            if st['P'][x] != tt or st['V'][tt & 1] != tt:
                raise ProtocolError('P V product read a stale P or V')
            if j == 0:
                if i > 0 and i - 1 not in st['o_read'][x]:
                    raise ProtocolError('O overwritten before it was read')
                st['O'][x], st['O_tiles'][x] = i, set()
            st['O_tiles'][x].add(tt)
            st['pv_done'].add((x, tt))
        else:
            bars[op[1]].arrive()

    actors = {'producer': producer(), 'mma': mma(), 'a': softmax(0), 'b': softmax(1)}
    rate = {a: rng.choice([0.05, 0.3, 1.0]) for a in list(actors) + ['tma', 'tc']}
    finished, idle = set(), 0
    while len(finished) < len(actors):
        moved = False
        names = [a for a in actors if a not in finished]
        rng.shuffle(names)
        for a in names:
            if rng.random() >= rate[a]:
                continue
            try:
                moved |= next(actors[a]) != 'blocked'
            except StopIteration:
                finished.add(a)
                moved = True
        if tma and rng.random() < rate['tma']:
            run_tma()
            moved = True
        if tc and rng.random() < rate['tc']:
            run_tc()
            moved = True
        idle = 0 if moved else idle + 1
        if idle > 2000:
            raise ProtocolError(f'deadlock; finished: {sorted(finished)}')
    while tc:
        run_tc()
    if any(len(r) != len(nkts) for r in st['o_read']):
        raise ProtocolError('an item was never written out')


def test_dual_protocol_holds_under_random_schedules():
    for nkts, seed in _cases(400):
        simulate_dual(nkts, seed)


@pytest.mark.parametrize('drop', ['o_done_before_s', 'softmax_o_final', 'q_empty', 'k_empty'])
def test_dual_dropping_a_wait_is_caught(drop):
    with pytest.raises(ProtocolError):
        for nkts, seed in _cases(400):
            simulate_dual(nkts, seed, drop=(drop,))
