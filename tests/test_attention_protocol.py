"""Model check of the persistent prefill attention kernel's barrier protocol
(attention_tc.cu, attn_prefill_tc_persistent_kernel), run on the CPU.

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


# ------------------------------------------------------- two CTAs per SM
def simulate_2cta(nkts, seed, drop=()):
    """The barrier protocol of attn_prefill_tc_2cta_kernel: single-stage Q, K
    and V buffers; one S buffer whose upper half takes P; the MMA issuer waits
    for the previous P V product before the next S overwrites that P."""
    rng = random.Random(seed)
    bars = {n: Bar() for n in ('q_full', 'q_empty', 'k_full', 'k_empty', 'v_full', 'v_empty', 's_full', 'p_full',
                               'o_done')}
    st = dict(Q=None, K=None, V=None, S=None, P=None, O_item=None, O_tiles=set(), o_read=set(), pv_done=set(),
              s_done=set(), s_read=set())
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
            if i > 0 and 'q_empty' not in drop:
                yield from wait('q_empty', i - 1)
            tma.append(('Q', i))
            for _ in range(n):
                if t > 0:
                    yield from wait('k_empty', t - 1)
                tma.append(('K', t))
                if t > 0:
                    yield from wait('v_empty', t - 1)
                tma.append(('V', t))
                t += 1
                yield 'step'

    def mma():
        t = 0
        for i, n in enumerate(nkts):
            yield from wait('q_full', i)
            for j in range(n):
                if t > 0 and 'mma_o_done' not in drop:
                    yield from wait('o_done', t - 1)
                yield from wait('k_full', t)
                tc.extend([('S', t, i), ('commit', 's_full'), ('commit', 'k_empty')])
                if j + 1 == n:
                    tc.append(('commit', 'q_empty'))
                yield from wait('p_full', t)
                yield from wait('v_full', t)
                tc.extend([('PV', t, i, j), ('commit', 'v_empty'), ('commit', 'o_done')])
                t += 1
                yield 'step'

    def softmax():
        t = 0
        for i, n in enumerate(nkts):
            for j in range(n):
                yield from wait('s_full', t)
                if st['S'] != t:
                    raise ProtocolError('softmax read a stale S')
                if j > 0 and (st['O_item'] != i or t - 1 not in st['pv_done']):
                    raise ProtocolError('rescaled an O that is not up to date')
                yield 'step'
                if st['S'] != t:
                    raise ProtocolError('S overwritten while the softmax read it')
                st['s_read'].add(t)
                st['P'] = t
                bars['p_full'].arrive()
                t += 1
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
        op = tma.pop(0)
        kind, x = op
        if kind == 'Q':
            if x > 0 and not set(range(first[x - 1], first[x - 1] + nkts[x - 1])) <= st['s_done']:
                raise ProtocolError('Q reloaded while still read')
        elif kind == 'K':
            if x > 0 and x - 1 not in st['s_done']:
                raise ProtocolError('K reloaded while still read')
        elif x > 0 and x - 1 not in st['pv_done']:
            raise ProtocolError('V reloaded while still read')
        st[kind] = x
        bars[f'{kind.lower()}_full'].arrive()

    def run_tc():
        op = tc.pop(0)
        if op[0] == 'S':
            _, t, i = op
            if st['Q'] != i or st['K'] != t:
                raise ProtocolError('S product read a stale Q or K')
            if t > 0 and t - 1 not in st['pv_done']:
                raise ProtocolError('S overwrote a P before its product ran')
            if t > 0 and t - 1 not in st['s_read']:
                raise ProtocolError('S overwritten before it was read')
            st['S'] = t
            st['s_done'].add(t)
        elif op[0] == 'PV':
            _, t, i, j = op
            if st['P'] != t or st['V'] != t:
                raise ProtocolError('P V product read a stale P or V')
            if j == 0:
                if i > 0 and i - 1 not in st['o_read']:
                    raise ProtocolError('O overwritten before it was read')
                st['O_item'], st['O_tiles'] = i, set()
            st['O_tiles'].add(t)
            st['pv_done'].add(t)
        else:
            bars[op[1]].arrive()

    actors = {'producer': producer(), 'mma': mma(), 'softmax': softmax()}
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


def test_2cta_protocol_holds_under_random_schedules():
    for nkts, seed in _cases(400):
        simulate_2cta(nkts, seed)


# (The MMA issuer's wait for the previous P V product before the next S is
# not in this list: the model's tensor engine completes operations in issue
# order, which already keeps S behind that product; the wait keeps the kernel
# correct without relying on that order.)
@pytest.mark.parametrize('drop', ['softmax_o_final', 'q_empty'])
def test_2cta_dropping_a_wait_is_caught(drop):
    with pytest.raises(ProtocolError):
        for nkts, seed in _cases(400):
            simulate_2cta(nkts, seed, drop=(drop,))
