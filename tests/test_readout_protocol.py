"""Barrier protocol of the persistent tensor-core readout (`tc_read`), on the CPU.

A step-by-step model of every role of the kernel -- TMA producer, the two MMA
issuers (alternate inter stages; scores Q K^T by issuer 0, reusing a score
buffer once the squaring warps have loaded it; weights times values by issuer
1), the output-store warp and the squaring warps -- with the same
ring sizes, barrier counts and phase arithmetic as the kernel, run over
sequences of work items (ragged tails, empty second tiles, single-segment
heads, several items per CTA, the quadratic form's longest-first order, and
first-segment items with an inter phase when the forward starts from a given
state).  TMA loads and MMA commits complete
asynchronously at random later times (one issuer's commits in order), and the
roles interleave at random, each at its own random speed.  Checked: no deadlock, and every wait observes
exactly the phase it intends (a barrier never runs two phases past a waiter,
which a parity wait could not tell apart).  Planted mistakes must be caught:
the score buffer reused across work items without waiting for its last
reader, and both item slots' outputs staged on one barrier (a real hazard of
an earlier version of the kernel, found by this model once each role ran at
its own speed).  The same model runs the KATA-Mg two-factor configuration
(9 inter stages, one score buffer per tile).
"""
import random

import pytest

KERNEL = dict(kQT=128, kTiles=2, kSB=64, kKB=64, kKVRing=4, kRStages=17, kRRing=3, kRBRing=4,
              kItemSlots=2, kSDepth=2)
# KATA-Mg with two factors: 9 inter stages, and one score buffer per tile
# (both factors' scores side by side), so a tile's next scores wait for the
# squaring warps to read the previous block
KERNEL_M2 = dict(KERNEL, kRStages=9, kSDepth=1)


class ProtocolError(AssertionError):
    pass


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase, self.tx = count, count, 0, 0

    def arrive(self, n=1):
        self.pending -= n
        if self.pending < 0:
            raise ProtocolError("too many arrivals")
        self.flip()

    def flip(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        return (self.phase & 1) != parity


def simulate(T, L, BH, items, seed, prm, planted=False, init=False, one_ostaged=False):
    kQT, kTiles, kSB, kKB = prm['kQT'], prm['kTiles'], prm['kSB'], prm['kKB']
    kKVRing, kRStages, kRRing, kRBRing, kSlots = (prm['kKVRing'], prm['kRStages'], prm['kRRing'],
                                                  prm['kRBRing'], prm['kItemSlots'])
    kCtaQ, kHalves, kGen, D = kQT * kTiles, kKB // kSB, 4 * kTiles, prm['kSDepth']
    rng = random.Random(seed)
    n_ct = (T + kCtaQ - 1) // kCtaQ
    B = {}
    for b in range(kSlots):
        B[f'qfull{b}'], B[f'qempty{b}'] = Bar(1), Bar(3)
    for b in range(kKVRing):
        B[f'kvfull{b}'], B[f'kvempty{b}'] = Bar(1), Bar(2)
    B.update(u=Bar(1), interdone=Bar(2), done=Bar(2), genin=Bar(kGen), drain0=Bar(1),
             drain1=Bar(1))
    for b in range(kSlots):  # output rows staged in item slot b
        B[f'ostaged{b}'] = Bar(kGen)
    # planted: one barrier for both slots (it may complete twice ahead of the store warp)
    osb = (lambda j: 'ostaged0') if one_ostaged else (lambda j: f'ostaged{j % kSlots}')
    osk = (lambda j: j) if one_ostaged else (lambda j: j // kSlots)
    for s in range(kRBRing):
        B[f'bfull{s}'], B[f'bempty{s}'] = Bar(1), Bar(1)
    for s in range(kRRing):
        B[f'afull{s}'], B[f'aempty{s}'] = Bar(kGen * 32), Bar(1)
    for t in range(kTiles):
        for x in range(2):
            B[f'pfull{t}{x}'], B[f'pempty{t}{x}'] = Bar(128), Bar(1)
        for x in range(D):
            B[f'sfull{t}{x}'], B[f'sload{t}{x}'] = Bar(1), Bar(128)

    def item(i):
        t0 = (i % n_ct) * kCtaQ
        seg0 = (t0 // L) * L
        return dict(t0=t0, seg0=seg0, inter=seg0 > 0 or init,
                    n_kv=(min(t0 + kCtaQ, T) - seg0 + kKB - 1) // kKB)

    def blocks(it, t):
        q0 = it['t0'] + kQT * t
        return 0 if q0 >= T else (min(q0 + kQT, T) - it['seg0'] + kSB - 1) // kSB

    def W(name, k):  # wait for phase k (k = -1: the fresh barrier's "previous" phase)
        return ('wait', name, k)

    def producer():
        n_q = n_bs = n_kv = 0
        for i in items:
            it = item(i)
            qb = n_q % kSlots
            yield W(f'qempty{qb}', n_q // kSlots - 1)
            yield ('load', f'qfull{qb}', kTiles + it['inter'])
            n_q += 1
            for _ in range(kRStages if it['inter'] else 0):
                s = n_bs % kRBRing
                yield W(f'bempty{s}', n_bs // kRBRing - 1)
                yield ('load', f'bfull{s}', 1)
                n_bs += 1
            for _ in range(it['n_kv']):
                s = n_kv % kKVRing
                yield W(f'kvempty{s}', n_kv // kKVRing - 1)
                yield ('load', f'kvfull{s}', 2)
                n_kv += 1

    def issuer(me):
        n_inter = g_kv = 0
        g_b = [0] * kTiles
        for j, i in enumerate(items):
            it = item(i)
            qb = j % kSlots
            yield W(f'qfull{qb}', j // kSlots)
            if it['inter']:
                if me == 0:
                    if j > 0:
                        yield W('done', j - 1)
                    yield ('commit', 'u')
                for st in range(me, kRStages, 2):
                    G = n_inter * kRStages + st
                    yield W(f'bfull{G % kRBRing}', G // kRBRing)
                    yield W(f'afull{G % kRRing}', G // kRRing)
                    yield ('commit', f'bempty{G % kRBRing}')
                    yield ('commit', f'aempty{G % kRRing}')
                yield ('commit', 'interdone')
                yield W('interdone', n_inter)
                n_inter += 1
            nb = [blocks(it, t) for t in range(kTiles)]
            gb, nbm = list(g_b), max(nb)
            for b in range(nbm):
                G, h = g_kv + b // kHalves, b % kHalves
                if h == 0:
                    yield W(f'kvfull{G % kKVRing}', G // kKVRing)
                for t in range(kTiles):
                    if b < nb[t]:
                        reuse = (b >= D) if planted else (gb[t] + b >= D)
                        if me == 0 and reuse:  # the squaring warps have loaded block n - D
                            yield W(f'sload{t}{(gb[t] + b - D) % D}', (gb[t] + b - D) // D)
                        if me == 1:
                            yield W(f'pfull{t}{(gb[t] + b) & 1}', (gb[t] + b) >> 1)
                for t in range(kTiles):
                    if b < nb[t]:
                        n = gb[t] + b
                        yield ('commit', f'sfull{t}{n % D}' if me == 0 else f'pempty{t}{n & 1}')
                if h == kHalves - 1 or b == nbm - 1:
                    yield ('commit', f'kvempty{G % kKVRing}')
            g_kv += it['n_kv']
            for t in range(kTiles):
                g_b[t] += nb[t]
            yield W('genin', j)
            yield ('commit', 'done')
            yield ('commit', f'qempty{qb}')
        yield ('commit', f'drain{me}')
        yield W(f'drain{me}', 0)

    def storer():
        for j in range(len(items)):
            yield W(osb(j), osk(j))
            yield ('arrive', f'qempty{j % kSlots}', 1)

    def gen(w):
        t, n_inter, g_b = w // 4, 0, 0
        for j, i in enumerate(items):
            it = item(i)
            yield ('arrive', 'genin', 1)
            yield W(f'qfull{j % kSlots}', j // kSlots)
            if it['inter']:
                yield W('u', n_inter)
                for st in range(kRStages):
                    G = n_inter * kRStages + st
                    yield W(f'aempty{G % kRRing}', G // kRRing - 1)
                    yield ('arrive', f'afull{G % kRRing}', 32)
                n_inter += 1
            for b in range(blocks(it, t)):
                n = g_b + b
                yield W(f'sfull{t}{n % D}', n // D)
                yield ('arrive', f'sload{t}{n % D}', 32)
                yield W(f'pempty{t}{n & 1}', (n >> 1) - 1)
                yield ('arrive', f'pfull{t}{n & 1}', 32)
            g_b += blocks(it, t)
            yield W('done', j)
            yield ('arrive', osb(j), 1)

    agents = {'prod': producer(), 'iss0': issuer(0), 'iss1': issuer(1), 'store': storer()}
    agents.update({f'gen{w}': gen(w) for w in range(kGen)})
    cur = dict.fromkeys(agents)
    # each role runs at its own random speed (the squaring warps share one), so
    # some runs starve a role and let the others race ahead of it
    role_speed = {r: rng.choice((0.02, 0.2, 1.0)) for r in ('prod', 'iss0', 'iss1', 'store', 'gen')}
    speed = {a: role_speed['gen' if a.startswith('gen') else a] for a in agents}
    loads, commits = [], {'iss0': [], 'iss1': []}
    while True:
        runnable = [a for a, g in agents.items() if g is not None and
                    (cur[a] is None or B[cur[a][1]].done(cur[a][2] & 1))]
        pending = len(loads) + len(commits['iss0']) + len(commits['iss1'])
        if not runnable and not pending:
            if all(g is None for g in agents.values()):
                return
            raise ProtocolError(f"deadlock: {[(a, cur[a]) for a in agents if agents[a] is not None]}")
        ready = [x for x in runnable if rng.random() < speed[x]]
        if pending and (not ready or rng.random() < 0.4):
            choice = rng.choice((['load'] if loads else []) + [a for a in commits if commits[a]])
            if choice == 'load':
                bar = B[loads.pop(rng.randrange(len(loads)))]
                bar.tx -= 1
                bar.flip()
            else:
                B[commits[choice].pop(0)].arrive()
            continue
        a = rng.choice(ready or runnable)
        if cur[a] is not None and B[cur[a][1]].phase != cur[a][2] + 1:
            raise ProtocolError(f"{a} woke on the wrong phase of {cur[a][1]}")
        try:
            act = next(agents[a])
        except StopIteration:
            agents[a], cur[a] = None, None
            continue
        cur[a] = None
        if act[0] == 'wait':
            if B[act[1]].phase not in (act[2], act[2] + 1):
                raise ProtocolError(f"{a} waits on {act[1]} two phases behind")
            cur[a] = act
        elif act[0] == 'arrive':
            B[act[1]].arrive(act[2])
        elif act[0] == 'load':  # arrive.expect_tx, then the bytes land later
            B[act[1]].tx += act[2]
            B[act[1]].arrive()
            loads.extend([act[1]] * act[2])
        else:
            commits[a].append(act[1])


CASES = [  # T, L, heads, CTAs
    (2300, 1024, 2, 4), (600, 1024, 160, 3), (130, 1024, 5, 1), (5000, 1024, 7, 5),
    (2048 + 129, 1024, 3, 2), (1152, 1024, 80, 7), (100, 1024, 9, 2),
]


def run_cases(prm, seeds, planted=False):
    cq = prm['kQT'] * prm['kTiles']
    for seed in seeds:
        for T, L, BH, grid in CASES:
            n_items = (T + cq - 1) // cq * BH
            g = min(grid, n_items)
            for c in range(g):
                simulate(T, L, BH, list(range(c * n_items // g, (c + 1) * n_items // g)),
                         1000 * seed + c, prm, planted)


QUADRATIC_CASES = [  # T, heads, CTAs (one segment: L = T)
    (2300, 2, 4), (600, 160, 3), (130, 5, 1), (5000, 3, 5), (1152, 80, 7), (257, 1, 1),
]


def quadratic_items(n_ct, BH, grid, c):
    """Items CTA c walks in the quadratic form: latest query tiles first, across
    heads, dealt round-robin to the CTAs."""
    return [(x % BH) * n_ct + (n_ct - 1 - x // BH) for x in range(c, n_ct * BH, grid)]


def test_readout_protocol_is_deadlock_free_and_phase_exact():
    run_cases(KERNEL, seeds=range(2))


def test_initial_state_gives_every_item_an_inter_phase():
    # a forward from a given state: first-segment items read a prefix too
    cq = KERNEL['kQT'] * KERNEL['kTiles']
    for T, L, BH, grid in CASES[:4]:
        n_items = (T + cq - 1) // cq * BH
        g = min(grid, n_items)
        for c in range(g):
            items = list(range(c * n_items // g, (c + 1) * n_items // g))
            simulate(T, L, BH, items, 11 * T + c, KERNEL, init=True)
        if T <= L:  # one segment: the longest-first order
            n_ct = (T + cq - 1) // cq
            for c in range(g):
                simulate(T, T, BH, quadratic_items(n_ct, BH, g, c), 13 * T + c, KERNEL, init=True)


def test_model_catches_one_output_barrier_for_both_slots():
    # the kernel once staged both slots' outputs on one barrier: with the store
    # warp slow, the squaring warps complete it twice before the store warp's
    # parity wait looks, which then never sees its phase
    cq = KERNEL['kQT'] * KERNEL['kTiles']
    with pytest.raises(ProtocolError):
        for seed in range(40):
            for T, BH, grid in QUADRATIC_CASES:
                n_ct = (T + cq - 1) // cq
                g = min(grid, n_ct * BH)
                for c in range(g):
                    simulate(T, T, BH, quadratic_items(n_ct, BH, g, c), 1000 * seed + 7 * T + c,
                             KERNEL, one_ostaged=True)


def test_quadratic_schedule_is_deadlock_free_and_phase_exact():
    cq = KERNEL['kQT'] * KERNEL['kTiles']
    for T, BH, grid in QUADRATIC_CASES:
        n_ct = (T + cq - 1) // cq
        g = min(grid, n_ct * BH)
        walked = []
        for c in range(g):
            items = quadratic_items(n_ct, BH, g, c)
            walked += items
            simulate(T, T, BH, items, 7 * T + c, KERNEL)
        assert sorted(walked) == list(range(n_ct * BH))  # every item exactly once


def test_model_catches_a_score_buffer_reused_across_items():
    with pytest.raises(ProtocolError):
        run_cases(KERNEL, seeds=range(4), planted=True)


def test_two_factor_readout_protocol():
    run_cases(KERNEL_M2, seeds=range(2))
    cq = KERNEL_M2['kQT'] * KERNEL_M2['kTiles']
    for T, L, BH, grid in CASES[:4]:
        n_items = (T + cq - 1) // cq * BH
        g = min(grid, n_items)
        for c in range(g):
            simulate(T, L, BH, list(range(c * n_items // g, (c + 1) * n_items // g)), 17 * T + c,
                     KERNEL_M2, init=True)


def test_model_catches_a_two_factor_score_buffer_reused_across_items():
    with pytest.raises(ProtocolError):
        run_cases(KERNEL_M2, seeds=range(4), planted=True)
