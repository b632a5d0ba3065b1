"""Barrier protocol of the persistent tensor-core readout (`tc_read`), on the CPU.

A step-by-step model of every role of the kernel -- TMA producer, the two MMA
issuers (alternate inter stages; in the intra phase, steps (key block b, tile
t) b-major on three score buffers shared round-robin by the tiles: issuer 0
forms a step's scores once the buffer's previous step has finished its
weights times values, issuer 1 multiplies the step's weights, written over its
scores, by the values), the output-store warp and the squaring warps -- with
the same ring sizes, barrier counts and phase arithmetic as the kernel, run
over sequences of work items (ragged tails, empty second tiles,
single-segment heads, several items per CTA, the quadratic form's
longest-first order, and first-segment items with an inter phase when the
forward starts from a given state).  TMA loads and MMA commits complete
asynchronously at random later times (one issuer's commits in order), and
the roles interleave at random, each at its own random speed.  Checked: no
deadlock, every wait observes exactly the phase it intends (a barrier never
runs two phases past a waiter, which a parity wait could not tell apart:
each tile waits on only some phases of a buffer's barrier), and no step's
scores are issued into a buffer whose previous step's products are still
running, and no key or value block is loaded over one whose scores or
products are still running.  Planted mistakes must be caught: a score buffer taking new scores
without waiting for its previous step's products, and both item slots'
outputs staged on one barrier (a real hazard of an earlier version of the
kernel, found by this model once each role ran at its own speed).  The same
model runs the KATA-Mg two-factor configuration (9 inter stages, 64-key
steps, rings of 6 key and 6 value blocks) and the configuration of
single-factor heads of d <= 32 (9 inter stages, 128-key steps).
"""
import random

import pytest

KERNEL = dict(kQT=128, kTiles=2, kKB=128, kKVRing=3, kRStages=17, kRRing=3, kRBRing=4,
              kItemSlots=2, kSBufs=3)
# KATA-Mg with two factors: 9 inter stages, and 64-key steps (both factors'
# scores side by side in a buffer) in a ring of 4 key/value blocks
KERNEL_M2 = dict(KERNEL, kRStages=9, kKB=64, kKVRing=6)
# A single-factor head of d <= 32 on the two-factor layout: 9 inter stages,
# the single factor's 128-key steps
KERNEL_SMALL = dict(KERNEL, kRStages=9)


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
    kQT, kTiles, kKB, kS = prm['kQT'], prm['kTiles'], prm['kKB'], prm['kSBufs']
    kKVRing, kRStages, kRRing, kRBRing, kSlots = (prm['kKVRing'], prm['kRStages'], prm['kRRing'],
                                                  prm['kRBRing'], prm['kItemSlots'])
    kCtaQ, kGen = kQT * kTiles, 4 * kTiles
    rng = random.Random(seed)
    n_ct = (T + kCtaQ - 1) // kCtaQ
    B = {}
    for b in range(kSlots):
        B[f'qfull{b}'], B[f'qempty{b}'] = Bar(1), Bar(3)
    for b in range(kKVRing):
        for r in 'kv':  # key and value rings apart; released by plain arrivals
            B[f'{r}full{b}'], B[f'{r}empty{b}'] = Bar(1), Bar(1)
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
    for x in range(kS):  # score buffers, shared round-robin by the tiles' steps
        B[f'sfull{x}'], B[f'pfull{x}'], B[f'bfree{x}'] = Bar(1), Bar(4), Bar(1)
    pv_done = set()  # steps whose weights times values have completed
    qk_done = set()  # steps whose scores have completed
    block_steps = {}  # key/value block -> its steps

    def item(i):
        t0 = (i % n_ct) * kCtaQ
        seg0 = (t0 // L) * L
        return dict(t0=t0, seg0=seg0, inter=seg0 > 0 or init,
                    n_kv=(min(t0 + kCtaQ, T) - seg0 + kKB - 1) // kKB)

    def blocks(it, t):
        q0 = it['t0'] + kQT * t
        return 0 if q0 >= T else (min(q0 + kQT, T) - it['seg0'] + kKB - 1) // kKB

    def before(b, t, nb):  # steps of the item before step (b, t), b-major
        return min(b, nb[0]) + min(b, nb[1]) + (1 if t == 1 and b < nb[0] else 0)

    def W(name, k):  # wait for phase k (k = -1: the fresh barrier's "previous" phase)
        return ('wait', name, k)

    def producer():
        n_q = n_bs = n_kv = 0
        for i in items:
            it = item(i)
            qb = n_q % kSlots
            yield W(f'qempty{qb}', n_q // kSlots - 1)
            yield ('load', f'qfull{qb}', kTiles)
            n_q += 1
            for _ in range(1 + kRStages if it['inter'] else 0):  # Z hi / lo, then the stages
                s = n_bs % kRBRing
                yield W(f'bempty{s}', n_bs // kRBRing - 1)
                yield ('load', f'bfull{s}', 1)
                n_bs += 1
            for _ in range(it['n_kv']):
                s = n_kv % kKVRing
                yield W(f'kempty{s}', n_kv // kKVRing - 1)
                yield ('load', f'kfull{s}', 1, n_kv)
                yield W(f'vempty{s}', n_kv // kKVRing - 1)
                yield ('load', f'vfull{s}', 1, n_kv)
                n_kv += 1

    def issuer(me):
        n_inter = g_kv = ns = 0
        vrel = [None] * kS  # per buffer: the slot whose values its step finishes reading
        for j, i in enumerate(items):
            it = item(i)
            qb = j % kSlots
            yield W(f'qfull{qb}', j // kSlots)
            if it['inter']:
                if me == 0:
                    if j > 0:
                        yield W('done', j - 1)
                    ze = n_inter * (kRStages + 1)  # Z hi / lo: the item's first prefix entry
                    yield W(f'bfull{ze % kRBRing}', ze // kRBRing)
                    yield ('commit', 'u')
                    yield ('commit', f'bempty{ze % kRBRing}')
                for st in range(me, kRStages, 2):
                    G, E = n_inter * kRStages + st, n_inter * (kRStages + 1) + 1 + st
                    yield W(f'afull{G % kRRing}', G // kRRing)
                    yield W(f'bfull{E % kRBRing}', E // kRBRing)
                    yield ('commit', f'bempty{E % kRBRing}')
                    yield ('commit', f'aempty{G % kRRing}')
                yield ('commit', 'interdone')
                yield W('interdone', n_inter)
                n_inter += 1
            nb = [blocks(it, t) for t in range(kTiles)]
            for b in range(max(nb)):
                G = g_kv + b
                if me == 0:  # issuer 1 learns of the values from the squaring warps
                    yield W(f'kfull{G % kKVRing}', G // kKVRing)
                for t in range(kTiles):
                    if b >= nb[t]:
                        continue
                    n, x = ns + before(b, t, nb), (ns + before(b, t, nb)) % kS
                    if me == 0:
                        # the buffer's previous step must have finished its products
                        # (planted: not waited for)
                        if n >= kS and not planted:
                            yield W(f'bfree{x}', (n - kS) // kS)
                            if vrel[x] is not None:  # step n - 3 ended its block: values read
                                yield ('arrive', f'vempty{vrel[x]}', 1)
                        vrel[x] = G % kKVRing if (t == 1 or b >= nb[1]) else None
                        yield ('qk', n, G)
                        yield ('commit', (f'sfull{x}', ('qk', n)))
                    else:
                        yield W(f'pfull{x}', n // kS)
                        yield ('mma',)
                        yield ('commit', (f'bfree{x}', ('pv', n)))
            g_kv += it['n_kv']
            ns += nb[0] + nb[1]
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
        t, n_inter, ns, g_kv = w // 4, 0, 0, 0
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
            nb = [blocks(it, 0), blocks(it, 1)]
            for b in range(nb[t]):
                n = ns + before(b, t, nb)
                yield W(f'sfull{n % kS}', n // kS)
                G = g_kv + b
                if w % 4 == 0 and (t == 1 or b >= nb[1]):  # the block's last scores: keys read
                    yield ('arrive', f'kempty{G % kKVRing}', 1)
                # the block's values landed, then the weights are handed over
                yield W(f'vfull{G % kKVRing}', G // kKVRing)
                yield ('arrive', f'pfull{n % kS}', 1)  # weights stored over the scores
            ns += nb[0] + nb[1]
            g_kv += it['n_kv']
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
                c = commits[choice].pop(0)
                if isinstance(c, tuple):  # the scores or products of a step are complete
                    c, (kind, step) = c
                    (qk_done if kind == 'qk' else pv_done).add(step)
                B[c].arrive()
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
            if len(act) > 3 and act[3] >= kKVRing:  # a key or value block into a used slot
                old = block_steps.get(act[3] - kKVRing, [])
                done_set = qk_done if act[1].startswith('k') else pv_done
                if len(old) < len(set(old)) or any(n not in done_set for n in old) or not old:
                    raise ProtocolError(f"block {act[3]} loaded over block {act[3] - kKVRing} "
                                        f"while MMAs still read its {'keys' if act[1][0] == 'k' else 'values'}")
            B[act[1]].tx += act[2]
            B[act[1]].arrive()
            loads.extend([act[1]] * act[2])
        elif act[0] == 'qk':
            n = act[1]
            block_steps.setdefault(act[2], []).append(n)
            if n >= kS and n - kS not in pv_done:
                raise ProtocolError(f"scores of step {n} issued over step {n - kS}'s weights "
                                    "before its products finished")
        elif act[0] == 'mma':
            pass
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


def test_model_catches_a_score_buffer_reused_before_its_products():
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


def test_model_catches_a_two_factor_score_buffer_reused_before_its_products():
    with pytest.raises(ProtocolError):
        run_cases(KERNEL_M2, seeds=range(4), planted=True)


def test_small_head_readout_protocol():
    # single-factor heads of d <= 32: the two-factor layout's 9 inter stages
    # with the single factor's 128-key intra steps
    run_cases(KERNEL_SMALL, seeds=range(2))
    cq = KERNEL_SMALL['kQT'] * KERNEL_SMALL['kTiles']
    for T, L, BH, grid in CASES[:4]:
        n_items = (T + cq - 1) // cq * BH
        g = min(grid, n_items)
        for c in range(g):
            simulate(T, L, BH, list(range(c * n_items // g, (c + 1) * n_items // g)), 19 * T + c,
                     KERNEL_SMALL, init=True)
