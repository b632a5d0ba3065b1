"""Barrier protocol of the persistent state builder (`tc_build`), on the CPU.

A step-by-step model of every role of the kernel, with its ring sizes,
barrier counts and phase arithmetic:
- the TMA producer, which loads key/value tiles into a ring of 5;
- the two MMA issuers, which take alternate stages (32-token stages of every
  tile; for an item with a single accumulator tile, 128-token stages of two
  tiles) and commit the A slot, the tiles and, per work item, `done` (an
  issuer with no stage in an item arrives on `done` instead: a commit must
  follow an MMA of the same thread, which the model checks);
- the 8 generation warps, which write the products of each stage into a ring
  of 3 A slots in tensor memory and, after each item, drain the accumulators
  to the staging buffer once the previous item's store has released it;
- the store warp, which stores each staged item and releases the buffer.

It runs over sequences of work items with ragged token-tile counts (a short
last segment, single-tile items).  TMA loads and MMA commits complete at
random later times (one issuer's commits in order) and the roles interleave
at random, each at its own random speed.  Checked: no deadlock, and every wait observes exactly the phase
it intends.  Planted mistakes (the drain not waiting for the staging buffer,
an issuer waiting for the wrong A-slot phase) must be caught.
"""
import random

import pytest

from tests.test_readout_protocol import Bar, ProtocolError

KERNEL = dict(kBTileRing=5, kBARing=3, kGenWarps=8)


def item_stages(n_tt, wide):
    """32-token stages of an item (two per 64-token tile), or for a wide item
    (a single accumulator tile) 128-token stages of up to two tiles."""
    return (n_tt + 1) // 2 if wide else 2 * n_tt


def simulate(items_ntt, seed, prm, planted=None):
    """items_ntt: per work item its token-tile count, or (count, wide)."""
    items = [x if isinstance(x, tuple) else (x, False) for x in items_ntt]
    R, A, n_gen = prm["kBTileRing"], prm["kBARing"], prm["kGenWarps"]
    rng = random.Random(seed)
    B = {}
    for x in range(R):
        B[f"tfull{x}"], B[f"tempty{x}"] = Bar(1), Bar(2)
    for x in range(A):
        B[f"afull{x}"], B[f"aempty{x}"] = Bar(32 * n_gen), Bar(1)
    B.update(done=Bar(2), staged=Bar(32 * n_gen), sfree=Bar(1), drain0=Bar(1), drain1=Bar(1))
    n_items = len(items)
    issued = {0: False, 1: False}  # whether an issuer has any MMA before a commit
    inflight = {0: [], 1: []}  # (sequence, item) of each issuer's MMAs not yet covered by a landed commit
    seq = {0: 0, 1: 0}

    def W(name, k):  # wait for phase k of `name` (k = -1: the fresh barrier's previous phase)
        return ("wait", name, k)

    def producer():
        tt = 0
        for n_tt, _ in items:
            for _ in range(n_tt):
                yield W(f"tempty{tt % R}", tt // R - 1)
                yield ("load", f"tfull{tt % R}", 2)  # keys^T and values
                tt += 1

    def issuer(me):
        tt = ns = 0
        for j, (n_tt, wide) in enumerate(items):
            mine = 0
            for s in range(item_stages(n_tt, wide)):
                g = ns + s
                if g % 2 != me:
                    continue
                a = g % A
                tiles = [tt + 2 * s + x for x in range(2) if 2 * s + x < n_tt] if wide else [tt + s // 2]
                for t in tiles:
                    yield W(f"tfull{t % R}", t // R)
                # planted: the wait one phase early (it would pass on the slot's previous fill)
                yield W(f"afull{a}", g // A - 1 if planted == "issuer_phase" else g // A)
                yield ("mma", me, j)
                yield ("commit", f"aempty{a}")
                for t in tiles:  # each tile takes two arrivals: one per 32-token half
                    for _ in range(2 if wide else 1):
                        yield ("commit", f"tempty{t % R}")
                mine += 1
            # an issuer with no stage in the item arrives on `done` itself (a
            # commit with no MMA of its own to track is not relied on), once
            # its commit for the previous item has landed: an arrival before
            # that would complete the previous item's phase early, while its
            # MMAs still run.  Planted: the arrival without that wait.
            if mine:
                yield ("commit", "done")
            else:
                if j > 0 and planted != "idle_arrive_early":
                    yield W("done", j - 1)
                yield ("arrive", "done", 1)
            tt += n_tt
            ns += item_stages(n_tt, wide)
        if issued[me]:
            yield ("commit", f"drain{me}")
            yield W(f"drain{me}", 0)

    def gen(w):
        tt = ns = 0
        wg = w // (n_gen // 2)
        for j, (n_tt, wide) in enumerate(items):
            if wide:
                for s in range(item_stages(n_tt, wide)):
                    g = ns + s
                    a = g % A
                    t = tt + 2 * s + wg  # this warpgroup's tile of the stage, if any
                    if 2 * s + wg < n_tt:
                        yield W(f"tfull{t % R}", t // R)
                    yield W(f"aempty{a}", g // A - 1)
                    yield ("arrive", f"afull{a}", 32)
            else:
                yield W(f"tfull{tt % R}", tt // R)
                for t in range(n_tt):
                    for half in range(2):
                        g = ns + 2 * t + half
                        a = g % A
                        yield W(f"aempty{a}", g // A - 1)
                        if half == 1 and t + 1 < n_tt:
                            yield W(f"tfull{(tt + t + 1) % R}", (tt + t + 1) // R)
                        yield ("arrive", f"afull{a}", 32)
            tt += n_tt
            ns += item_stages(n_tt, wide)
            yield W("done", j)
            if j > 0 and planted != "drain_no_sfree":
                yield W("sfree", j - 1)
            yield ("write_stage", j)  # the drain: accumulators -> staging buffer
            yield ("arrive", "staged", 32)

    def storer():
        for j in range(n_items):
            yield W("staged", j)
            yield ("read_stage", j)  # the store reads the staging buffer
            yield ("arrive", "sfree", 1)

    agents = {"prod": producer(), "iss0": issuer(0), "iss1": issuer(1), "store": storer()}
    agents.update({f"gen{w}": gen(w) for w in range(n_gen)})
    cur = dict.fromkeys(agents)
    # each role runs at its own random speed, so that some runs starve one of
    # them (a slow store warp, a slow issuer) and others race ahead
    role_speed = {r: rng.choice((0.02, 0.2, 1.0)) for r in ("prod", "iss0", "iss1", "store", "gen")}
    speed = {a: role_speed["gen" if a.startswith("gen") else a] for a in agents}
    loads, commits = [], {"iss0": [], "iss1": []}
    # the staging buffer: which item's rows it holds, and which item the store
    # has finished reading; a drain may overwrite it only once the store of
    # the previous item has read it
    stage = {"item": -1, "read": -1}
    while True:
        runnable = [a for a, g in agents.items() if g is not None and
                    (cur[a] is None or B[cur[a][1]].done(cur[a][2] & 1))]
        pending = len(loads) + len(commits["iss0"]) + len(commits["iss1"])
        if not runnable and not pending:
            if all(g is None for g in agents.values()):
                return
            raise ProtocolError(f"deadlock: {[(a, cur[a]) for a in agents if agents[a] is not None]}")
        # a role is ready this step with the probability of its speed; a slow
        # role's turn passes to the copies and MMAs in flight or to faster roles
        ready = [x for x in runnable if rng.random() < speed[x]]
        if pending and (not ready or rng.random() < 0.4):
            choice = rng.choice((["load"] if loads else []) + [a for a in commits if commits[a]])
            if choice == "load":
                bar = B[loads.pop(rng.randrange(len(loads)))]
                bar.tx -= 1
                bar.flip()
            else:
                # a landed commit covers every earlier MMA of its issuer
                name, upto = commits[choice].pop(0)
                B[name].arrive()
                m = int(choice[-1])
                inflight[m] = [x for x in inflight[m] if x[0] >= upto]
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
        if act[0] == "wait":
            if B[act[1]].phase not in (act[2], act[2] + 1):
                raise ProtocolError(f"{a} waits on {act[1]} two phases behind")
            cur[a] = act
        elif act[0] == "write_stage":
            if any(act[1] == it for m in (0, 1) for _, it in inflight[m]):
                raise ProtocolError(f"drain of item {act[1]} while its MMAs run")
            if stage["read"] < act[1] - 1:
                raise ProtocolError(f"drain of item {act[1]} overwrote item {act[1] - 1} before its store read it")
            stage["item"] = max(stage["item"], act[1])
        elif act[0] == "read_stage":
            if stage["item"] != act[1]:
                raise ProtocolError(f"store of item {act[1]} read the rows of item {stage['item']}")
            stage["read"] = act[1]
        elif act[0] == "mma":
            issued[act[1]] = True
            inflight[act[1]].append((seq[act[1]], act[2]))
            seq[act[1]] += 1
        elif act[0] == "arrive":
            B[act[1]].arrive(act[2])
        elif act[0] == "load":  # arrive.expect_tx, then the bytes land later
            B[act[1]].tx += act[2]
            B[act[1]].arrive()
            loads.extend([act[1]] * act[2])
        else:
            if not issued[int(a[-1])]:
                raise ProtocolError(f"{a} commits {act[1]} before issuing any MMA")
            commits[a].append((act[1], seq[int(a[-1])]))


# token tiles per work item, as one CTA walks them: full 1024-token segments
# (16 tiles of 64), a ragged last segment, single-tile segments, and runs
# longer than the rings
CASES = [[16, 16, 16], [16, 3, 16, 1], [1, 1, 1, 1, 1, 1], [2, 16, 5, 7, 16, 1, 4], [16], [4, 4],
         # wide items (one accumulator tile, 128-token stages), mixed with the others,
         # with odd tile counts and single-stage items (one issuer idle in the item)
         [16, 16, (16, True), 16, 16, (16, True)], [(1, True), 16, (2, True), (3, True), 5],
         [(16, True), (1, True), (16, True)], [(2, True)], [(1, True), (1, True), 3]]


def test_build_protocol_is_deadlock_free_and_phase_exact():
    for seed in range(12):
        for c, items in enumerate(CASES):
            simulate(items, 100 * seed + c, KERNEL)


@pytest.mark.parametrize("mistake", ["drain_no_sfree", "issuer_phase", "idle_arrive_early"])
def test_model_catches_planted_mistakes(mistake):
    with pytest.raises(ProtocolError):
        for seed in range(40):
            for c, items in enumerate(CASES):
                simulate(items, 100 * seed + c, KERNEL, planted=mistake)
