"""Barrier protocol of the persistent state builder (`tc_build`), on the CPU.

A step-by-step model of every role of the kernel, with its ring sizes,
barrier counts and phase arithmetic:
- the TMA producer, which loads key/value tiles into a ring of 5;
- the transposing warp, which transposes each key tile in place once it has
  landed and hands it to the generation warps;
- the two MMA issuers, which take alternate 32-token stages of every tile
  and commit the A slot, the tile and, per work item, `done`;
- the 8 generation warps, which write the products of each stage into a ring
  of 3 A slots in tensor memory and, after each item, drain the accumulators
  to the staging buffer once the previous item's store has released it;
- the store warp, which stores each staged item and releases the buffer.

It runs over sequences of work items with ragged token-tile counts (a short
last segment, single-tile items).  TMA loads and MMA commits complete at
random later times (one issuer's commits in order) and the roles interleave
at random, each at its own random speed.  Checked: no deadlock, every wait
observes exactly the phase it intends, no drain starts while an MMA of its
item runs, no issuer commits before it has issued an MMA (a commit with
nothing of its own to track is not relied on), no key tile is transposed
before it has landed, and no slot is refilled or rewritten while a generation
warp still reads its keys.  Planted mistakes (the drain not waiting for the
staging buffer, an issuer waiting for the wrong A-slot phase, a load not
waiting for its slot, a transpose not waiting for its keys) must be caught.
"""
import random

import pytest

from tests.test_readout_protocol import Bar, ProtocolError

KERNEL = dict(kBTileRing=5, kBARing=3, kGenWarps=8)


def simulate(items_ntt, seed, prm, planted=None):
    R, A, n_gen = prm["kBTileRing"], prm["kBARing"], prm["kGenWarps"]
    rng = random.Random(seed)
    B = {}
    for x in range(R):
        B[f"kraw{x}"], B[f"tfull{x}"], B[f"tempty{x}"] = Bar(1), Bar(32), Bar(2)
    for x in range(A):
        B[f"afull{x}"], B[f"aempty{x}"] = Bar(32 * n_gen), Bar(1)
    B.update(done=Bar(2), staged=Bar(32 * n_gen), sfree=Bar(1), drain0=Bar(1), drain1=Bar(1))
    n_items = len(items_ntt)
    issued = {0: False, 1: False}  # whether an issuer has any MMA before a commit
    inflight = {0: [], 1: []}  # (sequence, item) of each issuer's MMAs not yet covered by a landed commit
    seq = {0: 0, 1: 0}

    def W(name, k):  # wait for phase k of `name` (k = -1: the fresh barrier's previous phase)
        return ("wait", name, k)

    total = sum(items_ntt)
    readers = {}  # key tile -> generation warps reading it
    transposed = set()

    def loader():
        for tt in range(total):
            if planted != "load_no_tempty":
                yield W(f"tempty{tt % R}", tt // R - 1)
            yield ("load", tt)  # keys and values, landing on kraw

    def transposer():
        for tt in range(total):
            if planted != "transpose_early":
                yield W(f"kraw{tt % R}", tt // R)
            yield ("transpose", tt)
            yield ("arrive", f"tfull{tt % R}", 32)

    def issuer(me):
        tt = 0
        for j, n_tt in enumerate(items_ntt):
            for _ in range(n_tt):
                G = 2 * tt + me
                a = G % A
                yield W(f"kraw{tt % R}", tt // R)  # the values
                # planted: the wait one phase early (it would pass on the slot's previous fill)
                yield W(f"afull{a}", G // A - 1 if planted == "issuer_phase" else G // A)
                yield ("mma", me, j)
                yield ("commit", f"aempty{a}")
                yield ("commit", f"tempty{tt % R}")
                tt += 1
            yield ("commit", "done")
        yield ("commit", f"drain{me}")
        yield W(f"drain{me}", 0)

    def gen(w):
        tt = 0
        for j, n_tt in enumerate(items_ntt):
            yield W(f"tfull{tt % R}", tt // R)
            yield ("read_keys", tt)
            for t in range(n_tt):
                for half in range(2):
                    G = 2 * tt + half
                    a = G % A
                    yield W(f"aempty{a}", G // A - 1)
                    if half == 1 and t + 1 < n_tt:
                        yield W(f"tfull{(tt + 1) % R}", (tt + 1) // R)
                        yield ("read_keys", tt + 1)
                    if half == 0:  # both halves' products of the tile are formed
                        yield ("keys_read", tt)
                    yield ("arrive", f"afull{a}", 32)
                tt += 1
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

    agents = {"load": loader(), "trans": transposer(), "iss0": issuer(0), "iss1": issuer(1),
              "store": storer()}
    agents.update({f"gen{w}": gen(w) for w in range(n_gen)})
    cur = dict.fromkeys(agents)
    # each role runs at its own random speed, so that some runs starve one of
    # them (a slow store warp, a slow issuer) and others race ahead
    role_speed = {r: rng.choice((0.02, 0.2, 1.0)) for r in ("load", "trans", "iss0", "iss1", "store", "gen")}
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
        elif act[0] == "mma":
            issued[act[1]] = True
            inflight[act[1]].append((seq[act[1]], act[2]))
            seq[act[1]] += 1
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
        elif act[0] == "arrive":
            B[act[1]].arrive(act[2])
        elif act[0] == "load":  # arrive.expect_tx, then the keys and values land later
            tt = act[1]
            if readers.get(tt - R, 0):
                raise ProtocolError(f"tile {tt} loaded over tile {tt - R} while its keys are read")
            bar = f"kraw{tt % R}"
            B[bar].tx += 2
            B[bar].arrive()
            loads.extend([bar] * 2)
        elif act[0] == "transpose":
            tt = act[1]
            if B[f"kraw{tt % R}"].phase <= tt // R or B[f"kraw{tt % R}"].tx:
                raise ProtocolError(f"tile {tt} transposed before its keys landed")
            if readers.get(tt - R, 0):
                raise ProtocolError(f"tile {tt} transposed over tile {tt - R} while its keys are read")
            transposed.add(tt)
        elif act[0] == "read_keys":
            if act[1] not in transposed:
                raise ProtocolError(f"{a} reads the keys of tile {act[1]} before they are transposed")
            readers[act[1]] = readers.get(act[1], 0) + 1
        elif act[0] == "keys_read":
            readers[act[1]] -= 1
        else:
            if not issued[int(a[-1])]:
                raise ProtocolError(f"{a} commits {act[1]} before issuing any MMA")
            commits[a].append((act[1], seq[int(a[-1])]))


# token tiles per work item, as one CTA walks them: full 1024-token segments
# (16 tiles of 64), a ragged last segment, single-tile segments, and runs
# longer than the rings
CASES = [[16, 16, 16], [16, 3, 16, 1], [1, 1, 1, 1, 1, 1], [2, 16, 5, 7, 16, 1, 4], [16], [4, 4]]


def test_build_protocol_is_deadlock_free_and_phase_exact():
    for seed in range(12):
        for c, items in enumerate(CASES):
            simulate(items, 100 * seed + c, KERNEL)


@pytest.mark.parametrize("mistake", ["drain_no_sfree", "issuer_phase", "load_no_tempty", "transpose_early"])
def test_model_catches_planted_mistakes(mistake):
    with pytest.raises(ProtocolError):
        for seed in range(40):
            for c, items in enumerate(CASES):
                simulate(items, 100 * seed + c, KERNEL, planted=mistake)
