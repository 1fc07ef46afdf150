"""The mbarrier protocol of the decode-block kernel (tq4_decode.cu), modelled
on the CPU.

The kernel's roles synchronise only through mbarriers (plus one CTA barrier
and one cluster barrier that every thread reaches): the TMA producer and the
codes ring (full/empty), four-warp dequant groups filling half A stages
(afull) that their MMA issuer frees (afree, by tcgen05.commit), the rotation
warps' xready, the dequant warps' eready, the issuers' dfull and idone.  This model runs the roles as
actors in random interleavings, with TMA landings and MMA completions as
asynchronous events, for every k-range length a CTA can have (1..8
iterations), and checks that:
  * every actor finishes (no deadlock) and every barrier phase completes with
    exactly its initial arrival count;
  * no parity wait is ever evaluated two phases behind its barrier (the
    mbarrier parity ABA hazard);
  * with one arrival withheld (a rotation warp that never reports), the
    bounded waits run out, every role still ends, every issued TMA copy has
    landed and every issued MMA has completed before tensor memory would be
    released -- the wind-down the kernel promises on a timeout.
The arrival counts and ring depth are read from the kernel source, so a
change there is checked as it stands."""
import os
import random
import re

import pytest

SRC = open(os.path.join(os.path.dirname(__file__), "..", "bit_rotated_weight_b200", "csrc", "tq4_decode.cu")).read()


def _const(name):
    return int(re.search(rf"constexpr int {name} = (\d+);", SRC).group(1))


GROUPS = _const("kGroups")
STAGES = _const("kStagesD")
FIRST_DQ = _const("kFirstDqWarp")
WARPS = FIRST_DQ + 4 * GROUPS


def test_source_constants_and_counts():
    # the init counts the model assumes, as written in the kernel
    assert (GROUPS, STAGES, FIRST_DQ) == (3, 4, 4)
    assert "mbar_init(&sh.empty[i - kStagesD], 4)" in SRC           # one arrival per dequant warp
    assert "mbar_init(&sh.afull[(i - 2 * kStagesD) >> 1][i & 1], 4)" in SRC
    assert "mbar_init(&sh.xready, kThreads / 32)" in SRC             # one arrival per warp
    assert "mbar_init(&sh.dfull, kGroups)" in SRC
    assert "mbar_init(&sh.eready, 4 * kGroups)" in SRC               # one arrival per dequant warp


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, f"{self.name}: over-arrival in phase {self.phase}"
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1

    def done(self, p):
        # a parity wait for phase p: the hazard is a barrier two phases ahead
        assert self.phase <= p + 1, f"{self.name}: parity wait for phase {p} while at phase {self.phase}"
        return self.phase > p


class Timeout(Exception):
    pass


def run(cnt, seed, withhold_xready=False):
    rng = random.Random(seed)
    B = {}

    def bar(name, count):
        B[name] = Barrier(name, count)
        return B[name]

    full = [bar(f"full{s}", 1) for s in range(STAGES)]
    empty = [bar(f"empty{s}", 4) for s in range(STAGES)]
    afull = [[bar(f"afull{g}{h}", 4) for h in range(2)] for g in range(GROUPS)]
    afree = [[bar(f"afree{g}{h}", 1) for h in range(2)] for g in range(GROUPS)]
    xready = bar("xready", WARPS)
    dfull = bar("dfull", GROUPS)
    idone = [bar(f"idone{g}", 1) for g in range(GROUPS)]
    eready = bar("eready", 4 * GROUPS)
    state = {"abort": False, "landings": [], "mma": [], "issued": 0, "landed": 0, "mma_issued": 0, "mma_done": 0}

    def wait(b, p, bounded=True):
        # a bounded wait: yields until the phase completed; after an abort it
        # gives up (returns False); the scheduler raises Timeout into it when
        # nothing else can move
        while not b.done(p):
            if bounded and state["abort"]:
                return False
            try:
                yield ("wait", b.name, p, bounded)
            except Timeout:
                state["abort"] = True
                return False
        return True

    def issue(li):
        state["issued"] += 1
        state["landings"].append(full[li % STAGES])

    def producer():
        # warp 0, lane 0: the first copies, the warp's rotation, then the ring
        npre = min(cnt, STAGES)
        for li in range(npre):
            issue(li)
        yield from rotation(0)
        armed = npre - 1
        for li in range(npre, cnt):
            ok = yield from wait(empty[li % STAGES], li // STAGES - 1)
            if not ok:
                break
            issue(li)
            armed = li
        if state["abort"]:
            for li in range(max(armed - STAGES + 1, 0), armed + 1):
                yield from wait(full[li % STAGES], li // STAGES, bounded=False)

    def rotation(w):
        yield ("step", "rotate")
        if not (withhold_xready and w == 7):
            xready.arrive()

    def dequant(g, q):
        yield from rotation(FIRST_DQ + 4 * g + q)
        yield ("step", "row exponent")
        eready.arrive()
        use = 0
        for li in range(g, cnt, GROUPS):
            ok = yield from wait(full[li % STAGES], li // STAGES)
            if not ok:
                break
            empty[li % STAGES].arrive()
            for h in range(2):
                if use > 0:
                    ok = yield from wait(afree[g][h], use - 1)
                    if not ok:
                        break
                yield ("step", "dequant")
                afull[g][h].arrive()
            if not ok:
                break
            use += 1

    def issuer(g):
        yield from rotation(1 + g)
        ok = yield from wait(xready, 0)
        use = 0
        for li in range(g, cnt, GROUPS):
            if not ok:
                break
            for h in range(2):
                ok = yield from wait(afull[g][h], use)
                if not ok:
                    break
                state["mma_issued"] += 1
                state["mma"].append(afree[g][h])      # commit: arrives when the MMAs complete
            if not ok:
                break
            use += 1
        if use > 0:
            state["mma"].append(dfull)
        else:
            dfull.arrive()
        state["mma"].append(idone[g])
        yield from wait(idone[g], 0, bounded=False)

    def epilogue(w):
        if w == 0:
            yield from producer()
        ok = yield from wait(xready, 0)
        ok = ok and (yield from wait(eready, 0))
        ok = ok and (yield from wait(dfull, 0))

    actors = [epilogue(0)]
    actors += [issuer(g) for g in range(GROUPS)]
    actors += [dequant(g, q) for g in range(GROUPS) for q in range(4)]
    # the issuers' warps and warps 1-3 join the epilogue after their roles
    actors += [epilogue(w) for w in range(1, 4)]
    live = list(actors)
    pending = {id(a): None for a in live}
    for a in live:
        pending[id(a)] = next(a, "END")
    steps = 0
    while True:
        steps += 1
        assert steps < 100000
        events = []
        if state["landings"]:
            events.append("land")
        if state["mma"]:
            events.append("mma")
        runnable = [a for a in live if pending[id(a)] != "END"]
        if not runnable and not events:
            break
        choices = events + runnable
        pick = rng.choice(choices)
        if pick == "land":
            b = state["landings"].pop(rng.randrange(len(state["landings"])))
            b.arrive()
            state["landed"] += 1
            continue
        if pick == "mma":
            # MMAs of one CTA complete in issue order
            state["mma"].pop(0).arrive()
            state["mma_done"] += 1
            continue
        a = pick
        tag = pending[id(a)]
        if tag[0] == "wait":
            def can_move(o):
                t = pending[id(o)]
                if t == "END":
                    return False
                if t[0] == "step":
                    return True
                return B[t[1]].phase > t[2] or (t[3] and state["abort"])
            progress_possible = bool(events) or any(can_move(o) for o in live)
            if not progress_possible:
                # nothing can move: the bounded wait of this actor runs out
                try:
                    pending[id(a)] = a.throw(Timeout())
                except StopIteration:
                    pending[id(a)] = "END"
                continue
        try:
            pending[id(a)] = a.send(None)
        except StopIteration:
            pending[id(a)] = "END"
    return B, state


@pytest.mark.parametrize("cnt", range(1, 9))
def test_protocol_completes_with_exact_counts(cnt):
    for seed in range(40):
        B, state = run(cnt, seed)
        assert not state["abort"], f"cnt={cnt} seed={seed}: a wait ran out in a correct run"
        assert state["landed"] == state["issued"] == cnt
        assert not state["mma"] and state["mma_issued"] == 2 * cnt
        for b in B.values():
            assert b.arrived == 0, f"{b.name}: partial phase left at the end"
        assert B["xready"].phase == 1 and B["dfull"].phase == 1 and B["eready"].phase == 1
        for s in range(STAGES):
            assert B[f"full{s}"].phase == len(range(s, cnt, STAGES))


@pytest.mark.parametrize("cnt", [1, 3, 4, 8])
def test_withheld_arrival_winds_down(cnt):
    for seed in range(40):
        B, state = run(cnt, seed, withhold_xready=True)
        assert state["abort"], "the withheld arrival must make a wait run out"
        assert state["landed"] == state["issued"], "a TMA copy still in flight at exit"
        assert not state["mma"], "an MMA still in flight when tensor memory is released"
        assert B["xready"].phase == 0
