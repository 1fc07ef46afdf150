"""The mbarrier protocol of the decode-block kernel (tq4_decode.cu), modelled
on the CPU.

The kernel's roles synchronise through mbarriers (plus one CTA barrier and
one cluster barrier that every thread reaches, and one named barrier of the
eight rotation warps): the weight producer's codes tiles (full, one stage per
iteration) and scales tile (sfull), the x producer's x tiles (xland),
four-warp dequant groups filling half A stages (afull) -- iterations past the
tensor memory's stage count reuse a stage once the MMAs reading it complete
(afree, by tcgen05.commit) -- the rotation warps' xready, the dequant warps'
eready, the issuers' dfull and idone.  Static weights are requested at entry
and dequantized in part before the wait for the previous kernel.  This model runs the roles as
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
    released -- the wind-down the kernel promises on a timeout;
  * a withheld x copy (xland never completes) also winds down, through the
    rotation warps' named barrier.
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
FIRST_DQ = _const("kFirstDqWarp")
WARPS = _const("kRotWarps")            # rotation warps: 0-3 and 16-19
ISSUERS = 2 * GROUPS                   # one per (group, 64-k half)
MAX_ITERS = 8                                    # kFusedMaxIters
TMEM_COLS = _const("kTmemColsD")


def a_stages(nb):
    # as a_stages() in the kernel: tensor memory beside the accumulators
    return (TMEM_COLS - ISSUERS * 16 * nb) // 64


def all_stages(nb):
    return a_stages(nb)


def test_source_constants_and_counts():
    # the init counts and layout the model assumes, as written in the kernel
    assert (GROUPS, FIRST_DQ, TMEM_COLS) == (3, 4, 512)
    assert "constexpr int kStagesD = kMaxIters;" in SRC              # one codes stage per iteration
    assert "mbar_init(&sh.afull[i][0], 4);" in SRC and "mbar_init(&sh.afull[i][1], 4);" in SRC   # one arrival per warp
    assert "mbar_init(&sh.xready, kRotWarps)" in SRC                 # one arrival per rotation warp
    assert WARPS == 8 and "constexpr int kProducerWarp = kFirstDqWarp;" in SRC
    # dequant warps 4-15, rotation warps 0-3 and 16-19
    assert "(warp >= kFirstDqWarp && warp < kHiWarp) ? (warp - kFirstDqWarp) >> 2 : -1" in SRC
    assert "constexpr int kHiWarp = kFirstDqWarp + 4 * kGroups;" in SRC
    assert "warp < 4 ? warp : ((warp >= kHiWarp && warp < kHiWarp + 4) ? warp - kHiWarp + 4 : -1)" in SRC
    assert "mbar_init(&sh.dfull, kIssuers)" in SRC and "constexpr int kIssuers = 2 * kGroups;" in SRC
    assert "mbar_init(&sh.eready, 4 * kGroups)" in SRC               # one arrival per dequant warp
    assert "mbar_init(&sh.xland, 1)" in SRC and "mbar_init(&sh.sfull, 1)" in SRC
    # the x producer initialises its own barrier, waits and copies x before
    # the set-up barrier; its warp takes no part in the set-up stores; the
    # next-launch trigger precedes the set-up barrier (which the x producer
    # reaches only after its wait)
    i_xp = SRC.index("  if (warp == kHiWarp && lane == 0) {\n    mbar_init(&sh.xland, 1);\n    fence_mbar_init();\n    pdl_wait();")
    i_trig = SRC.index("  if (threadIdx.x == 0) pdl_launch_dependents();\n  tc_fence_before();\n  __syncthreads();")
    assert i_xp < i_trig
    assert SRC.count("mbar_init(&sh.xland, 1)") == 1
    assert "const bool setup_role = warp != kProducerWarp && warp != kHiWarp;" in SRC
    assert "if (warp == kHiWarp && lane == 0 && !stat) issue_weight();" in SRC
    assert "named_bar_sync(1, kRotWarps * 32)" in SRC                 # the eight rotation warps
    # tensor-core rotation: the bounded rdone wait, then the first conversion
    # and the token max, then the named barrier (every warp reaches it), then
    # the check of the token range and the second conversion where needed
    i_rdone = SRC.index("const bool rok = wwait(&sh.rdone, 0, abortp);")
    i_first = SRC.index("uint32_t mb = __float_as_uint(convert(std::false_type{}, 1.0f));")
    i_bar = SRC.index("named_bar_sync(1, kRotWarps * 32);", i_first)
    i_keep = SRC.index("const bool keep = tb == 0u || (tb >= 0x3D800000u && tb < 0x47000000u);")
    i_again = SRC.index("if (__any_sync(0xFFFFFFFFu, !keep && e != 0)) convert(std::true_type{}, exp2i(-e));")
    assert i_rdone < i_first < i_bar < i_keep < i_again
    # the factor r of x' is applied in the epilogue on this path
    assert "(kTcRot ? __uint_as_float(0x3E3504F3u) / kLevelScaleD : 1.0f / kLevelScaleD)" in SRC
    assert "mbar_init(&sh.rdone, 2)" in SRC
    # the cluster reduction: asynchronous stores counted in bytes on the
    # owner's barrier; every CTA sends all its rows (zeros after a timeout)
    # and waits for its own with a wait that ignores its abort flag, so no
    # store can reach a CTA that has left
    assert "if (ok || split > 1) {" in SRC and "st_async_v4(" in SRC
    assert "while (!mbar_try_wait(addr, 0)) {" in SRC and "wwait(&sh.redfull" not in SRC
    assert SRC.count("barrier.cluster.arrive") == 1 and SRC.count("barrier.cluster.wait") == 2 and "mma_commit(&sh.rdone)" in SRC and "drain(&sh.rdone, 0)" in SRC
    assert (a_stages(1), a_stages(2)) == (6, 5)
    assert "const int sa = li % kNA;" in SRC and SRC.count("dq_run(kMaxIters);") == 1   # one call site


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


def run(cnt, seed, withhold_xready=False, static=True, nb=1, withhold_x=False):
    rng = random.Random(seed)
    na = all_stages(nb)
    B = {}

    def bar(name, count):
        B[name] = Barrier(name, count)
        return B[name]

    full = [bar(f"full{s}", 1) for s in range(MAX_ITERS)]
    afull = [[bar(f"afull{s}{h}", 4) for h in range(2)] for s in range(MAX_ITERS)]
    afree = [[bar(f"afree{s}{h}", 1) for h in range(2)] for s in range(MAX_ITERS)]
    xready = bar("xready", WARPS)
    dfull = bar("dfull", ISSUERS)
    idone = [bar(f"idone{i}", 1) for i in range(ISSUERS)]
    eready = bar("eready", 4 * GROUPS)
    xland = bar("xland", 1)
    sfull = bar("sfull", 1)
    rotbar = bar("rotbar", WARPS)      # the named barrier (hardware: no timeout)
    rdone = bar("rdone", 2)            # the rotation MMAs (16 tokens of TQ4_1S: on the tensor core), per block
    state = {"abort": False, "landings": [], "mma": [], "issued": 0, "landed": 0, "mma_issued": 0,
             "waited": False}

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

    def issue_all():
        # codes tiles and the scales tile
        for li in range(cnt):
            state["issued"] += 1
            state["landings"].append(full[li])
        state["issued"] += 1
        state["landings"].append(sfull)

    def rotation(r):
        # rotation warp r (0-3: warps 0-3; 4-7: warps 16-19); lane 0 of warp
        # 16 issues the rotation MMAs once x landed (else arrives itself)
        xok = yield from wait(xland, 0)
        if r in (4, 5):
            # lane 0 of warp 16 (block 0) and 17 (block 1, more than 4 iterations)
            if xok and (r == 4 or cnt > 4):
                state["mma_issued"] += 1
                state["mma"].append(rdone)
            else:
                rdone.arrive()
        rok = yield from wait(rdone, 0)
        if xok and rok:
            yield ("step", "x' to fp16 at e = 0, token max |x'|")
        rotbar.arrive()
        yield from wait(rotbar, 0, bounded=False)
        if xok and rok:
            yield ("step", "tokens outside [2^-4, 2^15) converted again")
        if not (withhold_xready and r == 7):
            xready.arrive()

    def dq_run(g, done, li_end):
        # dequantize this group's iterations g + 3 done, ... below li_end
        while True:
            li = g + GROUPS * done[0]
            if li >= li_end or li >= cnt:
                return True
            sa = li % na
            ok = yield from wait(full[li], 0)
            if not ok:
                return False
            for h in range(2):
                if li >= na:
                    ok = yield from wait(afree[sa][h], li // na - 1)
                    if not ok:
                        return False
                yield ("step", "dequant")
                afull[sa][h].arrive()
            done[0] += 1

    def dequant(g, q):
        # warp 4 + 4g + q; lane 0 of warp 4 is also the weight producer
        if (g, q) == (0, 0) and static:
            issue_all()                              # at entry
        yield ("step", "set-up (CTA barrier)")
        done = [0]
        ok = True
        if static:
            ok = yield from wait(sfull, 0)           # the scales tile
            yield ("step", "row exponent")
            eready.arrive()
            if ok:
                ok = yield from dq_run(g, done, na)  # before the wait: stages not reused
        yield ("step", "wait for the previous kernel")
        if not static:
            ok = yield from wait(sfull, 0)
            yield ("step", "row exponent")
            eready.arrive()
        if ok:
            yield from dq_run(g, done, MAX_ITERS)

    def issuer(g, h):
        # lane 0 of warps 1-3 (h = 0) and 17-19 (h = 1), all rotation warps
        yield from rotation(1 + g if h == 0 else 5 + g)
        ok = yield from wait(xready, 0)
        use = 0
        for li in range(g, cnt, GROUPS):
            if not ok:
                break
            sa = li % na
            ok = yield from wait(afull[sa][h], li // na)
            if not ok:
                break
            state["mma_issued"] += 1
            state["mma"].append(afree[sa][h])          # commit: arrives when the MMAs complete
            use += 1
        if use > 0:
            state["mma"].append(dfull)
        else:
            dfull.arrive()
        state["mma"].append(idone[2 * g + h])
        yield from wait(idone[2 * g + h], 0, bounded=False)

    def epilogue(w):
        if w == 0:
            yield from rotation(0)
        ok = yield from wait(xready, 0)
        ok = ok and (yield from wait(eready, 0))
        ok = ok and (yield from wait(dfull, 0))

    def x_producer_rotation():
        # warp 16: lane 0 initialises xland, waits for the previous kernel and
        # issues the x tiles before the set-up barrier (the set-up is not
        # modelled: every actor here starts after it), then a weight not
        # flagged static; the warp rotates, and on an abort lane 0 waits for
        # every copy to land
        yield ("step", "wait for the previous kernel")
        state["issued"] += 1
        if not withhold_x:
            state["landings"].append(xland)
        else:
            state["issued"] -= 1                      # the copy never completes (models a lost transfer)
        if not static:
            issue_all()
        yield from rotation(4)
        if state["abort"]:
            for li in range(cnt):
                yield from wait(full[li], 0, bounded=False)
            yield from wait(sfull, 0, bounded=False)
            if not withhold_x:
                yield from wait(xland, 0, bounded=False)
            yield from wait(rdone, 0, bounded=False)

    actors = [epilogue(0), x_producer_rotation()]
    actors += [issuer(g, h) for g in range(GROUPS) for h in range(2)]
    actors += [dequant(g, q) for g in range(GROUPS) for q in range(4)]
    # the issuers' warps 1-3 join the epilogue after their roles
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
@pytest.mark.parametrize("static,nb", [(True, 1), (False, 1), (True, 2)])
def test_protocol_completes_with_exact_counts(cnt, static, nb):
    for seed in range(30):
        B, state = run(cnt, seed, static=static, nb=nb)
        assert not state["abort"], f"cnt={cnt} seed={seed}: a wait ran out in a correct run"
        assert state["landed"] == state["issued"] == cnt + 2   # codes, scales, x
        assert not state["mma"] and state["mma_issued"] == 2 * cnt + (2 if cnt > 4 else 1)   # + the rotation MMAs
        for b in B.values():
            assert b.arrived == 0, f"{b.name}: partial phase left at the end"
        assert B["xready"].phase == 1 and B["dfull"].phase == 1 and B["eready"].phase == 1
        assert B["xland"].phase == 1 and B["sfull"].phase == 1 and B["rotbar"].phase == 1
        na = all_stages(nb)
        for s in range(MAX_ITERS):
            uses = len(range(s, cnt, na)) if s < na else 0
            assert B[f"afull{s}0"].phase == uses and B[f"afree{s}1"].phase == uses


@pytest.mark.parametrize("cnt", [1, 3, 7, 8])
@pytest.mark.parametrize("static", [True, False])
def test_withheld_arrival_winds_down(cnt, static):
    for seed in range(30):
        B, state = run(cnt, seed, withhold_xready=True, static=static)
        assert state["abort"], "the withheld arrival must make a wait run out"
        assert state["landed"] == state["issued"], "a TMA copy still in flight at exit"
        assert not state["mma"], "an MMA still in flight when tensor memory is released"
        assert B["xready"].phase == 0


@pytest.mark.parametrize("cnt", [1, 4, 8])
@pytest.mark.parametrize("static", [True, False])
def test_lost_x_copy_winds_down(cnt, static):
    for seed in range(20):
        B, state = run(cnt, seed, withhold_x=True, static=static)
        assert state["abort"], "a lost x copy must make a wait run out"
        assert state["landed"] == state["issued"], "a TMA copy still in flight at exit"
        assert not state["mma"], "an MMA still in flight when tensor memory is released"
        assert B["xready"].phase == 1 and B["rotbar"].phase == 1
