"""Host-side checks of the work partition the small-m GEMM kernel uses
(no GPU): the kernel computes these integers on the device with the formulas
restated here, and relies on the invariants below."""
import random

import pytest


def range_begin(c, T, G):
    """First iteration of CTA c of G over T iterations, as the kernel forms
    it in 32-bit arithmetic: c*q + (c*r)//G with q = T//G, r = T%G."""
    q, r = T // G, T % G
    assert c * r < 2 ** 32        # the unsigned 32-bit product cannot wrap
    return c * q + (c * r) // G


def owner_of(i, T, G):
    """CTA whose range holds iteration i: ceil((i + 1) G / T) - 1."""
    return -(-((i + 1) * G) // T) - 1


@pytest.mark.parametrize("seed", range(4))
def test_range_begin_is_the_even_split(seed):
    rng = random.Random(seed)
    for _ in range(2000):
        G = rng.randint(1, 1024)
        T = rng.randint(1, 2 ** 31 - 1)
        for c in (0, 1, G // 2, G - 1, G, rng.randint(0, G)):
            assert range_begin(c, T, G) == (c * T) // G


def test_every_iteration_has_one_owner_and_ranges_tile_the_space():
    rng = random.Random(7)
    for _ in range(300):
        G = rng.randint(1, 160)
        T = rng.randint(1, 5000)
        covered = 0
        for c in range(G):
            b, e = range_begin(c, T, G), range_begin(c + 1, T, G)
            assert b == covered
            covered = e
            for i in range(b, e):
                assert owner_of(i, T, G) == c
        assert covered == T


@pytest.mark.parametrize("s", [2, 3, 4, 5, 8])
def test_cluster_split_gives_each_cta_part_of_one_tile(s):
    # grid = tiles * s over tiles * KI iterations: CTA (tile, rank) covers
    # k iterations [rank*KI//s, (rank+1)*KI//s) of its own tile, so the s CTAs
    # of a tile (one cluster) together cover it once
    rng = random.Random(s)
    for _ in range(200):
        tiles, KI = rng.randint(1, 40), rng.randint(s, 64)
        T, G = tiles * KI, tiles * s
        for c in range(G):
            b, e = range_begin(c, T, G), range_begin(c + 1, T, G)
            tile, rank = divmod(c, s)
            assert b == tile * KI + (rank * KI) // s
            assert e == tile * KI + ((rank + 1) * KI) // s
            assert e - b >= 1 and (b // KI) == ((e - 1) // KI) == tile


# ------------------------------------------------------- split-tile counters
MASK32 = 0xFFFFFFFF


def _contributors(tile, KI, T, G):
    """CTAs whose range touches tile (the kernel's c_first..c_last with a
    non-empty range)."""
    c0, c1 = owner_of(tile * KI, T, G), owner_of(tile * KI + KI - 1, T, G)
    return [c for c in range(c0, c1 + 1) if range_begin(c + 1, T, G) > range_begin(c, T, G)]


def _arrive(counters, tile, epoch, ncontrib, reset):
    """One contributor's compare-and-swap on the tile counter, as the kernel
    does it: a value of another epoch counts as zero arrivals; the arrival
    that brings the count to ncontrib finishes the tile (and, with reset,
    zeroes the counter)."""
    cur = counters[tile]
    want = cur + 1 if (cur >> 32) == epoch else (epoch << 32) | 1
    counters[tile] = want
    last = (want & MASK32) == ncontrib
    if last and reset:
        counters[tile] = 0
    return last


def _launch(counters, epoch, KI, T, G, rng, reset):
    """One launch: every contributor of every split tile arrives, in a random
    order; returns, per split tile, how many contributors saw themselves last."""
    finished = {}
    arrivals = []
    for tile in range(T // KI):
        cs = _contributors(tile, KI, T, G)
        if len(cs) > 1:
            arrivals += [(tile, len(cs))] * len(cs)
            finished[tile] = 0
    rng.shuffle(arrivals)
    for tile, n in arrivals:
        finished[tile] += _arrive(counters, tile, epoch, n, reset)
    return finished


@pytest.mark.parametrize("replays", [False, True])
def test_split_tiles_finish_exactly_once_per_launch(replays):
    # eager calls take a fresh epoch each; a CUDA graph replays a launch with
    # the epoch it was captured with.  Either way every split tile must have
    # exactly one finishing contributor in every launch, starting from
    # counters left by earlier launches (or never initialised).
    rng = random.Random(11)
    for _ in range(60):
        KI, tiles, G = rng.randint(1, 40), rng.randint(1, 30), rng.randint(2, 160)
        T = KI * tiles
        counters = [rng.getrandbits(64) & ~(0xFFFFFFFF << 32) for _ in range(tiles)]   # garbage, epoch 0
        epoch = 1
        for launch in range(5):
            if not replays:
                epoch += 1
            done = _launch(counters, epoch, KI, T, G, rng, reset=True)
            assert all(v == 1 for v in done.values()), (KI, tiles, G, launch, done)


def test_without_the_reset_a_replay_never_finishes_its_split_tiles():
    # the failure the counter reset removes: a replay with the same epoch
    # counts on from the previous launch's total
    rng = random.Random(12)
    KI, tiles, G = 7, 10, 31
    T = KI * tiles
    counters = [0] * tiles
    first = _launch(counters, 5, KI, T, G, rng, reset=False)
    second = _launch(counters, 5, KI, T, G, rng, reset=False)
    assert first and all(v == 1 for v in first.values())
    assert all(v == 0 for v in second.values())
