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
