"""The stream-K work split of the decode-sized tensor-core product, on the CPU.

The kernel (gemm_sk.cuh) gives CTA c of G the contiguous units
[U*c/G, U*(c+1)/G) of the (tile, K stage) stream, U = tiles * nk, with
G = min(SMs, U).  Its correctness rests on a few facts about that split,
checked here for every benchmark shape and a sweep of small ones:
  * every unit belongs to exactly one CTA, and cta_of(u) = ((u+1)*G - 1) // U
    names it;
  * a CTA's segments (one per tile it touches) are: at most one leading
    segment that starts after the tile's first stage (the CTA is a "helper"
    of that tile), then segments that start at a tile's first stage;
  * a tile cut between CTAs is finished by the CTA holding its first stage,
    for which it is the LAST segment, and its helpers are exactly the CTAs
    finisher+1 .. cta_of(last unit of the tile), for each of which it is the
    FIRST segment -- so one workspace slot per CTA suffices and the finisher
    reaches the tile after its helpers have started on it.
"""
import itertools

import pytest


def split(U, G):
    return [(U * c // G, U * (c + 1) // G) for c in range(G)]


def cta_of(u, U, G):
    return ((u + 1) * G - 1) // U


def segments(u0, u1, nk):
    out, u = [], u0
    while u < u1:
        t = u // nk
        end = min(u1, (t + 1) * nk)
        out.append((t, u - t * nk, end - t * nk))
        u = end
    return out


def check(tiles, nk, sms=148):
    U = tiles * nk
    G = min(sms, U)
    ranges = split(U, G)
    owner = {}
    for c, (u0, u1) in enumerate(ranges):
        assert u1 > u0, "every CTA has work when G <= U"
        for u in range(u0, u1):
            assert u not in owner
            owner[u] = c
            assert cta_of(u, U, G) == c
    assert len(owner) == U
    helper_of = {}
    for c, (u0, u1) in enumerate(ranges):
        segs = segments(u0, u1, nk)
        for i, (t, lo, hi) in enumerate(segs):
            if lo > 0:
                assert i == 0, "only a CTA's first segment can start after the tile's first stage"
                helper_of[c] = t
            if lo == 0 and hi < nk:
                assert i == len(segs) - 1, "a finisher's cut tile is its last segment"
                last = cta_of(t * nk + nk - 1, U, G)
                assert last > c
                for h in range(c + 1, last + 1):
                    assert helper_of.get(h, t) == t
                    hs = segments(*ranges[h], nk)
                    assert hs[0][0] == t and hs[0][1] > 0, "each helper holds the tile as its first segment"
    # every cut tile has exactly one finisher
    for t in range(tiles):
        holders = {owner[u] for u in range(t * nk, (t + 1) * nk)}
        first = owner[t * nk]
        assert holders == set(range(first, max(holders) + 1))


@pytest.mark.parametrize("N,M,K,rows,bn", [
    (21504, 16, 5376, 128, 16), (5376, 16, 21504, 128, 16),          # 27B decode batch of 16
    (3840, 64, 2560, 128, 64), (2560, 64, 2560, 128, 64), (13824, 64, 2560, 128, 64), (2560, 64, 6912, 128, 64),
    (6912, 64, 2560, 64, 64), (6912, 2048, 2560, 64, 64), (21504, 16, 5376, 64, 16),  # gated: 64 features a tile
    (128, 1, 64, 128, 16), (300, 5, 320, 128, 16), (777, 33, 1344, 64, 64)])
def test_benchmark_shapes(N, M, K, rows, bn):
    tiles = -(-N // rows) * -(-M // bn)
    nk = -(-K // 256)
    check(tiles, nk)


def test_small_sweep():
    for tiles, nk, sms in itertools.product(range(1, 40), range(1, 30), (1, 3, 7, 16, 148)):
        check(tiles, nk, sms)
