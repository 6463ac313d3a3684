"""Pins of the oracle's window mask against what the pages fix.

"CoWindow Attention: Full Causal Coverage Is a Collective Property":
the abstract and the paper digest's method key points state that all KV
heads share the prefix-sink and near-diagonal windows, that complementary
long-range windows split the remaining history into equal-width slices
between breakpoints, and that the union over heads is the full causal
prefix.  The digest's key results give the duplicated-window coverage
range.  Every check here is structural: none re-types the mask rule.
"""
import itertools
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def causal(Lq, Lk):
    """Bottom-right-aligned causal mask: row i sees keys j <= i + Lk - Lq."""
    return np.tril(np.ones((Lq, Lk), dtype=bool), k=Lk - Lq)


def shapes():
    grid = []
    for Lq, Lk in [(40, 40), (33, 57), (57, 33), (1, 50), (64, 64), (17, 17)]:
        for Hkv in (1, 2, 3, 4):
            for S, N in [(0, 1), (3, 5), (8, 0), (0, 0), (5, 12), (40, 3)]:
                grid.append((Lq, Lk, Hkv, S, N))
    return grid


@pytest.mark.parametrize("Lq,Lk,Hkv,S,N", shapes())
def test_union_is_causal_prefix(oracle_mod, Lq, Lk, Hkv, S, N):
    """G=0 and Hkv*W >= Lk-N: the union over KV heads is the causal mask."""
    S_, N_, G, W = oracle_mod.default_quad(Lk, Hkv, S, N)
    quad = (S_, N_, G, W)
    assert Hkv * W >= Lk - N
    union = np.zeros((Lq, Lk), dtype=bool)
    for h in range(Hkv):
        m = oracle_mod.mask(Lq, Lk, h, quad)
        assert not (m & ~causal(Lq, Lk)).any(), "a head sees the future"
        union |= m
    assert (union == causal(Lq, Lk)).all()


@pytest.mark.parametrize("Lq,Lk,Hkv,S,N", shapes())
@pytest.mark.parametrize("G,W", [(0, 4), (3, 6), (0, 1), (7, 2)])
def test_shared_windows_and_disjoint_long_slices(oracle_mod, Lq, Lk, Hkv, S, N, G, W):
    """Sink + near are identical for every head; long slices are disjoint."""
    quad = (S, N, G, W)
    shared = oracle_mod.mask(Lq, Lk, 0, (S, N, G, 0))   # no long window at all
    longs = []
    for h in range(Hkv):
        m = oracle_mod.mask(Lq, Lk, h, quad)
        assert (m | shared == m).all(), "sink/near not shared by head %d" % h
        longs.append(m & ~shared)
    for a, b in itertools.combinations(range(Hkv), 2):
        assert not (longs[a] & longs[b]).any(), "heads %d,%d overlap" % (a, b)


@pytest.mark.parametrize("Hkv,N,G,W", [(4, 5, 0, 7), (3, 2, 4, 9), (8, 16, 0, 6), (2, 1, 1, 1)])
def test_long_slices_are_equal_width_and_adjacent(oracle_mod, Hkv, N, G, W):
    """For a row that sees its whole history, head h's long window is one
    run of W consecutive distances and head h+1's run starts where head h's
    ends: equal-width slices between breakpoints, starting after the near
    window and the gap."""
    Lk = N + G + Hkv * W + 11
    quad = (0, N, G, W)
    last = Lk - 1
    shared = oracle_mod.mask(1, Lk, 0, (0, N, G, 0))[0]
    prev_end = None
    for h in range(Hkv):
        m = oracle_mod.mask(1, Lk, h, quad)[0] & ~shared
        dist = np.sort(last - np.nonzero(m)[0])
        assert len(dist) == W
        assert (np.diff(dist) == 1).all()
        if prev_end is None:
            assert dist[0] == N + G
        else:
            assert dist[0] == prev_end + 1
        prev_end = dist[-1]


def test_duplicated_window_coverage_matches_pages(oracle_mod):
    """Complementary windows give 100% collective coverage of the long-range
    history; one shared window gives 12.5% and four distinct windows 50% at
    8 KV heads -- the endpoints of the digest's duplicated-window range."""
    with open(os.path.join(GOLDEN, "coverage_ablation.json")) as f:
        gold = json.load(f)
    Hkv = gold["hkv"]
    N, G, W = 24, 0, 13
    Lk = N + G + Hkv * W
    quad = (0, N, G, W)
    last_row = Lk - 1
    long_range = np.arange(Lk) <= last_row - N - G   # keys at distance >= N+G

    def coverage(widx):
        union = np.zeros(Lk, dtype=bool)
        for h in range(Hkv):
            union |= oracle_mod.mask(1, Lk, widx[h], quad)[0]
        return (union & long_range).sum() / long_range.sum()

    assert coverage(list(range(Hkv))) == pytest.approx(gold["complementary_coverage"])
    assert coverage([0] * Hkv) == pytest.approx(gold["duplicated_coverage_low"])
    assert coverage([h % 4 for h in range(Hkv)]) == pytest.approx(gold["duplicated_coverage_high"])
    # and the control loses coverage of the whole causal mask too
    full = np.zeros((Lk, Lk), dtype=bool)
    dup = np.zeros((Lk, Lk), dtype=bool)
    for h in range(Hkv):
        full |= oracle_mod.mask(Lk, Lk, h, quad)
        dup |= oracle_mod.mask(Lk, Lk, 0, quad)
    assert (full == causal(Lk, Lk)).all()
    assert dup.sum() < full.sum()


@pytest.mark.parametrize("Lk,Hkv,S,N", [(512, 2, 16, 64), (8192, 4, 64, 1024),
                                        (32768, 8, 128, 4096), (131072, 8, 128, 8192)])
def test_default_quads_of_the_workloads(oracle_mod, Lk, Hkv, S, N):
    """Default W = ceil((Lk-N)/Hkv) at the four training workloads; the
    windows then cover the history exactly (Hkv*W >= Lk-N > (Hkv-1)*W)."""
    S_, N_, G, W = oracle_mod.default_quad(Lk, Hkv, S, N)
    assert (S_, N_, G) == (S, N, 0)
    assert Hkv * W >= Lk - N > Hkv * W - Hkv
    expected = {512: 224, 8192: 1792, 32768: 3584, 131072: 15360}[Lk]
    assert W == expected


def test_empty_rows_and_degenerate_quads(oracle_mod):
    # Lq > Lk: the first Lq-Lk rows have p < 0 and see nothing.
    m = oracle_mod.mask(10, 4, 0, (2, 2, 0, 2))
    assert not m[:6].any() and m[6:].any()
    # all-zero quad: nothing visible at all
    assert not oracle_mod.mask(8, 8, 0, (0, 0, 0, 0)).any()
    # N >= Lk: every head is dense causal regardless of W
    for h in range(3):
        assert (oracle_mod.mask(9, 9, h, (0, 9, 0, 0)) == causal(9, 9)).all()


def test_tile_counts_match_the_dense_mask(oracle_mod):
    for (Lq, Lk, BM, BN) in [(100, 100, 32, 64), (70, 130, 64, 64), (130, 70, 128, 64)]:
        quad = (5, 17, 3, 11)
        for w in range(3):
            m = oracle_mod.mask(Lq, Lk, w, quad)
            counts = oracle_mod.tile_counts(Lq, Lk, w, quad, BM, BN)
            for qt in range(counts.shape[0]):
                for kt in range(counts.shape[1]):
                    blk = m[qt * BM:(qt + 1) * BM, kt * BN:(kt + 1) * BN]
                    assert counts[qt, kt] == blk.sum()


def _window_keys_loop(p_lo, horizon, w, quad):
    # the visibility rule written out once more as a plain double loop
    S, N, G, W = quad
    keys = set()
    for p in range(p_lo, p_lo + horizon):
        for j in range(0, p + 1):
            d = p - j
            if j < S or d < N or (N + G + w * W <= d < N + G + (w + 1) * W):
                keys.add(j)
    return sorted(keys)


@pytest.mark.parametrize("p_lo,horizon,w,quad", [
    (200, 1, 0, (4, 16, 0, 24)), (200, 9, 3, (4, 16, 0, 24)), (37, 5, 1, (0, 8, 2, 5)),
    (500, 17, 7, (16, 32, 0, 60)), (3, 4, 0, (0, 0, 0, 0)), (90, 30, 2, (8, 8, 8, 8))])
def test_window_keys_match_the_rule(oracle_mod, p_lo, horizon, w, quad):
    got = oracle_mod.window_keys(p_lo, horizon, w, quad)
    assert list(got) == _window_keys_loop(p_lo, horizon, w, quad)


def test_window_keys_size_bound(oracle_mod):
    # a head's windowed key set never exceeds sink + near + long + 2 * horizon
    S, N, G, W = quad = (16, 64, 0, 96)
    for w in range(4):
        for p_lo, hz in ((1000, 1), (1000, 50), (300, 7)):
            n = len(oracle_mod.window_keys(p_lo, hz, w, quad))
            assert n <= S + N + W + 2 * hz
