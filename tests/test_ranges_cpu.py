"""The tile ranges each tcgen05 CTA computes for itself (query_tile_ranges /
key_tile_ranges in csrc/common.cuh, built here for the host): for every
query tile, the key tiles it visits are exactly those holding at least one
visible pair in the oracle's brute-force tile counts, and likewise for every
key tile and the query tiles that see it; the ranges are ascending, disjoint
and at most three.  The per-thread visible runs (row_key_runs /
key_pos_runs) hold exactly the keys of each row, and the positions seeing
each key, of the brute-force mask, as at most three ascending runs that
neither overlap nor touch.  Runs without a GPU (nvcc compiles host code)."""
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ranges_bin():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    out = os.path.join(tempfile.mkdtemp(), "ranges_host")
    subprocess.check_call([nvcc, "-std=c++17", "-O1", "-o", out, os.path.join(ROOT, "tests", "ranges_host.cu")])
    return out


def _ranges(binary, mode, Lq, Lk, quad, h, BM, BN):
    S, N, G, W = quad
    txt = subprocess.check_output([binary, mode, str(Lq), str(Lk), str(S), str(N), str(G), str(W), str(h),
                                   str(BM), str(BN)], text=True)
    out = []
    for line in txt.strip().splitlines():
        n, l0, n0, l1, n1, l2, n2 = (int(x) for x in line.split())
        spans = [(l0, n0), (l1, n1), (l2, n2)][:n]
        assert all(ln > 0 for _, ln in spans)
        assert all(spans[a][0] + spans[a][1] < spans[a + 1][0] for a in range(len(spans) - 1))  # disjoint, not touching
        out.append(set(t for lo, ln in spans for t in range(lo, lo + ln)))
    return out


@pytest.mark.parametrize("Lq,Lk,quad,BM,BN", [
    (512, 512, (16, 64, 0, 224), 128, 96), (700, 700, (5, 37, 0, 50), 128, 64),
    (300, 130, (3, 20, 0, 110), 64, 128), (200, 900, (64, 100, 7, 90), 128, 96),
    (384, 384, (0, 384, 0, 0), 32, 128), (1000, 1000, (1, 1, 0, 125), 64, 64),
    (257, 257, (0, 0, 0, 0), 128, 96), (9, 4000, (128, 256, 0, 900), 128, 128)])
def test_ranges_equal_the_visible_tiles(oracle_mod, ranges_bin, Lq, Lk, quad, BM, BN):
    for h in range(4):
        counts = oracle_mod.tile_counts(Lq, Lk, h, quad, BM, BN)  # [query tile, key tile] visible pairs
        q = _ranges(ranges_bin, "q", Lq, Lk, quad, h, BM, BN)
        k = _ranges(ranges_bin, "k", Lq, Lk, quad, h, BM, BN)
        assert len(q) == counts.shape[0] and len(k) == counts.shape[1]
        for qt in range(counts.shape[0]):
            assert q[qt] == set(np.nonzero(counts[qt])[0]), (h, "query tile", qt)
        for kt in range(counts.shape[1]):
            assert k[kt] == set(np.nonzero(counts[:, kt])[0]), (h, "key tile", kt)


def _runs(binary, mode, Lq, Lk, quad, h):
    S, N, G, W = quad
    txt = subprocess.check_output([binary, mode, str(Lq), str(Lk), str(S), str(N), str(G), str(W), str(h),
                                   "0", "0"], text=True)
    out = []
    for line in txt.strip().splitlines():
        v = [int(x) for x in line.split()]
        runs = [(v[2 * i], v[2 * i + 1]) for i in range(3) if v[2 * i] <= v[2 * i + 1]]
        # present runs come first, ascending, with a gap between neighbours
        assert all(v[2 * i] > v[2 * i + 1] for i in range(len(runs), 3))
        assert all(runs[a][1] + 1 < runs[a + 1][0] for a in range(len(runs) - 1))
        out.append(runs)
    return out


@pytest.mark.parametrize("Lq,Lk,quad", [
    (300, 300, (16, 64, 0, 60)), (200, 200, (5, 37, 0, 50)), (120, 250, (3, 20, 0, 110)),
    (250, 90, (0, 30, 7, 20)), (160, 160, (0, 160, 0, 0)), (130, 130, (1, 1, 0, 40)),
    (100, 100, (0, 0, 0, 0)), (140, 140, (200, 0, 0, 3)), (150, 150, (4, 10, 3, 0)),
    (180, 180, (0, 12, 0, 12))])
def test_runs_equal_the_mask(oracle_mod, ranges_bin, Lq, Lk, quad):
    for h in range(4):
        m = oracle_mod.mask(Lq, Lk, h, quad)  # [query row, key]
        rows = _runs(ranges_bin, "r", Lq, Lk, quad, h)
        keys = _runs(ranges_bin, "c", Lq, Lk, quad, h)
        for i in range(Lq):
            got = np.zeros(Lk, bool)
            for a, b in rows[i]:
                assert 0 <= a and b < Lk
                got[a:b + 1] = True
            np.testing.assert_array_equal(got, m[i], err_msg="h %d row %d" % (h, i))
        # key runs are in aligned positions p = i + Lk - Lq, at most Lk - 1
        for j in range(Lk):
            got = np.zeros(Lq, bool)
            for a, b in keys[j]:
                assert b <= Lk - 1
                lo, hi = max(a - (Lk - Lq), 0), b - (Lk - Lq)
                if lo <= hi:
                    got[lo:hi + 1] = True
            np.testing.assert_array_equal(got, m[:, j], err_msg="h %d key %d" % (h, j))
