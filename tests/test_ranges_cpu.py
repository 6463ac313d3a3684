"""The tile ranges each tcgen05 CTA computes for itself (query_tile_ranges /
key_tile_ranges in csrc/common.cuh, built here for the host): for every
query tile, the key tiles it visits are exactly those holding at least one
visible pair in the oracle's brute-force tile counts, and likewise for every
key tile and the query tiles that see it; the ranges are ascending, disjoint
and at most three.  Runs without a GPU (nvcc compiles host code)."""
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
