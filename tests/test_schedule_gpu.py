"""The visible-tile schedule the kernels walk, checked bit-exactly against the
oracle's brute-force visible-pair counts.

For every tile: skipped iff it holds no visible pair; unmasked iff every
in-range pair is visible and none of its columns lies past Lk; otherwise
masked.  This covers both the tile set (no invisible tile visited, none
missed, none twice -- the ranges are disjoint by construction and checked
here too) and the mask-free labels.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

def expected_classes(oracle_mod, Lq, Lk, h, quad, BM, BN):
    counts = oracle_mod.tile_counts(Lq, Lk, h, quad, BM, BN)
    nqt, nkt = counts.shape
    rows = np.minimum(BM, Lq - np.arange(nqt) * BM)[:, None]
    cols_in = (np.arange(nkt) * BN + BN <= Lk)[None, :]
    full = (counts == rows * BN) & cols_in
    return np.where(counts == 0, 0, np.where(full, 2, 1)).astype(np.uint8)


SMALL = [  # Lq, Lk, Hkv, quad
    (512, 512, 2, (16, 64, 0, 224)),
    (200, 200, 3, (5, 37, 0, 50)),
    (77, 300, 4, (16, 40, 3, 60)),
    (300, 130, 2, (3, 20, 0, 110)),
    (256, 256, 4, (0, 17, 5, 9)),
    (384, 384, 1, (0, 384, 0, 0)),
    (1000, 1000, 8, (1, 1, 0, 125)),
    (640, 640, 2, (64, 128, 0, 256)),
    (129, 129, 2, (0, 0, 0, 65)),
    (513, 1025, 3, (70, 0, 10, 0)),
]


# the tilings the kernels use: forward 128x128 (an earlier d=64 forward used 128x96);
# backward dQ 128x64, dK/dV key-tile major over 128 keys with 64 (d=64) or
# 32 (d=128) query rows per task; MALA blocks 128x64; and smaller tilings
TILINGS = [(128, 96, False), (128, 64, False), (128, 128, False), (64, 128, True), (32, 128, True),
           (64, 64, False), (32, 64, True), (64, 64, True)]


@pytest.mark.parametrize("Lq,Lk,Hkv,quad", SMALL)
@pytest.mark.parametrize("BM,BN,transposed", TILINGS)
def test_schedule_small(oracle_mod, Lq, Lk, Hkv, quad, BM, BN, transposed):
    import structured_sparse_attention_block_b200 as cowa
    for h in range(Hkv):
        got = cowa.cowa_tile_classes(Lq, Lk, h, quad, BM, BN, transposed).cpu().numpy()
        exp = expected_classes(oracle_mod, Lq, Lk, h, quad, BM, BN)
        np.testing.assert_array_equal(got, exp, err_msg="head %d" % h)


@pytest.mark.parametrize("name,heads", [("recall8k", None), ("llm14b_32k", None), ("op128k", (0, 7))])
def test_schedule_workloads(oracle_mod, name, heads):
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import WORKLOADS
    wl = WORKLOADS[name]
    heads = range(wl.Hkv) if heads is None else heads
    for h in heads:
        for BM, BN, tr in [(128, 96 if wl.d == 64 else 64, False), (128, 64 if wl.d == 64 else 128, False),
                           (64 if wl.d == 64 else 32, 128, True)]:
            got = cowa.cowa_tile_classes(wl.Lq, wl.Lk, h, wl.quad, BM, BN, tr).cpu().numpy()
            exp = expected_classes(oracle_mod, wl.Lq, wl.Lk, h, wl.quad, BM, BN)
            np.testing.assert_array_equal(got, exp, err_msg="%s head %d BM %d" % (name, h, BM))
