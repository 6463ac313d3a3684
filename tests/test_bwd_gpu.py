"""Backward parity: cowa_bwd against the oracle's analytic gradients on the
same bf16 inputs; dQ, dK, dV within max-abs 2e-2 * max|ref|.  The GPU
backward consumes the GPU forward's O and LSE, as a training step does."""
import numpy as np
import pytest
import torch

from helpers import assert_grad, sample_rows

pytestmark = pytest.mark.gpu

CASES = [  # B, Lq, Lk, Hq, Hkv, d, quad
    (1, 512, 512, 4, 2, 64, (16, 64, 0, 224)),       # the tiny workload
    (2, 200, 200, 6, 3, 64, (5, 37, 0, 50)),
    (1, 77, 300, 4, 4, 128, (16, 40, 3, 60)),
    (1, 300, 130, 2, 1, 64, (3, 20, 0, 110)),
    (1, 256, 256, 8, 4, 128, (0, 17, 5, 9)),
    (1, 384, 384, 2, 2, 128, (0, 384, 0, 0)),
    (1, 130, 130, 2, 2, 64, (0, 0, 0, 0)),
    (2, 700, 700, 8, 2, 128, (32, 100, 0, 300)),
]


def fwd_bwd(q, k, v, dout, quad, **kw):
    import structured_sparse_attention_block_b200 as cowa
    o, lse = cowa.cowa_fwd(q, k, v, quad, **kw)
    dq, dk, dv = cowa.cowa_bwd(q, k, v, o, lse, dout, quad, **kw)
    torch.cuda.synchronize()
    return dq, dk, dv


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,quad", CASES)
def test_bwd_matches_oracle(oracle_mod, B, Lq, Lk, Hq, Hkv, d, quad):
    from structured_sparse_attention_block_b200.inputs import bf16_bits, training_inputs
    q, k, v, do = training_inputs(B, Lq, Lk, Hq, Hkv, d, seed=B * 11 + Lk)
    dq, dk, dv = fwd_bwd(q, k, v, do, quad)
    rq, rk, rv = oracle_mod.bwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(do), quad)
    assert_grad(dq, rq, "dQ")
    assert_grad(dk, rk, "dK")
    assert_grad(dv, rv, "dV")


def test_bwd_strided_and_offset_heads(oracle_mod):
    from structured_sparse_attention_block_b200.inputs import bf16_bits
    B, L, Hq, Hkv, d = 1, 333, 4, 2, 128
    g = torch.Generator().manual_seed(9)
    packed = torch.randn(B, L, Hq + 2 * Hkv, d, generator=g).to(torch.bfloat16).cuda()
    q, k, v = packed[:, :, :Hq], packed[:, :, Hq:Hq + Hkv], packed[:, :, Hq + Hkv:]
    do = torch.randn(B, L, Hq, d, generator=g).to(torch.bfloat16).cuda()
    quad = (7, 30, 0, 40)
    import structured_sparse_attention_block_b200 as cowa
    o, lse = cowa.cowa_fwd(q, k, v, quad, kv_head_offset=5)
    dq, dk, dv = cowa.cowa_bwd(q, k, v, o, lse, do, quad, kv_head_offset=5)
    torch.cuda.synchronize()
    rq, rk, rv = oracle_mod.bwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(do), quad,
                                kv_head_offset=5)
    assert_grad(dq, rq, "dQ")
    assert_grad(dk, rk, "dK")
    assert_grad(dv, rv, "dV")


def key_columns(wl, per_head, seed):
    """(b, h, j): the last columns of every KV head, seen by few rows."""
    rng = np.random.default_rng(seed)
    cols = []
    for h in range(wl.Hkv):
        for j in range(wl.Lk - per_head, wl.Lk):
            cols.append((int(rng.integers(0, wl.B)), h, j))
    return cols


def heavy_columns(wl, heads, sink=True):
    """(b, h, j): a sink column (every query row sees it: the longest dK/dV
    CTA) and a column in the middle of the long window of the last query
    row, for each of `heads`."""
    S, N, G, W = wl.quad
    cols = []
    for n, h in enumerate(heads):
        b = n % wl.B
        if sink and S > 0:
            cols.append((b, h, min(S - 1, 3 + n)))
        c = N + G + h * W
        j = wl.Lk - 1 - (c + W // 2)
        if W > 0 and j >= S:
            cols.append((b, h, j))
    return cols


# the heavy columns: recall8k and llm14b_32k with sink columns; at op128k a
# sink column needs every one of the 524288 (row, query head) forwards of its
# KV head (about two minutes of the oracle), so there the long-window columns
# are compared element by element and the sink columns through the sums below
HEAVY = {"recall8k": ((1, 2), True), "llm14b_32k": ((0, 5), True), "op128k": ((1, 6), False)}


@pytest.mark.parametrize("name,per_head,ncols", [("recall8k", 32, 24), ("llm14b_32k", 6, 8),
                                                 ("op128k", 3, 4)])
def test_bwd_workloads_sampled(oracle_mod, name, per_head, ncols):
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, bf16_bits, workload_inputs
    wl = WORKLOADS[name]
    q, k, v, do = workload_inputs(wl, seed=0)
    dq, dk, dv = fwd_bwd(q, k, v, do, wl.quad)
    qb, kb, vb, db = (bf16_bits(x) for x in (q, k, v, do))
    rows = sample_rows(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.quad, per_head, seed=2)
    rq = oracle_mod.bwd_dq_rows(qb, kb, vb, db, wl.quad, rows)
    b, hq, i = (torch.tensor([r[a] for r in rows], device=q.device) for a in range(3))
    assert_grad(dq[b, i, hq], rq, "dQ rows")
    # few-row columns through the per-column C loops, the heavy columns
    # through the chunked form of the same definitions
    for cols, fn in ((key_columns(wl, ncols, seed=3), oracle_mod.bwd_dkv_cols),
                     (heavy_columns(wl, *HEAVY[name]), oracle_mod.bwd_dkv_cols_fast)):
        rk, rv = fn(qb, kb, vb, db, wl.quad, cols)
        cb, ch, cj = (torch.tensor([c[a] for c in cols], device=q.device) for a in range(3))
        # the tolerance scale is the largest |gradient| among the sampled columns
        assert_grad(dk[cb, cj, ch], rk, "dK cols %s" % cols[:2])
        assert_grad(dv[cb, cj, ch], rv, "dV cols %s" % cols[:2])
    # properties at any size, over every column (the sink columns included):
    # sum_j dK_j = 0 per (b, KV head), because the outputs do not change when
    # one vector is added to every key; sum_j dV_j = sum over the group's rows
    # of dO, because every row's probabilities sum to one (every row of these
    # workloads sees at least one key).  bf16 rounding of dK, dV leaves a
    # residue far below 1 % of the sums of magnitudes.
    dkf, dvf = dk.float(), dv.float()
    assert (dkf.sum(dim=1).abs() <= 1e-2 * dkf.abs().sum(dim=1) + 1e-6).all()
    g = wl.Hq // wl.Hkv
    want = do.float().sum(dim=1).view(wl.B, wl.Hkv, g, wl.d).sum(dim=2)
    assert ((dvf.sum(dim=1) - want).abs() <= 1e-2 * dvf.abs().sum(dim=1) + 1e-3).all()


@pytest.mark.parametrize("Lq,Lk", [(0, 200), (150, 0)])
def test_no_queries_or_no_keys_gives_zero_gradients(Lq, Lk):
    import structured_sparse_attention_block_b200 as cowa
    B, Hq, Hkv, d = 2, 4, 2, 128
    q = torch.randn(B, Lq, Hq, d, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, Lk, Hkv, d, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, Lk, Hkv, d, device="cuda").to(torch.bfloat16)
    o = torch.randn(B, Lq, Hq, d, device="cuda").to(torch.bfloat16)
    do = torch.randn(B, Lq, Hq, d, device="cuda").to(torch.bfloat16)
    lse = torch.full((B, Hq, Lq), float("-inf"), device="cuda")
    dq = torch.full_like(q, 3.0)
    dk, dv = torch.full_like(k, 3.0), torch.full_like(v, 3.0)
    cowa.cowa_bwd(q, k, v, o, lse, do, (4, 16, 0, 8), dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)
