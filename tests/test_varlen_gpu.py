"""Packed (variable-length) batches: every sequence of a packed forward and
backward equals the oracle run on that sequence alone (each aligned
bottom-right on its own: the pages' one position rule for training, prefill
and decoding), a packed batch of equal lengths reproduces the uniform-batch
path bit for bit, and offsets that do not fit the tensors are reported on
the device without any access outside them."""
import numpy as np
import pytest
import torch

from helpers import assert_grad, assert_lse, assert_o, to64

pytestmark = pytest.mark.gpu

SEQS = [(200, 200), (1, 57), (300, 431), (0, 10), (129, 129), (77, 300)]


def _packed_inputs(seqs, Hq, Hkv, d, seed):
    from structured_sparse_attention_block_b200.inputs import training_inputs
    Tq, Tk = sum(a for a, _ in seqs), sum(b for _, b in seqs)
    q, k, v, do = (t[0] for t in training_inputs(1, Tq, Tk, Hq, Hkv, d, seed=seed))
    cu_q = np.concatenate([[0], np.cumsum([a for a, _ in seqs])]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum([b for _, b in seqs])]).astype(np.int32)
    return q, k, v, do, cu_q, cu_k


@pytest.mark.parametrize("d", [64, 128])
def test_packed_sequences_match_the_oracle(oracle_mod, d):
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import bf16_bits
    Hq, Hkv, quad = 4, 2, (8, 40, 0, 80)
    q, k, v, do, cu_q, cu_k = _packed_inputs(SEQS, Hq, Hkv, d, seed=d)
    mq, mk = max(a for a, _ in SEQS), max(b for _, b in SEQS)
    cq, ck = torch.tensor(cu_q, device="cuda"), torch.tensor(cu_k, device="cuda")
    o, lse = cowa.cowa_fwd_varlen(q, k, v, cq, ck, mq, mk, quad)
    dq, dk, dv = cowa.cowa_bwd_varlen(q, k, v, o, lse, do, cq, ck, mq, mk, quad)
    torch.cuda.synchronize()
    cowa.cowa_get_device_error()
    for b, (Lq, Lk) in enumerate(SEQS):
        qs, qe, ks, ke = cu_q[b], cu_q[b + 1], cu_k[b], cu_k[b + 1]
        if Lq == 0:
            assert torch.all(dk[ks:ke] == 0) and torch.all(dv[ks:ke] == 0)
            continue
        args = [bf16_bits(t.unsqueeze(0)) for t in (q[qs:qe], k[ks:ke], v[ks:ke])]
        o_ref, lse_ref = oracle_mod.fwd(*args, quad)
        assert_o(o[qs:qe], o_ref[0], what="O of sequence %d" % b)
        assert_lse(lse[:, qs:qe], lse_ref[0], what="LSE of sequence %d" % b)
        rq, rk, rv = oracle_mod.bwd(*args, bf16_bits(do[qs:qe].unsqueeze(0)), quad)
        assert_grad(dq[qs:qe], rq[0], "dQ of sequence %d" % b)
        assert_grad(dk[ks:ke], rk[0], "dK of sequence %d" % b)
        assert_grad(dv[ks:ke], rv[0], "dV of sequence %d" % b)


def test_packed_equal_lengths_reproduce_the_uniform_batch():
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import training_inputs
    B, Lq, Lk, Hq, Hkv, d, quad = 3, 333, 520, 8, 4, 64, (16, 96, 0, 120)
    q, k, v, do = training_inputs(B, Lq, Lk, Hq, Hkv, d, seed=9)
    o_u, lse_u = cowa.cowa_fwd(q, k, v, quad)
    g_u = cowa.cowa_bwd(q, k, v, o_u, lse_u, do, quad)
    cq = torch.arange(0, (B + 1) * Lq, Lq, dtype=torch.int32, device="cuda")
    ck = torch.arange(0, (B + 1) * Lk, Lk, dtype=torch.int32, device="cuda")
    flat = lambda t: t.reshape(-1, t.shape[2], t.shape[3])
    o_p, lse_p = cowa.cowa_fwd_varlen(flat(q), flat(k), flat(v), cq, ck, Lq, Lk, quad)
    g_p = cowa.cowa_bwd_varlen(flat(q), flat(k), flat(v), o_p, lse_p, flat(do), cq, ck, Lq, Lk, quad)
    torch.cuda.synchronize()
    cowa.cowa_get_device_error()
    assert torch.equal(o_p, flat(o_u))
    assert torch.equal(lse_p, lse_u.permute(1, 0, 2).reshape(Hq, B * Lq))
    for a, b_ in zip(g_p, g_u):
        assert torch.equal(a, flat(b_))


def test_offsets_outside_the_tensors_are_reported():
    import structured_sparse_attention_block_b200 as cowa
    seqs = [(64, 64), (64, 64)]
    q, k, v, do, cu_q, cu_k = _packed_inputs(seqs, 4, 2, 64, seed=1)
    bad = torch.tensor([0, 64, 200], dtype=torch.int32, device="cuda")  # beyond the 128 rows
    ck = torch.tensor(cu_k, device="cuda")
    o, lse = cowa.cowa_fwd_varlen(q, k, v, bad, ck, 128, 64, quad=(4, 16, 0, 24))
    torch.cuda.synchronize()
    with pytest.raises(cowa.CowaError, match="COWA_ERR_DEVICE"):
        cowa.cowa_get_device_error()
