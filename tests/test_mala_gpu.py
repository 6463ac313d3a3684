"""MALA parity: cowa_mala_fwd / cowa_mala_bwd against the fp64 oracle of
oracle/mala.py (the reading: full causal scoring, blocks of 128 query rows x
64 keys kept when some row gives them at least tau of its softmax mass, the
dropped mass not redistributed, the gradient with the decisions fixed).

The block decision is a threshold on a floating-point sum, so tau is chosen
halfway between two of the oracle's block masses (far from every mass in
both precisions) and the decisions must then agree bit for bit; O, LSE and
the gradients use the operator's tolerances."""
import numpy as np
import pytest
import torch

from helpers import assert_grad, assert_lse, assert_o, to64

pytestmark = pytest.mark.gpu

BM, BN = 128, 64


def block_masses(q, k, scale=None):
    """Largest row mass of every (query block, key block), from the oracle's
    own scores and statistics: [B, Hq, nqt, nkt]."""
    from oracle import mala
    qf, kf = mala._f64(q), mala._f64(k)
    d = qf.shape[-1]
    s, _ = mala._scores(qf, kf, 1.0 / np.sqrt(d) if scale is None else scale)
    _, P = mala._stats(s)
    B, Hq, Lq, Lk = P.shape
    nqt, nkt = -(-Lq // BM), -(-Lk // BN)
    out = np.zeros((B, Hq, nqt, nkt))
    for a in range(nqt):
        for t in range(nkt):
            out[:, :, a, t] = P[:, :, a * BM:(a + 1) * BM, t * BN:(t + 1) * BN].sum(axis=-1).max(axis=-1)
    return out


def tau_between(masses, quantile):
    """A threshold halfway between two neighbouring distinct block masses near
    the quantile, so no mass lies within a relative 1e-3 of it."""
    m = np.unique(masses[masses > 0])
    i = int(np.clip(round(quantile * (len(m) - 1)), 0, len(m) - 2))
    for j in list(range(i, len(m) - 1)) + list(range(i - 1, -1, -1)):
        lo, hi = m[j], m[j + 1]
        if hi - lo > 4e-3 * hi:
            return 0.5 * (lo + hi)
    raise AssertionError("no threshold with a margin")


CASES = [  # B, Lq, Lk, Hq, Hkv, d, spread of q (sharper softmax)
    (1, 300, 300, 4, 2, 64, 2.0),
    (2, 200, 200, 2, 1, 128, 1.5),
    (1, 130, 400, 4, 4, 128, 2.0),   # chunked prefill: Lq < Lk
    (1, 257, 257, 8, 2, 64, 3.0),
    (1, 700, 700, 6, 2, 128, 2.0),   # g = 3: head pairs and a lone head; several 128-key tiles
    (1, 300, 130, 4, 2, 128, 2.0),   # Lq > Lk: the first rows see no key (O = 0, LSE = -inf)
    (2, 260, 100, 2, 1, 64, 2.0),    # the same at d = 64
]


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,spread", CASES)
@pytest.mark.parametrize("quantile", [0.3, 0.7])
def test_mala_matches_oracle(B, Lq, Lk, Hq, Hkv, d, spread, quantile):
    import structured_sparse_attention_block_b200 as cowa
    from oracle import mala
    from structured_sparse_attention_block_b200.inputs import bf16_bits, training_inputs
    q, k, v, do = training_inputs(B, Lq, Lk, Hq, Hkv, d, seed=Lq * 3 + Hq)
    q = (q.float() * spread).to(torch.bfloat16)
    qb, kb, vb, db = (bf16_bits(x) for x in (q, k, v, do))
    tau = tau_between(block_masses(qb, kb), quantile)
    o, lse, keep = cowa.cowa_mala_fwd(q, k, v, tau)
    dq, dk, dv = cowa.cowa_mala_bwd(q, k, v, o, lse, keep, do)
    torch.cuda.synchronize()
    assert cowa.lib().cowa_get_device_error(None) == 0
    o_ref, lse_ref, keep_ref, _ = mala.fwd(qb, kb, vb, tau, BM, BN)
    got_keep = keep.cpu().numpy().astype(bool)
    assert got_keep.shape == keep_ref.shape
    assert np.array_equal(got_keep, keep_ref), "block decisions differ at %s" % (
        np.argwhere(got_keep != keep_ref)[:4].tolist(),)
    assert 0 < keep_ref.sum() < np.prod(keep_ref.shape), "tau keeps all or none"
    assert_o(o, o_ref)
    assert_lse(lse, lse_ref)
    rq, rk, rv = mala.bwd(qb, kb, vb, db, tau, BM, BN)
    assert_grad(dq, rq, "dQ")
    assert_grad(dk, rk, "dK")
    assert_grad(dv, rv, "dV")


def test_mala_tau_zero_is_dense_causal():
    """tau = 0 keeps every causal block: the output is the library's own
    dense causal forward (the full-causal CoWA quadruple) up to rounding,
    and every causal block is marked kept."""
    import structured_sparse_attention_block_b200 as cowa
    from oracle import mala
    from structured_sparse_attention_block_b200.inputs import bf16_bits, training_inputs
    B, L, Hq, Hkv, d = 1, 333, 4, 2, 128
    q, k, v, _ = training_inputs(B, L, L, Hq, Hkv, d, seed=4)
    o, lse, keep = cowa.cowa_mala_fwd(q, k, v, 0.0)
    torch.cuda.synchronize()
    o_ref, lse_ref, keep_ref, _ = mala.fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), 0.0, BM, BN)
    # blocks holding a causal pair are all kept; a block past the diagonal
    # holds no pair (the oracle's max over an empty mass is 0 >= 0), and the
    # library marks it 0
    nqt, nkt = keep_ref.shape[2:]
    causal = np.array([[t * BN <= min(L, (a + 1) * BM) - 1 for t in range(nkt)] for a in range(nqt)])
    got = keep.cpu().numpy().astype(bool)
    assert np.array_equal(got[:, :, causal], keep_ref[:, :, causal]) and got[:, :, causal].all()
    assert not got[:, :, ~causal].any()
    assert_o(o, o_ref)
    assert_lse(lse, lse_ref)


def test_mala_tau_above_one_keeps_nothing():
    import structured_sparse_attention_block_b200 as cowa
    from oracle import mala
    from structured_sparse_attention_block_b200.inputs import bf16_bits, training_inputs
    q, k, v, do = training_inputs(1, 200, 200, 4, 2, 64, seed=5)
    o, lse, keep = cowa.cowa_mala_fwd(q, k, v, 1.5)
    dq, dk, dv = cowa.cowa_mala_bwd(q, k, v, o, lse, keep, do)
    torch.cuda.synchronize()
    assert int(keep.sum()) == 0 and torch.all(o == 0)
    _, lse_ref, _, _ = mala.fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), 1.5, BM, BN)
    assert_lse(lse, lse_ref)
    # O = 0 gives delta = 0; dP and dV vanish with every block skipped, so
    # every gradient is exactly zero
    assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)


def test_mala_rejects_bad_arguments():
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import training_inputs
    q, k, v, _ = training_inputs(1, 64, 64, 2, 1, 64, seed=6)
    for tau in (-0.1, float("nan"), float("inf")):
        with pytest.raises(cowa.CowaError):
            cowa.cowa_mala_fwd(q, k, v, tau)


def test_mala_workload_sampled_blocks():
    """The bench's MALA workload at full size (the 14B-like 32K shape, tau =
    2^-8, the same seed) in the launch configuration the bench times; sampled
    query blocks of 128 rows, one head each, against the oracle run on just
    those rows and their causal keys (rows [i0, i0 + 128) with keys
    [0, i0 + 128) keep the bottom-right alignment of the full problem).
    Decisions must agree wherever the oracle's block mass is not within 0.1 %
    of tau; O, LSE and the rows' dQ use the operator's tolerances (compared
    only when no decision of the block is that close)."""
    import structured_sparse_attention_block_b200 as cowa
    from oracle import mala
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, bf16_bits, workload_inputs
    wl = WORKLOADS["llm14b_32k"]
    tau = 2.0 ** -8
    q, k, v, do = workload_inputs(wl, seed=11)
    o, lse, keep = cowa.cowa_mala_fwd(q, k, v, tau)
    dq, _, _ = cowa.cowa_mala_bwd(q, k, v, o, lse, keep, do)
    torch.cuda.synchronize()
    assert cowa.lib().cowa_get_device_error(None) == 0
    g = wl.Hq // wl.Hkv
    nqt = -(-wl.Lq // BM)
    compared = 0
    for qb, hq in [(nqt - 1, 0), (nqt // 2, 21), (3, 39), (nqt - 2, 17)]:
        i0 = qb * BM
        rows = slice(i0, min(i0 + BM, wl.Lq))
        nk = min(i0 + BM, wl.Lk)
        h = hq // g
        q1 = bf16_bits(q[:, rows, hq:hq + 1])
        k1, v1 = bf16_bits(k[:, :nk, h:h + 1]), bf16_bits(v[:, :nk, h:h + 1])
        do1 = bf16_bits(do[:, rows, hq:hq + 1])
        o_ref, lse_ref, keep_ref, _ = mala.fwd(q1, k1, v1, tau, BM, BN)
        masses = block_masses(q1, k1)[0, 0, 0]
        got = keep[0, hq, qb].cpu().numpy().astype(bool)
        nb = keep_ref.shape[-1]
        near = np.abs(masses - tau) <= 1e-3 * tau
        assert np.array_equal(got[:nb][~near], keep_ref[0, 0, 0][~near]), "block decisions differ (block %d, head %d)" % (qb, hq)
        assert not got[nb:].any(), "a block past the causal diagonal is kept"
        if near.any():
            continue
        assert_o(o[:, rows, hq:hq + 1], o_ref)
        assert_lse(lse[:, hq:hq + 1, rows], lse_ref)
        rq, _, _ = mala.bwd(q1, k1, v1, do1, tau, BM, BN)
        assert_grad(dq[:, rows, hq:hq + 1], rq, "dQ")
        compared += 1
    assert compared >= 2
