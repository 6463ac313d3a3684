"""Pins of the oracle's attention arithmetic.

The pages define CoWA as ordinary softmax attention restricted to each
head's windows ("CoWindow Attention: Full Causal Coverage Is a Collective
Property", abstract and the digest's method key points), used the same way
in training, prefill and decoding through bottom-right-aligned causal
distance.  These tests pin the oracle to things other than itself:

* special cases that are textbook dense causal / sliding-window / sink-only
  attention, computed here by an independent numpy implementation;
* fp64 central finite differences of the forward for the gradients;
* identities every exact implementation satisfies (key translation
  invariance, probability normalisation, value shift);
* consistency of the three entry points (training rows, chunked prefill with
  Lq < Lk, decode) and of the global KV-head index and GQA grouping.
"""
import math

import numpy as np
import pytest


def rand(rng, *shape):
    return rng.standard_normal(shape)


def textbook_attention(q, k, v, allowed, scale):
    """Dense masked softmax attention in numpy, one (b, head) at a time.

    q [Lq, d], k/v [Lk, d], allowed [Lq, Lk] bool.  Rows with no allowed key
    give O = 0 and LSE = -inf.
    """
    s = (q @ k.T) * scale
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    empty = ~allowed.any(axis=1)
    m[empty] = 0.0
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    z[empty] = 1.0
    o = (e / z) @ v
    lse = (m + np.log(z))[:, 0]
    lse[empty] = -np.inf
    o[empty] = 0.0
    return o, lse


def textbook_all_heads(q, k, v, allowed_fn, scale):
    B, Lq, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for hq in range(Hq):
            h = hq // g
            o[b, :, hq], lse[b, hq] = textbook_attention(
                q[b, :, hq], k[b, :, h], v[b, :, h], allowed_fn(h), scale)
    return o, lse


def causal(Lq, Lk):
    return np.tril(np.ones((Lq, Lk), dtype=bool), k=Lk - Lq)


SHAPES = [  # B, Lq, Lk, Hq, Hkv, d
    (2, 37, 37, 4, 2, 16),
    (1, 20, 45, 6, 3, 8),
    (1, 45, 20, 2, 2, 8),
    (1, 1, 30, 4, 1, 16),
]


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d", SHAPES)
def test_near_window_covering_everything_is_dense_causal(oracle_mod, B, Lq, Lk, Hq, Hkv, d):
    rng = np.random.default_rng(1)
    q, k, v = rand(rng, B, Lq, Hq, d), rand(rng, B, Lk, Hkv, d), rand(rng, B, Lk, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle_mod.fwd(q, k, v, (3, Lk, 2, 5), scale)
    o_t, lse_t = textbook_all_heads(q, k, v, lambda h: causal(Lq, Lk), scale)
    np.testing.assert_allclose(o, o_t, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(lse), np.isinf(lse_t))
    fin = np.isfinite(lse_t)
    np.testing.assert_allclose(lse[fin], lse_t[fin], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N", [0, 1, 6])
def test_single_kv_head_with_full_long_window_is_dense_causal(oracle_mod, N):
    rng = np.random.default_rng(2)
    B, L, Hq, d = 1, 41, 3, 8
    q, k, v = rand(rng, B, L, Hq, d), rand(rng, B, L, 1, d), rand(rng, B, L, 1, d)
    W = L - N
    o, lse = oracle_mod.fwd(q, k, v, (0, N, 0, W), 0.7)
    o_t, lse_t = textbook_all_heads(q, k, v, lambda h: causal(L, L), 0.7)
    np.testing.assert_allclose(o, o_t, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_t, rtol=1e-12, atol=1e-12)


def test_head0_with_w_beyond_length_is_dense_causal(oracle_mod):
    """W >= Lk: KV head 0's long window reaches back to the start, so head 0
    is dense causal; heads >= 1 keep only their sink and near windows."""
    rng = np.random.default_rng(3)
    B, L, Hq, Hkv, d = 1, 50, 4, 2, 8
    q, k, v = rand(rng, B, L, Hq, d), rand(rng, B, L, Hkv, d), rand(rng, B, L, Hkv, d)
    quad = (4, 6, 0, L)
    o, lse = oracle_mod.fwd(q, k, v, quad)
    o_t, _ = textbook_all_heads(q, k, v, lambda h: causal(L, L), 1 / math.sqrt(d))
    np.testing.assert_allclose(o[:, :, :2], o_t[:, :, :2], rtol=1e-12, atol=1e-12)
    o_w0, _ = oracle_mod.fwd(q, k, v, (4, 6, 0, 0))
    np.testing.assert_allclose(o[:, :, 2:], o_w0[:, :, 2:], rtol=1e-12, atol=1e-12)


def test_sliding_window_special_case(oracle_mod):
    """S = 0, W = 0: textbook sliding-window attention of width N."""
    rng = np.random.default_rng(4)
    B, Lq, Lk, Hq, Hkv, d, N = 1, 30, 44, 2, 1, 8, 7
    q, k, v = rand(rng, B, Lq, Hq, d), rand(rng, B, Lk, Hkv, d), rand(rng, B, Lk, Hkv, d)
    band = causal(Lq, Lk) & ~np.tril(np.ones((Lq, Lk), dtype=bool), k=Lk - Lq - N)
    o, lse = oracle_mod.fwd(q, k, v, (0, N, 0, 0), 0.5)
    o_t, lse_t = textbook_all_heads(q, k, v, lambda h: band, 0.5)
    np.testing.assert_allclose(o, o_t, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_t, rtol=1e-12, atol=1e-12)


def test_sink_only_special_case(oracle_mod):
    """N = 0, W = 0: each row attends to the first S keys it can see."""
    rng = np.random.default_rng(5)
    B, L, Hq, Hkv, d, S = 1, 25, 2, 2, 8, 5
    q, k, v = rand(rng, B, L, Hq, d), rand(rng, B, L, Hkv, d), rand(rng, B, L, Hkv, d)
    cols = np.zeros((L, L), dtype=bool)
    cols[:, :S] = True
    o, lse = oracle_mod.fwd(q, k, v, (S, 0, 0, 0), 0.9)
    o_t, lse_t = textbook_all_heads(q, k, v, lambda h: cols & causal(L, L), 0.9)
    np.testing.assert_allclose(o, o_t, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_t, rtol=1e-12, atol=1e-12)


def test_empty_rows(oracle_mod):
    """Rows that see nothing (Lq > Lk, or an all-zero quadruple)."""
    rng = np.random.default_rng(6)
    q, k, v = rand(rng, 1, 12, 2, 8), rand(rng, 1, 5, 1, 8), rand(rng, 1, 5, 1, 8)
    o, lse = oracle_mod.fwd(q, k, v, (1, 2, 0, 1))
    assert np.isneginf(lse[:, :, :7]).all() and (o[:, :7] == 0).all()
    assert np.isfinite(lse[:, :, 7:]).all()
    o, lse = oracle_mod.fwd(q, k, v, (0, 0, 0, 0))
    assert np.isneginf(lse).all() and (o == 0).all()
    dq, dk, dv = oracle_mod.bwd(q, k, v, rand(rng, 1, 12, 2, 8), (0, 0, 0, 0))
    assert (dq == 0).all() and (dk == 0).all() and (dv == 0).all()


FD_CASES = [  # B, Lq, Lk, Hq, Hkv, d, quad
    (1, 24, 24, 4, 2, 8, (2, 3, 1, 4)),
    (1, 16, 29, 2, 2, 4, (3, 4, 0, 5)),
    (2, 11, 11, 2, 1, 4, (0, 2, 2, 3)),
]


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,quad", FD_CASES)
def test_gradients_match_finite_differences(oracle_mod, B, Lq, Lk, Hq, Hkv, d, quad):
    """Analytic dQ, dK, dV vs central differences of L = sum(O * dO)."""
    rng = np.random.default_rng(7)
    q, k, v = rand(rng, B, Lq, Hq, d), rand(rng, B, Lk, Hkv, d), rand(rng, B, Lk, Hkv, d)
    do = rand(rng, B, Lq, Hq, d)
    scale = 0.6
    dq, dk, dv = oracle_mod.bwd(q, k, v, do, quad, scale)

    def loss(q_, k_, v_):
        o, _ = oracle_mod.fwd(q_, k_, v_, quad, scale)
        return float((o * do).sum())

    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = x[idx]
            x[idx] = orig + eps
            lp = loss(q, k, v)
            x[idx] = orig - eps
            lm = loss(q, k, v)
            x[idx] = orig
            fd[idx] = (lp - lm) / (2 * eps)
        err = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert err < 1e-6, (name, err)
        assert np.abs(grad).max() > 1e-3, name


def test_gradient_identities(oracle_mod):
    """Exact identities of softmax attention:
    * adding one vector to every key leaves every output unchanged, so the
      dK of each (batch, KV head) sums to zero over keys;
    * probabilities of a row sum to one, so sum_j dV_j = sum of dO over the
      group's rows that see any key;
    * adding a vector c to every value shifts each non-empty row's O by c."""
    rng = np.random.default_rng(8)
    B, Lq, Lk, Hq, Hkv, d = 2, 40, 40, 4, 2, 8
    quad = (3, 5, 0, 9)
    q, k, v = rand(rng, B, Lq, Hq, d), rand(rng, B, Lk, Hkv, d), rand(rng, B, Lk, Hkv, d)
    do = rand(rng, B, Lq, Hq, d)
    dq, dk, dv = oracle_mod.bwd(q, k, v, do, quad)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    g = Hq // Hkv
    do_grouped = do.reshape(B, Lq, Hkv, g, d).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), do_grouped, rtol=1e-12, atol=1e-12)
    c = rand(rng, d)
    o, _ = oracle_mod.fwd(q, k, v, quad)
    o2, _ = oracle_mod.fwd(q, k, v + c, quad)
    np.testing.assert_allclose(o2 - o, np.broadcast_to(c, o.shape), atol=1e-12)


def test_chunked_prefill_equals_training_rows(oracle_mod):
    """Bottom-right alignment: a query chunk (Lq < Lk) equals the last Lq
    rows of the full training forward and backward (dQ rows)."""
    rng = np.random.default_rng(9)
    B, L, Hq, Hkv, d, Lq = 1, 48, 4, 2, 8, 13
    quad = (2, 6, 1, 10)
    q, k, v = rand(rng, B, L, Hq, d), rand(rng, B, L, Hkv, d), rand(rng, B, L, Hkv, d)
    o, lse = oracle_mod.fwd(q, k, v, quad)
    o_c, lse_c = oracle_mod.fwd(q[:, -Lq:], k, v, quad)
    np.testing.assert_allclose(o_c, o[:, -Lq:], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse_c, lse[:, :, -Lq:], rtol=1e-13, atol=1e-13)


def test_decode_equals_last_row(oracle_mod):
    """Decode over a cache with per-sequence lengths equals the last row of a
    forward over the first seqlens[b] keys."""
    rng = np.random.default_rng(10)
    B, Lcap, Hq, Hkv, d = 3, 40, 4, 2, 8
    quad = (2, 5, 0, 9)
    kc, vc = rand(rng, B, Lcap, Hkv, d), rand(rng, B, Lcap, Hkv, d)
    qd = rand(rng, B, Hq, d)
    seqlens = np.array([40, 17, 1], dtype=np.int32)
    o, lse = oracle_mod.decode(qd, kc, vc, seqlens, quad)
    for b in range(B):
        L = int(seqlens[b])
        o_f, lse_f = oracle_mod.fwd(qd[b:b + 1, None], kc[b:b + 1, :L], vc[b:b + 1, :L], quad)
        np.testing.assert_allclose(o[b], o_f[0, 0], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse[b], lse_f[0, :, 0], rtol=1e-13, atol=1e-13)
    o0, lse0 = oracle_mod.decode(qd, kc, vc, np.array([0, 0, 3], np.int32), quad)
    assert (o0[:2] == 0).all() and np.isneginf(lse0[:2]).all()


def test_global_kv_head_index_and_gqa_grouping(oracle_mod):
    """Running one KV head's slice with kv_head_offset = h reproduces that
    head's outputs of the full run: windows follow the global KV-head index
    and query heads g*h .. g*h+g-1 belong to KV head h."""
    rng = np.random.default_rng(11)
    B, L, Hq, Hkv, d = 1, 36, 6, 3, 8
    g = Hq // Hkv
    quad = (2, 4, 0, 11)
    q, k, v = rand(rng, B, L, Hq, d), rand(rng, B, L, Hkv, d), rand(rng, B, L, Hkv, d)
    do = rand(rng, B, L, Hq, d)
    o, lse = oracle_mod.fwd(q, k, v, quad)
    dq, dk, dv = oracle_mod.bwd(q, k, v, do, quad)
    for h in range(Hkv):
        sl = slice(g * h, g * h + g)
        o_h, lse_h = oracle_mod.fwd(q[:, :, sl], k[:, :, h:h + 1], v[:, :, h:h + 1], quad,
                                    kv_head_offset=h)
        np.testing.assert_allclose(o_h, o[:, :, sl], rtol=1e-13, atol=1e-13)
        dq_h, dk_h, dv_h = oracle_mod.bwd(q[:, :, sl], k[:, :, h:h + 1], v[:, :, h:h + 1],
                                          do[:, :, sl], quad, kv_head_offset=h)
        np.testing.assert_allclose(dq_h, dq[:, :, sl], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(dk_h, dk[:, :, h:h + 1], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(dv_h, dv[:, :, h:h + 1], rtol=1e-13, atol=1e-13)
    # heads really differ: the offset changes the outputs
    o_wrong, _ = oracle_mod.fwd(q[:, :, :g], k[:, :, 1:2], v[:, :, 1:2], quad, kv_head_offset=0)
    assert np.abs(o_wrong - o[:, :, g:2 * g]).max() > 1e-3


def test_sampled_entry_points_match_full(oracle_mod):
    rng = np.random.default_rng(12)
    B, L, Hq, Hkv, d = 2, 33, 4, 2, 8
    quad = (2, 5, 1, 8)
    q, k, v = rand(rng, B, L, Hq, d), rand(rng, B, L, Hkv, d), rand(rng, B, L, Hkv, d)
    do = rand(rng, B, L, Hq, d)
    o, lse = oracle_mod.fwd(q, k, v, quad)
    dq, dk, dv = oracle_mod.bwd(q, k, v, do, quad)
    rows = [(0, 0, 0), (1, 3, 32), (0, 2, 17), (1, 1, 5)]
    o_r, lse_r = oracle_mod.fwd_rows(q, k, v, quad, rows)
    dq_r = oracle_mod.bwd_dq_rows(q, k, v, do, quad, rows)
    for n, (b, hq, i) in enumerate(rows):
        np.testing.assert_allclose(o_r[n], o[b, i, hq], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse_r[n], lse[b, hq, i], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(dq_r[n], dq[b, i, hq], rtol=1e-12, atol=1e-12)
    cols = [(0, 0, 0), (1, 1, 32), (0, 1, 20), (1, 0, 1)]
    dk_c, dv_c = oracle_mod.bwd_dkv_cols(q, k, v, do, quad, cols)
    for n, (b, h, j) in enumerate(cols):
        np.testing.assert_allclose(dk_c[n], dk[b, j, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dv_c[n], dv[b, j, h], rtol=1e-12, atol=1e-12)


def test_bf16_inputs_are_widened_exactly(oracle_mod):
    rng = np.random.default_rng(13)
    q, k, v = rand(rng, 1, 20, 2, 8), rand(rng, 1, 20, 1, 8), rand(rng, 1, 20, 1, 8)
    qb, kb, vb = (oracle_mod.bf16_bits(x) for x in (q, k, v))
    o_b, lse_b = oracle_mod.fwd(qb, kb, vb, (1, 3, 0, 6))
    o_f, lse_f = oracle_mod.fwd(*(oracle_mod.bits_to_f64(x) for x in (qb, kb, vb)), (1, 3, 0, 6))
    np.testing.assert_array_equal(o_b, o_f)
    np.testing.assert_array_equal(lse_b, lse_f)
    # rounding is to nearest: error at most half a bf16 ulp (<= 2^-8 relative)
    back = oracle_mod.bits_to_f64(qb)
    assert (np.abs(back - q) <= np.abs(q) * 2.0 ** -8 + 1e-38).all()
    assert np.abs(back - q).max() > 0


def test_dkv_cols_fast_equals_per_column_loops(oracle_mod):
    """The chunked (matrix-product) dK/dV column routine that the full-size
    GPU tests use for the heavy columns reproduces the per-column C loops
    (themselves pinned above) on ragged shapes, offsets, gaps and chunk
    boundaries."""
    rng = np.random.default_rng(1)

    def bf(shape):
        x = rng.standard_normal(shape, dtype=np.float32)
        return (x.view(np.uint32) >> 16).astype(np.uint16)

    for B, Lq, Lk, Hq, Hkv, d, quad, off in [(2, 300, 300, 4, 2, 16, (5, 30, 0, 70), 0),
                                             (1, 200, 260, 6, 3, 8, (0, 17, 4, 50), 2),
                                             (1, 180, 150, 2, 1, 8, (3, 20, 0, 90), 0)]:
        q, k, v, do = bf((B, Lq, Hq, d)), bf((B, Lk, Hkv, d)), bf((B, Lk, Hkv, d)), bf((B, Lq, Hq, d))
        cols = [(b, h, j) for b in range(B) for h in range(Hkv) for j in (0, 1, 3, Lk // 2, Lk - 1, Lk - 40)]
        rk, rv = oracle_mod.bwd_dkv_cols(q, k, v, do, quad, cols, kv_head_offset=off)
        fk, fv = oracle_mod.bwd_dkv_cols_fast(q, k, v, do, quad, cols, kv_head_offset=off, chunk=37)
        assert np.abs(rk - fk).max() <= 1e-12 * max(1.0, np.abs(rk).max())
        assert np.abs(rv - fv).max() <= 1e-12 * max(1.0, np.abs(rv).max())
