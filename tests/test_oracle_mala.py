"""Pins of the MALA oracle (oracle/mala.py) against what its reading fixes:
tau = 0 keeps every tile and is dense causal attention (compared with a
separately written per-row softmax here); tau above 1 keeps none; the error
against dense attention is bounded by each row's dropped mass; the dropped
mass of a row is below tau per skipped tile; raising tau only removes tiles;
and the gradients equal central finite differences with the selection held
fixed."""
import math

import numpy as np
import pytest

from oracle import mala


def _inputs(B, Lq, Lk, Hq, Hkv, d, seed, spread=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Lq, Hq, d)) * spread
    k = rng.standard_normal((B, Lk, Hkv, d)) * spread
    v = rng.standard_normal((B, Lk, Hkv, d))
    return q, k, v


def _dense_causal(q, k, v):
    """Row by row: softmax over keys j <= i + Lk - Lq, max subtracted first."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    o = np.zeros_like(q)
    lse = np.full((B, Hq, Lq), -np.inf)
    for b in range(B):
        for hq in range(Hq):
            h = hq * Hkv // Hq
            for i in range(Lq):
                n = i + Lk - Lq + 1
                if n <= 0:
                    continue
                z = np.array([q[b, i, hq] @ k[b, j, h] for j in range(n)]) / math.sqrt(d)
                zm = z.max()
                w = np.exp(z - zm)
                o[b, i, hq] = (w[:, None] * v[b, :n, h]).sum(axis=0) / w.sum()
                lse[b, hq, i] = zm + math.log(w.sum())
    return o, lse


SHAPES = [(1, 40, 40, 4, 2, 8), (2, 23, 37, 2, 2, 8), (1, 30, 19, 3, 1, 4)]


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d", SHAPES)
def test_tau_zero_is_dense_causal_attention(B, Lq, Lk, Hq, Hkv, d):
    q, k, v = _inputs(B, Lq, Lk, Hq, Hkv, d, seed=Lq)
    o, lse, keep, dropped = mala.fwd(q, k, v, 0.0, 8, 8)
    o_ref, lse_ref = _dense_causal(q, k, v)
    assert keep.all() and np.abs(dropped).max() < 1e-15
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(lse), np.isinf(lse_ref))
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], atol=1e-12)


def test_tau_above_one_keeps_nothing():
    q, k, v = _inputs(1, 24, 24, 2, 1, 8, seed=1)
    o, lse, keep, dropped = mala.fwd(q, k, v, 1.5, 8, 8)
    assert not keep.any()
    assert np.abs(o).max() == 0.0
    np.testing.assert_allclose(dropped, 1.0, atol=1e-12)  # every row has keys
    _, lse_ref = _dense_causal(q, k, v)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)  # the statistics stay the full ones


@pytest.mark.parametrize("tau", [0.01, 0.05, 0.2])
@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d", SHAPES)
def test_error_bounded_by_dropped_mass(B, Lq, Lk, Hq, Hkv, d, tau):
    q, k, v = _inputs(B, Lq, Lk, Hq, Hkv, d, seed=7 + Lk, spread=1.5)
    BM, BN = 8, 4
    o, _, keep, dropped = mala.fwd(q, k, v, tau, BM, BN)
    o_ref, _ = _dense_causal(q, k, v)
    vmax = np.abs(v).max()
    err = np.abs(o - o_ref).max(axis=-1)  # [B, Lq, Hq]
    assert (err <= dropped.transpose(0, 2, 1) * vmax + 1e-12).all()
    # a row drops less than tau per skipped key tile of its query tile
    skipped = (~keep).sum(axis=-1)  # [B, Hq, nqt]
    per_row = np.repeat(skipped, BM, axis=-1)[..., :Lq]
    assert (dropped <= per_row * tau + 1e-12).all()


def test_tile_decision_by_brute_force_and_monotone():
    q, k, v = _inputs(1, 33, 33, 2, 1, 8, seed=3, spread=2.0)
    BM, BN = 8, 8
    scale = 1 / math.sqrt(8)
    prev = None
    for tau in (0.0, 0.02, 0.1, 0.3, 0.9):
        _, _, keep, _ = mala.fwd(q, k, v, tau, BM, BN)
        for hq in range(2):
            for a in range(keep.shape[2]):
                for t in range(keep.shape[3]):
                    best = 0.0
                    for i in range(a * BM, min(33, (a + 1) * BM)):
                        z = np.array([q[0, i, hq] @ k[0, j, 0] * scale for j in range(i + 1)])
                        p = np.exp(z - z.max())
                        p /= p.sum()
                        best = max(best, p[t * BN:(t + 1) * BN].sum())
                    assert keep[0, hq, a, t] == (best >= tau)
        if prev is not None:
            assert not (keep & ~prev).any()  # a higher tau keeps a subset
        prev = keep


@pytest.mark.parametrize("tau", [0.0, 0.15])
def test_gradients_match_finite_differences(tau):
    B, Lq, Lk, Hq, Hkv, d, BM, BN = 1, 20, 20, 2, 1, 4, 4, 4
    q, k, v = _inputs(B, Lq, Lk, Hq, Hkv, d, seed=16, spread=1.3)
    dout = np.random.default_rng(12).standard_normal((B, Lq, Hq, d))
    # keep the threshold away from every tile's mass, so the perturbations
    # below cannot flip a decision
    s, _ = mala._scores(q, k, 1 / math.sqrt(d))
    _, P = mala._stats(s)
    masses = np.array([[P[0, hq, a * BM:(a + 1) * BM, t * BN:(t + 1) * BN].sum(axis=-1).max()
                        for a in range(Lq // BM) for t in range(Lk // BN)] for hq in range(Hq)])
    assert tau == 0.0 or np.abs(masses - tau).min() > 1e-3
    _, _, keep, dropped = mala.fwd(q, k, v, tau, BM, BN)
    # at tau > 0 visible tiles holding real mass are skipped (not only the
    # empty tiles above the diagonal)
    assert tau == 0.0 or dropped.max() > 0.05
    dq, dk, dv = mala.bwd(q, k, v, dout, tau, BM, BN)

    def loss(q_, k_, v_):
        return (mala.fwd(q_, k_, v_, tau, BM, BN)[0] * dout).sum()

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            ap = [xp if a is x else a for a in (q, k, v)]
            am = [xm if a is x else a for a in (q, k, v)]
            num[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        err = np.abs(num - g).max() / max(np.abs(g).max(), 1e-12)
        assert err < 1e-6, (name, err)
