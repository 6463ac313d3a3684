"""fp64 CPU oracle of MassAlloc Attention (MALA), the companion method the
CoWA pages name ("Two new attention models slash redundancy...", first
section; "CoWindow Attention: Full Causal Coverage Is a Collective Property",
abstract).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``.  The library has no
kernel for this operator; this module defines what one must compute.

The pages state what MALA keeps and what it uses, not its rule.  It keeps the
full causal QK scoring and lets attention's own softmax statistics decide
where the remaining work of a tile is worth doing, dropping low-contribution
regions.  This module fixes the plainest reading of that, in the pages'
order:

1. Scores on every causal pair: s_ij = scale * <q_i, k_j> for j <= p_i,
   p_i = i + Lk - Lq (bottom-right alignment, as for CoWA); query head hq
   uses KV head hq // (Hq / Hkv).
2. The softmax statistics of each row over all of its causal keys:
   LSE_i = log sum_j exp(s_ij), P_ij = exp(s_ij - LSE_i).
3. Per (query tile of BM rows, key tile of BN keys) of one head, the mass
   each row gives the tile, M_it = sum_{j in t} P_ij.  The tile is
   low-contribution when every row of the query tile gives it less than tau:
   max_i M_it < tau.  Its remaining work (P V forward; dP and dV backward)
   is skipped.
4. O_i = sum over kept tiles of sum_j P_ij v_j.  The dropped mass is not
   redistributed: LSE stays the full-scoring statistic, so
   |O_i - O_i(dense)| <= (mass row i dropped) * max |v|.

The gradient is that of the output in step 4 with the tile selection held
fixed (selection is a threshold, not differentiable): with
delta_i = <dO_i, O_i>,
    dV_j  = sum over kept (i, j) of P_ij dO_i
    dS_ij = P_ij * (<dO_i, v_j> [j kept for i] - delta_i)   (every causal pair)
    dQ_i  = scale * sum_j dS_ij k_j,   dK_j = scale * sum_i dS_ij q_i.
Skipped pairs still carry -P_ij * delta_i through LSE, which depends on
every score: the full scoring the pages say MALA keeps.
"""
import math

import numpy as np


def _f64(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:  # bf16 bit patterns, widened exactly
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def _scores(q, k, scale):
    """Per (b, hq): the causal score matrix (-inf off the causal pairs)."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    p = np.arange(Lq)[:, None] + (Lk - Lq)
    causal = np.arange(Lk)[None, :] <= p
    s = np.full((B, Hq, Lq, Lk), -np.inf)
    for b in range(B):
        for hq in range(Hq):
            raw = scale * (q[b, :, hq] @ k[b, :, hq // g].T)
            s[b, hq] = np.where(causal, raw, -np.inf)
    return s, causal


def _stats(s):
    """LSE per row (-inf for a row without keys) and P = exp(s - LSE)."""
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    l = np.exp(s - m).sum(axis=-1, keepdims=True)
    lse = np.where(l > 0, m + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    P = np.where(np.isfinite(s), np.exp(s - np.where(np.isfinite(lse), lse, 0.0)), 0.0)
    return lse[..., 0], P


def keep_tiles(P, BM, BN, tau):
    """Step 3: bool [B, Hq, nqt, nkt], True where some row of the query tile
    gives the key tile a mass of at least tau."""
    B, Hq, Lq, Lk = P.shape
    nqt, nkt = -(-Lq // BM), -(-Lk // BN)
    keep = np.zeros((B, Hq, nqt, nkt), bool)
    for a in range(nqt):
        rows = P[:, :, a * BM:(a + 1) * BM]
        for t in range(nkt):
            mass = rows[..., t * BN:(t + 1) * BN].sum(axis=-1)  # [B, Hq, rows]
            keep[:, :, a, t] = mass.max(axis=-1) >= tau
    return keep


def _pair_keep(keep, Lq, Lk, BM, BN):
    """The tile decision spread over (row, key) pairs."""
    rows = np.arange(Lq) // BM
    cols = np.arange(Lk) // BN
    return keep[:, :, rows][:, :, :, cols]


def fwd(q, k, v, tau, BM, BN, scale=None):
    """(O [B, Lq, Hq, d], LSE [B, Hq, Lq], keep [B, Hq, nqt, nkt], dropped
    mass per row [B, Hq, Lq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    s, _ = _scores(q, k, scale)
    lse, P = _stats(s)
    keep = keep_tiles(P, BM, BN, tau)
    Pk = np.where(_pair_keep(keep, Lq, Lk, BM, BN), P, 0.0)
    o = np.zeros_like(q)
    for b in range(B):
        for hq in range(Hq):
            o[b, :, hq] = Pk[b, hq] @ v[b, :, hq // g]
    return o, lse, keep, (P - Pk).sum(axis=-1)


def bwd(q, k, v, dout, tau, BM, BN, scale=None):
    """(dQ, dK, dV) of fwd's O, the tile selection held fixed; dK and dV are
    summed over the query heads of each KV head."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    s, _ = _scores(q, k, scale)
    _, P = _stats(s)
    kp = _pair_keep(keep_tiles(P, BM, BN, tau), Lq, Lk, BM, BN)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for hq in range(Hq):
            h = hq // g
            Pk = np.where(kp[b, hq], P[b, hq], 0.0)
            o = Pk @ v[b, :, h]
            delta = (dout[b, :, hq] * o).sum(axis=-1, keepdims=True)
            dP = np.where(kp[b, hq], dout[b, :, hq] @ v[b, :, h].T, 0.0)
            dS = P[b, hq] * (dP - delta)
            dv[b, :, h] += Pk.T @ dout[b, :, hq]
            dq[b, :, hq] = scale * (dS @ k[b, :, h])
            dk[b, :, h] += scale * (dS.T @ q[b, :, hq])
    return dq, dk, dv
