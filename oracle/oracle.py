"""numpy front end of the fp64 CPU oracle (``cowa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's
CPU-baseline leg are its only users.  Arrays are numpy; an input given as
``np.uint16`` is read as bf16 bit patterns and widened exactly, anything else
is converted to fp64.  Layouts: Q/O [B, Lq, Hq, d], K/V [B, Lk, Hkv, d],
LSE [B, Hq, Lq], KV cache [B, Lcap, Hkv, d].

Every function follows the definitions written out at the top of
``cowa_oracle.c`` (mask rule of "CoWindow Attention: Full Causal Coverage Is
a Collective Property", method key points; softmax attention and its analytic
gradients).
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        sig = [_i64] * 11 + [_ptr, ctypes.c_double, ctypes.c_int]
        _lib.cowa_ref_fwd.argtypes = sig + [_ptr] * 5
        _lib.cowa_ref_fwd_rows.argtypes = sig + [_ptr] * 3 + [_i64] + [_ptr] * 3
        _lib.cowa_ref_bwd.argtypes = sig + [_ptr] * 7
        _lib.cowa_ref_bwd_dq_rows.argtypes = sig + [_ptr] * 4 + [_i64] + [_ptr] * 2
        _lib.cowa_ref_bwd_dkv_cols.argtypes = sig + [_ptr] * 4 + [_i64] + [_ptr] * 3
        _lib.cowa_ref_decode.argtypes = [_i64] * 10 + [_ptr, ctypes.c_double,
                                                       ctypes.c_int] + [_ptr] * 6
        _lib.cowa_ref_mask.argtypes = [_i64] * 7 + [_ptr]
        _lib.cowa_ref_visible.argtypes = [_i64] * 7
        _lib.cowa_ref_visible.restype = ctypes.c_int
        _lib.cowa_ref_threads.restype = ctypes.c_int
        _lib.cowa_ref_tile_counts.argtypes = [_i64] * 9 + [_ptr]
    return _lib


def threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().cowa_ref_threads())


def default_quad(Lk, Hkv, S, N):
    """Default quadruple: G = 0 and W = ceil((Lk - N) / Hkv), never negative."""
    return (int(S), int(N), 0, max(0, -(-(int(Lk) - int(N)) // int(Hkv))))


def _prep(x):
    """Contiguous array plus its bf16 flag."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 1
    return np.ascontiguousarray(x, dtype=np.float64), 0


def _inputs(*arrays):
    out, flags = [], set()
    for a in arrays:
        arr, f = _prep(a)
        out.append(arr)
        flags.add(f)
    if len(flags) != 1:
        raise TypeError("oracle inputs must be all bf16 bits or all floating")
    return out, flags.pop()


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _widx(widx):
    if widx is None:
        return None
    return np.ascontiguousarray(widx, dtype=np.int64)


def _head(q, k, quad, kv_head_offset, widx, scale):
    B, Lq, Hq, D = q.shape
    Bk, Lk, Hkv, Dk = k.shape
    if B != Bk or D != Dk or Hq % Hkv:
        raise ValueError("shape mismatch")
    S, N, G, W = (int(x) for x in quad)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return [B, Lq, Lk, Hq, Hkv, D, S, N, G, W, int(kv_head_offset)], scale


def visible(p, j, w, quad) -> bool:
    S, N, G, W = quad
    return bool(_load().cowa_ref_visible(p, j, w, S, N, G, W))


def mask(Lq, Lk, w, quad) -> np.ndarray:
    """Boolean [Lq, Lk] visibility of window index ``w``."""
    S, N, G, W = quad
    out = np.empty((Lq, Lk), dtype=np.uint8)
    _load().cowa_ref_mask(Lq, Lk, w, S, N, G, W, _p(out))
    return out.astype(bool)


def tile_counts(Lq, Lk, w, quad, BM, BN) -> np.ndarray:
    """int64 [ceil(Lq/BM), ceil(Lk/BN)]: visible pairs in each tile (brute force)."""
    S, N, G, W = quad
    out = np.zeros((-(-Lq // BM), -(-Lk // BN)), dtype=np.int64)
    _load().cowa_ref_tile_counts(Lq, Lk, w, S, N, G, W, BM, BN, _p(out))
    return out


def fwd(q, k, v, quad, scale=None, kv_head_offset=0, widx=None):
    """Forward: returns (O [B,Lq,Hq,d] fp64, LSE [B,Hq,Lq] fp64)."""
    (q, k, v), bf = _inputs(q, k, v)
    dims, scale = _head(q, k, quad, kv_head_offset, widx, scale)
    B, Lq, Lk, Hq = dims[:4]
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, Hq, Lq), dtype=np.float64)
    w = _widx(widx)
    _load().cowa_ref_fwd(*dims, _p(w), scale, bf, _p(q), _p(k), _p(v), _p(o), _p(lse))
    return o, lse


def fwd_rows(q, k, v, quad, rows, scale=None, kv_head_offset=0, widx=None):
    """Forward of selected rows ``rows`` [(b, hq, i), ...]: (O [n,d], LSE [n])."""
    (q, k, v), bf = _inputs(q, k, v)
    dims, scale = _head(q, k, quad, kv_head_offset, widx, scale)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.zeros((n, q.shape[3]), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    w = _widx(widx)
    _load().cowa_ref_fwd_rows(*dims, _p(w), scale, bf, _p(q), _p(k), _p(v),
                              n, _p(rows), _p(o), _p(lse))
    return o, lse


def bwd(q, k, v, dout, quad, scale=None, kv_head_offset=0, widx=None):
    """Backward: returns (dQ, dK, dV) in fp64, shapes of q, k, v."""
    (q, k, v, dout), bf = _inputs(q, k, v, dout)
    dims, scale = _head(q, k, quad, kv_head_offset, widx, scale)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    w = _widx(widx)
    _load().cowa_ref_bwd(*dims, _p(w), scale, bf, _p(q), _p(k), _p(v), _p(dout),
                         _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def bwd_dq_rows(q, k, v, dout, quad, rows, scale=None, kv_head_offset=0, widx=None):
    """dQ of selected rows [(b, hq, i), ...] -> [n, d]."""
    (q, k, v, dout), bf = _inputs(q, k, v, dout)
    dims, scale = _head(q, k, quad, kv_head_offset, widx, scale)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    dq = np.zeros((n, q.shape[3]), dtype=np.float64)
    w = _widx(widx)
    _load().cowa_ref_bwd_dq_rows(*dims, _p(w), scale, bf, _p(q), _p(k), _p(v),
                                 _p(dout), n, _p(rows), _p(dq))
    return dq


def bwd_dkv_cols(q, k, v, dout, quad, cols, scale=None, kv_head_offset=0, widx=None):
    """dK, dV of selected key columns [(b, hkv, j), ...] -> ([n, d], [n, d])."""
    (q, k, v, dout), bf = _inputs(q, k, v, dout)
    dims, scale = _head(q, k, quad, kv_head_offset, widx, scale)
    cols = np.ascontiguousarray(np.asarray(cols, dtype=np.int64).reshape(-1, 3))
    n = cols.shape[0]
    dk = np.zeros((n, q.shape[3]), dtype=np.float64)
    dv = np.zeros((n, q.shape[3]), dtype=np.float64)
    w = _widx(widx)
    _load().cowa_ref_bwd_dkv_cols(*dims, _p(w), scale, bf, _p(q), _p(k), _p(v),
                                  _p(dout), n, _p(cols), _p(dk), _p(dv))
    return dk, dv


def _visible_np(p, j, w, quad):
    """The mask rule of ``cowa_ref_visible`` on numpy arrays (broadcasting):
    key j visible from aligned position p under window index w iff
    d = p - j >= 0 and (j < S or d < N or N+G+w*W <= d < N+G+(w+1)*W)."""
    S, N, G, W = (int(x) for x in quad)
    d = p - j
    c = N + G + w * W
    return (d >= 0) & (j >= 0) & ((j < S) | (d < N) | ((d >= c) & (d < c + W)))


def bwd_dkv_cols_fast(q, k, v, dout, quad, cols, scale=None, kv_head_offset=0, chunk=256):
    """dK, dV of selected key columns [(b, hkv, j), ...] -> ([n, d], [n, d]),
    the same definitions as ``bwd_dkv_cols`` with numpy matrix products for
    the scores and the PV sums of whole chunks of rows (every row's softmax is
    still taken over exactly its visible keys, in fp64).  For the full-size
    workloads, where a sink column is seen by every query row: each of those
    rows needs its own LSE and O, which the per-row C loops cannot afford.

    Per KV head h of a column, over the rows i (of the g query heads of the
    group) that see column j: s_il = scale <q_i, k_l> on the row's visible
    keys l, LSE_i = log sum_l exp(s_il), P_il = exp(s_il - LSE_i),
    O_i = sum_l P_il v_l, delta_i = <dO_i, O_i>, dP_ij = <dO_i, v_j>,
    dS_ij = P_ij (dP_ij - delta_i); dK_j = scale sum_i dS_ij q_i,
    dV_j = sum_i P_ij dO_i."""
    def widen(x):  # slices are widened when taken: a full-size fp64 copy would not fit
        x = np.asarray(x)
        return (lambda *i: bits_to_f64(x[i])) if x.dtype == np.uint16 else (lambda *i: np.asarray(x[i], np.float64))

    qf, kf, vf, df = (widen(x) for x in (q, k, v, dout))
    B, Lq, Hq, D = np.shape(q)
    Lk, Hkv = np.shape(k)[1], np.shape(k)[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    S, N, G, W = (int(x) for x in quad)
    cols = [tuple(int(a) for a in c) for c in cols]
    dk = np.zeros((len(cols), D))
    dv = np.zeros((len(cols), D))
    by_head = {}
    for n, (b, h, j) in enumerate(cols):
        by_head.setdefault((b, h), []).append((n, j))
    shift = Lk - Lq
    for (b, h), members in by_head.items():
        w = h + int(kv_head_offset)
        p_all = np.arange(Lq, dtype=np.int64) + shift
        js = np.array([j for _, j in members], dtype=np.int64)
        sees = _visible_np(p_all[:, None], js[None, :], w, quad)  # [Lq, ncols]
        rows = np.nonzero(sees.any(axis=1))[0]
        for r0 in range(0, len(rows), chunk):
            ri = rows[r0:r0 + chunk]
            pr = ri + shift
            # candidate keys: the union over the chunk's rows of the sink
            # [0, S), near [p-N+1, p] and long [p-e+1, p-c] ranges (c =
            # N+G+w*W, e = c+W), a superset of every row's visible keys; each
            # row's own mask is then the rule itself
            lo, hi = int(pr.min()), int(pr.max())
            c = N + G + w * W
            parts = [np.arange(0, min(S, hi + 1, Lk)),
                     np.arange(max(0, lo - N + 1), min(hi + 1, Lk)),
                     np.arange(max(0, lo - (c + W) + 1), min(hi - c + 1, Lk))]
            kidx = np.unique(np.concatenate([x for x in parts if x.size] or [np.zeros(0, np.int64)]))
            m = _visible_np(pr[:, None], kidx[None, :], w, quad)
            kk, vv = kf(b, kidx, h), vf(b, kidx, h)
            kcol = {j: (kf(b, j, h), vf(b, j, h)) for _, j in members}
            for hq in range(h * g, (h + 1) * g):
                qi, di = qf(b, ri, hq), df(b, ri, hq)
                s = scale * (qi @ kk.T)
                s[~m] = -np.inf
                mx = s.max(axis=1, keepdims=True)
                np.subtract(s, mx, out=s)
                np.exp(s, out=s)  # exp(s - max): 0 off the mask
                tot = s.sum(axis=1)
                lse = mx[:, 0] + np.log(tot)
                o = (s @ vv) / tot[:, None]  # sum_l P_il v_l with P = exp(s - LSE)
                delta = (di * o).sum(axis=1)
                for n, j in members:
                    sel = _visible_np(pr, j, w, quad)
                    if not sel.any():
                        continue
                    kj, vj = kcol[j]
                    pij = np.exp(scale * (qi[sel] @ kj) - lse[sel])
                    dpij = di[sel] @ vj
                    dsij = pij * (dpij - delta[sel])
                    dk[n] += scale * (dsij @ qi[sel])
                    dv[n] += pij @ di[sel]
    return dk, dv


def decode(q, k_cache, v_cache, seqlens, quad, scale=None, kv_head_offset=0,
           widx=None):
    """Single-token decode: q [B,Hq,d], caches [B,Lcap,Hkv,d], seqlens [B].

    Returns (O [B,Hq,d], LSE [B,Hq]) in fp64.
    """
    (q, kc, vc), bf = _inputs(q, k_cache, v_cache)
    B, Hq, D = q.shape
    Bc, Lcap, Hkv, Dc = kc.shape
    if B != Bc or D != Dc or Hq % Hkv or vc.shape != kc.shape:
        raise ValueError("shape mismatch")
    seq = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    if seq.shape != (B,) or (seq < 0).any() or (seq > Lcap).any():
        raise ValueError("seqlens must be [B] within [0, Lcap]")
    S, N, G, W = (int(x) for x in quad)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    w = _widx(widx)
    _load().cowa_ref_decode(B, Lcap, Hq, Hkv, D, S, N, G, W, int(kv_head_offset),
                            _p(w), scale, bf, _p(q), _p(kc), _p(vc), _p(seq),
                            _p(o), _p(lse))
    return o, lse


def window_keys(p_lo, horizon, w, quad) -> np.ndarray:
    """Sorted keys that some query position in [p_lo, p_lo + horizon) sees
    through window index w: the key set a decode cache for those positions
    must hold for that KV head (Digest, execution notes: decoding reads only
    the windows, which is where its KV-cache saving comes from).  Brute force
    over the dense mask, so it restates no interval arithmetic."""
    if horizon <= 0:
        return np.zeros(0, dtype=np.int64)
    Lk = int(p_lo) + int(horizon)
    m = mask(int(horizon), Lk, int(w), quad)  # row i is position p_lo + i
    return np.nonzero(m.any(axis=0))[0].astype(np.int64)


def bf16_bits(x) -> np.ndarray:
    """Round fp32/fp64 values to bf16 (round to nearest even); return bit patterns.

    Used to give the oracle the same bf16-rounded values as the GPU when a
    workload is drawn in fp32.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bits_to_f64(bits) -> np.ndarray:
    """Widen bf16 bit patterns to fp64 exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


__all__ = ["threads", "default_quad", "visible", "mask", "tile_counts", "fwd", "fwd_rows", "bwd",
           "bwd_dq_rows", "bwd_dkv_cols", "bwd_dkv_cols_fast", "decode", "window_keys", "bf16_bits", "bits_to_f64"]
