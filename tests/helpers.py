"""Shared test helpers: tolerances, comparisons against the oracle, sampling.

Tolerances are the ones fixed for this operator: O within max-abs 1e-2 and
mean-abs 1e-3 of the fp64 oracle; dQ, dK, dV within max-abs 2e-2 * max|ref|.
LSE has no stated bound; fp32 scores of bf16 inputs give it an absolute error
far below 2e-3, which is the bound used here.

O is returned in bf16, rounded to nearest (ties to even) from the kernel's
fp32 result, so the max-abs bound is applied to that fp32 value: the bf16
output must be the rounding of some value within 1e-2 of the oracle's O,
i.e. lie in [rne(ref - 1e-2), rne(ref + 1e-2)] (rounding is monotone).  No
slack is added: an output outside that interval came from an fp32 value more
than 1e-2 away.  The mean-abs bound compares with rne(ref), the exact value
of a bf16 output.
"""
import numpy as np
import torch

O_MAX, O_MEAN, GRAD_REL, LSE_ABS = 1e-2, 1e-3, 2e-2, 2e-3


def to64(t):
    return t.detach().float().cpu().double().numpy()


def bf16_rne(x):
    """fp64 values rounded to bf16 (8 significant bits), nearest with ties
    to even, in one step (no intermediate fp32 rounding); returned as fp64."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    fin = np.isfinite(x) & (ax > 0)
    e = np.floor(np.log2(np.where(fin, ax, 1.0)))
    ulp = 2.0 ** (e - 7)
    return np.where(fin, np.round(x / ulp) * ulp, x)  # np.round: half to even


def assert_o(o_gpu, o_ref, what="O"):
    got = to64(o_gpu) if isinstance(o_gpu, torch.Tensor) else o_gpu
    assert np.isfinite(got).all(), "%s has non-finite values" % what
    lo, hi = bf16_rne(o_ref - O_MAX), bf16_rne(o_ref + O_MAX)
    out = np.maximum(lo - got, got - hi)  # > 0: no value within O_MAX rounds to got
    assert out.max() <= 0, "%s: bf16 output not the rounding of a value within %g of the oracle " \
        "(max-abs %.3g, %d elements)" % (what, O_MAX, np.abs(got - o_ref).max(), int((out > 0).sum()))
    diff = np.abs(got - bf16_rne(o_ref))
    assert diff.mean() <= O_MEAN, "%s mean-abs %.3g > %g" % (what, diff.mean(), O_MEAN)


def assert_lse(lse_gpu, lse_ref, what="LSE"):
    got = to64(lse_gpu) if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    ref_inf = np.isneginf(lse_ref)
    assert (np.isneginf(got) == ref_inf).all(), "%s: empty-row pattern differs" % what
    fin = ~ref_inf
    if fin.any():
        err = np.abs(got[fin] - lse_ref[fin]).max()
        assert err <= LSE_ABS, "%s max-abs %.3g > %g" % (what, err, LSE_ABS)


def assert_grad(g_gpu, g_ref, what):
    got = to64(g_gpu) if isinstance(g_gpu, torch.Tensor) else g_gpu
    assert np.isfinite(got).all(), "%s has non-finite values" % what
    scale = np.abs(g_ref).max()
    err = np.abs(got - g_ref).max()
    assert err <= GRAD_REL * max(scale, 1e-30), "%s max-abs %.3g > %g * %.3g" % (what, err, GRAD_REL, scale)


def sample_rows(B, Lq, Lk, Hq, quad, per_head, seed=0):
    """(b, hq, i) triples: per query head the first and last rows, rows at the
    window edges (distances S, N, N+G+h*W seen from the end) and random rows."""
    rng = np.random.default_rng(seed)
    S, N, G, W = quad
    rows = []
    for hq in range(Hq):
        cand = {0, Lq - 1, min(Lq - 1, max(0, S)), min(Lq - 1, max(0, N)),
                min(Lq - 1, max(0, N + G + W)), max(0, Lq - 1 - N)}
        cand |= set(int(x) for x in rng.integers(0, Lq, size=max(0, per_head - len(cand))))
        for i in sorted(cand)[:per_head]:
            rows.append((int(rng.integers(0, B)), hq, int(i)))
    return rows
