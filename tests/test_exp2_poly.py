"""The cubic base-2 exponential of the softmax kernels, checked on the CPU:
the header's coefficients are the ones the committed fit produces, and the
kernel's fp32 steps (clamp, round-to-integer by the 1.5*2^23 shift, cubic in
fused multiply-adds, exponent-field scale) reproduce 2^x within 1e-4
relative on [-126, 16], give exactly 0 for -inf and anything below -127,
and change by no more than the fit's error where the split moves from
f = +0.5 to f = -0.5."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "structured_sparse_attention_block_b200", "csrc", "sm100.cuh")


def header_coeffs():
    text = open(HDR).read()
    vals = dict(re.findall(r"kExp2C(\d)\s*=\s*([-+0-9.eE]+)f", text))
    return [np.float32(float(vals[str(k)])) for k in range(4)]


def emulate(x, c):
    """The kernel's steps in fp32 (fma emulated exactly through fp64)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-127.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    jf = (t - magic).astype(f32)
    f = (x - jf).astype(f32)
    fma = lambda a, b, d: (a.astype(np.float64) * b.astype(np.float64) + np.float64(d)).astype(f32)
    p = fma(np.full_like(f, c[3]), f, c[2])
    p = fma(p, f, c[1])
    p = fma(p, f, c[0])
    scale = ((t.view(np.uint32) << np.uint32(23)) + np.uint32(127 << 23)).view(f32)
    return (p * scale).astype(f32)


def test_header_matches_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "exp2_fit", os.path.join(ROOT, "structured_sparse_attention_block_b200", "exp2_fit.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    c = mod.fit()
    assert mod.max_rel_error(c) < 8e-5
    assert header_coeffs() == [np.float32(v) for v in c]


def test_emulated_kernel_steps():
    c = header_coeffs()
    x = np.concatenate([np.linspace(-126.0, 16.0, 2_000_003), np.arange(-126, 17) - 0.5,
                        np.arange(-126, 17) + 0.5]).astype(np.float32)
    y = emulate(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.abs(y / ref - 1.0).max() < 1e-4
    # masked entries and deep underflow give exact zeros
    z = emulate(np.array([-np.inf, -127.0, -200.0, -1e30], dtype=np.float32), c)
    assert (z == 0).all()
    # where j changes (f jumps from +0.5 to -0.5) the two sides agree to the fit's error
    for k in range(-20, 9):
        lo, hi = emulate(np.array([k + 0.4999, k + 0.5001], dtype=np.float32), c).astype(np.float64)
        assert abs(hi / lo - 2.0 ** 0.0002) < 2e-4
