"""The test helpers' bf16 rounding, checked against torch's conversion."""
import numpy as np
import torch

from helpers import bf16_rne


def test_bf16_rne_matches_torch_on_fp32_values():
    # fp32 inputs: torch rounds fp32 -> bf16 to nearest, ties to even, the
    # same single rounding bf16_rne applies to the (exact) fp64 widening
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    # exact ties: bf16 values plus half their spacing, both parities
    base = torch.randn(2000).to(torch.bfloat16).float().numpy()
    bits = base.view(np.uint32) + np.uint32(0x8000)
    ties = bits.view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1.0, 3.0, 65504.0])])
    want = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = bf16_rne(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_rne_keeps_bf16_values_and_specials():
    v = torch.randn(5000).to(torch.bfloat16).double().numpy()
    assert np.array_equal(bf16_rne(v), v)
    sp = np.array([np.inf, -np.inf, 0.0])
    assert np.array_equal(bf16_rne(sp), sp)
    assert np.isnan(bf16_rne(np.array([np.nan]))).all()


def test_o_bound_is_the_rounding_of_a_value_within_tolerance():
    from helpers import O_MAX, assert_o
    import pytest
    # ref + 0.01 lies past the midpoint above rne(ref) in the [2, 4) binade
    # (spacing 1/64), so the output one spacing up is the rounding of a value
    # within 1e-2 although it lies 0.0128 from ref
    ref = np.concatenate([[2.03405, 0.3, -3.1], np.linspace(-1, 1, 97)])  # 100 values: the mean
    ok = bf16_rne(ref)                                                    # bound sees one outlier
    assert ok[0] == 2.03125
    assert_o(ok, ref)
    assert_o(ok + np.eye(100)[0] / 64, ref)
    # two spacings up: no value within 1e-2 rounds there
    with pytest.raises(AssertionError):
        assert_o(ok + np.eye(100)[0] * 2 / 64, ref)
    # one spacing down: the nearest values within 1e-2 round to rne(ref)
    with pytest.raises(AssertionError):
        assert_o(ok - np.eye(100)[0] / 64, ref)
    with pytest.raises(AssertionError):
        assert_o(bf16_rne(ref + np.eye(100)[1] * 2 * O_MAX), ref)
