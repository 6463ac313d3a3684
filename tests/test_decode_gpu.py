"""Decode parity: cowa_decode against the oracle's decode on the same bf16
cache (O within max-abs 1e-2 / mean-abs 1e-3, LSE within 2e-3), and
consistency with the training forward's last row."""
import numpy as np
import pytest
import torch

from helpers import assert_lse, assert_o, to64

pytestmark = pytest.mark.gpu

CASES = [  # B, Lcap, Hq, Hkv, d, quad, seqlens
    (3, 700, 4, 2, 64, (16, 64, 0, 224), [700, 1, 333]),
    (2, 1000, 8, 4, 128, (5, 37, 3, 50), [0, 999]),
    (4, 4096, 16, 2, 128, (64, 512, 0, 1792), [4096, 4000, 129, 64]),
    (1, 300, 4, 4, 64, (0, 300, 0, 0), [300]),
    (2, 513, 32, 2, 64, (0, 0, 0, 0), [513, 100]),
    (5, 2000, 12, 4, 128, (1, 1, 0, 400), [2000, 1999, 1601, 7, 2]),
]


def run(q, kc, vc, sl, quad, **kw):
    import structured_sparse_attention_block_b200 as cowa
    o, lse = cowa.cowa_decode(q, kc, vc, sl, quad, **kw)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("B,Lcap,Hq,Hkv,d,quad,seqlens", CASES)
def test_decode_matches_oracle(oracle_mod, B, Lcap, Hq, Hkv, d, quad, seqlens):
    from structured_sparse_attention_block_b200.inputs import bf16_bits, decode_inputs
    q, kc, vc, sl = decode_inputs(B, Lcap, Hq, Hkv, d, seed=Lcap, seqlens=seqlens)
    o, lse = run(q, kc, vc, sl, quad)
    o_ref, lse_ref = oracle_mod.decode(bf16_bits(q[:, 0]), bf16_bits(kc), bf16_bits(vc),
                                       np.array(seqlens), quad)
    assert_o(o[:, 0], o_ref)
    assert_lse(lse, lse_ref)


def test_decode_equals_forward_last_row():
    """Same pattern in training and decoding: the decode of the last token
    equals the forward's last row on the same data."""
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import training_inputs
    B, L, Hq, Hkv, d = 2, 1500, 8, 2, 128
    quad = (32, 200, 0, 650)
    q, k, v, _ = training_inputs(B, L, L, Hq, Hkv, d, seed=4, with_dout=False)
    o, lse = cowa.cowa_fwd(q, k, v, quad)
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    od, lsed = run(q[:, -1:].contiguous(), k, v, sl, quad)
    assert (od[:, 0].float() - o[:, -1].float()).abs().max().item() <= 1e-2
    assert (lsed - lse[:, :, -1]).abs().max().item() <= 2e-3


def test_decode_workload(oracle_mod):
    """The 128K decode workload in full: 16 sequences x 32 query heads."""
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, bf16_bits, workload_inputs
    wl = WORKLOADS["decode128k"]
    q, kc, vc, sl = workload_inputs(wl, seed=0)
    o, lse = run(q, kc, vc, sl, wl.quad)
    o_ref, lse_ref = oracle_mod.decode(bf16_bits(q[:, 0]), bf16_bits(kc), bf16_bits(vc),
                                       sl.cpu().numpy(), wl.quad)
    assert_o(o[:, 0], o_ref)
    assert_lse(lse, lse_ref)


def test_bad_seqlens_are_reported_not_read():
    """seqlens past the cache capacity: the kernel reads nothing out of range
    and records a device error that cowa_get_device_error raises."""
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import decode_inputs
    q, kc, vc, _ = decode_inputs(2, 256, 4, 2, 64, seed=1)
    sl = torch.tensor([256, 10_000], dtype=torch.int32, device="cuda")
    o, lse = run(q, kc, vc, sl, (4, 16, 0, 120))
    with pytest.raises(cowa.CowaError) as e:
        cowa.cowa_get_device_error()
    assert e.value.status == 7
    cowa.cowa_get_device_error()  # cleared
    assert torch.isneginf(lse[1]).all() and (o[1] == 0).all()
