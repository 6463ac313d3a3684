"""Forward parity: the library's cowa_fwd against the fp64 oracle on the
same bf16 inputs (O within max-abs 1e-2 / mean-abs 1e-3; LSE within 2e-3)."""
import numpy as np
import pytest
import torch

from helpers import assert_lse, assert_o, sample_rows, to64

pytestmark = pytest.mark.gpu

CASES = [  # B, Lq, Lk, Hq, Hkv, d, quad
    (1, 512, 512, 4, 2, 64, (16, 64, 0, 224)),       # the tiny workload
    (2, 200, 200, 6, 3, 64, (5, 37, 0, 50)),         # ragged tiles, odd sink
    (1, 77, 300, 4, 4, 128, (16, 40, 3, 60)),        # chunked prefill Lq < Lk, gap
    (1, 300, 130, 2, 1, 64, (3, 20, 0, 110)),         # Lq > Lk: empty rows
    (1, 256, 256, 8, 4, 128, (0, 17, 5, 9)),          # W < tile, G > 0
    (1, 384, 384, 2, 2, 128, (0, 384, 0, 0)),         # full causal control quad
    (1, 130, 130, 2, 2, 64, (0, 0, 0, 0)),           # nothing visible
    (1, 1, 700, 4, 2, 128, (32, 100, 0, 300)),       # a single query row
    (3, 1000, 1000, 16, 8, 64, (1, 1, 0, 125)),       # many heads, 1-wide windows
    (2, 700, 700, 6, 2, 128, (8, 150, 0, 330)),      # g = 3: head pairs and a lone head in one launch
    (1, 1500, 1500, 4, 1, 128, (64, 256, 3, 512)),   # many 128-key tiles per query tile: the K/V rings wrap
]


def run(q, k, v, quad, **kw):
    import structured_sparse_attention_block_b200 as cowa
    o, lse = cowa.cowa_fwd(q, k, v, quad, **kw)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,quad", CASES)
def test_fwd_matches_oracle(oracle_mod, B, Lq, Lk, Hq, Hkv, d, quad):
    from structured_sparse_attention_block_b200.inputs import bf16_bits, training_inputs
    q, k, v, _ = training_inputs(B, Lq, Lk, Hq, Hkv, d, seed=B * 7 + Lq)
    o, lse = run(q, k, v, quad)
    o_ref, lse_ref = oracle_mod.fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), quad)
    assert_o(o, o_ref)
    assert_lse(lse, lse_ref)


def test_fwd_tiny_inputs_scaled_reading(oracle_mod):
    """The tiny workload's other reading: inputs multiplied by 1/sqrt(d)."""
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, bf16_bits, training_inputs
    wl = WORKLOADS["tiny"]
    q, k, v, _ = training_inputs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.d, seed=0)
    q, k, v = (x * wl.scale for x in (q, k, v))
    o, lse = run(q, k, v, wl.quad)
    o_ref, lse_ref = oracle_mod.fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), wl.quad)
    assert_o(o, o_ref)
    assert_lse(lse, lse_ref)


def test_fwd_large_logits(oracle_mod):
    """Logits x8 so the running max moves often (rescaling path)."""
    from structured_sparse_attention_block_b200.inputs import bf16_bits, training_inputs
    q, k, v, _ = training_inputs(1, 600, 600, 4, 2, 128, seed=3)
    q = q * 8
    quad = (20, 90, 0, 260)
    o, lse = run(q, k, v, quad)
    o_ref, lse_ref = oracle_mod.fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), quad)
    assert_o(o, o_ref)
    assert_lse(lse, lse_ref)


def test_fwd_strided_and_offset_heads(oracle_mod):
    """Q/K/V as views of one packed [B, L, Hq+2Hkv, d] tensor, O strided too,
    and a KV-head offset (a tensor-parallel rank holding global heads 3, 4)."""
    from structured_sparse_attention_block_b200.inputs import bf16_bits
    B, L, Hq, Hkv, d = 2, 333, 4, 2, 64
    g = torch.Generator().manual_seed(5)
    packed = torch.randn(B, L, Hq + 2 * Hkv, d, generator=g).to(torch.bfloat16).cuda()
    q, k, v = packed[:, :, :Hq], packed[:, :, Hq:Hq + Hkv], packed[:, :, Hq + Hkv:]
    out = torch.zeros(B, L, Hq + 8, d, dtype=torch.bfloat16, device="cuda")[:, :, 8:]
    quad = (7, 30, 0, 40)
    o, lse = run(q, k, v, quad, kv_head_offset=3, out=out)
    o_ref, lse_ref = oracle_mod.fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), quad, kv_head_offset=3)
    assert_o(o, o_ref)
    assert_lse(lse, lse_ref)
    assert (out.data_ptr() == o.data_ptr())


@pytest.mark.parametrize("name,per_head", [("recall8k", 96), ("llm14b_32k", 24), ("op128k", 12)])
def test_fwd_workloads_sampled_rows(oracle_mod, name, per_head):
    """Full-size workloads in the bench's launch configuration; the oracle
    computes sampled rows one by one."""
    from structured_sparse_attention_block_b200.inputs import WORKLOADS, bf16_bits, workload_inputs
    wl = WORKLOADS[name]
    q, k, v, _ = workload_inputs(wl, seed=0)
    o, lse = run(q, k, v, wl.quad)
    rows = sample_rows(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.quad, per_head, seed=1)
    o_ref, lse_ref = oracle_mod.fwd_rows(bf16_bits(q), bf16_bits(k), bf16_bits(v), wl.quad, rows)
    b, hq, i = (torch.tensor([r[a] for r in rows], device=o.device) for a in range(3))
    o_got = o[b, i, hq]
    lse_got = lse[b, hq, i]
    assert_o(o_got, o_ref)
    assert_lse(lse_got, lse_ref)


def test_no_keys_gives_empty_rows():
    # a sequence with no keys at all: every row sees nothing (O = 0, LSE = -inf)
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import training_inputs
    q, _, _, _ = training_inputs(2, 130, 1, 4, 2, 64, seed=2)
    k = torch.empty((2, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    o, lse = cowa.cowa_fwd(q, k, k, (4, 16, 0, 8), out=torch.full_like(q, 7.0))
    torch.cuda.synchronize()
    assert torch.all(o == 0)
    assert torch.all(torch.isneginf(lse))
