"""KV-head sharding on one GPU: the calls a tensor-parallel rank makes (its
contiguous block of KV heads and their query heads, as strided views of the
full tensors, with kv_head_offset = its first global head) reproduce the
unsharded call.  Forward and backward are bit-identical: every CTA works on
one KV head (or a pair of its query heads) with that head's global windows,
and neither its work nor its summation order depends on how many heads the
call holds.  The decode chooses its split count from the total work, so the
shards' outputs agree to the rounding of the split merge."""
import pytest
import torch

import structured_sparse_attention_block_b200 as cowa
from structured_sparse_attention_block_b200.inputs import training_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("B,L,Hq,Hkv,d,quad", [(2, 700, 8, 4, 64, (16, 100, 0, 150)),
                                              (1, 900, 12, 4, 128, (8, 128, 3, 200))])
def test_kv_head_shards_equal_the_full_run(world, B, L, Hq, Hkv, d, quad):
    q, k, v, do = training_inputs(B, L, L, Hq, Hkv, d, device="cuda", seed=31 + d)
    o, lse = cowa.cowa_fwd(q, k, v, quad)
    dq, dk, dv = cowa.cowa_bwd(q, k, v, o, lse, do, quad)
    qd = q[:, -1:].contiguous()
    seqlens = torch.tensor([L - 3 * b for b in range(B)], dtype=torch.int32, device="cuda")
    od, lsed = cowa.cowa_decode(qd, k, v, seqlens, quad)
    g, per = Hq // Hkv, Hkv // world
    for r in range(world):
        hs, qs = slice(r * per, (r + 1) * per), slice(r * per * g, (r + 1) * per * g)
        h0 = r * per
        o_r, lse_r = cowa.cowa_fwd(q[:, :, qs], k[:, :, hs], v[:, :, hs], quad, kv_head_offset=h0)
        assert torch.equal(o_r, o[:, :, qs]) and torch.equal(lse_r, lse[:, qs]), ("forward", r)
        g_r = cowa.cowa_bwd(q[:, :, qs], k[:, :, hs], v[:, :, hs], o[:, :, qs], lse[:, qs].contiguous(),
                            do[:, :, qs], quad, kv_head_offset=h0)
        full = (dq[:, :, qs], dk[:, :, hs], dv[:, :, hs])
        for name, got, ref in zip(("dq", "dk", "dv"), g_r, full):
            assert torch.equal(got, ref), (name, r)
        od_r, lsed_r = cowa.cowa_decode(qd[:, :, qs], k[:, :, hs], v[:, :, hs], seqlens, quad, kv_head_offset=h0)
        torch.testing.assert_close(od_r.float(), od[:, :, qs].float(), atol=4e-3, rtol=1e-2)
        torch.testing.assert_close(lsed_r, lsed[:, qs], atol=1e-5, rtol=1e-5)
    cowa.cowa_get_device_error()
