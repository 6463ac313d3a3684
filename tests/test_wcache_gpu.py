"""Windowed decode cache: for a horizon of decode steps from an origin
position, each KV head's cache holds only the keys those steps can see
(Digest, execution notes: decoding reads only the windows, which is where
the decode memory saving comes from).

* build: the stored rows of every (sequence, KV head), in order, are the
  full cache's rows of the oracle's brute-force key set (bit-exact);
* append: a new token's K/V lands where the next steps read it;
* decode over the windowed cache equals decode over the full cache (the
  oracle's), at every step of the horizon, including ragged origins;
* a query outside [origin, origin + horizon) is refused on the device."""
import numpy as np
import pytest
import torch

from helpers import LSE_ABS, assert_o, to64

pytestmark = pytest.mark.gpu


def _full_and_windowed(cowa, B, Lcap, Hq, Hkv, d, quad, origins, horizon, seed):
    from structured_sparse_attention_block_b200.inputs import decode_inputs
    q, kc, vc, _ = decode_inputs(B, Lcap, Hq, Hkv, d, seed=seed)
    org = torch.tensor(origins, dtype=torch.int32, device="cuda")
    kw, vw = cowa.cowa_wcache_build(kc, vc, org, quad, horizon)
    return q, kc, vc, org, kw, vw


@pytest.mark.parametrize("B,Lcap,Hq,Hkv,d,quad,origins,horizon", [
    (2, 1200, 4, 2, 64, (16, 64, 0, 300), [1000, 733], 5),
    (3, 700, 8, 4, 128, (8, 40, 4, 90), [699 - 9, 300, 45], 9),
    (1, 600, 2, 2, 64, (0, 32, 0, 0), [500], 3),
])
def test_build_stores_the_oracle_key_set(oracle_mod, B, Lcap, Hq, Hkv, d, quad, origins, horizon):
    import structured_sparse_attention_block_b200 as cowa
    q, kc, vc, org, kw, vw = _full_and_windowed(cowa, B, Lcap, Hq, Hkv, d, quad, origins, horizon, seed=5)
    assert kw.shape[1] == cowa.cowa_wcache_rows(quad, horizon)
    kc_h, vc_h, kw_h, vw_h = (t.cpu() for t in (kc, vc, kw, vw))
    for b in range(B):
        for h in range(Hkv):
            keys = oracle_mod.window_keys(origins[b], horizon, h, quad)
            have = keys[keys <= origins[b]]  # keys already in the full cache
            n = len(have)
            assert torch.equal(kw_h[b, :n, h], kc_h[b, have, h])
            assert torch.equal(vw_h[b, :n, h], vc_h[b, have, h])
            assert len(keys) <= kw.shape[1]


@pytest.mark.parametrize("d", [64, 128])
def test_decode_over_horizon_matches_full_cache(oracle_mod, d):
    import structured_sparse_attention_block_b200 as cowa
    from structured_sparse_attention_block_b200.inputs import bf16_bits, decode_inputs
    B, Lcap, Hq, Hkv, horizon = 3, 900, 8, 4, 6
    quad = (16, 48, 0, 160)
    origins = [880, 511, 200]
    q, kc, vc, org, kw, vw = _full_and_windowed(cowa, B, Lcap, Hq, Hkv, d, quad, origins, horizon, seed=11)
    for step in range(horizon):
        pos = torch.tensor([o + step for o in origins], dtype=torch.int32, device="cuda")
        if step > 0:
            # the new tokens' K/V: written to the full cache and appended to the windowed one
            _, kn, vn, _ = decode_inputs(B, 1, Hq, Hkv, d, seed=100 + step)
            for b in range(B):
                kc[b, origins[b] + step] = kn[b, 0]
                vc[b, origins[b] + step] = vn[b, 0]
            cowa.cowa_wcache_append(kw, vw, kn[:, 0], vn[:, 0], pos, org, quad, horizon)
        qs = decode_inputs(B, 1, Hq, Hkv, d, seed=200 + step)[0]
        seq = pos + 1
        o_w, lse_w = cowa.cowa_decode_windowed(qs, kw, vw, seq, org, quad, horizon)
        torch.cuda.synchronize()
        cowa.cowa_get_device_error()
        o_ref, lse_ref = oracle_mod.decode(bf16_bits(qs[:, 0]), bf16_bits(kc), bf16_bits(vc), seq.cpu().numpy(),
                                           quad)
        assert_o(o_w[:, 0], o_ref, what="windowed decode O, step %d" % step)
        assert np.abs(lse_w.cpu().numpy() - lse_ref).max() <= LSE_ABS


def test_query_outside_the_horizon_is_flagged():
    import structured_sparse_attention_block_b200 as cowa
    B, Lcap, Hq, Hkv, d, horizon = 2, 400, 4, 2, 64, 6
    quad = (8, 32, 0, 100)
    origins = [300, 100]
    q, kc, vc, org, kw, vw = _full_and_windowed(cowa, B, Lcap, Hq, Hkv, d, quad, origins, horizon, seed=3)
    seq = torch.tensor([300 + horizon + 1, 101], dtype=torch.int32, device="cuda")  # batch 0 past the horizon
    cowa.cowa_decode_windowed(q, kw, vw, seq, org, quad, horizon)
    with pytest.raises(cowa.CowaError, match="COWA_ERR_DEVICE"):
        cowa.cowa_get_device_error()
