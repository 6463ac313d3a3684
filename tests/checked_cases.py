"""Small ragged parity cases of every kernel, run in a process of their own
(see test_debug_gpu.py): forward, backward, decode, packed batches, the
windowed decode cache and MALA, each against the fp64 oracle, with the
device error word read after every case.  Prints "checked ok <library>" at the end."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import structured_sparse_attention_block_b200 as cowa  # noqa: E402
from helpers import assert_grad, assert_lse, assert_o  # noqa: E402
from oracle import oracle  # noqa: E402
from structured_sparse_attention_block_b200.inputs import bf16_bits, decode_inputs, training_inputs  # noqa: E402


def no_device_error(what):
    st = cowa.lib().cowa_get_device_error(None)
    assert st == 0, "%s: device error word %d" % (what, st)


def main():
    torch.cuda.set_device(0)
    for B, Lq, Lk, Hq, Hkv, d, quad in [(2, 200, 200, 6, 3, 64, (5, 37, 0, 50)),
                                        (1, 77, 300, 4, 4, 128, (16, 40, 3, 60)),
                                        (1, 300, 130, 2, 1, 64, (3, 20, 0, 110)),
                                        (1, 256, 256, 8, 4, 128, (0, 17, 5, 9)),
                                        (2, 700, 700, 8, 2, 128, (32, 100, 0, 300))]:
        q, k, v, do = training_inputs(B, Lq, Lk, Hq, Hkv, d, seed=Lq + Lk)
        o, lse = cowa.cowa_fwd(q, k, v, quad)
        dq, dk, dv = cowa.cowa_bwd(q, k, v, o, lse, do, quad)
        torch.cuda.synchronize()
        no_device_error("training %s" % ((B, Lq, Lk, Hq, Hkv, d, quad),))
        qb, kb, vb, db = (bf16_bits(x) for x in (q, k, v, do))
        o_ref, lse_ref = oracle.fwd(qb, kb, vb, quad)
        assert_o(o, o_ref)
        assert_lse(lse, lse_ref)
        rq, rk, rv = oracle.bwd(qb, kb, vb, db, quad)
        assert_grad(dq, rq, "dQ")
        assert_grad(dk, rk, "dK")
        assert_grad(dv, rv, "dV")
    # decode over a cache with ragged lengths, d = 64 and 128
    for d in (64, 128):
        quad = (16, 128, 0, 300)
        qd, kc, vc, sl = decode_inputs(3, 1000, 8, 2, d, seed=d, seqlens=[1000, 513, 2])
        od, lsed = cowa.cowa_decode(qd, kc, vc, sl, quad)
        torch.cuda.synchronize()
        no_device_error("decode d=%d" % d)
        o_ref, lse_ref = oracle.decode(bf16_bits(qd[:, 0]), bf16_bits(kc), bf16_bits(vc), [1000, 513, 2], quad)
        assert_o(od[:, 0], o_ref)
        assert_lse(lsed, lse_ref)
    # a packed batch of ragged sequences
    lens = [300, 77, 512, 1]
    T = sum(lens)
    q, k, v, do = (t[0] for t in training_inputs(1, T, T, 4, 2, 128, seed=11))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device="cuda")
    quad = (8, 64, 0, 100)
    o, lse = cowa.cowa_fwd_varlen(q, k, v, cu, cu, max(lens), max(lens), quad)
    dq, dk, dv = cowa.cowa_bwd_varlen(q, k, v, o, lse, do, cu, cu, max(lens), max(lens), quad)
    torch.cuda.synchronize()
    no_device_error("packed batch")
    # each sequence alone through the oracle; gradients compared over the
    # whole packed tensor (a one-token sequence has exactly zero dQ)
    refs = {"O": [], "dQ": [], "dK": [], "dV": []}
    for b, n in enumerate(lens):
        a = int(cu[b])
        sl = slice(a, a + n)
        qb, kb, vb, db = (bf16_bits(x[sl][None]) for x in (q, k, v, do))
        refs["O"].append(oracle.fwd(qb, kb, vb, quad)[0][0])
        rq, rk, rv = oracle.bwd(qb, kb, vb, db, quad)
        refs["dQ"].append(rq[0])
        refs["dK"].append(rk[0])
        refs["dV"].append(rv[0])
    assert_o(o, np.concatenate(refs["O"]), what="packed O")
    for name, got in (("dQ", dq), ("dK", dk), ("dV", dv)):
        assert_grad(got, np.concatenate(refs[name]), "packed " + name)
    # decode over a windowed cache built for the next 8 positions
    quad = (16, 128, 0, 300)
    qd, kc, vc, sl = decode_inputs(2, 900, 8, 2, 128, seed=3, seqlens=[700, 400])
    origin = sl - 1
    kw, vw = cowa.cowa_wcache_build(kc, vc, origin, quad, 8)
    od, lsed = cowa.cowa_decode_windowed(qd, kw, vw, sl, origin, quad, 8)
    torch.cuda.synchronize()
    no_device_error("windowed decode")
    o_ref, lse_ref = oracle.decode(bf16_bits(qd[:, 0]), bf16_bits(kc), bf16_bits(vc), [700, 400], quad)
    assert_o(od[:, 0], o_ref)
    # MALA at both ends of tau, where no decision is close to the threshold:
    # tau = 0 keeps every causal block (dense causal attention), tau > 1
    # keeps none (O = 0, zero gradients)
    from oracle import mala
    for d in (64, 128):
        q, k, v, do = training_inputs(1, 300, 300, 4, 2, d, seed=d + 5)
        qb, kb, vb, db = (bf16_bits(x) for x in (q, k, v, do))
        for tau in (0.0, 1.5):
            o, lse, keep = cowa.cowa_mala_fwd(q, k, v, tau)
            dq, dk, dv = cowa.cowa_mala_bwd(q, k, v, o, lse, keep, do)
            torch.cuda.synchronize()
            no_device_error("MALA d=%d tau=%g" % (d, tau))
            o_ref, lse_ref, _, _ = mala.fwd(qb, kb, vb, tau, 128, 64)
            assert_o(o, o_ref, what="MALA O")
            assert_lse(lse, lse_ref)
            if tau == 0.0:
                rq, rk, rv = mala.bwd(qb, kb, vb, db, tau, 128, 64)
                assert_grad(dq, rq, "MALA dQ")
                assert_grad(dk, rk, "MALA dK")
                assert_grad(dv, rv, "MALA dV")
            else:
                assert int(keep.sum()) == 0 and bool(torch.all(dq == 0)) and bool(torch.all(dk == 0))
    print("checked ok %s" % cowa.library_path())


if __name__ == "__main__":
    main()
