"""Host-side logic of bench.py, on the CPU: visible-pair counting, the
reference (oracle) arm, and the multi-rank reduction and KV-head sharding
under a world_size-2 gloo group."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("Lq,Lk,quad", [(50, 50, (3, 7, 0, 11)), (20, 61, (5, 4, 2, 9)),
                                        (61, 20, (0, 5, 0, 6)), (40, 40, (0, 0, 0, 0)),
                                        (33, 33, (40, 0, 0, 3)), (64, 64, (0, 64, 0, 0))])
def test_row_visible_counts_match_oracle_mask(oracle_mod, Lq, Lk, quad):
    for h in range(4):
        got = bench.row_visible_counts(Lq, Lk, quad, h)
        exp = oracle_mod.mask(Lq, Lk, h, quad).sum(axis=1)
        np.testing.assert_array_equal(got, exp)


def test_workload_pair_counts(oracle_mod):
    """Visible pairs of the recall workload, against brute-force tile counts."""
    from structured_sparse_attention_block_b200.inputs import WORKLOADS
    wl = WORKLOADS["recall8k"]
    exp = sum(int(oracle_mod.tile_counts(wl.Lq, wl.Lk, h, wl.quad, 128, 64).sum())
              for h in range(wl.Hkv)) * (wl.Hq // wl.Hkv) * wl.B
    assert bench.visible_pairs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.quad) == exp


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3", "--ref-rows", "16"],
                         capture_output=True, text=True, env=env, timeout=600)
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["value"] > 0
    assert res["cpu_baseline"]["kind"] == "oracle" and res["e2e"]["h2d_bytes_per_step"] == 0


def _worker(rank, world, port, q, k, v, quad, result):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import oracle
        # the slowest rank sets the step time; whole-job work adds up
        t = bench.max_over_ranks([1.0 + rank, 5.0 - rank], world, "cpu")
        tot = bench.sum_over_ranks([1.0 + rank, 10.0 * rank], world, "cpu")
        assert tot == [3.0, 10.0]
        # KV-head sharding: rank r owns KV heads [r*H/R, (r+1)*H/R) and their
        # query heads, and passes its first global head as kv_head_offset
        Hkv = k.shape[2]
        g = q.shape[2] // Hkv
        per = Hkv // world
        hs = slice(rank * per, (rank + 1) * per)
        qs = slice(rank * per * g, (rank + 1) * per * g)
        o, _ = oracle.fwd(q[:, :, qs], k[:, :, hs], v[:, :, hs], quad, kv_head_offset=rank * per)
        parts = [torch.zeros_like(torch.from_numpy(o)) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(o))
        if rank == 0:
            result.put((t, torch.cat(parts, dim=2).numpy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_head_sharding(oracle_mod):
    import multiprocessing as mp
    import socket
    rng = np.random.default_rng(0)
    B, L, Hq, Hkv, d = 1, 40, 4, 2, 8
    q, k, v = rng.standard_normal((B, L, Hq, d)), rng.standard_normal((B, L, Hkv, d)), rng.standard_normal((B, L, Hkv, d))
    quad = (2, 5, 0, 18)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, k, v, quad, result)) for r in range(2)]
    for p in procs:
        p.start()
    t, o_sharded = result.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert t == [2.0, 5.0]
    o_full, _ = oracle_mod.fwd(q, k, v, quad)
    np.testing.assert_allclose(o_sharded, o_full, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("name", ["recall8k", "llm14b_32k", "op128k", "decode128k"])
def test_head_shard_covers_every_head_once(name):
    """KV-head sharding: the ranks' head ranges tile [0, Hkv), query heads
    follow their KV heads, and the ranks' visible work adds up to the whole
    workload's (the windows are those of the global heads)."""
    from structured_sparse_attention_block_b200.inputs import WORKLOADS
    wl = WORKLOADS[name]
    for world in (1, 2, 4, 8):
        if wl.Hkv % world:
            with pytest.raises(SystemExit):
                bench.head_shard(wl, 0, world, "heads")
            continue
        seen, pairs = [], 0
        for r in range(world):
            w, h0 = bench.head_shard(wl, r, world, "heads")
            assert w.Hq * world == wl.Hq and w.Hkv * world == wl.Hkv
            assert (w.B, w.Lq, w.Lk, w.d, w.quad) == (wl.B, wl.Lq, wl.Lk, wl.d, wl.quad)
            seen += list(range(h0, h0 + w.Hkv))
            if wl.kind == "train" and wl.Lq <= 8192:
                pairs += bench.visible_pairs(w.B, w.Lq, w.Lk, w.Hq, w.Hkv, w.quad, kv_head_offset=h0)
            else:
                pairs += bench.decode_visible_keys([w.Lk] * w.B, w.Hkv, w.quad, kv_head_offset=h0)
        assert seen == list(range(wl.Hkv))
        if wl.kind == "train" and wl.Lq <= 8192:
            assert pairs == bench.visible_pairs(wl.B, wl.Lq, wl.Lk, wl.Hq, wl.Hkv, wl.quad)
        else:
            assert pairs == bench.decode_visible_keys([wl.Lk] * wl.B, wl.Hkv, wl.quad)
        # replicas keep the whole workload on every rank
        assert bench.head_shard(wl, world - 1, world, "dp") == (wl, 0)


def test_source_hash_ignores_comments_only():
    """The staleness check of the committed DRAM counters: comments and blank
    lines do not count as a kernel change, code (string literals included)
    does."""
    code = 'int f() { return 1; }  // one\n/* block\n comment */\nconst char *s = "// kept /* */";\n'
    assert bench.strip_comments(code) == 'int f() { return 1; }\nconst char *s = "// kept /* */";\n'
    assert bench.strip_comments(code) == bench.strip_comments(code.replace("// one", "// other\n\n"))
    assert bench.strip_comments(code) != bench.strip_comments(code.replace("return 1", "return 2"))
    assert bench.strip_comments(code) != bench.strip_comments(code.replace("// kept", "// kept!"))
    assert bench.strip_comments("char c = '\\'';  // q\n") == "char c = '\\'';\n"


def test_mala_pair_counts_match_brute_force():
    """The MALA leg's causal and kept pair counts from a block decision array
    equal a loop over every (row, key) pair."""
    from bench import mala_pair_counts
    rng = np.random.default_rng(0)
    for Lq, Lk in [(300, 400), (257, 257), (130, 64), (64, 300)]:
        nqt, nkt = -(-Lq // 128), -(-Lk // 64)
        keep = (rng.random((2, 3, nqt, nkt)) < 0.5).astype(np.uint8)
        causal, kept = mala_pair_counts(keep, Lq, Lk)
        cb = kb = 0
        for i in range(Lq):
            for j in range(Lk):
                if j <= i + Lk - Lq:
                    cb += 6
                    kb += int(keep[:, :, i // 128, j // 64].sum())
        assert (causal, kept) == (cb, kb)
