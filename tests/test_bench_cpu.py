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
        # the slowest rank sets the step time
        t = bench.max_over_ranks([1.0 + rank, 5.0 - rank], world, "cpu")
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
