"""The multi-GPU path on CPU: two gloo ranks.

* The benchmark's aggregation takes the slowest rank's time and counts all
  ranks' work.
* Head sharding needs no exchange: each rank plans its own heads with the
  oracle, and the gathered plans equal the single-process plan bit for bit
  (the sampling uniforms are counter-based on (b, h, q-block, KV block)).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_12_b200 import inputs, multigpu

W = inputs.TINY


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _aggregate_worker(rank, world, port, out):
    _init(rank, world, port)
    try:
        ms = multigpu.max_over_ranks(10.0 + 5.0 * rank)
        out[rank] = (ms, multigpu.job_throughput(1e12, ms, world))
    finally:
        dist.destroy_process_group()


def _plan_worker(rank, world, port, out):
    import oracle
    _init(rank, world, port)
    try:
        Q, K, _ = inputs.make_qkv(W)
        heads = multigpu.head_shard(W.H, rank, world)
        scale = 1 / math.sqrt(W.d)
        sel = oracle.selector_all(Q[:, heads.start:heads.stop], K[:, heads.start:heads.stop], 128,
                                  W.kv_block, W.n_clusters, W.kmeans_iters, scale)
        # each rank plans its heads; the RNG counter needs the global head index,
        # so plan rows one by one with their true (b, h, qb)
        nkvb = W.N // W.kv_block
        rows = []
        for i, h in enumerate(heads):
            for qb in range(W.N // 128):
                pi, _, _ = oracle.waterfill(sel["S"][0, i, qb], W.budget * nkvb)
                idx, _, _ = oracle.sample(pi.astype(np.float32), W.seed, 0, h, qb)
                rows.append(torch.tensor([h, qb, idx.size] + idx.tolist() + [-1] * (nkvb - idx.size), dtype=torch.int64))
        mine = torch.stack(rows)
        gathered = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)
        if rank == 0:
            out["sharded"] = torch.cat(gathered).numpy()
    finally:
        dist.destroy_process_group()


def _gather_worker(rank, world, port, out):
    _init(rank, world, port)
    try:
        H = 5
        hs = multigpu.head_shard(H, rank, world)
        # each rank's slice holds its global head indices
        O = torch.arange(hs.start, hs.stop, dtype=torch.float32).view(1, -1, 1, 1).expand(1, len(hs), 3, 2).contiguous()
        full = multigpu.gather_heads(O, H, world)
        out[rank] = full.numpy()
    finally:
        dist.destroy_process_group()


def _run(fn, world):
    port = 29500 + (os.getpid() % 1000)
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(fn, args=(world, port, out), nprocs=world, join=True)
        return dict(out)


def test_aggregation_takes_slowest_rank_and_all_work():
    out = _run(_aggregate_worker, 2)
    for r in range(2):
        ms, thr = out[r]
        assert ms == 15.0
        assert thr == pytest.approx(2 * 1e12 / 0.015)


def test_head_shard_covers_all_heads_once():
    for H, world in [(40, 8), (24, 8), (12, 8), (40, 3), (2, 2)]:
        got = [h for r in range(world) for h in multigpu.head_shard(H, r, world)]
        assert got == list(range(H))


def test_sharded_plan_equals_single_process_plan():
    import oracle
    out = _run(_plan_worker, 2)
    sharded = out["sharded"]
    Q, K, _ = inputs.make_qkv(W)
    sel = oracle.selector_all(Q, K, 128, W.kv_block, W.n_clusters, W.kmeans_iters, 1 / math.sqrt(W.d))
    full = oracle.plan_all(sel["S"], W.budget, 0, W.seed, cap=W.N // W.kv_block)
    for row in sharded:
        h, qb, n = int(row[0]), int(row[1]), int(row[2])
        assert full["counts"][0, h, qb] == n
        np.testing.assert_array_equal(row[3:3 + n], full["idx"][0, h, qb, :n])


@pytest.mark.parametrize("world", [2, 3])
def test_gather_heads_assembles_the_layer(world):
    out = _run(_gather_worker, world)
    want = np.arange(5, dtype=np.float32).reshape(1, 5, 1, 1) * np.ones((1, 5, 3, 2), dtype=np.float32)
    for r in range(world):
        np.testing.assert_array_equal(out[r], want)


def test_head_slice_inputs_equal_the_layer():
    Q, K, V = inputs.make_qkv(W)
    Qs, Ks, Vs = inputs.make_qkv_heads(W, range(1, 2))
    assert torch.equal(Qs, Q[:, 1:2]) and torch.equal(Ks, K[:, 1:2]) and torch.equal(Vs, V[:, 1:2])
