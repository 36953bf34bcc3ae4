"""The N>1 host path of bench.py on CPU: two gloo ranks.

The sparse-prefill path has no exchange step, so N GPUs either run
independent replicas (weak scaling) or split one workload's tokens (strong
scaling); the only collectives are the barrier and the max-over-ranks
timing reduction.  These tests run those pieces on two gloo ranks.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    from top_sparse_attention_qsa_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        m = bench.max_over_ranks(1.5 * (rank + 1), dist, "cpu")
        w = W.make("tiny")
        part = bench.shard_workload(w, world, rank)
        t0, t1 = bench.shard_range(w.shape["T"], world, rank)
        same = torch.equal(part.q, w.q[t0:t1]) and torch.equal(part.topk_idx, w.topk_idx[t0:t1])
        # KV-head split: each rank's oracle result on its heads is the full
        # result's head slice
        import oracle
        wh = W.generic_case(T=5, S=40, Hq=16, Hkv=2, K=9, seed=7)
        wh.n_valid = torch.tensor([[9, 3], [0, 9], [5, 5], [9, 1], [2, 9]], dtype=torch.int32)
        mine = bench.shard_heads(wh, world, rank)
        full = oracle.sparse_prefill(wh.q, wh.k_cache, wh.v_cache, wh.topk_idx, wh.n_valid, 0.0)
        part_res = oracle.sparse_prefill(mine.q, mine.k_cache, mine.v_cache, mine.topk_idx, mine.n_valid, 0.0)
        h0 = rank * 8
        heads_ok = bool((part_res[0] == full[0][:, h0:h0 + 8]).all() and (part_res[1] == full[1][:, h0:h0 + 8]).all())
        queue.put((rank, m, (t0, t1), part.shape["T"], bool(same and heads_ok)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_shard_range_partitions():
    sys.path.insert(0, ROOT)
    import bench
    for n in (0, 1, 7, 256, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert [r[1] for r in results] == [3.0, 3.0]                  # max over ranks, on every rank
    assert results[0][2] == (0, 128) and results[1][2] == (128, 256)
    assert sum(r[3] for r in results) == 256                       # the shards cover the workload
    assert all(r[4] for r in results)                              # and are views of the same tokens
