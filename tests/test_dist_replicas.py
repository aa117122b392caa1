"""Replica data parallelism on the host: sequences are independent, so a batch
sharded over ranks must give exactly the single-process results, and the
reported time is the max over ranks.  Runs as two gloo ranks on the CPU."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_gqa_indexer_b200 import synth as S


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global():
    return S.Workload(ctx=[4500, 300, 9000, 77, 6000], nq=[1, 2, 1, 3, 1], seed=21)


def _results(w):
    from tests.harness import oracle_selection, oracle_sparse
    rows = list(range(w.total_q))
    sel = oracle_selection(w, rows)
    out, lse = oracle_sparse(w, rows, sel)
    return sel, out, lse


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        shard = S.shard(_global(), rank, world)
        sel, out, lse = _results(shard)
        gathered = [None] * world
        dist.all_gather_object(gathered, (sel, out, lse))
        t = bench.max_over_ranks(1.0 + rank, dist, torch.device("cpu"))
        if rank == 0:
            q.put((gathered, t))
    finally:
        dist.destroy_process_group()


def test_sharded_batch_matches_single_process():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    gathered, tmax = q.get(timeout=300)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert tmax == 2.0
    sel, out, lse = _results(_global())
    assert np.array_equal(np.concatenate([g[0] for g in gathered]), sel)
    assert np.array_equal(np.concatenate([g[1] for g in gathered]), out)
    assert np.array_equal(np.concatenate([g[2] for g in gathered]), lse)


def test_shards_partition_the_batch():
    w = S.config_workloads(3)[0]
    parts = [S.shard(w, r, 4) for r in range(4)]
    assert sum(p.batch for p in parts) == w.batch
    assert [c for p in parts for c in p.ctx] == w.ctx
    # row r of shard k is global row row_base + r
    qx = w.qx_rows(torch.arange(w.total_q))
    got = torch.cat([p.qx_rows(torch.arange(p.total_q)) for p in parts])
    assert torch.equal(got, qx)
    k_full = w.k_tokens(5, torch.arange(10))
    p1 = parts[0] if 5 < parts[0].batch else parts[1]
    s_local = 5 - (p1.seq_base - w.seq_base)
    assert torch.equal(p1.k_tokens(s_local, torch.arange(10)), k_full)
