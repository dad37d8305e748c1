"""Sharded search, host side, on CPU: two gloo ranks each hold half of a
database; each rank's local top-k comes from the oracle (test
infrastructure), gather_topk all-gathers the lists, and a merge written here
from the definition (score descending, global id ascending) combines them.
The result must equal the oracle's top-k over the whole database: this checks
the shard offsets, the gather order and the rank bookkeeping of
compressed_kv_cache_tq_b200.sharded (the merge itself is tq_topk_merge,
checked against the same definition on the GPU)."""

from __future__ import annotations

import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _merge_by_definition(scores, ids, first_rows, k):
    import torch

    P, nq, _ = scores.shape
    out_i = torch.empty((nq, k), dtype=torch.int64)
    out_s = torch.empty((nq, k), dtype=torch.float32)
    for i in range(nq):
        cand = [(float(scores[p, i, j]), int(ids[p, i, j]) + int(first_rows[p])) for p in range(P) for j in range(k)]
        cand.sort(key=lambda c: (-c[0], c[1]))
        out_s[i] = torch.tensor([c[0] for c in cand[:k]])
        out_i[i] = torch.tensor([c[1] for c in cand[:k]])
    return out_i, out_s


def _rank_main(rank, world, port, results):
    import datetime

    import torch
    import torch.distributed as dist

    from compressed_kv_cache_tq_b200 import sharded
    from compressed_kv_cache_tq_b200 import workloads as W
    from oracle import tq_oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        n, d, k = 601, 32, 7
        tb = O.make_tables(d, 3, 42)
        db = W.search_vectors(n, d, seed=5, which=0).astype(np.float64)
        qs = W.search_vectors(9, d, seed=5, which=1).astype(np.float64)
        first, count = sharded.shard_rows(n, world, rank)
        firsts = [sharded.shard_rows(n, world, r)[0] for r in range(world)]
        qz = O.quantize(db[first:first + count], tb)
        ids, sc, _, _ = O.topk(qs, qz.codes, qz.bits, qz.n16, qz.rho16, tb, k)
        gi, gs = sharded.gather_topk(torch.from_numpy(ids), torch.from_numpy(sc.astype(np.float32)), firsts, k,
                                     merge=_merge_by_definition)
        results[rank] = (gi.numpy().tolist(), gs.numpy().tolist())
    finally:
        dist.destroy_process_group()


def test_sharded_topk_two_gloo_ranks_equal_the_whole_database():
    from compressed_kv_cache_tq_b200 import workloads as W
    from oracle import tq_oracle as O

    world = 2
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, start_method="spawn",
                           join=True)
        got = dict(results)
    assert got[0] == got[1]
    n, d, k = 601, 32, 7
    tb = O.make_tables(d, 3, 42)
    db = W.search_vectors(n, d, seed=5, which=0).astype(np.float64)
    qs = W.search_vectors(9, d, seed=5, which=1).astype(np.float64)
    qz = O.quantize(db, tb)
    ids, sc, _, _ = O.topk(qs, qz.codes, qz.bits, qz.n16, qz.rho16, tb, k)
    assert got[0][0] == ids.tolist()
    np.testing.assert_allclose(got[0][1], sc.astype(np.float32), rtol=0, atol=0)


def test_shard_rows_cover_the_database():
    from compressed_kv_cache_tq_b200 import sharded

    for n, world in ((10, 3), (1_000_000, 8), (7, 7)):
        blocks = [sharded.shard_rows(n, world, r) for r in range(world)]
        assert blocks[0][0] == 0 and sum(c for _, c in blocks) == n
        assert all(blocks[r][0] + blocks[r][1] == blocks[r + 1][0] for r in range(world - 1))
