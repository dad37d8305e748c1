"""GPU: merge of per-shard top-k lists (tq_topk_merge) and the sharded search
path on one device.  A database split into shards and searched shard by
shard must give the single search's answer (rows whose fp32 scores tie may
swap places; the merge orders them by id)."""

import numpy as np
import pytest
import torch

from compressed_kv_cache_tq_b200 import sharded
from compressed_kv_cache_tq_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_topk_merge_follows_score_then_id(lib):
    rng = np.random.default_rng(3)
    parts, nq, k = 3, 5, 6
    # few distinct scores, so that ties across and within shards are common
    sc = rng.integers(0, 4, size=(parts, nq, k)).astype(np.float32) * 0.5
    ids = np.stack([np.stack([rng.permutation(50)[:k] for _ in range(nq)]) for _ in range(parts)]).astype(np.int64)
    first = [0, 100, 1000]
    gi, gs = lib.tq_topk_merge(torch.from_numpy(sc).to(DEV), torch.from_numpy(ids).to(DEV), first, k)
    torch.cuda.synchronize()
    for q in range(nq):
        cand = sorted(((float(sc[p, q, j]), int(ids[p, q, j]) + first[p]) for p in range(parts) for j in range(k)),
                      key=lambda c: (-c[0], c[1]))[:k]
        assert gi[q].cpu().tolist() == [c[1] for c in cand]
        assert gs[q].cpu().tolist() == [c[0] for c in cand]


@pytest.mark.parametrize("bits,k", [(3, 10), (4, 1), (2, 32)])
def test_shards_merged_equal_one_search(lib, bits, k):
    n, d, nq = 5000, 128, 20
    ctx = lib.tq_init(d, bits, 17)
    db = torch.from_numpy(W.search_vectors(n, d, seed=40 + bits, which=0)).to(DEV)
    qs = torch.from_numpy(W.search_vectors(nq, d, seed=40 + bits, which=1)).to(DEV)
    payload, norms = lib.tq_quantize(ctx, db)
    ids1, sc1 = lib.tq_topk(ctx, qs, payload, norms, k)
    bounds = [0, 1700, 3300, n]
    parts = [lib.tq_topk(ctx, qs, payload[a:b], norms[a:b], k) for a, b in zip(bounds[:-1], bounds[1:])]
    gi, gs = lib.tq_topk_merge(torch.stack([p[1] for p in parts]), torch.stack([p[0] for p in parts]), bounds[:-1], k)
    torch.cuda.synchronize()
    assert torch.equal(gs, sc1)                     # the same exact scores, rounded once
    same = (gi == ids1).all(1)
    for q in torch.nonzero(~same).flatten().tolist():
        # the scores agree position by position (checked above), so ids can
        # only differ among rows whose fp32 scores tie
        diff = (gi[q] != ids1[q]).nonzero().flatten().tolist()
        for j in diff:
            assert (sc1[q] == sc1[q, j]).sum() > 1


def test_sharded_topk_on_one_rank_is_the_search(lib):
    n, d, nq, k = 3000, 128, 8, 10
    ctx = lib.tq_init(d, 3, 21)
    db = torch.from_numpy(W.search_vectors(n, d, seed=7, which=0)).to(DEV)
    qs = torch.from_numpy(W.search_vectors(nq, d, seed=7, which=1)).to(DEV)
    payload, norms = lib.tq_quantize(ctx, db)
    ids1, sc1 = lib.tq_topk(ctx, qs, payload, norms, k)
    gi, gs = sharded.sharded_topk(ctx, qs, payload, norms, [0], k)
    torch.cuda.synchronize()
    assert torch.equal(gi, ids1) and torch.equal(gs, sc1)


def test_topk_merge_argument_errors(lib):
    sc = torch.zeros((2, 3, 4), device=DEV)
    ids = torch.zeros((2, 3, 4), dtype=torch.int64, device=DEV)
    with pytest.raises(ValueError):
        lib.tq_topk_merge(sc, ids, [0], 4)               # one offset per part
    with pytest.raises(lib.TQError):
        lib.tq_topk_merge(sc, ids, [0, -5], 4)           # negative first row
    big = torch.zeros((65, 1, 1), device=DEV)
    with pytest.raises(lib.TQError):
        lib.tq_topk_merge(big, torch.zeros((65, 1, 1), dtype=torch.int64, device=DEV), list(range(65)), 1)
