"""Host side of corpus sharding, without a GPU: shard bounds, mask slices,
and the exchange step over a gloo process group of two ranks. Each rank
scores its shard with the fp64 oracle (standing in for the GPU scorer),
the lists are all-gathered with the package's own helper, and a plain
merge written here must reproduce the oracle's top-k of the whole corpus."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

shard = pytest.importorskip("exact_inner_product_b200.shard")


def test_shard_bounds_cover_and_align():
    for n in (0, 1, 31, 32, 33, 400, 1000, 10 ** 6 + 7):
        for world in (1, 2, 3, 4, 7, 8):
            b = shard.shard_bounds(n, world)
            assert len(b) == world
            pos = 0
            for start, count in b:
                assert start == pos or count == 0
                assert start % 32 == 0 or start == n
                assert count >= 0
                pos = max(pos, start + count)
            assert pos == n
            assert sum(c for _, c in b) == n
            counts = [c for _, c in b if c]
            if len(counts) > 1 and n >= 32 * world:
                assert max(counts) - min(counts) <= 32
    with pytest.raises(ValueError):
        shard.shard_bounds(10, 0)


def test_exclude_slice_words():
    words = torch.arange(10, dtype=torch.int32)
    assert shard.exclude_slice(words, 64, 100).tolist() == [2, 3, 4, 5]
    assert shard.exclude_slice(words, 0, 32).tolist() == [0]
    assert shard.exclude_slice(None, 0, 5) is None
    with pytest.raises(ValueError):
        shard.exclude_slice(words, 16, 10)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _keys_sorted(ids, scores):
    """(score desc, id asc) order of valid entries."""
    pairs = [(-s, i) for i, s in zip(ids, scores) if i >= 0]
    pairs.sort()
    return [(i, -s) for s, i in pairs]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    import workloads as W
    from exact_inner_product_b200 import shard as sh
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.workload("tiny_f32", n=1000, b=8, k=25, mask_rate=0.1)
        raw_c = W.to_numpy_rows(W.corpus(w))
        raw_q = W.queries(w).numpy()
        excl = W.exclusion_bits(w)
        corpus = oracle.normalize(raw_c, "f32")
        queries = oracle.normalize(raw_q, "f32")
        bounds = sh.shard_bounds(w.n, world)
        start, count = bounds[rank]
        ex = sh.exclude_slice(excl, start, count)
        ex_np = None if ex is None else ex.numpy().view(np.uint32)
        ids, scores = oracle.topk(queries, corpus[start:start + count], w.k, tau=w.tau, exclude=ex_np)
        all_ids, all_scores = sh.gather_lists(torch.from_numpy(ids.astype(np.int32)),
                                              torch.from_numpy(scores.astype(np.float64)))
        merged = []
        for q in range(w.b):
            cand_i, cand_s = [], []
            for p, (s0, _) in enumerate(bounds):
                for i, s in zip(all_ids[p, q].tolist(), all_scores[p, q].tolist()):
                    if i >= 0:
                        cand_i.append(i + s0)
                        cand_s.append(s)
            merged.append(_keys_sorted(cand_i, cand_s)[:w.k])
        ex_full = None if excl is None else excl.numpy().view(np.uint32)
        full_ids, full_scores = oracle.topk(queries, corpus, w.k, tau=w.tau, exclude=ex_full)
        ok = all([i for i, _ in merged[q]] == [i for i in full_ids[q].tolist() if i >= 0]
                 for q in range(w.b))
        out[rank] = bool(ok)
    finally:
        dist.destroy_process_group()


def test_exchange_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert out[0] and out[1]
