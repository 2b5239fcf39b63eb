"""Corpus sharding on one GPU: the corpus is split into row shards, each shard
is scored as its own index, and tt_merge_topk combines the lists. The merged
result is checked against the fp64 oracle's top-k of the whole corpus (the
comparison rule of the parity tests), and must also equal the single-corpus
call bit for bit (ids and scores), on every scorer path, with masks, per-row
norms, k larger than a shard and lists too long for the merge's
shared-memory staging. (GPU)"""
import numpy as np
import pytest
import torch

import parity
import workloads as W

pytestmark = pytest.mark.gpu

tt = pytest.importorskip("exact_inner_product_b200")
from exact_inner_product_b200 import shard  # noqa: E402


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _shard_and_merge(index, qn, k, tau, excl, parts, **options):
    bounds = shard.shard_bounds(index.n, parts)
    lists_i, lists_s = [], []
    for start, count in bounds:
        rows = index.rows[start:start + count]
        inv = None if index.inv_norm is None else index.inv_norm[start:start + count]
        local = tt.tt_index_wrap(rows, inv)
        ids, scores = tt.tt_score_topk(local, qn, k, tau=tau, exclude=shard.exclude_slice(excl, start, count),
                                       **options)
        lists_i.append(ids)
        lists_s.append(scores)
    return tt.tt_merge_topk(torch.stack(lists_i), torch.stack(lists_s), [s for s, _ in bounds], k)


@pytest.mark.parametrize("name,over,parts", [
    ("stream_b1", {"n": 200_037, "b": 3, "k": 100}, 3),
    ("small_batch", {"n": 300_077, "b": 40, "k": 500}, 2),
    ("large_batch", {"n": 400_005, "b": 300, "k": 1000}, 5),
    ("masked_fused", {"n": 200_099, "b": 260, "k": 256}, 4),
    ("tiny_f32", {}, 3),
])
def test_sharded_equals_single(name, over, parts):
    _cuda()
    w = W.workload(name, **over)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    excl = W.exclusion_bits(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    want_ids, want_scores = tt.tt_score_topk(index, qn, w.k, tau=w.tau, exclude=excl)
    path = tt.tt_last_stats(index)["path"]
    got_ids, got_scores = _shard_and_merge(index, qn, w.k, w.tau, excl, parts)
    # the merged lists against the oracle's top-k of the whole corpus
    qids = W.oracle_query_ids(w)
    side = parity.OracleSide(w, W.to_numpy_rows(raw_c), raw_q.cpu().numpy(),
                             None if excl is None else excl.cpu().numpy().view(np.uint32), qids)
    res = parity.compare(got_ids.cpu().numpy()[qids], got_scores.cpu().numpy()[qids], side, w.k, w.tolerance)
    assert res["max_abs_err"] <= w.tolerance and res.get("sure_checked", 0) > 0, res
    assert torch.equal(got_ids, want_ids), name
    assert torch.equal(got_scores, want_scores), name
    if name == "masked_fused":  # the SM-pair kernel too, forced on every shard and on the whole
        want = tt.tt_score_topk(index, qn, w.k, tau=w.tau, exclude=excl, path=3)
        got = _shard_and_merge(index, qn, w.k, w.tau, excl, parts, path=3)
        assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
    assert path in (1, 2, 3)


def test_merge_edge_cases():
    _cuda()
    dev = "cuda"
    # two parts of b=2 queries, k_in=4; padding entries (-1) are ignored
    ids = torch.tensor([[[0, 1, 2, -1], [3, -1, -1, -1]],
                        [[1, 0, -1, -1], [-1, -1, -1, -1]]], dtype=torch.int32, device=dev)
    scores = torch.tensor([[[0.9, 0.5, 0.5, float("-inf")], [0.1, float("-inf"), float("-inf"), float("-inf")]],
                           [[0.7, 0.5, float("-inf"), float("-inf")], [float("-inf")] * 4]], device=dev)
    out_ids, out_scores = tt.tt_merge_topk(ids, scores, [0, 100], 4)
    # query 0: 0.9 (id 0), 0.7 (id 101), then 0.5 ties: ids 1, 2, 100 -> lower ids first
    assert out_ids[0].tolist() == [0, 101, 1, 2]
    assert out_scores[0].tolist() == pytest.approx([0.9, 0.7, 0.5, 0.5])
    # query 1: one entry, the rest padded
    assert out_ids[1].tolist() == [3, -1, -1, -1]
    assert out_scores[1, 0].item() == pytest.approx(0.1) and torch.isinf(out_scores[1, 1:]).all()
    # k_out < k_in
    out_ids, _ = tt.tt_merge_topk(ids, scores, [0, 100], 2)
    assert out_ids.tolist() == [[0, 101], [3, -1]]
    # b = 0
    e = torch.empty((2, 0, 4), dtype=torch.int32, device=dev)
    out_ids, _ = tt.tt_merge_topk(e, torch.empty((2, 0, 4), device=dev), [0, 100], 4)
    assert out_ids.shape == (0, 4)
    # bad arguments are refused before any device work
    with pytest.raises(tt.TTError) as err:
        tt.tt_merge_topk(ids, scores, [0, 100], 5)  # k_out > k_in
    assert err.value.status == tt.TT_ERR_INVALID_ARG
    with pytest.raises(tt.TTError) as err:
        tt.tt_merge_topk(ids, scores, [0, -1], 2)
    assert err.value.status == tt.TT_ERR_INVALID_ARG


def test_merge_long_lists_use_scratch():
    """parts * k_in above the shared-memory staging (4096 keys): the keys go
    through the stream-ordered scratch buffer."""
    _cuda()
    g = torch.Generator(device="cpu").manual_seed(7)
    parts, b, k = 6, 5, 1000
    scores = torch.rand((parts, b, k), generator=g).cuda()
    scores, _ = torch.sort(scores, dim=2, descending=True)
    ids = torch.arange(k, dtype=torch.int32).repeat(parts, b, 1).cuda()
    offsets = [p * 10_000 for p in range(parts)]
    out_ids, out_scores = tt.tt_merge_topk(ids.contiguous(), scores.contiguous(), offsets, k)
    flat_s = scores.permute(1, 0, 2).reshape(b, parts * k)
    flat_i = (ids + torch.tensor(offsets, dtype=torch.int32, device="cuda")[:, None, None]).permute(1, 0, 2)
    flat_i = flat_i.reshape(b, parts * k)
    # score descending, ties by ascending id: stable sort by id, then by score
    by_id = torch.argsort(flat_i, dim=1, stable=True)
    s1, i1 = torch.gather(flat_s, 1, by_id), torch.gather(flat_i, 1, by_id)
    order = torch.sort(s1, dim=1, descending=True, stable=True).indices
    want_s = torch.gather(s1, 1, order[:, :k])
    want_i = torch.gather(i1, 1, order[:, :k])
    assert torch.equal(out_scores, want_s)
    assert torch.equal(out_ids, want_i)
