"""Several result sets from one call (recsys_two_tower_model.py `forward`:
`dataset_ranges` and `target_dataset_types`): each set's list must equal
the single-set call over the same candidates bit for bit, and agree with the
oracle. (GPU)"""
import numpy as np
import pytest
import torch

import oracle
import oracle_pins
import parity
import workloads as W

pytestmark = pytest.mark.gpu

tt = pytest.importorskip("exact_inner_product_b200")


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _mask_from_bool(excluded: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(oracle_pins.pack_bits(excluded).view(np.int32)).cuda()


def _bits(excl: torch.Tensor | None, n: int) -> np.ndarray:
    if excl is None:
        return np.zeros(n, dtype=bool)
    return np.unpackbits(excl.cpu().numpy().view(np.uint8), bitorder="little")[:n].astype(bool)


@pytest.mark.parametrize("name,over", [("small_batch", {"n": 200_011, "b": 24, "k": 100}),
                                       ("large_batch", {"n": 150_007, "b": 300, "k": 200}),
                                       ("masked_fused", {"n": 100_003, "b": 3, "k": 50})])
def test_ranges_equal_single_calls(name, over):
    _cuda()
    w = W.workload(name, **over)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    excl = W.exclusion_bits(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    n = w.n
    ranges = [(0, n // 3), (n // 3, n // 3 + 12_345), (n // 3 + 12_345, n), (777, 778), (5, 5), (1000, 60_001)]
    ids, scores = tt.tt_score_topk_ranges(index, qn, w.k, ranges, tau=w.tau, exclude=excl)
    ex_all = _bits(excl, n)
    for r, (a, b) in enumerate(ranges):
        rows = index.rows[a:b]
        inv = None if index.inv_norm is None else index.inv_norm[a:b]
        if b > a:
            sub = tt.tt_index_wrap(rows.contiguous(), None if inv is None else inv.contiguous())
            sub_ex = _mask_from_bool(ex_all[a:b]) if excl is not None else None
            wi, ws = tt.tt_score_topk(sub, qn, w.k, tau=w.tau, exclude=sub_ex)
            wi = torch.where(wi >= 0, wi + a, wi)
        else:
            wi = torch.full((w.b, w.k), -1, dtype=torch.int32, device="cuda")
            ws = torch.full((w.b, w.k), float("-inf"), device="cuda")
        assert torch.equal(ids[r], wi), (name, r)
        assert torch.equal(scores[r], ws), (name, r)


def test_ranges_against_oracle():
    _cuda()
    w = W.workload("small_batch", n=120_001, b=16, k=60, tau=1.0)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    a, b = 30_017, 90_001
    ids, scores = tt.tt_score_topk_ranges(index, qn, w.k, [(a, b)])
    corpus = oracle.normalize(W.to_numpy_rows(raw_c), w.store)
    queries = oracle.normalize(raw_q.cpu().numpy(), w.query_dtype)
    oi, os_ = oracle.topk(queries, corpus[a:b], w.k)
    got_i = ids[0].cpu().numpy()
    got_s = scores[0].cpu().numpy().astype(np.float64)
    assert ((got_i >= a) & (got_i < b)).all()
    for q in range(w.b):
        so = oracle.scores_for(queries, q, corpus, got_i[q])
        assert np.abs(so - got_s[q]).max() <= w.tolerance
        sure = oi[q][os_[q] > os_[q][-1] + w.tolerance] + a
        assert set(sure.tolist()) <= set(got_i[q].tolist())


@pytest.mark.parametrize("b,path", [(3, 1), (40, 2), (260, 3)])
def test_types_equal_masked_calls_and_oracle(b, path):
    """One fused pass for all the requested types (a type asked twice gets the
    same lists twice), on each scorer."""
    _cuda()
    w = W.workload("large_batch", n=90_001, b=b, k=80, mask_rate=0.1)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    excl = W.exclusion_bits(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    g = torch.Generator(device="cpu").manual_seed(31)
    types_np = torch.randint(0, 4, (w.n,), generator=g, dtype=torch.uint8).numpy()
    types = torch.from_numpy(types_np).cuda()
    sets = [2, 0, 7, 2]  # type 7 has no candidates: all padding
    ids, scores = tt.tt_score_topk_types(index, qn, w.k, types, sets, exclude=excl)
    assert tt.tt_last_stats(index)["path"] == path
    ex_all = _bits(excl, w.n)
    corpus = oracle.normalize(W.to_numpy_rows(raw_c), w.store)
    queries = oracle.normalize(raw_q.cpu().numpy()[:8], w.query_dtype)
    nq_check = min(8, w.b)
    for t_i, t in enumerate(sets):
        combined = ex_all | (types_np != t)
        wi, ws = tt.tt_score_topk(index, qn, w.k, exclude=_mask_from_bool(combined))
        assert torch.equal(ids[t_i], wi) and torch.equal(scores[t_i], ws), t
        if t == 7:
            assert (ids[t_i] == -1).all()
            continue
        oi, os_ = oracle.topk(queries, corpus, w.k, exclude=oracle_pins.pack_bits(combined))
        got = ids[t_i, :nq_check].cpu().numpy()
        assert (types_np[got[got >= 0]] == t).all()
        for q in range(nq_check):
            sure = oi[q][os_[q] > os_[q][-1] + w.tolerance]
            assert set(sure.tolist()) <= set(got[q].tolist())


def test_set_calls_reject_bad_arguments():
    _cuda()
    rows = torch.nn.functional.normalize(torch.randn(100, 64), dim=1).to("cuda", torch.bfloat16)
    index = tt.tt_index_wrap(rows.contiguous())
    q = torch.randn(4, 64, device="cuda").to(torch.bfloat16)
    for bad in ([(5, 3)], [(0, 101)], [(-1, 4)]):
        with pytest.raises(tt.TTError) as e:
            tt.tt_score_topk_ranges(index, q, 3, bad)
        assert e.value.status == tt.TT_ERR_INVALID_ARG
    types = torch.zeros(100, dtype=torch.uint8, device="cuda")
    with pytest.raises(tt.TTError) as e:
        tt.tt_score_topk_types(index, q, 3, types, [256])
    assert e.value.status == tt.TT_ERR_INVALID_ARG
