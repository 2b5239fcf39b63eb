"""CUDA path vs the fp64 oracle on seeded inputs (GPU).

Sizes are small enough for the oracle to finish in seconds, yet span several
tiles (32-row streaming tiles, 128-row tensor-core tiles, 256-query tiles,
256-row tiles of the SM-pair kernel) with ragged tails. Each case calls the library through its C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import workloads as W

pytestmark = pytest.mark.gpu

tt = pytest.importorskip("exact_inner_product_b200")


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


CASES = [
    # name, overrides, expected path
    ("tiny_f32", {}, 1),
    ("stream_b1", {"n": 200_037}, 1),
    ("stream_b1", {"n": 150_001, "b": 5, "k": 64}, 1),
    ("small_batch", {"n": 300_077}, 2),
    ("small_batch", {"n": 100_003, "b": 9, "k": 17}, 2),
    ("large_batch", {"n": 400_005, "b": 300, "k": 1000, "oracle_queries": 12}, 3),
    ("large_batch", {"n": 250_001, "b": 200, "k": 300, "oracle_queries": 12}, 2),
    ("masked_fused", {"n": 200_099, "b": 520, "oracle_queries": 12}, 2),
    ("masked_fused", {"n": 120_031, "b": 3, "k": 256}, 1),
]


@pytest.mark.parametrize("name,over,path", CASES, ids=[f"{c[0]}-{i}" for i, c in enumerate(CASES)])
def test_parity_scaled(name, over, path):
    _cuda()
    w = W.workload(name, **over)
    res, st = parity.run_case(w)
    assert st["path"] == path, st
    assert res["max_abs_err"] <= w.tolerance


@pytest.mark.parametrize("path,b", [(1, 3), (2, 40), (3, 260)])
def test_limits_widest_rows_and_largest_k(path, b):
    """d = 512 (the widest rows) with k = 2048 (the largest k) on every
    scorer: the query tile and ring shrink to fit shared memory, and the
    final selection sorts 2048 keys."""
    _cuda()
    w = W.workload("large_batch", n=30_011, d=512, b=b, k=2048, n_clusters=64, oracle_queries=6)
    res, st = parity.run_case(w, path=path)
    assert st["path"] == path
    assert res["max_abs_err"] <= w.tolerance


@pytest.mark.parametrize("path", [1, 2, 3])
def test_every_scorer_agrees_with_oracle(path):
    _cuda()
    w = W.workload("small_batch", n=70_001, b=40, k=100, tau=1.0)
    res, st = parity.run_case(w, path=path)
    assert st["path"] == path


def test_pair_kernel_with_norms_and_mask():
    """The SM-pair kernel on a raw corpus with per-row norms, tau and an
    exclusion mask (the automatic choice sends such corpora to the single-SM
    kernel, so it is forced here)."""
    _cuda()
    w = W.workload("masked_fused", n=200_099, b=520, oracle_queries=12)
    res, st = parity.run_case(w, path=3)
    assert st["path"] == 3
    assert res["max_abs_err"] <= w.tolerance


def test_normalize_matches_oracle():
    _cuda()
    for name, n in (("tiny_f32", 400), ("stream_b1", 50_003), ("masked_fused", 20_011)):
        w = W.workload(name, n=n)
        raw = W.corpus(w, "cuda")
        raw_np = W.to_numpy_rows(raw)
        if w.store == "raw":
            inv = torch.empty((n,), dtype=torch.float32, device="cuda")
            tt.tt_normalize_candidates(raw, inv, tt.TT_NORM_FUSED, make_index=False)
            ref = 1.0 / oracle.row_norms(raw_np)
            got = inv.cpu().numpy().astype(np.float64)
            assert np.allclose(got, ref, rtol=3e-7, atol=0)
            continue
        dt = torch.float32 if w.store == "f32" else torch.bfloat16
        out = torch.empty((n, w.d), dtype=dt, device="cuda")
        tt.tt_normalize_candidates(raw, out, tt.TT_NORM_STORE, make_index=False)
        ref = oracle.normalize(raw_np, w.store)
        got = W.to_numpy_rows(out)
        if w.store == "bf16":
            # each element equals the once-rounded fp64 value or is one bf16 ulp away
            diff = np.abs(got.astype(np.int32) - ref.astype(np.int32))
            assert diff.max() <= 1
            assert (diff == 0).mean() > 0.999
        else:
            assert np.allclose(got, ref, rtol=4e-7, atol=1e-30)


def _index_from_rows(rows_np, dtype=torch.float32):
    rows = torch.from_numpy(np.ascontiguousarray(rows_np)).to("cuda", dtype)
    return tt.tt_index_wrap(rows), rows


def _pad16(a):
    a = np.asarray(a, dtype=np.float32)
    out = np.zeros((a.shape[0], 16), dtype=np.float32)
    out[:, :a.shape[1]] = a
    return out


@pytest.mark.parametrize("path", [1, 2, 3])
def test_hand_worked_h2(path):
    """The hand-worked d=4 example (zero-padded to d=16) through both scorers."""
    _cuda()
    import oracle_pins
    g = oracle_pins.golden()["H2_topk"]
    V = _pad16(g["corpus"])
    if path >= 2:  # tensor cores need a bf16 corpus with d >= 64
        V = np.pad(V, ((0, 0), (0, 48)))
    dtype = torch.float32 if path == 1 else torch.bfloat16
    index, rows = _index_from_rows(V, dtype)
    q = torch.from_numpy(np.pad(np.array([g["query"]], dtype=np.float32), ((0, 0), (0, V.shape[1] - 4))))
    q = q.repeat(16, 1).to("cuda", dtype).contiguous()
    for case in g["cases"]:
        excl = None
        if case["exclude"]:
            bits = np.zeros(6, dtype=bool)
            bits[case["exclude"]] = True
            excl = torch.from_numpy(oracle_pins.pack_bits(bits).view(np.int32)).cuda()
        ids, scores = tt.tt_score_topk(index, q, case["k"], tau=case["tau"], exclude=excl, path=path)
        want = [float("-inf") if s == "-inf" else s for s in case["scores"]]
        for row in range(q.shape[0]):
            assert ids[row].tolist() == case["ids"], (case, ids[row])
            assert scores[row].tolist() == want


def test_ties_across_tiles():
    """All rows identical: every score ties; ids must be 0..k-1 on every path."""
    _cuda()
    n, d = 70_000, 64
    row = torch.randn(1, d)
    rows = (row / row.norm()).repeat(n, 1).to("cuda", torch.bfloat16).contiguous()
    index = tt.tt_index_wrap(rows)
    for path, b in ((1, 2), (2, 40), (3, 300)):
        q = torch.randn(b, d, device="cuda").to(torch.bfloat16)
        ids, scores = tt.tt_score_topk(index, q, 700, path=path)
        assert (ids.cpu() == torch.arange(700, dtype=torch.int32)[None, :]).all()
        assert (scores == scores[:, :1]).all()


def test_identity_corpus():
    _cuda()
    d = 64
    E = torch.eye(d)
    index, rows = _index_from_rows(E.numpy(), torch.bfloat16)
    q = E[[0, 7, 63] * 4].to("cuda", torch.bfloat16).contiguous()
    for path in (1, 2, 3):
        ids, scores = tt.tt_score_topk(index, q, 6, path=path)
        for r, t in enumerate([0, 7, 63] * 4):
            assert ids[r].tolist() == [t] + [j for j in range(d) if j != t][:5]
            assert scores[r].tolist() == [1.0, 0, 0, 0, 0, 0]


def test_edge_cases():
    _cuda()
    d = 64
    rows = torch.nn.functional.normalize(torch.randn(300, d), dim=1).to("cuda", torch.bfloat16)
    index = tt.tt_index_wrap(rows.contiguous())
    q = torch.randn(12, d, device="cuda").to(torch.bfloat16)
    # k > n: padding
    ids, scores = tt.tt_score_topk(index, q, 400)
    assert (ids[:, 300:] == -1).all() and torch.isinf(scores[:, 300:]).all()
    assert sorted(ids[0, :300].tolist()) == list(range(300))
    # everything excluded
    excl = torch.full(((300 + 31) // 32,), -1, dtype=torch.int32, device="cuda")
    ids, scores = tt.tt_score_topk(index, q, 5, exclude=excl)
    assert (ids == -1).all()
    # b = 0
    ids, scores = tt.tt_score_topk(index, q[:0], 5)
    assert ids.shape == (0, 5)
    # empty corpus
    empty = tt.tt_index_wrap(torch.empty((0, d), dtype=torch.bfloat16, device="cuda"))
    ids, scores = tt.tt_score_topk(empty, q, 3)
    assert (ids == -1).all() and torch.isinf(scores).all()
    # a tiny corpus below one tile, on every path
    small = tt.tt_index_wrap(rows[:7].contiguous())
    for path in (1, 2, 3):
        ids, _ = tt.tt_score_topk(small, q, 3, path=path)
        s = (q.float() @ rows[:7].float().T)
        ref = torch.sort(s, dim=1, descending=True, stable=True).indices[:, :3].to(torch.int32)
        assert (ids == ref).all()


@pytest.mark.parametrize("opts", [{"rank_scale_pct": 3}, {"cap": 256, "force_levels": 2},
                                  {"force_levels": 1}, {"force_levels": 4},
                                  {"rank_scale_pct": 3, "path": 3}, {"cap": 256, "path": 3}])
def test_rescans_stay_exact(opts):
    """Thresholds deliberately mis-estimated (tiny ranks, tiny buffers): the
    on-device exactness check must hand the lists to the exact fallback scan,
    and the answer must still match the oracle."""
    _cuda()
    k = 60 if "cap" in opts else 200
    w = W.workload("small_batch", n=200_003, b=24, k=k)
    res, st = parity.run_case(w, **opts)
    if "rank_scale_pct" in opts or "cap" in opts:
        assert st["rescans"] >= 1, st


def test_repeat_runs_are_bitwise_identical():
    _cuda()
    w = W.workload("large_batch", n=300_001, b=260, k=100)
    raw_c = W.corpus(w, "cuda")
    raw_q = W.queries(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    first = tt.tt_score_topk(index, qn, w.k)
    for _ in range(3):
        again = tt.tt_score_topk(index, qn, w.k)
        assert torch.equal(first[0], again[0]) and torch.equal(first[1], again[1])
    assert tt.tt_last_stats(index)["path"] == 3
    # batch invariance: a query's result does not depend on the rest of the
    # batch, nor on which tensor-core kernel the batch size selects
    sub = tt.tt_score_topk(index, qn[5:6].repeat(20, 1).contiguous(), w.k)
    assert tt.tt_last_stats(index)["path"] == 2
    assert torch.equal(sub[0][0], first[0][5])
    assert torch.equal(sub[1][0], first[1][5])
    single = tt.tt_score_topk(index, qn, w.k, path=2)
    assert torch.equal(single[0], first[0]) and torch.equal(single[1], first[1])


def test_bounded_wait_expiry_is_reported():
    """The tensor-core pass is told (test hook) to withhold its first corpus
    copy: the wait for it gives up after its time limit and every role of the
    kernel drains and exits. The search was only enqueued (the call returned
    TT_OK); its outputs become (id -1, score NaN), and the expiry is reported
    once, as TT_ERR_TIMEOUT, by tt_index_check or else by the next call on the
    handle. The device and the handle stay usable: the next search gives the
    earlier answer."""
    import time
    _cuda()
    w = W.workload("small_batch", n=100_003, b=40, k=50)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    good = [t.clone() for t in tt.tt_score_topk(index, qn, w.k, path=2)]
    torch.cuda.synchronize()
    t0 = time.time()
    bad_ids, bad_scores = tt.tt_score_topk(index, qn, w.k, path=2, force_levels=1, withhold_copy=1)
    with pytest.raises(tt.TTError) as e:
        tt.tt_index_check(index)
    assert e.value.status == tt.TT_ERR_TIMEOUT
    assert time.time() - t0 < 60
    assert (bad_ids == -1).all() and torch.isnan(bad_scores).all()
    tt.tt_index_check(index)  # reported once
    again = tt.tt_score_topk(index, qn, w.k, path=2)
    torch.cuda.synchronize()
    assert torch.equal(good[0], again[0]) and torch.equal(good[1], again[1])
    # unchecked: the next call reports it, without enqueueing anything
    tt.tt_score_topk(index, qn, w.k, path=2, force_levels=1, withhold_copy=1)
    torch.cuda.synchronize()
    with pytest.raises(tt.TTError) as e:
        tt.tt_score_topk(index, qn, w.k, path=2)
    assert e.value.status == tt.TT_ERR_TIMEOUT
    again = tt.tt_score_topk(index, qn, w.k, path=2)
    tt.tt_index_check(index)
    assert torch.equal(good[0], again[0]) and torch.equal(good[1], again[1])


def test_search_is_asynchronous():
    """tt_score_topk only enqueues: two searches issued back to back return
    before the stream has finished the first, and both results are right."""
    import time
    _cuda()
    n, d, k = 8_000_000, 128, 100
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    rows = torch.randn(n, d, device="cuda", generator=g).to(torch.bfloat16)
    q = torch.randn(1024, d, device="cuda", generator=g).to(torch.bfloat16)
    index = tt.tt_index_wrap(rows)
    ref = [t.clone() for t in tt.tt_score_topk(index, q, k)]  # warm-up: grows the work memory
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0 = time.perf_counter()
    first = tt.tt_score_topk(index, q, k)
    second = tt.tt_score_topk(index, q[:512].contiguous(), k)
    t_calls = time.perf_counter() - t0
    pending = not stream.query()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    tt.tt_score_topk(index, q, k)
    e1.record(stream)
    torch.cuda.synchronize()
    assert pending, "the calls waited for their own work"
    assert t_calls * 1e3 < 2 * e0.elapsed_time(e1), (t_calls, e0.elapsed_time(e1))
    assert torch.equal(first[0], ref[0]) and torch.equal(first[1], ref[1])
    assert torch.equal(second[0], ref[0][:512]) and torch.equal(second[1], ref[1][:512])
    tt.tt_index_check(index)


def test_host_buffer_entry_point():
    """tt_score_topk_host (host queries in, host results out, queries
    normalised on the device) equals the device-buffer call."""
    _cuda()
    w = W.workload("small_batch", n=200_003, b=40, k=100)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    ids, scores = tt.tt_score_topk(index, qn, w.k, tau=w.tau)
    torch.cuda.synchronize()
    hid, hsc = tt.tt_score_topk_host(index, raw_q.cpu().pin_memory(), w.k, tau=w.tau, normalize=True,
                                     norm_dtype=torch.bfloat16)
    assert not hid.is_cuda
    assert torch.equal(hid, ids.cpu()) and torch.equal(hsc, scores.cpu())
    # pageable memory, queries already normalised
    hid, hsc = tt.tt_score_topk_host(index, qn.cpu(), w.k, tau=w.tau, normalize=False)
    assert torch.equal(hid, ids.cpu()) and torch.equal(hsc, scores.cpu())
    # the streaming scorer with an fp32 query
    w1 = W.workload("stream_b1", n=150_001)
    raw_c, raw_q = W.corpus(w1, "cuda"), W.queries(w1, "cuda")
    index, qn = parity.gpu_prepare(w1, raw_c, raw_q)
    ids, scores = tt.tt_score_topk(index, qn, w1.k)
    hid, hsc = tt.tt_score_topk_host(index, raw_q.cpu(), w1.k, normalize=True, norm_dtype=torch.float32)
    assert torch.equal(hid, ids.cpu()) and torch.equal(hsc, scores.cpu())


def test_rejects_host_pointers_and_bad_args():
    _cuda()
    rows = torch.randn(100, 64, device="cuda").to(torch.bfloat16)
    index = tt.tt_index_wrap(rows)
    q_host = torch.randn(4, 64).to(torch.bfloat16)
    with pytest.raises(tt.TTError) as e:
        tt.tt_score_topk(index, q_host, 5, out_ids=torch.empty(4, 5, dtype=torch.int32, device="cuda"),
                         out_scores=torch.empty(4, 5, device="cuda"))
    assert e.value.status == tt.TT_ERR_INVALID_ARG
    q = torch.randn(4, 64, device="cuda").to(torch.bfloat16)
    for bad in ({"tau": 0.0}, {"tau": float("nan")}, {"k": 0}):
        with pytest.raises(tt.TTError) as e:
            kw = {"k": 5, **bad}
            tt.tt_score_topk(index, q, kw.pop("k"), **kw)
        assert e.value.status == tt.TT_ERR_INVALID_ARG
    with pytest.raises(tt.TTError) as e:
        tt.tt_score_topk(index, q, 4096)
    assert e.value.status == tt.TT_ERR_UNSUPPORTED


@pytest.mark.parametrize("name,over,opts", [
    ("stream_b1", {"n": 300_007, "k": 100}, {}),
    ("stream_b1", {"n": 250_013, "b": 6, "k": 333}, {}),
    ("masked_fused", {"n": 180_017, "b": 2, "k": 64, "oracle_queries": 0}, {}),
    ("stream_b1", {"n": 200_003, "b": 3, "k": 100}, {"rank_scale_pct": 3}),
])
def test_sampled_plan_small_batches(name, over, opts):
    """A few queries on the streaming scorer: one sample of the corpus sets
    the threshold in one launch (a two-level plan whose level 1 is every S-th
    row, S odd). The result matches the oracle; with the rank scaled down the
    filter keeps too few candidates and the exact fallback restores the
    answer."""
    _cuda()
    w = W.workload(name, **over)
    res, st = parity.run_case(w, **opts)
    assert st["path"] == 1 and st["levels"] == 2 and st["sampled"], st
    stride = st["level_stride"][1]
    assert stride % 2 == 1 and st["level_rows"][1] == -(-w.n // stride)
    assert res["max_abs_err"] <= w.tolerance
    if opts:
        assert st["rescans"] >= 1, st
    else:
        assert st["rescans"] == 0, st


def test_sampled_plan_int8_and_f32_rows():
    """The sample is scored with each row type's own arithmetic."""
    _cuda()
    w = W.workload("stream_b1", n=120_011, b=4, k=50)
    res, st = parity.run_case_q8(w)
    assert st["path"] == 1 and st["levels"] == 2 and st["rescans"] == 0, st
    w = W.workload("tiny_f32", n=90_001, d=64, b=3, k=40, oracle_queries=0)
    res, st = parity.run_case(w)
    assert st["path"] == 1 and st["levels"] == 2 and st["rescans"] == 0, st
    assert res["max_abs_err"] <= w.tolerance


@pytest.mark.parametrize("k", [1, 31, 32, 33, 64, 65, 128, 129, 256, 257, 513, 1000, 1024])
@pytest.mark.parametrize("path,b", [(1, 2), (2, 24), (3, 256)])
def test_select_widths(path, b, k):
    """The selects rank up to 4096 kept keys by buckets (r <= 1024), keep
    the best r <= 256 keys sorted in registers (32, 64, 128 or 256 per warp)
    where the buckets cannot decide, and use the radix select beyond that; k
    on both sides of each width, on every scorer (on the streaming scorer
    the sample estimate's rank varies with k too)."""
    _cuda()
    w = W.workload("small_batch", n=60_013, b=b, k=k, tau=1.0, oracle_queries=6)
    res, st = parity.run_case(w, path=path)
    assert st["path"] == path and st["rescans"] == 0, st
    assert res["max_abs_err"] <= w.tolerance and res["set_checked"] + res["rank_checked"] > 0, res


@pytest.mark.parametrize("name,over", [
    ("tiny_f32", {"n": 200_003, "d": 64, "b": 1, "k": 50, "oracle_queries": 0}),   # fp32 rows
    ("stream_b1", {"n": 1_500_007, "b": 1, "k": 100}),                            # rows after the deferred four
    ("masked_fused", {"n": 400_009, "b": 2, "k": 64, "oracle_queries": 0}),       # two queries, mask, norms
])
def test_pass_scores_rows_before_the_threshold(name, over):
    """After the one-sample estimate the streaming pass scores each thread's
    first rows before waiting for the threshold and filters them afterwards
    (one or two queries per block). Every form of that pass matches the
    oracle: fp32 rows, a corpus with more rows per thread than are deferred,
    and a masked raw corpus with norms."""
    _cuda()
    w = W.workload(name, **over)
    res, st = parity.run_case(w)
    assert st["path"] == 1 and st["sampled"] and st["rescans"] == 0, st
    assert res["max_abs_err"] <= w.tolerance
