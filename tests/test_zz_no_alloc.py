"""tt_score_topk_noalloc, the entry point for callers that must not allocate
device memory while they run (for instance a serving process whose memory
pool reserved the GPU at start-up, where a late cudaMalloc would fail or
stall the device). It works in a fixed array the library reserves on each
GPU instead of buffers grown with cudaMalloc.

The test calls it through the C ABI, twice on the same inputs with a
different call between them (the array keeps each call's leftovers, which
the next call must not see), and checks every result against the regular
tt_score_topk within the score tolerance of the other parity tests. Another
test checks that calls after the first leave the device's free memory
unchanged. It sits in a file of its own that
pytest collects last, and passes alone in a fresh process as well as after
the other tests.
"""
import ctypes
import math

import pytest
import torch

import parity
import workloads as W

pytestmark = pytest.mark.gpu

tt = pytest.importorskip("exact_inner_product_b200")


def _noalloc(rows, inv, q, k, tau, excl, ids, scores):
    return tt._lib.tt_score_topk_noalloc(
        ctypes.c_void_p(rows.data_ptr()), tt._dtype(rows), rows.shape[0], rows.shape[1],
        None if inv is None else ctypes.c_void_p(inv.data_ptr()), ctypes.c_void_p(q.data_ptr()),
        tt._dtype(q), q.shape[0], None if excl is None else ctypes.c_void_p(excl.data_ptr()),
        float(tau), int(k), ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(scores.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [
    ("small_batch", {"n": 150_001, "b": 40, "k": 300}),      # tensor-core scorer
    ("stream_b1", {"n": 120_003, "k": 100}),                  # streaming scorer, fp32 query
    ("masked_fused", {"n": 60_013, "b": 33, "k": 64}),        # raw corpus + norms, mask
]


@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_regular_entry_point(name, over):
    """Two calls with the same arguments, with a different call between them
    (more queries, a larger k, another tau, no mask), which leaves larger
    counts and looser thresholds in the shared array: every call must still
    equal tt_score_topk."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.workload(name, **over)
    raw_c = W.corpus(w, "cuda")
    raw_q = W.queries(w, "cuda")
    excl = W.exclusion_bits(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    ref_ids, ref_scores = tt.tt_score_topk(index, qn, w.k, tau=w.tau, exclude=excl)
    # the call in between: twice the queries (repeated), k * 3, tau 0.5, no mask
    q2 = torch.cat([qn, qn.flip(0)]).contiguous()
    k2 = min(3 * w.k, 2048)
    ref2_ids, ref2_scores = tt.tt_score_topk(index, q2, k2, tau=0.5)
    torch.cuda.synchronize()

    def check(ids, scores, want_ids, want_scores, tol):
        assert torch.equal(ids, want_ids)
        pad = torch.isinf(want_scores)
        assert torch.equal(pad, torch.isinf(scores))
        assert (scores[~pad] - want_scores[~pad]).abs().max().item() <= tol

    for step in range(3):
        if step == 1:
            ids = torch.full((q2.shape[0], k2), -7, dtype=torch.int32, device="cuda")
            scores = torch.full((q2.shape[0], k2), math.nan, dtype=torch.float32, device="cuda")
            st = _noalloc(index.rows, index.inv_norm, q2, k2, 0.5, None, ids, scores)
            assert st == tt.TT_OK, tt._lib.tt_last_error().decode()
            torch.cuda.synchronize()
            check(ids, scores, ref2_ids, ref2_scores, 2 * w.tolerance)
            continue
        ids = torch.full((w.b, w.k), -7, dtype=torch.int32, device="cuda")
        scores = torch.full((w.b, w.k), math.nan, dtype=torch.float32, device="cuda")
        st = _noalloc(index.rows, index.inv_norm, qn, w.k, w.tau, excl, ids, scores)
        assert st == tt.TT_OK, tt._lib.tt_last_error().decode()
        torch.cuda.synchronize()
        check(ids, scores, ref_ids, ref_scores, w.tolerance)


def test_noalloc_allocates_nothing_after_the_first_call():
    """After one warm-up call on the GPU (which may commit the fixed array:
    CUDA loads a module's device memory when first used), further calls leave
    the device's free memory unchanged: the single-SM tensor-core plan, the
    one-sample plan of a few queries on the streaming scorer and a wider
    batch, each called several times."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = W.workload("small_batch", n=150_001, b=200, k=300)
    raw_c = W.corpus(w, "cuda")
    raw_q = W.queries(w, "cuda")
    index, qn = parity.gpu_prepare(w, raw_c, raw_q)
    calls = []
    for b in (40, 4, 200):  # tensor-core levels, one sample (b <= 8), a wider batch
        ids = torch.empty((b, w.k), dtype=torch.int32, device="cuda")
        scores = torch.empty((b, w.k), dtype=torch.float32, device="cuda")
        calls.append((qn[:b].contiguous(), ids, scores))
    for q, ids, scores in calls:  # warm-up
        assert _noalloc(index.rows, None, q, w.k, w.tau, None, ids, scores) == tt.TT_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        for q, ids, scores in calls:
            assert _noalloc(index.rows, None, q, w.k, w.tau, None, ids, scores) == tt.TT_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def test_noalloc_rejects_batches_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rows = torch.nn.functional.normalize(torch.randn(1000, 64, device="cuda"), dim=1).to(torch.bfloat16)
    q = torch.randn(1000, 64, device="cuda").to(torch.bfloat16)
    ids = torch.empty((1000, 10), dtype=torch.int32, device="cuda")
    scores = torch.empty((1000, 10), dtype=torch.float32, device="cuda")
    st = _noalloc(rows, None, q, 10, 1.0, None, ids, scores)
    assert st == tt.TT_ERR_UNSUPPORTED
    assert "bytes" in tt._lib.tt_last_error().decode()
