"""The int8 path (recsys_two_tower_model.py `compute_top_k_int8`) against
the oracle: corpus coding on the GPU against the oracle's codes, and exact
top-k over int8 codes on the streaming (dp4a) and tensor-core (kind::i8)
scorers, with masks, tau, ties and edge cases. (GPU)"""
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


@pytest.mark.parametrize("name,n", [("stream_b1", 50_003), ("masked_fused", 20_011), ("tiny_f32", 400)])
def test_coding_matches_oracle(name, n):
    """Codes equal the oracle's except where the two sides' normalised values
    (fp32 norm here, fp64 there) straddle a rounding half step: then they
    differ by one. Scales agree to fp32 rounding."""
    _cuda()
    w = W.workload(name, n=n)
    raw = W.corpus(w, "cuda")
    codes = torch.empty((n, w.d), dtype=torch.int8, device="cuda")
    scales = torch.empty((n,), dtype=torch.float32, device="cuda")
    tt.tt_quantize_candidates(raw, codes, scales, make_index=False)
    oc, os_ = oracle.quantize(W.to_numpy_rows(raw), True)
    diff = np.abs(codes.cpu().numpy().astype(np.int32) - oc.astype(np.int32))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.9995
    assert np.allclose(scales.cpu().numpy(), os_, rtol=5e-7, atol=0)
    assert np.abs(codes.cpu().numpy().astype(np.int32)).max() <= 127


@pytest.mark.parametrize("dtype,d", [(torch.float32, 128), (torch.bfloat16, 256), (torch.float32, 64)])
def test_coding_is_the_ieee_fp32_formula_bitwise(dtype, d):
    """The coding of tt_quantize_candidates is the page's formula in IEEE fp32
    (w = fl(v / norm), scale = max(fl(max|w| / 127), 1e-12), code =
    round_half_even(fl(w / scale)), clipped), bit for bit, although the kernel
    divides once per row: torch's fp32 operations (IEEE division and square
    root on the GPU) evaluate the formula as written. Rows of small integers
    make the sum of squares exact, so the norm does not depend on the order
    of the sum; rows with a value on a half step of the code grid test the
    kernel's near-tie fallback."""
    _cuda()
    g = torch.Generator(device="cpu").manual_seed(11)
    n = 60_000
    v = torch.randint(-40, 41, (n, d), generator=g).to(torch.float32)
    v[::7, 0] = 0.0
    v[1::97] = 0.0                                   # zero rows: scale 1e-12, codes 0
    # rows whose values sit on code half steps: max|v| = 254 puts v = 1 at code 0.5
    v[2::11, 0] = 254.0
    v[2::11, 1:6] = torch.tensor([1.0, 3.0, -5.0, 127.0, -253.0])
    x = v.to(dtype).cuda()
    codes = torch.empty((n, d), dtype=torch.int8, device="cuda")
    scales = torch.empty((n,), dtype=torch.float32, device="cuda")
    tt.tt_quantize_candidates(x, codes, scales, make_index=False)
    xf = x.float()
    ss = (xf * xf).sum(1)                            # exact: small integers
    norm = torch.sqrt(torch.clamp(ss, min=1e-12))
    # every division tensor by tensor: a Python-scalar divisor may be turned
    # into a multiply by its reciprocal, which is not the IEEE quotient
    w = xf / norm[:, None]
    sc = torch.clamp(w.abs().amax(1) / torch.full_like(ss, 127.0), min=1e-12)
    want = torch.clamp(torch.round(w / sc[:, None]), -127, 127).to(torch.int8)
    bad = (scales != sc).nonzero()
    assert bad.numel() == 0, (bad.numel(), bad[:3].tolist(), scales[bad[:3, 0]].tolist(), sc[bad[:3, 0]].tolist())
    bad = (codes != want).nonzero()
    assert bad.numel() == 0, (bad.numel(), bad[:3].tolist())
    # quotients within the kernel's margin of a half step occurred (v = +-1, +-3, ... -> code +-0.5, +-1.5, ...)
    q = (w / sc[:, None])[2::11, 1:6]
    assert ((q - q.floor() - 0.5).abs() < 1e-5).float().mean() > 0.5


CASES = [
    # name, overrides, expected path
    ("stream_b1", {"n": 200_037}, 1),
    ("stream_b1", {"n": 150_001, "b": 5, "k": 64}, 1),
    ("small_batch", {"n": 300_077, "tau": 1.0}, 2),
    ("small_batch", {"n": 100_003, "b": 9, "k": 17}, 2),
    ("large_batch", {"n": 400_005, "b": 300, "k": 1000, "oracle_queries": 12}, 3),
    ("large_batch", {"n": 250_001, "b": 200, "k": 300, "oracle_queries": 12}, 2),
    ("masked_fused", {"n": 200_099, "b": 260, "oracle_queries": 12}, 3),
    ("masked_fused", {"n": 120_031, "b": 3, "k": 256}, 1),
    # the pass after the one-sample estimate scores its first rows before the
    # threshold lands: two queries per block with a mask, and a corpus with
    # more rows per thread than are deferred
    ("masked_fused", {"n": 150_011, "b": 2, "k": 64}, 1),
    ("stream_b1", {"n": 1_500_007, "k": 100}, 1),
]


@pytest.mark.parametrize("name,over,path", CASES, ids=[f"{c[0]}-{i}" for i, c in enumerate(CASES)])
def test_int8_parity(name, over, path):
    _cuda()
    w = W.workload(name, **over)
    res, st = parity.run_case_q8(w)
    assert st["path"] == path, st
    assert res["max_abs_err"] <= parity.q8_tolerance(w)
    assert res.get("sure_checked", 0) > 0


def test_int8_both_scorers_agree():
    """The dp4a streaming scorer, the kind::i8 tensor-core scorer and its
    SM-pair form compute the same exact integer sums and the same score
    arithmetic, so their results are identical."""
    _cuda()
    w = W.workload("small_batch", n=70_001, b=40, k=100, tau=1.0)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    index, qn = parity.gpu_prepare_q8(w, raw_c, raw_q)
    a = tt.tt_score_topk(index, qn, w.k, path=1)
    assert tt.tt_last_stats(index)["path"] == 1
    b = tt.tt_score_topk(index, qn, w.k, path=2)
    assert tt.tt_last_stats(index)["path"] == 2
    c = tt.tt_score_topk(index, qn, w.k, path=3)
    assert tt.tt_last_stats(index)["path"] == 3
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])
    res, _ = parity.run_case_q8(w, path=1)
    assert res["max_abs_err"] <= parity.q8_tolerance(w)


def test_int8_ties_and_edges():
    _cuda()
    d = 64
    # identical rows: every score ties; ids must come out 0..k-1 on both scorers
    row = torch.nn.functional.normalize(torch.randn(1, d), dim=1)
    raw = row.repeat(5000, 1).cuda().contiguous()
    codes = torch.empty((5000, d), dtype=torch.int8, device="cuda")
    scales = torch.empty((5000,), dtype=torch.float32, device="cuda")
    index = tt.tt_quantize_candidates(raw, codes, scales)
    for path, b in ((1, 2), (2, 40), (3, 260)):
        q = torch.randn(b, d, device="cuda")
        ids, sc = tt.tt_score_topk(index, q, 300, path=path)
        assert (ids.cpu() == torch.arange(300, dtype=torch.int32)[None, :]).all()
        assert (sc == sc[:, :1]).all()
    # k > n pads; everything excluded pads
    small = tt.tt_index_wrap(codes[:40].contiguous(), scales[:40].contiguous())
    q = torch.randn(12, d, device="cuda")
    ids, sc = tt.tt_score_topk(small, q, 50)
    assert (ids[:, 40:] == -1).all() and torch.isinf(sc[:, 40:]).all()
    excl = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    ids, _ = tt.tt_score_topk(small, q, 5, exclude=excl)
    assert (ids == -1).all()
    # int8 rows need the scales and d % 32 == 0
    with pytest.raises(tt.TTError) as e:
        tt.tt_index_wrap(codes)
    assert e.value.status == tt.TT_ERR_INVALID_ARG
    odd = torch.empty((10, 48), dtype=torch.int8, device="cuda")
    ix48 = tt.tt_index_wrap(odd, torch.ones(10, device="cuda"))
    with pytest.raises(tt.TTError) as e:
        tt.tt_score_topk(ix48, torch.randn(2, 48, device="cuda"), 3)
    assert e.value.status == tt.TT_ERR_UNSUPPORTED
    # several result sets by type stay on the single-SM kernel for int8 rows
    types = torch.zeros(5000, dtype=torch.uint8, device="cuda")
    ids_t, _ = tt.tt_score_topk_types(index, torch.randn(300, d, device="cuda"), 3, types, [0])
    assert tt.tt_last_stats(index)["path"] == 2 and (ids_t[0] == torch.arange(3, dtype=torch.int32, device="cuda")).all()


def test_int8_pair_negative_thresholds():
    """k close to n: the k-th best score is negative, so the integer fast test
    of the SM-pair kernel (which needs a positive threshold) is bypassed and
    every score takes the exact test; the result still equals the other
    scorers' and the oracle's."""
    _cuda()
    w = W.workload("large_batch", n=3_001, b=270, k=2048, oracle_queries=6)
    raw_c, raw_q = W.corpus(w, "cuda"), W.queries(w, "cuda")
    index, qn = parity.gpu_prepare_q8(w, raw_c, raw_q)
    a = tt.tt_score_topk(index, qn, w.k, path=2)
    c = tt.tt_score_topk(index, qn, w.k, path=3)
    assert tt.tt_last_stats(index)["path"] == 3
    assert torch.equal(a[0], c[0]) and torch.equal(a[1], c[1])
    assert (c[1][:, -1] < 0).float().mean() > 0.5  # mostly negative k-th scores
    res, _ = parity.run_case_q8(w, path=3)
    assert res["max_abs_err"] <= parity.q8_tolerance(w)
