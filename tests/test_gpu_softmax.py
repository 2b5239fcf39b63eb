"""In-batch sampled softmax on the GPU against the fp64 oracle. (GPU)

Both sides take the same seeded bf16 batch. Small batches are compared row
by row in full; the full-size batches on a seeded sample of rows, which the
oracle scores against every column (the columns are reordered so that the
sampled rows' positives come first; a log-sum-exp does not depend on the
order of its terms), plus properties that hold at any size.

Tolerance, from the arithmetic: each logit is an fp32 sum of d exact bf16
products, off by at most gamma_d * sum_k |u_k v_k| <= gamma_d |u| |v|
(gamma_d = d 2^-24 / (1 - d 2^-24)), divided by tau. lse moves by at most the
largest logit error; loss = lse - l_ii by twice that. On top come the
single-precision steps (the biased logit in base-2 units, ex2.approx with
relative error below 2^-22, fp32 sums over up to nc / 8 terms per thread,
log2): a relative 4e-6 of (1 + |lse|)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

tt = pytest.importorskip("exact_inner_product_b200")


def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _tolerances(inp, tau):
    u = inp["users"].float()
    v = inp["items"].float()
    d = u.shape[1]
    gamma = d * 2.0 ** -24 / (1 - d * 2.0 ** -24)
    bound = gamma * float(u.norm(dim=1).max()) * float(v.norm(dim=1).max()) / tau
    return bound, 2 * bound


def _oracle(inp, rows, tau, use):
    """fp64 lse and loss of the listed rows, each against every column."""
    nc = inp["items"].shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    rest = np.setdiff1d(np.arange(nc), rows)
    cols = np.concatenate([rows, rest])
    users = W.bf16_bits(inp["users"][torch.from_numpy(rows).to(inp["users"].device)])
    items = W.bf16_bits(inp["items"][torch.from_numpy(cols).to(inp["items"].device)])
    logq = inp["logq"].cpu().numpy().astype(np.float64)[cols] if "logq" in use else None
    ids = inp["item_ids"].cpu().numpy()[cols] if "ids" in use else None
    valid = inp["valid"].cpu().numpy()[cols] if "valid" in use else None
    lse, loss, _ = oracle.inbatch_softmax(users, items, tau, logq=logq, item_ids=ids, valid=valid)
    return lse, loss


def _run(inp, tau, use):
    return tt.tt_inbatch_softmax(inp["users"], inp["items"], tau,
                                 logq=inp["logq"] if "logq" in use else None,
                                 item_ids=inp["item_ids"] if "ids" in use else None,
                                 valid=inp["valid"] if "valid" in use else None)


def _compare(inp, tau, use, rows):
    lse, loss, mean = _run(inp, tau, use)
    want_lse, want_loss = _oracle(inp, rows, tau, use)
    tol_lse, tol_loss = _tolerances(inp, tau)
    got_lse = lse.double().cpu().numpy()[rows]
    got_loss = loss.double().cpu().numpy()[rows]
    fin = np.isfinite(want_lse)
    assert (np.isfinite(got_lse) == fin).all()
    assert (got_lse[~fin] == want_lse[~fin]).all()  # -inf where no column enters
    slack = 4e-6 * (1 + np.abs(want_lse[fin]))
    err_lse = np.abs(got_lse[fin] - want_lse[fin])
    assert (err_lse <= tol_lse + slack).all(), (err_lse.max(), tol_lse)
    err_loss = np.abs(got_loss - want_loss)
    slack_all = 4e-6 * (1 + np.abs(np.where(fin, want_lse, 0)))
    assert (err_loss <= tol_loss + slack_all).all(), (err_loss.max(), tol_loss)
    # the mean is the mean of the kernel's own per-row losses over valid rows
    rows_valid = inp["valid"].cpu().numpy()[:inp["users"].shape[0]] if "valid" in use else \
        np.ones(inp["users"].shape[0], dtype=bool)
    lv = loss.double().cpu().numpy()
    want_mean = lv[rows_valid].mean() if rows_valid.any() else 0.0
    assert abs(float(mean) - want_mean) <= 1e-6 * max(1.0, abs(want_mean))
    assert (lv[~rows_valid] == 0).all()
    return lse, loss, mean, err_lse.max() if err_lse.size else 0.0


FULL = ("logq", "ids", "valid")


@pytest.mark.parametrize("over,use", [
    ({"b": 384, "nc": 384, "d": 64, "catalogue": 500}, FULL),  # many accidental hits
    ({"b": 300, "nc": 1100, "d": 96, "catalogue": 3000}, FULL),  # shared negatives, ragged K and tiles
    ({"b": 129, "nc": 257, "d": 64, "catalogue": 50}, FULL),  # one row and one column past a tile
    ({"b": 256, "nc": 256, "d": 128}, ()),  # the plain in-batch loss
    ({"b": 200, "nc": 700, "d": 512, "catalogue": 400}, FULL),  # widest rows: two pipeline stages
    ({"b": 640, "nc": 2000, "d": 64, "tau": 1.0}, ("logq",)),
    ({"b": 512, "nc": 512, "d": 64, "pad_rate": 0.3}, ("ids", "valid")),
    # twenty items: groups of hundreds of rows, hits in every chunk of every warp
    ({"b": 4096, "nc": 6000, "d": 64, "catalogue": 20}, FULL),
    # uniform ids from a large catalogue: almost every row's only hit is its own positive
    ({"b": 3000, "nc": 3500, "d": 64, "zipf_s": 0.0}, FULL),
])
def test_small_batches_every_row(over, use):
    _cuda()
    w = W.batch("inbatch_b8192_d64", oracle_rows=0, **over)
    inp = W.batch_inputs(w, "cuda")
    _compare(inp, w.tau, use, np.arange(w.b))


@pytest.mark.parametrize("name", sorted(W.BATCHES))
def test_full_size_sampled_rows(name):
    _cuda()
    w = W.batch(name)
    inp = W.batch_inputs(w, "cuda")
    rows = W.oracle_row_ids(w)
    lse, loss, mean, _ = _compare(inp, w.tau, FULL, rows)
    # the same call again gives the same bits
    lse2, loss2, mean2 = _run(inp, w.tau, FULL)
    assert torch.equal(lse, lse2) and torch.equal(loss, loss2) and torch.equal(mean, mean2)


def test_many_columns_sampled_rows():
    """More than 2^20 columns: the bin order cuts each part into tiles of
    2048 elements."""
    _cuda()
    w = W.batch("inbatch_b8192_d64", b=700, nc=(1 << 20) + 3000, catalogue=5000)
    inp = W.batch_inputs(w, "cuda")
    rows = np.array([0, 1, 31, 32, 255, 256, 511, 600, 699], dtype=np.int64)
    _compare(inp, w.tau, FULL, rows)


def test_edge_cases():
    _cuda()
    dev = "cuda"
    d = 64
    # b = 0: the mean is 0 and nothing else is written
    u = torch.empty((0, d), dtype=torch.bfloat16, device=dev)
    v = torch.randn((5, d), device=dev).to(torch.bfloat16)
    lse, loss, mean = tt.tt_inbatch_softmax(u, v, 0.5)
    assert lse.numel() == 0 and float(mean) == 0.0
    # one row, one column: lse is the logit and the loss is 0
    u1 = torch.full((1, d), 0.125, device=dev).to(torch.bfloat16)
    v1 = torch.full((1, d), 0.25, device=dev).to(torch.bfloat16)
    lq = torch.tensor([-2.0], device=dev)
    lse, loss, mean = tt.tt_inbatch_softmax(u1, v1, 0.5, logq=lq)
    want = d * 0.125 * 0.25 / 0.5 + 2.0
    assert abs(float(lse[0]) - want) <= 1e-5 * want and float(loss[0]) == 0.0 and float(mean) == 0.0
    # every row invalid: loss 0, mean 0, lse -inf
    w = W.batch("inbatch_b8192_d64", b=70, nc=90, d=d)
    inp = W.batch_inputs(w, dev)
    none = torch.zeros(90, dtype=torch.bool, device=dev)
    lse, loss, mean = tt.tt_inbatch_softmax(inp["users"], inp["items"], w.tau, valid=none)
    assert torch.isinf(lse).all() and (lse < 0).all() and (loss == 0).all() and float(mean) == 0.0
    # all columns hold one item: each row keeps only its own positive, loss 0
    same = torch.full((90,), 7, dtype=torch.int64, device=dev)
    lse, loss, mean = tt.tt_inbatch_softmax(inp["users"], inp["items"], w.tau, item_ids=same)
    assert float(loss.abs().max()) <= 1e-6 and abs(float(mean)) <= 1e-6
    # the id the library's table reserves (INT64_MIN) is an ordinary id to the caller
    ids = inp["item_ids"].clone()
    ids[3] = ids[11] = -(2 ** 63)
    ws = torch.empty(tt.tt_inbatch_softmax_workspace(70, 90, d, True), dtype=torch.uint8, device=dev)
    lse, loss, _ = tt.tt_inbatch_softmax(inp["users"], inp["items"], w.tau, logq=inp["logq"], item_ids=ids,
                                         valid=inp["valid"], workspace=ws)
    want_lse, want_loss = _oracle({**inp, "item_ids": ids}, np.arange(70), w.tau, FULL)
    tol_lse, tol_loss = _tolerances(inp, w.tau)
    fin = np.isfinite(want_lse)
    assert np.allclose(lse.double().cpu().numpy()[fin], want_lse[fin], rtol=4e-6, atol=tol_lse + 4e-6)
    assert np.allclose(loss.double().cpu().numpy(), want_loss, rtol=4e-6, atol=tol_loss + 4e-6)


def test_validation():
    _cuda()
    dev = "cuda"
    u = torch.randn((8, 64), device=dev).to(torch.bfloat16)
    v = torch.randn((6, 64), device=dev).to(torch.bfloat16)
    with pytest.raises(tt.TTError) as err:  # nc < b
        tt.tt_inbatch_softmax(u, v, 1.0)
    assert err.value.status == tt.TT_ERR_INVALID_ARG
    with pytest.raises(tt.TTError) as err:  # fp32 rows: cast to bf16 first
        tt.tt_inbatch_softmax(u.float(), u.float(), 1.0)
    assert err.value.status == tt.TT_ERR_UNSUPPORTED
    with pytest.raises(tt.TTError) as err:
        tt.tt_inbatch_softmax(u, u, 0.0)
    assert err.value.status == tt.TT_ERR_INVALID_ARG
    small = torch.empty(16, dtype=torch.uint8, device=dev)
    with pytest.raises(tt.TTError) as err:
        tt.tt_inbatch_softmax(u, u, 1.0, workspace=small)
    assert err.value.status == tt.TT_ERR_INVALID_ARG
