"""Parity harness: run a workload through the CUDA library and through the
fp64 oracle from the same raw inputs, and compare.

Both sides start from the raw vectors drawn by ``workloads``; each side
normalises them with its own code (the CUDA path with
``tt_normalize_candidates``, the oracle in fp64 followed by one rounding to
the storage type), so no oracle input comes from the CUDA path.

Comparison rule (tol = the workload's score tolerance), per query:
 1. every returned id j has |s_gpu - s_oracle(j)| <= tol;
 2. returned ids are distinct and eligible, scores non-increasing, and the
    number of valid entries is min(k, eligible); padding is (-1, -inf);
 3. where the oracle's gap s_(k) - s_(k+1) exceeds tol, the returned id set
    equals the oracle's top-k set;
 4. at every rank whose neighbouring oracle gaps both exceed tol, the id
    equals the oracle's id at that rank;
 5. every returned id has s_oracle(j) >= s_(k) - tol;
 6. where the GPU's own scores tie exactly, ids ascend;
 7. every oracle top-k member whose score exceeds the k-th score by more
    than tol is returned (it cannot be displaced by rounding).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import workloads as W


def gpu_prepare(w: W.Workload, raw_corpus: torch.Tensor, raw_queries: torch.Tensor):
    """Normalise corpus and queries on the GPU; returns (index, queries_stored)."""
    import exact_inner_product_b200 as tt
    if w.store == "raw":
        inv = torch.empty((w.n,), dtype=torch.float32, device=raw_corpus.device)
        index = tt.tt_normalize_candidates(raw_corpus, inv, tt.TT_NORM_FUSED)
    else:
        dt = torch.float32 if w.store == "f32" else torch.bfloat16
        rows = torch.empty((w.n, w.d), dtype=dt, device=raw_corpus.device)
        index = tt.tt_normalize_candidates(raw_corpus, rows, tt.TT_NORM_STORE)
    qdt = torch.float32 if w.query_dtype == "f32" else torch.bfloat16
    qn = torch.empty((w.b, w.d), dtype=qdt, device=raw_queries.device)
    tt.tt_normalize_candidates(raw_queries, qn, tt.TT_NORM_STORE, make_index=False)
    return index, qn


class OracleSide:
    """The oracle's view of a workload: its own normalised corpus/queries."""

    def __init__(self, w: W.Workload, raw_corpus_np: np.ndarray, raw_queries_np: np.ndarray,
                 exclude_np: np.ndarray | None, qids: np.ndarray):
        self.w = w
        self.qids = qids
        self.exclude = exclude_np
        if w.store == "raw":
            self.corpus = raw_corpus_np
            self.norms = oracle.row_norms(raw_corpus_np)
        else:
            self.corpus = oracle.normalize(raw_corpus_np, w.store)
            self.norms = None
        self.queries = oracle.normalize(np.ascontiguousarray(raw_queries_np[qids]), w.query_dtype)

    def topk(self, k: int):
        return oracle.topk(self.queries, self.corpus, k, tau=self.tau, norms=self.norms,
                           exclude=self.exclude)

    @property
    def tau(self) -> float:
        return float(np.float32(self.w.tau))

    def scores_for(self, row: int, ids) -> np.ndarray:
        return oracle.scores_for(self.queries, row, self.corpus, ids, tau=self.tau, norms=self.norms)

    def eligible_count(self) -> int:
        if self.exclude is None:
            return self.w.n
        bits = np.unpackbits(self.exclude.view(np.uint8), bitorder="little")[:self.w.n]
        return int(self.w.n - bits.sum())

    def excluded(self, ids: np.ndarray) -> np.ndarray:
        if self.exclude is None:
            return np.zeros(ids.shape, dtype=bool)
        words = self.exclude.view(np.uint32)
        return ((words[ids >> 5] >> (ids & 31).astype(np.uint32)) & 1).astype(bool)


class OracleSideQ8(OracleSide):
    """The oracle's view of an int8 index: its own codes of its own
    normalised corpus rows, and of its own stored queries coded as given."""

    def __init__(self, w: W.Workload, raw_corpus_np: np.ndarray, raw_queries_np: np.ndarray,
                 exclude_np: np.ndarray | None, qids: np.ndarray):
        self.w = w
        self.qids = qids
        self.exclude = exclude_np
        self.vcodes, self.vscales = oracle.quantize(raw_corpus_np, True)
        stored_q = oracle.normalize(np.ascontiguousarray(raw_queries_np[qids]), w.query_dtype)
        self.qcodes, self.qscales = oracle.quantize(stored_q, False)

    def topk(self, k: int):
        return oracle.topk_q8(self.qcodes, self.qscales, self.vcodes, self.vscales, k, tau=self.tau,
                              exclude=self.exclude)

    def scores_for(self, row: int, ids) -> np.ndarray:
        return oracle.scores_for_q8(self.qcodes, self.qscales, row, self.vcodes, self.vscales, ids, tau=self.tau)


def gpu_prepare_q8(w: W.Workload, raw_corpus: torch.Tensor, raw_queries: torch.Tensor):
    """int8 index of the corpus (normalise + code on the GPU) and the stored
    (normalised) queries; tt_score_topk codes the queries itself."""
    import exact_inner_product_b200 as tt
    codes = torch.empty((w.n, w.d), dtype=torch.int8, device=raw_corpus.device)
    scales = torch.empty((w.n,), dtype=torch.float32, device=raw_corpus.device)
    index = tt.tt_quantize_candidates(raw_corpus, codes, scales)
    qdt = torch.float32 if w.query_dtype == "f32" else torch.bfloat16
    qn = torch.empty((w.b, w.d), dtype=qdt, device=raw_queries.device)
    tt.tt_normalize_candidates(raw_queries, qn, tt.TT_NORM_STORE, make_index=False)
    return index, qn


def q8_tolerance(w: W.Workload) -> float:
    """Score tolerance of the int8 path: 2e-3 / tau. A code that rounds the
    other way on the two sides (their normalised rows can differ in the last
    fp32 bit) moves a score by us * scale * |code| / tau <= max|u| max|v| / 127
    / tau, about 7e-4 / tau for unit rows at d = 128; such flips are rare (a
    value must sit within ~1e-5 of a half step)."""
    return 2e-3 / float(np.float32(w.tau))


def run_case_q8(w: W.Workload, device="cuda", **options):
    """int8 index: generate, run both sides, compare."""
    import exact_inner_product_b200 as tt
    raw_c = W.corpus(w, device)
    raw_q = W.queries(w, device)
    excl = W.exclusion_bits(w, device)
    index, qn = gpu_prepare_q8(w, raw_c, raw_q)
    ids, scores = tt.tt_score_topk(index, qn, w.k, tau=w.tau, exclude=excl, **options)
    torch.cuda.synchronize()
    qids = W.oracle_query_ids(w)
    gi = ids.cpu().numpy()[qids]
    gs = scores.cpu().numpy()[qids]
    st = tt.tt_last_stats(index)
    side = OracleSideQ8(w, W.to_numpy_rows(raw_c), raw_q.cpu().numpy(),
                        None if excl is None else excl.cpu().numpy().view(np.uint32), qids)
    del raw_c
    res = compare(gi, gs, side, w.k, q8_tolerance(w))
    return res, st


def compare(gpu_ids: np.ndarray, gpu_scores: np.ndarray, side: OracleSide, k: int, tol: float,
            o_ids: np.ndarray | None = None, o_scores: np.ndarray | None = None) -> dict:
    """Apply the comparison rule to the sampled rows. gpu_* are [len(qids), k]."""
    if o_ids is None:
        o_ids, o_scores = side.topk(k + 1)
    eligible = side.eligible_count()
    want_valid = min(k, eligible)
    stats = {"queries": len(side.qids), "max_abs_err": 0.0, "set_checked": 0, "rank_checked": 0}
    for r_i in range(len(side.qids)):
        ids = gpu_ids[r_i]
        sc = gpu_scores[r_i]
        valid = ids >= 0
        nv = int(valid.sum())
        assert nv == want_valid, (r_i, nv, want_valid)
        assert valid[:nv].all() and not valid[nv:].any(), "padding must be at the tail"
        assert np.isneginf(sc[nv:]).all(), "padding scores must be -inf"
        vid = ids[:nv].astype(np.int64)
        assert len(np.unique(vid)) == nv, "duplicate ids"
        assert (vid < side.w.n).all()
        assert not side.excluded(vid).any(), "excluded candidate returned"
        vs = sc[:nv].astype(np.float64)
        assert (np.diff(vs) <= 0).all(), "scores must be non-increasing"
        tie = np.diff(vs) == 0
        assert (np.diff(vid)[tie] > 0).all(), "equal scores must come in ascending id order"
        so = side.scores_for(r_i, vid)
        err = np.abs(vs - so).max() if nv else 0.0
        stats["max_abs_err"] = max(stats["max_abs_err"], float(err))
        assert err <= tol, (r_i, err)
        oi = o_ids[r_i]
        os_ = o_scores[r_i]
        if nv == 0:
            continue
        kth = os_[nv - 1]
        assert (so >= kth - tol).all(), "a returned candidate is not near the top-k"
        sure = oi[:nv][os_[:nv] > kth + tol]
        missing = set(sure.tolist()) - set(vid.tolist())
        assert not missing, (r_i, "oracle top-k members missing", sorted(missing)[:5])
        stats["sure_checked"] = stats.get("sure_checked", 0) + len(sure)
        nxt = os_[nv] if nv < len(os_) else -math.inf
        if kth - nxt > tol:
            assert set(vid.tolist()) == set(oi[:nv].tolist()), (r_i, "top-k set differs")
            stats["set_checked"] += 1
        for r in range(nv):
            gap_above = (os_[r - 1] - os_[r]) if r > 0 else math.inf
            gap_below = (os_[r] - os_[r + 1]) if r + 1 < len(os_) else math.inf
            if gap_above > tol and gap_below > tol:
                assert vid[r] == oi[r], (r_i, r, vid[r], oi[r])
                stats["rank_checked"] += 1
    return stats


def run_case(w: W.Workload, device="cuda", **options):
    """Generate, run both sides, compare. Returns (stats, tt_stats)."""
    import exact_inner_product_b200 as tt
    raw_c = W.corpus(w, device)
    raw_q = W.queries(w, device)
    excl = W.exclusion_bits(w, device)
    index, qn = gpu_prepare(w, raw_c, raw_q)
    ids, scores = tt.tt_score_topk(index, qn, w.k, tau=w.tau, exclude=excl, **options)
    torch.cuda.synchronize()
    qids = W.oracle_query_ids(w)
    gi = ids.cpu().numpy()[qids]
    gs = scores.cpu().numpy()[qids]
    st = tt.tt_last_stats(index)
    side = OracleSide(w, W.to_numpy_rows(raw_c), raw_q.cpu().numpy(),
                      None if excl is None else excl.cpu().numpy().view(np.uint32), qids)
    del raw_c
    res = compare(gi, gs, side, w.k, w.tolerance)
    return res, st
