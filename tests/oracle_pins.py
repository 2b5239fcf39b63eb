"""Pins for the fp64 oracle: checks that tie it to something other than itself.

Each ``check_*`` takes an ``oracle.OracleLib`` and raises ``AssertionError`` on
a mismatch. ``test_oracle_pins.py`` runs them against the oracle as built;
``test_oracle_mutants.py`` runs them against copies of ``oracle.c`` with one
planted mistake each and expects every copy to fail at least one check.

The pins are: hand-worked closed forms (``golden/hand_worked.json``, H1-H3
for the fp path, H5-H7 for int8 coding and scoring), the
rank characterisation of top-k evaluated in exact rational arithmetic on tiny
inputs, fp32 -> bf16 rounding by an independent library routine, and
invariants that any correct implementation satisfies (unit norms, scaling by
powers of two, permutation of the corpus, prefix property of top-k, 1/tau
scaling, masks that exclude nothing, duplicate queries). For the in-batch
sampled softmax: the logQ article's printed three-item example (H8), torch's
fp64 cross-entropy on the dense masked logits, the two-column logistic form,
equal-logit counts, and invariants (a constant shift of log q, permutation of
the batch, accidental hits as dropped columns, power-of-two scaling).
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_worked.json")


def golden() -> dict:
    with open(GOLDEN) as f:
        return json.load(f)


def pack_bits(excluded: np.ndarray) -> np.ndarray:
    """Pack a boolean [n] array into uint32 words, bit (j & 31) of word j >> 5."""
    n = excluded.shape[0]
    words = np.zeros((n + 31) // 32, dtype=np.uint32)
    for j in np.nonzero(excluded)[0]:
        words[j >> 5] |= np.uint32(1) << np.uint32(j & 31)
    return words


def _as_float(x):
    return -math.inf if x == "-inf" else float(x)


def bf16_bits_via_torch(values_f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (nearest-even) by torch's own conversion, as uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(values_f32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits: int) -> float:
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


# ---------------------------------------------------------------------------


def check_bf16_rounding(o):
    # closed forms
    assert o.bf16_from_double(0.6) == 0x3F1A
    assert o.bf16_from_double(0.8) == 0x3F4D
    assert o.bf16_from_double(0.1) == 0x3DCD
    assert o.bf16_from_double(1.0) == 0x3F80
    assert o.bf16_from_double(-2.0) == 0xC000
    assert o.bf16_from_double(0.0) == 0x0000
    assert o.bf16_from_double(-0.0) == 0x8000
    # ties to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> 1 (even)
    assert o.bf16_from_double(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even) -> 1 + 2^-6
    assert o.bf16_from_double(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above a tie rounds up
    assert o.bf16_from_double(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    # subnormal: 2^-130 is exactly representable (bf16 subnormal quantum 2^-133)
    assert o.bf16_from_double(2.0 ** -130) == 0x0008
    # independent route: for fp32-representable values, one rounding to bf16
    # must agree with torch's fp32 -> bf16 conversion
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-3).astype(np.float32),
        (rng.integers(-2 ** 15, 2 ** 15, 2000) * 2.0 ** -20).astype(np.float32),
    ])
    ref = bf16_bits_via_torch(vals)
    mine = np.array([o.bf16_from_double(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(mine, ref), "bf16 rounding disagrees with torch's fp32->bf16"


def check_h1_normalize(o):
    g = golden()["H1_normalize"]
    rows = np.array(g["rows"], dtype=np.float32)
    out_bf = o.normalize(rows, "bf16")
    assert np.array_equal(out_bf, np.array(g["expected_bf16_bits"], dtype=np.uint16)), out_bf
    out_f = o.normalize(rows, "f32")
    exp_f = np.array(g["expected_f64"], dtype=np.float64)
    assert np.allclose(out_f, exp_f, rtol=2e-7, atol=0), (out_f, exp_f)
    norms = o.row_norms(rows)
    assert np.allclose(norms, [5.0, 1e-6, 1e-6, 5.0], rtol=1e-7), norms


def check_normalize_invariants(o):
    rng = np.random.default_rng(11)
    for d in (16, 48, 128, 256):
        x = rng.standard_normal((64, d)).astype(np.float32)
        x[3] = 0.0
        x[5] *= 1e-9  # below the norm floor
        y = o.normalize(x, "f32").astype(np.float64)
        big = (x.astype(np.float64) ** 2).sum(1) >= 1e-12
        # unit length where the floor is not active
        assert np.allclose(np.linalg.norm(y[big], axis=1), 1.0, atol=1e-6)
        # below the floor: divided by exactly 1e-6
        assert np.allclose(y[~big], x[~big].astype(np.float64) * 1e6, rtol=1e-6, atol=1e-30)
        # scaling a row by a power of two changes nothing (above the floor)
        for s in (-3, 5):
            xs = (x * np.float32(2.0 ** s)).astype(np.float32)
            keep = big & ((xs.astype(np.float64) ** 2).sum(1) >= 1e-12)
            assert np.array_equal(o.normalize(xs, "f32")[keep], o.normalize(x, "f32")[keep])
            assert np.array_equal(o.normalize(xs, "bf16")[keep], o.normalize(x, "bf16")[keep])
        # flipping the sign of a row flips its output; permuting coordinates permutes it
        assert np.array_equal(o.normalize(-x, "f32"), -o.normalize(x, "f32"))
        perm = rng.permutation(d)
        assert np.array_equal(o.normalize(x[:, perm], "f32"), o.normalize(x, "f32")[:, perm])
        # direction is kept: y_i * x_j == y_j * x_i
        xd = x[big].astype(np.float64)
        cross = y[big][:, :, None] * xd[:, None, :] - y[big][:, None, :] * xd[:, :, None]
        assert np.abs(cross).max() < 1e-5 * np.abs(xd).max()
        # row norms: |a e_i| = |a|; scaling by powers of two
        assert np.allclose(o.row_norms(np.eye(d, dtype=np.float32) * -3.0), 3.0)
        nrm = o.row_norms(x)
        assert np.allclose(o.row_norms(x * np.float32(4.0))[big], 4.0 * nrm[big], rtol=1e-12)
    # bf16 input: the same invariants hold for bf16-stored raw rows
    xb = bf16_bits_via_torch(rng.standard_normal((32, 64)).astype(np.float32)).reshape(32, 64)
    yb = o.normalize(xb, "f32").astype(np.float64)
    assert np.allclose(np.linalg.norm(yb, axis=1), 1.0, atol=1e-6)


def check_h2_topk(o):
    g = golden()["H2_topk"]
    V = np.array(g["corpus"], dtype=np.float32)
    u = np.array([g["query"]], dtype=np.float32)
    for case in g["cases"]:
        excl = np.zeros(V.shape[0], dtype=bool)
        excl[case["exclude"]] = True
        mask = pack_bits(excl) if case["exclude"] else None
        ids, scores = o.topk(u, V, case["k"], tau=case["tau"], exclude=mask)
        assert ids[0].tolist() == case["ids"], (case, ids)
        assert np.array_equal(scores[0], np.array([_as_float(s) for s in case["scores"]])), (case, scores)


def check_h3_fused(o):
    g = golden()["H3_fused"]
    V = np.array(g["corpus_raw"], dtype=np.float32)
    u = np.array([g["query"]], dtype=np.float32)
    norms = o.row_norms(V)
    assert np.allclose(norms, g["norms"], rtol=1e-9), norms
    for case in g["cases"]:
        ids, scores = o.topk(u, V, case["k"], tau=case["tau"], norms=norms)
        assert ids[0].tolist() == case["ids"], (case, ids)
        assert np.allclose(scores[0], case["scores"], rtol=1e-7, atol=0), (case, scores)


def check_exact_rational(o):
    """Rank characterisation in exact arithmetic: the entry at rank r has
    exactly r eligible candidates better than it (higher score, or equal score
    and lower id), and its score is the exact dot product over tau."""
    rng = np.random.default_rng(3)
    for trial in range(60):
        n = int(rng.integers(1, 40))
        d = int(rng.integers(1, 6))
        b = 3
        k = int(rng.integers(1, n + 4))
        V = (rng.integers(-4, 5, size=(n, d)) / 4.0).astype(np.float32)
        Q = (rng.integers(-4, 5, size=(b, d)) / 4.0).astype(np.float32)
        tau = float(rng.choice([1.0, 0.5, 0.25, 2.0]))
        excl = rng.random(n) < (0.25 if trial % 2 else 0.0)
        mask = pack_bits(excl) if excl.any() else None
        ids, scores = o.topk(Q, V, k, tau=tau, exclude=mask)
        for qi in range(b):
            exact = [sum(Fraction(float(Q[qi, i])) * Fraction(float(V[j, i])) for i in range(d))
                     / Fraction(tau) for j in range(n)]
            eligible = [j for j in range(n) if not excl[j]]
            got = ids[qi].tolist()
            for r in range(k):
                if r >= len(eligible):
                    assert got[r] == -1 and scores[qi, r] == -math.inf, (trial, qi, r)
                    continue
                j = got[r]
                assert 0 <= j < n and not excl[j], (trial, qi, r, j)
                assert Fraction(float(scores[qi, r])) == exact[j], (trial, qi, r)
                better = sum(1 for i in eligible
                             if exact[i] > exact[j] or (exact[i] == exact[j] and i < j))
                assert better == r, (trial, qi, r, better)
            assert len(set(x for x in got if x >= 0)) == min(k, len(eligible))


def check_invariants(o):
    rng = np.random.default_rng(5)
    n, d, b, k = 300, 32, 6, 20
    V = o.normalize(rng.standard_normal((n, d)).astype(np.float32), "f32")
    Q = o.normalize(rng.standard_normal((b, d)).astype(np.float32), "f32")
    ids, scores = o.topk(Q, V, k)
    # corpus permutation: ids map through the permutation, scores are unchanged
    perm = rng.permutation(n)
    ids_p, scores_p = o.topk(Q, V[perm], k)
    assert np.array_equal(perm[ids_p], ids)
    assert np.array_equal(scores_p, scores)
    # top-k is the prefix of top-(k+1)
    ids1, scores1 = o.topk(Q, V, k + 1)
    assert np.array_equal(ids1[:, :k], ids) and np.array_equal(scores1[:, :k], scores)
    # scores are non-increasing
    assert (np.diff(scores, axis=1) <= 0).all()
    # tau = 0.25: same ids, scores times 4 exactly
    ids_t, scores_t = o.topk(Q, V, k, tau=0.25)
    assert np.array_equal(ids_t, ids) and np.array_equal(scores_t, 4.0 * scores)
    # a mask that excludes nothing equals no mask
    ids_m, scores_m = o.topk(Q, V, k, exclude=np.zeros((n + 31) // 32, dtype=np.uint32))
    assert np.array_equal(ids_m, ids) and np.array_equal(scores_m, scores)
    # excluding each query's best candidate removes it and shifts the rest up
    for qi in range(b):
        excl = np.zeros(n, dtype=bool)
        excl[ids[qi, 0]] = True
        ids_x, _ = o.topk(Q[qi:qi + 1], V, k, exclude=pack_bits(excl))
        assert np.array_equal(ids_x[0, :k - 1], ids[qi, 1:])
    # excluded candidates never appear
    excl = rng.random(n) < 0.5
    ids_e, _ = o.topk(Q, V, k, exclude=pack_bits(excl))
    assert not excl[ids_e[ids_e >= 0]].any()
    # duplicate queries give identical rows; a query's row does not depend on the batch
    Qd = np.concatenate([Q, Q[:2]])
    ids_d, scores_d = o.topk(Qd, V, k)
    assert np.array_equal(ids_d[b:], ids[:2]) and np.array_equal(scores_d[b:], scores[:2])
    ids_s, scores_s = o.topk(Q[3:4], V, k)
    assert np.array_equal(ids_s[0], ids[3]) and np.array_equal(scores_s[0], scores[3])
    # k > n pads with (-1, -inf)
    ids_big, scores_big = o.topk(Q[:1], V[:5], 8)
    assert (ids_big[0, 5:] == -1).all() and np.isneginf(scores_big[0, 5:]).all()
    assert sorted(ids_big[0, :5].tolist()) == list(range(5))
    # fused norms: scaling a raw row by a power of two leaves its fused score unchanged
    raw = rng.standard_normal((n, d)).astype(np.float32)
    scale = (2.0 ** rng.integers(-4, 5, size=(n, 1))).astype(np.float32)
    ids_f, sc_f = o.topk(Q, raw, k, norms=o.row_norms(raw))
    ids_g, sc_g = o.topk(Q, raw * scale, k, norms=o.row_norms(raw * scale))
    assert np.array_equal(ids_f, ids_g) and np.array_equal(sc_f, sc_g)


def check_ties(o):
    # all rows identical: every score ties, ids come out 0..k-1
    row = np.array([[0.25, -0.5, 0.75, 0.125]], dtype=np.float32)
    V = np.repeat(row, 1000, axis=0)
    Q = np.array([[1.0, 1.0, 1.0, 1.0], [-1.0, 0.5, 0.0, 2.0]], dtype=np.float32)
    ids, scores = o.topk(Q, V, 300)
    assert (ids == np.arange(300)[None, :]).all()
    assert (scores == scores[:, :1]).all()
    # identity corpus: query e_t scores 1 at t and 0 elsewhere
    d = 24
    E = np.eye(d, dtype=np.float32)
    for t in (0, 7, 23):
        ids, scores = o.topk(E[t:t + 1], E, 6)
        expect = [t] + [j for j in range(d) if j != t][:5]
        assert ids[0].tolist() == expect, (t, ids)
        assert scores[0].tolist() == [1.0, 0, 0, 0, 0, 0]


def check_scores_for(o):
    rng = np.random.default_rng(9)
    V = rng.standard_normal((50, 8)).astype(np.float32)
    Q = rng.standard_normal((2, 8)).astype(np.float32)
    norms = o.row_norms(V)
    ids, scores = o.topk(Q, V, 10, tau=0.5, norms=norms)
    for qi in range(2):
        s = o.scores_for(Q, qi, V, ids[qi], tau=0.5, norms=norms)
        assert np.array_equal(s, scores[qi])
    # closed form: e_0 against the H2 corpus
    g = golden()["H2_topk"]
    s = o.scores_for(np.array([g["query"]], dtype=np.float32), 0,
                     np.array(g["corpus"], dtype=np.float32), [0, 1, 2, 3, 4, 5])
    assert s.tolist() == [0.5, 1.0, 0.5, -1.0, 0.0, 0.75]


def check_bf16_inputs(o):
    """bf16-stored inputs: the closed forms of H1/H2/H3 hold when the rows and
    queries are handed over as bf16 (all values there are exact in bf16)."""
    g1 = golden()["H1_normalize"]
    rows = np.array(g1["rows"], dtype=np.float32)[[0, 1, 3]]
    rows_bf = bf16_bits_via_torch(rows).reshape(rows.shape)
    assert np.array_equal(o.normalize(rows_bf, "bf16"),
                          np.array(g1["expected_bf16_bits"], dtype=np.uint16)[[0, 1, 3]])
    assert np.allclose(o.row_norms(rows_bf), [5.0, 1e-6, 5.0], rtol=1e-12)
    g2 = golden()["H2_topk"]
    V = bf16_bits_via_torch(np.array(g2["corpus"], dtype=np.float32)).reshape(6, 4)
    u = bf16_bits_via_torch(np.array([g2["query"]], dtype=np.float32)).reshape(1, 4)
    for case in g2["cases"]:
        excl = np.zeros(6, dtype=bool)
        excl[case["exclude"]] = True
        ids, scores = o.topk(u, V, case["k"], tau=case["tau"],
                             exclude=pack_bits(excl) if case["exclude"] else None)
        assert ids[0].tolist() == case["ids"], (case, ids)
        assert np.array_equal(scores[0], np.array([_as_float(s) for s in case["scores"]]))
    g3 = golden()["H3_fused"]
    raw = np.array(g3["corpus_raw"], dtype=np.float32)[:6]
    raw_bf = bf16_bits_via_torch(raw).reshape(raw.shape)
    ids, scores = o.topk(u, raw_bf, 3, norms=o.row_norms(raw_bf))
    assert ids[0].tolist() == [1, 5, 0]
    assert np.allclose(scores[0], [1.0, 0.8017837257372732, 0.5], rtol=1e-12)


def _check_quantize_golden(o, g):
    rows = np.array(g["rows"], dtype=np.float32)
    codes, scales = o.quantize(rows, g["normalise"])
    assert codes.tolist() == g["expected_codes"], (codes, g["expected_codes"])
    for s, want in zip(scales.tolist(), g["expected_scales"]):
        assert abs(s - want) <= g["scale_rel_tol"] * abs(want) + 1e-30, (s, want)


def check_h5_quantize(o):
    _check_quantize_golden(o, golden()["H5_quantize"])


def check_h6_quantize_ties(o):
    _check_quantize_golden(o, golden()["H6_quantize_ties"])


def check_h7_int8_score(o):
    g = golden()["H7_int8_score"]
    vc, vs = o.quantize(np.array(g["corpus_raw"], dtype=np.float32), True)
    qc, qs = o.quantize(np.array([g["query"]], dtype=np.float32), False)
    ids, scores = o.topk_q8(qc, qs, vc, vs, g["k"], tau=g["tau"])
    assert ids[0].tolist() == g["expected_ids"]
    for s, want in zip(scores[0].tolist(), g["expected_scores"]):
        assert abs(s - want) <= g["rel_tol"] * abs(want) + 1e-12, (s, want)
    # the listed-candidate scorer agrees
    s2 = o.scores_for_q8(qc, qs, 0, vc, vs, [2, 0], tau=g["tau"])
    assert s2.tolist() == [scores[0, 2], scores[0, 0]]


def check_quantize_invariants(o):
    """Codes stay in [-127, 127]; a non-zero row reaches 127 in magnitude; each
    dequantised value is within half a scale step of the fp32 row value it
    codes; signs agree; the scale is max|w| / 127 to fp32 rounding; a power of
    two times a row (not normalised) keeps the codes and scales the scale."""
    rng = np.random.default_rng(17)
    for d in (16, 64, 128, 256):
        x = (rng.standard_normal((80, d)) * rng.lognormal(0, 1, (80, 1))).astype(np.float32)
        for normalise in (False, True):
            codes, scales = o.quantize(x, normalise)
            assert codes.dtype == np.int8 and np.abs(codes.astype(np.int32)).max() <= 127
            assert (np.abs(codes.astype(np.int32)).max(axis=1) == 127).all()
            w = x.astype(np.float64)
            if normalise:
                w = w / np.sqrt(np.maximum((w * w).sum(axis=1, keepdims=True), 1e-12))
            w32 = w.astype(np.float32).astype(np.float64)
            maxabs = np.abs(w32).max(axis=1)
            assert np.allclose(scales, maxabs / 127, rtol=2.4e-7, atol=0)
            deq = codes.astype(np.float64) * scales.astype(np.float64)[:, None]
            assert (np.abs(deq - w32) <= 0.5 * scales.astype(np.float64)[:, None] * (1 + 2e-5)).all()
            nz = codes != 0
            assert (np.sign(codes[nz]) == np.sign(w32[nz])).all()
        c1, s1 = o.quantize(x, False)
        c2, s2 = o.quantize((x * 8).astype(np.float32), False)
        assert (c1 == c2).all() and np.allclose(s2, s1 * 8, rtol=0, atol=0)
        # normalising first makes the codes independent of the row's length
        c3, _ = o.quantize((x * 8).astype(np.float32), True)
        c4, _ = o.quantize(x, True)
        assert (c3 == c4).all()


def check_int8_topk_invariants(o):
    """The int8 top-k is the top-k of the dequantised vectors' dot products:
    compared with the fp64 top-k of (codes * scale) rows, and 1/tau only scales."""
    rng = np.random.default_rng(23)
    n, d, b, k = 400, 32, 5, 25
    V = rng.standard_normal((n, d)).astype(np.float32)
    Q = rng.standard_normal((b, d)).astype(np.float32)
    vc, vs = o.quantize(V, True)
    qc, qs = o.quantize(Q, False)
    ids, scores = o.topk_q8(qc, qs, vc, vs, k)
    deq_v = (vc.astype(np.float64) * vs.astype(np.float64)[:, None])
    deq_q = (qc.astype(np.float64) * qs.astype(np.float64)[:, None])
    full = deq_q @ deq_v.T
    for q in range(b):
        order = sorted(range(n), key=lambda j: (-full[q, j], j))[:k]
        assert ids[q].tolist() == order
        assert np.allclose(scores[q], full[q, order], rtol=1e-12, atol=1e-15)
    ids2, scores2 = o.topk_q8(qc, qs, vc, vs, k, tau=0.25)
    assert (ids2 == ids).all() and np.allclose(scores2, scores * 4, rtol=1e-15)
    # exclusion removes exactly the excluded ids
    ex = np.zeros(n, dtype=bool)
    ex[ids[:, 0]] = True
    ids3, _ = o.topk_q8(qc, qs, vc, vs, k, exclude=pack_bits(ex))
    assert not np.isin(ids3, np.nonzero(ex)[0]).any()


# ---- in-batch sampled softmax ----------------------------------------------


def _unit_rows(idx, d):
    """Rows of the identity: row t is e_{idx[t]} (exact in every storage type)."""
    out = np.zeros((len(idx), d), dtype=np.float32)
    out[np.arange(len(idx)), idx] = 1.0
    return out


def check_h8_logq_worked(o):
    """The logQ article's three-item example: a batch that holds each item in
    proportion to q recovers the full-softmax denominator (times the batch
    size) once log q is subtracted, and reproduces the printed pressure
    ratios without it."""
    g = golden()["H8_logq_worked"]
    mult = g["multiplicities"]
    col_item = np.repeat(np.arange(3), mult)
    ncol = len(col_item)
    d = 16
    V = _unit_rows(col_item, d)
    U = np.zeros((ncol, d), dtype=np.float32)
    U[0, :3] = [2.0, 1.0, 0.0]  # user 0's logits against A, B, C (its positive is a copy of A)
    q = np.array(g["q"], dtype=np.float64)[col_item]
    press = g["printed_corrected_pressures"]
    tol = 0.5 * 10.0 ** -g["printed_digits"]
    lse, _, _ = o.inbatch_softmax(U, V, 1.0, logq=np.log(q))
    assert abs(math.exp(lse[0]) - ncol * sum(press)) <= ncol * 3 * tol, (math.exp(lse[0]), ncol * sum(press))
    lse_u, _, _ = o.inbatch_softmax(U, V, 1.0)
    z_unc = math.exp(lse_u[0])
    assert abs(z_unc - sum(m * p for m, p in zip(mult, press))) <= 20 * tol, z_unc
    share_full = [p / sum(press) for p in press]
    ratio_a = mult[0] * press[0] / z_unc / share_full[0]
    ratio_c = mult[2] * press[2] / z_unc / share_full[2]
    assert round(ratio_a, 2) == g["printed_ratio_uncorrected_to_correct"]["A"], ratio_a
    assert round(ratio_c, 2) == g["printed_ratio_uncorrected_to_correct"]["C"], ratio_c


def _random_batch(seed, b, nc, d, dup=True, invalid=True):
    rng = np.random.default_rng(seed)
    U = (rng.standard_normal((b, d)) / math.sqrt(d)).astype(np.float32)
    V = (rng.standard_normal((nc, d)) / math.sqrt(d)).astype(np.float32)
    logq = np.log(rng.uniform(1e-4, 1.0, nc))
    ids = rng.integers(0, nc * 4, nc).astype(np.int64)
    if dup:  # a few accidental hits: rows sharing an item, and a shared negative equal to a positive
        ids[3] = ids[7]
        ids[b - 1] = ids[5] = ids[0]
        if nc > b:
            ids[nc - 1] = ids[2]
    valid = np.ones(nc, dtype=bool)
    if invalid:
        valid[[1, b - 2]] = False
    return U, V, logq, ids, valid


def _dense_reference(U, V, tau, logq, ids, valid):
    """Row-wise cross-entropy of the masked logit matrix by torch's own
    fp64 routine (the form `in_batch_loss` / `corrected_in_batch_loss` call)."""
    b, nc = U.shape[0], V.shape[0]
    logits = torch.from_numpy(U.astype(np.float64)) @ torch.from_numpy(V.astype(np.float64)).T / tau
    if logq is not None:
        logits = logits - torch.from_numpy(logq)[None, :]
    keep = torch.ones((b, nc), dtype=torch.bool)
    if valid is not None:
        keep &= torch.from_numpy(valid)[None, :]
    if ids is not None:
        t = torch.from_numpy(ids)
        hit = t[:b, None] == t[None, :]
        hit[torch.arange(b), torch.arange(b)] = False
        keep &= ~hit
    logits = logits.masked_fill(~keep, -math.inf)
    ce = torch.nn.functional.cross_entropy(logits, torch.arange(b), reduction="none")
    lse = torch.logsumexp(logits, dim=1)
    return lse.numpy(), ce.numpy()


def check_inbatch_library(o):
    """Against torch's fp64 cross-entropy and logsumexp on the dense masked
    logits, with and without each of logq, item ids, validity and shared
    negatives."""
    for seed, b, nc, d in ((1, 12, 12, 16), (2, 16, 23, 32), (3, 9, 9, 64)):
        U, V, logq, ids, valid = _random_batch(seed, b, nc, d)
        for use_q in (False, True):
            for use_ids in (False, True):
                for use_valid in (False, True):
                    tau = 0.07 if use_q else 1.0
                    args = dict(logq=logq if use_q else None, item_ids=ids if use_ids else None,
                                valid=valid if use_valid else None)
                    lse, loss, mean = o.inbatch_softmax(U, V, tau, **args)
                    want_lse, want_ce = _dense_reference(U, V, tau, args["logq"], args["item_ids"], args["valid"])
                    assert np.allclose(lse, want_lse, rtol=1e-12, atol=1e-12), (seed, use_q, use_ids, use_valid)
                    rows = valid[:b] if use_valid else np.ones(b, dtype=bool)
                    assert np.allclose(loss[rows], want_ce[rows], rtol=1e-12, atol=1e-12)
                    assert (loss[~rows] == 0).all()
                    assert abs(mean - want_ce[rows].mean()) <= 1e-12 * max(1.0, abs(mean))


def check_inbatch_closed_forms(o):
    """Two columns: the softmax cross-entropy is the logistic loss
    log(1 + exp(-margin)). Equal logits: the loss is log of the number of
    columns in the row's denominator, counted from the masks."""
    d = 16
    U = np.zeros((2, d), dtype=np.float32)
    V = np.zeros((2, d), dtype=np.float32)
    U[0, 0], U[1, 1] = 1.0, 2.0
    V[0, 0], V[1, 1], V[1, 0] = 2.0, 1.0, 0.5
    logq = np.array([math.log(0.25), math.log(0.5)])
    _, loss, _ = o.inbatch_softmax(U, V, 0.5, logq=logq)
    # row 0: logits 2/0.5 - log 0.25 and 0.5/0.5 - log 0.5; row 1: 0 - log 0.25 and 2/0.5 - log 0.5
    m0 = (4.0 - math.log(0.25)) - (1.0 - math.log(0.5))
    m1 = (4.0 - math.log(0.5)) - (0.0 - math.log(0.25))
    assert abs(loss[0] - math.log1p(math.exp(-m0))) <= 1e-14, loss
    assert abs(loss[1] - math.log1p(math.exp(-m1))) <= 1e-14, loss
    # equal logits (zero users): loss_i = log |D_i|
    b, nc = 10, 14
    _, _, _, ids, valid = _random_batch(5, b, nc, d)
    Uz = np.zeros((b, d), dtype=np.float32)
    Vr = np.ones((nc, d), dtype=np.float32)
    lse, loss, mean = o.inbatch_softmax(Uz, Vr, 1.0, item_ids=ids, valid=valid)
    for i in range(b):
        count = sum(1 for j in range(nc) if valid[j] and (j == i or ids[j] != ids[i]))
        assert abs(lse[i] - math.log(count)) <= 1e-14, (i, lse[i], count)
        assert loss[i] == (lse[i] if valid[i] else 0.0)
    # no valid row: the mean is 0
    _, loss, mean = o.inbatch_softmax(Uz, Vr, 1.0, valid=np.zeros(nc, dtype=bool))
    assert mean == 0.0 and (loss == 0).all()


def check_inbatch_invariants(o):
    """A constant added to every log q moves lse by minus that constant and
    leaves the loss alone (the correction applies to every column, the
    positive included); permuting the batch permutes the outputs; masking an
    accidental hit equals dropping that column for the row; users scaled by 2
    with tau scaled by 2 change nothing."""
    b, nc, d = 14, 20, 32
    U, V, logq, ids, valid = _random_batch(9, b, nc, d)
    lse, loss, mean = o.inbatch_softmax(U, V, 0.1, logq=logq, item_ids=ids, valid=valid)
    lse2, loss2, mean2 = o.inbatch_softmax(U, V, 0.1, logq=logq + 3.0, item_ids=ids, valid=valid)
    assert np.allclose(lse2, lse - 3.0, rtol=0, atol=1e-12)
    assert np.allclose(loss2, loss, rtol=0, atol=1e-12) and abs(mean2 - mean) <= 1e-12
    # permutation of rows (with their columns) and of the shared negatives
    rng = np.random.default_rng(4)
    pr = rng.permutation(b)
    pg = b + rng.permutation(nc - b)
    cols = np.concatenate([pr, pg])
    lse3, loss3, mean3 = o.inbatch_softmax(U[pr], V[cols], 0.1, logq=logq[cols], item_ids=ids[cols],
                                           valid=valid[cols])
    assert np.allclose(lse3, lse[pr], rtol=1e-13, atol=1e-13)
    assert np.allclose(loss3, loss[pr], rtol=1e-13, atol=1e-13) and abs(mean3 - mean) <= 1e-12
    # row 3 shares its item with row 7: its loss equals the loss with column 7 dropped and no id mask
    assert ids[3] == ids[7] and valid[3] and valid[7]
    drop7 = valid.copy()
    drop7[7] = False
    lse4, loss4, _ = o.inbatch_softmax(U, V, 0.1, logq=logq, valid=drop7)
    assert abs(loss4[3] - loss[3]) <= 1e-12 and abs(lse4[3] - lse[3]) <= 1e-12
    # the shared item does not mask the positive itself: row 0's item is also held by rows 5 and b-1
    assert np.isfinite(loss[0]) and loss[0] > 0
    # power-of-two scaling of users and tau
    lse5, loss5, _ = o.inbatch_softmax((U * 2).astype(np.float32), V, 0.2, logq=logq, item_ids=ids, valid=valid)
    assert np.array_equal(lse5, lse) and np.array_equal(loss5, loss)


ALL_CHECKS = [
    check_h8_logq_worked,
    check_inbatch_library,
    check_inbatch_closed_forms,
    check_inbatch_invariants,
    check_h5_quantize,
    check_h6_quantize_ties,
    check_h7_int8_score,
    check_quantize_invariants,
    check_int8_topk_invariants,
    check_bf16_rounding,
    check_bf16_inputs,
    check_h1_normalize,
    check_normalize_invariants,
    check_h2_topk,
    check_h3_fused,
    check_exact_rational,
    check_invariants,
    check_ties,
    check_scores_for,
]
