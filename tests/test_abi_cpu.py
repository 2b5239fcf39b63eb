"""The C-ABI library on a machine without a GPU: it loads, exports every
function ``include/tt.h`` declares, validates arguments on the host before
any device call, and plans its scans. No compute call is made here."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tt.h")

tt = pytest.importorskip("exact_inner_product_b200")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TT_API\s+[\w\s\*]+?\b(tt_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("tt_normalize_candidates", "tt_score_topk", "tt_free"):
        assert required in names
    assert len(names) >= 10


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tt.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in tt.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", tt.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tt_\w+)", out))
    assert set(declared_functions()) <= exported
    assert set(tt.EXPORTED) <= exported


def test_status_strings_and_version():
    assert tt.tt_version().startswith("tt ")
    for st, name in ((0, "TT_OK"), (1, "TT_ERR_INVALID_ARG"), (2, "TT_ERR_UNSUPPORTED"),
                     (5, "TT_ERR_TIMEOUT")):
        assert tt._lib.tt_status_string(st).decode() == name


def _empty_index(d=64, dtype=tt.TT_BF16):
    h = ctypes.c_void_p()
    st = tt._lib.tt_index_wrap(None, dtype, 0, d, None, ctypes.byref(h))
    assert st == tt.TT_OK
    return h


def test_host_validation_rejects_before_any_device_call():
    lib = tt._lib
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    h = ctypes.c_void_p()
    # tt_normalize_candidates
    assert lib.tt_normalize_candidates(fake, 0, -1, 64, fake, 1, 0, None, None) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_normalize_candidates(fake, 0, 10, 15, fake, 1, 0, None, None) == tt.TT_ERR_UNSUPPORTED
    assert lib.tt_normalize_candidates(fake, 0, 10, 1024, fake, 1, 0, None, None) == tt.TT_ERR_UNSUPPORTED
    assert lib.tt_normalize_candidates(fake, 0, 10, 0, fake, 1, 0, None, None) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_normalize_candidates(fake, 7, 10, 64, fake, 1, 0, None, None) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_normalize_candidates(fake, 0, 10, 64, fake, 1, 9, None, None) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_normalize_candidates(None, 0, 10, 64, fake, 1, 0, None, None) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_normalize_candidates(ctypes.c_void_p(0x10004), 0, 10, 64, fake, 1, 0, None,
                                       None) == tt.TT_ERR_INVALID_ARG  # misaligned
    assert lib.tt_normalize_candidates(fake, 0, 1 << 31, 64, fake, 1, 0, None, None) == tt.TT_ERR_UNSUPPORTED
    # n = 0 is a valid no-op, and may produce a handle
    assert lib.tt_normalize_candidates(None, 0, 0, 64, None, 1, 0, None, ctypes.byref(h)) == tt.TT_OK
    lib.tt_free(h)
    # tt_index_wrap
    assert lib.tt_index_wrap(fake, 1, 10, 64, None, None) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_index_wrap(None, 1, 10, 64, None, ctypes.byref(h)) == tt.TT_ERR_INVALID_ARG
    # tt_score_topk on an empty handle: every bad argument is caught on the host
    ix = _empty_index()
    ids = ctypes.c_void_p(0x20000)
    sc = ctypes.c_void_p(0x30000)
    call = lambda **kw: lib.tt_score_topk(kw.get("ix", ix), kw.get("q", fake), kw.get("qdt", 1), kw.get("b", 4),
                                          kw.get("excl", None), kw.get("tau", 1.0), kw.get("k", 10),
                                          kw.get("ids", ids), kw.get("sc", sc), None)
    assert call(ix=None) == tt.TT_ERR_INVALID_ARG
    assert call(k=0) == tt.TT_ERR_INVALID_ARG
    assert call(k=-3) == tt.TT_ERR_INVALID_ARG
    assert call(k=4096) == tt.TT_ERR_UNSUPPORTED
    assert call(tau=0.0) == tt.TT_ERR_INVALID_ARG
    assert call(tau=-1.0) == tt.TT_ERR_INVALID_ARG
    assert call(tau=float("nan")) == tt.TT_ERR_INVALID_ARG
    assert call(tau=float("inf")) == tt.TT_ERR_INVALID_ARG
    assert call(b=-1) == tt.TT_ERR_INVALID_ARG
    assert call(qdt=5) == tt.TT_ERR_INVALID_ARG
    assert call(q=None) == tt.TT_ERR_INVALID_ARG
    assert call(ids=None) == tt.TT_ERR_INVALID_ARG
    assert call(q=ctypes.c_void_p(0x10008)) == tt.TT_ERR_INVALID_ARG  # queries must be 16-byte aligned
    assert call(sc=ctypes.c_void_p(0x30002)) == tt.TT_ERR_INVALID_ARG
    assert call(excl=ctypes.c_void_p(0x40001)) == tt.TT_ERR_INVALID_ARG
    # b = 0: nothing to do
    assert call(b=0) == tt.TT_OK
    lib.tt_free(ix)
    lib.tt_free(None)  # NULL-safe
    # tensor-core path requested for an fp32 corpus: unsupported
    ixf = _empty_index(dtype=tt.TT_F32)
    opt = tt.tt_options(2, 0, 0, 0)
    assert lib.tt_score_topk_ex(ixf, fake, 0, 4, None, 1.0, 10, ids, sc, None, ctypes.byref(opt)) \
        == tt.TT_ERR_UNSUPPORTED
    opt3 = tt.tt_options(3, 0, 0, 0)
    assert lib.tt_score_topk_ex(ixf, fake, 0, 4, None, 1.0, 10, ids, sc, None, ctypes.byref(opt3)) \
        == tt.TT_ERR_UNSUPPORTED
    bad = tt.tt_options(4, 0, 0, 0)
    assert lib.tt_score_topk_ex(ixf, fake, 0, 4, None, 1.0, 10, ids, sc, None, ctypes.byref(bad)) \
        == tt.TT_ERR_INVALID_ARG
    lib.tt_free(ixf)
    # an fp32 corpus wider than 256 is outside the streaming scorer
    ixw = _empty_index(d=512, dtype=tt.TT_F32)
    assert call(ix=ixw) == tt.TT_ERR_UNSUPPORTED
    lib.tt_free(ixw)


def test_merge_validation_before_device_calls():
    lib = tt._lib
    fake = ctypes.c_void_p(0x10000)
    offs = (ctypes.c_int64 * 3)(0, 100, 200)
    call = lambda **kw: lib.tt_merge_topk(kw.get("ids", fake), kw.get("sc", fake), kw.get("parts", 3),
                                          kw.get("b", 4), kw.get("k_in", 10), kw.get("offs", offs),
                                          kw.get("k_out", 10), fake, fake, None)
    assert call(parts=0) == tt.TT_ERR_INVALID_ARG
    assert call(parts=65) == tt.TT_ERR_UNSUPPORTED
    assert call(k_in=4096, k_out=10) == tt.TT_ERR_UNSUPPORTED
    assert call(k_out=11) == tt.TT_ERR_INVALID_ARG  # k_out > k_in
    assert call(k_out=0) == tt.TT_ERR_INVALID_ARG
    assert call(b=-1) == tt.TT_ERR_INVALID_ARG
    assert call(offs=None) == tt.TT_ERR_INVALID_ARG
    assert call(offs=(ctypes.c_int64 * 3)(0, -5, 10)) == tt.TT_ERR_INVALID_ARG
    assert call(offs=(ctypes.c_int64 * 3)(0, 1 << 31, 10)) == tt.TT_ERR_INVALID_ARG
    assert call(ids=ctypes.c_void_p(0x10002)) == tt.TT_ERR_INVALID_ARG  # misaligned
    assert call(b=0) == tt.TT_OK


def test_set_calls_validate_before_device_calls():
    lib = tt._lib
    fake = ctypes.c_void_p(0x10000)
    ix = _empty_index()
    rng = (ctypes.c_int64 * 2)(0, 0)
    call = lambda **kw: lib.tt_score_topk_ranges(kw.get("ix", ix), fake, 1, kw.get("b", 0), None, 1.0,
                                                 kw.get("k", 5), kw.get("nr", 1), kw.get("rng", rng), fake,
                                                 fake, None)
    assert call() == tt.TT_OK  # b = 0: nothing to do
    assert call(ix=None) == tt.TT_ERR_INVALID_ARG
    assert call(nr=0) == tt.TT_ERR_INVALID_ARG
    assert call(nr=65) == tt.TT_ERR_UNSUPPORTED
    assert call(k=0) == tt.TT_ERR_INVALID_ARG
    assert call(k=4096) == tt.TT_ERR_UNSUPPORTED
    assert call(rng=None) == tt.TT_ERR_INVALID_ARG
    assert call(rng=(ctypes.c_int64 * 2)(0, 1)) == tt.TT_ERR_INVALID_ARG  # end past n = 0
    types_call = lambda st, n=1: lib.tt_score_topk_types(ix, fake, 1, 0, None, 1.0, 5, None, n, st, fake, fake,
                                                         None)
    assert types_call((ctypes.c_int32 * 1)(3)) == tt.TT_OK
    assert types_call(None) == tt.TT_ERR_INVALID_ARG
    assert types_call((ctypes.c_int32 * 1)(256)) == tt.TT_ERR_INVALID_ARG
    assert types_call((ctypes.c_int32 * 1)(3), n=0) == tt.TT_ERR_INVALID_ARG
    # too many (set, query) lists: refused before any device call
    many = lib.tt_score_topk_types(ix, fake, 1, 1 << 20, None, 1.0, 5, None, 32, (ctypes.c_int32 * 32)(*range(32)),
                                   fake, fake, None)
    assert many == tt.TT_ERR_UNSUPPORTED
    lib.tt_free(ix)


def test_softmax_validation_before_device_calls():
    lib = tt._lib
    fake = ctypes.c_void_p(0x10000)
    size = ctypes.c_size_t(0)
    assert lib.tt_inbatch_softmax_workspace(100, 300, 64, 1, ctypes.byref(size)) == tt.TT_OK
    need = size.value
    assert need > 300 * 8  # at least the per-column data
    assert lib.tt_inbatch_softmax_workspace(100, 300, 64, 0, ctypes.byref(size)) == tt.TT_OK
    assert size.value < need  # no hash table without item ids
    assert lib.tt_inbatch_softmax_workspace(300, 100, 64, 0, ctypes.byref(size)) == tt.TT_ERR_INVALID_ARG
    assert lib.tt_inbatch_softmax_workspace(10, 10, 24, 0, ctypes.byref(size)) == tt.TT_ERR_UNSUPPORTED
    assert lib.tt_inbatch_softmax_workspace(10, 10, 64, 0, None) == tt.TT_ERR_INVALID_ARG

    def call(**kw):
        return lib.tt_inbatch_softmax(fake, fake, kw.get("dt", tt.TT_BF16), kw.get("b", 100), kw.get("nc", 300),
                                      kw.get("d", 64), kw.get("tau", 0.05), None, kw.get("ids", fake), None, fake,
                                      fake, kw.get("mean", fake), kw.get("ws", fake), kw.get("wsb", 1), None)
    assert call(dt=tt.TT_F32) == tt.TT_ERR_UNSUPPORTED
    assert call(dt=9) == tt.TT_ERR_INVALID_ARG
    assert call(b=400) == tt.TT_ERR_INVALID_ARG  # nc < b
    assert call(b=-1) == tt.TT_ERR_INVALID_ARG
    assert call(d=40) == tt.TT_ERR_UNSUPPORTED
    assert call(d=48) == tt.TT_ERR_UNSUPPORTED  # narrower than one 64-element box
    assert call(d=1024) == tt.TT_ERR_UNSUPPORTED
    assert call(tau=0.0) == tt.TT_ERR_INVALID_ARG
    assert call(tau=float("inf")) == tt.TT_ERR_INVALID_ARG
    assert call(mean=None) == tt.TT_ERR_INVALID_ARG
    assert call(ws=ctypes.c_void_p(0x10010)) == tt.TT_ERR_INVALID_ARG  # workspace not 256-byte aligned
    assert call(wsb=need - 1) == tt.TT_ERR_INVALID_ARG  # workspace too small
    assert call(ids=ctypes.c_void_p(0x10004)) == tt.TT_ERR_INVALID_ARG  # misaligned ids
    assert lib.tt_inbatch_softmax_check(None, None) == tt.TT_ERR_INVALID_ARG


def test_plan_levels():
    # the deepest level holds at most `cap` rows; strides are powers of 61
    for n, k in ((400, 10), (10 ** 6, 100), (10 ** 7, 500), (5 * 10 ** 7, 1000), (2 * 10 ** 7, 256),
                 (2 ** 31 - 1, 2048), (1, 1), (0, 7)):
        p = tt.tt_plan(n, k)
        assert p["rows"][-1] <= 4096 or p["levels"] == 4
        assert p["rows"][0] == n
        for i, (r, s) in enumerate(zip(p["rows"], p["strides"])):
            assert s == 61 ** i
            assert r == (n + s - 1) // s
        # expected survivors at each finer level ~ rank * 61, comfortably above
        # the rank needed there and within the buffer
        for i in range(1, p["levels"]):
            need = p["ranks"][i - 1]
            assert p["ranks"][i] * 61 >= 3 * need
            assert p["ranks"][i] * 61 <= p["cap"] // 2
    assert tt.tt_plan(400, 10)["levels"] == 1
    assert tt.tt_plan(10 ** 6, 100) == {"levels": 3, "rows": [10 ** 6, 16394, 269], "strides": [1, 61, 3721],
                                        "ranks": [100, 32, 10], "cap": 16384}
    assert tt.tt_plan(5 * 10 ** 7, 1000)["ranks"] == [1000, 50, 10, 10]
    assert tt.tt_plan(4096, 10)["levels"] == 1 and tt.tt_plan(4097, 10)["levels"] == 2
    assert tt.tt_plan(10 ** 6, 100, force_levels=1)["levels"] == 1
    assert tt.tt_plan(10 ** 6, 100, force_levels=3)["levels"] == 3
    assert tt.tt_plan(10 ** 6, 100, rank_scale_pct=50)["ranks"] == [100, 16, 5]
    with pytest.raises(tt.TTError):
        tt.tt_plan(10, 0)
    with pytest.raises(tt.TTError):
        tt.tt_plan(10, 200, cap=256)  # cap must hold 2k keys
    with pytest.raises(tt.TTError):
        tt.tt_plan(10, 10, cap=1000)  # not a power of two


def test_package_fails_loudly_without_the_library(tmp_path):
    """Without libtt.so the package refuses to import (no CPU fallback)."""
    pkg = tmp_path / "exact_inner_product_b200"
    pkg.mkdir()
    src = open(os.path.join(ROOT, "exact_inner_product_b200", "__init__.py")).read()
    (pkg / "__init__.py").write_text(src)
    r = subprocess.run([sys.executable, "-c", "import exact_inner_product_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "exact_inner_product_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "oracle.c" not in text and "liboracle" not in text, f
