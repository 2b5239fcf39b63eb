"""fp64 CPU oracle for exact maximum-inner-product search (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It wraps ``oracle.c`` (plain C, fp64)
through ctypes; nothing here touches the CUDA library and nothing in the CUDA
library touches this.

Arrays are numpy. bf16 data travels as ``uint16`` bit patterns.

What each function computes and which passage it follows is stated in
``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile ``oracle.c`` (or another source) into a shared library (gcc, OpenMP, strict IEEE)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
               "-fPIC", "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle takes float32 or bf16-as-uint16 arrays, got {a.dtype}")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c2(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.ndim != 2:
        raise ValueError("expected a 2-D [rows, d] array")
    return a


class OracleLib:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        lib.oracle_bf16_from_double.restype = ctypes.c_uint16
        lib.oracle_row_norms.argtypes = [vp, i32, i64, i32, vp]
        lib.oracle_row_norms.restype = None
        lib.oracle_normalize.argtypes = [vp, i32, i64, i32, vp, i32]
        lib.oracle_normalize.restype = None
        lib.oracle_topk.argtypes = [vp, i32, i64, vp, i32, i64, i32, vp, vp, ctypes.c_double, i64,
                                    vp, vp]
        lib.oracle_topk.restype = ctypes.c_int
        lib.oracle_scores.argtypes = [vp, i32, i64, vp, i32, i32, vp, ctypes.c_double, vp, i64, vp]
        lib.oracle_scores.restype = None
        lib.oracle_quantize_rows.argtypes = [vp, i32, i64, i32, i32, vp, vp]
        lib.oracle_quantize_rows.restype = None
        lib.oracle_topk_q8.argtypes = [vp, vp, i64, vp, vp, i64, i32, vp, ctypes.c_double, i64, vp, vp]
        lib.oracle_topk_q8.restype = ctypes.c_int
        lib.oracle_scores_q8.argtypes = [vp, vp, i64, vp, vp, i32, ctypes.c_double, vp, i64, vp]
        lib.oracle_scores_q8.restype = None
        lib.oracle_inbatch_softmax.argtypes = [vp, i32, i64, vp, i32, i64, i32, vp, vp, vp, ctypes.c_double,
                                               vp, vp, vp]
        lib.oracle_inbatch_softmax.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [i32]
        lib.oracle_set_threads.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def bf16_from_double(self, x: float) -> int:
        """Bit pattern of x rounded once to bf16 (nearest, ties to even)."""
        return int(self.lib.oracle_bf16_from_double(float(x)))

    def row_norms(self, rows: np.ndarray) -> np.ndarray:
        """fp64 ``sqrt(max(sum v^2, 1e-12))`` per row."""
        rows = _c2(rows)
        out = np.empty(rows.shape[0], dtype=np.float64)
        self.lib.oracle_row_norms(_ptr(rows), _dtype_code(rows), rows.shape[0], rows.shape[1],
                                  _ptr(out))
        return out

    def normalize(self, rows: np.ndarray, out_dtype: str) -> np.ndarray:
        """Rows divided by their norm in fp64, rounded once to ``out_dtype``
        (``"f32"`` -> float32, ``"bf16"`` -> uint16 bit patterns)."""
        rows = _c2(rows)
        if out_dtype == "f32":
            out = np.empty(rows.shape, dtype=np.float32)
        elif out_dtype == "bf16":
            out = np.empty(rows.shape, dtype=np.uint16)
        else:
            raise ValueError(out_dtype)
        self.lib.oracle_normalize(_ptr(rows), _dtype_code(rows), rows.shape[0], rows.shape[1],
                                  _ptr(out), _dtype_code(out))
        return out

    def topk(self, queries: np.ndarray, corpus: np.ndarray, k: int, tau: float = 1.0,
             norms: np.ndarray | None = None, exclude: np.ndarray | None = None):
        """Exact top-k by sorting every eligible score (fp64).

        Returns ``(ids int32 [b,k], scores float64 [b,k])``; padding is
        ``(-1, -inf)``. ``norms`` (fp64 [n]) divides each score by the row norm
        (corpus kept raw); ``exclude`` is the packed uint32 exclusion bitmask.
        """
        queries, corpus = _c2(queries), _c2(corpus)
        b, d = queries.shape
        n = corpus.shape[0]
        if corpus.shape[1] != d:
            raise ValueError("queries and corpus disagree on d")
        if norms is not None:
            norms = np.ascontiguousarray(norms, dtype=np.float64)
            assert norms.shape == (n,)
        if exclude is not None:
            exclude = np.ascontiguousarray(exclude).view(np.uint32)
            assert exclude.size >= (n + 31) // 32
        ids = np.empty((b, k), dtype=np.int32)
        scores = np.empty((b, k), dtype=np.float64)
        rc = self.lib.oracle_topk(_ptr(queries), _dtype_code(queries), b, _ptr(corpus),
                                  _dtype_code(corpus), n, d, _ptr(norms), _ptr(exclude), float(tau),
                                  int(k), _ptr(ids), _ptr(scores))
        if rc != 0:
            raise MemoryError("oracle_topk could not allocate its work buffer")
        return ids, scores

    def scores_for(self, queries: np.ndarray, qrow: int, corpus: np.ndarray, ids, tau: float = 1.0,
                   norms: np.ndarray | None = None) -> np.ndarray:
        """fp64 scores of the listed candidate ids for query ``qrow``."""
        queries, corpus = _c2(queries), _c2(corpus)
        ids = np.ascontiguousarray(ids, dtype=np.int64)
        if norms is not None:
            norms = np.ascontiguousarray(norms, dtype=np.float64)
        out = np.empty(ids.shape[0], dtype=np.float64)
        self.lib.oracle_scores(_ptr(queries), _dtype_code(queries), int(qrow), _ptr(corpus),
                               _dtype_code(corpus), queries.shape[1], _ptr(norms), float(tau),
                               _ptr(ids), ids.shape[0], _ptr(out))
        return out

    def quantize(self, rows: np.ndarray, normalise: bool):
        """Symmetric per-row int8 codes in fp32 arithmetic: ``(codes int8
        [n,d], scales float32 [n])``; with ``normalise`` the row is first
        L2-normalised (fp64 norm, value held in fp32)."""
        rows = _c2(rows)
        codes = np.empty(rows.shape, dtype=np.int8)
        scales = np.empty(rows.shape[0], dtype=np.float32)
        self.lib.oracle_quantize_rows(_ptr(rows), _dtype_code(rows), rows.shape[0], rows.shape[1],
                                      1 if normalise else 0, _ptr(codes), _ptr(scales))
        return codes, scales

    def topk_q8(self, qcodes: np.ndarray, qscales: np.ndarray, vcodes: np.ndarray, vscales: np.ndarray,
                k: int, tau: float = 1.0, exclude: np.ndarray | None = None):
        """Exact top-k of (sum q8 v8) * qscale * vscale / tau (fp64, every score sorted)."""
        qcodes, vcodes = _c2(qcodes), _c2(vcodes)
        assert qcodes.dtype == np.int8 and vcodes.dtype == np.int8
        b, d = qcodes.shape
        n = vcodes.shape[0]
        qscales = np.ascontiguousarray(qscales, dtype=np.float32)
        vscales = np.ascontiguousarray(vscales, dtype=np.float32)
        if exclude is not None:
            exclude = np.ascontiguousarray(exclude).view(np.uint32)
        ids = np.empty((b, k), dtype=np.int32)
        scores = np.empty((b, k), dtype=np.float64)
        rc = self.lib.oracle_topk_q8(_ptr(qcodes), _ptr(qscales), b, _ptr(vcodes), _ptr(vscales), n, d,
                                     _ptr(exclude), float(tau), int(k), _ptr(ids), _ptr(scores))
        if rc != 0:
            raise MemoryError("oracle_topk_q8 could not allocate its work buffer")
        return ids, scores

    def scores_for_q8(self, qcodes, qscales, qrow, vcodes, vscales, ids, tau=1.0) -> np.ndarray:
        qcodes, vcodes = _c2(qcodes), _c2(vcodes)
        ids = np.ascontiguousarray(ids, dtype=np.int64)
        out = np.empty(ids.shape[0], dtype=np.float64)
        self.lib.oracle_scores_q8(_ptr(qcodes), _ptr(np.ascontiguousarray(qscales, dtype=np.float32)),
                                  int(qrow), _ptr(vcodes), _ptr(np.ascontiguousarray(vscales, dtype=np.float32)),
                                  qcodes.shape[1], float(tau), _ptr(ids), ids.shape[0], _ptr(out))
        return out

    def inbatch_softmax(self, users: np.ndarray, items: np.ndarray, tau: float = 1.0,
                        logq: np.ndarray | None = None, item_ids: np.ndarray | None = None,
                        valid: np.ndarray | None = None):
        """In-batch sampled softmax in fp64: row i's positive is candidate i,
        every other valid column not holding row i's item is a negative.

        ``users`` [b,d] and ``items`` [nc,d] (nc >= b) as float32 or bf16 bits;
        ``logq`` [nc] is subtracted from every logit of its column; ``item_ids``
        [nc] int64 marks accidental hits; ``valid`` [nc] bool drops columns and
        (for i < b) rows. Returns ``(lse [b], loss [b], mean)`` as float64.
        """
        users, items = _c2(users), _c2(items)
        b, d = users.shape
        nc = items.shape[0]
        if items.shape[1] != d or nc < b:
            raise ValueError("need items [nc, d] with nc >= b")
        if logq is not None:
            logq = np.ascontiguousarray(logq, dtype=np.float64)
            assert logq.shape == (nc,)
        if item_ids is not None:
            item_ids = np.ascontiguousarray(item_ids, dtype=np.int64)
            assert item_ids.shape == (nc,)
        if valid is not None:
            valid = np.ascontiguousarray(valid, dtype=bool).view(np.uint8)
            assert valid.shape == (nc,)
        lse = np.empty(b, dtype=np.float64)
        loss = np.empty(b, dtype=np.float64)
        mean = np.empty(1, dtype=np.float64)
        rc = self.lib.oracle_inbatch_softmax(_ptr(users), _dtype_code(users), b, _ptr(items),
                                             _dtype_code(items), nc, d, _ptr(logq), _ptr(item_ids),
                                             _ptr(valid), float(tau), _ptr(lse), _ptr(loss), _ptr(mean))
        if rc != 0:
            raise MemoryError("oracle_inbatch_softmax could not allocate its work buffer")
        return lse, loss, float(mean[0])

    def set_threads(self, n: int) -> None:
        self.lib.oracle_set_threads(int(n))

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())


_default = None


def default() -> OracleLib:
    """The oracle built from ``oracle.c`` next to this file."""
    global _default
    if _default is None:
        _default = OracleLib(build())
    return _default


def bf16_from_double(x):
    return default().bf16_from_double(x)


def row_norms(rows):
    return default().row_norms(rows)


def normalize(rows, out_dtype):
    return default().normalize(rows, out_dtype)


def topk(queries, corpus, k, tau=1.0, norms=None, exclude=None):
    return default().topk(queries, corpus, k, tau=tau, norms=norms, exclude=exclude)


def scores_for(queries, qrow, corpus, ids, tau=1.0, norms=None):
    return default().scores_for(queries, qrow, corpus, ids, tau=tau, norms=norms)


def quantize(rows, normalise):
    return default().quantize(rows, normalise)


def topk_q8(qcodes, qscales, vcodes, vscales, k, tau=1.0, exclude=None):
    return default().topk_q8(qcodes, qscales, vcodes, vscales, k, tau=tau, exclude=exclude)


def scores_for_q8(qcodes, qscales, qrow, vcodes, vscales, ids, tau=1.0):
    return default().scores_for_q8(qcodes, qscales, qrow, vcodes, vscales, ids, tau=tau)


def inbatch_softmax(users, items, tau=1.0, logq=None, item_ids=None, valid=None):
    return default().inbatch_softmax(users, items, tau=tau, logq=logq, item_ids=item_ids, valid=valid)


def set_threads(n):
    default().set_threads(n)


def max_threads():
    return default().max_threads()
