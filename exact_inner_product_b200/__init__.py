"""Exact top-k inner-product search on B200: Python binding of ``libtt.so``.

Thin ctypes layer over the C ABI declared in ``include/tt.h``: every function
here only marshals arguments (tensor pointers, sizes, the current CUDA stream)
and raises ``TTError`` on a non-OK status. All computation runs in the CUDA
kernels of the library. PyTorch supplies device memory and streams.

    import exact_inner_product_b200 as tt
    index = tt.tt_normalize_candidates(raw_corpus, torch.empty_like(raw_corpus, dtype=torch.bfloat16))
    ids, scores = tt.tt_score_topk(index, queries, k=100)

There is no fallback: if ``libtt.so`` has not been built, importing this
package raises ``ImportError``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtt.so")

TT_OK = 0
TT_ERR_INVALID_ARG = 1
TT_ERR_UNSUPPORTED = 2
TT_ERR_CUDA = 3
TT_ERR_NO_MEMORY = 4
TT_ERR_TIMEOUT = 5
TT_ERR_INTERNAL = 6

TT_F32 = 0
TT_BF16 = 1
TT_I8 = 2
TT_NORM_STORE = 0
TT_NORM_FUSED = 1
TT_MAX_D = 512
TT_MAX_K = 2048

KIND_NAMES = ("normalize", "cast", "stream", "tensor", "select", "aux", "softmax", "estimate")
TT_NUM_KINDS = len(KIND_NAMES)

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python exact_inner_product_b200/build.py` "
        "(there is no CPU fallback)")


class tt_options(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("rank_scale_pct", ctypes.c_int32),
                ("force_levels", ctypes.c_int32), ("cap", ctypes.c_int32), ("withhold_copy", ctypes.c_int32)]


class tt_stats(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("levels", ctypes.c_int32), ("rescans", ctypes.c_int32),
                ("launches", ctypes.c_int32), ("level_rows", ctypes.c_int64 * 4),
                ("level_stride", ctypes.c_int64 * 4), ("cap", ctypes.c_int32),
                ("sampled", ctypes.c_int32)]


_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("tt_normalize_candidates", ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _vp, ctypes.c_int, _i32, _vp,
                                               ctypes.POINTER(_vp)])
_sig("tt_index_wrap", ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _vp, ctypes.POINTER(_vp)])
_sig("tt_quantize_candidates", ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _vp, _vp, _vp, ctypes.POINTER(_vp)])
_sig("tt_score_topk", ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _vp, ctypes.c_float, _i32, _vp, _vp,
                                     _vp])
_sig("tt_score_topk_ex", ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _vp, ctypes.c_float, _i32, _vp,
                                        _vp, _vp, ctypes.POINTER(tt_options)])
_sig("tt_last_stats", ctypes.c_int, [_vp, ctypes.POINTER(tt_stats)])
_sig("tt_index_check", ctypes.c_int, [_vp, _vp])
_sig("tt_score_topk_host", ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _i32, ctypes.c_int, _vp, ctypes.c_float,
                                          _i32, _vp, _vp, _vp])
_sig("tt_plan", ctypes.c_int, [_i64, _i32, ctypes.POINTER(tt_options), ctypes.POINTER(_i32),
                               ctypes.POINTER(_i64), ctypes.POINTER(_i64), ctypes.POINTER(_i32),
                               ctypes.POINTER(_i32)])
_sig("tt_score_topk_noalloc", ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _vp, _vp, ctypes.c_int, _i32,
                                             _vp, ctypes.c_float, _i32, _vp, _vp, _vp])
_sig("tt_merge_topk", ctypes.c_int, [_vp, _vp, _i32, _i32, _i32, ctypes.POINTER(_i64), _i32, _vp, _vp, _vp])
_sig("tt_score_topk_ranges", ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _vp, ctypes.c_float, _i32, _i32,
                                            ctypes.POINTER(_i64), _vp, _vp, _vp])
_sig("tt_score_topk_types", ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _vp, ctypes.c_float, _i32, _vp, _i32,
                                           ctypes.POINTER(_i32), _vp, _vp, _vp])
_sig("tt_inbatch_softmax_workspace", ctypes.c_int, [_i32, _i32, _i32, _i32, ctypes.POINTER(ctypes.c_size_t)])
_sig("tt_inbatch_softmax", ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _i32, _i32, ctypes.c_float, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp])
_sig("tt_inbatch_softmax_check", ctypes.c_int, [_vp, _vp])
_sig("tt_free", None, [_vp])
_sig("tt_launch_count", _i64, [])
_sig("tt_profile_begin", ctypes.c_int, [])
_sig("tt_profile_end", ctypes.c_int, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)])
_sig("tt_profile_launches", ctypes.c_int, [ctypes.POINTER(_i32), ctypes.POINTER(ctypes.c_double), _i32,
                                           ctypes.POINTER(_i32)])
_sig("tt_status_string", ctypes.c_char_p, [ctypes.c_int])
_sig("tt_last_error", ctypes.c_char_p, [])
_sig("tt_version", ctypes.c_char_p, [])

EXPORTED = ("tt_normalize_candidates", "tt_quantize_candidates", "tt_index_wrap", "tt_score_topk", "tt_score_topk_ex",
            "tt_index_check", "tt_score_topk_host",
            "tt_score_topk_noalloc", "tt_merge_topk", "tt_score_topk_ranges", "tt_score_topk_types",
            "tt_inbatch_softmax_workspace", "tt_inbatch_softmax", "tt_inbatch_softmax_check",
            "tt_last_stats", "tt_plan", "tt_free", "tt_launch_count", "tt_profile_begin",
            "tt_profile_end", "tt_profile_launches", "tt_status_string", "tt_last_error", "tt_version")


class TTError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _lib.tt_status_string(status).decode()
        detail = _lib.tt_last_error().decode()
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))


def _check(status: int, where: str) -> None:
    if status != TT_OK:
        raise TTError(status, where)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TT_F32
    if t.dtype == torch.bfloat16:
        return TT_BF16
    if t.dtype == torch.int8:
        return TT_I8
    raise TypeError(f"tensors must be float32, bfloat16 or int8 (codes), got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _options(path=0, rank_scale_pct=0, force_levels=0, cap=0, withhold_copy=0):
    return tt_options(int(path), int(rank_scale_pct), int(force_levels), int(cap), int(withhold_copy))


class Index:
    """A prepared corpus (handle from the C library). Keeps the tensors it
    refers to alive; releases the handle (``tt_free``) when collected."""

    def __init__(self, handle: int, rows: torch.Tensor, inv_norm: torch.Tensor | None, n: int, d: int):
        self.handle = ctypes.c_void_p(handle)
        self.rows = rows
        self.inv_norm = inv_norm
        self.n = n
        self.d = d

    def free(self) -> None:
        if self.handle is not None and self.handle.value:
            _lib.tt_free(self.handle)
        self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def tt_normalize_candidates(x: torch.Tensor, out: torch.Tensor, mode: int = TT_NORM_STORE,
                            stream=None, make_index: bool = True) -> Index | None:
    """Row-wise L2 normalisation (``tt_normalize_candidates``).

    ``x``: [n, d] float32/bfloat16 on the GPU. ``mode=TT_NORM_STORE``: ``out``
    is [n, d] (float32 or bfloat16) and receives the normalised rows.
    ``mode=TT_NORM_FUSED``: ``out`` is [n] float32 and receives 1/norm; the
    index then scores the raw rows. Returns an ``Index`` (or None when
    ``make_index`` is False, e.g. for normalising queries)."""
    if x.dim() != 2 or not x.is_contiguous() or not out.is_contiguous():
        raise ValueError("x must be a contiguous [n, d] tensor and out contiguous")
    n, d = x.shape
    handle = ctypes.c_void_p()
    st = _lib.tt_normalize_candidates(_ptr(x), _dtype(x), n, d, _ptr(out),
                                      _dtype(out), int(mode), _stream(stream),
                                      ctypes.byref(handle) if make_index else None)
    _check(st, "tt_normalize_candidates")
    if not make_index:
        return None
    if mode == TT_NORM_STORE:
        return Index(handle.value, out, None, n, d)
    return Index(handle.value, x, out, n, d)


def tt_quantize_candidates(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, stream=None,
                           make_index: bool = True) -> Index | None:
    """L2-normalise each row and code it in int8 with one scale per row
    (``tt_quantize_candidates``). ``x``: [n, d] float32/bfloat16 on the GPU;
    ``codes``: [n, d] int8; ``scales``: [n] float32. Returns an int8 ``Index``
    (or None when ``make_index`` is False)."""
    if x.dim() != 2 or not x.is_contiguous() or not codes.is_contiguous() or not scales.is_contiguous():
        raise ValueError("x, codes and scales must be contiguous")
    if codes.dtype != torch.int8 or scales.dtype != torch.float32:
        raise TypeError("codes must be int8 and scales float32")
    n, d = x.shape
    handle = ctypes.c_void_p()
    _check(_lib.tt_quantize_candidates(_ptr(x), _dtype(x), n, d, _ptr(codes), _ptr(scales), _stream(stream),
                                       ctypes.byref(handle) if make_index else None), "tt_quantize_candidates")
    if not make_index:
        return None
    return Index(handle.value, codes, scales, n, d)


def tt_index_wrap(rows: torch.Tensor, inv_norm: torch.Tensor | None = None) -> Index:
    """Handle over an already prepared corpus (``tt_index_wrap``)."""
    if rows.dim() != 2 or not rows.is_contiguous():
        raise ValueError("rows must be a contiguous [n, d] tensor")
    n, d = rows.shape
    handle = ctypes.c_void_p()
    _check(_lib.tt_index_wrap(_ptr(rows), _dtype(rows), n, d, _ptr(inv_norm), ctypes.byref(handle)),
           "tt_index_wrap")
    return Index(handle.value, rows, inv_norm, n, d)


def tt_score_topk(index: Index, queries: torch.Tensor, k: int, tau: float = 1.0,
                  exclude: torch.Tensor | None = None, out_ids: torch.Tensor | None = None,
                  out_scores: torch.Tensor | None = None, stream=None, **options):
    """Exact top-k by inner product (``tt_score_topk`` / ``tt_score_topk_ex``).

    ``queries``: [b, d] float32/bfloat16 on the GPU. ``exclude``: packed
    exclusion bits, int32 tensor of ceil(n/32) words (bit j&31 of word j>>5).
    Returns ``(ids int32 [b,k], scores float32 [b,k])``, complete once the
    stream reaches the call's work (the call itself does not wait; see
    ``tt_index_check``). Keyword options (``path``, ``rank_scale_pct``,
    ``force_levels``, ``cap``, ``withhold_copy``) go to ``tt_score_topk_ex``."""
    if queries.dim() != 2 or not queries.is_contiguous():
        raise ValueError("queries must be a contiguous [b, d] tensor")
    b, d = queries.shape
    if d != index.d:
        raise ValueError(f"queries have d={d}, index has d={index.d}")
    dev = queries.device
    if out_ids is None:
        out_ids = torch.empty((b, k), dtype=torch.int32, device=dev)
    if out_scores is None:
        out_scores = torch.empty((b, k), dtype=torch.float32, device=dev)
    if exclude is not None and (exclude.dtype not in (torch.int32,) or not exclude.is_contiguous()):
        raise TypeError("exclude must be a contiguous int32 tensor of packed bits")
    if options:
        opt = _options(**options)
        st = _lib.tt_score_topk_ex(index.handle, _ptr(queries), _dtype(queries), b, _ptr(exclude),
                                   float(tau), int(k), _ptr(out_ids), _ptr(out_scores), _stream(stream),
                                   ctypes.byref(opt))
    else:
        st = _lib.tt_score_topk(index.handle, _ptr(queries), _dtype(queries), b, _ptr(exclude),
                                float(tau), int(k), _ptr(out_ids), _ptr(out_scores), _stream(stream))
    _check(st, "tt_score_topk")
    return out_ids, out_scores


def tt_score_topk_noalloc(rows: torch.Tensor, queries: torch.Tensor, k: int, tau: float = 1.0,
                          inv_norm: torch.Tensor | None = None, exclude: torch.Tensor | None = None,
                          out_ids: torch.Tensor | None = None, out_scores: torch.Tensor | None = None,
                          stream=None):
    """``tt_score_topk`` for callers that must not allocate device memory
    (``tt_score_topk_noalloc``): the library works in a fixed array reserved
    on each GPU, so this call makes no allocation of its own. ``rows`` is the
    prepared corpus (normalised rows, or raw rows with ``inv_norm``). Output
    tensors are allocated here only when not given; pass them in to keep the
    whole call allocation-free. At most about 255 queries per call."""
    if rows.dim() != 2 or queries.dim() != 2 or not rows.is_contiguous() or not queries.is_contiguous():
        raise ValueError("rows and queries must be contiguous 2-D tensors")
    n, d = rows.shape
    b = queries.shape[0]
    if queries.shape[1] != d:
        raise ValueError(f"queries have d={queries.shape[1]}, rows have d={d}")
    dev = queries.device
    if out_ids is None:
        out_ids = torch.empty((b, k), dtype=torch.int32, device=dev)
    if out_scores is None:
        out_scores = torch.empty((b, k), dtype=torch.float32, device=dev)
    for name, t, dt in (("out_ids", out_ids, torch.int32), ("out_scores", out_scores, torch.float32)):
        if t.dtype != dt or tuple(t.shape) != (b, k) or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"{name} must be a contiguous {dt} tensor of shape ({b}, {k}) on {dev}")
    if exclude is not None and (exclude.dtype != torch.int32 or not exclude.is_contiguous()
                                or exclude.numel() < (n + 31) // 32):
        raise TypeError("exclude must be a contiguous int32 tensor of ceil(n/32) packed words")
    if inv_norm is not None and (inv_norm.dtype != torch.float32 or not inv_norm.is_contiguous()
                                 or inv_norm.numel() != n):
        raise TypeError("inv_norm must be a contiguous float32 tensor of n elements")
    st = _lib.tt_score_topk_noalloc(_ptr(rows), _dtype(rows), n, d, _ptr(inv_norm), _ptr(queries),
                                    _dtype(queries), b, _ptr(exclude), float(tau), int(k), _ptr(out_ids),
                                    _ptr(out_scores), _stream(stream))
    _check(st, "tt_score_topk_noalloc")
    return out_ids, out_scores


def tt_index_check(index: Index, stream=None) -> None:
    """Wait for the work enqueued on ``stream`` and raise ``TTError``
    (TT_ERR_TIMEOUT) if a device-side wait of a search on this handle
    expired (``tt_index_check``)."""
    _check(_lib.tt_index_check(index.handle, _stream(stream)), "tt_index_check")


def tt_score_topk_host(index: Index, queries: torch.Tensor, k: int, tau: float = 1.0,
                       exclude: torch.Tensor | None = None, normalize: bool = True,
                       norm_dtype=torch.bfloat16, out_ids: torch.Tensor | None = None,
                       out_scores: torch.Tensor | None = None, stream=None):
    """The search from host to host (``tt_score_topk_host``): ``queries`` is
    a CPU [b, d] tensor (pinned memory copies faster), copied to the device,
    L2-normalised there into ``norm_dtype`` when ``normalize``, scored against
    the resident index; returns CPU ``(ids int32 [b, k], scores float32 [b, k])``
    once they are there. ``exclude`` stays a device tensor."""
    if queries.dim() != 2 or not queries.is_contiguous() or queries.is_cuda:
        raise ValueError("queries must be a contiguous [b, d] CPU tensor")
    b, d = queries.shape
    if d != index.d:
        raise ValueError(f"queries have d={d}, index has d={index.d}")
    if out_ids is None:
        out_ids = torch.empty((b, k), dtype=torch.int32, pin_memory=torch.cuda.is_available())
    if out_scores is None:
        out_scores = torch.empty((b, k), dtype=torch.float32, pin_memory=torch.cuda.is_available())
    for name, t, dt in (("out_ids", out_ids, torch.int32), ("out_scores", out_scores, torch.float32)):
        if t.dtype != dt or tuple(t.shape) != (b, k) or not t.is_contiguous() or t.is_cuda:
            raise ValueError(f"{name} must be a contiguous CPU {dt} tensor of shape ({b}, {k})")
    if exclude is not None and (exclude.dtype != torch.int32 or not exclude.is_contiguous() or not exclude.is_cuda):
        raise TypeError("exclude must be a contiguous int32 CUDA tensor of packed bits")
    norm_dt = TT_F32 if norm_dtype == torch.float32 else TT_BF16
    _check(_lib.tt_score_topk_host(index.handle, _ptr(queries), _dtype(queries), b, 1 if normalize else 0,
                                   norm_dt, _ptr(exclude), float(tau), int(k), _ptr(out_ids), _ptr(out_scores),
                                   _stream(stream)), "tt_score_topk_host")
    return out_ids, out_scores


def tt_merge_topk(ids: torch.Tensor, scores: torch.Tensor, id_offsets, k_out: int,
                  out_ids: torch.Tensor | None = None, out_scores: torch.Tensor | None = None, stream=None):
    """Top-k_out of the union of per-shard lists (``tt_merge_topk``).

    ``ids`` int32 / ``scores`` float32, contiguous [parts, b, k_in] on the GPU
    (each part: one shard's tt_score_topk output, local ids); ``id_offsets``:
    the global id of each shard's row 0. Returns ``(ids int32 [b, k_out],
    scores float32 [b, k_out])`` with global ids."""
    if ids.dim() != 3 or ids.shape != scores.shape or not ids.is_contiguous() or not scores.is_contiguous():
        raise ValueError("ids and scores must be contiguous [parts, b, k_in] tensors of one shape")
    if ids.dtype != torch.int32 or scores.dtype != torch.float32:
        raise TypeError("ids must be int32 and scores float32")
    parts, b, k_in = ids.shape
    offs = (_i64 * max(1, parts))(*[int(o) for o in id_offsets])
    if len(id_offsets) != parts:
        raise ValueError("one offset per part")
    dev = ids.device
    if out_ids is None:
        out_ids = torch.empty((b, k_out), dtype=torch.int32, device=dev)
    if out_scores is None:
        out_scores = torch.empty((b, k_out), dtype=torch.float32, device=dev)
    _check(_lib.tt_merge_topk(_ptr(ids), _ptr(scores), parts, b, k_in, offs, int(k_out), _ptr(out_ids),
                              _ptr(out_scores), _stream(stream)), "tt_merge_topk")
    return out_ids, out_scores


def tt_inbatch_softmax_workspace(b: int, nc: int, d: int, with_item_ids: bool) -> int:
    """Bytes of device workspace ``tt_inbatch_softmax`` needs for these sizes."""
    out = ctypes.c_size_t(0)
    _check(_lib.tt_inbatch_softmax_workspace(int(b), int(nc), int(d), 1 if with_item_ids else 0,
                                             ctypes.byref(out)), "tt_inbatch_softmax_workspace")
    return int(out.value)


def tt_inbatch_softmax(users: torch.Tensor, items: torch.Tensor, tau: float = 1.0,
                       logq: torch.Tensor | None = None, item_ids: torch.Tensor | None = None,
                       valid: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                       out: tuple | None = None, stream=None, check: bool = True):
    """In-batch sampled softmax loss (``tt_inbatch_softmax``): row i of
    ``users`` [b, d] has candidate row i of ``items`` [nc, d] (bf16, nc >= b)
    as its positive. ``logq`` float32 [nc] is subtracted from every logit of
    its column, ``item_ids`` int64 [nc] masks accidental hits, ``valid`` bool
    or uint8 [nc] drops padding. Returns ``(lse [b], loss [b], mean [])`` as
    float32 tensors on the device. ``workspace`` (uint8, at least
    ``tt_inbatch_softmax_workspace`` bytes) and ``out`` (lse, loss, mean) may
    be passed to avoid allocations; ``check`` waits for the result and raises
    on a device-side timeout."""
    if users.dim() != 2 or items.dim() != 2 or not users.is_contiguous() or not items.is_contiguous():
        raise ValueError("users and items must be contiguous [b, d] and [nc, d] tensors")
    if users.shape[1] != items.shape[1]:
        raise ValueError("users and items disagree on d")
    b, d = users.shape
    nc = items.shape[0]
    for name, t, dt in (("logq", logq, torch.float32), ("item_ids", item_ids, torch.int64)):
        if t is not None and (t.dtype != dt or not t.is_contiguous() or t.numel() != nc):
            raise TypeError(f"{name} must be a contiguous {dt} tensor of nc elements")
    if valid is not None:
        if valid.dtype == torch.bool:
            valid = valid.view(torch.uint8)
        if valid.dtype != torch.uint8 or not valid.is_contiguous() or valid.numel() != nc:
            raise TypeError("valid must be a contiguous bool or uint8 tensor of nc elements")
    need = tt_inbatch_softmax_workspace(b, nc, d, item_ids is not None)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=users.device)
    if out is None:
        out = (torch.empty(b, dtype=torch.float32, device=users.device),
               torch.empty(b, dtype=torch.float32, device=users.device),
               torch.empty((), dtype=torch.float32, device=users.device))
    lse, loss, mean = out
    _check(_lib.tt_inbatch_softmax(_ptr(users), _ptr(items), _dtype(users), b, nc, d, float(tau), _ptr(logq), _ptr(item_ids),
                                   _ptr(valid), _ptr(lse), _ptr(loss), _ptr(mean), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "tt_inbatch_softmax")
    if check:
        _check(_lib.tt_inbatch_softmax_check(_ptr(workspace), _stream(stream)), "tt_inbatch_softmax")
    return lse, loss, mean


def _check_queries(index: Index, queries: torch.Tensor, exclude):
    if queries.dim() != 2 or not queries.is_contiguous():
        raise ValueError("queries must be a contiguous [b, d] tensor")
    if queries.shape[1] != index.d:
        raise ValueError(f"queries have d={queries.shape[1]}, index has d={index.d}")
    if exclude is not None and (exclude.dtype != torch.int32 or not exclude.is_contiguous()):
        raise TypeError("exclude must be a contiguous int32 tensor of packed bits")


def tt_score_topk_ranges(index: Index, queries: torch.Tensor, k: int, ranges, tau: float = 1.0,
                         exclude: torch.Tensor | None = None, stream=None):
    """One top-k per candidate range [start, end) (``tt_score_topk_ranges``).
    Returns ``(ids int32 [R, b, k], scores float32 [R, b, k])`` with corpus ids."""
    _check_queries(index, queries, exclude)
    b = queries.shape[0]
    R = len(ranges)
    flat = (_i64 * (2 * max(1, R)))(*[int(v) for rng in ranges for v in rng])
    out_ids = torch.empty((R, b, k), dtype=torch.int32, device=queries.device)
    out_scores = torch.empty((R, b, k), dtype=torch.float32, device=queries.device)
    _check(_lib.tt_score_topk_ranges(index.handle, _ptr(queries), _dtype(queries), b, _ptr(exclude), float(tau),
                                     int(k), R, flat, _ptr(out_ids), _ptr(out_scores), _stream(stream)),
           "tt_score_topk_ranges")
    return out_ids, out_scores


def tt_score_topk_types(index: Index, queries: torch.Tensor, k: int, types: torch.Tensor, set_types,
                        tau: float = 1.0, exclude: torch.Tensor | None = None, stream=None):
    """One top-k per candidate type (``tt_score_topk_types``): ``types`` is a
    uint8 [n] tensor on the GPU, ``set_types`` the types to report. Returns
    ``(ids int32 [T, b, k], scores float32 [T, b, k])``."""
    _check_queries(index, queries, exclude)
    if types.dtype != torch.uint8 or not types.is_contiguous():
        raise TypeError("types must be a contiguous uint8 tensor")
    b = queries.shape[0]
    T = len(set_types)
    st_arr = (_i32 * max(1, T))(*[int(t) for t in set_types])
    out_ids = torch.empty((T, b, k), dtype=torch.int32, device=queries.device)
    out_scores = torch.empty((T, b, k), dtype=torch.float32, device=queries.device)
    _check(_lib.tt_score_topk_types(index.handle, _ptr(queries), _dtype(queries), b, _ptr(exclude), float(tau),
                                    int(k), _ptr(types), T, st_arr, _ptr(out_ids), _ptr(out_scores),
                                    _stream(stream)), "tt_score_topk_types")
    return out_ids, out_scores


def tt_free(index: Index) -> None:
    index.free()


def tt_last_stats(index: Index) -> dict:
    """What the last search on the handle did; ``rescans`` (lists the exact
    fallback recomputed) is -1 until that search's work has completed."""
    s = tt_stats()
    _check(_lib.tt_last_stats(index.handle, ctypes.byref(s)), "tt_last_stats")
    return {"path": s.path, "levels": s.levels, "rescans": s.rescans, "launches": s.launches,
            "level_rows": list(s.level_rows[:s.levels]), "level_stride": list(s.level_stride[:s.levels]),
            "cap": s.cap, "sampled": bool(s.sampled)}


def tt_plan(n: int, k: int, **options) -> dict:
    levels, cap = _i32(), _i32()
    rows, strides, ranks = (_i64 * 4)(), (_i64 * 4)(), (_i32 * 4)()
    opt = _options(**options)
    _check(_lib.tt_plan(int(n), int(k), ctypes.byref(opt), ctypes.byref(levels), rows, strides, ranks,
                        ctypes.byref(cap)), "tt_plan")
    L = levels.value
    return {"levels": L, "rows": list(rows[:L]), "strides": list(strides[:L]), "ranks": list(ranks[:L]),
            "cap": cap.value}


def tt_launch_count() -> int:
    return int(_lib.tt_launch_count())


def tt_profile_begin() -> None:
    _check(_lib.tt_profile_begin(), "tt_profile_begin")


def tt_profile_end() -> dict:
    ms = (ctypes.c_double * TT_NUM_KINDS)()
    cnt = (_i64 * TT_NUM_KINDS)()
    _check(_lib.tt_profile_end(ms, cnt), "tt_profile_end")
    return {name: {"ms": ms[i], "launches": cnt[i]} for i, name in enumerate(KIND_NAMES)}


def tt_profile_launches(max_records: int = 4096) -> list:
    """Launches recorded since tt_profile_begin: [(kind name, device ms), ...]."""
    kinds = (_i32 * max_records)()
    ms = (ctypes.c_double * max_records)()
    n = _i32()
    _check(_lib.tt_profile_launches(kinds, ms, max_records, ctypes.byref(n)), "tt_profile_launches")
    return [(KIND_NAMES[kinds[i]], ms[i]) for i in range(n.value)]


def tt_version() -> str:
    return _lib.tt_version().decode()


def search(corpus: torch.Tensor, queries: torch.Tensor, k: int, tau: float = 1.0,
           exclude: torch.Tensor | None = None, store_dtype=torch.bfloat16,
           query_dtype=None, fused: bool = False, device="cuda"):
    """End-to-end call from host tensors: copy the raw corpus and queries to
    the GPU, normalise both, score, and copy ``(ids, scores)`` back.

    ``corpus`` [n, d] and ``queries`` [b, d] are CPU tensors (pinned memory
    makes the copies asynchronous). ``fused`` keeps the corpus raw and folds
    the norms into the scores; ``store_dtype=torch.int8`` codes the
    normalised corpus in int8 (``tt_quantize_candidates``) and scores with
    int8 codes. ``query_dtype`` defaults to float32 for small batches
    (b <= 8) and bfloat16 otherwise."""
    n, d = corpus.shape
    b = queries.shape[0]
    dc = corpus.to(device, non_blocking=True)
    dq = queries.to(device, non_blocking=True)
    dx = exclude.to(device, non_blocking=True) if exclude is not None else None
    if fused:
        inv = torch.empty((n,), dtype=torch.float32, device=device)
        index = tt_normalize_candidates(dc, inv, TT_NORM_FUSED)
    elif store_dtype == torch.int8:
        codes = torch.empty((n, d), dtype=torch.int8, device=device)
        scales = torch.empty((n,), dtype=torch.float32, device=device)
        index = tt_quantize_candidates(dc, codes, scales)
    else:
        rows = torch.empty((n, d), dtype=store_dtype, device=device)
        index = tt_normalize_candidates(dc, rows, TT_NORM_STORE)
    if query_dtype is None:
        query_dtype = torch.float32 if b <= 8 else torch.bfloat16
    qn = torch.empty((b, d), dtype=query_dtype, device=device)
    tt_normalize_candidates(dq, qn, TT_NORM_STORE, make_index=False)
    ids, scores = tt_score_topk(index, qn, k, tau=tau, exclude=dx)
    out_ids = torch.empty((b, k), dtype=torch.int32, pin_memory=True)
    out_scores = torch.empty((b, k), dtype=torch.float32, pin_memory=True)
    out_ids.copy_(ids, non_blocking=True)
    out_scores.copy_(scores, non_blocking=True)
    torch.cuda.current_stream().synchronize()
    index.free()
    return out_ids, out_scores
