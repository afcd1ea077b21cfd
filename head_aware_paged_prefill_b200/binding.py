"""ctypes binding of librk.so (the C ABI declared in include/rk.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
library is missing, every call raises; there is no fallback.
"""
from __future__ import annotations

import copy
import ctypes
import dataclasses
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librk.so")

RK_OK, RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY, RK_ERR_CUDA, RK_ERR_DEVICE = range(6)
RK_DEV_BAD_PAGE, RK_DEV_TIMEOUT, RK_DEV_CAPACITY = 1, 2, 4
STATUS_NAMES = {0: "RK_OK", 1: "RK_ERR_INVALID_ARG", 2: "RK_ERR_UNALIGNED", 3: "RK_ERR_CAPACITY",
                4: "RK_ERR_CUDA", 5: "RK_ERR_DEVICE"}


class RkError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class RkDims(ctypes.Structure):
    _fields_ = [("n_req", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("n_pages", ctypes.c_int64), ("total_tokens", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class RkLayout(ctypes.Structure):
    _fields_ = [("n_segments", ctypes.c_int32), ("segments", ctypes.c_void_p),
                ("page_base", ctypes.c_void_p), ("cu_seqlens", ctypes.c_void_p),
                ("class_map", ctypes.c_void_p), ("class_window", ctypes.c_void_p),
                ("retr_indptr", ctypes.c_void_p), ("retr_pages", ctypes.c_void_p)]


class RkVisible(ctypes.Structure):
    _fields_ = [("entries", ctypes.c_void_p), ("entry_start", ctypes.c_void_p),
                ("entry_count", ctypes.c_void_p), ("ranges", ctypes.c_void_p),
                ("range_start", ctypes.c_void_p), ("range_count", ctypes.c_void_p),
                ("entry_capacity", ctypes.c_int64), ("range_capacity", ctypes.c_int64)]


class RkSizes(ctypes.Structure):
    _fields_ = [("n_tables", ctypes.c_int64), ("entry_capacity", ctypes.c_int64),
                ("range_capacity", ctypes.c_int64), ("item_capacity", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64)]


EXPORTS = ("rk_query_sizes", "rk_select_visible", "rk_relocate_rope", "rk_segpaged_prefill",
           "rk_get_device_status", "rk_select_visible_noalloc", "rk_selftest_bounded_wait",
           "rk_score_query_sizes", "rk_score_retrieval_pages", "rk_decode_query_sizes",
           "rk_segpaged_decode", "rk_importance_query_sizes", "rk_attention_importance",
           "rk_ffn_query_sizes", "rk_sparse_ffn", "rk_relocation_query_sizes",
           "rk_relocation_plan")

_lib = None


def lib() -> ctypes.CDLL:
    """Loads librk.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m head_aware_paged_prefill_b200.csrc.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.rk_query_sizes.argtypes = [vp, vp, vp]
        L.rk_select_visible.argtypes = [vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.rk_relocate_rope.argtypes = [vp, i64, vp, i64, vp, i32, i32, i32, ctypes.c_double, vp,
                                       vp]
        L.rk_segpaged_prefill.argtypes = [vp, vp, vp, vp, vp, i32, ctypes.c_double, ctypes.c_float,
                                          vp, vp, vp, ctypes.c_size_t, vp]
        L.rk_get_device_status.argtypes = [vp, vp, vp]
        L.rk_select_visible_noalloc.argtypes = [vp, vp, vp, vp, vp]
        L.rk_selftest_bounded_wait.argtypes = [vp, i32, vp]
        L.rk_score_query_sizes.argtypes = [vp, vp, i32, vp]
        L.rk_decode_query_sizes.argtypes = [vp, vp, vp]
        L.rk_segpaged_decode.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                         ctypes.c_size_t, vp]
        L.rk_score_retrieval_pages.argtypes = [vp, vp, vp, vp, ctypes.c_double, i32, vp, vp, vp,
                                               i64, vp, ctypes.c_size_t, vp]
        L.rk_importance_query_sizes.argtypes = [vp, vp, vp]
        L.rk_attention_importance.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, vp,
                                              vp, vp, vp, ctypes.c_size_t, vp]
        L.rk_ffn_query_sizes.argtypes = [vp, i32, vp, i32, vp]
        L.rk_relocation_query_sizes.argtypes = [vp, vp, vp]
        L.rk_relocation_plan.argtypes = [vp, vp, vp, i64, vp, i64, vp, vp]
        L.rk_sparse_ffn.argtypes = [vp, i32, vp, vp, i32, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        for name in EXPORTS:
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != RK_OK:
        raise RkError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class RkDecodeSizes(ctypes.Structure):
    _fields_ = [("n_pieces", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


class RkRelocationSizes(ctypes.Structure):
    _fields_ = [("n_jobs_k", ctypes.c_int64), ("n_jobs_v", ctypes.c_int64),
                ("n_extra_pages", ctypes.c_int64)]


class RkFfnDims(ctypes.Structure):
    _fields_ = [("n_rows", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class RkFfnSizes(ctypes.Structure):
    _fields_ = [("n_selected", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


class RkImportanceSizes(ctypes.Structure):
    _fields_ = [("n_items", ctypes.c_int64), ("workspace_bytes", ctypes.c_int64)]


class RkScoreSizes(ctypes.Structure):
    _fields_ = [("n_tables", ctypes.c_int64), ("max_pages", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_int64)]


class HostLayout:
    """ctypes view of a host-side layout (an object with the attributes of
    ``synth.Layout``).  Keeps the contiguous arrays it points into alive."""

    def __init__(self, lay):
        self.lay = lay
        seg = np.ascontiguousarray(lay.segments, dtype=np.int32).reshape(-1, 5)
        pb = np.ascontiguousarray(lay.page_base, dtype=np.int32)
        cu = np.ascontiguousarray(lay.cu_seqlens, dtype=np.int32)
        cm = np.ascontiguousarray(lay.class_map, dtype=np.int8)
        cw = np.ascontiguousarray(lay.class_window, dtype=np.int32)
        ri = np.ascontiguousarray(lay.retr_indptr, dtype=np.int32)
        rp = np.ascontiguousarray(np.concatenate([np.asarray(lay.retr_pages, np.int32),
                                                  np.zeros(1, np.int32)]))
        self._keep = (seg, pb, cu, cm, cw, ri, rp)
        self.layout = RkLayout(seg.shape[0], seg.ctypes.data, pb.ctypes.data, cu.ctypes.data,
                               cm.ctypes.data, cw.ctypes.data, ri.ctypes.data, rp.ctypes.data)
        self.dims = RkDims(lay.n_req, lay.n_layers, lay.hq, lay.hkv, lay.d, lay.p, lay.n_pages,
                           int(cu[-1]), 0)

    def sizes(self) -> RkSizes:
        s = RkSizes()
        _check(lib().rk_query_sizes(ctypes.byref(self.dims), ctypes.byref(self.layout),
                                    ctypes.byref(s)), "rk_query_sizes")
        return s


class Visible:
    """Device buffers of rk_visible, sized by rk_query_sizes."""

    def __init__(self, sizes: RkSizes, device):
        nt = max(1, int(sizes.n_tables))
        dev = torch.device(device)
        self.entries = torch.zeros((max(1, int(sizes.entry_capacity)), 4), dtype=torch.int32,
                                   device=dev)
        self.entry_start = torch.zeros(nt, dtype=torch.int32, device=dev)
        self.entry_count = torch.zeros(nt, dtype=torch.int32, device=dev)
        self.ranges = torch.zeros((max(1, int(sizes.range_capacity)), 2), dtype=torch.int32,
                                  device=dev)
        self.range_start = torch.zeros(nt, dtype=torch.int32, device=dev)
        self.range_count = torch.zeros(nt, dtype=torch.int32, device=dev)
        self.struct = RkVisible(self.entries.data_ptr(), self.entry_start.data_ptr(),
                                self.entry_count.data_ptr(), self.ranges.data_ptr(),
                                self.range_start.data_ptr(), self.range_count.data_ptr(),
                                self.entries.shape[0], self.ranges.shape[0])

    def tables(self):
        """Per-table (entries [n, 4], ranges [m, 2]) as numpy, in table order."""
        es, ec = self.entry_start.cpu().numpy(), self.entry_count.cpu().numpy()
        rs, rc = self.range_start.cpu().numpy(), self.range_count.cpu().numpy()
        E, R = self.entries.cpu().numpy(), self.ranges.cpu().numpy()
        return ([E[a:a + n] for a, n in zip(es, ec)], [R[a:a + n] for a, n in zip(rs, rc)])


def workspace(sizes: RkSizes, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.zeros(int(sizes.workspace_bytes), dtype=torch.uint8, device=torch.device(device))


def select_visible(hl: HostLayout, vis: Visible, ws: torch.Tensor, stream=None):
    _check(lib().rk_select_visible(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                   ctypes.byref(vis.struct), _ptr(ws), ws.numel(),
                                   _stream(stream)), "rk_select_visible")


def select_visible_noalloc(hl: HostLayout, vis: Visible,
                           device_error: Optional[torch.Tensor] = None, stream=None):
    """Page tables and row ranges into ``vis`` without a caller workspace:
    the library's own fixed-size device scratch is used (see include/rk.h)."""
    _check(lib().rk_select_visible_noalloc(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                           ctypes.byref(vis.struct), _ptr(device_error),
                                           _stream(stream)), "rk_select_visible_noalloc")


def relocate_rope(k_src: torch.Tensor, k_dst: torch.Tensor, jobs: torch.Tensor, theta: float,
                  device_error: Optional[torch.Tensor] = None, stream=None):
    n_src, p, d = k_src.shape
    assert k_dst.shape[1:] == k_src.shape[1:] and k_src.dtype == k_dst.dtype == torch.bfloat16
    assert jobs.dtype == torch.int32 and jobs.is_contiguous()
    _check(lib().rk_relocate_rope(_ptr(k_src), n_src, _ptr(k_dst), k_dst.shape[0], _ptr(jobs),
                                  jobs.shape[0], p, d, float(theta), _ptr(device_error),
                                  _stream(stream)),
           "rk_relocate_rope")


def segpaged_prefill(hl: HostLayout, q: torch.Tensor, k_pool: torch.Tensor,
                     v_pool: torch.Tensor, vis: Visible, ws: torch.Tensor, o: torch.Tensor,
                     lse: Optional[torch.Tensor] = None, fuse_rope: bool = False,
                     stream=None):
    lay = hl.lay
    for t in (q, k_pool, v_pool, o):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    _check(lib().rk_segpaged_prefill(ctypes.byref(hl.dims), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                     ctypes.byref(vis.struct), 1 if fuse_rope else 0,
                                     float(lay.theta), float(lay.softmax_scale), _ptr(o),
                                     _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "rk_segpaged_prefill")


def selftest_bounded_wait(word: torch.Tensor, wait_ms: int, stream=None):
    _check(lib().rk_selftest_bounded_wait(_ptr(word), int(wait_ms), _stream(stream)),
           "rk_selftest_bounded_wait")


def device_status(ws: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(0)
    st = lib().rk_get_device_status(_ptr(ws), ctypes.byref(v), _stream(stream))
    if st not in (RK_OK, RK_ERR_DEVICE):
        raise RkError(st, "rk_get_device_status")
    return int(v.value)


# ------------------------------------------------------ retrieval page scoring

def score_sizes(hl: HostLayout, top_k: int = 16) -> RkScoreSizes:
    s = RkScoreSizes()
    _check(lib().rk_score_query_sizes(ctypes.byref(hl.dims), ctypes.byref(hl.layout), int(top_k),
                                      ctypes.byref(s)), "rk_score_query_sizes")
    return s


class ScoreOutputs:
    """Device outputs of rk_score_retrieval_pages for one layout."""

    def __init__(self, sizes: RkScoreSizes, top_k: int, device, with_scores: bool = True):
        dev = torch.device(device)
        n = int(sizes.n_tables)
        self.top_k = int(top_k)
        self.pages = torch.zeros((n, self.top_k), dtype=torch.int32, device=dev)
        self.count = torch.zeros(n, dtype=torch.int32, device=dev)
        self.stride = max(int(sizes.max_pages), 1)
        self.scores = (torch.empty((n, self.stride), dtype=torch.float32, device=dev)
                       if with_scores else None)
        self.ws = torch.zeros(max(int(sizes.workspace_bytes), 256), dtype=torch.uint8, device=dev)

    def lists(self):
        """The picks as a host CSR (retr_indptr, retr_pages) over tables."""
        count = self.count.cpu().numpy()
        pages = self.pages.cpu().numpy()
        indptr = np.zeros(count.shape[0] + 1, dtype=np.int32)
        indptr[1:] = np.cumsum(count)
        flat = np.concatenate([pages[t, :count[t]] for t in range(count.shape[0])] +
                              [np.zeros(0, np.int32)]).astype(np.int32)
        return indptr, flat


def score_retrieval_pages(hl: HostLayout, q: torch.Tensor, k_store: torch.Tensor, theta: float,
                          out: ScoreOutputs, stream=None):
    _check(lib().rk_score_retrieval_pages(
        ctypes.byref(hl.dims), ctypes.byref(hl.layout), _ptr(q), _ptr(k_store), float(theta),
        out.top_k, _ptr(out.pages), _ptr(out.count), _ptr(out.scores),
        out.stride if out.scores is not None else 0, _ptr(out.ws), out.ws.numel(),
        _stream(stream)), "rk_score_retrieval_pages")


# ------------------------------------------------------------------ decode

def decode_sizes(hl: HostLayout) -> RkDecodeSizes:
    s = RkDecodeSizes()
    _check(lib().rk_decode_query_sizes(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                       ctypes.byref(s)), "rk_decode_query_sizes")
    return s


def decode_workspace(sizes: RkDecodeSizes, device) -> torch.Tensor:
    return torch.zeros(int(sizes.workspace_bytes), dtype=torch.uint8, device=torch.device(device))


def segpaged_decode(hl: HostLayout, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                    vis: Visible, ws: torch.Tensor, o: torch.Tensor,
                    lse: Optional[torch.Tensor] = None, stream=None):
    """q, o: bf16 [n_layers][n_req][Hq][D] (one row per request)."""
    for t in (q, k_pool, v_pool, o):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    _check(lib().rk_segpaged_decode(ctypes.byref(hl.dims), ctypes.byref(hl.layout), _ptr(q),
                                    _ptr(k_pool), _ptr(v_pool), ctypes.byref(vis.struct),
                                    float(hl.lay.softmax_scale), _ptr(o), _ptr(lse), _ptr(ws),
                                    ws.numel(), _stream(stream)), "rk_segpaged_decode")


def importance_sizes(hl: HostLayout) -> RkImportanceSizes:
    s = RkImportanceSizes()
    _check(lib().rk_importance_query_sizes(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                           ctypes.byref(s)), "rk_importance_query_sizes")
    return s


def importance_workspace(sizes: RkImportanceSizes, device) -> torch.Tensor:
    return torch.zeros(int(sizes.workspace_bytes), dtype=torch.uint8, device=torch.device(device))


def attention_importance(hl: HostLayout, q: torch.Tensor, k_pool: torch.Tensor, vis: Visible,
                         lse: torch.Tensor, ws: torch.Tensor, importance: torch.Tensor,
                         top_k: int = 0, tokens: Optional[torch.Tensor] = None,
                         token_count: Optional[torch.Tensor] = None, stream=None):
    """q: bf16 [n_layers][T][Hq][D]; k_pool: relocated bf16 [n_pages][P][D];
    lse: fp32 [n_layers][Hq][T] from the prefill; importance: fp32
    [n_layers][T]; tokens: int32 [n_layers][n_req][top_k] and token_count:
    int32 [n_layers][n_req], or both None."""
    for t in (q, k_pool):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    for t in (lse, importance):
        assert t.dtype == torch.float32 and t.is_contiguous()
    for t in (tokens, token_count):
        assert t is None or (t.dtype == torch.int32 and t.is_contiguous())
    _check(lib().rk_attention_importance(ctypes.byref(hl.dims), ctypes.byref(hl.layout), _ptr(q),
                                         _ptr(k_pool), ctypes.byref(vis.struct), _ptr(lse),
                                         float(hl.lay.softmax_scale), int(top_k),
                                         _ptr(importance), _ptr(tokens), _ptr(token_count),
                                         _ptr(ws), ws.numel(), _stream(stream)),
           "rk_attention_importance")


# ------------------------------------------------------ token-selective FFN

def _ffn_args(n_rows: int, d_model: int, d_ff: int, cu_seqlens):
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    return RkFfnDims(int(n_rows), int(d_model), int(d_ff), 0), cu


def ffn_sizes(n_rows: int, d_model: int, d_ff: int, cu_seqlens, top_k: int) -> RkFfnSizes:
    dims, cu = _ffn_args(n_rows, d_model, d_ff, cu_seqlens)
    s = RkFfnSizes()
    _check(lib().rk_ffn_query_sizes(ctypes.byref(dims), cu.shape[0] - 1, cu.ctypes.data,
                                    int(top_k), ctypes.byref(s)), "rk_ffn_query_sizes")
    return s


def ffn_workspace(sizes: RkFfnSizes, device) -> torch.Tensor:
    return torch.empty(max(256, int(sizes.workspace_bytes)), dtype=torch.uint8,
                       device=torch.device(device))


def sparse_ffn(x: torch.Tensor, cu_seqlens, tokens: Optional[torch.Tensor], top_k: int,
               w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, ws: torch.Tensor,
               stream=None):
    """rk_sparse_ffn: x [n_rows][d_model] bf16 (updated in place at the
    selected rows); tokens int32 [n_req][top_k] request-local picks (one
    layer of rk_attention_importance's output); w_gate / w_up [d_ff][d_model],
    w_down [d_model][d_ff] bf16."""
    n_rows, d_model = x.shape
    d_ff = w_gate.shape[0]
    assert x.dtype == w_gate.dtype == w_up.dtype == w_down.dtype == torch.bfloat16
    assert w_up.shape == w_gate.shape == (d_ff, d_model) and w_down.shape == (d_model, d_ff)
    dims, cu = _ffn_args(n_rows, d_model, d_ff, cu_seqlens)
    _check(lib().rk_sparse_ffn(ctypes.byref(dims), cu.shape[0] - 1, cu.ctypes.data, _ptr(tokens),
                               int(top_k), _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                               _ptr(ws), ws.numel(), _stream(stream)), "rk_sparse_ffn")


# ------------------------------------------------------ relocation plan

@dataclasses.dataclass
class RelocationPlan:
    jobs_k: np.ndarray   # int32 [n, 3] (src_page in the K store, dst_page in the working K pool, delta)
    jobs_v: np.ndarray   # int32 [m, 3] (src_page, dst_page >= n_pages, 0) within the working V pool
    layout: object       # the relocated layout: every segment at delta 0, appended runs in page_base
    n_extra: int         # pages appended to both working pools


def relocation_plan(lay) -> RelocationPlan:
    """rk_relocation_plan (host only): the relocate-mode step's job lists and
    relocated layout for a layout (an object with synth.Layout's fields)."""
    hl = HostLayout(lay)
    sz = RkRelocationSizes()
    _check(lib().rk_relocation_query_sizes(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                           ctypes.byref(sz)), "rk_relocation_query_sizes")
    nk, nv = int(sz.n_jobs_k), int(sz.n_jobs_v)
    jk = np.zeros((max(nk, 1), 3), dtype=np.int32)
    jv = np.zeros((max(nv, 1), 3), dtype=np.int32)
    n_seg = int(np.asarray(lay.segments).reshape(-1, 5).shape[0])
    segs = np.zeros((max(n_seg, 1), 5), dtype=np.int32)
    pb = np.zeros((max(n_seg, 1), lay.n_layers * lay.hkv), dtype=np.int32)
    _check(lib().rk_relocation_plan(ctypes.byref(hl.dims), ctypes.byref(hl.layout), jk.ctypes.data,
                                    nk, jv.ctypes.data, nv, segs.ctypes.data, pb.ctypes.data),
           "rk_relocation_plan")
    out = copy.copy(lay)
    out.segments = segs[:n_seg].copy()
    out.page_base = pb[:n_seg].copy()
    out.n_pages = int(lay.n_pages) + int(sz.n_extra_pages)
    return RelocationPlan(jk[:nk].copy(), jv[:nv].copy(), out, int(sz.n_extra_pages))
