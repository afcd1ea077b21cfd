"""fp64 CPU oracle for SegPagedAttention prefill.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  Nothing here is shared
with the CUDA path (``head_aware_paged_prefill_b200``); the two meet only in
the seeded input module ``head_aware_paged_prefill_b200.synth``.

The arithmetic lives in ``rk_oracle.c`` (plain C, fp64, pthreads); its header
states the definitions and the RedKnot passages they follow.  This module
marshals numpy arrays into it, fans independent tables out over threads, and
adds the closed-form restatements of the per-class rules that the pins compare
the brute-force derivations against (``page_tables_closed_form``,
``visible_pairs_closed_form``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from typing import List, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rk_oracle.c")
_SO = os.path.join(_HERE, "librk_oracle.so")
_lib = None

GLOBAL, LOCAL, RETRIEVAL, DENSE = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no GPU involved)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-D_DEFAULT_SOURCE", "-shared", "-fPIC",
                               "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        lib.ora_rope_rotate.argtypes = [P(ctypes.c_double), ctypes.c_int, ctypes.c_double,
                                        ctypes.c_double, P(ctypes.c_double)]
        lib.ora_page_table.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_int, P(ctypes.c_int),
                                       ctypes.c_void_p, ctypes.c_int, P(ctypes.c_int)]
        lib.ora_count_pairs.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int]
        lib.ora_count_pairs.restype = ctypes.c_int64
        lib.ora_relocate.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_double, ctypes.c_void_p]
        lib.ora_attention.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_double, ctypes.c_double,
                                      ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.ora_score_pages.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
        lib.ora_score_pages.restype = ctypes.c_int
        lib.ora_importance.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_void_p]
        lib.ora_importance.restype = ctypes.c_int
        lib.ora_sparse_ffn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                       ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        lib.ora_sparse_ffn.restype = ctypes.c_int
        _lib = lib
    return _lib


class _Problem(ctypes.Structure):
    _fields_ = [("n_req", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("hq", ctypes.c_int32),
                ("hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("p", ctypes.c_int32),
                ("n_seg", ctypes.c_int32), ("seg", ctypes.c_void_p), ("page_base", ctypes.c_void_p),
                ("cu_seqlens", ctypes.c_void_p), ("class_map", ctypes.c_void_p),
                ("class_window", ctypes.c_void_p), ("retr_indptr", ctypes.c_void_p),
                ("retr_pages", ctypes.c_void_p)]


class _ProblemRef:
    """A ctypes problem plus the contiguous arrays it points into."""

    def __init__(self, lay):
        self.keep = [np.ascontiguousarray(a) for a in (
            lay.segments.astype(np.int32), lay.page_base.astype(np.int32),
            lay.cu_seqlens.astype(np.int32), lay.class_map.astype(np.int8),
            lay.class_window.astype(np.int32), lay.retr_indptr.astype(np.int32),
            np.concatenate([lay.retr_pages.astype(np.int32), np.zeros(1, np.int32)]))]
        seg, pb, cu, cm, cw, ri, rp = self.keep
        self.s = _Problem(lay.n_req, lay.n_layers, lay.hq, lay.hkv, lay.d, lay.p,
                          seg.shape[0], seg.ctypes.data, pb.ctypes.data, cu.ctypes.data,
                          cm.ctypes.data, cw.ctypes.data, ri.ctypes.data, rp.ctypes.data)

    @property
    def ptr(self):
        return ctypes.addressof(self.s)


def _threads(n=None) -> int:
    return int(n or os.cpu_count() or 1)


def _tables(lay):
    for r in range(lay.n_req):
        for layer in range(lay.n_layers):
            for h in range(lay.hkv):
                yield lay.table_index(r, layer, h), r, layer, h


# ---------------------------------------------------------------- RoPE

def rope_rotate(x, theta: float, pos: float) -> np.ndarray:
    """R(pos) x for one D-vector (rotate-half pairs (m, m + D/2)), fp64."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    y = np.empty_like(x)
    P = ctypes.POINTER(ctypes.c_double)
    _load().ora_rope_rotate(x.ctypes.data_as(P), x.shape[0], float(theta), float(pos),
                            y.ctypes.data_as(P))
    return y


def relocate(k_pool_u16: np.ndarray, jobs: np.ndarray, p: int, d: int, theta: float) -> np.ndarray:
    """fp64 R(delta) K_stored for each job (src_page, dst_page, delta): [n, p, d]."""
    k = np.ascontiguousarray(k_pool_u16.view(np.uint16))
    jobs = np.ascontiguousarray(jobs.astype(np.int32))
    out = np.empty((jobs.shape[0], p, d), dtype=np.float64)
    _load().ora_relocate(k.ctypes.data, jobs.ctypes.data, jobs.shape[0], p, d, float(theta),
                         out.ctypes.data)
    return out


# ------------------------------------------------------------ page tables

def page_tables(lay, threads=None) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Brute-force per-table entries [n, 4] (phys_page, logical_pos, delta,
    n_valid) and merged row ranges [m, 2], indexed by table id."""
    lib = _load()
    pref = _ProblemRef(lay)
    n_t = lay.n_tables
    entries: List[np.ndarray] = [None] * n_t
    ranges: List[np.ndarray] = [None] * n_t
    n_seg_of = np.bincount(lay.segments[:, 0], minlength=lay.n_req)

    def one(args):
        t, r, layer, h = args
        L = lay.req_len(r)
        cap = -(-L // lay.p) + 1
        rcap = int(n_seg_of[r]) + 1
        e = np.zeros((cap, 4), dtype=np.int32)
        rg = np.zeros((rcap, 2), dtype=np.int32)
        ne, nr = ctypes.c_int(0), ctypes.c_int(0)
        rc = lib.ora_page_table(pref.ptr, r, layer, h, e.ctypes.data, cap, ctypes.byref(ne),
                                rg.ctypes.data, rcap, ctypes.byref(nr))
        assert rc == 0
        entries[t] = e[: ne.value].copy()
        ranges[t] = rg[: nr.value].copy()

    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(one, list(_tables(lay))))
    return entries, ranges


# ------------------------------------------------- retrieval page scoring

def score_pages(lay, q_u16: np.ndarray, k_pool_u16: np.ndarray, top_k: int = 16,
                threads=None) -> Tuple[List[np.ndarray], List[np.ndarray]]:
    """Per table: the retrieval page picks (ascending page indices within the
    request) and the fp64 score of every page of the request (NaN for pages
    that are not candidates).  The reading is stated in ``ora_score_pages``.
    q: bf16 bits [n_layers][T][Hq][D]; k_pool: bf16 bits [n_pages][P][D]."""
    lib = _load()
    pref = _ProblemRef(lay)
    q = np.ascontiguousarray(q_u16.view(np.uint16))
    k = np.ascontiguousarray(k_pool_u16.view(np.uint16))
    n_t = lay.n_tables
    picks: List[np.ndarray] = [None] * n_t
    scores: List[np.ndarray] = [None] * n_t

    def one(args):
        t, r, layer, h = args
        npg = -(-lay.req_len(r) // lay.p)
        pg = np.zeros(max(npg, 1), dtype=np.int32)
        sc = np.zeros(max(npg, 1), dtype=np.float64)
        n = lib.ora_score_pages(pref.ptr, q.ctypes.data, k.ctypes.data, float(lay.theta),
                                int(top_k), r, layer, h, pg.ctypes.data, sc.ctypes.data)
        picks[t] = pg[:n].copy()
        scores[t] = sc[:npg].copy()

    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(one, list(_tables(lay))))
    return picks, scores


# ------------------------------------------------- attention importance

def importance(lay, q_u16: np.ndarray, k_pool_u16: np.ndarray, threads=None) -> np.ndarray:
    """fp64 token importance [n_layers][T] (the reading is stated in
    ``ora_importance``): per request and layer, the prefill's softmax weights
    summed over q heads and computed rows.  q: bf16 bits [n_layers][T][Hq][D];
    k_pool: bf16 bits [n_pages][P][D] (stored, not relocated)."""
    lib = _load()
    pref = _ProblemRef(lay)
    q = np.ascontiguousarray(q_u16.view(np.uint16))
    k = np.ascontiguousarray(k_pool_u16.view(np.uint16))
    T = int(lay.cu_seqlens[-1])
    out = np.zeros((lay.n_layers, T), dtype=np.float64)

    def one(args):
        r, layer = args
        L = lay.req_len(r)
        if L == 0:
            return
        buf = np.zeros(L, dtype=np.float64)
        lib.ora_importance(pref.ptr, q.ctypes.data, k.ctypes.data, float(lay.theta),
                           float(lay.softmax_scale), r, layer, buf.ctypes.data)
        c0 = int(lay.cu_seqlens[r])
        out[layer, c0:c0 + L] = buf

    jobs = [(r, layer) for r in range(lay.n_req) for layer in range(lay.n_layers)]
    with ThreadPoolExecutor(_threads(threads)) as ex:
        list(ex.map(one, jobs))
    return out


def select_tokens(imp, top_k: int) -> np.ndarray:
    """The top_k positions by importance, ties to the lower position, in
    ascending order (all positions when there are at most top_k)."""
    vals = [float(x) for x in imp]
    ranked = sorted(range(len(vals)), key=lambda j: (-vals[j], j))
    return np.array(sorted(ranked[:max(int(top_k), 0)]), dtype=np.int32)


def _uncached_ranges(lay, r) -> List[Tuple[int, int]]:
    out: List[Tuple[int, int]] = []
    for seg in lay.segments_of(r):
        if seg[4]:
            continue
        a, b = int(seg[1]), int(seg[1] + seg[2])
        if out and out[-1][1] == a:
            out[-1] = (out[-1][0], b)
        else:
            out.append((a, b))
    return out


def _entry(lay, r, layer, h, k) -> Tuple[int, int, int, int]:
    P, L = lay.p, lay.req_len(r)
    pos = k * P
    for s, seg in enumerate(lay.segments):
        if seg[0] == r and seg[1] <= pos < seg[1] + seg[2]:
            pis = (pos - int(seg[1])) // P
            phys = int(lay.page_base[s, layer * lay.hkv + h]) + pis
            return phys, pos, pos - (int(seg[3]) + pis * P), min(P, L - pos)
    raise AssertionError("position outside every segment")


def page_tables_closed_form(lay):
    """Second derivation of the page tables, from each class's rule in closed
    form (the brute-force routine above is the primary one)."""
    P = lay.p
    W = int(lay.class_window[LOCAL])
    entries, ranges = [], []
    for t, r, layer, h in _tables(lay):
        L = lay.req_len(r)
        npg = -(-L // P)
        cls = int(lay.class_map[layer * lay.hkv + h])
        unc = _uncached_ranges(lay, r)
        if cls in (GLOBAL, DENSE):
            rows = [(0, L)] if L > 0 else []
            pages = list(range(npg))
        else:
            rows = unc
            cached_page = np.ones(npg, dtype=bool)
            for a, b in unc:
                cached_page[a // P: -(-b // P)] = False
            if cls == LOCAL:
                pages = [k for k in range(npg)
                         if any(max(k * P, a - W + 1) <= min(k * P + P, L, b) - 1
                                for a, b in rows)]
            else:
                sel = set(int(x) for x in lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]])
                last_row = rows[-1][1] - 1 if rows else -1
                pages = [k for k in range(npg)
                         if (not cached_page[k]) or (k in sel and k * P <= last_row)]
        entries.append(np.asarray([_entry(lay, r, layer, h, k) for k in pages],
                                  dtype=np.int32).reshape(-1, 4))
        ranges.append(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
    return entries, ranges


# ---------------------------------------------------------- pair counts

def visible_pairs(lay, threads=None, chunk: int = 2048) -> int:
    """Brute-force sum over (layer, q head, row) of visible keys."""
    lib = _load()
    pref = _ProblemRef(lay)
    g = lay.hq // lay.hkv
    units = []
    for t, r, layer, h in _tables(lay):
        L = lay.req_len(r)
        for a in range(0, L, chunk):
            units.append((r, layer, h, a, min(L, a + chunk)))
    with ThreadPoolExecutor(_threads(threads)) as ex:
        counts = list(ex.map(lambda u: lib.ora_count_pairs(pref.ptr, *u), units))
    return int(sum(counts)) * g


def visible_pairs_closed_form(lay) -> int:
    P = lay.p
    W = int(lay.class_window[LOCAL])
    g = lay.hq // lay.hkv
    total = 0
    for t, r, layer, h in _tables(lay):
        L = lay.req_len(r)
        cls = int(lay.class_map[layer * lay.hkv + h])
        if cls in (GLOBAL, DENSE):
            total += L * (L + 1) // 2
            continue
        unc = _uncached_ranges(lay, r)
        rows = np.concatenate([np.arange(a, b) for a, b in unc]) if unc else np.zeros(0, np.int64)
        if cls == LOCAL:
            total += int(np.minimum(rows + 1, W).sum())
        else:
            is_unc = np.zeros(L, dtype=np.int64)
            for a, b in unc:
                is_unc[a:b] = 1
            unc_before = np.cumsum(is_unc)  # uncached keys <= i
            sel = set(int(x) for x in lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]])
            sel = [k for k in sel if k * P < L and not is_unc[k * P]]
            for i in rows:
                c = int(unc_before[i])
                for k in sel:
                    c += max(0, min(k * P + P - 1, int(i)) - k * P + 1)
                total += c
    return total * g


# ------------------------------------------------------------ attention

def attention(lay, q_rows_u16: np.ndarray, k_pool_u16: np.ndarray, v_pool_u16: np.ndarray,
              rows: np.ndarray, threads=None):
    """fp64 attention for requested rows.

    rows: int32 [n, 3] of (layer, q_head, token); q_rows: bf16 bits [n, d],
    the query of each requested row.  Returns (o [n, d] fp64, lse [n] fp64,
    computed [n] int32), lse in natural log; rows outside their table's row
    set come back with computed = 0.
    """
    rows = np.ascontiguousarray(rows.astype(np.int32))
    n = rows.shape[0]
    q = np.ascontiguousarray(q_rows_u16.view(np.uint16).reshape(n, lay.d))
    kp = np.ascontiguousarray(k_pool_u16.view(np.uint16))
    vp = np.ascontiguousarray(v_pool_u16.view(np.uint16))
    o = np.zeros((n, lay.d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    comp = np.zeros(n, dtype=np.int32)
    pref = _ProblemRef(lay)
    _load().ora_attention(pref.ptr, q.ctypes.data, kp.ctypes.data, vp.ctypes.data,
                          float(lay.theta), float(lay.softmax_scale), rows.ctypes.data, n,
                          o.ctypes.data, lse.ctypes.data, comp.ctypes.data, _threads(threads))
    return o, lse, comp


# ------------------------------------------------------------ sparse FFN

def sparse_ffn(x_u16: np.ndarray, rows, w_gate_u16: np.ndarray, w_up_u16: np.ndarray,
               w_down_u16: np.ndarray, threads=None) -> np.ndarray:
    """fp64 token-selective FFN (rk_oracle.c, ora_sparse_ffn): for each listed
    row i of x [., d_model], y_i = x_i + W_down (silu(W_gate x_i) * W_up x_i).
    Weights are bf16 bits [d_ff][d_model] (gate, up) and [d_model][d_ff]
    (down).  Returns fp64 [len(rows)][d_model]; unlisted rows are x itself."""
    x = np.ascontiguousarray(x_u16.view(np.uint16))
    wg = np.ascontiguousarray(w_gate_u16.view(np.uint16))
    wu = np.ascontiguousarray(w_up_u16.view(np.uint16))
    wd = np.ascontiguousarray(w_down_u16.view(np.uint16))
    d_ff, d_model = wg.shape
    assert x.shape[-1] == d_model and wu.shape == wg.shape and wd.shape == (d_model, d_ff)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    y = np.zeros((rows.shape[0], d_model), dtype=np.float64)
    _load().ora_sparse_ffn(x.ctypes.data, d_model, rows.ctypes.data, rows.shape[0], wg.ctypes.data,
                           wu.ctypes.data, wd.ctypes.data, d_ff, y.ctypes.data, _threads(threads))
    return y
