"""The C-ABI library loads, exports what include/rk.h declares, and rejects
bad arguments on the host before any GPU work (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from head_aware_paged_prefill_b200.csrc import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return binding.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "rk.h")).read()
    return sorted(set(re.findall(r"^rk_status\s+(rk_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert set(names) == set(binding.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def _hl(lay):
    return binding.HostLayout(lay)


@pytest.mark.parametrize("name", ["cfg1", "cfg2", "cfg3", "cfg4", "cfg5"])
def test_query_sizes(lib, name):
    lay = synth.CONFIGS[name]().layout
    s = _hl(lay).sizes()
    n_lh = lay.n_layers * lay.hkv
    total_pages = sum(-(-lay.req_len(r) // lay.p) for r in range(lay.n_req))
    assert s.n_tables == lay.n_tables
    assert s.entry_capacity == n_lh * total_pages
    assert s.range_capacity == n_lh * lay.segments.shape[0]
    assert s.workspace_bytes % 256 == 0 and s.workspace_bytes > 256 + 96 * s.item_capacity


def _status_sizes(lay, mutate):
    hl = _hl(lay)
    mutate(hl)
    s = binding.RkSizes()
    return binding.lib().rk_query_sizes(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                        ctypes.byref(s))


def test_rejects_bad_dims(lib):
    lay = synth.cfg1().layout
    E = binding.RK_ERR_INVALID_ARG
    assert _status_sizes(lay, lambda h: setattr(h.dims, "head_dim", 96)) == E
    assert _status_sizes(lay, lambda h: setattr(h.dims, "page_size", 32)) == E
    assert _status_sizes(lay, lambda h: setattr(h.dims, "num_q_heads", 3)) == E
    assert _status_sizes(lay, lambda h: setattr(h.dims, "n_pages", 0)) == E
    assert _status_sizes(lay, lambda h: setattr(h.dims, "total_tokens", 447)) == E
    assert _status_sizes(lay, lambda h: setattr(h.dims, "reserved", 1)) == E
    assert _status_sizes(lay, lambda h: setattr(h.dims, "n_req", 0)) == E


def test_rejects_bad_layouts(lib):
    base = synth.cfg1().layout

    def with_(**kw):
        lay = synth.Layout(**{**base.__dict__})
        for k, v in kw.items():
            setattr(lay, k, v)
        return lay

    E, U = binding.RK_ERR_INVALID_ARG, binding.RK_ERR_UNALIGNED
    seg = base.segments.copy()
    seg[0, 2] = 120
    seg[1, 1] = 120
    seg[1, 2] = 136
    assert _status_sizes(with_(segments=seg), lambda h: None) == U  # 120 % 16 != 0
    pb = base.page_base.copy()
    pb[3, 1] = base.n_pages - 1  # tail needs 4 pages
    assert _status_sizes(with_(page_base=pb), lambda h: None) == E
    seg = base.segments.copy()
    seg[2, 1] = 250  # gap
    assert _status_sizes(with_(segments=seg), lambda h: None) == E
    assert _status_sizes(with_(class_map=np.asarray([0, 4], np.int8)), lambda h: None) == E
    cw = base.class_window.copy()
    cw[1] = 0
    assert _status_sizes(with_(class_window=cw), lambda h: None) == E
    cu = base.cu_seqlens.copy()
    cu[1] = 440
    assert _status_sizes(with_(cu_seqlens=cu), lambda h: None) == E
    # retrieval class without lists
    lay = with_(class_map=np.asarray([0, 2], np.int8))
    assert _status_sizes(lay, lambda h: setattr(h.layout, "retr_indptr", None)) == E
    assert _status_sizes(base, lambda h: setattr(h.layout, "segments", None)) == E


def test_select_rejects_on_host_without_gpu(lib):
    lay = synth.cfg1().layout
    hl = _hl(lay)
    s = hl.sizes()
    vis = binding.RkVisible()  # null pointers
    st = lib.rk_select_visible(ctypes.byref(hl.dims), ctypes.byref(hl.layout), ctypes.byref(vis),
                               ctypes.c_void_p(256), s.workspace_bytes, None)
    assert st == binding.RK_ERR_INVALID_ARG
    fake = 1 << 20  # never dereferenced: the capacity check fails first
    vis = binding.RkVisible(fake, fake, fake, fake, fake, fake, s.entry_capacity - 1,
                            s.range_capacity)
    st = lib.rk_select_visible(ctypes.byref(hl.dims), ctypes.byref(hl.layout), ctypes.byref(vis),
                               ctypes.c_void_p(fake), s.workspace_bytes, None)
    assert st == binding.RK_ERR_CAPACITY
    vis = binding.RkVisible(fake, fake, fake, fake, fake, fake, s.entry_capacity,
                            s.range_capacity)
    st = lib.rk_select_visible(ctypes.byref(hl.dims), ctypes.byref(hl.layout), ctypes.byref(vis),
                               ctypes.c_void_p(fake), s.workspace_bytes - 256, None)
    assert st == binding.RK_ERR_CAPACITY


def test_relocate_and_prefill_reject_on_host(lib):
    E = binding.RK_ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    # (k_src, n_src_pages, k_dst, n_dst_pages, jobs, n_jobs, P, D, theta, error, stream)
    assert lib.rk_relocate_rope(fake, 8, fake, 8, fake, 1, 64, 96, 1e4, None, None) == E
    assert lib.rk_relocate_rope(fake, 8, fake, 8, fake, -1, 64, 128, 1e4, None, None) == E
    assert lib.rk_relocate_rope(fake, 8, fake, 8, fake, 1, 64, 128, -1.0, None, None) == E
    assert lib.rk_relocate_rope(None, 8, fake, 8, fake, 1, 64, 128, 1e4, None, None) == E
    assert lib.rk_relocate_rope(fake, 0, fake, 8, fake, 1, 64, 128, 1e4, None, None) == E
    assert lib.rk_relocate_rope(fake, 8, fake, 0, fake, 1, 64, 128, 1e4, None, None) == E
    assert lib.rk_relocate_rope(fake, 8, fake, 8, fake, 1, 0, 128, 1e4, None, None) == E
    assert lib.rk_relocate_rope(ctypes.c_void_p((1 << 20) + 2), 8, fake, 8, fake, 1, 64, 128,
                                1e4, None, None) == E
    # no jobs: nothing to do, no pointer needed
    assert lib.rk_relocate_rope(None, 8, None, 8, None, 0, 64, 128, 1e4, None, None) == 0
    lay = synth.cfg1().layout
    hl = _hl(lay)
    vis = binding.RkVisible(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1, 1)
    args = [ctypes.byref(hl.dims), fake, fake, fake, ctypes.byref(vis), 0, 1e4, 0.125, fake,
            None, fake, 1 << 20, None]
    bad_scale = list(args)
    bad_scale[7] = 0.0
    assert lib.rk_segpaged_prefill(*bad_scale) == E
    bad_fuse = list(args)
    bad_fuse[5] = 2
    assert lib.rk_segpaged_prefill(*bad_fuse) == E
    null_q = list(args)
    null_q[1] = None
    assert lib.rk_segpaged_prefill(*null_q) == E
    small_ws = list(args)
    small_ws[11] = 16
    assert lib.rk_segpaged_prefill(*small_ws) == binding.RK_ERR_CAPACITY
    assert lib.rk_get_device_status(None, None, None) == E



def test_score_calls_validate_on_host(lib):
    """Retrieval page scoring: sizes follow the layout, and every argument
    error is returned before any GPU work."""
    E, C = binding.RK_ERR_INVALID_ARG, binding.RK_ERR_CAPACITY
    lay = synth.cfg4().layout
    hl = _hl(lay)
    s = binding.score_sizes(hl, 16)
    assert s.n_tables == lay.n_tables and s.max_pages == -(-lay.req_len(0) // lay.p)
    assert s.workspace_bytes > 0 and s.workspace_bytes % 256 == 0
    # the layout's retrieval lists are optional here
    hl.layout.retr_indptr = None
    hl.layout.retr_pages = None
    s2 = binding.score_sizes(hl, 16)
    assert s2.workspace_bytes == s.workspace_bytes
    out = binding.RkScoreSizes()
    for k in (0, 65):
        assert lib.rk_score_query_sizes(ctypes.byref(hl.dims), ctypes.byref(hl.layout), k,
                                        ctypes.byref(out)) == E
    fake = ctypes.c_void_p(1 << 20)
    # (dims, layout, q, k_store, theta, top_k, pages, count, scores, stride, ws, ws_bytes, stream)
    args = [ctypes.byref(hl.dims), ctypes.byref(hl.layout), fake, fake, 1e6, 16, fake, fake, fake,
            s.max_pages, fake, s.workspace_bytes, None]

    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.rk_score_retrieval_pages(*a)

    assert call(a2=None) == E               # q
    assert call(a3=None) == E               # k_store
    assert call(a4=-1.0) == E               # theta
    assert call(a5=0) == E                  # top_k
    assert call(a6=None) == E               # out_pages
    assert call(a3=ctypes.c_void_p((1 << 20) + 2)) == E  # unaligned k_store
    assert call(a9=s.max_pages - 1) == C    # scores row too short
    assert call(a11=s.workspace_bytes - 1) == C


def test_importance_calls_validate_on_host(lib):
    """Attention importance: sizes follow the layout, and argument errors are
    returned before any GPU work."""
    E, C = binding.RK_ERR_INVALID_ARG, binding.RK_ERR_CAPACITY
    lay = synth.cfg1().layout
    hl = _hl(lay)
    s = binding.importance_sizes(hl)
    assert s.n_items == _importance_items_brute(lay)
    assert s.workspace_bytes >= 256 + 4 * 256 * s.n_items
    assert s.workspace_bytes % 256 == 0
    sz = hl.sizes()
    fake = ctypes.c_void_p(1 << 20)
    vis = binding.RkVisible(fake.value, fake.value, fake.value, fake.value, fake.value,
                            fake.value, sz.entry_capacity, sz.range_capacity)
    # (dims, layout, q, k_pool, vis, lse, scale, top_k, importance, tokens,
    #  token_count, ws, ws_bytes, stream)
    args = [ctypes.byref(hl.dims), ctypes.byref(hl.layout), fake, fake, ctypes.byref(vis), fake,
            0.125, 8, fake, fake, fake, fake, s.workspace_bytes, None]

    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.rk_attention_importance(*a)

    assert call(a2=None) == E                # q
    assert call(a5=None) == E                # lse
    assert call(a6=0.0) == E                 # softmax scale
    assert call(a7=-1) == E                  # top_k
    assert call(a8=None) == E                # importance
    assert call(a10=None) == E               # tokens without token_count
    assert call(a3=ctypes.c_void_p((1 << 20) + 8)) == E  # unaligned k_pool
    assert call(a12=s.workspace_bytes - 1) == C
    small = binding.RkVisible(fake.value, fake.value, fake.value, fake.value, fake.value,
                              fake.value, sz.entry_capacity - 1, sz.range_capacity)
    assert call(a4=ctypes.byref(small)) == C


KB = 256          # keys per importance work item
CHUNK_COLS = 4096  # (row, q head) columns per row chunk


def _importance_items_brute(lay) -> int:
    """Importance work items by brute force: for every table and every block
    of 256 consecutive page-table keys, the row chunks (CHUNK_COLS / G rows)
    from the one holding the first row that sees a key of the block to the
    one holding the last such row (visibility from the oracle's brute-force
    page tables and the class rule)."""
    entries, ranges = oracle.page_tables(lay)
    g = lay.hq // lay.hkv
    rpc = CHUNK_COLS // g
    W = int(lay.class_window[synth.LOCAL])
    n = 0
    for t in range(lay.n_tables):
        r, rem = divmod(t, lay.n_layers * lay.hkv)
        cls = int(lay.class_map[rem])
        rows = [i for a, b in ranges[t] for i in range(a, b)]
        epk = KB // lay.p
        ent = entries[t]
        for kb in range(-(-ent.shape[0] // epk)):
            blk = [int(e[1]) + k for e in ent[kb * epk: kb * epk + epk] for k in range(int(e[3]))]
            seeing = [i for i in rows
                      if any(k <= i and (cls != synth.LOCAL or i - k < W) for k in blk)]
            if seeing:
                n += seeing[-1] // rpc - seeing[0] // rpc + 1
    return n


def _importance_items_tail_layout(lay) -> int:
    """The same count in closed form for layouts whose only uncached segment
    is each request's last (the full-size workloads)."""
    P, g, W = lay.p, lay.hq // lay.hkv, int(lay.class_window[synth.LOCAL])
    rpc = CHUNK_COLS // g
    entries, _ = oracle.page_tables_closed_form(lay)
    n = 0
    for t in range(lay.n_tables):
        r, rem = divmod(t, lay.n_layers * lay.hkv)
        cls = int(lay.class_map[rem])
        L = lay.req_len(r)
        segs = lay.segments_of(r)
        unc = segs[segs[:, 4] == 0]
        assert unc.shape[0] <= 1 and (unc.shape[0] == 0 or int(unc[0, 1] + unc[0, 2]) == L)
        a = int(unc[0, 1]) if unc.shape[0] else L
        rows = (0, L) if cls in (synth.GLOBAL, synth.DENSE) else (a, L)
        if rows[0] >= rows[1]:
            continue
        e = entries[t]
        epk = KB // P
        for kb in range(-(-e.shape[0] // epk)):
            blk = e[kb * epk: kb * epk + epk]
            lo, hi = int(blk[0, 1]), int(blk[-1, 1] + blk[-1, 3] - 1)
            first = max(lo, rows[0])
            last = min(L - 1, hi + W - 1) if cls == synth.LOCAL else L - 1
            if first <= last:
                n += last // rpc - first // rpc + 1
    return n


def test_importance_items_match_brute_force(lib):
    """The library's exact item count equals the brute-force count on random
    small layouts (every class, windows, uncached segments anywhere)."""
    rng = np.random.default_rng(12)
    for _ in range(40):
        lay = synth.random_small(rng, max_pages=40)
        assert binding.importance_sizes(_hl(lay)).n_items == _importance_items_brute(lay)


@pytest.mark.parametrize("name", ["cfg2", "cfg3", "cfg4", "cfg5"])
def test_importance_workspace_exact(lib, name):
    """The workspace holds one 1 KB partial per work item plus small index
    arrays: no dense per-(chunk, token) buffer (the serving mix needs about
    260 MB, not GBs)."""
    lay = synth.CONFIGS[name]().layout
    s = binding.importance_sizes(_hl(lay))
    assert s.n_items == _importance_items_tail_layout(lay)
    g = lay.hq // lay.hkv
    max_pages = max(-(-lay.req_len(r) // lay.p) for r in range(lay.n_req))
    index = 8 * lay.n_tables * (max_pages * lay.p // KB + 1 + max_pages // 8 + 1) + 4 * lay.n_tables * max_pages
    assert 1024 * s.n_items <= s.workspace_bytes <= 1040 * s.n_items + index + 4096 + 8 * lay.n_tables


def test_ffn_calls_validate_on_host(lib):
    """Token-selective FFN: sizes follow the selection, and bad shapes or
    pointers are refused before any GPU work."""
    E, C = binding.RK_ERR_INVALID_ARG, binding.RK_ERR_CAPACITY
    s = binding.ffn_sizes(700, 256, 384, [0, 300, 700], 200)
    assert s.n_selected == 400
    assert s.workspace_bytes >= 2 * 400 * (256 + 384) and s.workspace_bytes % 256 == 0
    assert binding.ffn_sizes(700, 256, 384, [0, 300, 700], 1000).n_selected == 700
    for bad in ((700, 200, 384), (700, 256, 100), (699, 256, 384)):
        with pytest.raises(binding.RkError):
            binding.ffn_sizes(*bad, [0, 300, 700], 8)
    fake = ctypes.c_void_p(1 << 20)
    dims = binding.RkFfnDims(700, 256, 384, 0)
    cu = np.asarray([0, 300, 700], dtype=np.int32)
    args = [ctypes.byref(dims), 2, cu.ctypes.data, fake, 200, fake, fake, fake, fake, fake,
            s.workspace_bytes, None]

    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.rk_sparse_ffn(*a)

    assert call(a3=None) == E                           # tokens
    assert call(a5=None) == E                           # x
    assert call(a5=ctypes.c_void_p((1 << 20) + 2)) == E  # unaligned x
    assert call(a9=ctypes.c_void_p((1 << 20) + 16)) == E  # unaligned workspace
    assert call(a4=-1) == E                             # top_k
    assert call(a10=s.workspace_bytes - 1) == C
