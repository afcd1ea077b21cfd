"""The relocation plan (rk_relocation_plan, host only, no GPU): its jobs must
leave, in the working pools, exactly the rotated pages that the relocated
layout's page tables point at, and nothing more.  The library's plan is
also compared with a Python restatement (relocation_plan_ref) built from
the oracle's page tables."""
import numpy as np
import pytest

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from relocation_plan_ref import relocation_plan, visible_pages


def _check(lay, plan=None):
    entries, _ = oracle.page_tables(lay)
    if plan is None:
        plan = binding.relocation_plan(lay)
    n = int(lay.n_pages)
    n_all = n + plan.n_extra
    assert plan.layout.n_pages == n_all
    # every segment of the relocated layout sits at delta 0
    assert (plan.layout.segments[:, 1] == plan.layout.segments[:, 3]).all()
    # symbolic working pools: K page -> (store page, rotation), V page -> pool page
    kc = {p: (p, 0) for p in range(n)}
    vc = {p: p for p in range(n)}
    dst_k = plan.jobs_k[:, 1].tolist()
    assert len(set(dst_k)) == len(dst_k), "two K jobs write one page"
    for s, d, dl in plan.jobs_k.tolist():
        assert 0 <= s < n and 0 <= d < n_all
        assert d == s or d >= n, "an in-place job moved a page"
        assert dl != 0 or d >= n, "a delta-0 job on a page that already holds it"
        kc[d] = (s, dl)
    dst_v = plan.jobs_v[:, 1].tolist()
    assert len(set(dst_v)) == len(dst_v)
    for s, d, dl in plan.jobs_v.tolist():
        assert dl == 0 and 0 <= s < n <= d < n_all
        vc[d] = vc[s]
    new_entries, _ = oracle.page_tables(plan.layout)
    read = set()
    for t, (a, b) in enumerate(zip(entries, new_entries)):
        assert a.shape == b.shape, f"table {t}"
        np.testing.assert_array_equal(a[:, 1], b[:, 1])
        np.testing.assert_array_equal(a[:, 3], b[:, 3])
        assert (b[:, 2] == 0).all()
        for (p0, _, dl, _), p1 in zip(a.tolist(), b[:, 0].tolist()):
            assert kc[p1] == (p0, dl), f"table {t}: K page {p1} holds {kc[p1]}, want {(p0, dl)}"
            assert vc[p1] == p0, f"table {t}: V page {p1}"
            read.add(p1)
    # no job writes a page that attention never reads
    assert set(dst_k) <= read and set(dst_v) <= read
    return plan


@pytest.mark.parametrize("seed", range(40))
def test_reference_plan_random_tiny(seed):
    """The Python restatement on the oracle's page tables of tiny layouts
    (page sizes 1-4, below the library's)."""
    lay = synth.random_tiny(np.random.default_rng(1000 + seed))
    _check(lay, relocation_plan(lay, oracle.page_tables(lay)[0]))


def _same_plan(a, b):
    np.testing.assert_array_equal(a.jobs_k, b.jobs_k)
    np.testing.assert_array_equal(a.jobs_v, b.jobs_v)
    np.testing.assert_array_equal(a.layout.segments, b.layout.segments)
    np.testing.assert_array_equal(a.layout.page_base, b.layout.page_base)
    assert a.n_extra == b.n_extra and a.layout.n_pages == b.layout.n_pages


@pytest.mark.parametrize("seed", range(40))
def test_library_plan_random_small(seed):
    """rk_relocation_plan on random layouts of the library's page sizes:
    the symbolic pool check, and the same jobs as the Python restatement."""
    lay = synth.random_small(np.random.default_rng(2000 + seed), max_pages=16)
    plan = _check(lay)
    _same_plan(plan, relocation_plan(lay, oracle.page_tables(lay)[0]))


def test_plan_some_random_layout_needs_appended_pages():
    # shared contents reused at two offsets must occur in the random family
    extra = sum(binding.relocation_plan(
        synth.random_small(np.random.default_rng(2000 + s), max_pages=16)).n_extra for s in range(40))
    assert extra > 0


@pytest.mark.parametrize("name", ["cfg2", "cfg3", "cfg4", "cfg5"])
def test_library_plan_full_size_matches_reference(name):
    lay = synth.CONFIGS[name]().layout
    _same_plan(binding.relocation_plan(lay),
               relocation_plan(lay, oracle.page_tables_closed_form(lay)[0]))


def test_plan_cfg1():
    plan = _check(synth.cfg1().layout)
    # kv head 0 (global) sees all 3 x 8 cached pages; kv head 1 (window 128)
    # sees the 8 pages of the last cached segment; the first segment has delta 0
    assert plan.jobs_k.shape[0] == 16 + 8 and plan.n_extra == 0


def test_plan_cfg3_duplicate_content():
    lay = synth.cfg3().layout
    plan = _check(lay)
    # the duplicated content is seen at two offsets by the global head
    assert plan.n_extra > 0 and plan.jobs_v.shape[0] > 0


def test_visible_pages_cfg2_counts():
    lay = synth.cfg2().layout
    entries, _ = oracle.page_tables_closed_form(lay)
    need = visible_pages(lay, entries)
    g_pages = sum(len(v) for (s, lh), v in need.items() if lh == 0 and lay.segments[s, 4])
    l_pages = sum(len(v) for (s, lh), v in need.items() if lh > 0 and lay.segments[s, 4])
    assert g_pages == 7 * 64          # the global head reads every cached page
    assert l_pages == 7 * 64          # each local head: the last cached segment (window 4096)


def test_scoring_bytes_by_hand():
    """One retrieval table: 2 cached segments of 2 pages (P 8, D 16) and a
    10-token tail, 2 q heads: 10 rows x 2 heads of queries and 32 cached
    keys, 2 bytes each, times D; other classes read nothing."""
    from head_aware_paged_prefill_b200 import metrics
    segs = [("a", 16, 3, True), ("b", 16, 9, True), ("t", 10, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=4, hkv=2, d=16, p=8, theta=1e4, requests=[segs],
                             class_map=[synth.RETRIEVAL, synth.GLOBAL], window=8, retrieval={})
    assert metrics.scoring_bytes(lay) == 2 * 16 * (2 * 10 + 32)


def test_decode_bytes_by_hand():
    """One request of 40 tokens (2 cached pages of 8 + a 24-token tail), P 8,
    D 16, 2 q heads per kv head: a global head reads 40 keys, a local head
    (W 8) 8, a retrieval head the tail (24) plus its listed cached page (8);
    K and V, 2 bytes each, plus the queries and outputs of 6 rows."""
    from head_aware_paged_prefill_b200 import metrics
    segs = [("a", 16, 3, True), ("t", 24, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=6, hkv=3, d=16, p=8, theta=1e4, requests=[segs],
                             class_map=[synth.GLOBAL, synth.LOCAL, synth.RETRIEVAL], window=8,
                             retrieval={2: [1]})
    keys = 40 + 8 + (24 + 8)
    assert metrics.decode_bytes(lay) == 2 * 16 * 2 * keys + 2 * 2 * 16 * 6
    rep = synth.replicate_requests(lay, 3)
    assert rep.n_req == 3 and rep.n_pages == 3 * lay.n_pages and rep.total_tokens == 120
    assert metrics.decode_bytes(rep) == 3 * metrics.decode_bytes(lay)
