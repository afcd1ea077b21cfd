"""Pins of the oracle's retrieval page scoring (``oracle.score_pages``).

The RedKnot pages say retrieval heads choose their cached pages "by query
semantics" (paooo page, "how to use" section, SELECTVISIBLESTATE) and give
no rule, so the oracle implements a stated reading: page summary = mean of
the page's relocated keys, query summary = sum over the kv head's q heads of
the mean query over the table's rows, score = their dot product, top-k with
ties to the lower page index.  These pins restate that reading by other
routes, independent of the oracle's code:

* the score is the bilinear mean of q . k' over (q head, row, page row),
  evaluated term by term with complex-number RoPE;
* planted pages (keys aligned with the query summary) win;
* top-k covers all candidates when there are few, and ties go to the lower
  page index;
* non-retrieval tables, tables without rows and uncached pages get nothing;
* swapping two tail rows leaves the scores unchanged (a mean).
"""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import synth
from test_oracle_pins import _complex_rope, _u16


def _layout(n_cached=6, p=8, d=16, g=2, hkv=2, tail=20, cmap=None, theta=1e4, stored=None):
    stored = stored or [5 * i + 3 for i in range(n_cached)]
    segs = [(f"c{i}", 2 * p, stored[i], True) for i in range(n_cached)]
    segs.append(("tail", tail, 0, False))
    cmap = cmap if cmap is not None else [synth.RETRIEVAL] + [synth.GLOBAL] * (hkv - 1)
    return synth._make_layout(n_layers=1, hq=hkv * g, hkv=hkv, d=d, p=p, theta=theta,
                              requests=[segs], class_map=cmap, window=p, retrieval={})


def _scores_by_expansion(lay, q, k_pool, r, layer, kvh):
    """score_pg = mean over (row i, page row) of sum over q heads of
    q_{h,i} . R(delta) k: the bilinear form expanded term by term."""
    P, d = lay.p, lay.d
    g = lay.hq // lay.hkv
    L = lay.req_len(r)
    t0 = int(lay.cu_seqlens[r])
    unc = np.zeros(L, dtype=bool)
    seg_of = np.full(L, -1)
    for s, seg in enumerate(lay.segments):
        if seg[0] != r:
            continue
        seg_of[seg[1]:seg[1] + seg[2]] = s
        if not seg[4]:
            unc[seg[1]:seg[1] + seg[2]] = True
    rows = np.nonzero(unc)[0]
    qf = q.double().numpy()
    kf = k_pool.double().numpy()
    out = {}
    for pg in range(-(-L // P)):
        j0 = pg * P
        if unc[j0] or j0 > rows.max():
            continue
        s = seg_of[j0]
        seg = lay.segments[s]
        delta = float(seg[1] - seg[3])
        nv = min(P, L - j0)
        base = int(lay.page_base[s, layer * lay.hkv + kvh])
        acc = 0.0
        for rr in range(nv):
            off = j0 + rr - int(seg[1])
            kr = _complex_rope(kf[base + off // P, off % P], lay.theta, np.asarray(delta))
            for h in range(kvh * g, kvh * g + g):
                for i in rows:
                    acc += float(qf[layer, t0 + i, h] @ kr)
        out[pg] = acc / (nv * len(rows))
    return out


def test_scores_equal_bilinear_expansion():
    lay = _layout(n_cached=5, tail=13, theta=1e4)
    wl = synth.tiny_workload(lay, seed=4)
    q, k_pool, _ = wl.materialize("cpu")
    picks, scores = oracle.score_pages(lay, _u16(q), _u16(k_pool), top_k=3)
    want = _scores_by_expansion(lay, q, k_pool, 0, 0, 0)
    got = {pg: scores[0][pg] for pg in range(scores[0].shape[0]) if not np.isnan(scores[0][pg])}
    assert set(got) == set(want)
    for pg in want:
        assert abs(got[pg] - want[pg]) <= 1e-10 * (1 + abs(want[pg])), pg
    order = sorted(want, key=lambda pg: (-want[pg], pg))
    np.testing.assert_array_equal(picks[0], np.sort(order[:3]))


def test_planted_pages_win():
    """Pages whose relocated keys point along the query summary win (their
    stored keys are that direction rotated back by the page's delta)."""
    lay = _layout(n_cached=6, tail=16, d=16, theta=100.0, stored=[0, 40, 80, 120, 160, 200])
    wl = synth.tiny_workload(lay, seed=9)
    q, k_pool, _ = wl.materialize("cpu")
    g = lay.hq // lay.hkv
    t0, L = 0, lay.req_len(0)
    tail = slice(L - 16, L)
    u = q[0, tail, 0:g].double().mean(dim=0).sum(dim=0).numpy()
    planted = [3, 8]  # pages 3 and 8: segments 1 and 4 (2 pages per segment)
    kp = k_pool.clone()
    for pg in planted:
        s = pg // 2
        seg = lay.segments[s]
        delta = float(seg[1] - seg[3])
        base = int(lay.page_base[s, 0])
        stored = _complex_rope(5.0 * u / np.linalg.norm(u), lay.theta, np.asarray(-delta))
        kp[base + pg % 2] = torch.from_numpy(np.tile(stored, (lay.p, 1))).to(torch.bfloat16)
    picks, _ = oracle.score_pages(lay, _u16(q), _u16(kp), top_k=2)
    np.testing.assert_array_equal(picks[0], planted)


def test_few_candidates_all_picked_and_other_tables_empty():
    lay = _layout(n_cached=3, tail=9, hkv=3, cmap=[synth.RETRIEVAL, synth.LOCAL, synth.GLOBAL])
    wl = synth.tiny_workload(lay, seed=1)
    q, k_pool, _ = wl.materialize("cpu")
    picks, scores = oracle.score_pages(lay, _u16(q), _u16(k_pool), top_k=16)
    np.testing.assert_array_equal(picks[0], np.arange(6))  # 3 cached segments x 2 pages
    assert picks[1].size == 0 and picks[2].size == 0
    assert np.isnan(scores[1]).all() and np.isnan(scores[2]).all()
    assert np.isnan(scores[0][6:]).all()  # the uncached tail pages are not candidates


def test_ties_go_to_the_lower_page():
    """Two pages of one segment (same delta) with identical keys pointing
    along the query summary tie for first: top-1 is the lower one, top-2
    both."""
    lay = _layout(n_cached=3, tail=8, stored=[0, 7, 21])
    wl = synth.tiny_workload(lay, seed=2)
    q, k_pool, _ = wl.materialize("cpu")
    g = lay.hq // lay.hkv
    L = lay.req_len(0)
    u = q[0, L - 8:L, 0:g].double().mean(dim=0).sum(dim=0).numpy()
    seg = lay.segments[1]  # pages 2 and 3
    delta = float(seg[1] - seg[3])
    base = int(lay.page_base[1, 0])
    stored = _complex_rope(4.0 * u / np.linalg.norm(u), lay.theta, np.asarray(-delta))
    kp = k_pool.clone()
    kp[base] = torch.from_numpy(np.tile(stored, (lay.p, 1))).to(torch.bfloat16)
    kp[base + 1] = kp[base]
    picks, scores = oracle.score_pages(lay, _u16(q), _u16(kp), top_k=1)
    assert scores[0][2] == scores[0][3] and scores[0][2] == np.nanmax(scores[0])
    np.testing.assert_array_equal(picks[0], [2])
    picks2, _ = oracle.score_pages(lay, _u16(q), _u16(kp), top_k=2)
    np.testing.assert_array_equal(picks2[0], [2, 3])


def test_no_rows_no_picks():
    """A request whose positions are all cached has no rows: no picks."""
    segs = [("a", 16, 3, True), ("b", 16, 9, True)]
    lay = synth._make_layout(n_layers=1, hq=2, hkv=1, d=16, p=8, theta=1e4, requests=[segs],
                             class_map=[synth.RETRIEVAL], window=8, retrieval={})
    wl = synth.tiny_workload(lay, seed=1)
    q, k, _ = wl.materialize("cpu")
    picks, scores = oracle.score_pages(lay, _u16(q), _u16(k))
    assert picks[0].size == 0 and np.isnan(scores[0]).all()


def test_tail_row_order_does_not_matter():
    """The query summary is a mean: swapping two tail rows' queries (of every
    head) leaves the scores unchanged up to rounding."""
    lay = _layout(n_cached=4, tail=12)
    wl = synth.tiny_workload(lay, seed=6)
    q, k_pool, _ = wl.materialize("cpu")
    _, scores = oracle.score_pages(lay, _u16(q), _u16(k_pool), top_k=16)
    L = lay.req_len(0)
    q2 = q.clone()
    q2[0, L - 1], q2[0, L - 5] = q[0, L - 5].clone(), q[0, L - 1].clone()
    _, scores2 = oracle.score_pages(lay, _u16(q2), _u16(k_pool), top_k=16)
    np.testing.assert_allclose(scores2[0], scores[0], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["cfg4", "cfg5"])
def test_workload_picks_are_top_scores(name):
    """On the workloads with retrieval heads: each retrieval table picks
    min(16, candidates) pages, and they are the highest-scoring ones."""
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    if lay.total_tokens * lay.hq * lay.d * lay.n_layers > 4e8:
        pytest.skip("values of this workload are drawn on the GPU")
    q, k_pool, _ = wl.materialize("cpu")
    picks, scores = oracle.score_pages(lay, _u16(q), _u16(k_pool))
    n_retr = 0
    for t in range(lay.n_tables):
        sc = scores[t]
        cand = np.nonzero(~np.isnan(sc))[0]
        if cand.size == 0:
            assert picks[t].size == 0
            continue
        n_retr += 1
        assert picks[t].size == min(16, cand.size)
        order = sorted(cand, key=lambda pg: (-sc[pg], pg))
        np.testing.assert_array_equal(picks[t], np.sort(order[:picks[t].size]))
    assert n_retr > 0
