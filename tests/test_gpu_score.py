"""rk_score_retrieval_pages (retrieval page scoring) against the fp64 oracle.

Scores are compared element by element.  The picks are compared as sets when
the oracle's scores separate the k-th and (k+1)-th candidates by more than
the fp32 tolerance.  Otherwise either order is correct, and the picks are
checked to be valid: no pick scores clearly below a non-pick."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from gpu_util import u16

pytestmark = pytest.mark.gpu


def _run(lay, q, k, top_k):
    hl = binding.HostLayout(lay)
    sizes = binding.score_sizes(hl, top_k)
    out = binding.ScoreOutputs(sizes, top_k, "cuda")
    binding.score_retrieval_pages(hl, q, k, lay.theta, out)
    torch.cuda.synchronize()
    return out


def _check(lay, q, k, top_k=16, what=""):
    out = _run(lay, q.cuda(), k.cuda(), top_k)
    picks_ref, scores_ref = oracle.score_pages(lay, u16(q), u16(k), top_k)
    count = out.count.cpu().numpy()
    pages = out.pages.cpu().numpy()
    scores = out.scores.cpu().numpy()
    n_checked = 0
    for t in range(lay.n_tables):
        ref = scores_ref[t]
        got = scores[t, :ref.shape[0]]
        assert np.array_equal(np.isnan(got), np.isnan(ref)), f"{what} table {t}: candidates"
        assert np.isnan(scores[t, ref.shape[0]:]).all()
        cand = np.nonzero(~np.isnan(ref))[0]
        if cand.size == 0:
            assert count[t] == 0
            continue
        scale = np.abs(ref[cand]).max() + 1e-30
        tol = 1e-4 * scale
        err = np.abs(got[cand] - ref[cand]).max()
        assert err <= tol, f"{what} table {t}: score error {err:.3e} > {tol:.3e}"
        n = min(top_k, cand.size)
        assert count[t] == n, f"{what} table {t}: {count[t]} picks, want {n}"
        mine = np.sort(pages[t, :n])
        assert np.all(np.diff(pages[t, :n]) > 0), "picks in ascending page order"
        order = sorted(cand, key=lambda pg: (-ref[pg], pg))
        if n < cand.size and ref[order[n - 1]] - ref[order[n]] <= 2 * tol:
            kth = ref[order[n - 1]]
            assert np.all(ref[mine] >= kth - 2 * tol)
            rest = np.setdiff1d(cand, mine)
            assert np.all(ref[rest] <= kth + 2 * tol)
        else:
            np.testing.assert_array_equal(mine, picks_ref[t], err_msg=f"{what} table {t}")
        n_checked += 1
    return n_checked


def test_score_cfg4():
    wl = synth.cfg4()
    q, k, _ = wl.materialize("cuda")
    assert _check(wl.layout, q, k, 16, "cfg4") == 1


def test_score_many_retrieval_heads():
    """The 32K layer with every kv head a retrieval head (8 tables of 448
    candidate pages), top 16 and top 64."""
    base = synth.cfg2().layout
    lay = synth.with_classes(base, [synth.RETRIEVAL] * base.hkv)
    wl = synth.tiny_workload(lay, seed=21)
    q, k, _ = wl.materialize("cuda")
    assert _check(lay, q, k, 16, "all-retrieval") == base.hkv
    assert _check(lay, q, k, 64, "all-retrieval top 64") == base.hkv


@pytest.mark.parametrize("top_k", [1, 3, 16])
def test_score_random_small(top_k):
    rng = np.random.default_rng(55)
    checked = 0
    for n in range(30):
        lay = synth.random_small(rng, max_pages=24)
        wl = synth.tiny_workload(lay, seed=n)
        q, k, _ = wl.materialize("cpu")
        checked += _check(lay, q, k, top_k, f"random layout {n}")
    assert checked > 0


def test_score_is_deterministic():
    wl = synth.cfg4()
    q, k, _ = wl.materialize("cuda")
    a = _run(wl.layout, q, k, 16)
    b = _run(wl.layout, q, k, 16)
    assert torch.equal(a.pages, b.pages) and torch.equal(a.count, b.count)
    assert torch.equal(a.scores.view(torch.int32), b.scores.view(torch.int32))


def test_scored_lists_drive_attention():
    """End to end: the device picks become the layout's retrieval lists, and
    attention over that layout (select, relocation, attention) matches the
    oracle on the same layout (sampled rows of the retrieval head)."""
    from head_aware_paged_prefill_b200.api import SegPagedPrefill, score_retrieval
    from gpu_util import assert_close, oracle_rows
    wl = synth.cfg4()
    q, k, v = wl.materialize("cuda")
    lay, out = score_retrieval(wl.layout, q, k, top_k=16)
    t = lay.table_index(0, 0, 1)  # kv head 1 is the retrieval head
    picks_ref, _ = oracle.score_pages(wl.layout, u16(q), u16(k), 16)
    assert lay.retr_indptr[t + 1] - lay.retr_indptr[t] == 16
    np.testing.assert_array_equal(lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]],
                                  picks_ref[t])
    pre = SegPagedPrefill(lay, "cuda")
    o = pre.run(q, k, v)
    torch.cuda.synchronize()
    assert pre.status() == 0
    g = lay.hq // lay.hkv
    L = lay.req_len(0)
    rng = np.random.default_rng(3)
    rows = np.array([(0, h, int(i)) for h in range(g, 2 * g)
                     for i in rng.integers(L - 2048, L, 12)], dtype=np.int32)
    o_ref, _, comp = oracle_rows(lay, q.cpu(), k.cpu(), v.cpu(), rows)
    assert comp.all()
    idx = [torch.from_numpy(rows[:, c]).long().cuda() for c in (0, 2, 1)]
    got = o[idx[0], idx[1], idx[2]].double().cpu().numpy()
    assert_close(got, o_ref, "scored retrieval o")


def _retrieval_layout(seg_len, n_seg, tail, p=16, hq=2, hkv=1, d=64):
    segs = [(f"c{i}", seg_len, 0, True) for i in range(n_seg)] + [("tail", tail, 0, False)]
    return synth._make_layout(n_layers=1, hq=hq, hkv=hkv, d=d, p=p, theta=1e4, requests=[segs],
                              class_map=[synth.RETRIEVAL] * hkv, window=0)


@pytest.mark.parametrize("top_k", [1, 7, 64])
def test_score_ties_go_to_the_lower_pages(top_k):
    """Zero queries make every candidate's score exactly zero: the picks are
    then decided by the page alone (ties to the lower page), so every byte
    of the (score, page) key takes part in the selection."""
    lay = _retrieval_layout(1024, 3, 64, hkv=2, hq=4)
    q, k, _ = synth.tiny_workload(lay, seed=31).materialize("cuda")
    q.zero_()
    out = _run(lay, q, k, top_k)
    for t in range(lay.n_tables):
        assert out.count[t].item() == top_k
        assert out.pages[t, :top_k].cpu().numpy().tolist() == list(range(top_k))
        assert (out.scores[t, :192] == 0).all()


@pytest.mark.parametrize("n_seg,top_k", [(9, 16), (16, 64)])
def test_score_thousands_of_candidates(n_seg, top_k):
    """2304 and 4096 (the most a table takes) candidate pages of 16 keys."""
    lay = _retrieval_layout(4096, n_seg, 128)
    wl = synth.tiny_workload(lay, seed=32 + n_seg)
    q, k, _ = wl.materialize("cpu")
    assert _check(lay, q, k, top_k, f"{n_seg * 256} candidates") == 1
