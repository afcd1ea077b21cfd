"""Pins of the oracle's token importance (``ora_importance``) and token
selection (``select_tokens``).

The RedKnot pages send the tokens with the highest attention scores through
the dense FFN (README "About", Elastic Sparsity / Sparse FFN; paooo page,
"main functions"), and print no worked example.  The pins are:
* an independent dense restatement (complex-number RoPE, explicit per-class
  masks, torch softmax in fp64, column sums);
* the invariant that each computed row's weights sum to one;
* a closed form (zero keys: harmonic sums);
* brute force for the selection rule.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import synth
from test_oracle_pins import _dense_kv, _retrieval_layout, _u16

GLOBAL, LOCAL, RETRIEVAL, DENSE = 0, 1, 2, 3


def _uncached(lay, r):
    unc = np.zeros(lay.req_len(r), dtype=bool)
    for seg in lay.segments:
        if int(seg[0]) == r and int(seg[4]) == 0:
            unc[int(seg[1]):int(seg[1]) + int(seg[2])] = True
    return unc


def _mask(lay, r, layer, kvh):
    """[L, L] visibility of key j to row i under the class rules, restated
    from the definitions (rows outside the table's row set see nothing)."""
    L, P = lay.req_len(r), lay.p
    unc = _uncached(lay, r)
    c = int(lay.class_map[layer * lay.hkv + kvh])
    rows = np.ones(L, dtype=bool) if c in (GLOBAL, DENSE) else unc
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    m = j <= i
    if c == LOCAL:
        m = m & (j > i - int(lay.class_window[LOCAL]))
    if c == RETRIEVAL:
        t = lay.table_index(r, layer, kvh)
        listed = {int(pg) for pg in lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]]
                  if 0 <= pg < -(-L // P) and not unc[int(pg) * P]}
        key_ok = unc | np.isin(np.arange(L) // P, sorted(listed))
        m = m & key_ok[None, :]
    return m & rows[:, None]


def _dense_importance(lay, q, k_pool, v_pool):
    """[n_layers][T]: column sums of the masked fp64 softmax, per table and
    q head, added over the layer's heads."""
    T = int(lay.cu_seqlens[-1])
    g = lay.hq // lay.hkv
    out = np.zeros((lay.n_layers, T))
    for r in range(lay.n_req):
        L = lay.req_len(r)
        if L == 0:
            continue
        t0 = int(lay.cu_seqlens[r])
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                K, _ = _dense_kv(lay, k_pool, v_pool, r, layer, kvh)
                m = _mask(lay, r, layer, kvh)
                live = m.any(axis=1)
                for h in range(kvh * g, kvh * g + g):
                    qd = q[layer, t0:t0 + L, h].double().numpy()
                    s = torch.from_numpy((qd @ K.T) * lay.softmax_scale)
                    s[~torch.from_numpy(m)] = -math.inf
                    p = torch.softmax(s[torch.from_numpy(live)], dim=1)
                    out[layer, t0:t0 + L] += p.sum(dim=0).numpy()
    return out


def _check_dense(wl):
    lay = wl.layout
    q, k, v = wl.materialize("cpu")
    got = oracle.importance(lay, _u16(q), _u16(k))
    want = _dense_importance(lay, q, k, v)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10)
    return lay, got


def test_importance_is_dense_softmax_column_sums_cfg1():
    _check_dense(synth.cfg1())


def test_importance_is_dense_softmax_column_sums_retrieval():
    _check_dense(_retrieval_layout())


def test_importance_is_dense_softmax_column_sums_random():
    rng = np.random.default_rng(17)
    for n in range(6):
        lay = synth.random_small(rng, max_pages=10)
        _check_dense(synth.tiny_workload(lay, seed=100 + n))


def test_importance_sums_to_computed_rows():
    """Every computed (q head, row) pair spreads a total weight of one."""
    rng = np.random.default_rng(23)
    for n in range(4):
        lay = synth.random_small(rng, max_pages=10)
        wl = synth.tiny_workload(lay, seed=200 + n)
        q, k, _ = wl.materialize("cpu")
        imp = oracle.importance(lay, _u16(q), _u16(k))
        g = lay.hq // lay.hkv
        for r in range(lay.n_req):
            L = lay.req_len(r)
            t0 = int(lay.cu_seqlens[r])
            n_unc = int(_uncached(lay, r).sum())
            for layer in range(lay.n_layers):
                rows = 0
                for kvh in range(lay.hkv):
                    c = int(lay.class_map[layer * lay.hkv + kvh])
                    rows += g * (L if c in (GLOBAL, DENSE) else n_unc)
                assert imp[layer, t0:t0 + L].sum() == pytest.approx(rows, rel=1e-12, abs=1e-12)
                assert (imp[layer, t0:t0 + L] >= 0).all()


def test_zero_keys_give_harmonic_sums():
    """K = 0: every visible key of row i weighs 1 / (i + 1) on a global head,
    so I(j) = Hq * (H_L - H_j) with H_n the n-th harmonic number."""
    segs = [("doc", 40, 11, True), ("tail", 24, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=4, hkv=2, d=16, p=8, theta=1e4, requests=[segs],
                             class_map=[GLOBAL, DENSE], window=0)
    wl = synth.tiny_workload(lay, seed=9)
    q, k, _ = wl.materialize("cpu")
    imp = oracle.importance(lay, _u16(q), _u16(torch.zeros_like(k)))
    L = lay.req_len(0)
    harm = np.concatenate([[0.0], np.cumsum(1.0 / np.arange(1, L + 1))])
    want = lay.hq * (harm[L] - harm[np.arange(L)])
    np.testing.assert_allclose(imp[0], want, rtol=1e-12, atol=1e-12)


def test_select_tokens_by_hand():
    imp = [1.0, 3.0, 3.0, 2.0, 3.0, 0.5]
    assert oracle.select_tokens(imp, 2).tolist() == [1, 2]  # ties to the lower position
    assert oracle.select_tokens(imp, 4).tolist() == [1, 2, 3, 4]
    assert oracle.select_tokens(imp, 10).tolist() == [0, 1, 2, 3, 4, 5]
    assert oracle.select_tokens(imp, 0).tolist() == []
    assert oracle.select_tokens([], 3).tolist() == []


def test_select_tokens_brute_force():
    """Against the threshold rule: everything above the k-th value, then the
    lowest positions among the values equal to it."""
    rng = np.random.default_rng(3)
    for _ in range(300):
        n = int(rng.integers(0, 40))
        imp = rng.integers(0, 6, size=n).astype(float)
        k = int(rng.integers(0, n + 3))
        if k >= n:
            want = list(range(n))
        elif k == 0:
            want = []
        else:
            kth = sorted(imp, reverse=True)[k - 1]
            above = [j for j in range(n) if imp[j] > kth]
            ties = [j for j in range(n) if imp[j] == kth][:k - len(above)]
            want = sorted(above + ties)
        assert oracle.select_tokens(imp, k).tolist() == want
