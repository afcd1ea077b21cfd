"""Pins of the fp64 oracle against facts fixed outside of it.

The RedKnot pages print no worked numeric example, so every pin here is a
closed form, a textbook special case computed by an independent routine
(numpy complex arithmetic, torch SDPA in fp64), an invariance, or brute force
on tiny inputs:

* RoPE relocation "guarantees numerical alignment" (README excerpt, "Offline
  KV Reuse + RoPE Relocation"): R(delta) R(p) x = R(p + delta) x.
* The paged, mask-free kernel must equal dense attention with a mask (paooo
  page, "paged storage removes the mask penalty"): global heads reduce to
  causal attention, local heads to a sliding-window mask, retrieval heads to
  a union mask.
* Global heads recompute everything, local heads see only their window
  (paooo page, "how to use", EXECUTE step): perturbations outside the window
  leave a row bit-unchanged.
* Position-independent reuse (paooo page, main features): a segment shared
  through the same physical pages equals the same segment copied twice.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import synth

# ----------------------------------------------------------------- helpers


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _complex_rope(x: np.ndarray, theta: float, pos: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE as complex multiplication: (x_m + i x_{m+D/2}) e^{i pos f_m}."""
    d = x.shape[-1]
    h = d // 2
    f = theta ** (-2.0 * np.arange(h) / d)
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * np.multiply.outer(pos, f))
    return np.concatenate([z.real, z.imag], axis=-1)


def _dense_kv(lay, k_pool, v_pool, r, layer, kvh):
    """Dense [L, D] relocated K (complex-number RoPE) and V of one table,
    assembled from the layout without any oracle routine."""
    L = lay.req_len(r)
    P = lay.p
    kf = k_pool.double().numpy()
    vf = v_pool.double().numpy()
    K = np.zeros((L, lay.d))
    V = np.zeros((L, lay.d))
    for s, seg in enumerate(lay.segments):
        if seg[0] != r:
            continue
        base = int(lay.page_base[s, layer * lay.hkv + kvh])
        for off in range(int(seg[2])):
            j = int(seg[1]) + off
            page, row = base + off // P, off % P
            delta = int(seg[1]) - int(seg[3])
            K[j] = _complex_rope(kf[page, row], lay.theta, np.asarray(delta, dtype=np.float64))
            V[j] = vf[page, row]
    return K, V


def _oracle_rows(lay, q, k_pool, v_pool, rows):
    rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
    qr = torch.stack([q[int(l), int(t), int(h)] for l, h, t in rows])
    return oracle.attention(lay, _u16(qr), _u16(k_pool), _u16(v_pool), rows)


def _sdpa(qd, K, V, mask, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qd)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        attn_mask=torch.from_numpy(mask)[None], scale=scale)
    return out[0].numpy()


# ---------------------------------------------------------------- P1 RoPE

@pytest.mark.parametrize("d", [2, 4, 64, 128])
def test_rope_matches_complex_rotation(d):
    rng = np.random.default_rng(d)
    for theta in (1e4, 1e6, 100.0):
        for pos in (0.0, 1.0, -3.0, 127.0, 4096.0, -30720.0, 65535.0):
            x = rng.standard_normal(d)
            y = oracle.rope_rotate(x, theta, pos)
            np.testing.assert_allclose(y, _complex_rope(x, theta, np.asarray(pos)),
                                       rtol=0, atol=1e-9)


def test_rope_quarter_turn_by_hand():
    # D = 2: one pair with frequency 1; a quarter turn maps (1, 0) to (0, 1)
    y = oracle.rope_rotate([1.0, 0.0], 1e4, math.pi / 2)
    np.testing.assert_allclose(y, [0.0, 1.0], atol=1e-15)
    # D = 4, theta = 1e4: frequencies 1 and 1e-2 on pairs (0, 2) and (1, 3)
    x = [1.0, 2.0, 3.0, 4.0]
    y = oracle.rope_rotate(x, 1e4, 1.0)
    c1, s1, c2, s2 = math.cos(1.0), math.sin(1.0), math.cos(0.01), math.sin(0.01)
    np.testing.assert_allclose(
        y, [1 * c1 - 3 * s1, 2 * c2 - 4 * s2, 1 * s1 + 3 * c1, 2 * s2 + 4 * c2], atol=1e-14)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_composition(d):
    rng = np.random.default_rng(7 + d)
    for _ in range(50):
        x = rng.standard_normal(d)
        p = float(rng.integers(0, 65536))
        delta = float(rng.integers(-65536, 65536))
        a = oracle.rope_rotate(oracle.rope_rotate(x, 1e6, p), 1e6, delta)
        b = oracle.rope_rotate(x, 1e6, p + delta)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)
        assert np.linalg.norm(a) == pytest.approx(np.linalg.norm(x), rel=1e-12)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_relocation_after_bf16_storage(d):
    """Stored keys are bf16(R(p) x); relocating them by delta stays within the
    bf16 rounding bound of R(p + delta) x."""
    rng = np.random.default_rng(11 + d)
    for _ in range(50):
        x = rng.standard_normal(d)
        p = float(rng.integers(0, 4096))
        delta = float(rng.integers(-32768, 32768))
        stored = torch.tensor(oracle.rope_rotate(x, 1e6, p)).to(torch.bfloat16).double().numpy()
        got = oracle.rope_rotate(stored, 1e6, delta)
        want = oracle.rope_rotate(x, 1e6, p + delta)
        bound = 2.0 ** -8 * np.abs(oracle.rope_rotate(x, 1e6, p)).max() * math.sqrt(2)
        assert np.abs(got - want).max() <= bound


def test_relocate_matches_rotation_per_row():
    lay = synth.cfg1().layout
    _, k_pool, _ = synth.cfg1().materialize("cpu")
    jobs = np.asarray([[0, 0, 128], [5, 5, -37], [9, 9, 0]], dtype=np.int32)
    out = oracle.relocate(_u16(k_pool), jobs, lay.p, lay.d, lay.theta)
    for n, (src, _, delta) in enumerate(jobs):
        want = _complex_rope(k_pool[src].double().numpy(), lay.theta,
                             np.full(lay.p, float(delta)))
        np.testing.assert_allclose(out[n], want, rtol=0, atol=1e-9)
    np.testing.assert_array_equal(out[2], k_pool[9].double().numpy())


# -------------------------------------------- P2-P4 special cases via SDPA

def _check_table_against_sdpa(lay, q, k_pool, v_pool, r, layer, kvh, mask_fn):
    L = lay.req_len(r)
    K, V = _dense_kv(lay, k_pool, v_pool, r, layer, kvh)
    g = lay.hq // lay.hkv
    t0 = int(lay.cu_seqlens[r])
    for h in range(kvh * g, kvh * g + g):
        rows_i = [i for i in range(L) if mask_fn(i, 0) is not None]
        mask = np.zeros((len(rows_i), L), dtype=bool)
        for a, i in enumerate(rows_i):
            mask[a] = [mask_fn(i, j) for j in range(L)]
        qd = q[layer, t0 + np.asarray(rows_i), h].double().numpy()
        want = _sdpa(qd, K, V, mask, lay.softmax_scale)
        o, lse, comp = _oracle_rows(lay, q, k_pool, v_pool,
                                    [(layer, h, t0 + i) for i in rows_i])
        assert comp.all()
        np.testing.assert_allclose(o, want, rtol=0, atol=1e-10)
        s = (qd @ K.T) * lay.softmax_scale
        s[~mask] = -np.inf
        m = s.max(axis=1)
        np.testing.assert_allclose(lse, m + np.log(np.exp(s - m[:, None]).sum(axis=1)),
                                   rtol=0, atol=1e-10)


def test_global_head_is_causal_attention():
    wl = synth.cfg1()
    lay = wl.layout
    q, k_pool, v_pool = wl.materialize("cpu")
    _check_table_against_sdpa(lay, q, k_pool, v_pool, 0, 0, 0, lambda i, j: j <= i)


def test_local_head_is_sliding_window():
    wl = synth.cfg1()
    lay = wl.layout
    q, k_pool, v_pool = wl.materialize("cpu")
    W = 128

    def mask_fn(i, j):
        if i < 384:
            return None  # not a row of the local table
        return i - W < j <= i

    _check_table_against_sdpa(lay, q, k_pool, v_pool, 0, 0, 1, mask_fn)


def _retrieval_layout():
    segs = [(f"c{i}", 32, 7 * i, True) for i in range(4)] + [("tail", 20, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=2, hkv=1, d=16, p=8, theta=1e4, requests=[segs],
                             class_map=[synth.RETRIEVAL], window=0,
                             retrieval={0: [1, 6, 9, 15, 17]})
    return synth.tiny_workload(lay, seed=3)


def test_retrieval_head_is_union_mask():
    wl = _retrieval_layout()
    lay = wl.layout
    q, k_pool, v_pool = wl.materialize("cpu")
    sel = {1, 6, 9, 15}  # page 17 is in the uncached tail: visible anyway

    def mask_fn(i, j):
        if i < 128:
            return None
        return j <= i and (j >= 128 or (j // 8) in sel)

    _check_table_against_sdpa(lay, q, k_pool, v_pool, 0, 0, 0, mask_fn)


def test_local_window_perturbation():
    """Changing K/V of a key outside (i - W, i] leaves o_i bit-unchanged;
    changing one inside changes it."""
    wl = synth.cfg1()
    lay = wl.layout
    q, k_pool, v_pool = wl.materialize("cpu")
    i, h, W = 400, 2, 128
    rows = [(0, h, i)]
    o0, _, _ = _oracle_rows(lay, q, k_pool, v_pool, rows)

    def page_row(j):  # kv head 1 of cfg1: find its page
        for s, seg in enumerate(lay.segments):
            if seg[1] <= j < seg[1] + seg[2]:
                off = j - int(seg[1])
                return int(lay.page_base[s, 1]) + off // lay.p, off % lay.p

    for j, inside in ((i - W, False), (10, False), (i - W + 1, True), (i, True), (i + 1, False)):
        pg, rw = page_row(j)
        k2, v2 = k_pool.clone(), v_pool.clone()
        k2[pg, rw] += 1.0
        v2[pg, rw] -= 2.0
        o1, _, _ = _oracle_rows(lay, q, k2, v2, rows)
        if inside:
            assert not np.array_equal(o0, o1), j
        else:
            np.testing.assert_array_equal(o0, o1)


# ------------------------------------------------------------- P5 sharing

def test_shared_pages_equal_private_copies():
    wl = synth.cfg3()
    lay = wl.layout
    # shrink cfg3's structure: keep its slot permutation, scale lengths down
    segs = []
    for s in lay.segments_of(0):
        segs.append((f"c{int(s[3]) // 2048}" if s[4] else "tail", 16, int(s[3]) // 128,
                     bool(s[4])))
    shared = synth._make_layout(n_layers=1, hq=4, hkv=2, d=16, p=4, theta=1e6,
                                requests=[segs], class_map=[synth.GLOBAL, synth.LOCAL], window=20)
    private_segs = [(f"{name}_{k}", ln, st, c) for k, (name, ln, st, c) in enumerate(segs)]
    private = synth._make_layout(n_layers=1, hq=4, hkv=2, d=16, p=4, theta=1e6,
                                 requests=[private_segs], class_map=[synth.GLOBAL, synth.LOCAL],
                                 window=20)
    assert private.n_pages > shared.n_pages  # the duplicate got its own pages
    q, k_sh, v_sh = synth.tiny_workload(shared, 5).materialize("cpu")
    # materialise the private pool by copying each instance's pages
    k_pr = torch.zeros((private.n_pages, 4, 16), dtype=torch.bfloat16)
    v_pr = torch.zeros_like(k_pr)
    for s in range(shared.segments.shape[0]):
        for lh in range(2):
            a, b = int(shared.page_base[s, lh]), int(private.page_base[s, lh])
            k_pr[b:b + 4] = k_sh[a:a + 4]
            v_pr[b:b + 4] = v_sh[a:a + 4]
    rows = [(0, h, t) for h in range(4) for t in range(shared.total_tokens)]
    o1, l1, c1 = _oracle_rows(shared, q, k_sh, v_sh, rows)
    o2, l2, c2 = _oracle_rows(private, q, k_pr, v_pr, rows)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_physical_page_permutation_invariance():
    wl = synth.cfg1()
    lay = wl.layout
    q, k_pool, v_pool = wl.materialize("cpu")
    # pages of one segment stay consecutive: permute whole segment blocks
    lay2 = synth.Layout(**{**lay.__dict__})
    blocks = []
    for s in range(lay.segments.shape[0]):
        for lh in range(lay.n_layers * lay.hkv):
            n = -(-int(lay.segments[s, 2]) // lay.p)
            blocks.append((s, lh, int(lay.page_base[s, lh]), n))
    order = np.random.default_rng(1).permutation(len(blocks))
    new_base = lay.page_base.copy()
    k2 = torch.empty_like(k_pool)
    v2 = torch.empty_like(v_pool)
    nxt = 0
    for b in order:
        s, lh, old, n = blocks[b]
        new_base[s, lh] = nxt
        k2[nxt:nxt + n] = k_pool[old:old + n]
        v2[nxt:nxt + n] = v_pool[old:old + n]
        nxt += n
    lay2.page_base = new_base
    rows = [(0, h, t) for h in range(lay.hq) for t in range(0, lay.total_tokens, 7)]
    o1, l1, _ = _oracle_rows(lay, q, k_pool, v_pool, rows)
    o2, l2, _ = _oracle_rows(lay2, q, k2, v2, rows)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ------------------------------------------------- P6 page tables, P7 pairs

def _assert_tables_equal(a, b):
    ea, ra = a
    eb, rb = b
    assert len(ea) == len(eb)
    for t in range(len(ea)):
        np.testing.assert_array_equal(ea[t], eb[t], err_msg=f"entries of table {t}")
        np.testing.assert_array_equal(ra[t], rb[t], err_msg=f"ranges of table {t}")


def test_page_tables_brute_force_vs_closed_form_random():
    rng = np.random.default_rng(2024)
    for _ in range(1000):
        lay = synth.random_tiny(rng)
        _assert_tables_equal(oracle.page_tables(lay, threads=1),
                             oracle.page_tables_closed_form(lay))
        assert oracle.visible_pairs(lay, threads=1) == oracle.visible_pairs_closed_form(lay)


@pytest.mark.parametrize("name", ["cfg1", "cfg2", "cfg3", "cfg4", "cfg5"])
def test_page_tables_brute_force_vs_closed_form_configs(name):
    lay = synth.CONFIGS[name]().layout
    _assert_tables_equal(oracle.page_tables(lay), oracle.page_tables_closed_form(lay))


def test_cfg1_page_table_by_hand():
    """cfg1: three cached segments stored at 0..127 placed at 0/128/256
    (deltas 0/128/256), 64-token tail; kv_head 0 global sees all 28 pages,
    kv_head 1 (window 128, rows 384..447) sees pages 16..27."""
    lay = synth.cfg1().layout
    ent, rng_ = oracle.page_tables(lay)
    e0, e1 = ent[0], ent[1]
    assert e0.shape == (28, 4) and e1.shape == (12, 4)
    np.testing.assert_array_equal(e0[:, 1], np.arange(28) * 16)
    np.testing.assert_array_equal(e0[:, 2], [0] * 8 + [128] * 8 + [256] * 8 + [0] * 4)
    np.testing.assert_array_equal(e0[:, 3], [16] * 28)
    np.testing.assert_array_equal(e1[:, 1], np.arange(16, 28) * 16)
    np.testing.assert_array_equal(rng_[0], [[0, 448]])
    np.testing.assert_array_equal(rng_[1], [[384, 448]])


PAIRS = {"cfg1": 217_536, "cfg2": 2_617_311_232, "cfg3": 4_529_979_392,
         "cfg4": 17_280_802_816}


@pytest.mark.parametrize("name", ["cfg1", "cfg2", "cfg3"])
def test_visible_pairs_brute_force(name):
    lay = synth.CONFIGS[name]().layout
    assert oracle.visible_pairs(lay) == PAIRS[name]


@pytest.mark.parametrize("name", ["cfg1", "cfg2", "cfg3", "cfg4"])
def test_visible_pairs_closed_form(name):
    lay = synth.CONFIGS[name]().layout
    assert oracle.visible_pairs_closed_form(lay) == PAIRS[name]


def test_empty_row_set_and_empty_request():
    # a request with no uncached segment: local / retrieval tables have no rows
    segs = [("a", 8, 0, True), ("b", 8, 3, True)]
    lay = synth._make_layout(n_layers=1, hq=2, hkv=2, d=8, p=4, theta=1e4, requests=[segs],
                             class_map=[synth.LOCAL, synth.RETRIEVAL], window=4,
                             retrieval={1: [0, 2]})
    ent, rg = oracle.page_tables(lay)
    assert all(e.shape[0] == 0 for e in ent) and all(r.shape[0] == 0 for r in rg)
    assert oracle.visible_pairs(lay) == 0 == oracle.visible_pairs_closed_form(lay)


def test_partial_last_page_by_hand():
    """13 tokens over 4-token pages: a cached segment of 8 stored at 0..7
    placed at 0 (delta 0) and a 5-token uncached tail; a global head sees all
    four pages, the last holding one key; a local head (W=3) computes rows
    8..12 and sees the pages holding keys 6..12."""
    segs = [("a", 8, 0, True), ("t", 5, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=2, hkv=2, d=8, p=4, theta=1e4, requests=[segs],
                             class_map=[synth.GLOBAL, synth.LOCAL], window=3)
    ent, rg = oracle.page_tables(lay)
    np.testing.assert_array_equal(ent[0][:, 1], [0, 4, 8, 12])
    np.testing.assert_array_equal(ent[0][:, 3], [4, 4, 4, 1])
    np.testing.assert_array_equal(ent[1][:, 1], [4, 8, 12])
    np.testing.assert_array_equal(ent[1][:, 3], [4, 4, 1])
    np.testing.assert_array_equal(rg[0], [[0, 13]])
    np.testing.assert_array_equal(rg[1], [[8, 13]])
    assert oracle.visible_pairs(lay) == 13 * 14 // 2 + 5 * 3
