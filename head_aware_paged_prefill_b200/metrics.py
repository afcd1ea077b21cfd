"""Work counts used to report throughput.

visible_pairs(layout): sum over layers, q heads and computed rows of the
number of keys the row attends to, counted from each class's rule in closed
form.  Algorithmic FLOPs of the attention are 4 * D per visible pair
(2 D for q.k, 2 D for p.v); exp, masking and rotation are not counted.

row_visible_keys / table_rows: the same rules per sampled row (the CPU
baseline's row samples).

relocate_bytes(jobs, p, d): bytes an rk_relocate_rope pass must move
(read + write of every page it touches).

decode_bytes(layout): bytes rk_segpaged_decode must move: the keys and
values visible to every table's last row (once per kv head), the new rows'
queries and the outputs.

scoring_bytes(layout): bytes rk_score_retrieval_pages must read: the
queries of every retrieval table's rows (all q heads of its kv head) and the
keys of its candidate pages, each once.
"""
from __future__ import annotations

import numpy as np

LOCAL, RETRIEVAL = 1, 2


def _uncached_mask(lay, r):
    L = lay.req_len(r)
    m = np.zeros(L, dtype=bool)
    for seg in lay.segments[lay.segments[:, 0] == r]:
        if not seg[4]:
            m[int(seg[1]):int(seg[1] + seg[2])] = True
    return m


def visible_pairs(lay) -> int:
    g = lay.hq // lay.hkv
    W = int(lay.class_window[LOCAL])
    P = lay.p
    total = 0
    for r in range(lay.n_req):
        L = lay.req_len(r)
        unc = _uncached_mask(lay, r)
        rows = np.nonzero(unc)[0].astype(np.int64)
        n_unc_le = np.cumsum(unc.astype(np.int64))  # uncached keys at positions <= i
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                c = int(lay.class_map[layer * lay.hkv + kvh])
                if c == LOCAL:
                    total += g * int(np.minimum(rows + 1, W).sum())
                elif c == RETRIEVAL:
                    t = lay.table_index(r, layer, kvh)
                    pages = np.unique(lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]])
                    pages = pages[(pages >= 0) & (pages * P < L)]
                    pages = pages[~unc[pages * P]]
                    cnt = n_unc_le[rows].sum() if rows.size else 0
                    for k in pages:
                        first, last = int(k) * P, min(int(k) * P + P, L) - 1
                        # keys first..last visible to rows i >= first: min(i, last) - first + 1
                        cnt += int(np.clip(rows - first + 1, 0, last - first + 1).sum())
                    total += g * int(cnt)
                else:
                    total += g * L * (L + 1) // 2
    return int(total)


def row_visible_keys(lay, r: int, layer: int, kvh: int, rows: np.ndarray) -> np.ndarray:
    """Visible keys of each request-local row in ``rows`` (rows of the table's
    row set) for table (r, layer, kvh), from the class rules in closed form."""
    rows = np.asarray(rows, dtype=np.int64)
    c = int(lay.class_map[layer * lay.hkv + kvh])
    if c == LOCAL:
        return np.minimum(rows + 1, int(lay.class_window[LOCAL]))
    if c != RETRIEVAL:
        return rows + 1
    P, L = lay.p, lay.req_len(r)
    unc = _uncached_mask(lay, r)
    n_unc_le = np.cumsum(unc.astype(np.int64))
    t = lay.table_index(r, layer, kvh)
    pages = np.unique(lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]])
    pages = pages[(pages >= 0) & (pages * P < L)]
    pages = pages[~unc[pages * P]]
    cnt = n_unc_le[rows].copy()
    for k in pages:
        first, last = int(k) * P, min(int(k) * P + P, L) - 1
        cnt += np.clip(rows - first + 1, 0, last - first + 1)
    return cnt


def table_rows(lay, r: int, layer: int, kvh: int) -> np.ndarray:
    """Request-local rows a table computes: every position for global and
    dense heads, the uncached positions for local and retrieval heads."""
    c = int(lay.class_map[layer * lay.hkv + kvh])
    L = lay.req_len(r)
    if c in (LOCAL, RETRIEVAL):
        return np.nonzero(_uncached_mask(lay, r))[0].astype(np.int64)
    return np.arange(L, dtype=np.int64)


def attention_flops(lay) -> int:
    return 4 * lay.d * visible_pairs(lay)


def relocate_bytes(n_jobs: int, p: int, d: int) -> int:
    return 2 * n_jobs * p * d * 2


def scoring_bytes(lay) -> int:
    g = lay.hq // lay.hkv
    P, D = lay.p, lay.d
    total = 0
    for r in range(lay.n_req):
        L = lay.req_len(r)
        unc = _uncached_mask(lay, r)
        rows = np.nonzero(unc)[0]
        if rows.size == 0:
            continue
        last = int(rows.max())
        cand_keys = sum(min(P, L - k * P) for k in range(-(-L // P))
                        if not unc[k * P] and k * P <= last)
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                if int(lay.class_map[layer * lay.hkv + kvh]) == RETRIEVAL:
                    total += 2 * D * (g * rows.size + cand_keys)
    return int(total)


def decode_bytes(lay) -> int:
    """Last-row attention of every table whose last position is a row."""
    g = lay.hq // lay.hkv
    W = int(lay.class_window[LOCAL])
    P, D = lay.p, lay.d
    keys = 0
    for r in range(lay.n_req):
        L = lay.req_len(r)
        if L == 0:
            continue
        unc = _uncached_mask(lay, r)
        i = L - 1
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                c = int(lay.class_map[layer * lay.hkv + kvh])
                if c in (LOCAL, RETRIEVAL) and not unc[i]:
                    continue
                if c == LOCAL:
                    keys += min(L, W)
                elif c == RETRIEVAL:
                    t = lay.table_index(r, layer, kvh)
                    pages = np.unique(lay.retr_pages[lay.retr_indptr[t]:lay.retr_indptr[t + 1]])
                    pages = pages[(pages >= 0) & (pages * P < L)]
                    pages = pages[~unc[pages * P]]
                    keys += int(unc.sum()) + sum(min(P, L - int(k) * P) for k in pages)
                else:
                    keys += L
    rows = sum(1 for r in range(lay.n_req) if lay.req_len(r) > 0) * lay.n_layers * lay.hq
    return int(2 * D * 2 * keys + 2 * 2 * D * rows)
