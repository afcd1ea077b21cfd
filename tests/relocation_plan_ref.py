"""Python restatement of the relocation plan, kept as a CPU cross-check of
the library's rk_relocation_plan (tests only).

Host-side planning for the relocation pass (BUILDSTATE's relocation part in
the RedKnot pages: cached segment KV is re-rotated to the offset it is reused
at, "Offline KV Reuse + RoPE Relocation" in the README excerpt).

Two pools take part.  The *store* holds every page as written (cached pages
rotated at their stored positions); the *working K pool* mirrors the store's
page ids and is what the attention kernel reads keys from.  The plan lists
one rk_relocate_rope job per page that (a) belongs to a cached segment
instance with a non-zero delta and (b) appears in at least one page table:
attention reads no other page, so no other page needs rotating.  Such a page
is rotated into the working pool at its own id, and V is read from the
caller's pool unchanged.

A physical page can be visible through two instances placed at different
offsets (the same stored content reused twice).  The first instance that
sees it keeps the page id; a later instance with another delta gets a fresh
run of pages appended to both pools, filled by K jobs (rotated) and V jobs
(delta 0, a copy).  Running the jobs and then rk_segpaged_prefill(fuse_rope=0)
on the returned layout computes the same attention as
rk_segpaged_prefill(fuse_rope=1) on the original layout.
"""
from __future__ import annotations

import copy
from dataclasses import dataclass
from typing import Dict, List, Sequence, Set, Tuple

import numpy as np


@dataclass
class RelocationPlan:
    jobs_k: np.ndarray   # int32 [n, 3] (src_page in the store, dst_page in the working K pool, delta)
    jobs_v: np.ndarray   # int32 [m, 3] (src_page, dst_page >= n_pages, 0) within the V pool
    layout: object       # every segment at delta 0; page_base moved for appended runs
    n_extra: int         # pages appended to the working pools


def _segment_of(lay) -> List[Tuple[np.ndarray, np.ndarray]]:
    """Per request: (segment indices, their logical starts), ascending."""
    out = []
    for r in range(lay.n_req):
        idx = np.nonzero(lay.segments[:, 0] == r)[0]
        starts = lay.segments[idx, 1]
        order = np.argsort(starts, kind="stable")
        out.append((idx[order], starts[order]))
    return out


def visible_pages(lay, entries: Sequence[np.ndarray]) -> Dict[Tuple[int, int], Set[int]]:
    """{(segment, layer * Hkv + kv_head): page offsets within the segment that
    some page table lists}.  entries[t] is table t's [n, 4] entries
    (phys_page, logical_pos, delta, n_valid), t = (r * n_layers + layer) * Hkv + kvh."""
    n_lh = lay.n_layers * lay.hkv
    segs = _segment_of(lay)
    need: Dict[Tuple[int, int], Set[int]] = {}
    for t, e in enumerate(entries):
        if e is None or len(e) == 0:
            continue
        r, lh = divmod(t, n_lh)
        idx, starts = segs[r]
        pos = np.asarray(e)[:, 1]
        which = np.searchsorted(starts, pos, side="right") - 1
        for s_i, p in zip(which.tolist(), pos.tolist()):
            s = int(idx[s_i])
            need.setdefault((s, lh), set()).add((p - int(lay.segments[s, 1])) // lay.p)
    return need


def relocation_plan(lay, entries: Sequence[np.ndarray]) -> RelocationPlan:
    """Relocation jobs for ``lay`` given its page tables (``entries`` as the
    page-table builder returns them, indexed by table id)."""
    n_lh = lay.n_layers * lay.hkv
    P = lay.p
    need = visible_pages(lay, entries)
    claim: Dict[int, int] = {}  # physical page -> delta its working copy holds
    jobs_k: List[Tuple[int, int, int]] = []
    jobs_v: List[Tuple[int, int, int]] = []
    new_base = lay.page_base.copy().astype(np.int64)
    segs = lay.segments.copy()
    nxt = int(lay.n_pages)
    for s in range(segs.shape[0]):
        _, start, ln, stored, cached = (int(x) for x in segs[s])
        delta = start - stored if cached else 0
        segs[s, 3] = start
        npg = -(-ln // P)
        for lh in range(n_lh):
            ks = sorted(need.get((s, lh), ()))
            if not ks:
                continue
            base = int(lay.page_base[s, lh])
            if any(claim.get(base + k, delta) != delta for k in ks):
                new_base[s, lh] = nxt
                for k in ks:
                    jobs_k.append((base + k, nxt + k, delta))
                    jobs_v.append((base + k, nxt + k, 0))
                nxt += npg
                continue
            for k in ks:
                if base + k in claim:
                    continue
                claim[base + k] = delta
                if delta != 0:
                    jobs_k.append((base + k, base + k, delta))
    out = copy.copy(lay)
    out.segments = segs
    out.page_base = new_base.astype(np.int32)
    out.n_pages = nxt
    return RelocationPlan(np.asarray(jobs_k, dtype=np.int32).reshape(-1, 3),
                          np.asarray(jobs_v, dtype=np.int32).reshape(-1, 3), out,
                          nxt - int(lay.n_pages))
