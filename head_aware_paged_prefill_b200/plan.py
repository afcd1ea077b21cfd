"""Host-side planning for the relocation pass (BUILDSTATE's relocation part in
the RedKnot pages: cached segment KV is re-rotated to the offset it is reused
at, "Offline KV Reuse + RoPE Relocation" in the README excerpt).

``relocation_plan`` lists one rk_relocate_rope job per page of every cached
segment instance whose delta is non-zero, writing into fresh pages appended to
the pool, and returns the layout that reads those pages with delta 0.  Running
rk_relocate_rope on the jobs and then rk_segpaged_prefill(fuse_rope=0) on the
returned layout computes the same attention as rk_segpaged_prefill(fuse_rope=1)
on the original layout.
"""
from __future__ import annotations

import copy
from typing import Tuple

import numpy as np


def relocation_plan(lay) -> Tuple[np.ndarray, object]:
    """Returns (jobs int32 [n, 3] of (src_page, dst_page, delta), new_layout).

    new_layout.n_pages covers the appended destination pages; every segment of
    new_layout has delta 0.  Instances sharing pages get private copies.
    """
    n_lh = lay.n_layers * lay.hkv
    P = lay.p
    jobs = []
    new_base = lay.page_base.copy().astype(np.int64)
    segs = lay.segments.copy()
    nxt = int(lay.n_pages)
    for s in range(segs.shape[0]):
        _, start, ln, stored, cached = (int(x) for x in segs[s])
        delta = start - stored
        if not cached:
            continue
        segs[s, 3] = start
        if delta == 0:
            continue
        npg = -(-ln // P)
        for lh in range(n_lh):
            src = int(lay.page_base[s, lh])
            new_base[s, lh] = nxt
            for k in range(npg):
                jobs.append((src + k, nxt + k, delta))
            nxt += npg
    out = copy.copy(lay)
    out.segments = segs
    out.page_base = new_base.astype(np.int32)
    out.n_pages = nxt
    return np.asarray(jobs, dtype=np.int32).reshape(-1, 3), out
