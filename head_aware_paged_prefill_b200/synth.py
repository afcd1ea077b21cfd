"""Seeded synthetic workloads for SegPagedAttention prefill.

This module only builds inputs: the segment layout of each request, the head
class map, the retrieval page lists, and the bf16 Q / K-pool / V-pool values.
It holds none of the method's arithmetic (no RoPE, no visibility rule, no
attention), so both the CUDA path and the fp64 oracle can consume it.

Recipe (RedKnot pages, "Offline KV Reuse + RoPE Relocation" and
"SegPagedAttention Runtime" in the README excerpt; the per-(layer, kv_head)
class map of the "Head Classification" bullet):

* Structure is drawn with ``numpy.random.default_rng(seed)``.
* Values are drawn with ``torch.Generator(device).manual_seed(seed)`` as
  float32 ``randn`` and rounded to bf16 (round to nearest even), in this order:
  Q for every layer (``[T, Hq, D]`` per layer), then the whole K pool
  (``[n_pages, P, D]``), then the whole V pool.  The device is part of the
  recipe: CPU for the small cases, CUDA for the full-size ones (the host
  cannot draw 10^10 normals in reasonable time).
* Cached K is drawn directly in its stored (rotated) form.  A rotation of an
  i.i.d. N(0, 1) vector is again i.i.d. N(0, 1), so this has the distribution
  of ``bf16(R(stored_pos) k_raw)`` without doing RoPE arithmetic here.
* Page rows past the end of a request (the tail's last, partial page) are
  zero.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

GLOBAL, LOCAL, RETRIEVAL, DENSE = 0, 1, 2, 3
CLASS_NAMES = {GLOBAL: "global", LOCAL: "local", RETRIEVAL: "retrieval", DENSE: "dense"}


@dataclasses.dataclass
class Layout:
    """Host-side description of one prefill batch over a paged KV pool.

    segments: int32 [n_seg, 5] rows of (req, logical_start, len,
        stored_pos_base, cached), grouped by request in ascending
        logical_start and tiling [0, L_r) of each request.
    page_base: int32 [n_seg, n_layers * hkv]; the physical page holding the
        first page of the segment for one (layer, kv_head).  The segment's
        pages for that (layer, kv_head) are consecutive page ids.
    cu_seqlens: int32 [n_req + 1] token offsets of the requests.
    class_map: int8 [n_layers * hkv], class of each (layer, kv_head).
    class_window: int32 [4], key window of the local class (others unused).
    retr_indptr / retr_pages: CSR over tables t = (req * n_layers + layer) *
        hkv + kvh of request-logical page numbers (page k covers positions
        [k P, k P + P)) chosen for retrieval heads.
    """

    n_req: int
    n_layers: int
    hq: int
    hkv: int
    d: int
    p: int
    n_pages: int
    theta: float
    segments: np.ndarray
    page_base: np.ndarray
    cu_seqlens: np.ndarray
    class_map: np.ndarray
    class_window: np.ndarray
    retr_indptr: np.ndarray
    retr_pages: np.ndarray
    softmax_scale: float
    # per-page value scale of K and V (cfg3 draws one per kv head); None = 1
    kv_page_scale: Optional[np.ndarray] = None

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def n_tables(self) -> int:
        return self.n_req * self.n_layers * self.hkv

    def req_len(self, r: int) -> int:
        return int(self.cu_seqlens[r + 1] - self.cu_seqlens[r])

    def table_index(self, r: int, layer: int, kvh: int) -> int:
        return (r * self.n_layers + layer) * self.hkv + kvh

    def segments_of(self, r: int) -> np.ndarray:
        return self.segments[self.segments[:, 0] == r]


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    layout: Layout
    value_device: str = "cpu"

    def materialize(self, device: Optional[str] = None):
        """Draw (q, k_pool, v_pool) as bf16 tensors on ``device``.

        q is [n_layers, T, Hq, D]; the pools are [n_pages, P, D].
        """
        dev = torch.device(device or self.value_device)
        lay = self.layout
        g = torch.Generator(device=dev).manual_seed(self.seed)
        T = lay.total_tokens
        q = torch.empty((lay.n_layers, T, lay.hq, lay.d), dtype=torch.bfloat16, device=dev)
        for layer in range(lay.n_layers):
            q[layer] = torch.randn((T, lay.hq, lay.d), generator=g, device=dev).to(torch.bfloat16)
        pools = []
        for _ in range(2):
            x = torch.randn((lay.n_pages, lay.p, lay.d), generator=g, device=dev)
            if lay.kv_page_scale is not None:
                x *= torch.from_numpy(lay.kv_page_scale).to(dev).view(-1, 1, 1)
            pools.append(x.to(torch.bfloat16))
        k_pool, v_pool = pools
        for page, nv in _partial_pages(lay):
            k_pool[page, nv:] = 0
            v_pool[page, nv:] = 0
        return q, k_pool, v_pool


def _partial_pages(lay: Layout) -> List[Tuple[int, int]]:
    """Physical pages whose last rows lie past the end of their segment."""
    out = []
    for s in range(lay.segments.shape[0]):
        ln = int(lay.segments[s, 2])
        rem = ln % lay.p
        if rem:
            last = ln // lay.p
            for lh in range(lay.n_layers * lay.hkv):
                out.append((int(lay.page_base[s, lh]) + last, rem))
    return out


class _PoolBuilder:
    """Assigns physical pages to segment contents, per (layer, kv_head)."""

    def __init__(self, n_layers: int, hkv: int, p: int):
        self.n_lh = n_layers * hkv
        self.p = p
        self.next_page = 0
        self.bases = {}
        self.owner_lh: List[int] = []  # lh index of every allocated page

    def base_of(self, content, length: int) -> np.ndarray:
        if content in self.bases:
            return self.bases[content]
        npg = -(-length // self.p)
        base = np.empty(self.n_lh, dtype=np.int64)
        for lh in range(self.n_lh):
            base[lh] = self.next_page
            self.next_page += npg
            self.owner_lh.extend([lh] * npg)
        self.bases[content] = base
        return base


def _make_layout(*, n_layers, hq, hkv, d, p, theta, requests, class_map, window,
                 retrieval=None, kv_scale_per_lh=None) -> Layout:
    """requests: per request, a list of (content, len, stored_pos_base, cached).

    ``content`` names the stored KV: equal names share physical pages.
    """
    pb = _PoolBuilder(n_layers, hkv, p)
    seg_rows, bases, cu = [], [], [0]
    for r, segs in enumerate(requests):
        pos = 0
        for content, ln, stored, cached in segs:
            base = pb.base_of(content, ln)
            seg_rows.append((r, pos, ln, stored if cached else pos, 1 if cached else 0))
            bases.append(base)
            pos += ln
        cu.append(cu[-1] + pos)
    n_req = len(requests)
    n_tables = n_req * n_layers * hkv
    retr_lists = [[] for _ in range(n_tables)]
    if retrieval is not None:
        for t, pages in retrieval.items():
            retr_lists[t] = list(pages)
    indptr = np.zeros(n_tables + 1, dtype=np.int32)
    for t in range(n_tables):
        indptr[t + 1] = indptr[t] + len(retr_lists[t])
    flat = [x for lst in retr_lists for x in lst]
    cw = np.zeros(4, dtype=np.int32)
    cw[LOCAL] = window
    page_scale = None
    if kv_scale_per_lh is not None:
        page_scale = np.asarray(kv_scale_per_lh, dtype=np.float32)[np.asarray(pb.owner_lh)]
    return Layout(
        n_req=n_req, n_layers=n_layers, hq=hq, hkv=hkv, d=d, p=p, n_pages=pb.next_page,
        theta=float(theta),
        segments=np.asarray(seg_rows, dtype=np.int32).reshape(-1, 5),
        page_base=np.asarray(bases, dtype=np.int32).reshape(len(seg_rows), n_layers * hkv),
        cu_seqlens=np.asarray(cu, dtype=np.int32),
        class_map=np.asarray(class_map, dtype=np.int8),
        class_window=cw,
        retr_indptr=indptr,
        retr_pages=np.asarray(flat, dtype=np.int32),
        softmax_scale=1.0 / float(np.sqrt(d)),
        kv_page_scale=page_scale,
    )


# ---------------------------------------------------------------------------
# The five workloads.  Shapes follow the RedKnot pages' model families
# (Mistral-7B, Qwen3-32B, a 64K long-context layer) and their share of
# global heads (about 12-15 %, "core advantages" section of the paooo page).
# ---------------------------------------------------------------------------

def cfg1(seed: int = 1) -> Workload:
    """Tiny layer: Hq 4, Hkv 2, D 64, P 16, three cached 128-token segments
    stored at local positions 0..127 and placed at 0/128/256, 64-token tail.
    kv_head 0 global, kv_head 1 local with a 128-key window."""
    segs = [(f"c{i}", 128, 0, True) for i in range(3)] + [("tail", 64, 0, False)]
    lay = _make_layout(n_layers=1, hq=4, hkv=2, d=64, p=16, theta=1e4, requests=[segs],
                       class_map=[GLOBAL, LOCAL], window=128)
    return Workload("cfg1_tiny_L448", seed, lay, "cpu")


def cfg2(seed: int = 2) -> Workload:
    """Mistral-7B-shaped layer at 32K: 7 cached 4096-token segments at local
    positions plus a 4096-token tail; kv_head 0 global, 1-7 local W=4096."""
    segs = [(f"c{i}", 4096, 0, True) for i in range(7)] + [("tail", 4096, 0, False)]
    lay = _make_layout(n_layers=1, hq=32, hkv=8, d=128, p=64, theta=1e6, requests=[segs],
                       class_map=[GLOBAL] + [LOCAL] * 7, window=4096)
    return Workload("cfg2_mistral7b_L32768", seed, lay, "cuda")


def cfg3(seed: int = 3) -> Workload:
    """Qwen3-32B-shaped layer at 32K: 15 slots of 2048 whose contents are a
    seeded permutation of 14 distinct segments plus one duplicate (shared
    pages, two deltas); segment s is stored at base 2048 s.  Per-kv-head K/V
    scale drawn in [0.5, 2]."""
    rng = np.random.default_rng(seed)
    contents = list(range(14)) + [int(rng.integers(14))]
    order = rng.permutation(15)
    slots = [contents[k] for k in order]
    segs = [(f"c{s}", 2048, 2048 * s, True) for s in slots] + [("tail", 2048, 0, False)]
    scale = rng.uniform(0.5, 2.0, size=8)
    lay = _make_layout(n_layers=1, hq=64, hkv=8, d=128, p=64, theta=1e6, requests=[segs],
                       class_map=[GLOBAL] + [LOCAL] * 7, window=2048,
                       kv_scale_per_lh=scale)
    return Workload("cfg3_qwen3_32b_L32768", seed, lay, "cuda")


def cfg4(seed: int = 4) -> Workload:
    """64K layer with three windowed classes: 31 cached 2048-token segments
    plus a 2048 tail; kv_head 0 global, 1 retrieval (16 seeded cached pages),
    2-3 local W=2048."""
    rng = np.random.default_rng(seed)
    segs = [(f"c{i}", 2048, 0, True) for i in range(31)] + [("tail", 2048, 0, False)]
    n_cached_pages = 31 * 2048 // 64
    picks = np.sort(rng.choice(n_cached_pages, size=16, replace=False)).tolist()
    lay = _make_layout(n_layers=1, hq=32, hkv=4, d=128, p=64, theta=1e6, requests=[segs],
                       class_map=[GLOBAL, RETRIEVAL, LOCAL, LOCAL], window=2048,
                       retrieval={1: picks})
    return Workload("cfg4_longctx_L65536", seed, lay, "cuda")


def cfg5(seed: int = 5) -> Workload:
    """Serving mix: 8 requests x 4 layers, Hq 64, Hkv 8, D 128, P 64.
    Lengths ~ U[8192, 65536] (multiple of 64), segments of 1024-4096 tokens
    (step 64), the last one the uncached tail; about 30 % of cached segment
    instances come from a shared set, so the same pages sit in several
    requests at different offsets.  Layers 0-1 hold one dense head each and
    local heads otherwise; layers 2-3 hold the four global heads (12.5 % of
    32) and one retrieval head each.  Windows: local 4096, retrieval 16
    pages."""
    rng = np.random.default_rng(seed)
    n_req, n_layers, hkv, p = 8, 4, 8, 64
    shared = [int(rng.integers(16, 65)) * 64 for _ in range(10)]
    requests = []
    for r in range(n_req):
        L = int(rng.integers(8192, 65537)) // 64 * 64
        segs, pos, k = [], 0, 0
        while pos < L:
            ln = int(rng.integers(16, 65)) * 64
            if pos + ln >= L or L - (pos + ln) < 64:
                segs.append((f"tail{r}", L - pos, 0, False))
                break
            if rng.random() < 0.3:
                sid = int(rng.integers(len(shared)))
                ln = shared[sid]
                if pos + ln > L - 64:
                    segs.append((f"tail{r}", L - pos, 0, False))
                    break
                segs.append((f"s{sid}", ln, 0, True))
            else:
                segs.append((f"r{r}_{k}", ln, 0, True))
            pos += ln
            k += 1
        requests.append(segs)
    cmap = np.full((n_layers, hkv), LOCAL, dtype=np.int8)
    for layer in range(2):
        cmap[layer, int(rng.integers(hkv))] = DENSE
    for layer in (2, 3):
        heads = rng.permutation(hkv)
        cmap[layer, heads[0]] = GLOBAL
        cmap[layer, heads[1]] = GLOBAL
        cmap[layer, heads[2]] = RETRIEVAL
    lay_tmp = _make_layout(n_layers=n_layers, hq=64, hkv=hkv, d=128, p=p, theta=1e6,
                           requests=requests, class_map=cmap.reshape(-1), window=4096)
    retrieval = {}
    for r in range(n_req):
        segs = lay_tmp.segments_of(r)
        cached_pages = []
        for seg in segs:
            if seg[4]:
                cached_pages.extend(range(seg[1] // p, (seg[1] + seg[2]) // p))
        for layer in range(n_layers):
            for h in range(hkv):
                if cmap[layer, h] == RETRIEVAL:
                    k = min(16, len(cached_pages))
                    pick = np.sort(rng.choice(np.asarray(cached_pages), size=k, replace=False))
                    retrieval[lay_tmp.table_index(r, layer, h)] = pick.tolist()
    lay = _make_layout(n_layers=n_layers, hq=64, hkv=hkv, d=128, p=p, theta=1e6,
                       requests=requests, class_map=cmap.reshape(-1), window=4096,
                       retrieval=retrieval)
    return Workload("cfg5_serving_mix_8req_4layer", seed, lay, "cuda")


CONFIGS = {"cfg1": cfg1, "cfg2": cfg2, "cfg3": cfg3, "cfg4": cfg4, "cfg5": cfg5}


def random_tiny(rng: np.random.Generator, *, p: Optional[int] = None, d: int = 8,
                max_len: int = 40, n_req: Optional[int] = None) -> Layout:
    """A small random layout for brute-force comparisons: 1-3 requests of
    length <= max_len, any mix of classes, windows and retrieval lists,
    shared contents, and uncached segments anywhere (not only at the end)."""
    p = p or int(rng.choice([1, 2, 4]))
    n_req = n_req or int(rng.integers(1, 4))
    n_layers = int(rng.integers(1, 3))
    hkv = int(rng.integers(1, 4))
    g = int(rng.integers(1, 3))
    shared = [(f"sh{i}", p * int(rng.integers(1, 4))) for i in range(2)]
    requests = []
    for r in range(n_req):
        L = int(rng.integers(1, max_len + 1))
        segs, pos, k = [], 0, 0
        while pos < L:
            ln = p * int(rng.integers(1, max(2, 8 // p + 1)))
            if pos + ln >= L:
                cached = bool(rng.random() < 0.3) and (L - pos) % p == 0
                segs.append((f"t{r}_{k}", L - pos, int(rng.integers(0, 50)), cached))
                break
            u = rng.random()
            if u < 0.25:
                name, ln = shared[int(rng.integers(2))]
                if pos + ln > L:
                    segs.append((f"t{r}_{k}", L - pos, 0, False))
                    break
                segs.append((name, ln, int(rng.integers(0, 50)), True))
            elif u < 0.5:
                segs.append((f"u{r}_{k}", ln, 0, False))
            else:
                segs.append((f"c{r}_{k}", ln, int(rng.integers(0, 50)), True))
            pos += ln
            k += 1
        requests.append(segs)
    cmap = rng.integers(0, 4, size=n_layers * hkv).astype(np.int8)
    lay = _make_layout(n_layers=n_layers, hq=hkv * g, hkv=hkv, d=d, p=p, theta=100.0,
                       requests=requests, class_map=cmap, window=int(rng.integers(1, 12)))
    retrieval = {}
    for t in range(lay.n_tables):
        r = t // (n_layers * hkv)
        npg = -(-lay.req_len(r) // p)
        k = int(rng.integers(0, min(5, npg) + 1))
        retrieval[t] = np.sort(rng.choice(npg, size=k, replace=False)).tolist()
    lay.retr_pages = np.asarray([x for t in range(lay.n_tables) for x in retrieval[t]],
                                dtype=np.int32)
    ind = np.zeros(lay.n_tables + 1, dtype=np.int32)
    for t in range(lay.n_tables):
        ind[t + 1] = ind[t] + len(retrieval[t])
    lay.retr_indptr = ind
    return lay


def with_classes(lay: Layout, class_map, retrieval=None) -> Layout:
    """The same segments and pages under another head-class map; retrieval
    lists empty unless given as (indptr, pages)."""
    indptr, pages = retrieval if retrieval is not None else (
        np.zeros(lay.n_tables + 1, np.int32), np.zeros(0, np.int32))
    return dataclasses.replace(lay, class_map=np.asarray(class_map, dtype=np.int8),
                               retr_indptr=np.asarray(indptr, dtype=np.int32),
                               retr_pages=np.asarray(pages, dtype=np.int32))


def replicate_requests(lay: Layout, n: int) -> Layout:
    """n requests with the segments and retrieval lists of a one-request
    layout, each on its own copy of the pages (request r's pages follow the
    pool r times over)."""
    assert lay.n_req == 1
    seg = np.asarray(lay.segments, dtype=np.int32)
    segs = np.concatenate([np.column_stack([np.full(seg.shape[0], r, np.int32), seg[:, 1:]])
                           for r in range(n)]).astype(np.int32)
    pb = np.concatenate([np.asarray(lay.page_base, np.int64) + r * lay.n_pages
                         for r in range(n)]).astype(np.int32)
    L = lay.req_len(0)
    # every request keeps the retrieval lists of the original request's tables
    counts = np.diff(np.asarray(lay.retr_indptr, np.int64))
    indptr = np.concatenate([[0], np.cumsum(np.tile(counts, n))]).astype(np.int32)
    pages = np.tile(np.asarray(lay.retr_pages, np.int32), n)
    return dataclasses.replace(lay, n_req=n, n_pages=lay.n_pages * n, segments=segs,
                               page_base=pb, cu_seqlens=(np.arange(n + 1) * L).astype(np.int32),
                               retr_indptr=indptr, retr_pages=pages, kv_page_scale=None)


def tiny_workload(lay: Layout, seed: int = 0) -> Workload:
    return Workload("tiny", seed, lay, "cpu")


def random_small(rng: np.random.Generator, *, p: Optional[int] = None, d: Optional[int] = None,
                 max_pages: int = 24, n_req: Optional[int] = None) -> Layout:
    """Random layout with the library's page sizes and head dims: 1-3
    requests of up to max_pages pages (last page possibly partial), every
    class, odd and even GQA groups, shared and private cached segments,
    uncached segments anywhere, windows from 1 to 4 pages."""
    p = p or int(rng.choice([16, 64]))
    d = d or int(rng.choice([64, 128]))
    n_req = n_req or int(rng.integers(1, 4))
    n_layers = int(rng.integers(1, 3))
    hkv = int(rng.integers(1, 4))
    g = int(rng.choice([1, 2, 3, 4]))
    shared = [(f"sh{i}", p * int(rng.integers(1, 4))) for i in range(2)]
    requests = []
    for r in range(n_req):
        L = int(rng.integers(1, max_pages * p + 1))
        segs, pos, k = [], 0, 0
        while pos < L:
            ln = p * int(rng.integers(1, 6))
            if pos + ln >= L:
                cached = bool(rng.random() < 0.3) and (L - pos) % p == 0
                segs.append((f"t{r}_{k}", L - pos, int(rng.integers(0, 5000)), cached))
                break
            u = rng.random()
            if u < 0.25:
                name, ln = shared[int(rng.integers(2))]
                if pos + ln > L:
                    segs.append((f"t{r}_{k}", L - pos, 0, False))
                    break
                segs.append((name, ln, int(rng.integers(0, 5000)), True))
            elif u < 0.45:
                segs.append((f"u{r}_{k}", ln, 0, False))
            else:
                segs.append((f"c{r}_{k}", ln, int(rng.integers(0, 5000)), True))
            pos += ln
            k += 1
        requests.append(segs)
    cmap = rng.integers(0, 4, size=n_layers * hkv).astype(np.int8)
    n_tables = n_req * n_layers * hkv
    retrieval = {}
    lens = [sum(s[1] for s in segs) for segs in requests]
    for t in range(n_tables):
        r = t // (n_layers * hkv)
        npg = -(-lens[r] // p)
        k = int(rng.integers(0, min(6, npg) + 1))
        retrieval[t] = np.sort(rng.choice(npg, size=k, replace=False)).tolist()
    return _make_layout(n_layers=n_layers, hq=hkv * g, hkv=hkv, d=d, p=p,
                        theta=float(rng.choice([1e4, 1e6])), requests=requests, class_map=cmap,
                        window=int(rng.integers(1, 4 * p + 1)), retrieval=retrieval)


def ffn_inputs(n_rows: int, d_model: int, d_ff: int, seed: int, device="cpu"):
    """Synthetic hidden state and FFN weights for the token-selective FFN:
    x ~ N(0, 1) [n_rows][d_model]; W_gate, W_up ~ N(0, 1 / d_model)
    [d_ff][d_model]; W_down ~ N(0, 1 / d_ff) [d_model][d_ff] (so every
    product is of unit scale), all drawn in fp32 in that order from
    torch.Generator(device).manual_seed(seed) and rounded to bf16.  The
    width of the bench's FFN is Mistral-7B's (d_model 4096, d_ff 14336)."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(seed)
    bf = torch.bfloat16
    x = torch.randn((n_rows, d_model), generator=g, device=dev).to(bf)
    wg = (torch.randn((d_ff, d_model), generator=g, device=dev) * d_model ** -0.5).to(bf)
    wu = (torch.randn((d_ff, d_model), generator=g, device=dev) * d_model ** -0.5).to(bf)
    wd = (torch.randn((d_model, d_ff), generator=g, device=dev) * d_ff ** -0.5).to(bf)
    return x, wg, wu, wd
