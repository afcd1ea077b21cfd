#!/usr/bin/env python
"""SegPagedAttention prefill benchmark (visible-pair TFLOP/s on B200).

One step = one pass of the whole hot path over the Mistral-7B-shaped 32K
layer (Hq 32, Hkv 8, D 128, P 64; 7 cached 4096-token segments + 4096 tail;
kv_head 0 global, 1-7 local with a 4096 window), inputs resident in HBM, L2
flushed (256 MiB write, then 256 MiB read of another buffer) between timed
steps.  Default mode "relocate":
rk_relocate_rope (every visible page of a cached segment with a non-zero
delta, rotated from the K store into the working K pool) ->
rk_select_visible -> rk_segpaged_prefill.  Mode "fused":
rk_select_visible -> rk_segpaged_prefill with the relocation done inside the
attention kernel.  The line reports the other mode too, and the standalone
relocation kernel against the HBM roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs its own replica
(the work items are independent: weak scaling, no collective on the data
path); time is the max over ranks of the summed device step times.
``--impl reference`` times the fp64 CPU oracle on a bounded row sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SegPagedAttn prefill visible-pair TFLOP/s & % BF16 peak at 32K"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS = 2250.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


KERNEL_SOURCES = {"segpaged_prefill_kernel": ("rk_prefill.cu", "sm100.cuh", "rk_internal.h"),
                  "relocate_kernel": ("rk_relocate.cu", "sm100.cuh", "rk_internal.h"),
                  "decode_split_kernel": ("rk_decode.cu", "rk_internal.h"),
                  "importance_colsum_kernel": ("rk_importance.cu", "rk_internal.h"),
                  "ffn_gemm_kernel": ("rk_ffn.cu", "sm100.cuh", "rk_internal.h")}


def _kernel_hash(kernel: str = "segpaged_prefill_kernel") -> str:
    """Hash of the sources a kernel is compiled from (ties a recorded ncu
    figure to the code it was taken on)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "head_aware_paged_prefill_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _recorded_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {})
    # a later source state counts only where its device code was checked
    # byte-identical to the captured one (recorded beside the figure)
    hashes = {e.get("source_hash")} | {x["source_hash"] for x in e.get("same_device_code", [])}
    if _kernel_hash(kernel) not in hashes or e.get("workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


class L2Flush:
    """Evicts the workload from the 126 MB L2 between timed steps: a write of
    one 256 MiB buffer, then a read of another, so the L2 is left holding
    clean, unrelated lines (a write alone leaves dirty lines whose write-back
    would land inside the next timed kernel)."""

    DESCRIPTION = "flushed between timed steps (256 MiB write, then 256 MiB read)"

    def __init__(self, torch, dev):
        self.a = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.b = torch.ones(256 << 20, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.a.zero_()
        self.b.sum()


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (every rank gets it); plain x without a
    process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, work_per_rank: float, steps: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank ran `steps` steps of `work_per_rank`;
    the job took as long as the slowest rank."""
    return world * work_per_rank * steps / (max_total_ms * 1e-3)


def _gpu_id(torch, dev) -> str:
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev.index or 0)


def _oracle_sample_rows(lay, n_rows: int, seed: int):
    """A seeded sample of computed (layer, q_head, token) rows, uniform over
    every computed row of the workload, and the number of visible keys of
    the sampled rows (closed form per class), for the CPU baseline."""
    from head_aware_paged_prefill_b200 import metrics
    rng = np.random.default_rng(seed)
    g = lay.hq // lay.hkv
    tabs, sizes = [], []
    for r in range(lay.n_req):
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                rows = metrics.table_rows(lay, r, layer, kvh)
                if rows.size:
                    tabs.append((r, layer, kvh, rows))
                    sizes.append(rows.size)
    w = np.asarray(sizes, dtype=np.float64)
    pick = rng.choice(len(tabs), size=n_rows, p=w / w.sum())
    out, pairs = [], 0
    for ti in np.unique(pick):
        r, layer, kvh, rows = tabs[ti]
        n = int((pick == ti).sum())
        i = rows[rng.integers(rows.size, size=n)]
        h = kvh * g + rng.integers(g, size=n)
        pairs += int(metrics.row_visible_keys(lay, r, layer, kvh, i).sum())
        t0 = int(lay.cu_seqlens[r])
        out.append(np.column_stack([np.full(n, layer), h, t0 + i]))
    return np.concatenate(out).astype(np.int32), pairs


def _time_oracle(lay, q, k, v, rows):
    import torch
    import oracle

    def u16(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    idx = torch.from_numpy(rows).long().to(q.device)
    qr = q[idx[:, 0], idx[:, 2], idx[:, 1]].cpu()
    t0 = time.perf_counter()
    oracle.attention(lay, u16(qr), u16(k), u16(v), rows)
    return time.perf_counter() - t0


def _bench_relocate(torch, lay, k_pool, dev, flush, stream, reps, peaks, peak_kind, copies=4):
    """rk_relocate_rope alone over every page of every cached segment with
    delta != 0 (all (layer, kv_head) pairs, visible or not), from the store
    into a working pool at the same page ids.  The main figure runs that job
    list over `copies` distinct copies of the store into as many distinct
    destination pools, so the pages read and written (several times the
    126 MB L2) stream from and to HBM; the single-copy figure, whose 50 MB
    of writes can stay in L2 until after the timed launch, is kept beside
    it as "in_l2"."""
    from head_aware_paged_prefill_b200 import binding, metrics
    n_lh = lay.n_layers * lay.hkv
    jobs = []
    for s in range(lay.segments.shape[0]):
        _, start, ln, stored, cached = (int(x) for x in lay.segments[s])
        if cached and start != stored:
            for lh in range(n_lh):
                b0 = int(lay.page_base[s, lh])
                jobs += [(b0 + k, b0 + k, start - stored) for k in range(-(-ln // lay.p))]
    if not jobs:
        return None
    jobs = np.asarray(jobs, dtype=np.int32)
    peak = float(peaks["hbm_gbs"])

    def timed(src, dst, jt):
        for _ in range(3):
            binding.relocate_rope(src, dst, jt, lay.theta)
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            binding.relocate_rope(src, dst, jt, lay.theta)
            b.record(stream)
            ms.append((a, b))
        torch.cuda.synchronize()
        return statistics.mean(x.elapsed_time(y) for x, y in ms)

    n = jobs.shape[0]
    t1 = timed(k_pool, torch.empty_like(k_pool), torch.from_numpy(jobs).to(dev))
    b1 = metrics.relocate_bytes(n, lay.p, lay.d)
    npg = int(k_pool.shape[0])
    big = np.concatenate([jobs + np.asarray([c * npg, c * npg, 0], np.int32) for c in range(copies)])
    src = k_pool.repeat(copies, 1, 1)
    dst = torch.empty_like(src)
    t = timed(src, dst, torch.from_numpy(big).to(dev))
    del src, dst
    torch.cuda.empty_cache()
    byts = metrics.relocate_bytes(big.shape[0], lay.p, lay.d)
    gbs = byts / (t * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "relocate_kernel", "jobs": int(big.shape[0]),
            "workload": f"every delta != 0 page of the layer's cached segments, {copies} "
                        "distinct copies (sources and destinations)",
            "bytes": byts, "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
            "peak_kind": peak_kind, "us": t * 1e3,
            "traffic": _recorded_traffic("relocate_kernel", "relocate_" + str(big.shape[0])),
            "in_l2": {"jobs": n, "bytes": b1, "us": t1 * 1e3,
                      "achieved": b1 / (t1 * 1e-3) / 1e9, "frac": b1 / (t1 * 1e-3) / 1e9 / peak}}


def cpu_values(wl):
    """(q, k, v) on the host for the oracle (drawn on the GPU when the workload's
    recipe says so, then copied back)."""
    import torch
    dev = wl.value_device if (wl.value_device == "cpu" or torch.cuda.is_available()) else "cpu"
    q, k, v = wl.materialize(dev)
    return q.cpu(), k.cpu(), v.cpu()


def run_reference(args, rank, world):
    """The fp64 oracle on a bounded row sample per step (rank 0 only)."""
    if rank != 0:
        return 0
    from head_aware_paged_prefill_b200 import synth
    wl = synth.CONFIGS[args.config]()
    lay = wl.layout
    q, k, v = cpu_values(wl)
    cores = os.cpu_count() or 1
    # size the per-step sample: one oracle call has a fixed cost (layout
    # setup, key relocation) besides its cost per row, so two calls of
    # different sizes give both; a step then takes about 4x the fixed cost
    # (at least --ref-step-s), within a budget that ends the whole run in
    # about four minutes
    rows, _ = _oracle_sample_rows(lay, 64, seed=0)
    t_a = _time_oracle(lay, q, k, v, rows)
    rows, _ = _oracle_sample_rows(lay, 512, seed=0)
    t_b = _time_oracle(lay, q, k, v, rows)
    per_row = max((t_b - t_a) / (512 - 64), 1e-7)
    fixed = max(t_a - 64 * per_row, 0.0)
    budget = max(240.0 / (args.warmup + args.steps), args.ref_step_s)
    step_s = min(max(args.ref_step_s, 4 * fixed), budget)
    n_rows = int(max(64, min(65536, (step_s - fixed) / per_row)))
    tot_t, tot_pairs = 0.0, 0
    for s in range(args.warmup + args.steps):
        rows, pairs = _oracle_sample_rows(lay, n_rows, seed=1 + s)
        dt = _time_oracle(lay, q, k, v, rows)
        if s >= args.warmup:
            tot_t += dt
            tot_pairs += pairs
    value = 4 * lay.d * tot_pairs / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "step": f"oracle on {n_rows} sampled rows"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n_rows} seeded (layer, q head, row) samples per step, "
                                   f"{args.steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _bench_scoring(torch, lay, q, k_store, dev, flush, stream, reps, peaks, peak_kind):
    """rk_score_retrieval_pages on the same layer with every kv head a
    retrieval head (its cached pages ranked against its tail queries, top
    16): a bandwidth measurement of the scoring launches."""
    from head_aware_paged_prefill_b200 import binding, metrics, synth
    lay_r = synth.with_classes(lay, [synth.RETRIEVAL] * (lay.n_layers * lay.hkv))
    hl = binding.HostLayout(lay_r)
    out = binding.ScoreOutputs(binding.score_sizes(hl, 16), 16, dev, with_scores=False)
    for _ in range(3):
        binding.score_retrieval_pages(hl, q, k_store, lay.theta, out)
    torch.cuda.synchronize()
    ms = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        binding.score_retrieval_pages(hl, q, k_store, lay.theta, out)
        b.record(stream)
        ms.append((a, b))
    torch.cuda.synchronize()
    t = statistics.mean(x.elapsed_time(y) for x, y in ms)
    nbytes = metrics.scoring_bytes(lay_r)
    gbs = nbytes / (t * 1e-3) / 1e9
    n_tables = int((out.count > 0).sum().item())
    return {"bound": "hbm", "kernel": "score_query + score_page + score_pick",
            "workload": "the same layer, every kv head a retrieval head, top 16",
            "tables": n_tables, "bytes": nbytes, "achieved": gbs,
            "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
            "frac": gbs / float(peaks["hbm_gbs"]), "peak_kind": peak_kind, "us": t * 1e3,
            "launches": 3}


def _mask_penalty(torch, pre, lay, q, k3_ms, reps=5):
    """Context for the pages' claim that a dense layout with an attention
    mask loses the fast attention path (paooo page, "paged storage removes
    the mask penalty"): torch SDPA on the dense relocated K / V of the same
    layer, one call per head class with an explicit boolean mask over the
    same visible (row, key) pairs, timed against the paged kernel."""
    from head_aware_paged_prefill_b200 import synth
    if lay.n_req != 1 or lay.n_layers != 1:
        return None
    L, P, d, g = lay.req_len(0), lay.p, lay.d, lay.hq // lay.hkv
    W = int(lay.class_window[synth.LOCAL])
    dev = q.device
    # dense [Hkv, L, D] K and V from the working pools (relocated pages)
    page_of = torch.empty((lay.hkv, -(-L // P)), dtype=torch.long)
    for s_, seg in enumerate(lay.segments):
        first = int(seg[1]) // P
        for h in range(lay.hkv):
            base = int(lay.page_base[s_, h])
            page_of[h, first:first + -(-int(seg[2]) // P)] = torch.arange(base, base + -(-int(seg[2]) // P))
    page_of = page_of.to(dev)
    K = pre.k_work[page_of].reshape(lay.hkv, -1, d)[:, :L]
    V = pre.v_work[page_of].reshape(lay.hkv, -1, d)[:, :L]
    unc = torch.zeros(L, dtype=torch.bool, device=dev)
    for seg in lay.segments:
        if not seg[4]:
            unc[int(seg[1]):int(seg[1] + seg[2])] = True
    tail = torch.nonzero(unc).flatten()
    i_all = torch.arange(L, device=dev)
    causal = i_all[None, :] <= i_all[:, None]
    window = causal[tail] & (i_all[None, :] > tail[:, None] - W)
    calls = []
    for cls, rows, mask in ((synth.GLOBAL, i_all, causal), (synth.LOCAL, tail, window)):
        heads = [h for h in range(lay.hkv) if int(lay.class_map[h]) == cls]
        if not heads:
            continue
        qh = torch.cat([q[0, rows, h * g:(h + 1) * g] for h in heads], dim=1).transpose(0, 1)
        kh = torch.cat([K[h:h + 1].expand(g, -1, -1) for h in heads])
        vh = torch.cat([V[h:h + 1].expand(g, -1, -1) for h in heads])
        calls.append((qh[None].contiguous(), kh[None].contiguous(), vh[None].contiguous(),
                      mask, heads, rows))
    sdpa = torch.nn.functional.scaled_dot_product_attention
    scale = 1.0 / math.sqrt(d)
    for c in calls:
        sdpa(c[0], c[1], c[2], attn_mask=c[3], scale=scale)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        outs = [sdpa(c[0], c[1], c[2], attn_mask=c[3], scale=scale) for c in calls]
    b.record()
    torch.cuda.synchronize()
    sdpa_ms = a.elapsed_time(b) / reps
    # the two paths agree on a sample of rows (bf16 outputs)
    diff = 0.0
    for (qh, kh, vh, mask, heads, rows), o in zip(calls, outs):
        pick = torch.linspace(0, rows.numel() - 1, 16, device=dev).long()
        for j, h in enumerate(heads):
            mine = pre.o[0, rows[pick], h * g:(h + 1) * g].float()
            ref = o[0, j * g:(j + 1) * g, pick].transpose(0, 1).float()
            diff = max(diff, float((mine - ref).abs().max()))
    del calls, outs, causal, window
    torch.cuda.empty_cache()
    return {"sdpa_masked_ms": sdpa_ms, "k3_ms": k3_ms, "ratio": sdpa_ms / k3_ms,
            "sample_max_abs_diff": diff,
            "note": "torch SDPA on dense relocated K/V with an explicit boolean mask per head "
                    "class, the same visible pairs; context for the pages' 4.9-7.6x"}


def _bench_decode(torch, lay, pre, dev, flush, stream, reps, peaks, peak_kind, batch):
    """rk_segpaged_decode on a batch of `batch` requests shaped like the
    bench's layer, each on its own copy of the relocated pages (so every
    request's keys come from HBM): one decode row per request and q head."""
    from head_aware_paged_prefill_b200 import binding, metrics, synth
    if lay.n_req != 1 or batch < 1:
        return None
    lay_b = synth.replicate_requests(lay, batch)
    n = lay.n_pages
    k_b = pre.k_work[:n].repeat(batch, 1, 1)
    v_b = pre.v_work[:n].repeat(batch, 1, 1)
    hl = binding.HostLayout(lay_b)
    vis = binding.Visible(hl.sizes(), dev)
    ws_sel = binding.workspace(hl.sizes(), dev)
    binding.select_visible(hl, vis, ws_sel)
    g = torch.Generator(device=dev).manual_seed(7)
    q_d = torch.randn((lay.n_layers, batch, lay.hq, lay.d), generator=g, device=dev).to(torch.bfloat16)
    o_d = torch.empty_like(q_d)
    sizes = binding.decode_sizes(hl)
    ws = binding.decode_workspace(sizes, dev)
    for _ in range(3):
        binding.segpaged_decode(hl, q_d, k_b, v_b, vis, ws, o_d)
    torch.cuda.synchronize()
    st = binding.device_status(ws)
    ms = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        binding.segpaged_decode(hl, q_d, k_b, v_b, vis, ws, o_d)
        b.record(stream)
        ms.append((a, b))
    torch.cuda.synchronize()
    t = statistics.mean(x.elapsed_time(y) for x, y in ms)
    nbytes = metrics.decode_bytes(lay_b)
    gbs = nbytes / (t * 1e-3) / 1e9
    del k_b, v_b
    torch.cuda.empty_cache()
    return {"bound": "hbm", "kernel": "decode_split + decode_combine",
            "workload": f"{batch} requests shaped like the bench's layer, own pages each, "
                        "one decode row per request and q head",
            "bytes": nbytes, "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
            "frac": gbs / float(peaks["hbm_gbs"]), "peak_kind": peak_kind, "us": t * 1e3,
            "rows_per_s": batch * lay.n_layers * lay.hq / (t * 1e-3), "device_status": st,
            "traffic": _recorded_traffic("decode_split_kernel", f"decode_{batch}req")}


def _bench_importance(torch, lay, lay_name, q, k, v, dev, flush, stream, reps, peaks, peak_kind):
    """rk_attention_importance on the bench's layer after its prefill (with
    lse): every visible (q head, row, key) pair's weight exp(s - lse) summed
    per token, then the top L/4 tokens.  One exp per visible pair and a
    QK^T product: bound by the exp unit (16 results per clock per SM), the
    roofline given here."""
    from head_aware_paged_prefill_b200 import metrics
    from head_aware_paged_prefill_b200.api import SegPagedPrefill
    pre = SegPagedPrefill(lay, dev, with_lse=True)
    pre.load(q, k, v)
    pre.compute()
    top_k = max(lay.req_len(r) for r in range(lay.n_req)) // 4
    for _ in range(3):
        pre.attention_importance(top_k)
    torch.cuda.synchronize()
    st = pre.importance_status()
    ms = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        pre.attention_importance(top_k)
        b.record(stream)
        ms.append((a, b))
    torch.cuda.synchronize()
    t = statistics.mean(x.elapsed_time(y) for x, y in ms)
    pairs = metrics.visible_pairs(lay)
    sm_mhz = float(peaks.get("sm_max_mhz", 1965.0))
    exp_peak = 148 * 16 * sm_mhz * 1e6 / 1e9  # G exp / s
    achieved = pairs / (t * 1e-3) / 1e9
    del pre
    torch.cuda.empty_cache()
    return {"bound": "alu", "kernel": "importance_colsum + importance_select",
            "workload": f"the bench's layer, top {top_k} tokens", "pairs": pairs,
            "achieved": achieved, "peak": exp_peak, "unit": "Gexp/s",
            "frac": achieved / exp_peak, "peak_kind": "derived: 148 SMs x 16 ex2 / clock x max SM clock",
            "us": t * 1e3, "qk_tflops": 2 * lay.d * pairs / (t * 1e-3) / 1e12,
            "traffic": _recorded_traffic("importance_colsum_kernel", lay_name),
            "device_status": st}


def _bench_ffn(torch, lay, dev, flush, stream, reps, peaks, peak_kind, d_model=4096, d_ff=14336):
    """rk_sparse_ffn on the layer's rows at Mistral-7B's FFN width with the
    top quarter of each request's tokens selected (seeded synthetic hidden
    state and weights): three GEMM-sized products (gate, up, down) on the
    selected rows only, bound by the tensor cores."""
    from head_aware_paged_prefill_b200 import binding, synth
    T = lay.total_tokens
    top_k = max(lay.req_len(r) for r in range(lay.n_req)) // 4
    x, wg, wu, wd = synth.ffn_inputs(T, d_model, d_ff, seed=21, device=dev)
    rng = np.random.default_rng(22)
    tok = np.zeros((lay.n_req, top_k), dtype=np.int32)
    for r in range(lay.n_req):
        L = lay.req_len(r)
        k = min(top_k, L)
        tok[r, :k] = np.sort(rng.choice(L, size=k, replace=False))
    tok = torch.from_numpy(tok).to(dev)
    sizes = binding.ffn_sizes(T, d_model, d_ff, lay.cu_seqlens, top_k)
    ws = binding.ffn_workspace(sizes, dev)
    for _ in range(3):
        binding.sparse_ffn(x, lay.cu_seqlens, tok, top_k, wg, wu, wd, ws)
    torch.cuda.synchronize()
    ms = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        binding.sparse_ffn(x, lay.cu_seqlens, tok, top_k, wg, wu, wd, ws)
        b.record(stream)
        ms.append((a, b))
    torch.cuda.synchronize()
    t = statistics.mean(x_.elapsed_time(y_) for x_, y_ in ms)
    m = int(sizes.n_selected)
    flops = 2 * m * d_model * d_ff * 3
    achieved = flops / (t * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    st = binding.device_status(ws)
    del x, wg, wu, wd, ws
    torch.cuda.empty_cache()
    return {"bound": "tensor", "kernel": "ffn_gather + ffn_gemm (gate/up, SwiGLU) + ffn_gemm (down, residual)",
            "workload": f"the layer's {T} rows, top {top_k} per request selected, d_model {d_model}, "
                        f"d_ff {d_ff} (Mistral-7B's FFN), seeded synthetic x and weights",
            "selected_rows": m, "flops": flops, "achieved": achieved, "peak": peak,
            "unit": UNIT, "frac": achieved / peak, "peak_kind": f"bf16 burst, {peak_kind}",
            "us": t * 1e3, "launches": 3, "device_status": st,
            "traffic": _recorded_traffic("ffn_gemm_kernel", f"ffn_{m}x{d_model}x{d_ff}")}


def _cpu_baseline(lay, q, kc, vc, seconds: float, total_pairs: int):
    """The fp64 oracle timed on seeded row samples of the workload (batches of
    growing size until about `seconds` of oracle time), with the full-run
    time it implies (labelled as an extrapolation)."""
    n_rows, tot_rows, tot_pairs, tot_t, seed = 1024, 0, 0, 0.0, 1
    while tot_t < seconds:
        rows, pairs = _oracle_sample_rows(lay, n_rows, seed=seed)
        tot_t += _time_oracle(lay, q, kc, vc, rows)
        tot_rows += n_rows
        tot_pairs += pairs
        seed += 1
        n_rows = min(2 * n_rows, 65536)
    return {"value": 4 * lay.d * tot_pairs / tot_t / 1e12, "unit": UNIT,
            "cores": os.cpu_count() or 1, "kind": "oracle",
            "sample": f"{tot_rows} seeded (layer, q head, row) samples, uniform over the "
                      f"workload's computed rows, in {seed - 1} batches: {tot_pairs} visible "
                      f"pairs in {tot_t:.1f} s",
            "rows_per_s": tot_rows / tot_t,
            "full_run_s_extrapolated": tot_t * total_pairs / max(tot_pairs, 1)}


def _bench_config(torch, name, dev, flush, stream, steps, warmup, peaks, peak_kind, cpu_s):
    """One more workload, timed like the headline one in both modes: the
    attention kernel's TFLOP/s against the bf16 roofline, the whole step's
    TFLOP/s and tokens/s, and a CPU-oracle baseline on a row sample."""
    from head_aware_paged_prefill_b200 import metrics, synth
    from head_aware_paged_prefill_b200.api import SegPagedPrefill
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    q, k, v = wl.materialize(str(dev))
    flops = metrics.attention_flops(lay)
    tokens = lay.total_tokens * lay.n_layers
    peak = float(peaks["bf16_tflops"])
    out = {"workload": wl.name, "requests": lay.n_req, "layers": lay.n_layers,
           "tokens": lay.total_tokens, "heads": f"Hq {lay.hq} / Hkv {lay.hkv}",
           "head_dim": lay.d, "page_size": lay.p, "visible_pairs": flops // (4 * lay.d),
           "steps": steps, "l2": L2Flush.DESCRIPTION}
    for mode in ("relocate", "fused"):
        pre = SegPagedPrefill(lay, dev, mode=mode)
        pre.load(q, k, v)
        for _ in range(warmup):
            pre.compute()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(2 * steps)]
        for s_ in range(steps):
            flush()
            ev[2 * s_][0].record(stream)
            pre.compute(k3_events=ev[2 * s_ + 1])
            ev[2 * s_][1].record(stream)
        torch.cuda.synchronize()
        step_ms = statistics.mean(ev[2 * i][0].elapsed_time(ev[2 * i][1]) for i in range(steps))
        k3_ms = statistics.mean(ev[2 * i + 1][0].elapsed_time(ev[2 * i + 1][1])
                                for i in range(steps))
        k3 = flops / (k3_ms * 1e-3) / 1e12
        out[mode] = {"step_tflops": flops / (step_ms * 1e-3) / 1e12, "ms_per_step": step_ms,
                     "tokens_per_s": tokens / (step_ms * 1e-3), "k3_ms": k3_ms,
                     "k3_tflops": k3, "k3_frac": k3 / peak, "device_status": pre.status(),
                     "launches_per_step": pre.launches_per_run}
        del pre
        torch.cuda.empty_cache()
    k3 = out["relocate"]["k3_tflops"]
    out["roofline"] = {"bound": "tensor", "kernel": "segpaged_prefill_kernel", "mode": "relocate",
                       "achieved": k3, "peak": peak, "unit": UNIT, "frac": k3 / peak,
                       "peak_kind": f"bf16 burst, {peak_kind}",
                       "traffic": _recorded_traffic("segpaged_prefill_kernel", wl.name)}
    if cpu_s > 0:
        out["cpu_baseline"] = _cpu_baseline(lay, q, k.cpu(), v.cpu(), cpu_s, flops // (4 * lay.d))
    del q, k, v
    return out


def _bench_e2e(torch, pre, q, k, v, stream, E, world, dist, dev, flops):
    """The same metric end to end through SegPagedPrefill with host buffers:
    pinned q / K / V in and o out every step, E steps pipelined."""
    q_h = q.cpu().pin_memory()
    k_h = k.cpu().pin_memory()
    v_h = v.cpu().pin_memory()
    o_h = torch.empty(pre.o.shape, dtype=pre.o.dtype, pin_memory=True)
    pre.run_host_pipelined([(q_h, k_h, v_h)] * 2, [o_h] * 2)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    pre.run_host_pipelined([(q_h, k_h, v_h)] * E, [o_h] * E)
    b.record(stream)
    b.synchronize()
    e2e_ms = a.elapsed_time(b)
    # the same steps one after another (copy in, compute, copy out), for context
    a2, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a2.record(stream)
    for _ in range(min(E, 5)):
        pre.run(q_h, k_h, v_h, out="host", host_out=o_h)
    b2.record(stream)
    b2.synchronize()
    serial_ms_per_step = a2.elapsed_time(b2) / min(E, 5)
    e2e_ms = max_over_ranks(e2e_ms, dist if world > 1 else None, dev)
    e2e_value = weak_scaling_value(world, flops, E, e2e_ms) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = o_h.numel() * o_h.element_size()
    del q_h, k_h, v_h, o_h
    return {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / E, "pipelined": True,
            "serial_ms_per_step": serial_ms_per_step}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="cfg2")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--mode", default="relocate", choices=["fused", "relocate"])
    ap.add_argument("--reloc-reps", type=int, default=50)
    ap.add_argument("--ref-step-s", type=float, default=0.25)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mask-penalty", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=32)
    ap.add_argument("--no-importance", action="store_true")
    ap.add_argument("--no-ffn", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--per-config", default="cfg1,cfg3,cfg4,cfg5",
                    help="other workloads timed after the headline one ('' for none)")
    ap.add_argument("--pc-steps", type=int, default=20)
    ap.add_argument("--pc-cpu-seconds", type=float, default=6.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from head_aware_paged_prefill_b200 import metrics, synth
    from head_aware_paged_prefill_b200.api import SegPagedPrefill

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    wl = synth.CONFIGS[args.config]()
    lay = wl.layout
    q, k, v = wl.materialize(str(dev))
    pre = SegPagedPrefill(lay, dev, mode=args.mode)
    pre.load(q, k, v)
    flops = metrics.attention_flops(lay)
    tokens = lay.total_tokens * lay.n_layers
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        pre.compute()
    torch.cuda.synchronize()
    st = pre.status()
    if st != 0:
        raise SystemExit(f"device error word {st:#x} after warm-up")

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    ev3 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    sampler = ClockSampler(_gpu_id(torch, dev))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(K):
        flush()
        ev[s][0].record(stream)
        pre.compute(k3_events=ev3[s])
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    k3_ms = [a.elapsed_time(b) for a, b in ev3]
    total_ms = max_over_ranks(sum(step_ms), dist if world > 1 else None, dev)
    st = pre.status()
    if st != 0:
        raise SystemExit(f"device error word {st:#x} after the timed steps")
    ms_per_step = total_ms / K
    launches = K * pre.launches_per_run
    value = weak_scaling_value(world, flops, K, total_ms) / 1e12

    # end to end through the public API: pinned host inputs in, o back to
    # host, E steps pipelined (step n + 1's inputs and step n - 1's o cross
    # the host link while step n computes); every step moves its full inputs
    # and output, each larger than L2
    e2e = _bench_e2e(torch, pre, q, k, v, stream, args.e2e_steps, world, dist, dev, flops) \
        if not args.no_e2e else None
    peaks, peak_kind = _peaks()
    k3_mean = statistics.mean(k3_ms)
    achieved = flops / (k3_mean * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = _recorded_traffic("segpaged_prefill_kernel", wl.name)

    reloc = _bench_relocate(torch, lay, k, dev, flush, stream, args.reloc_reps, peaks, peak_kind)
    scoring = _bench_scoring(torch, lay, q, k, dev, flush, stream, args.reloc_reps, peaks,
                             peak_kind)
    decode = (_bench_decode(torch, lay, pre, dev, flush, stream, args.reloc_reps, peaks,
                            peak_kind, args.decode_batch)
              if args.mode == "relocate" else None)
    importance = (_bench_importance(torch, lay, wl.name, q, k, v, dev, flush, stream,
                                    args.reloc_reps, peaks, peak_kind)
                  if args.mode == "relocate" and not args.no_importance else None)
    ffn = (_bench_ffn(torch, lay, dev, flush, stream, args.reloc_reps, peaks, peak_kind)
           if args.mode == "relocate" and not args.no_ffn else None)
    mask_penalty = (_mask_penalty(torch, pre, lay, q, k3_mean)
                    if args.mode == "relocate" and not args.no_mask_penalty else None)

    # the other mode of the same path, timed the same way (context)
    other = "relocate" if args.mode == "fused" else "fused"
    alt = SegPagedPrefill(lay, dev, mode=other)
    alt.load(q, k, v)
    for _ in range(args.warmup):
        alt.compute()
    torch.cuda.synchronize()
    alt_ms, alt_k3 = 0.0, 0.0
    for s_ in range(K):
        flush()
        ev[s_][0].record(stream)
        alt.compute(k3_events=ev3[s_])
        ev[s_][1].record(stream)
    torch.cuda.synchronize()
    alt_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    alt_k3 = statistics.mean(a.elapsed_time(b) for a, b in ev3)
    st = alt.status()
    other_mode = {"mode": other, "value": flops / (alt_ms * 1e-3) / 1e12, "unit": UNIT,
                  "ms_per_step": alt_ms, "k3_tflops": flops / (alt_k3 * 1e-3) / 1e12,
                  "device_status": st}
    del alt

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_baseline = _cpu_baseline(lay, q, k.cpu(), v.cpu(), args.cpu_seconds, flops // (4 * lay.d))

    per_config = None
    if world == 1 and args.per_config:
        per_config = {}
        del pre
        torch.cuda.empty_cache()
        for name in [c for c in args.per_config.split(",") if c and c != args.config]:
            per_config[name] = _bench_config(torch, name, dev, flush, stream, min(K, args.pc_steps),
                                             args.warmup, peaks, peak_kind,
                                             0.0 if args.no_cpu_baseline else args.pc_cpu_seconds)
            torch.cuda.empty_cache()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "layers": lay.n_layers, "seq_len": lay.total_tokens,
                   "heads": f"Hq {lay.hq} / Hkv {lay.hkv}", "head_dim": lay.d,
                   "page_size": lay.p, "visible_pairs": flops // (4 * lay.d),
                   "parallelism": f"replicas x{world}",
                   "l2": L2Flush.DESCRIPTION},
        "pct_bf16_peak": 100.0 * value / world / peak,
        "pct_bf16_spec": 100.0 * value / world / SPEC_BF16_TFLOPS,
        "tokens_per_s": weak_scaling_value(world, tokens, K, total_ms),
        "roofline": {"bound": "tensor", "kernel": "segpaged_prefill_kernel",
                     "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                     "peak_kind": f"bf16 burst, {peak_kind}", "traffic": traffic,
                     "k3_ms": k3_mean},
        "cpu_baseline": cpu_baseline,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "mode": args.mode,
        "other_mode": other_mode,
        "relocate_roofline": reloc,
        "retrieval_scoring_roofline": scoring,
        "mask_penalty": mask_penalty,
        "decode_roofline": decode,
        "importance_roofline": importance,
        "sparse_ffn_roofline": ffn,
        "per_config": per_config,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
