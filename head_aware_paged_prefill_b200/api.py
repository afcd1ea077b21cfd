"""Public Python API: one SegPagedAttention prefill pass over a paged pool.

``SegPagedPrefill(layout)`` plans the buffers of one layout once (page
tables, work list, workspace); ``run(q, k_pool, v_pool)`` then executes the
C-ABI calls on the current CUDA stream.  Two modes:

  "fused"     rk_select_visible, then rk_segpaged_prefill(fuse_rope=1): cached
              keys are rotated by their page's delta as they are loaded.
  "relocate"  rk_relocate_rope rotates every visible page of a cached
              segment with a non-zero delta from the K store into the working
              K pool (same page id; pages reused at two offsets get an
              appended copy, V copied alongside), then rk_select_visible and
              rk_segpaged_prefill(fuse_rope=0) read the working pools.  The
              jobs and the relocated layout come from rk_relocation_plan
              (host only), once, when the object is created.

Inputs may live on the host (pinned tensors are copied asynchronously) or on
the device; ``run(..., out="host")`` returns o on the host.
``run_host_pipelined`` runs a sequence of host-resident steps with the copies
of one step overlapping the computation of its neighbours (two device buffer
sets, a copy-in, a compute and a copy-out stream).
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import binding, synth


def score_retrieval(layout, q: torch.Tensor, k_store: torch.Tensor, top_k: int = 16,
                    stream=None):
    """Chooses every retrieval head's cached pages on the device
    (rk_score_retrieval_pages: the top_k pages by the score of their mean
    relocated key against the head's mean tail query) and returns the layout
    with those retrieval lists, plus the device outputs.  q and k_store are
    device tensors ([n_layers][T][Hq][D] post-RoPE queries, the K pool as
    stored).  Reading the picks back synchronises the stream."""
    hl = binding.HostLayout(layout)
    out = binding.ScoreOutputs(binding.score_sizes(hl, top_k), top_k, q.device)
    binding.score_retrieval_pages(hl, q, k_store, layout.theta, out, stream)
    indptr, pages = out.lists()
    return synth.with_classes(layout, layout.class_map, (indptr, pages)), out


class SegPagedPrefill:
    def __init__(self, layout, device="cuda", with_lse: bool = False, mode: str = "relocate"):
        if mode not in ("fused", "relocate"):
            raise ValueError(mode)
        self.layout = layout
        self.mode = mode
        self.device = torch.device(device)
        lay = layout
        # attention work items: 128-row tiles of each table's row ranges x
        # pairs of q heads (the library's own rule), for the launch count
        npairs = (layout.hq // layout.hkv + 1) // 2
        self.n_items = npairs * sum(-(-(b - a) // 128) for a, b in self._row_ranges(layout))
        if mode == "relocate":
            self.plan = binding.relocation_plan(layout)
        else:
            empty = np.zeros((0, 3), np.int32)
            self.plan = binding.RelocationPlan(empty, empty, layout, 0)
        self.rel_layout = self.plan.layout
        self.hl = binding.HostLayout(self.rel_layout)
        self.sizes = self.hl.sizes()
        self.vis = binding.Visible(self.sizes, self.device)
        self.ws = binding.workspace(self.sizes, self.device)
        self.n_extra = self.plan.n_extra
        self._sets = [self._buffers()]
        self.k_work, self.v_work = self._sets[0]["k_work"], self._sets[0]["v_work"]
        self.k_store, self.q_dev, self.o = (self._sets[0][n] for n in ("k_store", "q", "o"))
        self.lse = (torch.empty((lay.n_layers, lay.hq, lay.total_tokens), dtype=torch.float32,
                                device=self.device) if with_lse else None)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.jobs_k = torch.from_numpy(self.plan.jobs_k).to(self.device)
        self.jobs_v = torch.from_numpy(self.plan.jobs_v).to(self.device)
        # relocation and selection are independent: the relocation runs on a
        # side stream that the attention launch waits for
        self.side = torch.cuda.Stream(self.device) if mode == "relocate" else None

    def _buffers(self) -> dict:
        """One set of device buffers a step reads and writes."""
        lay, dev, bf = self.layout, self.device, torch.bfloat16
        shape = (lay.n_pages + self.n_extra, lay.p, lay.d)
        q = torch.empty((lay.n_layers, lay.total_tokens, lay.hq, lay.d), dtype=bf, device=dev)
        return {
            "q": q,
            "o": torch.empty_like(q),
            "k_work": torch.empty(shape, dtype=bf, device=dev),
            "v_work": torch.empty(shape, dtype=bf, device=dev),
            # the K store (pages as written) is the relocation's source
            "k_store": (torch.empty((lay.n_pages, lay.p, lay.d), dtype=bf, device=dev)
                        if self.mode == "relocate" else None),
        }

    @staticmethod
    def _row_ranges(lay):
        """Every table's row ranges by the class rule: the whole request for
        global and dense heads, the merged uncached segments otherwise."""
        out = []
        for r in range(lay.n_req):
            L = lay.req_len(r)
            unc = []
            for seg in lay.segments_of(r):
                if not seg[4]:
                    a, b = int(seg[1]), int(seg[1] + seg[2])
                    if unc and unc[-1][1] == a:
                        unc[-1] = (unc[-1][0], b)
                    else:
                        unc.append((a, b))
            for lh in range(lay.n_layers * lay.hkv):
                c = int(lay.class_map[lh])
                out.extend([(0, L)] if c in (synth.GLOBAL, synth.DENSE) and L > 0 else
                           ([] if c in (synth.GLOBAL, synth.DENSE) else unc))
        return out

    # Number of library kernel launches one run() makes.
    @property
    def launches_per_run(self) -> int:
        # selection (one kernel; a second one moves the work list into cost
        # order above 16384 items), attention, and the relocation launches
        select = 1 if self.n_items <= 16384 else 2
        return (select + 1 + int(self.plan.jobs_k.shape[0] > 0) +
                int(self.plan.jobs_v.shape[0] > 0))

    def _copy_in(self, b: dict, q, k_pool, v_pool):
        """Copies a step's inputs (host or device) into buffer set b on the
        current stream; the K store copy into the working K pool is left to
        the step's computation."""
        n = self.layout.n_pages
        b["q"].copy_(q, non_blocking=True)
        if b["k_store"] is not None:
            b["k_store"].copy_(k_pool, non_blocking=True)
        else:
            b["k_work"][:n].copy_(k_pool, non_blocking=True)
        b["v_work"][:n].copy_(v_pool, non_blocking=True)

    def load(self, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor):
        """Copies inputs (host or device) into the device working buffers."""
        b = self._sets[0]
        self._copy_in(b, q, k_pool, v_pool)
        if b["k_store"] is not None:
            b["k_work"][:self.layout.n_pages].copy_(b["k_store"])

    def compute(self, stream=None, k3_events=None):
        """Runs relocation, selection and attention on the loaded inputs.
        k3_events: optional (start, end) CUDA events recorded around the
        attention kernel on the launching stream."""
        self._compute(self._sets[0], stream, k3_events)

    def _compute(self, b: dict, stream=None, k3_events=None):
        s = stream if stream is not None else torch.cuda.current_stream()
        relocating = self.plan.jobs_k.shape[0] > 0 or self.plan.jobs_v.shape[0] > 0
        if relocating:
            self.side.wait_stream(s)
            if self.plan.jobs_k.shape[0]:
                binding.relocate_rope(b["k_store"], b["k_work"], self.jobs_k, self.layout.theta,
                                      self.dev_err, self.side)
            if self.plan.jobs_v.shape[0]:
                binding.relocate_rope(b["v_work"], b["v_work"], self.jobs_v, self.layout.theta,
                                      self.dev_err, self.side)
        binding.select_visible(self.hl, self.vis, self.ws, s)
        if relocating:
            s.wait_stream(self.side)
        if k3_events is not None:
            k3_events[0].record(s)
        binding.segpaged_prefill(self.hl, b["q"], b["k_work"], b["v_work"], self.vis,
                                 self.ws, b["o"], self.lse, fuse_rope=self.mode == "fused",
                                 stream=s)
        if k3_events is not None:
            k3_events[1].record(s)

    def attention_importance(self, top_k: int, stream=None):
        """Token importance for the sparse FFN from the last compute()
        (rk_attention_importance: the attention weights each token received,
        summed over q heads and computed rows, and the top_k tokens per
        (request, layer)).  Needs relocate mode (relocated K pool) and
        with_lse=True.  Returns device tensors (importance [n_layers][T] fp32,
        tokens [n_layers][n_req][top_k] int32, token_count [n_layers][n_req]
        int32), reused across calls with the same top_k."""
        if self.mode != "relocate" or self.lse is None:
            raise ValueError("attention_importance needs mode='relocate' and with_lse=True")
        lay = self.layout
        key = int(top_k)
        if getattr(self, "_imp", None) is None or self._imp[0] != key:
            sizes = binding.importance_sizes(self.hl)
            self._imp = (key, binding.importance_workspace(sizes, self.device),
                         torch.empty((lay.n_layers, lay.total_tokens), dtype=torch.float32,
                                     device=self.device),
                         torch.empty((lay.n_layers, lay.n_req, max(key, 1)), dtype=torch.int32,
                                     device=self.device),
                         torch.empty((lay.n_layers, lay.n_req), dtype=torch.int32,
                                     device=self.device))
        _, ws, imp, tokens, count = self._imp
        b = self._sets[0]
        binding.attention_importance(self.hl, b["q"], b["k_work"], self.vis, self.lse, ws, imp,
                                     key, tokens if key > 0 else None, count if key > 0 else None,
                                     stream)
        return imp, tokens, count

    def importance_status(self) -> int:
        """Device error word of the last attention_importance call."""
        return binding.device_status(self._imp[1])

    def sparse_ffn(self, x: torch.Tensor, tokens: torch.Tensor, top_k: int, w_gate: torch.Tensor,
                   w_up: torch.Tensor, w_down: torch.Tensor, stream=None) -> torch.Tensor:
        """The token-selective FFN of one layer (rk_sparse_ffn): the picked
        tokens (``tokens`` [n_req][top_k], one layer of attention_importance's
        output) of the hidden state x [T][d_model] take x + W_down (silu(W_gate
        x) * W_up x), every other row keeps x.  Updates x in place and returns
        it; the workspace is kept across calls of the same shape."""
        lay = self.layout
        key = (int(top_k), int(x.shape[1]), int(w_gate.shape[0]))
        if getattr(self, "_ffn", None) is None or self._ffn[0] != key:
            sizes = binding.ffn_sizes(lay.total_tokens, x.shape[1], w_gate.shape[0],
                                      lay.cu_seqlens, top_k)
            self._ffn = (key, binding.ffn_workspace(sizes, self.device))
        binding.sparse_ffn(x, lay.cu_seqlens, tokens, top_k, w_gate, w_up, w_down, self._ffn[1],
                           stream)
        return x

    def ffn_status(self) -> int:
        """Device error word of the last sparse_ffn call."""
        return binding.device_status(self._ffn[1])

    def run(self, q, k_pool, v_pool, out: str = "device", host_out: Optional[torch.Tensor] = None):
        self.load(q, k_pool, v_pool)
        self.compute()
        if out == "host":
            dst = host_out if host_out is not None else torch.empty(
                self.o.shape, dtype=self.o.dtype, pin_memory=True)
            dst.copy_(self.o, non_blocking=True)
            return dst
        return self.o

    def run_host_pipelined(self, inputs, outs, stream=None):
        """Runs one step per entry of ``inputs`` ((q, k_pool, v_pool), pinned
        host tensors) and copies each step's o into the pinned host tensor at
        the same index of ``outs``.

        Step n's inputs cross to the device on a copy-in stream and its o
        comes back on a copy-out stream, each step in one of two device buffer
        sets, so the copies of steps n + 1 and n - 1 overlap step n's
        relocation, selection and attention on ``stream`` (default: the
        current stream).  Every step waits for its own inputs; a buffer set is
        refilled only after the step that last read it, and its o rewritten
        only after that o reached the host.  Returns once all work is queued;
        ``stream`` is ordered after the last copy out."""
        if len(inputs) != len(outs):
            raise ValueError("one output per step")
        s = stream if stream is not None else torch.cuda.current_stream()
        while len(self._sets) < 2:
            self._sets.append(self._buffers())
        if not hasattr(self, "_cp_in"):
            self._cp_in = torch.cuda.Stream(self.device)
            self._cp_out = torch.cuda.Stream(self.device)
        n = self.layout.n_pages
        consumed = [None, None]  # compute of the step that last read set i
        drained = [None, None]   # copy out of the o last written in set i
        self._cp_in.wait_stream(s)
        self._cp_out.wait_stream(s)
        for step, ((q, k_pool, v_pool), dst) in enumerate(zip(inputs, outs)):
            i = step % 2
            b = self._sets[i]
            with torch.cuda.stream(self._cp_in):
                if consumed[i] is not None:
                    self._cp_in.wait_event(consumed[i])
                self._copy_in(b, q, k_pool, v_pool)
                loaded = torch.cuda.Event()
                loaded.record(self._cp_in)
            s.wait_event(loaded)
            if drained[i] is not None:
                s.wait_event(drained[i])
            with torch.cuda.stream(s):
                if b["k_store"] is not None:
                    b["k_work"][:n].copy_(b["k_store"])
            self._compute(b, s)
            done = torch.cuda.Event()
            done.record(s)
            consumed[i] = done
            with torch.cuda.stream(self._cp_out):
                self._cp_out.wait_event(done)
                dst.copy_(b["o"], non_blocking=True)
                out_done = torch.cuda.Event()
                out_done.record(self._cp_out)
            drained[i] = out_done
        s.wait_stream(self._cp_out)
        s.wait_stream(self._cp_in)

    def status(self) -> int:
        """Device error bits of the last run (synchronises the stream)."""
        torch.cuda.current_stream().synchronize()
        return binding.device_status(self.ws) | int(self.dev_err.item())
