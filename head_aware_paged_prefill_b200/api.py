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
              jobs come from the page tables, built once on the device when
              the object is created.

Inputs may live on the host (pinned tensors are copied asynchronously) or on
the device; ``run(..., out="host")`` returns o on the host.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import binding
from .plan import RelocationPlan, relocation_plan


class SegPagedPrefill:
    def __init__(self, layout, device="cuda", with_lse: bool = False, mode: str = "relocate"):
        if mode not in ("fused", "relocate"):
            raise ValueError(mode)
        self.layout = layout
        self.mode = mode
        self.device = torch.device(device)
        lay = layout
        if mode == "relocate":
            self.plan = self._plan(layout)
        else:
            empty = np.zeros((0, 3), np.int32)
            self.plan = RelocationPlan(empty, empty, layout, 0)
        self.rel_layout = self.plan.layout
        self.hl = binding.HostLayout(self.rel_layout)
        self.sizes = self.hl.sizes()
        self.vis = binding.Visible(self.sizes, self.device)
        self.ws = binding.workspace(self.sizes, self.device)
        self.n_extra = self.plan.n_extra
        shape = (lay.n_pages + self.n_extra, lay.p, lay.d)
        self.k_work = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        self.v_work = torch.empty(shape, dtype=torch.bfloat16, device=self.device)
        # the K store (pages as written) is the relocation's source
        self.k_store = (torch.empty((lay.n_pages, lay.p, lay.d), dtype=torch.bfloat16,
                                    device=self.device) if mode == "relocate" else None)
        self.q_dev = torch.empty((lay.n_layers, lay.total_tokens, lay.hq, lay.d),
                                 dtype=torch.bfloat16, device=self.device)
        self.o = torch.empty_like(self.q_dev)
        self.lse = (torch.empty((lay.n_layers, lay.hq, lay.total_tokens), dtype=torch.float32,
                                device=self.device) if with_lse else None)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.jobs_k = torch.from_numpy(self.plan.jobs_k).to(self.device)
        self.jobs_v = torch.from_numpy(self.plan.jobs_v).to(self.device)
        # relocation and selection are independent: the relocation runs on a
        # side stream that the attention launch waits for
        self.side = torch.cuda.Stream(self.device) if mode == "relocate" else None

    def _plan(self, layout) -> RelocationPlan:
        """Page tables of the original layout (built by the library on the
        device), read back once, turned into relocation jobs."""
        hl = binding.HostLayout(layout)
        sizes = hl.sizes()
        vis = binding.Visible(sizes, self.device)
        ws = binding.workspace(sizes, self.device)
        binding.select_visible(hl, vis, ws)
        torch.cuda.current_stream(self.device).synchronize()
        st = binding.device_status(ws)
        if st:
            raise binding.RkError(binding.RK_ERR_DEVICE, f"rk_select_visible (device {st:#x})")
        entries, _ = vis.tables()
        return relocation_plan(layout, entries)

    # Number of library kernel launches one run() makes.
    @property
    def launches_per_run(self) -> int:
        # select (one kernel) + attention, plus the relocation launches
        return 2 + int(self.plan.jobs_k.shape[0] > 0) + int(self.plan.jobs_v.shape[0] > 0)

    def load(self, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor):
        """Copies inputs (host or device) into the device working buffers."""
        n = self.layout.n_pages
        self.q_dev.copy_(q, non_blocking=True)
        if self.k_store is not None:
            self.k_store.copy_(k_pool, non_blocking=True)
            self.k_work[:n].copy_(self.k_store)
        else:
            self.k_work[:n].copy_(k_pool, non_blocking=True)
        self.v_work[:n].copy_(v_pool, non_blocking=True)

    def compute(self, stream=None, k3_events=None):
        """Runs relocation, selection and attention on the loaded inputs.
        k3_events: optional (start, end) CUDA events recorded around the
        attention kernel on the launching stream."""
        s = stream if stream is not None else torch.cuda.current_stream()
        relocating = self.plan.jobs_k.shape[0] > 0 or self.plan.jobs_v.shape[0] > 0
        if relocating:
            self.side.wait_stream(s)
            if self.plan.jobs_k.shape[0]:
                binding.relocate_rope(self.k_store, self.k_work, self.jobs_k, self.layout.theta,
                                      self.dev_err, self.side)
            if self.plan.jobs_v.shape[0]:
                binding.relocate_rope(self.v_work, self.v_work, self.jobs_v, self.layout.theta,
                                      self.dev_err, self.side)
        binding.select_visible(self.hl, self.vis, self.ws, s)
        if relocating:
            s.wait_stream(self.side)
        if k3_events is not None:
            k3_events[0].record(s)
        binding.segpaged_prefill(self.hl, self.q_dev, self.k_work, self.v_work, self.vis,
                                 self.ws, self.o, self.lse, fuse_rope=self.mode == "fused",
                                 stream=s)
        if k3_events is not None:
            k3_events[1].record(s)

    def run(self, q, k_pool, v_pool, out: str = "device", host_out: Optional[torch.Tensor] = None):
        self.load(q, k_pool, v_pool)
        self.compute()
        if out == "host":
            dst = host_out if host_out is not None else torch.empty(
                self.o.shape, dtype=self.o.dtype, pin_memory=True)
            dst.copy_(self.o, non_blocking=True)
            return dst
        return self.o

    def status(self) -> int:
        """Device error bits of the last run (synchronises the stream)."""
        torch.cuda.current_stream().synchronize()
        return binding.device_status(self.ws) | int(self.dev_err.item())
