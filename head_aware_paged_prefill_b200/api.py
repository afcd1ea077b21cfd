"""Public Python API: one SegPagedAttention prefill pass over a paged pool.

``SegPagedPrefill(layout)`` plans the buffers of one layout once (page
tables, work list, workspace); ``run(q, k_pool, v_pool)`` then executes the
C-ABI calls on the current CUDA stream.  Two modes:

  "fused"     rk_select_visible, then rk_segpaged_prefill(fuse_rope=1): cached
              keys are rotated by their page's delta as they are loaded.
  "relocate"  rk_relocate_rope writes relocated copies of every cached page
              with a non-zero delta (K rotated, V copied), then
              rk_select_visible and rk_segpaged_prefill(fuse_rope=0) read them.

Inputs may live on the host (pinned tensors are copied asynchronously) or on
the device; ``run(..., out="host")`` returns o on the host.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import binding
from .plan import relocation_plan


class SegPagedPrefill:
    def __init__(self, layout, device="cuda", with_lse: bool = False, mode: str = "fused"):
        if mode not in ("fused", "relocate"):
            raise ValueError(mode)
        self.layout = layout
        self.mode = mode
        self.device = torch.device(device)
        if mode == "relocate":
            self.jobs_np, self.rel_layout = relocation_plan(layout)
        else:
            self.jobs_np, self.rel_layout = np.zeros((0, 3), np.int32), layout
        self.hl = binding.HostLayout(self.rel_layout)
        self.sizes = self.hl.sizes()
        self.vis = binding.Visible(self.sizes, self.device)
        self.ws = binding.workspace(self.sizes, self.device)
        lay = layout
        self.n_extra = int(self.rel_layout.n_pages - lay.n_pages)
        self.jobs = torch.from_numpy(self.jobs_np).to(self.device)
        self.k_work = torch.empty((self.rel_layout.n_pages, lay.p, lay.d), dtype=torch.bfloat16,
                                  device=self.device)
        self.v_work = torch.empty_like(self.k_work)
        self.q_dev = torch.empty((lay.n_layers, lay.total_tokens, lay.hq, lay.d),
                                 dtype=torch.bfloat16, device=self.device)
        self.o = torch.empty_like(self.q_dev)
        self.lse = (torch.empty((lay.n_layers, lay.hq, lay.total_tokens), dtype=torch.float32,
                                device=self.device) if with_lse else None)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=self.device)
        # V is not rotated: its relocated pages are delta-0 copies (a page gather)
        jobs_v = self.jobs_np.copy()
        jobs_v[:, 2] = 0
        self.jobs_v = torch.from_numpy(jobs_v).to(self.device)

    # Number of library kernel launches one run() makes.
    @property
    def launches_per_run(self) -> int:
        return 3 + (2 if self.jobs_np.shape[0] else 0)

    def load(self, q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor):
        """Copies inputs (host or device) into the device working buffers."""
        n = self.layout.n_pages
        self.q_dev.copy_(q, non_blocking=True)
        self.k_work[:n].copy_(k_pool, non_blocking=True)
        self.v_work[:n].copy_(v_pool, non_blocking=True)

    def compute(self, stream=None, k3_events=None):
        """Runs relocation, selection and attention on the loaded inputs.
        k3_events: optional (start, end) CUDA events recorded around the
        attention kernel on the launching stream."""
        if self.jobs_np.shape[0]:
            binding.relocate_rope(self.k_work, self.k_work, self.jobs, self.layout.theta,
                                  self.dev_err, stream)
            binding.relocate_rope(self.v_work, self.v_work, self.jobs_v, self.layout.theta,
                                  self.dev_err, stream)
        binding.select_visible(self.hl, self.vis, self.ws, stream)
        s = stream if stream is not None else torch.cuda.current_stream()
        if k3_events is not None:
            k3_events[0].record(s)
        binding.segpaged_prefill(self.hl, self.q_dev, self.k_work, self.v_work, self.vis,
                                 self.ws, self.o, self.lse, fuse_rope=self.mode == "fused",
                                 stream=stream)
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
