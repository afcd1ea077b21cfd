"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from head_aware_paged_prefill_b200 import binding

# tolerances for bf16-in / fp32-accumulate outputs (max abs, mean relative)
MAX_ABS = 2e-2
MEAN_REL = 5e-3
SENTINEL = 0x7FC0  # a bf16 NaN the kernels never write


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def assert_close(got: np.ndarray, want: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU values"
    err = np.abs(got - want)
    mx = float(err.max()) if err.size else 0.0
    rel = float(err.sum() / max(np.abs(want).sum(), 1e-300)) if err.size else 0.0
    assert mx <= MAX_ABS, f"{what}: max abs err {mx:.3e} > {MAX_ABS}"
    assert rel <= MEAN_REL, f"{what}: mean rel err {rel:.3e} > {MEAN_REL}"
    return mx, rel


def assert_bf16_rounded(got: np.ndarray, want: np.ndarray, what: str = ""):
    """A bf16 tensor computed in fp32 against its fp64 value: every element
    within one bf16 ulp of the exact value (round-to-nearest gives half an
    ulp; the fp32 evaluation may push a value across a rounding midpoint),
    ulp taken at the bottom of the value's binade, 2^-7 |want|, plus an
    absolute floor of 1e-5 for values that cancel to near zero."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU values"
    err = np.abs(got - want)
    bound = np.abs(want) * 2.0 ** -7 + 1e-5
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond one bf16 ulp, worst "
                           f"err {float(err[bad].max()):.3e} at |want| "
                           f"{float(np.abs(want[bad][np.argmax(err[bad])])):.3e}")
    return float(err.max()) if err.size else 0.0


def run_select(lay, device="cuda"):
    hl = binding.HostLayout(lay)
    s = hl.sizes()
    vis = binding.Visible(s, device)
    ws = binding.workspace(s, device)
    binding.select_visible(hl, vis, ws)
    return hl, vis, ws


class PrefillRun:
    """One pass of the CUDA path through the C ABI.

    mode "relocate": rk_relocation_plan gives the jobs and the relocated
    layout; rk_relocate_rope rotates the visible cached K pages from the
    input pool (the store) into a working copy, then rk_select_visible and
    rk_segpaged_prefill(fuse_rope=0) run on the relocated layout.  mode "fused": rk_select_visible and
    rk_segpaged_prefill(fuse_rope=1) on the original layout.
    ``o`` starts filled with the sentinel so untouched rows can be checked."""

    def __init__(self, lay, q, k_pool, v_pool, with_lse=True, mode="relocate"):
        dev = q.device
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        if mode == "fused":
            rel, self.plan = lay, None
            self.k_rel, self.v_rel = k_pool, v_pool
        else:
            # relocation jobs and the relocated layout (rk_relocation_plan)
            self.plan = binding.relocation_plan(lay)
            rel = self.plan.layout
            extra = self.plan.n_extra
            pad = torch.zeros((extra,) + tuple(k_pool.shape[1:]), dtype=k_pool.dtype, device=dev)
            self.k_rel = torch.cat([k_pool, pad])
            self.v_rel = torch.cat([v_pool, pad])
            if self.plan.jobs_k.shape[0]:
                binding.relocate_rope(k_pool, self.k_rel, torch.from_numpy(self.plan.jobs_k).to(dev),
                                      lay.theta, self.dev_err)
            if self.plan.jobs_v.shape[0]:
                binding.relocate_rope(self.v_rel, self.v_rel,
                                      torch.from_numpy(self.plan.jobs_v).to(dev), lay.theta,
                                      self.dev_err)
        self.lay, self.rel = lay, rel
        self.hl, self.vis, self.ws = run_select(rel, dev)
        self.o = torch.full(q.shape, SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
        self.lse = (torch.full((lay.n_layers, lay.hq, lay.total_tokens), float("nan"),
                               device=dev) if with_lse else None)
        binding.segpaged_prefill(self.hl, q, self.k_rel, self.v_rel, self.vis, self.ws, self.o,
                                 self.lse, fuse_rope=mode == "fused")
        torch.cuda.synchronize()
        self.status = binding.device_status(self.ws) | int(self.dev_err.item())


def table_rows(lay):
    """(table -> list of row ranges) from the oracle's brute-force row sets."""
    _, ranges = oracle.page_tables(lay)
    return ranges


def sample_rows(lay, per_table: int, seed: int):
    """(layer, q_head, token) rows: for each table, its first and last rows,
    rows around 128-row tile boundaries, and random rows; every q head."""
    rng = np.random.default_rng(seed)
    ranges = table_rows(lay)
    g = lay.hq // lay.hkv
    out = []
    for r in range(lay.n_req):
        t0 = int(lay.cu_seqlens[r])
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                rg = ranges[lay.table_index(r, layer, kvh)]
                if rg.shape[0] == 0:
                    continue
                rows = np.concatenate([np.arange(a, b) for a, b in rg])
                pick = {int(rows[0]), int(rows[-1])}
                for a, b in rg:
                    for x in (a + 127, a + 128, b - 129, b - 128):
                        if a <= x < b:
                            pick.add(int(x))
                extra = rng.choice(rows, size=min(len(rows), per_table), replace=False)
                pick.update(int(x) for x in extra)
                for h in range(kvh * g, kvh * g + g):
                    for i in sorted(pick):
                        out.append((layer, h, t0 + i))
    return np.asarray(out, dtype=np.int32).reshape(-1, 3)


def oracle_rows(lay, q, k_pool, v_pool, rows):
    qr = q[torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 2]).long(),
           torch.from_numpy(rows[:, 1]).long()]
    return oracle.attention(lay, u16(qr), u16(k_pool), u16(v_pool), rows)


def gpu_rows(run: PrefillRun, rows):
    o = run.o[torch.from_numpy(rows[:, 0]).long().to(run.o.device),
              torch.from_numpy(rows[:, 2]).long().to(run.o.device),
              torch.from_numpy(rows[:, 1]).long().to(run.o.device)]
    lse = None
    if run.lse is not None:
        lse = run.lse[torch.from_numpy(rows[:, 0]).long().to(run.o.device),
                      torch.from_numpy(rows[:, 1]).long().to(run.o.device),
                      torch.from_numpy(rows[:, 2]).long().to(run.o.device)]
        lse = lse.double().cpu().numpy()
    return o.double().cpu().numpy(), lse
