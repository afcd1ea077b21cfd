"""The Python API above the C ABI: the pipelined host path gives, step by
step, the bytes the one-step path gives, in both modes."""
import numpy as np
import pytest
import torch

from head_aware_paged_prefill_b200 import synth
from head_aware_paged_prefill_b200.api import SegPagedPrefill

pytestmark = pytest.mark.gpu


def _steps(wl, n):
    """n different host input triples of one layout (q, K and V rescaled or
    negated per step, so a step reading another step's buffers shows)."""
    q, k, v = wl.materialize("cpu")
    out = []
    for s in range(n):
        f = (1.0, -0.5, 2.0, 0.25)[s % 4]
        out.append(tuple((t.float() * f).to(torch.bfloat16).pin_memory() for t in (q, k, v)))
    return out


def _workload(case):
    if case == "cfg1":
        return synth.cfg1()
    # shared segments: pages reused at two offsets, so V is relocated too
    lay = synth.random_small(np.random.default_rng(100 + case), max_pages=24)
    return synth.tiny_workload(lay, seed=case)


def _one_step_outputs(pre, steps):
    """o of each step through run(); every buffer set's o starts as NaN, so
    the rows no head computes (left untouched) agree between the paths."""
    pre.run_host_pipelined([], [])  # creates the second buffer set
    for b in pre._sets:
        b["o"].fill_(float("nan"))
    want = []
    for q, k, v in steps:
        want.append(pre.run(q, k, v, out="host"))
        torch.cuda.synchronize()
    return want


@pytest.mark.parametrize("mode", ["relocate", "fused"])
@pytest.mark.parametrize("case", ["cfg1", 0, 1, 2])
def test_pipelined_matches_one_step(case, mode):
    wl = _workload(case)
    lay = wl.layout
    steps = _steps(wl, 5)
    pre = SegPagedPrefill(lay, "cuda", mode=mode)
    want = _one_step_outputs(pre, steps)
    outs = [torch.full_like(w, float("nan")).pin_memory() for w in want]
    pre.run_host_pipelined(steps, outs)
    torch.cuda.synchronize()
    assert pre.status() == 0
    for n, (got, w) in enumerate(zip(outs, want)):
        assert torch.equal(got.view(torch.int16), w.view(torch.int16)), f"step {n}"


def test_pipelined_one_step_and_reuse():
    """A single step, then a second call on the same object: the buffer sets
    and streams carry no state between calls."""
    wl = synth.cfg1()
    lay = wl.layout
    steps = _steps(wl, 3)
    pre = SegPagedPrefill(lay, "cuda")
    want = _one_step_outputs(pre, steps)
    o1 = [torch.empty_like(want[0]).pin_memory()]
    pre.run_host_pipelined(steps[:1], o1)
    o2 = [torch.empty_like(w).pin_memory() for w in want]
    pre.run_host_pipelined(steps, o2)
    torch.cuda.synchronize()
    assert torch.equal(o1[0].view(torch.int16), want[0].view(torch.int16))
    for got, w in zip(o2, want):
        assert torch.equal(got.view(torch.int16), w.view(torch.int16))
    with pytest.raises(ValueError):
        pre.run_host_pipelined(steps, o2[:1])


def test_c_abi_relocate_step_cfg3():
    """The step the bench times in relocate mode, written with the C ABI's
    calls only (through the ctypes binding): rk_relocation_plan ->
    rk_relocate_rope (K store -> working K pool; V copies into the pages
    appended for the duplicated segment) -> rk_select_visible ->
    rk_segpaged_prefill(fuse_rope = 0).  On cfg3 (a segment placed twice,
    sharing pages) its output matches the oracle on sampled rows, and
    SegPagedPrefill gives the same bytes."""
    import oracle
    from head_aware_paged_prefill_b200 import binding
    from gpu_util import assert_close, oracle_rows, sample_rows
    wl = synth.cfg3()
    lay = wl.layout
    q, k, v = wl.materialize("cuda")
    plan = binding.relocation_plan(lay)
    assert plan.n_extra > 0 and plan.jobs_v.shape[0] > 0
    n, extra = lay.n_pages, plan.n_extra
    pad = torch.zeros((extra, lay.p, lay.d), dtype=torch.bfloat16, device="cuda")
    k_work, v_work = torch.cat([k, pad]), torch.cat([v, pad])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.relocate_rope(k, k_work, torch.from_numpy(plan.jobs_k).cuda(), lay.theta, err)
    binding.relocate_rope(v_work, v_work, torch.from_numpy(plan.jobs_v).cuda(), lay.theta, err)
    hl = binding.HostLayout(plan.layout)
    s = hl.sizes()
    vis, ws = binding.Visible(s, "cuda"), binding.workspace(s, "cuda")
    binding.select_visible(hl, vis, ws)
    o = torch.full_like(q, float("nan"))
    binding.segpaged_prefill(hl, q, k_work, v_work, vis, ws, o, None, fuse_rope=False)
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0 and int(err.item()) == 0
    rows = sample_rows(lay, per_table=12, seed=31)
    want, _, _ = oracle_rows(lay, q.cpu(), k.cpu(), v.cpu(), rows)
    idx = [torch.from_numpy(rows[:, c]).long().cuda() for c in (0, 2, 1)]
    assert_close(o[idx[0], idx[1], idx[2]].double().cpu().numpy(), want, "cfg3 C-ABI step")
    pre = SegPagedPrefill(lay, "cuda")
    pre.load(q, k, v)
    pre.compute()
    torch.cuda.synchronize()
    got = pre.o[idx[0], idx[1], idx[2]]
    assert torch.equal(got.view(torch.int16), o[idx[0], idx[1], idx[2]].view(torch.int16))
