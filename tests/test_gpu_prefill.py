"""rk_segpaged_prefill (K3) against the fp64 oracle, element by element.

Two CUDA paths are checked against the same oracle rows: "fused" runs K1 and
K3 with the RoPE relocation fused into K3's K loads; "relocate" runs K2 on
every cached page with delta != 0, then K1 on the relocated layout and K3.
The oracle runs on the original layout and rotates the stored keys itself."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import synth
from gpu_util import (SENTINEL, PrefillRun, assert_close, gpu_rows, oracle_rows, sample_rows,
                      u16)

pytestmark = pytest.mark.gpu


def _all_rows(lay):
    _, ranges = oracle.page_tables(lay)
    g = lay.hq // lay.hkv
    out = []
    for r in range(lay.n_req):
        t0 = int(lay.cu_seqlens[r])
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                for a, b in ranges[lay.table_index(r, layer, kvh)]:
                    for h in range(kvh * g, kvh * g + g):
                        out.extend((layer, h, t0 + i) for i in range(a, b))
    return np.asarray(out, dtype=np.int32).reshape(-1, 3)


def _check(lay, q_cpu, k_cpu, v_cpu, run, rows, what):
    assert run.status == 0, f"device status {run.status}"
    o_ref, lse_ref, comp = oracle_rows(lay, q_cpu, k_cpu, v_cpu, rows)
    assert comp.all()
    o_got, lse_got = gpu_rows(run, rows)
    assert_close(o_got, o_ref, f"{what} o")
    if lse_got is not None:
        assert np.abs(lse_got - lse_ref).max() <= 1e-2, f"{what} lse"


def _untouched(lay, run):
    """Rows outside every table's row set keep the sentinel."""
    _, ranges = oracle.page_tables(lay)
    g = lay.hq // lay.hkv
    o16 = run.o.view(torch.int16)
    bad = 0
    for r in range(lay.n_req):
        t0, L = int(lay.cu_seqlens[r]), lay.req_len(r)
        for layer in range(lay.n_layers):
            for kvh in range(lay.hkv):
                mask = np.ones(L, dtype=bool)
                for a, b in ranges[lay.table_index(r, layer, kvh)]:
                    mask[a:b] = False
                idx = np.nonzero(mask)[0]
                if idx.size == 0:
                    continue
                idx = idx[:: max(1, idx.size // 64)]
                sl = o16[layer, torch.from_numpy(t0 + idx).long().cuda(), kvh * g:kvh * g + g]
                bad += int((sl != SENTINEL).sum().item())
    assert bad == 0


MODES = ("fused", "relocate")


@pytest.mark.parametrize("mode", MODES)
def test_prefill_cfg1_all_rows(mode):
    wl = synth.cfg1()
    lay = wl.layout
    q, k, v = wl.materialize("cpu")
    run = PrefillRun(lay, q.cuda(), k.cuda(), v.cuda(), mode=mode)
    _check(lay, q, k, v, run, _all_rows(lay), f"cfg1 {mode}")
    _untouched(lay, run)


@pytest.mark.parametrize("mode", MODES)
def test_prefill_random_small_all_rows(mode):
    rng = np.random.default_rng(7)
    for n in range(40):
        lay = synth.random_small(rng, max_pages=12)
        wl = synth.tiny_workload(lay, seed=n)
        q, k, v = wl.materialize("cpu")
        run = PrefillRun(lay, q.cuda(), k.cuda(), v.cuda(), mode=mode)
        rows = _all_rows(lay)
        if rows.shape[0]:
            _check(lay, q, k, v, run, rows, f"random layout {n} {mode}")
        _untouched(lay, run)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("cmap", [(0, 1, 2), (3, 2, 1)])
def test_prefill_edge_layout_all_rows(mode, cmap):
    """An empty request between others, a request whose rows are all cached
    (no local / retrieval rows), a one-token request, window 1, retrieval
    lists that name pages before and after the rows, D 64 with 16-token
    pages and a partial last page."""
    reqs = [[("a", 64, 0, True), ("t0", 37, 0, False)], [],
            [("b", 64, 5, True), ("c", 128, 9, True)], [("t3", 1, 0, False)]]
    lay = synth._make_layout(n_layers=1, hq=3, hkv=3, d=64, p=16, theta=1e4, requests=reqs,
                             class_map=list(cmap), window=1,
                             retrieval={0: [0, 3], 1: [1], 2: [2, 5], 7: [0, 1]})
    wl = synth.tiny_workload(lay, seed=11)
    q, k, v = wl.materialize("cpu")
    run = PrefillRun(lay, q.cuda(), k.cuda(), v.cuda(), mode=mode)
    rows = _all_rows(lay)
    assert rows.shape[0] > 0
    _check(lay, q, k, v, run, rows, f"edge layout {cmap} {mode}")
    _untouched(lay, run)


@pytest.mark.parametrize("name,per_table", [("cfg2", 24), ("cfg3", 16), ("cfg4", 16),
                                            ("cfg5", 3)])
def test_prefill_full_size_sampled(name, per_table):
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    q, k, v = wl.materialize("cuda")
    rows = sample_rows(lay, per_table, seed=11)
    # the oracle needs the sampled queries and the pools on the host
    o_ref, lse_ref, comp = oracle_rows(lay, q, k.cpu(), v.cpu(), rows)
    assert comp.all()
    for mode in MODES:
        run = PrefillRun(lay, q, k, v, mode=mode)
        assert run.status == 0, f"{name} {mode}: device status {run.status}"
        o_got, lse_got = gpu_rows(run, rows)
        assert_close(o_got, o_ref, f"{name} {mode} o")
        assert np.abs(lse_got - lse_ref).max() <= 1e-2, f"{name} {mode} lse"
        _untouched(lay, run)
        del run
        torch.cuda.empty_cache()


def _many_items_odd_group():
    """GQA group of 3 (work items alternate between two q heads and one) and
    enough rows that every CTA runs several items of both kinds in a row: the
    four global / dense kv heads alone give 4 x 108 row tiles x 2 head pairs."""
    segs = [(f"c{i}", 2048, 0, True) for i in range(6)] + [("tail", 1536, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=24, hkv=8, d=128, p=64, theta=1e6,
                             requests=[segs], class_map=[0, 1, 0, 1, 3, 1, 0, 1], window=1024)
    return synth.Workload("odd_group_L13824", 21, lay, "cuda")


def test_prefill_many_items_odd_group():
    wl = _many_items_odd_group()
    lay = wl.layout
    q, k, v = wl.materialize("cuda")
    rows = sample_rows(lay, 12, seed=5)
    o_ref, lse_ref, comp = oracle_rows(lay, q, k.cpu(), v.cpu(), rows)
    assert comp.all()
    for mode in MODES:
        run = PrefillRun(lay, q, k, v, mode=mode)
        assert run.status == 0, f"{mode}: device status {run.status}"
        o_got, lse_got = gpu_rows(run, rows)
        assert_close(o_got, o_ref, f"odd group {mode} o")
        assert np.abs(lse_got - lse_ref).max() <= 1e-2, f"odd group {mode} lse"
        _untouched(lay, run)
        del run
        torch.cuda.empty_cache()


@pytest.mark.parametrize("mode", MODES)
def test_prefill_deterministic(mode):
    wl = synth.cfg3()
    q, k, v = wl.materialize("cuda")
    a = PrefillRun(wl.layout, q, k, v, mode=mode)
    b = PrefillRun(wl.layout, q, k, v, mode=mode)
    assert torch.equal(a.o.view(torch.int16), b.o.view(torch.int16))


def test_prefill_repeated_on_one_selection():
    """Work items are handed out from a counter in the workspace: three
    attention launches on one selection must each cover every item (the
    last CTA of a launch resets the counter for the next), bit-identically."""
    from head_aware_paged_prefill_b200 import binding
    wl = synth.cfg2()
    q, k, v = wl.materialize("cuda")
    run = PrefillRun(wl.layout, q, k, v, mode="relocate")
    assert run.status == 0
    first = run.o.clone()
    for _ in range(2):
        run.o.view(torch.int16).fill_(SENTINEL)
        binding.segpaged_prefill(run.hl, q, run.k_rel, run.v_rel, run.vis, run.ws, run.o, run.lse)
        torch.cuda.synchronize()
        assert binding.device_status(run.ws) == 0
        assert torch.equal(run.o.view(torch.int16), first.view(torch.int16))


def test_prefill_reports_bad_page_without_faulting():
    """A page id outside the pool (corrupted after selection) is skipped by the
    kernel (the tile loads zeros) and reported through the error word."""
    from head_aware_paged_prefill_b200 import binding
    from gpu_util import run_select
    wl = synth.cfg1()
    lay = wl.layout
    q, k, v = (t.cuda() for t in wl.materialize("cpu"))
    for fuse in (True, False):
        hl, vis, ws = run_select(lay)
        torch.cuda.synchronize()
        vis.entries[3, 0] = lay.n_pages + 7
        vis.entries[30, 0] = -2  # a local-head entry
        o = torch.zeros_like(q)
        binding.segpaged_prefill(hl, q, k, v, vis, ws, o, fuse_rope=fuse)
        torch.cuda.synchronize()
        assert binding.device_status(ws) & binding.RK_DEV_BAD_PAGE
        assert torch.isfinite(o.float()).all()


def test_bounded_wait_gives_up_and_context_survives():
    """The kernels' bounded wait on a barrier that nothing completes raises
    RK_DEV_TIMEOUT and returns; the context is usable afterwards."""
    from head_aware_paged_prefill_b200 import binding
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.selftest_bounded_wait(word, 20)
    torch.cuda.synchronize()
    assert int(word.item()) == binding.RK_DEV_TIMEOUT
    wl = synth.cfg1()
    q, k, v = (t.cuda() for t in wl.materialize("cpu"))
    run = PrefillRun(wl.layout, q, k, v, mode="fused")
    assert run.status == 0
