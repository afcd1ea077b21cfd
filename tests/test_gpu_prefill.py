"""rk_segpaged_prefill (K3) against the fp64 oracle, element by element.

The CUDA path runs K2 (relocation of every cached page with delta != 0),
K1 on the relocated layout and K3; the oracle runs on the original layout and
rotates the stored keys itself, so the comparison covers all three calls."""
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


def test_prefill_cfg1_all_rows():
    wl = synth.cfg1()
    lay = wl.layout
    q, k, v = wl.materialize("cpu")
    run = PrefillRun(lay, q.cuda(), k.cuda(), v.cuda())
    _check(lay, q, k, v, run, _all_rows(lay), "cfg1")
    _untouched(lay, run)


def test_prefill_random_small_all_rows():
    rng = np.random.default_rng(7)
    for n in range(40):
        lay = synth.random_small(rng, max_pages=12)
        wl = synth.tiny_workload(lay, seed=n)
        q, k, v = wl.materialize("cpu")
        run = PrefillRun(lay, q.cuda(), k.cuda(), v.cuda())
        rows = _all_rows(lay)
        if rows.shape[0]:
            _check(lay, q, k, v, run, rows, f"random layout {n}")
        _untouched(lay, run)


@pytest.mark.parametrize("name,per_table", [("cfg2", 24), ("cfg3", 16), ("cfg4", 16),
                                            ("cfg5", 3)])
def test_prefill_full_size_sampled(name, per_table):
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    q, k, v = wl.materialize("cuda")
    run = PrefillRun(lay, q, k, v)
    rows = sample_rows(lay, per_table, seed=11)
    # the oracle needs the sampled queries and the pools on the host
    _check(lay, q, k.cpu(), v.cpu(), run, rows, name)
    _untouched(lay, run)


def test_prefill_deterministic():
    wl = synth.cfg1()
    q, k, v = (t.cuda() for t in wl.materialize("cpu"))
    a = PrefillRun(wl.layout, q, k, v)
    b = PrefillRun(wl.layout, q, k, v)
    assert torch.equal(a.o.view(torch.int16), b.o.view(torch.int16))
