"""rk_segpaged_decode (one row per request: its last position) against the
fp64 oracle's attention at that row, on the relocated pools and the page
tables the prefill path uses.  Tables whose request ends in a cached segment
(the last position is not one of their rows) must leave o untouched."""
import numpy as np
import pytest
import torch

from head_aware_paged_prefill_b200 import binding, synth
from gpu_util import SENTINEL, PrefillRun, assert_close, oracle_rows

pytestmark = pytest.mark.gpu


def _decode(run, lay, q):
    """Decode of every request's last row through the C ABI."""
    dev = q.device
    last = [int(lay.cu_seqlens[r + 1]) - 1 for r in range(lay.n_req)]
    q_dec = torch.zeros((lay.n_layers, lay.n_req, lay.hq, lay.d), dtype=torch.bfloat16, device=dev)
    for r, i in enumerate(last):
        if lay.req_len(r) > 0:
            q_dec[:, r] = q[:, i]
    o = torch.full(q_dec.shape, SENTINEL, dtype=torch.int16, device=dev).view(torch.bfloat16)
    lse = torch.full((lay.n_layers, lay.hq, lay.n_req), float("nan"), device=dev)
    sizes = binding.decode_sizes(run.hl)
    ws = binding.decode_workspace(sizes, dev)
    binding.segpaged_decode(run.hl, q_dec, run.k_rel, run.v_rel, run.vis, ws, o, lse)
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0
    return o, lse, last


def _check(lay, q, k, v, what):
    run = PrefillRun(lay, q, k, v, mode="relocate")
    assert run.status == 0
    o, lse, last = _decode(run, lay, q)
    rows = np.array([(layer, h, last[r]) for r in range(lay.n_req) if lay.req_len(r) > 0
                     for layer in range(lay.n_layers) for h in range(lay.hq)], dtype=np.int32)
    o_ref, lse_ref, comp = oracle_rows(lay, q.cpu(), k.cpu(), v.cpu(), rows)
    req_of = {last[r]: r for r in range(lay.n_req)}
    got = np.stack([o[l, req_of[t], h].double().cpu().numpy() for l, h, t in rows])
    got_lse = np.array([float(lse[l, h, req_of[t]]) for l, h, t in rows])
    if comp.any():
        assert_close(got[comp == 1], o_ref[comp == 1], f"{what} decode o")
        assert np.abs(got_lse[comp == 1] - lse_ref[comp == 1]).max() <= 1e-2, f"{what} lse"
        # the prefill's own last row agrees with the decode row
        pre = np.stack([run.o[l, t, h].double().cpu().numpy() for l, h, t in rows])
        assert np.abs(pre[comp == 1] - got[comp == 1]).max() <= 2e-2
    untouched = o.view(torch.int16).cpu().numpy()
    for (l, h, t), c in zip(rows, comp):
        if not c:
            assert (untouched[l, req_of[t], h] == SENTINEL).all(), f"{what}: row written"
    return int(comp.sum())


def test_decode_cfg1():
    wl = synth.cfg1()
    q, k, v = wl.materialize("cpu")
    assert _check(wl.layout, q.cuda(), k.cuda(), v.cuda(), "cfg1") > 0


@pytest.mark.parametrize("name", ["cfg2", "cfg3", "cfg4"])
def test_decode_full_size(name):
    wl = synth.CONFIGS[name]()
    q, k, v = wl.materialize("cuda")
    n = _check(wl.layout, q, k, v, name)
    assert n == wl.layout.hq  # one request, one layer: every head's last row


def test_decode_random_small():
    rng = np.random.default_rng(31)
    total = 0
    for n in range(40):
        lay = synth.random_small(rng, max_pages=40)
        wl = synth.tiny_workload(lay, seed=n)
        q, k, v = wl.materialize("cpu")
        total += _check(lay, q.cuda(), k.cuda(), v.cuda(), f"random layout {n}")
    assert total > 0


def test_decode_rejects_on_host():
    lay = synth.cfg1().layout
    hl = binding.HostLayout(lay)
    with pytest.raises(binding.RkError):
        binding.segpaged_decode(hl, torch.zeros(1, dtype=torch.bfloat16, device="cuda"),
                                torch.zeros(1, dtype=torch.bfloat16, device="cuda"),
                                torch.zeros(1, dtype=torch.bfloat16, device="cuda"),
                                binding.Visible(hl.sizes(), "cuda"),
                                torch.zeros(16, dtype=torch.uint8, device="cuda"),
                                torch.zeros(1, dtype=torch.bfloat16, device="cuda"))
