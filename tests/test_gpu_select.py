"""rk_select_visible (K1) against the oracle's brute-force page tables:
bit-exact entries and row ranges on every workload and on random layouts."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from gpu_util import run_select

pytestmark = pytest.mark.gpu


def _compare(lay):
    want_e, want_r = oracle.page_tables(lay)
    _, vis, ws = run_select(lay)
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0
    got_e, got_r = vis.tables()
    assert len(got_e) == len(want_e)
    for t in range(len(want_e)):
        np.testing.assert_array_equal(got_e[t], want_e[t], err_msg=f"entries of table {t}")
        np.testing.assert_array_equal(got_r[t], want_r[t], err_msg=f"ranges of table {t}")


@pytest.mark.parametrize("name", ["cfg1", "cfg2", "cfg3", "cfg4", "cfg5"])
def test_select_bit_exact_configs(name):
    _compare(synth.CONFIGS[name]().layout)


def test_select_bit_exact_random():
    rng = np.random.default_rng(99)
    for _ in range(200):
        _compare(synth.random_small(rng))


def test_select_edge_cases():
    # empty request in the middle, a request with no uncached rows, window 1
    reqs = [[("a", 64, 0, True), ("t0", 37, 0, False)], [],
            [("b", 64, 5, True), ("c", 128, 9, True)], [("t3", 1, 0, False)]]
    for cmap in ([0, 1, 2], [3, 2, 1]):
        lay = synth._make_layout(n_layers=1, hq=3, hkv=3, d=64, p=16, theta=1e4, requests=reqs,
                                 class_map=cmap, window=1,
                                 retrieval={0: [0, 3], 1: [1], 2: [2, 5], 7: [0, 1]})
        _compare(lay)


def test_select_is_deterministic():
    lay = synth.cfg4().layout
    _, vis1, _ = run_select(lay)
    _, vis2, _ = run_select(lay)
    torch.cuda.synchronize()
    assert torch.equal(vis1.entries, vis2.entries) and torch.equal(vis1.ranges, vis2.ranges)
