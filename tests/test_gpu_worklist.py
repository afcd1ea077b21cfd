"""The attention work list the selection builds in the workspace: a
permutation of the per-table items, longest first inside each (request,
layer) group, the groups one after another.  Small lists are sorted by
the selection kernel's last CTA, large ones by the per-table scatter launch;
both are checked.  White-box: reads the workspace through its internal map
(a 256-byte header, then the sorted list, then the unsorted list)."""
import numpy as np
import pytest
import torch

from head_aware_paged_prefill_b200 import binding, synth

pytestmark = pytest.mark.gpu

HEADER = 256
ITEM_WORDS = 12  # q_row0, row_begin, row_end, e_begin, e_end, qh0, nh, window, layer, req, table, cost
COST_BUCKETS = 2048


def _align(x, a):
    return (x + a - 1) // a * a


def _work_lists(lay):
    hl = binding.HostLayout(lay)
    sz = hl.sizes()
    vis = binding.Visible(sz, "cuda")
    ws = binding.workspace(sz, "cuda")
    binding.select_visible(hl, vis, ws)
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0
    raw = ws.cpu().numpy().view(np.uint8)
    n_items = int(raw[4:8].view(np.int32)[0])
    cap = int(sz.item_capacity)
    sorted_off = HEADER
    tmp_off = _align(HEADER + 48 * cap, 256)
    items = raw[sorted_off:sorted_off + 48 * n_items].view(np.int32).reshape(-1, ITEM_WORDS)
    tmp = raw[tmp_off:tmp_off + 48 * n_items].view(np.int32).reshape(-1, ITEM_WORDS)
    return n_items, items, tmp, cap


def _check(lay, expect_large=None):
    n, items, tmp, cap = _work_lists(lay)
    assert 0 <= n <= cap
    if expect_large is not None:
        assert (n > 16384) == expect_large
    # a permutation of the per-table items
    key = lambda a: np.lexsort(a.T[::-1])
    assert np.array_equal(items[key(items)], tmp[key(tmp)])
    # groups in order, longest first inside a group (costs past the last
    # bucket of a group share it): a group is one (request, layer) when the
    # layout has several (up to 256), the buckets split evenly between a
    # power of two of groups
    n_groups = lay.n_req * lay.n_layers
    groups = 1
    if 1 < n_groups <= 256:
        while groups < n_groups:
            groups *= 2
    bpg = COST_BUCKETS // groups
    ept = 128 // lay.p
    max_pages = max(-(-lay.req_len(r) // lay.p) for r in range(lay.n_req))
    max_cost = -(-max_pages // ept) + 1
    width = max(1, -(-(max_cost + 1) // bpg))
    g = items[:, 9] * lay.n_layers + items[:, 8] if groups > 1 else np.zeros(len(items), np.int64)
    c = np.minimum(items[:, 11] // width, bpg - 1)
    order = g * bpg + (bpg - 1 - c)
    assert np.all(order[:-1] <= order[1:])
    # every item of a table lies in that table and has a cost of its entries
    assert np.all(items[:, 4] >= items[:, 3])
    assert np.all(items[:, 6] >= 1) and np.all(items[:, 6] <= 2)


@pytest.mark.parametrize("name,large", [("cfg1", False), ("cfg2", False), ("cfg4", False),
                                        ("cfg5", True)])
def test_work_list_sorted_permutation(name, large):
    _check(synth.CONFIGS[name]().layout, expect_large=large)


def test_work_list_random_small():
    rng = np.random.default_rng(77)
    for _ in range(20):
        _check(synth.random_small(rng))


@pytest.mark.parametrize("name", ["cfg1", "cfg3", "cfg5"])
def test_api_item_count_matches_library(name):
    """The API's launch accounting counts work items by the library's rule."""
    from head_aware_paged_prefill_b200.api import SegPagedPrefill
    lay = synth.CONFIGS[name]().layout
    n, _, _, _ = _work_lists(lay)
    assert SegPagedPrefill(lay, "cuda", mode="fused").n_items == n
