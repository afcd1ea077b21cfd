"""The no-allocation page-table entry point (rk_select_visible_noalloc).

It serves callers that cannot allocate device memory (a framework that owns
every allocation, or a thread that must avoid the synchronisation a
cudaMalloc can bring): its scratch is a fixed 1 MiB array inside the library.
Its outputs must equal rk_select_visible's, bit for bit, and a second call must
not see anything left over from the first.  This file is collected last so a
run that stops at the first failure has run every other test before it.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from head_aware_paged_prefill_b200 import binding, synth


def _tables_with(lay, noalloc: bool):
    hl = binding.HostLayout(lay)
    s = hl.sizes()
    vis = binding.Visible(s, "cuda")
    if noalloc:
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        binding.select_visible_noalloc(hl, vis, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    else:
        ws = binding.workspace(s, "cuda")
        binding.select_visible(hl, vis, ws)
        torch.cuda.synchronize()
        assert binding.device_status(ws) == 0
    return vis.tables()


@pytest.mark.gpu
def test_noalloc_matches_select_visible_on_two_calls():
    # two calls in a row; the second layout is much smaller than the first, so
    # anything stale in the shared scratch would show up in its tables
    for name in ("cfg4", "cfg1"):
        lay = synth.CONFIGS[name]().layout
        got_e, got_r = _tables_with(lay, noalloc=True)
        want_e, want_r = _tables_with(lay, noalloc=False)
        assert len(got_e) == len(want_e) == lay.n_tables
        for t in range(lay.n_tables):
            np.testing.assert_array_equal(got_e[t], want_e[t], err_msg=f"{name} entries {t}")
            np.testing.assert_array_equal(got_r[t], want_r[t], err_msg=f"{name} ranges {t}")


def test_noalloc_rejects_layout_beyond_scratch():
    # 300 segments x 1024 (layer, kv_head) page bases: a 1.2 MB layout copy
    segs = [(f"c{i}", 16, 0, True) for i in range(299)] + [("tail", 16, 0, False)]
    lay = synth._make_layout(n_layers=64, hq=16, hkv=16, d=64, p=16, theta=1e4,
                             requests=[segs], class_map=[0] * 1024, window=16)
    hl = binding.HostLayout(lay)
    s = hl.sizes()
    fake = 1 << 20  # never dereferenced: the size check fails first
    vis = binding.RkVisible(fake, fake, fake, fake, fake, fake, s.entry_capacity,
                            s.range_capacity)
    st = binding.lib().rk_select_visible_noalloc(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                                 ctypes.byref(vis), None, None)
    assert st == binding.RK_ERR_CAPACITY


@pytest.mark.gpu
def test_noalloc_rejected_call_leaves_no_trace():
    """A page id outside the pool is caught on the host (RK_ERR_INVALID_ARG)
    before any GPU work: the caller's error word keeps its old value.  The
    next, valid call rewrites the shared scratch header and reports 0."""
    lay = synth.cfg1().layout
    bad = dataclasses.replace(lay, page_base=lay.page_base.copy())
    bad.page_base[0, 0] = lay.n_pages  # the segment's pages run past the pool
    hl = binding.HostLayout(bad)
    s = binding.HostLayout(lay).sizes()
    vis = binding.Visible(s, "cuda")
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = binding.lib().rk_select_visible_noalloc(ctypes.byref(hl.dims), ctypes.byref(hl.layout),
                                                 ctypes.byref(vis.struct), ctypes.c_void_p(err.data_ptr()),
                                                 None)
    assert st == binding.RK_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert int(err.item()) == -1
    got_e, got_r = _tables_with(lay, noalloc=True)
    want_e, want_r = _tables_with(lay, noalloc=False)
    for t in range(lay.n_tables):
        np.testing.assert_array_equal(got_e[t], want_e[t])
        np.testing.assert_array_equal(got_r[t], want_r[t])
