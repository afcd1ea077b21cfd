"""rk_relocate_rope (K2) against the oracle's fp64 R(delta) K_stored."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from head_aware_paged_prefill_b200.plan import relocation_plan
from gpu_util import assert_close, u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("p,d,theta", [(16, 64, 1e4), (64, 128, 1e6), (16, 128, 1e6),
                                       (64, 64, 1e4)])
def test_relocate_random_jobs(p, d, theta):
    g = torch.Generator().manual_seed(p * d)
    n_pages = 64
    src = torch.randn((n_pages, p, d), generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(p + d)
    deltas = np.concatenate([[0, 1, -1, 65535, -65536, 4096], rng.integers(-70000, 70000, 26)])
    jobs = np.stack([rng.permutation(32), 32 + np.arange(32), deltas], 1)
    jobs = jobs.astype(np.int32)
    src_d = src.cuda()
    dst = torch.zeros_like(src_d)
    dst[:32] = src_d[:32]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.relocate_rope(src_d, dst, torch.from_numpy(jobs).cuda(), theta, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = oracle.relocate(u16(src), jobs, p, d, theta)
    got = dst[32:].double().cpu().numpy()
    assert_close(got, want, "relocated K")
    # delta = 0 copies bit-exactly
    np.testing.assert_array_equal(u16(dst[32]), u16(src[jobs[0, 0]]))


def test_relocate_in_place_and_bad_page():
    g = torch.Generator().manual_seed(5)
    src = torch.randn((8, 64, 128), generator=g).to(torch.bfloat16)
    pool = src.cuda()
    jobs = np.asarray([[1, 1, 300], [2, 2, -77], [3, 9, 5], [-1, 4, 2]], dtype=np.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.relocate_rope(pool, pool, torch.from_numpy(jobs).cuda(), 1e6, err)
    torch.cuda.synchronize()
    assert int(err.item()) == binding.RK_DEV_BAD_PAGE  # pages 9 and -1 are outside
    want = oracle.relocate(u16(src), jobs[:2], 64, 128, 1e6)
    assert_close(pool[1:3].double().cpu().numpy(), want, "in-place relocation")
    np.testing.assert_array_equal(u16(pool[3]), u16(src[3]))  # skipped job wrote nothing
    np.testing.assert_array_equal(u16(pool[4]), u16(src[4]))


@pytest.mark.parametrize("name", ["cfg2", "cfg3"])
def test_relocate_full_plan_sampled(name):
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    _, k_pool, _ = wl.materialize("cuda")
    jobs, rel = relocation_plan(lay)
    extra = rel.n_pages - lay.n_pages
    pool = torch.cat([k_pool, torch.zeros((extra, lay.p, lay.d), dtype=torch.bfloat16,
                                          device="cuda")])
    binding.relocate_rope(pool, pool, torch.from_numpy(jobs).cuda(), lay.theta)
    torch.cuda.synchronize()
    pick = np.random.default_rng(0).choice(jobs.shape[0], 64, replace=False)
    sub = jobs[pick]
    want = oracle.relocate(u16(k_pool), sub, lay.p, lay.d, lay.theta)
    got = pool[torch.from_numpy(sub[:, 1]).long().cuda()].double().cpu().numpy()
    assert_close(got, want, f"{name} relocation")
