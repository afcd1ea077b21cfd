"""rk_relocate_rope (K2) against the oracle's fp64 R(delta) K_stored: every
element within one bf16 ulp, the max-abs / mean-relative bar on unit-scale
data, delta-0 copies bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from gpu_util import assert_bf16_rounded, assert_close, run_select, u16

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
    assert_bf16_rounded(got, want, "relocated K")
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
    assert_bf16_rounded(pool[1:3].double().cpu().numpy(), want, "in-place relocation")
    np.testing.assert_array_equal(u16(pool[3]), u16(src[3]))  # skipped job wrote nothing
    np.testing.assert_array_equal(u16(pool[4]), u16(src[4]))


def test_relocate_separate_pools_bounds():
    g = torch.Generator().manual_seed(6)
    store = torch.randn((8, 16, 64), generator=g).to(torch.bfloat16).cuda()
    work = torch.zeros((12, 16, 64), dtype=torch.bfloat16, device="cuda")
    # src 8 is outside the 8-page store though inside the 12-page working pool
    jobs = np.asarray([[7, 11, 3], [0, 0, -5], [8, 1, 2], [2, 12, 1]], dtype=np.int32)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.relocate_rope(store, work, torch.from_numpy(jobs).cuda(), 1e4, err)
    torch.cuda.synchronize()
    assert int(err.item()) == binding.RK_DEV_BAD_PAGE
    want = oracle.relocate(u16(store), jobs[:2], 16, 64, 1e4)
    assert_bf16_rounded(work[[11, 0]].double().cpu().numpy(), want, "separate pools")
    assert int(work[1].abs().sum().item()) == 0 and int(work[2].abs().sum().item()) == 0


@pytest.mark.parametrize("d", [64, 128])
def test_relocate_many_jobs_delta_runs(d):
    """More jobs than CTAs, so every CTA walks a block of jobs: runs of equal
    delta (the shared table is reused), delta changes inside a block, and
    delta-0 copies in between."""
    p, n = 16, 5000
    g = torch.Generator().manual_seed(d)
    store = torch.randn((n, p, d), generator=g).to(torch.bfloat16)
    rng = np.random.default_rng(d)
    run = rng.integers(1, 9, size=n)
    deltas = np.repeat(rng.integers(-50000, 50000, size=n), run)[:n]
    deltas[rng.choice(n, 200, replace=False)] = 0
    jobs = np.stack([np.arange(n), rng.permutation(n), deltas], 1).astype(np.int32)
    work = torch.zeros((n, p, d), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.relocate_rope(store.cuda(), work, torch.from_numpy(jobs).cuda(), 1e6, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    pick = rng.choice(n, 400, replace=False)
    want = oracle.relocate(u16(store), jobs[pick], p, d, 1e6)
    got = work[torch.from_numpy(jobs[pick, 1]).long().cuda()].double().cpu().numpy()
    assert_bf16_rounded(got, want, "blocked jobs")
    assert_close(got, want, "blocked jobs")
    z = jobs[jobs[:, 2] == 0][:20]
    np.testing.assert_array_equal(u16(work[torch.from_numpy(z[:, 1]).long().cuda()]),
                                  u16(store[torch.from_numpy(z[:, 0]).long()]))


@pytest.mark.parametrize("name", ["cfg2", "cfg3"])
def test_relocate_full_plan_sampled(name):
    """The plan of the full-size layout (rk_relocation_plan): the
    rotated pages match the oracle, and every page no K job writes still holds
    the store's bits."""
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    _, k_pool, _ = wl.materialize("cuda")
    plan = binding.relocation_plan(lay)
    jobs = plan.jobs_k
    work = torch.cat([k_pool, torch.zeros((plan.n_extra, lay.p, lay.d), dtype=torch.bfloat16,
                                          device="cuda")])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.relocate_rope(k_pool, work, torch.from_numpy(jobs).cuda(), lay.theta, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    pick = np.random.default_rng(0).choice(jobs.shape[0], 64, replace=False)
    sub = jobs[pick]
    want = oracle.relocate(u16(k_pool), sub, lay.p, lay.d, lay.theta)
    got = work[torch.from_numpy(sub[:, 1]).long().cuda()].double().cpu().numpy()
    assert_bf16_rounded(got, want, f"{name} relocation")
    # the max-abs / mean-relative bar is stated for unit-scale data: a layout
    # whose pages carry a K scale is compared after dividing it out
    if lay.kv_page_scale is not None:
        sc = lay.kv_page_scale[sub[:, 0]].astype(np.float64)[:, None, None]
        got, want = got / sc, want / sc
    assert_close(got, want, f"{name} relocation")
    untouched = np.setdiff1d(np.arange(lay.n_pages), jobs[:, 1])
    idx = torch.from_numpy(untouched).long().cuda()
    assert torch.equal(work[idx].view(torch.int16), k_pool[idx].view(torch.int16))
