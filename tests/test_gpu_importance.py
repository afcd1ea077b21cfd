"""rk_attention_importance (token importance for the sparse FFN and its top-k
tokens) against the fp64 oracle, on the relocated pools, page tables and lse
the prefill path produces.

Bar: elementwise |I_gpu - I_ref| <= 2e-2 * max(1, I_ref) and
sum |I_gpu - I_ref| / sum I_ref <= 5e-3.  Each weight is exp(s - lse) with s
from bf16 relocated keys (one bf16 rounding, as in the attention's own bar)
and fp32 sums of up to Hq * L terms.  The picks must equal the oracle's
wherever the k-th and (k+1)-th oracle values are further apart than the
bar; otherwise they only have to be a valid top k of the kernel's own
values.  At full size, where the oracle cannot run, the invariants hold:
every computed (q head, row) pair spreads a weight of one, and the picks are
exactly the top k of the returned importance."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from gpu_util import PrefillRun

pytestmark = pytest.mark.gpu

ABS, REL = 2e-2, 5e-3


def _u16(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _run(lay, q, k, v, top_k):
    run = PrefillRun(lay, q, k, v, mode="relocate")
    assert run.status == 0
    dev = q.device
    T = int(lay.cu_seqlens[-1])
    imp = torch.full((lay.n_layers, T), float("nan"), device=dev)
    tokens = torch.full((lay.n_layers, lay.n_req, max(top_k, 1)), -7, dtype=torch.int32, device=dev)
    count = torch.full((lay.n_layers, lay.n_req), -7, dtype=torch.int32, device=dev)
    ws = binding.importance_workspace(binding.importance_sizes(run.hl), dev)
    binding.attention_importance(run.hl, q, run.k_rel, run.vis, run.lse, ws, imp, top_k,
                                 tokens if top_k > 0 else None, count if top_k > 0 else None)
    torch.cuda.synchronize()
    assert binding.device_status(ws) == 0
    return imp.cpu().numpy().astype(np.float64), tokens.cpu().numpy(), count.cpu().numpy()


def _computed_pairs(lay, r, layer):
    g = lay.hq // lay.hkv
    L = lay.req_len(r)
    unc = np.zeros(L, dtype=bool)
    for seg in lay.segments:
        if int(seg[0]) == r and int(seg[4]) == 0:
            unc[int(seg[1]):int(seg[1]) + int(seg[2])] = True
    n = 0
    for kvh in range(lay.hkv):
        c = int(lay.class_map[layer * lay.hkv + kvh])
        n += g * (L if c in (synth.GLOBAL, synth.DENSE) else int(unc.sum()))
    return n


def _check_invariants(lay, imp, tokens, count, top_k, what):
    assert np.isfinite(imp).all() and (imp >= 0).all(), what
    for r in range(lay.n_req):
        t0, L = int(lay.cu_seqlens[r]), lay.req_len(r)
        for layer in range(lay.n_layers):
            row = imp[layer, t0:t0 + L].astype(np.float32)
            want = _computed_pairs(lay, r, layer)
            assert abs(float(row.astype(np.float64).sum()) - want) <= 1e-3 * max(want, 1), \
                f"{what}: weights of (r {r}, layer {layer}) do not sum to the row count"
            if top_k > 0:
                k = int(count[layer, r])
                assert k == min(top_k, L)
                got = tokens[layer, r, :k]
                assert got.tolist() == oracle.select_tokens(row, top_k).tolist(), \
                    f"{what}: picks are not the top k of the returned importance"


def _check_against_oracle(lay, imp, tokens, count, q, k, top_k, what):
    ref = oracle.importance(lay, _u16(q), _u16(k))
    err = np.abs(imp - ref)
    assert (err <= ABS * np.maximum(1.0, ref)).all(), f"{what}: max err {err.max():.3e}"
    assert err.sum() <= REL * max(ref.sum(), 1e-300), f"{what}: mean rel {err.sum() / ref.sum():.3e}"
    if top_k <= 0:
        return
    for r in range(lay.n_req):
        t0, L = int(lay.cu_seqlens[r]), lay.req_len(r)
        for layer in range(lay.n_layers):
            kk = min(top_k, L)
            got = tokens[layer, r, :kk].tolist()
            want = oracle.select_tokens(ref[layer, t0:t0 + L], top_k).tolist()
            srt = np.sort(ref[layer, t0:t0 + L])[::-1]
            if kk < L:
                gap = srt[kk - 1] - srt[kk] if kk > 0 else np.inf
                if gap > 2 * ABS * max(1.0, srt[kk - 1]):
                    assert got == want, f"{what}: picks differ (r {r}, layer {layer})"


def _case(wl, top_k, what):
    lay = wl.layout
    q, k, v = wl.materialize("cpu")
    imp, tokens, count = _run(lay, q.cuda(), k.cuda(), v.cuda(), top_k)
    _check_invariants(lay, imp, tokens, count, top_k, what)
    _check_against_oracle(lay, imp, tokens, count, q, k, top_k, what)


def test_importance_cfg1():
    _case(synth.cfg1(), 32, "cfg1")


def test_importance_retrieval_layout():
    segs = [(f"c{i}", 32, 7 * i, True) for i in range(4)] + [("tail", 20, 0, False)]
    lay = synth._make_layout(n_layers=1, hq=2, hkv=1, d=16 * 4, p=16, theta=1e4,
                             requests=[segs], class_map=[synth.RETRIEVAL], window=0,
                             retrieval={0: [1, 3, 6, 8]})
    _case(synth.tiny_workload(lay, seed=3), 10, "retrieval")


def test_importance_random_small():
    rng = np.random.default_rng(41)
    for n in range(24):
        lay = synth.random_small(rng, max_pages=12)
        _case(synth.tiny_workload(lay, seed=500 + n), int(rng.integers(0, 40)), f"random {n}")


def test_importance_top_k_edges():
    wl = synth.cfg1()
    lay = wl.layout
    q, k, v = wl.materialize("cuda")
    L = lay.req_len(0)
    for top_k in (0, 1, L - 1, L, L + 5):
        imp, tokens, count = _run(lay, q, k, v, top_k)
        _check_invariants(lay, imp, tokens, count, top_k, f"top_k {top_k}")
        if top_k >= L:
            assert tokens[0, 0, :L].tolist() == list(range(L))


def _multi_chunk_layout(kind: str):
    """Layouts whose tables span several row chunks of the column-sum kernel
    (a chunk holds 8192 (row, q head) columns, 8192 / G rows), so partial
    sums from different chunks and key blocks must land in the right slots.
      "g4": Hq 12, Hkv 3 (G 4, 2048-row chunks), L 6220: one global, one
            local (W 1536) and one retrieval head (16 cached pages), tail
            ending mid-page.
      "g8": Hq 16, Hkv 2 (G 8, 1024-row chunks), L 4100: a dense and a local
            (W 700) head, P 16, D 128."""
    if kind == "g4":
        segs = [(f"c{i}", 1024, 512 * i, True) for i in range(5)] + [("tail", 1100, 0, False)]
        picks = [1, 4, 9, 15, 22, 30, 37, 41, 50, 55, 58, 61, 66, 70, 74, 79]
        lay = synth._make_layout(n_layers=1, hq=12, hkv=3, d=64, p=64, theta=1e6,
                                 requests=[segs],
                                 class_map=[synth.GLOBAL, synth.LOCAL, synth.RETRIEVAL],
                                 window=1536, retrieval={2: picks})
    else:
        segs = [(f"c{i}", 1024, 3000 - 1000 * i, True) for i in range(3)] + [("tail", 1028, 0, False)]
        lay = synth._make_layout(n_layers=1, hq=16, hkv=2, d=128, p=16, theta=1e4,
                                 requests=[segs], class_map=[synth.DENSE, synth.LOCAL],
                                 window=700)
    return synth.tiny_workload(lay, seed=77 if kind == "g4" else 78)


@pytest.mark.parametrize("kind", ["g4", "g8"])
def test_importance_multi_chunk_against_oracle(kind):
    """Element by element against the oracle on layouts of 3-4 row chunks
    (the full-size cases below can only check invariants)."""
    wl = _multi_chunk_layout(kind)
    lay = wl.layout
    g = lay.hq // lay.hkv
    assert lay.req_len(0) > 2 * (8192 // g)  # at least three chunks
    _case(wl, lay.req_len(0) // 4, f"multi-chunk {kind}")


@pytest.mark.parametrize("name", ["cfg2", "cfg3", "cfg4", "cfg5"])
def test_importance_full_size_invariants(name):
    wl = synth.CONFIGS[name]()
    lay = wl.layout
    q, k, v = wl.materialize("cuda")
    top_k = lay.req_len(0) // 4
    imp, tokens, count = _run(lay, q, k, v, top_k)
    _check_invariants(lay, imp, tokens, count, top_k, name)
    del q, k, v
    torch.cuda.empty_cache()


def test_importance_deterministic():
    wl = synth.cfg1()
    q, k, v = wl.materialize("cuda")
    a = _run(wl.layout, q, k, v, 16)
    b = _run(wl.layout, q, k, v, 16)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_importance_through_api():
    """SegPagedPrefill.attention_importance after a prefill with lse: the
    same bar against the oracle, and the same invariants."""
    from head_aware_paged_prefill_b200.api import SegPagedPrefill
    wl = synth.cfg1()
    lay = wl.layout
    q, k, v = wl.materialize("cpu")
    pre = SegPagedPrefill(lay, "cuda", with_lse=True)
    pre.load(q.cuda(), k.cuda(), v.cuda())
    pre.compute()
    imp, tokens, count = pre.attention_importance(24)
    torch.cuda.synchronize()
    assert pre.importance_status() == 0
    imp = imp.cpu().numpy().astype(np.float64)
    tokens, count = tokens.cpu().numpy(), count.cpu().numpy()
    _check_invariants(lay, imp, tokens, count, 24, "api")
    _check_against_oracle(lay, imp, tokens, count, q, k, 24, "api")


def test_importance_rejects_on_host():
    lay = synth.cfg1().layout
    hl = binding.HostLayout(lay)
    vis = binding.Visible(hl.sizes(), "cuda")
    z = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(1, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.RkError):
        binding.attention_importance(hl, z, z, vis, f, torch.zeros(16, dtype=torch.uint8,
                                                                    device="cuda"), f, 4)
