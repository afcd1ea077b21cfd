"""rk_sparse_ffn (the token-selective FFN) against the fp64 oracle.

Selected rows: max abs <= 2e-2 and mean relative <= 5e-3 against
oracle.sparse_ffn (bf16 inputs, fp32 tensor-core sums, h rounded to bf16
between the two products, the result rounded to bf16).  Every other row of
the hidden state must be bit-identical to its input (the residual path)."""
import numpy as np
import pytest
import torch

import oracle
from head_aware_paged_prefill_b200 import binding, synth
from gpu_util import assert_close, u16

pytestmark = pytest.mark.gpu


def _tokens(rng, cu, top_k, dev):
    n_req = len(cu) - 1
    tok = np.full((n_req, max(top_k, 1)), -1, dtype=np.int32)
    for r in range(n_req):
        L = cu[r + 1] - cu[r]
        k = min(top_k, L)
        tok[r, :k] = np.sort(rng.choice(L, size=k, replace=False))
    return torch.from_numpy(tok).to(dev)


def _rows(cu, tok, top_k):
    tok = tok.cpu().numpy()
    return np.concatenate([cu[r] + tok[r, :min(top_k, cu[r + 1] - cu[r])]
                           for r in range(len(cu) - 1)]).astype(np.int32)


def _run(x, cu, tok, top_k, wg, wu, wd):
    ws = binding.ffn_workspace(binding.ffn_sizes(x.shape[0], x.shape[1], wg.shape[0], cu, top_k),
                               x.device)
    y = x.clone()
    binding.sparse_ffn(y, cu, tok, top_k, wg, wu, wd, ws)
    torch.cuda.synchronize()
    return y, binding.device_status(ws)


def _check(x, y, rows, wg, wu, wd, sample=None, what=""):
    sel = rows if sample is None else rows[sample]
    ref = oracle.sparse_ffn(u16(x), sel, u16(wg), u16(wu), u16(wd))
    got = y[torch.from_numpy(sel).long().to(y.device)].double().cpu().numpy()
    assert_close(got, ref, what)
    keep = torch.ones(x.shape[0], dtype=torch.bool, device=x.device)
    keep[torch.from_numpy(rows).long().to(x.device)] = False
    assert torch.equal(y[keep].view(torch.int16), x[keep].view(torch.int16)), \
        f"{what}: unselected rows changed"


@pytest.mark.parametrize("d_model,d_ff,cu,top_k", [
    (256, 384, [0, 300, 700], 200),    # 400 rows: three full M tiles and a ragged one
    (512, 256, [0, 1000], 129),        # one row past a tile
    (256, 128, [0, 5, 90, 90, 400], 64),  # short and empty requests
])
def test_sparse_ffn_small(d_model, d_ff, cu, top_k):
    rng = np.random.default_rng(d_model + d_ff + top_k)
    x, wg, wu, wd = synth.ffn_inputs(cu[-1], d_model, d_ff, seed=11, device="cuda")
    tok = _tokens(rng, cu, top_k, "cuda")
    y, st = _run(x, cu, tok, top_k, wg, wu, wd)
    assert st == 0
    _check(x, y, _rows(cu, tok, top_k), wg, wu, wd, what=f"{d_model}x{d_ff}")


def test_sparse_ffn_edges():
    cu = [0, 200]
    x, wg, wu, wd = synth.ffn_inputs(200, 256, 128, seed=12, device="cuda")
    rng = np.random.default_rng(3)
    # top_k 0: nothing changes
    y, st = _run(x, cu, _tokens(rng, cu, 0, "cuda"), 0, wg, wu, wd)
    assert st == 0 and torch.equal(y.view(torch.int16), x.view(torch.int16))
    # top_k >= L: every row runs the FFN
    tok = torch.arange(200, dtype=torch.int32, device="cuda").view(1, -1)
    y, st = _run(x, cu, tok, 250, wg, wu, wd)
    assert st == 0
    _check(x, y, np.arange(200, dtype=np.int32), wg, wu, wd, what="all rows")
    # a position outside the request is skipped and reported
    tok = _tokens(rng, cu, 20, "cuda")
    tok[0, 5] = 999
    y, st = _run(x, cu, tok, 20, wg, wu, wd)
    assert st == binding.RK_DEV_BAD_PAGE
    rows = _rows(cu, tok, 20)
    good = rows[rows < 200]
    _check(x, y, good, wg, wu, wd, what="bad token")


def test_sparse_ffn_deterministic():
    cu = [0, 700]
    x, wg, wu, wd = synth.ffn_inputs(700, 256, 256, seed=13, device="cuda")
    tok = _tokens(np.random.default_rng(4), cu, 300, "cuda")
    a, _ = _run(x, cu, tok, 300, wg, wu, wd)
    b, _ = _run(x, cu, tok, 300, wg, wu, wd)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_sparse_ffn_full_size_sampled():
    """Mistral-7B's FFN width (d_model 4096, d_ff 14336) on the 32K layer's
    rows with the top quarter selected (the bench's launch configuration):
    sampled selected rows (tile edges included) against the oracle, every
    other row unchanged."""
    T, dm, dff, top_k = 32768, 4096, 14336, 8192
    cu = [0, T]
    x, wg, wu, wd = synth.ffn_inputs(T, dm, dff, seed=14, device="cuda")
    tok = _tokens(np.random.default_rng(5), cu, top_k, "cuda")
    y, st = _run(x, cu, tok, top_k, wg, wu, wd)
    assert st == 0
    rows = _rows(cu, tok, top_k)
    sample = np.unique(np.concatenate([[0, 127, 128, 4095, 4096, top_k - 1],
                                       np.random.default_rng(6).choice(top_k, 18, replace=False)]))
    _check(x, y, rows, wg, wu, wd, sample=sample, what="full size")


def test_importance_picks_drive_the_ffn():
    """The pipeline: prefill with lse, attention importance, then the FFN on
    the picked tokens of the layer.  The picks must be the oracle's (the
    importance values here are well separated at the cut) and the updated
    rows must match the oracle's FFN on the oracle's picks.  top_k 415 of
    the tiny layer's 448 tokens sits at a clear gap of the oracle's values
    (about 0.1, against the importance bar of 2e-2)."""
    from head_aware_paged_prefill_b200.api import SegPagedPrefill
    wl = synth.cfg1()
    lay = wl.layout
    q, k, v = wl.materialize("cpu")
    pre = SegPagedPrefill(lay, "cuda", with_lse=True)
    pre.load(q.cuda(), k.cuda(), v.cuda())
    pre.compute()
    top_k = 415
    imp, tokens, count = pre.attention_importance(top_k)
    x, wg, wu, wd = synth.ffn_inputs(lay.total_tokens, 256, 256, seed=15, device="cuda")
    y = pre.sparse_ffn(x.clone(), tokens[0], top_k, wg, wu, wd)
    torch.cuda.synchronize()
    assert pre.ffn_status() == 0
    ref_imp = oracle.importance(lay, u16(q), u16(k))[0]
    want = oracle.select_tokens(ref_imp, top_k)
    srt = np.sort(ref_imp)[::-1]
    assert srt[top_k - 1] - srt[top_k] > 4e-2 * max(1.0, srt[top_k - 1])
    assert tokens[0, 0, :top_k].cpu().numpy().tolist() == want.tolist()
    _check(x, y, want.astype(np.int32), wg, wu, wd, what="pipeline")
