"""Pins of the fp64 token-selective FFN oracle (oracle.sparse_ffn).

Reading (README "About", Elastic Sparsity / Sparse FFN; paooo page, "main
functions"): a listed row takes y = x + W_down (silu(W_gate x) * W_up x), the
gated SiLU MLP of the Mistral / Qwen3 families the pages name; every other
row keeps x (the residual path).  The pins fix it without restating it:
values worked out by hand, the odd-part identity silu(z) - silu(-z) = z
(which turns a mirrored pair of features into a plain bilinear form that
numpy evaluates directly), a zero gate, and a scaled down-projection."""
import numpy as np
import torch

import oracle


def _bf(a):
    """bf16 bits of an array (values chosen exactly representable where a
    test writes them by hand)."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _f(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def test_one_feature_by_hand():
    # x = (1, 2); gate row (1, 0) -> g = 1; up row (0, 1) -> u = 2;
    # h = silu(1) * 2 = 2 / (1 + e^-1) = 1.4621171572600098;
    # down column (1, 1) adds h to both features
    y = oracle.sparse_ffn(_bf([[1.0, 2.0]]), [0], _bf([[1.0, 0.0]]), _bf([[0.0, 1.0]]),
                          _bf([[1.0], [1.0]]))
    np.testing.assert_allclose(y, [[2.4621171572600098, 3.4621171572600098]], rtol=0, atol=1e-14)


def test_two_features_by_hand():
    # x = (2, -1); gate rows (1, 0), (0, 1) -> g = (2, -1); up rows (1, 1),
    # (0, -1) -> u = (1, 1); h = (silu(2), silu(-1)) = (2 / (1 + e^-2),
    # -1 / (1 + e)) = (1.7615941559557646, -0.2689414213699951);
    # down rows (1, 0), (0, 2): y = (2 + h0, -1 + 2 h1)
    y = oracle.sparse_ffn(_bf([[2.0, -1.0]]), [0], _bf([[1.0, 0.0], [0.0, 1.0]]),
                          _bf([[1.0, 1.0], [0.0, -1.0]]), _bf([[1.0, 0.0], [0.0, 2.0]]))
    np.testing.assert_allclose(y, [[3.7615941559557646, -1.5378828427399902]], rtol=0, atol=1e-14)


def test_mirrored_features_give_a_bilinear_form():
    """Two features with gate rows w and -w, the same up row v and down
    columns a and -a contribute a (silu(g) - silu(-g)) u = a g u, with
    g = w.x and u = v.x: silu's odd part is the identity."""
    rng = np.random.default_rng(5)
    dm, n = 24, 7
    x = _bf(rng.standard_normal((n, dm)))
    w = rng.standard_normal(dm)
    v = rng.standard_normal(dm)
    a = rng.standard_normal(dm)
    wg = _bf(np.stack([w, -w]))
    wu = _bf(np.stack([v, v]))
    wd = _bf(np.stack([a, -a], axis=1))
    y = oracle.sparse_ffn(x, np.arange(n), wg, wu, wd)
    xd, wgd, wud, wdd = _f(x), _f(wg), _f(wu), _f(wd)
    g = xd @ wgd[0]
    u = xd @ wud[0]
    want = xd + (g * u)[:, None] * wdd[:, 0][None, :]
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)


def test_zero_gate_is_the_residual_path():
    rng = np.random.default_rng(6)
    dm, df = 16, 40
    x = _bf(rng.standard_normal((5, dm)))
    y = oracle.sparse_ffn(x, [4, 0, 2], _bf(np.zeros((df, dm))), _bf(rng.standard_normal((df, dm))),
                          _bf(rng.standard_normal((dm, df))))
    np.testing.assert_array_equal(y, _f(x)[[4, 0, 2]])


def test_down_projection_scales_the_update_and_rows_follow_the_list():
    rng = np.random.default_rng(7)
    dm, df = 16, 40
    x = _bf(rng.standard_normal((6, dm)))
    wg = _bf(rng.standard_normal((df, dm)) * 0.3)
    wu = _bf(rng.standard_normal((df, dm)) * 0.3)
    wd_f = rng.standard_normal((dm, df)) * 0.2
    y1 = oracle.sparse_ffn(x, [1, 3, 5], wg, wu, _bf(wd_f))
    y2 = oracle.sparse_ffn(x, [5, 1, 3], wg, wu, _bf(2.0 * wd_f))
    xd = _f(x)
    d1 = y1 - xd[[1, 3, 5]]
    d2 = y2 - xd[[5, 1, 3]]
    np.testing.assert_allclose(d2[[1, 2, 0]], 2.0 * d1, rtol=1e-12, atol=1e-12)
    assert np.abs(d1).max() > 1e-3
