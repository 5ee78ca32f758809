"""Pins for the oracle's causal statistical top-k (oracle.stat_topk_causal).

"Statistical Top-k" on attention-shaped score rows under a causal mask: row i
is query i mod n_q of its head at position offset + i mod n_q and sees that
many entries plus one (capped at d); the threshold theta = mean + std Q(1 - k/n)
is taken over the n visible entries ("Spark Attention": a token attends to at
most k_attn tokens, min{k_attn, n_ctx}); rows with n <= k keep every visible
entry.  Each test names what fixes the expected value: a sort (brute force), a
library routine on a standardised prefix, the non-causal operator on full
rows, or an invariant.  CPU only.
"""
import math

import numpy as np
import pytest
import scipy.special as sp

import oracle


def _rows(rng, rows, d):
    return rng.standard_normal((rows, d)).astype(np.float32)


def test_selection_is_the_sorted_top_m_of_the_visible_prefix():
    rng = np.random.default_rng(11)
    for d, k in ((8, 1), (8, 3), (16, 2), (40, 5), (40, 13)):
        x = _rows(rng, 3 * d, d)
        out, th = oracle.stat_topk_causal(x, k, n_q=d)
        for i in range(x.shape[0]):
            n = min(d, i % d + 1)
            xr = x[i, :n].astype(np.float64)
            kept = out[i, :n] > 0
            if n <= k:
                continue
            m = int(kept.sum())
            order = np.argsort(-xr, kind="stable")
            assert set(np.flatnonzero(kept)) == set(order[:m]), (d, k, i)
            # one threshold for every kept entry: x - out is constant there
            if m:
                assert np.allclose(xr[kept] - out[i, :n][kept], th[i], rtol=0, atol=1e-12)
            assert np.all(out[i, n:] == 0.0)


def test_theta_closed_form_on_standardised_prefixes():
    rng = np.random.default_rng(12)
    d, n_q, k = 64, 64, 7
    x = _rows(rng, n_q, d)
    _, th = oracle.stat_topk_causal(x, k, n_q=n_q)
    for i in range(n_q):
        n = i + 1
        if n <= k:
            assert th[i] == -math.inf
            continue
        xr = x[i, :n].astype(np.float64)
        ref = xr.mean() + xr.std() * sp.ndtri(1.0 - k / n)  # numpy population std, scipy quantile
        assert th[i] == pytest.approx(ref, rel=1e-12, abs=1e-12), i


def test_rows_with_at_most_k_visible_entries_pass_through():
    rng = np.random.default_rng(13)
    d, k = 32, 10
    x = _rows(rng, 2 * d, d)
    out, th = oracle.stat_topk_causal(x, k, n_q=d)
    for i in range(2 * d):
        n = i % d + 1
        if n <= k:
            assert th[i] == -math.inf
            assert np.array_equal(out[i, :n], x[i, :n].astype(np.float64))
            assert np.all(out[i, n:] == 0.0)


def test_full_rows_equal_the_plain_operator():
    rng = np.random.default_rng(14)
    d, k = 300, 24
    x = _rows(rng, 17, d)
    out, th = oracle.stat_topk_causal(x, k, n_q=5, offset=d - 1)  # every row sees all d entries
    ref, rth, _, _ = oracle.stat_topk(x, k)
    assert np.array_equal(out, ref) and np.array_equal(th, rth)


def test_masked_entries_do_not_matter():
    rng = np.random.default_rng(15)
    d, n_q, k, off = 50, 20, 6, 9
    x = _rows(rng, 2 * n_q, d)
    y = x.copy()
    for i in range(2 * n_q):
        n = min(d, off + i % n_q + 1)
        y[i, n:] = rng.standard_normal(d - n).astype(np.float32) * 1e3
    a, ta = oracle.stat_topk_causal(x, k, n_q=n_q, offset=off)
    b, tb = oracle.stat_topk_causal(y, k, n_q=n_q, offset=off)
    assert np.array_equal(a, b) and np.array_equal(ta, tb)


def test_position_rule_heads_and_offset():
    """Rows i and i + n_q (the same query of two heads) see the same prefix; the offset shifts it."""
    rng = np.random.default_rng(16)
    d, n_q, k = 24, 6, 2
    base = _rows(rng, n_q, d)
    x = np.concatenate([base, base, base])
    out, th = oracle.stat_topk_causal(x, k, n_q=n_q, offset=3)
    assert np.array_equal(out[:n_q], out[n_q:2 * n_q]) and np.array_equal(th[:n_q], th[2 * n_q:])
    for i in range(n_q):
        n = 3 + i + 1
        assert np.all(out[i, n:] == 0.0)
        ref, rth, _, _ = oracle.stat_topk(base[i:i + 1, :n], k)
        assert np.array_equal(out[i, :n], ref[0]) and th[i] == rth[0]


def test_constant_prefix_keeps_nothing():
    d, k = 16, 3
    x = np.full((d, d), 2.5, dtype=np.float32)
    out, th = oracle.stat_topk_causal(x, k, n_q=d)
    for i in range(d):
        if i + 1 > k:
            assert th[i] == 2.5 and np.all(out[i] == 0.0)


def test_counts_on_long_gaussian_prefixes_follow_theorem_3_1():
    rng = np.random.default_rng(17)
    d, k = 4096, 256
    x = _rows(rng, 8, d)
    out, _ = oracle.stat_topk_causal(x, k, n_q=4096, offset=4088)
    for i in range(8):
        n = 4088 + i + 1
        m = int((out[i, :n] > 0).sum())
        assert abs(m - k) <= math.sqrt(n * math.log(n)), (n, m)


def test_invalid_arguments():
    x = np.zeros((2, 8), np.float32)
    for kw in ({"k": 0, "n_q": 2}, {"k": 2, "n_q": 0}, {"k": 2, "n_q": 2, "offset": -1}):
        with pytest.raises(ValueError):
            oracle.stat_topk_causal(x, **kw)
