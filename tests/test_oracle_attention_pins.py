"""Pins of the fp64 Spark Attention oracle (one decoding position) against what the paper-notes page
("Spark Transformer: Reactivating Sparsity in FFN and Attention", 关键设计 / "Spark Attention" and
"Statistical Top-k") and the mathematics fix: closed forms of softplus, the reduction of the dense case
to library attention, selection = sorted top-m, invariants, grouped heads, degenerate rows and a brute
force on tiny inputs.  No GPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def widen(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bits)


def make(n_heads, n_kv, n_ctx, d_head, seed):
    rng = np.random.default_rng(seed)
    q = bf16_bits(rng.standard_normal((n_heads, d_head)))
    K = bf16_bits(rng.standard_normal((n_kv, n_ctx, d_head)))
    V = bf16_bits(rng.standard_normal((n_kv, n_ctx, d_head)))
    return q, K, V


def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    for a in (-30.0, -3.5, -0.25, 0.5, 7.0, 40.0):
        # softplus(a) - softplus(-a) = a, and softplus(a) = log(1 + e^a) where that is representable
        assert oracle.softplus(a) - oracle.softplus(-a) == pytest.approx(a, rel=1e-12, abs=1e-15)
        assert oracle.softplus(a) == pytest.approx(float(np.logaddexp(0.0, a)), rel=1e-14)


def test_dense_case_is_library_attention_with_constant_gate():
    """k_attn >= n_ctx selects every key.  With the K2 block of every key zero, a_j = 0 and
    softplus(a_j) = ln 2, so out = ln 2 * softmax(scale * q[:r] K1^T) V: the library's attention."""
    n_heads, n_kv, n_ctx, d_head, r = 4, 2, 40, 16, 8
    q, K, V = make(n_heads, n_kv, n_ctx, d_head, 1)
    K = K.copy()
    K[:, :, r:] = 0
    scale = 0.37
    res = oracle.spark_attention(q, K, V, r, k_attn=n_ctx, scale=scale)
    assert np.all(res["active"])
    qq = torch.from_numpy(widen(q)[:, :r]).reshape(1, n_heads, 1, r)
    kk = torch.from_numpy(widen(K)[:, :, :r]).repeat_interleave(n_heads // n_kv, dim=0).reshape(1, n_heads, n_ctx, r)
    vv = torch.from_numpy(widen(V)).repeat_interleave(n_heads // n_kv, dim=0).reshape(1, n_heads, n_ctx, d_head)
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale).reshape(n_heads, d_head).numpy()
    np.testing.assert_allclose(res["out"], math.log(2.0) * ref, rtol=1e-11, atol=1e-13)


def test_selection_is_the_sorted_top_m():
    """A threshold keeps a prefix of the scores sorted in descending order."""
    for seed in range(40):
        q, K, V = make(2, 1, 64, 8, 100 + seed)
        res = oracle.spark_attention(q, K, V, 4, k_attn=6, scale=1.0)
        for h in range(2):
            s, act = res["s"][h], res["active"][h]
            m = int(act.sum())
            top = np.argsort(-s, kind="stable")[:m]
            assert set(np.flatnonzero(act)) == set(top.tolist())
            assert np.all(s[act] > res["theta"][h]) and np.all(s[~act] <= res["theta"][h])


def test_count_within_theorem_bound_on_gaussian_scores():
    """Statistical top-k selects about k_attn keys: |m - k| <= sqrt(n ln n) (constant 1)."""
    n_ctx, k = 4096, 256
    q, K, V = make(8, 4, n_ctx, 32, 5)
    res = oracle.spark_attention(q, K, V, 16, k_attn=k, scale=1.0 / math.sqrt(32), n_threads=4)
    counts = res["active"].sum(axis=1)
    assert np.all(np.abs(counts - k) <= math.sqrt(n_ctx * math.log(n_ctx))), counts


def test_key_permutation_and_linearity_in_v():
    q, K, V = make(4, 2, 96, 16, 9)
    base = oracle.spark_attention(q, K, V, 8, k_attn=12, scale=0.5)["out"]
    perm = np.random.default_rng(3).permutation(96)
    permuted = oracle.spark_attention(q, K[:, perm], V[:, perm], 8, k_attn=12, scale=0.5)["out"]
    np.testing.assert_allclose(permuted, base, rtol=1e-12, atol=1e-14)
    # out is linear in V: V -> 2 V (exact in bf16) doubles it
    V2 = bf16_bits(2.0 * widen(V))
    doubled = oracle.spark_attention(q, K, V2, 8, k_attn=12, scale=0.5)["out"]
    np.testing.assert_allclose(doubled, 2.0 * base, rtol=1e-13, atol=1e-15)


def test_grouped_heads_share_their_key_value_head():
    """Heads 2g and 2g+1 read key/value head g; with the same query they give the same output, and
    each equals a one-head call on that key/value head alone."""
    q, K, V = make(4, 2, 80, 16, 11)
    q = q.copy()
    q[1] = q[0]
    res = oracle.spark_attention(q, K, V, 8, k_attn=10, scale=0.25)
    np.testing.assert_array_equal(res["out"][0], res["out"][1])
    for h in range(4):
        one = oracle.spark_attention(q[h:h + 1], K[h // 2:h // 2 + 1], V[h // 2:h // 2 + 1], 8, k_attn=10,
                                     scale=0.25)
        np.testing.assert_array_equal(one["out"][0], res["out"][h])


def test_degenerate_scores_select_nothing():
    """Identical predictor keys give scores of zero spread: theta = mean, nothing passes, out = 0."""
    q, K, V = make(2, 1, 50, 8, 13)
    K = K.copy()
    K[0, :, :4] = K[0, 0, :4]
    res = oracle.spark_attention(q, K, V, 4, k_attn=5, scale=1.0)
    assert not res["active"].any() and np.all(res["out"] == 0.0)


def test_brute_force_tiny():
    """A separate plain-Python evaluation of the same definition on n_ctx = 7 keys."""
    n_ctx, d_head, r, k = 7, 6, 3, 2
    q, K, V = make(1, 1, n_ctx, d_head, 21)
    qf, Kf, Vf = widen(q)[0], widen(K)[0], widen(V)[0]
    scale = 0.8
    s = [scale * sum(Kf[j][i] * qf[i] for i in range(r)) for j in range(n_ctx)]
    mean = sum(s) / n_ctx
    sd = math.sqrt(sum((x - mean) ** 2 for x in s) / n_ctx)
    theta = mean + sd * oracle.topk_quantile(k, n_ctx)
    sel = [j for j in range(n_ctx) if s[j] > theta]
    z = sum(math.exp(s[j]) for j in sel)
    expect = [0.0] * d_head
    for j in sel:
        a = sum(Kf[j][r + i] * qf[r + i] for i in range(d_head - r))
        w = math.exp(s[j]) / z * math.log1p(math.exp(a))
        for c in range(d_head):
            expect[c] += w * Vf[j][c]
    res = oracle.spark_attention(q, K, V, r, k_attn=k, scale=scale)
    assert res["theta"][0] == pytest.approx(theta, rel=1e-13)
    np.testing.assert_allclose(res["out"][0], expect, rtol=1e-12, atol=1e-14)


def test_override_set_renormalises_over_the_given_keys():
    """override_active replaces the selected set A: the softmax weights are renormalised over the given
    keys (checked against a plain numpy evaluation), an empty set gives 0, A itself gives the plain
    result, and the reported mask stays the predictor's own (s > theta)."""
    n_heads, n_kv, n_ctx, d_head, r, k = 4, 2, 40, 16, 8, 6
    q, K, V = make(n_heads, n_kv, n_ctx, d_head, 31)
    base = oracle.spark_attention(q, K, V, r, k_attn=k, scale=0.5)
    same = oracle.spark_attention(q, K, V, r, k_attn=k, scale=0.5, override_active=base["active"])
    assert np.array_equal(same["out"], base["out"]) and np.array_equal(same["active"], base["active"])
    none = oracle.spark_attention(q, K, V, r, k_attn=k, scale=0.5,
                                  override_active=np.zeros((n_heads, n_ctx), bool))
    assert np.all(none["out"] == 0.0) and np.array_equal(none["active"], base["active"])
    # a different set: drop each head's first selected key, add its two highest unselected ones
    ov = base["active"].copy()
    for h in range(n_heads):
        on = np.flatnonzero(ov[h])
        off = np.flatnonzero(~ov[h])
        ov[h, on[0]] = False
        ov[h, off[np.argsort(base["s"][h, off])[-2:]]] = True
    res = oracle.spark_attention(q, K, V, r, k_attn=k, scale=0.5, override_active=ov)
    assert np.array_equal(res["active"], base["active"])
    qf, Kf, Vf = widen(q), widen(K), widen(V)
    for h in range(n_heads):
        g = h // (n_heads // n_kv)
        sel = np.flatnonzero(ov[h])
        s = 0.5 * (Kf[g, sel, :r] @ qf[h, :r])
        p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
        a = Kf[g, sel, r:] @ qf[h, r:]
        expect = (p * np.log1p(np.exp(a))) @ Vf[g, sel]
        np.testing.assert_allclose(res["out"][h], expect, rtol=1e-12, atol=1e-14)
