"""GPU parity of the standalone statistical top-k + soft threshold against the oracle.

Workload of the attention-shaped case: 8 heads x 4096 queries = 32768 score
rows of n_ctx = 4096 fp32, k = 256, rows ~N(0,1) and Student-t(4).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import synthetic

from .parity import compare_active

pytestmark = pytest.mark.gpu


def check_rows(x_cpu, out_gpu, k, rows=None):
    """Values within the fp32 threshold error; active sets exact outside the band."""
    xs = x_cpu.numpy() if rows is None else x_cpu.numpy()[rows]
    go = out_gpu.cpu().numpy().astype(np.float64)
    go = go if rows is None else go[rows]
    ref, th, mu, sd = oracle.stat_topk(xs, k, n_threads=8)
    Q = abs(oracle.topk_quantile(k, xs.shape[1]))
    # fp32 statistics: |theta_gpu - theta| <= 64 u (|mu| + sd (1 + |Q|)) with u = 2^-24 (a few
    # dozen rounding steps in the sums and merges); plus the fp32 rounding of x - theta
    tol = (64 * 2.0 ** -24 * (np.abs(mu) + sd * (1 + Q)) + 2.0 ** -23 * np.abs(th))[:, None] + \
        2.0 ** -23 * np.abs(xs.astype(np.float64))
    assert np.all(np.abs(go - ref) <= tol)
    cmp = compare_active(go > 0, xs.astype(np.float64), th, sd)
    assert cmp["outside_band"] == 0, cmp
    return cmp


@pytest.mark.parametrize("rows,d,k", [(64, 4096, 256), (33, 1024, 82), (5, 8192, 655), (7, 4097, 256),
                                      (9, 1000, 80), (3, 7, 1), (2, 2, 1), (4, 12000, 960), (1, 96, 95)])
def test_shapes(rows, d, k):
    x = synthetic.score_rows(rows, d, base=rows * 7 + d)
    out = spark.stat_topk_soft_threshold(x.cuda(), k)
    check_rows(x, out, k)


def test_in_place_and_misaligned():
    x = synthetic.score_rows(16, 4096, base=3)
    xg = x.cuda()
    spark.stat_topk_soft_threshold(xg, 256, out=xg)
    check_rows(x, xg, 256)
    # rows that start at an odd float offset take the generic kernel
    buf = torch.zeros(16 * 4096 + 1, device="cuda")
    buf[1:] = x.cuda().reshape(-1)
    out = torch.empty(16 * 4096 + 1, device="cuda")
    spark.stat_topk_soft_threshold(buf[1:].view(16, 4096), 256, out=out[1:].view(16, 4096))
    check_rows(x, out[1:].view(16, 4096), 256)


def test_constant_and_shifted_rows():
    x = torch.full((4, 4096), 3.25)
    x[1] = -7.0
    x[2, :] = torch.linspace(1000.0, 1000.001, 4096)  # |mean| >> std
    x[3] = synthetic.score_rows(1, 4096, base=9)[0] * 1e-3 + 1e4
    out = spark.stat_topk_soft_threshold(x.cuda(), 256)
    assert torch.all(out[0] == 0) and torch.all(out[1] == 0)
    check_rows(x, out, 256)


@pytest.mark.parametrize("dist", ["normal", "student_t4"])
def test_attention_shaped_full_size_sampled(dist):
    rows, d, k = 8 * 4096, 4096, 256
    x = synthetic.score_rows(rows, d, dist=dist)
    out = spark.stat_topk_soft_threshold(x.cuda(), k)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    sample = np.sort(rng.choice(rows, size=128, replace=False))
    cmp = check_rows(x, out, k, rows=sample)
    counts = (out > 0).sum(dim=1).double()
    if dist == "normal":
        # Theorem 3.1 (C = 1) on every row; mean count near k
        assert float((counts - k).abs().max()) <= math.sqrt(d * math.log(d))
        assert abs(float(counts.mean()) - k) < 2.0
    else:
        # heavy tails: t4 has std sqrt(2); expected count d * P(t4 > sqrt(2) Q) ~ 196 < k
        assert 150 < float(counts.mean()) < 240


# ---------------------------------------------------------------- causal mask
def check_causal(x_cpu, out_gpu, th_gpu, k, n_q, offset, rows=None):
    """Against the oracle's causal operator: kept values within the fp32 threshold error, active sets
    exact outside the band, rows with at most k visible entries passed through bit for bit, masked 0."""
    idx = np.arange(x_cpu.shape[0]) if rows is None else np.asarray(rows)
    xs = x_cpu.numpy()[idx]
    go = out_gpu.cpu().numpy()[idx].astype(np.float64)
    gth = th_gpu.cpu().numpy()[idx].astype(np.float64)
    d = xs.shape[1]
    # the oracle on each sampled row, at its own position (n_q = 1 with the row's offset)
    for t, i in enumerate(idx):
        pos = offset + int(i) % n_q
        n = min(d, pos + 1)
        ref, rth = oracle.stat_topk_causal(xs[t:t + 1], k, n_q=1, offset=pos)
        assert np.all(go[t, n:] == 0.0), i
        if n <= k:
            assert gth[t] == -np.inf and np.array_equal(go[t, :n], xs[t, :n].astype(np.float64)), i
            continue
        xv = xs[t, :n].astype(np.float64)
        mu, sd = xv.mean(), xv.std()
        Q = abs(oracle.topk_quantile(k, n))
        tol = 64 * 2.0 ** -24 * (abs(mu) + sd * (1 + Q)) + 2.0 ** -23 * abs(rth[0]) + 2.0 ** -23 * np.abs(xv)
        assert np.all(np.abs(go[t, :n] - ref[0, :n]) <= tol), i
        assert abs(gth[t] - rth[0]) <= 64 * 2.0 ** -24 * (abs(mu) + sd * (1 + Q)) + 2.0 ** -23 * abs(rth[0]), i
        cmp = compare_active((go[t:t + 1, :n] > 0), xv[None, :], rth, np.array([sd]))
        assert cmp["outside_band"] == 0, (i, cmp)


@pytest.mark.parametrize("rows,d,k,n_q,offset", [
    (512, 512, 64, 512, 0),        # square causal scores of one prompt, vectorised path
    (64, 4096, 256, 64, 4032),     # the last 64 queries of a 4096-position context
    (300, 1000, 80, 300, 0),       # visible prefixes ending inside a 16-byte group
    (130, 4097, 256, 130, 3967),   # d % 4 != 0: generic path
    (96, 9000, 700, 48, 8900),     # longer than the register budget: generic path, two heads
    (40, 24, 5, 8, 0),             # tiny rows, five heads
])
def test_causal_shapes(rows, d, k, n_q, offset):
    x = synthetic.score_rows(rows, d, base=rows + d)
    out = torch.empty_like(x, device="cuda")
    th = torch.empty(rows, dtype=torch.float32, device="cuda")
    spark.stat_topk_soft_threshold_causal(x.cuda(), k, n_q=n_q, offset=offset, out=out, theta=th)
    torch.cuda.synchronize()
    sample = None if rows <= 160 else np.unique(np.r_[np.arange(0, 80), np.linspace(0, rows - 1, 60).astype(int)])
    check_causal(x, out, th, k, n_q, offset, rows=sample)


def test_causal_in_place_and_misaligned():
    x = synthetic.score_rows(70, 256, base=3)
    ref = torch.empty_like(x, device="cuda")
    th = torch.empty(70, dtype=torch.float32, device="cuda")
    spark.stat_topk_soft_threshold_causal(x.cuda(), 20, n_q=70, offset=100, out=ref, theta=th)
    xg = x.cuda()
    spark.stat_topk_soft_threshold_causal(xg, 20, n_q=70, offset=100, out=xg)  # in place
    buf = torch.empty(70 * 256 + 1, device="cuda")
    buf[1:].copy_(x.flatten())
    mis = torch.empty(70 * 256 + 1, device="cuda")
    spark.stat_topk_soft_threshold_causal(buf[1:].view(70, 256), 20, n_q=70, offset=100, out=mis[1:].view(70, 256))
    torch.cuda.synchronize()
    assert torch.equal(xg, ref)
    check_causal(x, mis[1:].view(70, 256), th, 20, 70, 100)


def test_causal_attention_workload_sampled():
    """8 heads x 4096 queries over 4096 positions (square causal scores), k = 256: sampled rows of
    every head against the oracle, the first queries (at most k visible keys) passed through."""
    rows, d, k = 8 * 4096, 4096, 256
    x = synthetic.score_rows(rows, d, base=21)
    xg = x.cuda()
    out = torch.empty_like(xg)
    th = torch.empty(rows, dtype=torch.float32, device="cuda")
    spark.stat_topk_soft_threshold_causal(xg, k, n_q=4096, out=out, theta=th)
    torch.cuda.synchronize()
    assert spark.query_status() == 0
    sample = np.unique(np.r_[[0, 1, 255, 256, 257, 4095, 4096, 4096 + 256], rng_rows(rows, 48)])
    check_causal(x, out, th, k, 4096, 0, rows=sample)


def rng_rows(rows, n):
    return np.random.default_rng(7).integers(0, rows, n)
