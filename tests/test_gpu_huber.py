"""GPU parity of the Huber-smoothed statistical top-k and its backward
(stat_topk_huber, stat_topk_huber_backward) against the fp64 oracle.

"Statistical Top-k", Theorem 3.2 (continuously differentiable after a Huber
smoothing).  Error bounds follow the fp32 arithmetic: theta carries at most
eps_t = 64 u (|mean| + std (1 + |Q|)); rho is 1-Lipschitz and rho' is
(1/delta)-Lipschitz, so w = g rho'(z) carries |g| (eps_t / delta + 4 u), W their
sum, and the dtheta/dx factor c_j = 1/d + |Q| |x_j - mean| / (d std) its own
rounding.  delta = 0 uses the band of the forward tests instead (rho' is a step).
"""
import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import synthetic

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _stats(x64, k):
    d = x64.shape[1]
    mu, sd = x64.mean(axis=1), x64.std(axis=1)
    Q = oracle.topk_quantile(k, d)
    eps_t = 64 * U * (np.abs(mu) + sd * (1 + abs(Q)))
    return mu, sd, Q, eps_t


@pytest.mark.parametrize("rows,d,k,delta", [(64, 4096, 256, 0.25), (33, 1024, 82, 1.0), (9, 1000, 80, 0.05),
                                            (7, 4097, 256, 0.5), (3, 9000, 720, 0.3), (5, 4096, 256, 0.0)])
def test_huber_forward(rows, d, k, delta):
    x = synthetic.score_rows(rows, d, base=d + rows)
    out = spark.stat_topk_huber(x.cuda(), k, delta).cpu().numpy().astype(np.float64)
    x64 = x.numpy().astype(np.float64)
    ref, th = oracle.stat_topk_huber(x64, k, delta)
    _, _, _, eps_t = _stats(x64, k)
    tol = eps_t[:, None] + 2.0 ** -23 * (np.abs(x64) + np.abs(th)[:, None])
    assert np.all(np.abs(out - ref) <= tol)


@pytest.mark.parametrize("rows,d,k,delta", [(64, 4096, 256, 0.25), (33, 1024, 82, 1.0), (17, 512, 40, 0.1),
                                            (7, 4097, 256, 0.5), (3, 9000, 720, 0.3)])
def test_huber_backward(rows, d, k, delta):
    x = synthetic.score_rows(rows, d, base=3 * d + rows)
    g = synthetic.score_rows(rows, d, base=5 * d + rows)
    gx = spark.stat_topk_huber_backward(x.cuda(), g.cuda(), k, delta).cpu().numpy().astype(np.float64)
    x64, g64 = x.numpy().astype(np.float64), g.numpy().astype(np.float64)
    ref = oracle.stat_topk_huber_backward(x64, g64, k, delta)
    mu, sd, Q, eps_t = _stats(x64, k)
    _, th = oracle.stat_topk_huber(x64, k, delta)
    z = x64 - th[:, None]
    slope = np.where(z <= 0, 0.0, np.where(z < delta, z / delta, 1.0))
    w = g64 * slope
    W = w.sum(axis=1)
    c = 1.0 / d + abs(Q) * np.abs(x64 - mu[:, None]) / (d * sd[:, None])
    ew = np.abs(g64) * (eps_t[:, None] / delta + 4 * U)
    tol = ew + c * (ew.sum(axis=1) + 32 * U * np.abs(w).sum(axis=1))[:, None] + \
        np.abs(W)[:, None] * c * (16 * U + (eps_t / sd)[:, None]) + 8 * U * np.abs(ref)
    assert np.all(np.abs(gx - ref) <= tol), np.max(np.abs(gx - ref) / tol)


def test_huber_backward_in_place_and_zero_spread():
    x = synthetic.score_rows(12, 256, base=77)
    g = synthetic.score_rows(12, 256, base=78)
    ref = spark.stat_topk_huber_backward(x.cuda(), g.cuda(), 20, 0.5)
    xg, gg = x.cuda(), g.cuda()
    spark.stat_topk_huber_backward(xg, gg, 20, 0.5, grad_x=gg)  # in place over grad_out
    torch.cuda.synchronize()
    assert torch.equal(gg, ref)
    flat = torch.full((2, 64), 1.5, device="cuda")
    gz = spark.stat_topk_huber_backward(flat, torch.ones_like(flat), 5, 0.2)
    torch.cuda.synchronize()
    assert torch.all(gz == 0)


def test_huber_backward_sums_to_zero_per_row():
    """Translation invariance of the operator: each row's gradient sums to ~0 (fp32)."""
    x = synthetic.score_rows(32, 4096, base=91)
    g = synthetic.score_rows(32, 4096, base=92)
    gx = spark.stat_topk_huber_backward(x.cuda(), g.cuda(), 256, 0.25).cpu().numpy().astype(np.float64)
    scale = np.abs(gx).sum(axis=1)
    assert np.all(np.abs(gx.sum(axis=1)) <= 1e-4 * scale)
