"""Pins for the oracle's Huber-smoothed statistical top-k and its backward.

"Statistical Top-k", Theorem 3.2: smoothed with a Huber function the
operator is continuously differentiable.  Reading: rho_delta(z) replaces
max{z, 0} (0 for z <= 0, z^2 / (2 delta) below delta, z - delta/2 above),
z = x - theta(x).  The backward is pinned to central finite differences of
the (separately pinned) forward, to delta -> 0 reducing to the plain
operator, and to invariants (translation: gradients sum to zero; linearity in
the upstream gradient).  CPU only.
"""
import numpy as np
import pytest

import oracle


def _rows(seed, rows, d, scale=1.0):
    return np.random.default_rng(seed).standard_normal((rows, d)) * scale


def test_delta_zero_is_the_soft_threshold():
    x = _rows(1, 6, 300).astype(np.float32)
    out, th = oracle.stat_topk_huber(x.astype(np.float64), 24, 0.0)
    ref, rth, _, _ = oracle.stat_topk(x, 24)
    assert np.array_equal(out, ref) and np.array_equal(th, rth)


def test_forward_pieces_and_continuity():
    x = _rows(2, 4, 500)
    delta = 0.25
    out, th = oracle.stat_topk_huber(x, 40, delta)
    z = x - th[:, None]
    assert np.all(out[z <= 0] == 0.0)
    big = z >= delta
    assert np.allclose(out[big], z[big] - delta / 2, rtol=0, atol=1e-14)  # parallel to the plain ramp
    mid = (z > 0) & (z < delta)
    assert np.all((out[mid] > 0) & (out[mid] < delta / 2))
    # C^1 at the joints: values and slopes meet from both sides
    for z0 in (0.0, delta):
        e = 1e-7
        xs = np.array([[-1.0] * 40 + [0.0]])  # a row whose theta we read back
        _, t = oracle.stat_topk_huber(xs, 4, delta)
        lo, _ = oracle.stat_topk_huber(xs + np.r_[[0.0] * 40, [t[0] + z0 - e]][None, :], 4, delta)
        hi, _ = oracle.stat_topk_huber(xs + np.r_[[0.0] * 40, [t[0] + z0 + e]][None, :], 4, delta)
        assert abs(hi[0, -1] - lo[0, -1]) < 1e-3


def test_shrinking_delta_converges_to_the_soft_threshold():
    x = _rows(3, 3, 200)
    ref, _ = oracle.stat_topk_huber(x, 16, 0.0)
    for delta in (1e-2, 1e-4, 1e-6):
        out, _ = oracle.stat_topk_huber(x, 16, delta)
        assert np.max(np.abs(out - ref)) <= delta / 2 + 1e-15


@pytest.mark.parametrize("d,k,delta", [(8, 2, 0.5), (16, 3, 0.3), (64, 8, 0.2), (200, 16, 1.0)])
def test_backward_matches_finite_differences(d, k, delta):
    rng = np.random.default_rng(d + k)
    x = rng.standard_normal((3, d))
    g = rng.standard_normal((3, d))
    dx = oracle.stat_topk_huber_backward(x, g, k, delta)
    h = 1e-6
    for r in range(3):
        fd = np.empty(d)
        for j in range(d):
            xp, xm = x[r:r + 1].copy(), x[r:r + 1].copy()
            xp[0, j] += h
            xm[0, j] -= h
            fp, _ = oracle.stat_topk_huber(xp, k, delta)
            fm, _ = oracle.stat_topk_huber(xm, k, delta)
            fd[j] = (g[r] @ fp[0] - g[r] @ fm[0]) / (2 * h)
        assert np.allclose(dx[r], fd, rtol=1e-5, atol=1e-6 * np.abs(g[r]).sum()), (r, np.abs(dx[r] - fd).max())


def test_backward_invariants():
    rng = np.random.default_rng(9)
    d, k, delta = 128, 10, 0.4
    x = rng.standard_normal((5, d))
    g1, g2 = rng.standard_normal((5, d)), rng.standard_normal((5, d))
    a = oracle.stat_topk_huber_backward(x, g1, k, delta)
    b = oracle.stat_topk_huber_backward(x, g2, k, delta)
    c = oracle.stat_topk_huber_backward(x, 2.0 * g1 - 3.0 * g2, k, delta)
    assert np.allclose(c, 2.0 * a - 3.0 * b, rtol=1e-12, atol=1e-12)
    # shifting a row by a constant moves theta with it: the output, so the loss, is unchanged
    assert np.allclose(a.sum(axis=1), 0.0, atol=1e-12)
    assert np.array_equal(oracle.stat_topk_huber_backward(x, np.zeros_like(x), k, delta), np.zeros_like(x))


def test_backward_delta_zero_is_the_almost_everywhere_gradient():
    """delta = 0: the soft threshold's gradient (away from the kink), from finite differences."""
    rng = np.random.default_rng(10)
    d, k = 32, 4
    x = rng.standard_normal((1, d))
    g = rng.standard_normal((1, d))
    dx = oracle.stat_topk_huber_backward(x, g, k, 0.0)
    h = 1e-7
    for j in range(d):
        xp, xm = x.copy(), x.copy()
        xp[0, j] += h
        xm[0, j] -= h
        fp, _ = oracle.stat_topk_huber(xp, k, 0.0)
        fm, _ = oracle.stat_topk_huber(xm, k, 0.0)
        assert dx[0, j] == pytest.approx((g[0] @ fp[0] - g[0] @ fm[0]) / (2 * h), rel=1e-5, abs=1e-6)


def test_constant_row_has_zero_gradient():
    x = np.full((1, 20), 3.0)
    g = np.random.default_rng(4).standard_normal((1, 20))
    assert np.array_equal(oracle.stat_topk_huber_backward(x, g, 3, 0.5), np.zeros((1, 20)))


def test_invalid_arguments():
    x = np.zeros((1, 8))
    with pytest.raises(ValueError):
        oracle.stat_topk_huber(x, 0, 0.1)
    with pytest.raises(ValueError):
        oracle.stat_topk_huber(x, 4, -0.1)
    with pytest.raises(ValueError):
        oracle.stat_topk_huber_backward(x, x, 8, 0.1)
