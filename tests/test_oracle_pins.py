"""Pins for the fp64 oracle, against things other than the oracle itself.

Each test names what fixes the expected value: a textbook table, a closed
form, a library routine on a special case the method reduces to, an
invariant, or brute force.  The method is from the paper-notes page "Spark
Transformer: Reactivating Sparsity in FFN and Attention", 方法详解/关键设计
("Spark FFN", "Statistical Top-k").  CPU only.
"""
import math
import os

import numpy as np
import pytest
import scipy.special as sp

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _to_bf16_bits(a):
    """Round fp32 values to bf16 (round to nearest even) and return the bit patterns."""
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (f + 0x7FFF + ((f >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def _widen(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- bf16 widening
def test_bf16_widening_known_patterns():
    # IEEE binary32 truncated to its top 16 bits: known values.
    cases = {0x3F80: 1.0, 0xC000: -2.0, 0x3F81: 1.0078125, 0x0000: 0.0,
             0x0001: 2.0 ** -133, 0x7F7F: 3.3895313892515355e38, 0x3E80: 0.25}
    bits = np.array(list(cases), dtype=np.uint16)
    got = oracle.bf16_bits_to_f64(bits)
    assert got.tolist() == list(cases.values())
    assert math.isinf(oracle.bf16_bits_to_f64(np.array([0x7F80], dtype=np.uint16))[0])


# ---------------------------------------------------------------- quantile Q
def test_quantile_matches_textbook_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "normal_quantiles.txt"))
            if l.strip() and not l.startswith("#")]
    for p_s, z_s in rows:
        p, z = float(p_s), float(z_s)
        # Q(1 - k/d) evaluated with d = 1 and k = 1 - p (the upper-tail mass)
        got = oracle.topk_quantile(1.0 - p, 1.0)
        assert abs(got - z) <= 1e-12 * max(1.0, abs(z)), (p, got, z)


def test_quantile_matches_library_and_symmetry():
    for d in (8, 16, 64, 1024, 4096, 9216):
        for k in sorted({1, 2, d // 16, d // 12, d // 4, d // 2, d - 1} - {0, d}):
            q = oracle.topk_quantile(k, d)
            ref = float(sp.ndtri(1.0 - k / d))
            assert abs(q - ref) <= 1e-11 * max(1.0, abs(ref)), (d, k, q, ref)
            assert abs(q + oracle.topk_quantile(d - k, d)) <= 1e-12 * max(1.0, abs(q))
    assert oracle.topk_quantile(2048, 4096) == pytest.approx(0.0, abs=1e-15)
    assert math.isnan(oracle.topk_quantile(0, 10)) and math.isnan(oracle.topk_quantile(10, 10))


# ---------------------------------------------------------------- theta
def test_theta_hand_worked_population_std():
    # x = [1,2,3,4], k = 1: mean 2.5, population std sqrt(1.25), Q(0.75) from the table.
    x = np.array([1.0, 2.0, 3.0, 4.0])
    expect = 2.5 + math.sqrt(1.25) * 0.6744897501960817
    assert oracle.theta(x, 1) == pytest.approx(expect, rel=1e-13)
    # the sample-std reading would give 2.5 + sqrt(5/3) * Q: must not match
    assert abs(oracle.theta(x, 1) - (2.5 + math.sqrt(5 / 3) * 0.6744897501960817)) > 1e-3
    m, s = oracle.row_stats(x)
    assert m == 2.5 and s == pytest.approx(math.sqrt(1.25), rel=1e-15)


@pytest.mark.parametrize("d,k", [(64, 5), (1024, 82), (4096, 256), (9216, 737)])
def test_theta_closed_form_on_standardised_rows(d, k):
    rng = _rng(d)
    for mu, sigma in [(0.0, 1.0), (3.5, 0.25), (-2.0, 7.0), (1e3, 1e-2)]:
        z = rng.standard_normal(d)
        z = (z - z.mean()) / z.std()  # exact population mean 0, std 1 (up to rounding)
        x = mu + sigma * z
        expect = mu + sigma * float(sp.ndtri(1.0 - k / d))
        got = oracle.theta(x, k)
        assert abs(got - expect) <= 1e-11 * max(abs(mu), sigma), (mu, sigma, got, expect)


def test_theta_random_gaussian_rows_within_sampling_bound():
    rng = _rng(7)
    d, k = 9216, 737
    Q = float(sp.ndtri(1 - k / d))
    bound = 4.0 * math.sqrt((1 + Q * Q / 2) / d)  # asymptotic sd of mean + std*Q estimates
    for _ in range(50):
        mu, sigma = rng.uniform(-5, 5), rng.uniform(0.1, 10)
        x = rng.normal(mu, sigma, d)
        assert abs(oracle.theta(x, k) - (mu + sigma * Q)) <= bound * sigma


# ---------------------------------------------------------------- selection
@pytest.mark.parametrize("d", [8, 16, 64])
def test_selection_equals_sorted_top_m(d):
    """A threshold keeps a sorted prefix: the active set is the top-m by a full sort."""
    rng = _rng(100 + d)
    k = max(1, d // 8)
    n_rows = 2000
    x = rng.standard_normal((n_rows, d)).astype(np.float32)
    out, th, _, _ = oracle.stat_topk(x, k)
    for i in range(n_rows):
        active = out[i] > 0
        m = int(active.sum())
        order = np.argsort(-x[i].astype(np.float64), kind="stable")
        assert set(np.nonzero(active)[0]) == set(order[:m].tolist())
        # soft threshold values: max(x - theta, 0): exactly zero off the active set
        assert np.all(out[i][~active] == 0.0)
        np.testing.assert_allclose(out[i][active], x[i][active].astype(np.float64) - th[i], rtol=0,
                                   atol=1e-12)


@pytest.mark.parametrize("d,k", [(1024, 82), (4096, 256), (9216, 737)])
def test_selected_count_theorem_3_1(d, k):
    """Theorem 3.1: for Gaussian scores the count deviates from k by O(sqrt(log d / d)) d.

    The constant is unstated; C = 1 gives |m - k| <= sqrt(d ln d).  The mean count over
    many rows must also sit near k (binomial spread)."""
    rng = _rng(d + k)
    rows = 200
    x = rng.standard_normal((rows, d)).astype(np.float32) * 3.0 + 1.0
    out, _, _, _ = oracle.stat_topk(x, k, n_threads=4)
    m = (out > 0).sum(axis=1)
    assert np.all(np.abs(m - k) <= math.sqrt(d * math.log(d)))
    sd = math.sqrt(k * (1 - k / d))
    assert abs(m.mean() - k) <= 4 * 2 * sd / math.sqrt(rows)


def test_stat_topk_constant_row_is_empty():
    x = np.full((3, 100), 2.5, dtype=np.float32)
    out, th, mu, sd = oracle.stat_topk(x, 10)
    assert np.all(out == 0) and np.all(sd == 0) and np.all(th == 2.5)


def test_stat_topk_rejects_bad_k():
    with pytest.raises(ValueError):
        oracle.stat_topk(np.zeros((1, 8), np.float32), 0)
    with pytest.raises(ValueError):
        oracle.stat_topk(np.zeros((1, 8), np.float32), 8)


# ---------------------------------------------------------------- GELU
def test_gelu_forms():
    assert oracle.gelu(0.0) == 0.0 and oracle.gelu(0.0, oracle.GELU_ERF) == 0.0
    s = np.linspace(-6, 6, 1201)
    for v in s:
        erf_form = oracle.gelu(v, oracle.GELU_ERF)
        assert erf_form == pytest.approx(v * float(sp.ndtr(v)), rel=1e-14, abs=1e-300)
        # the tanh form approximates x*Phi(x); max deviation ~4.7e-4 near |x| = 2.7
        assert abs(oracle.gelu(v) - v * float(sp.ndtr(v))) <= 5e-4
        # GELU(s) - GELU(-s) = s for both forms (Phi(s) + Phi(-s) = 1; tanh is odd)
        assert oracle.gelu(v) - oracle.gelu(-v) == pytest.approx(v, abs=1e-14)
    assert oracle.gelu(1.0) == pytest.approx(float(sp.ndtr(1.0)), abs=2e-4)
    assert oracle.gelu(30.0) == pytest.approx(30.0, rel=1e-15)


def _gelu_tanh_decimal(s: str, digits: int = 50):
    """GELU, tanh form, evaluated as s / (1 + exp(-2u)), u = sqrt(2/pi) (s + 0.044715 s^3), in
    `digits`-digit decimal arithmetic with pi from Machin's formula 16 atan(1/5) - 4 atan(1/239).
    A different route from the oracle's (no tanh, no libm constant), exact to far below fp64."""
    from decimal import Decimal, localcontext

    def atan_inv(n):
        x = Decimal(1) / n
        term, total, k = x, x, 1
        while True:
            term *= -x * x
            k += 2
            if abs(term / k) < Decimal(10) ** -(digits - 2):
                return total
            total += term / k

    with localcontext() as ctx:
        ctx.prec = digits
        pi = 16 * atan_inv(5) - 4 * atan_inv(239)
        v = Decimal(s)
        u = (Decimal(2) / pi).sqrt() * (v + Decimal("0.044715") * v ** 3)
        return float(v / (1 + (-2 * u).exp()))


def test_gelu_tanh_closed_form_values():
    # closed-form values: GELU_tanh(1) = 0.8411919906, GELU_tanh(2) = 1.9545976941 (to 10 digits)
    assert oracle.gelu(1.0) == pytest.approx(0.8411919906, abs=1e-10)
    assert oracle.gelu(2.0) == pytest.approx(1.9545976941, abs=1e-10)
    # the same points and more, to full double precision, from the 50-digit evaluation
    assert oracle.gelu(1.0) == pytest.approx(0.8411919906082768, rel=1e-14)
    assert oracle.gelu(2.0) == pytest.approx(1.954597694087775, rel=1e-14)
    for s in ("0.5", "1", "2", "3", "-1.5", "0.125", "4.75"):
        assert oracle.gelu(float(s)) == pytest.approx(_gelu_tanh_decimal(s), rel=1e-13, abs=1e-300), s


# ---------------------------------------------------------------- FFN
def _layer(rng, d_model, r, d_ff, T):
    K1 = _to_bf16_bits(rng.standard_normal((d_ff, r)) / math.sqrt(r))
    K2 = _to_bf16_bits(rng.standard_normal((d_ff, d_model - r)) / math.sqrt(d_model - r))
    V = _to_bf16_bits(rng.standard_normal((d_ff, d_model)) / math.sqrt(d_ff))
    q = _to_bf16_bits(rng.standard_normal((T, d_model)))
    return q, K1, K2, V


def _dense_formula(q, K1, K2, V, r, k):
    """The gated-FFN form with the Top_k mask applied densely, from library routines:
    numpy matmul for the contractions, numpy mean/std for the statistics, scipy ndtri for Q,
    scipy ndtr for the exact GELU s*Phi(s)."""
    qf, K1f, K2f, Vf = _widen(q), _widen(K1), _widen(K2), _widen(V)
    X = qf[:, :r] @ K1f.T
    d_ff = K1.shape[0]
    theta = X.mean(axis=1) + X.std(axis=1) * sp.ndtri(1.0 - k / d_ff)
    S = np.maximum(X - theta[:, None], 0.0)
    H = S * sp.ndtr(S) * (qf[:, r:] @ K2f.T)
    return H @ Vf, X, theta


@pytest.mark.parametrize("shape", [(256, 128, 1024, 82, 4), (48, 16, 96, 9, 3), (64, 8, 200, 17, 2)])
def test_ffn_equals_dense_gated_form(shape):
    """Spark FFN equals the dense gated-FFN formula under the same mask (inactive neurons
    contribute exactly 0 because GELU(0) = 0)."""
    d_model, r, d_ff, k, T = shape
    q, K1, K2, V = _layer(_rng(sum(shape)), d_model, r, d_ff, T)
    res = oracle.spark_ffn(q, K1, K2, V, r, k, gelu_kind=oracle.GELU_ERF)
    ref, X, theta = _dense_formula(q, K1, K2, V, r, k)
    np.testing.assert_allclose(res["x"], X, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["theta"], theta, rtol=1e-12, atol=1e-13)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(res["out"], ref, rtol=0, atol=1e-12 * scale)
    assert np.array_equal(res["active"], X > theta[:, None])


def test_ffn_reduces_to_gelu_of_soft_threshold():
    """With a_i = 1 (K2 column of ones against q[r] = 1) and V = [I | 0], out_i = GELU(max(x_i -
    theta, 0)): the FFN reduces to statistical top-k followed by GELU."""
    rng = _rng(5)
    d_ff, r = 16, 16
    d_model = r + 1
    K1 = _to_bf16_bits(rng.standard_normal((d_ff, r)))
    K2 = _to_bf16_bits(np.ones((d_ff, 1)))
    V = _to_bf16_bits(np.hstack([np.eye(d_ff), np.zeros((d_ff, 1))]))
    q = _to_bf16_bits(np.hstack([rng.standard_normal((2, r)), np.ones((2, 1))]))
    k = 3
    res = oracle.spark_ffn(q, K1, K2, V, r, k, gelu_kind=oracle.GELU_ERF)
    X = _widen(q)[:, :r] @ _widen(K1).T
    theta = X.mean(axis=1) + X.std(axis=1) * sp.ndtri(1 - k / d_ff)
    S = np.maximum(X - theta[:, None], 0)
    np.testing.assert_allclose(res["out"][:, :d_ff], S * sp.ndtr(S), rtol=1e-13, atol=1e-15)
    assert np.all(res["out"][:, d_ff] == 0)


def test_ffn_invariants():
    d_model, r, d_ff, k, T = 96, 40, 300, 24, 3
    rng = _rng(11)
    q, K1, K2, V = _layer(rng, d_model, r, d_ff, T)
    base = oracle.spark_ffn(q, K1, K2, V, r, k)
    assert base["active"].any()
    # 1. theta is scale-equivariant: doubling q[:r] (exact in bf16) keeps the active set.
    q2 = q.copy()
    q2[:, :r] = _to_bf16_bits(_widen(q[:, :r]) * 2)
    assert np.array_equal(oracle.spark_ffn(q2, K1, K2, V, r, k)["active"], base["active"])
    # 2. out is linear in V and in q[r:] (doubling is exact at every step).
    assert np.array_equal(oracle.spark_ffn(q, K1, K2, _to_bf16_bits(_widen(V) * 2), r, k)["out"],
                          2 * base["out"])
    q3 = q.copy()
    q3[:, r:] = _to_bf16_bits(_widen(q[:, r:]) * 2)
    assert np.array_equal(oracle.spark_ffn(q3, K1, K2, V, r, k)["out"], 2 * base["out"])
    # 3. permuting neurons (rows of K1, K2, V together) permutes the active set, keeps out.
    perm = rng.permutation(d_ff)
    pr = oracle.spark_ffn(q, K1[perm], K2[perm], V[perm], r, k)
    assert np.array_equal(pr["active"], base["active"][:, perm])
    np.testing.assert_allclose(pr["out"], base["out"], rtol=0, atol=1e-13 * np.abs(base["out"]).max())
    # 4. permuting only V's rows changes the output (catches a V index that ignores i)
    assert not np.allclose(oracle.spark_ffn(q, K1, K2, V[perm], r, k)["out"], base["out"])


def test_ffn_degenerate_rows_give_zero():
    d_model, r, d_ff, k = 32, 16, 64, 5
    rng = _rng(3)
    q, K1, K2, V = _layer(rng, d_model, r, d_ff, 2)
    q[:, :r] = 0  # x = 0 for every neuron: sigma = 0, theta = mean, nothing active
    res = oracle.spark_ffn(q, K1, K2, V, r, k)
    assert not res["active"].any() and np.all(res["out"] == 0)
    K1c = np.tile(K1[:1], (d_ff, 1))  # identical predictor rows: constant x
    q, _, _, _ = _layer(rng, d_model, r, d_ff, 2)
    res = oracle.spark_ffn(q, K1c, K2, V, r, k)
    assert not res["active"].any() and np.all(res["out"] == 0)


def test_ffn_override_active_set():
    d_model, r, d_ff, k, T = 64, 32, 128, 10, 2
    q, K1, K2, V = _layer(_rng(21), d_model, r, d_ff, T)
    base = oracle.spark_ffn(q, K1, K2, V, r, k)
    same = oracle.spark_ffn(q, K1, K2, V, r, k, override_active=base["active"])
    assert np.array_equal(same["out"], base["out"])
    none = oracle.spark_ffn(q, K1, K2, V, r, k, override_active=np.zeros((T, d_ff), bool))
    assert np.all(none["out"] == 0)
    assert np.array_equal(none["active"], base["active"])  # the reported mask stays x > theta
    # every neuron "active": inactive ones have max(x - theta, 0) = 0 and GELU(0) = 0
    allon = oracle.spark_ffn(q, K1, K2, V, r, k, override_active=np.ones((T, d_ff), bool))
    np.testing.assert_allclose(allon["out"], base["out"], rtol=0, atol=1e-14)


def test_ffn_rejects_bad_sizes():
    q, K1, K2, V = _layer(_rng(1), 32, 16, 64, 1)
    with pytest.raises(ValueError):
        oracle.spark_ffn(q, K1, K2, V, 16, 0)
    with pytest.raises(ValueError):
        oracle.spark_ffn(q, K1, K2, V, 16, 64)


def test_rmsnorm():
    rng = _rng(9)
    h = rng.standard_normal(2304) * 3 + 0.5
    y = oracle.rmsnorm(h, 1e-6)
    ms = float(np.mean(h * h))
    assert float(np.mean(y * y)) == pytest.approx(ms / (ms + 1e-6), rel=1e-12)
    np.testing.assert_allclose(y / h, np.full_like(h, 1 / math.sqrt(ms + 1e-6)), rtol=1e-13)
