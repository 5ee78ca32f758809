"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of ``oracle/spark_oracle.c``
(a dropped term, a wrong sign, a wrong index, a wrong reading of std), builds
it with gcc, and runs ``tests/test_oracle_pins.py`` against it in a
subprocess.  The pin suite must fail for every planted mistake.  CPU only; the
committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "spark_oracle.c")

MUTATIONS = {
    "sample_std": ("sqrt(ss / (double)d)", "sqrt(ss / (double)(d - 1))"),
    "theta_sign": ("return mean + sd * oracle_topk_quantile", "return mean - sd * oracle_topk_quantile"),
    "variance_drops_mean": ("double c = x[i] - mean;", "double c = x[i];"),
    "gelu_cubic_term": ("0.044715 * s * s * s", "0.044715 * s * s"),
    "gelu_truncated_constant": ("sqrt(2.0 / M_PI)", "0.7979"),
    "gelu_cubic_coefficient": ("0.044715 * s * s * s", "0.04472 * s * s * s"),
    "bisection_direction": ("lo = mid; /* too much", "hi = mid; /* too much"),
    "a_uses_q_head": ("* oracle_bf16_to_f64(qt[r + j])", "* oracle_bf16_to_f64(qt[j])"),
    "K1_transposed": ("K1[i * r + j]", "K1[j * r + i]"),
    "V_wrong_row": ("V[i * d_model + c]", "V[(d_ff - 1 - i) * d_model + c]"),
    "gelu_of_x_not_s": ("double g = gelu_of_kind(s, gelu_kind);", "double g = gelu_of_kind(x[i], gelu_kind);"),
    "drops_a": ("double h = g * a;", "double h = g;"),
    "soft_threshold_not_clamped": ("out[row * d + i] = s > 0.0 ? s : 0.0;", "out[row * d + i] = s;"),
    "mean_wrong_divisor": ("double mean = sum / (double)d;", "double mean = sum / (double)(d - 1);"),
    "gelu_half_dropped": ("return 0.5 * s * (1.0 + tanh(", "return s * (1.0 + tanh("),
    "gelu_one_dropped": ("(1.0 + tanh(c * (s", "(tanh(c * (s"),
    "quantile_tail_complement": ("double tail = k / d;", "double tail = 1.0 - k / d;"),
    "gelu_erf_sign": ("s * 0.5 * erfc(-s / sqrt(2.0))", "s * 0.5 * erfc(s / sqrt(2.0))"),
    "rmsnorm_eps_dropped": ("1.0 / sqrt(ss / (double)d + eps);", "1.0 / sqrt(ss / (double)d);"),
    "rmsnorm_sum_not_mean": ("1.0 / sqrt(ss / (double)d + eps);", "1.0 / sqrt(ss + eps);"),
    "ffn_override_unclamped": ("            if (s < 0.0) s = 0.0;\n            double g = gelu_of_kind", "            double g = gelu_of_kind"),
    "ffn_mask_from_override": ("if (active_out) active_out[t * d_ff + i] = (uint8_t)(x[i] > theta);",
                               "if (active_out) active_out[t * d_ff + i] = (uint8_t)active;"),
}


# Mistakes planted in the Spark Attention oracle; the attention pins must catch each.
ATTN_MUTATIONS = {
    "attn_scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "attn_softplus_sign": ("return a > 0.0 ? a + log1p(exp(-a)) : log1p(exp(a));",
                           "return a > 0.0 ? a - log1p(exp(-a)) : log1p(exp(a));"),
    "attn_a_uses_predictor_dims": ("a += oracle_bf16_to_f64(Kg[j * d_head + r + i]) * oracle_bf16_to_f64(qh[r + i]);",
                                   "a += oracle_bf16_to_f64(Kg[j * d_head + i]) * oracle_bf16_to_f64(qh[i]);"),
    "attn_no_normalisation": ("for (long c = 0; c < d_head; ++c) o[c] /= z;",
                              "for (long c = 0; c < d_head; ++c) o[c] /= 1.0;"),
    "attn_wrong_kv_head": ("const long g = h / group;", "const long g = h % n_kv_heads;"),
    "attn_theta_ignored": ("if (k_attn < n_ctx) theta = oracle_theta(s, n_ctx, k_attn, NULL, NULL);", ""),
    "attn_value_from_key": ("o[c] += f * oracle_bf16_to_f64(Vg[j * d_head + c]);",
                            "o[c] += f * oracle_bf16_to_f64(Kg[j * d_head + c]);"),
    "attn_softmax_over_all_keys": ("            if (!act) continue;\n            double w = exp(s[j] - smax);",
                                   "            double w = exp(s[j] - smax);\n            if (!act) { z += w; continue; }"),
    "attn_softplus_to_identity": ("double f = w * oracle_softplus(a);", "double f = w * a;"),
    "attn_theta_at_k_equal_n": ("if (k_attn < n_ctx) theta", "if (k_attn <= n_ctx) theta"),
    "attn_mask_from_override": ("if (active_out) active_out[h * n_ctx + j] = (uint8_t)(s[j] > theta);",
                                "if (active_out) active_out[h * n_ctx + j] = (uint8_t)act;"),
}


# Mistakes planted in the causal statistical top-k; the causal pins must catch each.
CAUSAL_MUTATIONS = {
    "causal_visible_count_off_by_one": ("const long n = pos + 1 < d ? pos + 1 : d;", "const long n = pos < d ? pos : d;"),
    "causal_heads_not_wrapped": ("const long pos = offset + row % n_q;", "const long pos = offset + row;"),
    "causal_offset_ignored": ("const long pos = offset + row % n_q;", "const long pos = row % n_q;"),
    "causal_masked_not_zeroed": ("for (long j = n; j < d; ++j) out[row * d + j] = 0.0;",
                                 "for (long j = n; j < d; ++j) out[row * d + j] = (double)x[row * d + j];"),
    "causal_select_all_zeroed": ("for (long j = 0; j < n; ++j) out[row * d + j] = xr[j];",
                                 "for (long j = 0; j < n; ++j) out[row * d + j] = 0.0;"),
    "causal_select_all_boundary": ("        if (k < n) {\n            double mean, sd;", "        if (k <= n) {\n            double mean, sd;"),
    "causal_theta_misses_last_visible": ("theta = oracle_theta(xr, n, k, &mean, &sd);",
                                         "theta = oracle_theta(xr, n > 1 ? n - 1 : n, k, &mean, &sd);"),
    "causal_pass_through_clamped": ("for (long j = 0; j < n; ++j) out[row * d + j] = xr[j];",
                                    "for (long j = 0; j < n; ++j) out[row * d + j] = xr[j] > 0.0 ? xr[j] : 0.0;"),
}


# Mistakes planted in the Huber-smoothed forward and its backward; the Huber pins must catch each.
HUBER_MUTATIONS = {
    "huber_backward_drops_theta": ("grad_x[row * d + j] = w[j] - W * dtheta;", "grad_x[row * d + j] = w[j];"),
    "huber_backward_theta_sign": ("grad_x[row * d + j] = w[j] - W * dtheta;", "grad_x[row * d + j] = w[j] + W * dtheta;"),
    "huber_backward_drops_std_term": ("if (sd > 0.0) dtheta += Q * (xr[j] - mean) / ((double)d * sd);",
                                      "if (sd > 0.0) dtheta += 0.0;"),
    "huber_middle_slope": ("if (z < delta) return z / delta;", "if (z < delta) return z / (2.0 * delta);"),
    "huber_forward_offset": ("return z - 0.5 * delta;", "return z - delta;"),
    "huber_forward_square": ("if (z < delta) return z * z / (2.0 * delta);", "if (z < delta) return z * z / delta;"),
    "huber_backward_drops_mean_term": ("double dtheta = 1.0 / (double)d;", "double dtheta = 0.0;"),
}


def _pins_fail_on(old, new, pin_file, tmp_path):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fopenmp",
                           "-fPIC", "-shared", str(mutated), "-o", str(lib), "-lm"])
    env = dict(os.environ, SPARK_ORACLE_LIB=str(lib))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", pin_file)],
                          env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    return proc.returncode != 0, proc.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(ATTN_MUTATIONS))
def test_attention_pins_catch_planted_mistake(name, tmp_path):
    old, new = ATTN_MUTATIONS[name]
    caught, log = _pins_fail_on(old, new, "test_oracle_attention_pins.py", tmp_path)
    assert caught, f"attention pins did not catch mutation {name}:\n{log}"


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fopenmp",
                           "-fPIC", "-shared", str(mutated), "-o", str(lib), "-lm"])
    env = dict(os.environ, SPARK_ORACLE_LIB=str(lib))
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert proc.returncode != 0, f"pins did not catch mutation {name}:\n{proc.stdout[-2000:]}"


@pytest.mark.parametrize("name", sorted(CAUSAL_MUTATIONS))
def test_causal_pins_catch_planted_mistake(name, tmp_path):
    old, new = CAUSAL_MUTATIONS[name]
    caught, log = _pins_fail_on(old, new, "test_oracle_causal_pins.py", tmp_path)
    assert caught, f"causal pins did not catch mutation {name}:\n{log}"


@pytest.mark.parametrize("name", sorted(HUBER_MUTATIONS))
def test_huber_pins_catch_planted_mistake(name, tmp_path):
    old, new = HUBER_MUTATIONS[name]
    caught, log = _pins_fail_on(old, new, "test_oracle_huber_pins.py", tmp_path)
    assert caught, f"Huber pins did not catch mutation {name}:\n{log}"
