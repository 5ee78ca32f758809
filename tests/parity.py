"""Comparison rules between the CUDA path and the fp64 oracle (test helper).

Readings (Spark Transformer notes, 关键设计; tolerance as the method's target
states it):
* active sets: bit-exact, except neurons with |x - theta| <= 1e-4 * std (oracle
  values), which are counted and reported.  The GPU compares x and theta in
  fp32, so the band also covers the fp32 spacing at theta (this only matters
  for rows whose |mean| exceeds ~1e3 std, where fp32 cannot resolve theta to
  1e-4 std);
* outputs, evaluated by the oracle on the GPU's own active set: relative L2
  error <= 2e-3, and max-abs error <= 1e-2 * rms(out) beyond the rounding of
  the bf16 output itself (at most 2^-8 |out| per element).
"""
import math

import numpy as np

BAND = 1e-4
REL_L2_MAX = 2e-3
MAX_ABS_REL_RMS = 1e-2
BF16_HALF_ULP_REL = 2.0 ** -8


def bf16_to_f64(t):
    """bf16 torch tensor (any device) -> float64 numpy."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare_active(gpu_active, ox, otheta, ostd, band=BAND):
    gpu_active = np.asarray(gpu_active).astype(bool)
    oracle_active = ox > otheta[:, None]
    mismatch = gpu_active != oracle_active
    spacing = np.spacing(np.abs(otheta).astype(np.float32)).astype(np.float64)
    in_band = np.abs(ox - otheta[:, None]) <= np.maximum(band * ostd, spacing)[:, None]
    return {"outside_band": int((mismatch & ~in_band).sum()), "band_flips": int((mismatch & in_band).sum()),
            "band_size": int(in_band.sum()), "gpu_count": gpu_active.sum(axis=1),
            "oracle_count": oracle_active.sum(axis=1)}


def output_errors(gpu_out, ref):
    diff = gpu_out - ref
    norm = float(np.linalg.norm(ref))
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    rel_l2 = float(np.linalg.norm(diff)) / norm if norm > 0 else float(np.linalg.norm(diff))
    excess = np.abs(diff) - BF16_HALF_ULP_REL * np.abs(ref)
    max_excess = float(excess.max()) if ref.size else 0.0
    return {"rel_l2": rel_l2, "rms": rms, "max_abs": float(np.abs(diff).max()) if ref.size else 0.0,
            "max_excess_over_rms": max_excess / rms if rms > 0 else max_excess}


def assert_outputs_close(gpu_out, ref):
    e = output_errors(gpu_out, ref)
    if e["rms"] == 0.0:
        assert np.all(gpu_out == 0.0), e
        return e
    assert e["rel_l2"] <= REL_L2_MAX, e
    assert e["max_excess_over_rms"] <= MAX_ABS_REL_RMS, e
    return e


def x_tolerance(K1f, q1f, r):
    """Rigorous bound on the kernel's fp32 predictor error: each lane accumulates at most
    8*ceil(r/256) products with FMA, then a 5-level tree; (n + slack) u sum|K1_ij q_j|."""
    n = 8 * math.ceil(r / 256) + 8
    return n * 2.0 ** -24 * (np.abs(q1f) @ np.abs(K1f).T)
