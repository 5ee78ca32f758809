"""GPU parity of Spark Attention (one decoding position) against the fp64 oracle, through the C ABI.

The Gemma-2-2B-like case: 8 query heads over 4 key/value heads, head dimension 256 split r = 128,
4096 cached positions, k_attn = 256, scale 1/sqrt(256); plus ragged contexts, the dense case
(k_attn >= n_ctx), degenerate keys, poisoned unselected rows and repeatability.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import _binding, synthetic

from .gpu_util import widen
from .parity import assert_outputs_close, bf16_to_f64, compare_active, x_tolerance

pytestmark = pytest.mark.gpu


def run_attention(n_heads, n_kv, n_ctx, d_head, r, k_attn, scale=None, layer=0, inputs=None):
    host = inputs if inputs is not None else synthetic.attention_inputs(n_heads, n_kv, n_ctx, d_head, layer=layer)
    dev = {k: v.cuda() for k, v in host.items()}
    if scale is None:
        scale = 1.0 / math.sqrt(d_head)
    res = spark.attention_decode(dev["q"], dev["K"], dev["V"], r, k_attn, scale=scale, debug=True)
    torch.cuda.synchronize()
    bits = {k: synthetic.bf16_bits(v) for k, v in host.items()}
    orc = oracle.spark_attention(bits["q"], bits["K"], bits["V"], r, k_attn, scale, n_threads=8)
    gs = res["s"].cpu().numpy().astype(np.float64)
    gth = res["theta"].cpu().numpy().astype(np.float64)
    gact = res["active"].cpu().numpy().astype(bool)
    group = n_heads // n_kv
    qf, Kf = widen(bits["q"]), widen(bits["K"])
    for h in range(n_heads):
        # scaled predictor scores within the kernel's fp32 bound (one more rounding for the scale)
        tol = scale * x_tolerance(Kf[h // group][:, :r], qf[h:h + 1, :r], r)[0] + 2.0 ** -23 * np.abs(orc["s"][h])
        assert np.all(np.abs(gs[h] - orc["s"][h]) <= tol), h
    if k_attn >= n_ctx:
        assert np.all(np.isneginf(gth)) and np.all(gact)
    else:
        std = orc["s"].std(axis=1)
        assert np.all(np.abs(gth - orc["theta"]) <= 1e-5 * std)
        # the GPU decides s > theta in fp32 on its own values: reproduce exactly
        assert np.array_equal(gact, res["s"].cpu().numpy() > res["theta"].cpu().numpy()[:, None])
        cmp = compare_active(gact, orc["s"], orc["theta"], std)
        assert cmp["outside_band"] == 0, cmp
    # output on the GPU's selection
    ref = oracle.spark_attention(bits["q"], bits["K"], bits["V"], r, k_attn, scale, override_active=gact,
                                 n_threads=8)["out"]
    out = bf16_to_f64(res["out"]).reshape(n_heads, d_head)
    assert_outputs_close(out, ref)
    # the plain entry point gives the same bits
    plain = spark.attention_decode(dev["q"], dev["K"], dev["V"], r, k_attn, scale=scale)
    assert torch.equal(plain, res["out"])
    return res, orc


def test_gemma_like_heads():
    res, orc = run_attention(8, 4, 4096, 256, 128, 256, layer=1)
    counts = res["active"].sum(dim=1).cpu().numpy()
    assert np.all(np.abs(counts - 256) <= math.sqrt(4096 * math.log(4096))), counts


@pytest.mark.parametrize("shape", [
    (8, 4, 1000, 256, 128, 64),   # ragged context: the last CTA of each cluster is partial
    (4, 4, 4097, 128, 64, 256),   # one past a multiple of the cluster size
    (2, 1, 300, 64, 8, 20),       # r = 8, small head
    (4, 2, 129, 256, 248, 16),    # r close to d_head
    (3, 1, 16384, 64, 32, 512),   # long context
])
def test_ragged_and_edge_shapes(shape):
    n_heads, n_kv, n_ctx, d_head, r, k = shape
    run_attention(n_heads, n_kv, n_ctx, d_head, r, k, layer=sum(shape) % 89)


@pytest.mark.parametrize("n_ctx", [1, 7, 256])
def test_dense_when_k_attn_covers_the_context(n_ctx):
    run_attention(4, 2, n_ctx, 128, 64, 256, layer=3)


def test_degenerate_keys_select_nothing():
    host = synthetic.attention_inputs(2, 1, 512, 64, layer=4)
    host["K"][0, :, :32] = host["K"][0, 0, :32]  # identical predictor parts: zero spread
    res = spark.attention_decode(host["q"].cuda(), host["K"].cuda(), host["V"].cuda(), 32, 20, debug=True)
    torch.cuda.synchronize()
    assert int(res["active"].sum()) == 0 and torch.all(res["out"] == 0)


def test_poisoned_unselected_rows_are_never_read():
    """NaN in the K2 part and the value row of every unselected key leaves out bit-identical."""
    host = synthetic.attention_inputs(8, 4, 4096, 256, layer=5)
    dev = {k: v.cuda() for k, v in host.items()}
    res = spark.attention_decode(dev["q"], dev["K"], dev["V"], 128, 256, debug=True)
    used = res["active"].bool().reshape(4, 2, 4096).any(dim=1)  # per key/value head
    K2, V2 = dev["K"].clone(), dev["V"].clone()
    K2[:, :, 128:][~used] = float("nan")
    V2[~used] = float("nan")
    out2 = spark.attention_decode(dev["q"], K2, V2, 128, 256)
    assert torch.isfinite(out2.float()).all()
    assert torch.equal(out2, res["out"])


def test_repeatable_and_errors_refused():
    host = synthetic.attention_inputs(8, 4, 2048, 256, layer=6)
    dev = {k: v.cuda() for k, v in host.items()}
    a = spark.attention_decode(dev["q"], dev["K"], dev["V"], 128, 128)
    b = spark.attention_decode(dev["q"], dev["K"], dev["V"], 128, 128)
    assert torch.equal(a, b)
    L = _binding.lib()
    st = _binding.stream_handle()
    q, K, V = dev["q"], dev["K"], dev["V"]
    out = torch.empty_like(q)
    # 8 heads do not divide over 3 key/value heads; r must lie inside the head; scale must be positive
    assert L.spark_attention_decode(q.data_ptr(), K.data_ptr(), V.data_ptr(), 8, 3, 2048, 256, 128, 128, 0.0625,
                                    out.data_ptr(), st) == -1
    assert L.spark_attention_decode(q.data_ptr(), K.data_ptr(), V.data_ptr(), 8, 4, 2048, 256, 256, 128, 0.0625,
                                    out.data_ptr(), st) == -1
    assert L.spark_attention_decode(q.data_ptr(), K.data_ptr(), V.data_ptr(), 8, 4, 2048, 256, 128, 128, -1.0,
                                    out.data_ptr(), st) == -1
    assert L.spark_attention_decode(q.data_ptr(), K.data_ptr(), V.data_ptr(), 8, 4, 2048, 256, 12, 128, 0.0625,
                                    out.data_ptr(), st) == -2


def test_portable_cluster_size():
    """Caches shorter than 512 positions run on 8-CTA clusters (the portable size, also the
    fallback where 16-CTA clusters are unavailable); parity holds there and at the switch."""
    run_attention(8, 4, 511, 256, 128, 64, layer=8)
    run_attention(2, 1, 500, 128, 64, 100, layer=9)
    run_attention(8, 4, 512, 256, 128, 64, layer=10)
