"""GPU parity of the Spark FFN forward against the fp64 oracle, through the C ABI.

Shapes: the tiny layer (d_model 256, r 128, d_ff 1024, k 82, T 4), the
Gemma-2-2B-shaped layer (2304 / 1152 / 9216, k 737) at decode T = 1 and a
prefill sweep, ragged shapes and the edge cases of the method.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import _binding

from .gpu_util import make_layer, widen
from .parity import assert_outputs_close, bf16_to_f64, compare_active, x_tolerance

pytestmark = pytest.mark.gpu

TINY = (256, 128, 1024, 82)
GEMMA = (2304, 1152, 9216, 737)


def run_parity(d_model, r, d_ff, k, T, layer=0, sample_tokens=None, threads=8):
    dev, bits = make_layer(d_model, r, d_ff, T, layer=layer)
    res = spark.ffn_forward_debug(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    torch.cuda.synchronize()
    assert spark.query_status() == 0
    toks = np.arange(T) if sample_tokens is None else np.asarray(sample_tokens)
    q_bits = bits["q"][toks]
    orc = oracle.spark_ffn(q_bits, bits["K1"], bits["K2"], bits["V"], r, k, n_threads=threads)
    gx = res["x"].cpu().numpy().astype(np.float64)[toks]
    gth = res["theta"].cpu().numpy().astype(np.float64)[toks]
    gact = res["active"].cpu().numpy().astype(bool)[toks]
    # predictor scores within the kernel's rigorous fp32 bound
    tol = x_tolerance(widen(bits["K1"]), widen(q_bits[:, :r]), r)
    assert np.all(np.abs(gx - orc["x"]) <= tol)
    # thresholds well inside the 1e-4*std band
    assert np.all(np.abs(gth - orc["theta"]) <= 1e-5 * orc["std"])
    # the GPU decides x > theta in fp32 on its own x and theta: reproduce exactly
    assert np.array_equal(gact, res["x"].cpu().numpy()[toks] > res["theta"].cpu().numpy()[toks][:, None])
    cmp = compare_active(gact, orc["x"], orc["theta"], orc["std"])
    assert cmp["outside_band"] == 0, cmp
    # output on the GPU's active set
    ref = oracle.spark_ffn(q_bits, bits["K1"], bits["K2"], bits["V"], r, k, override_active=gact,
                           n_threads=threads)["out"]
    out = bf16_to_f64(res["out"]).reshape(T, d_model)[toks]
    err = assert_outputs_close(out, ref)
    # the plain entry point gives the same bits as the debug one
    plain = spark.ffn_forward(dev["q"] if T > 1 else dev["q"][0], dev["K1"], dev["K2"], dev["V"], k)
    assert torch.equal(plain.reshape(T, d_model), res["out"].reshape(T, d_model))
    return err, cmp


def test_tiny_layer_T4():
    run_parity(*TINY, T=4)


@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_gemma_decode_T1(layer):
    err, cmp = run_parity(*GEMMA, T=1, layer=layer)
    # selected count within Theorem 3.1's deviation (C = 1): |m - k| <= sqrt(d ln d)
    assert abs(int(cmp["gpu_count"][0]) - 737) <= math.sqrt(9216 * math.log(9216))


@pytest.mark.parametrize("T", [2, 3, 8, 9, 16])
def test_gemma_small_batches(T):
    run_parity(*GEMMA, T=T, layer=10 + T)


@pytest.mark.parametrize("T", [5, 64, 100, 128, 129, 256])
def test_gemma_prefill(T):
    """One 128-token band up to 128 tokens, two from 129 on; 64-row token boxes up to 64 tokens."""
    run_parity(*GEMMA, T=T, layer=20 + T)


@pytest.mark.parametrize("T", [1024, 4096])
def test_gemma_prefill_large_sampled(T):
    rng = np.random.default_rng(T)
    sample = np.sort(rng.choice(T, size=24, replace=False))
    sample[0], sample[-1] = 0, T - 1
    run_parity(*GEMMA, T=T, layer=30 + T, sample_tokens=sample)


def test_prefill_wide_predictor_ragged_last_unit():
    """Enough tokens for the predictor GEMM's 128 x 256 units, with d_ff = 2496 so that the last
    unit's second 128-column half is only half inside the layer."""
    T = 1920
    rng = np.random.default_rng(7)
    sample = np.sort(rng.choice(T, size=16, replace=False))
    sample[0], sample[-1] = 0, T - 1
    run_parity(512, 256, 2496, 200, T=T, layer=77, sample_tokens=sample)


def test_prefill_wide_output_gemm_ragged_model_width():
    """Enough token tiles for the 128 x 256 output units; d_model = 1088 leaves the last unit one
    64-column box of V inside the matrix and one wholly outside it."""
    T = 1536
    sample = np.arange(0, T, 61)
    run_parity(1088, 512, 2048, 160, T=T, layer=78, sample_tokens=sample)


@pytest.mark.parametrize("shape", [
    (264, 136, 1001, 80, 3),    # ragged d_ff: last CTA owns one neuron
    (64, 32, 200, 17, 2),       # tiny, few CTAs
    (512, 256, 2048, 1, 1),     # k = 1: extreme quantile
    (512, 256, 2048, 2047, 2),  # k = d_ff - 1
    (4096, 2048, 7104, 568, 1), # largest r and d_model - r of the fused kernel
    (1024, 8, 4096, 328, 5),    # r = 8
])
def test_ragged_and_edge_shapes(shape):
    d_model, r, d_ff, k, T = shape
    run_parity(d_model, r, d_ff, k, T, layer=sum(shape) % 97)


def test_degenerate_rows_select_nothing():
    d_model, r, d_ff, k = TINY
    dev, _ = make_layer(d_model, r, d_ff, 3)
    q = dev["q"].clone()
    q[0, :r] = 0  # x = 0 everywhere
    K1 = dev["K1"].clone()
    res = spark.ffn_forward_debug(q, K1, dev["K2"], dev["V"], k)
    assert int(res["active"][0].sum()) == 0 and torch.all(res["out"][0] == 0)
    K1c = K1[:1].repeat(d_ff, 1).contiguous()  # identical predictor rows: constant x
    res = spark.ffn_forward_debug(dev["q"], K1c, dev["K2"], dev["V"], k)
    assert int(res["active"].sum()) == 0 and torch.all(res["out"] == 0)
    # prefill with an empty union (every token's x constant): h is zero everywhere
    d_model, r, d_ff, k = GEMMA
    dev, _ = make_layer(d_model, r, d_ff, 12, layer=4)
    K1c = dev["K1"][:1].repeat(d_ff, 1).contiguous()
    res = spark.ffn_forward_debug(dev["q"], K1c, dev["K2"], dev["V"], k)
    torch.cuda.synchronize()
    assert spark.query_status() == 0
    assert int(res["active"].sum()) == 0 and torch.all(res["out"] == 0)


@pytest.mark.parametrize("shape,T", [(GEMMA, 1), (GEMMA, 4), (TINY, 4), (TINY, 3)])
def test_poisoned_inactive_rows_are_never_read(shape, T):
    """NaN in every K2 / V row outside the union of the tokens' active sets leaves out bit-identical:
    decode and small batches (T <= 4) read only the active rows.  (Prefill, T >= 5, reads every row by
    design: see spark.h.)"""
    d_model, r, d_ff, k = shape
    dev, _ = make_layer(d_model, r, d_ff, T, layer=5)
    res = spark.ffn_forward_debug(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    used = res["active"].bool().any(dim=0)
    K2p, Vp = dev["K2"].clone(), dev["V"].clone()
    K2p[~used] = float("nan")
    Vp[~used] = float("nan")
    out2 = spark.ffn_forward(dev["q"], dev["K1"], K2p, Vp, k)
    assert torch.isfinite(out2.float()).all()
    assert torch.equal(out2, res["out"])


def test_deterministic_across_runs():
    d_model, r, d_ff, k = GEMMA
    dev, _ = make_layer(d_model, r, d_ff, 3, layer=7)
    a = spark.ffn_forward(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    b = spark.ffn_forward(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    assert torch.equal(a, b)


def test_side_stream_and_empty_batch():
    d_model, r, d_ff, k = TINY
    dev, _ = make_layer(d_model, r, d_ff, 2)
    ref = spark.ffn_forward(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = spark.ffn_forward(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    s.synchronize()
    assert torch.equal(out, ref)
    assert spark.query_status(s) == 0
    empty = torch.empty((0, d_model), dtype=torch.bfloat16, device="cuda")
    spark.ffn_forward(empty, dev["K1"], dev["K2"], dev["V"], k)


def test_errors_are_reported_not_launched():
    d_model, r, d_ff, k = TINY
    dev, _ = make_layer(d_model, r, d_ff, 1)
    with pytest.raises(_binding.SparkError) as e:
        spark.ffn_forward(dev["q"], dev["K1"], dev["K2"], dev["V"], d_ff)
    assert e.value.status == -1
    with pytest.raises(_binding.SparkError) as e:
        spark.ffn_forward(dev["q"], dev["K1"], dev["K2"], dev["V"], k, out=dev["q"])
    assert e.value.status == -1
    # r beyond what this build's kernels take: refused on the host
    big = make_layer(8192, 4096, 512, 1)[0]
    with pytest.raises(_binding.SparkError) as e:
        spark.ffn_forward(big["q"], big["K1"], big["K2"], big["V"], 40)
    assert e.value.status == -1


def test_bounded_wait_times_out_and_recovers():
    assert spark.selftest_wait_timeout() == -5  # SPARK_ETIMEOUT, then cleared
    assert spark.query_status() == 0
    run_parity(*TINY, T=4)


def test_decode_weight_overlap_in_graph_is_bit_identical():
    """Score kernels launched behind the previous call (programmatic dependent launch), in a
    stream and inside a CUDA graph, give the same bits as plain stream order; each call's q
    is produced by the kernel just before it, so an early read of q would show."""
    d_model, r, d_ff, k = GEMMA
    layers = [make_layer(d_model, r, d_ff, 1, layer=60 + i)[0] for i in range(3)]
    n = 6
    q0 = layers[0]["q"][0].contiguous()

    def chain(outs):
        q = q0
        for i in range(n):
            L = layers[i % 3]
            spark.ffn_forward(q, L["K1"], L["K2"], L["V"], k, out=outs[i])
            q = outs[i]

    ref = [torch.empty(d_model, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    spark.set_weight_overlap(False)
    chain(ref)
    torch.cuda.synchronize()
    try:
        spark.set_weight_overlap(True)
        got = [torch.empty_like(ref[0]) for _ in range(n)]
        chain(got)
        torch.cuda.synchronize()
        assert all(torch.equal(a, b) for a, b in zip(got, ref))
        s = torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        gout = [torch.empty_like(ref[0]) for _ in range(n)]
        with torch.cuda.stream(s):
            chain(gout)  # workspace of this stream exists before capture
            s.synchronize()
            with torch.cuda.graph(g, stream=s):
                chain(gout)
        for _ in range(3):
            for t in gout:
                t.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert all(torch.equal(a, b) for a, b in zip(gout, ref))
        assert spark.query_status(s) == 0
    finally:
        spark.set_weight_overlap(False)
    assert spark.query_status() == 0


@pytest.mark.parametrize("shape,T", [(GEMMA, 1), (TINY, 4), (GEMMA, 100)])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_buffers_give_the_device_entry_points_bits(shape, T, pinned):
    """spark_ffn_forward_host (q in and out back through host memory) on two calls in a row on one
    stream (its device copies of q and out are reused) against the device-pointer entry point."""
    d_model, r, d_ff, k = shape
    for layer in (90 + T, 91 + T):
        dev, _ = make_layer(d_model, r, d_ff, T, layer=layer)
        q = dev["q"] if T > 1 else dev["q"][0]
        ref = spark.ffn_forward(q, dev["K1"], dev["K2"], dev["V"], k)
        qh = q.cpu()
        if pinned:
            qh = qh.pin_memory()
        out = spark.ffn_forward_host(qh, dev["K1"], dev["K2"], dev["V"], k)
        torch.cuda.synchronize()
        assert spark.query_status() == 0
        assert out.shape == qh.shape and torch.equal(out, ref.cpu())


def test_host_buffers_in_a_decode_loop_with_weight_overlap():
    """Single-token calls from mapped pinned buffers back to back with weight overlap on (the first
    kernel of each call reads q from host memory while the next call's K1 streams), against the
    device entry point, one layer per call."""
    d_model, r, d_ff, k = GEMMA
    layers = [make_layer(d_model, r, d_ff, 1, layer=120 + i) for i in range(3)]
    refs = [spark.ffn_forward(dv["q"][0], dv["K1"], dv["K2"], dv["V"], k).cpu() for dv, _ in layers]
    qh = [dv["q"][0].cpu().pin_memory() for dv, _ in layers]
    oh = [torch.empty_like(q).pin_memory() for q in qh]
    spark.set_weight_overlap(True)
    try:
        for rep in range(2):
            for i, (dv, _) in enumerate(layers):
                spark.ffn_forward_host(qh[i], dv["K1"], dv["K2"], dv["V"], k, out_host=oh[i])
            torch.cuda.synchronize()
            assert spark.query_status() == 0
            for i in range(3):
                assert torch.equal(oh[i], refs[i]), (rep, i)
                oh[i].zero_()
    finally:
        spark.set_weight_overlap(False)


def test_host_buffers_unaligned_pinned_q_takes_the_copy_path():
    """A pinned q_host that is not 16-byte aligned cannot be read by the first kernel in 16-byte chunks:
    the call copies it with the copy engine instead, with the same bits."""
    d_model, r, d_ff, k = GEMMA
    dev, _ = make_layer(d_model, r, d_ff, 1, layer=130)
    ref = spark.ffn_forward(dev["q"][0], dev["K1"], dev["K2"], dev["V"], k).cpu()
    buf = torch.empty(d_model + 1, dtype=torch.bfloat16).pin_memory()
    qh = buf[1:]
    qh.copy_(dev["q"][0].cpu())
    assert qh.data_ptr() % 16 != 0
    out = spark.ffn_forward_host(qh, dev["K1"], dev["K2"], dev["V"], k)
    torch.cuda.synchronize()
    assert spark.query_status() == 0
    assert torch.equal(out, ref)
