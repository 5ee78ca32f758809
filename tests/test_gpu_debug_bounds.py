"""The bounds-checked build (libspark_debug.so, compiled with SPARK_DEBUG) on the
paths that gather by computed indices: single-token decode, the fused 2-4 token
kernel, the three prefill GEMMs (one and two 128-token bands, split-K and not),
the predictor alone, the decode stack, the no-allocation entry point and the
attention decode.  Each runs through both libraries on the same inputs: the
checked build must count no violation and give the release build's bits."""
import pytest
import torch

import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import _binding, synthetic

from .gpu_util import make_layer

pytestmark = pytest.mark.gpu

TINY = (256, 128, 1024, 82)
GEMMA = (2304, 1152, 9216, 737)


def both(fn):
    """fn() under the release library, then under the checked one; the checked
    run's violation count (read and cleared)."""
    rel = fn()
    torch.cuda.synchronize()
    D = _binding.debug_lib()
    with _binding.using_library(D):
        assert spark.debug_violations() >= 0  # clear whatever an earlier test left
        dbg = fn()
        torch.cuda.synchronize()
        assert spark.query_status() == 0
        n = spark.debug_violations()
    return rel, dbg, n


def test_release_build_has_no_checks():
    assert spark.debug_violations() == -1


@pytest.mark.parametrize("shape,T", [(GEMMA, 1), (TINY, 1), (TINY, 4), (GEMMA, 2), (GEMMA, 5), (GEMMA, 100),
                                     (GEMMA, 129), (GEMMA, 1024), ((264, 136, 1001, 80), 1),
                                     ((264, 136, 1001, 80), 3), ((1088, 512, 2048, 160), 70)])
def test_ffn_paths_count_no_violation(shape, T):
    d_model, r, d_ff, k = shape
    dev, _ = make_layer(d_model, r, d_ff, T, layer=40 + T)
    rel, dbg, n = both(lambda: spark.ffn_forward_debug(dev["q"], dev["K1"], dev["K2"], dev["V"], k))
    assert n == 0
    for key in ("out", "x", "theta", "active"):
        assert torch.equal(rel[key], dbg[key]), key


@pytest.mark.parametrize("T", [16, 256])
def test_predictor_counts_no_violation(T):
    d_model, r, d_ff, _ = GEMMA
    dev, _ = make_layer(d_model, r, d_ff, T, layer=60 + T)
    rel, dbg, n = both(lambda: spark.ffn_predictor(dev["q"], dev["K1"]))
    assert n == 0 and torch.equal(rel, dbg)


def test_decode_stack_counts_no_violation():
    d_model, r, d_ff, k = GEMMA
    layers = [synthetic.ffn_layer(d_model, r, d_ff, layer=l) for l in range(3)]
    dev = [(w["K1"].cuda(), w["K2"].cuda(), w["V"].cuda()) for w in layers]
    h0 = synthetic.residual(1, d_model)[0].cuda()
    rel, dbg, n = both(lambda: spark.ffn_decode_stack(h0, dev, k, debug=True))
    assert n == 0
    for a, b in zip(rel, dbg):
        assert torch.equal(a, b)


def test_noalloc_counts_no_violation():
    d_model, r, d_ff, k = GEMMA
    dev, _ = make_layer(d_model, r, d_ff, 1, layer=77)

    def call():
        out = torch.empty(d_model, dtype=torch.bfloat16, device="cuda")
        rc = _binding.lib().spark_ffn_forward_noalloc(dev["q"].data_ptr(), dev["K1"].data_ptr(),
                                                      dev["K2"].data_ptr(), dev["V"].data_ptr(), d_model, r, d_ff,
                                                      k, out.data_ptr(), _binding.stream_handle())
        _binding.check("spark_ffn_forward_noalloc", rc)
        return out

    rel, dbg, n = both(call)
    assert n == 0 and torch.equal(rel, dbg)


@pytest.mark.parametrize("n_ctx,k_attn", [(4096, 256), (500, 64), (100, 200)])
def test_attention_counts_no_violation(n_ctx, k_attn):
    host = synthetic.attention_inputs(8, 4, n_ctx, 256, layer=3)
    dev = {key: v.cuda() for key, v in host.items()}
    rel, dbg, n = both(lambda: spark.attention_decode(dev["q"], dev["K"], dev["V"], 128, k_attn, debug=True))
    assert n == 0
    for key in ("out", "s", "theta", "active"):
        assert torch.equal(rel[key], dbg[key]), key


def test_checked_library_is_separate():
    assert _binding.debug_lib()._handle != _binding.lib()._handle
