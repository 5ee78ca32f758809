"""The allocation-free decode entry point, spark_ffn_forward_noalloc.

Some callers cannot allocate device memory while they run -- the execute hook
of an inference-engine plugin, or a runtime that plans all of its device memory
ahead of time.  For them the library has one entry point whose scratch is a
fixed buffer inside the library instead of an allocated workspace.  These tests
call it through the C ABI, twice in a row (the buffer keeps the previous
call's contents), and compare each result with the allocating entry point's
and with the fp64 oracle's, under the same tolerance as the other parity tests.  The file name makes
pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import _binding

from .gpu_util import make_layer
from .parity import assert_outputs_close, bf16_to_f64

pytestmark = pytest.mark.gpu

SPARK_ESCRATCH = -7


def _noalloc(q, K1, K2, V, k, out):
    d_ff, r = K1.shape
    return _binding.lib().spark_ffn_forward_noalloc(q.data_ptr(), K1.data_ptr(), K2.data_ptr(), V.data_ptr(),
                                                    q.shape[-1], r, d_ff, int(k), out.data_ptr(),
                                                    _binding.stream_handle())


@pytest.mark.parametrize("shape", [(2304, 1152, 9216, 737), (256, 128, 1024, 82)])
def test_noalloc_matches_allocating_entry_point_on_two_calls(shape):
    d_model, r, d_ff, k = shape
    for call, layer in enumerate((40, 41)):
        dev, bits = make_layer(d_model, r, d_ff, 1, layer=layer)
        q = dev["q"][0].contiguous()
        ref = spark.ffn_forward(q, dev["K1"], dev["K2"], dev["V"], k)
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(q, dev["K1"], dev["K2"], dev["V"], k, out) == 0, f"call {call}"
        torch.cuda.synchronize()
        assert spark.query_status() == 0
        assert torch.isfinite(out.float()).all()
        # against the allocating entry point ...
        assert_outputs_close(bf16_to_f64(out), bf16_to_f64(ref))
        # ... and against the fp64 oracle (its own active set: neurons that may flip between the
        # two sit within 1e-4 std of theta and contribute GELU(s) ~ s / 2 ~ 0)
        orc = oracle.spark_ffn(bits["q"], bits["K1"], bits["K2"], bits["V"], r, k, n_threads=8)["out"]
        assert_outputs_close(bf16_to_f64(out)[None, :], orc)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # d_model 4096 needs ~4 * 4096 * 148 bytes of partial outputs: more than 2 MiB
    dev, _ = make_layer(4096, 2048, 7104, 1, layer=2)
    q = dev["q"][0].contiguous()
    out = torch.zeros_like(q)
    assert _noalloc(q, dev["K1"], dev["K2"], dev["V"], 568, out) == SPARK_ESCRATCH
    torch.cuda.synchronize()
    assert torch.all(out == 0)  # nothing was enqueued
