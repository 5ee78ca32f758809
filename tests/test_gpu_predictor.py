"""GPU parity of the predictor-only entry point (spark_ffn_predictor): the
low-rank predictor x = K1^T q[:r] of the Spark FFN (Spark Transformer notes,
关键设计 / "Spark FFN") on the tensor cores, against the fp64 oracle's x within
the kernel's rigorous fp32 error bound, at token counts that take each GEMM
unit shape (64-row token boxes, 128 x 128 and 128 x 256 units) and ragged edges."""
import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark

from .gpu_util import make_layer, widen
from .parity import x_tolerance

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,T", [
    ((2304, 1152, 9216, 737), 1),
    ((2304, 1152, 9216, 737), 16),      # one token band: 128 x 64 units, 64-row token boxes
    ((2304, 1152, 9216, 737), 64),
    ((2304, 1152, 9216, 737), 100),     # one token band: 128 x 64 units, 128-row token boxes
    ((2304, 1152, 9216, 737), 200),
    ((2304, 1152, 9216, 737), 1100),     # 128 x 256 units, ragged last token band
    ((264, 136, 1008, 80), 7),          # ragged r (two partial K blocks) and d_ff
])
def test_predictor_matches_oracle_scores(shape, T):
    d_model, r, d_ff, k = shape
    dev, bits = make_layer(d_model, r, d_ff, T, layer=T % 89)
    x = spark.ffn_predictor(dev["q"], dev["K1"])
    torch.cuda.synchronize()
    assert spark.query_status() == 0
    toks = np.arange(T) if T <= 64 else np.unique(np.linspace(0, T - 1, 24).astype(int))
    gx = x.cpu().numpy().astype(np.float64)[toks]
    orc = oracle.spark_ffn(bits["q"][toks], bits["K1"], bits["K2"], bits["V"], r, k, n_threads=8)
    tol = x_tolerance(widen(bits["K1"]), widen(bits["q"][toks][:, :r]), r)
    assert np.all(np.abs(gx - orc["x"]) <= tol)


@pytest.mark.parametrize("T", [100, 256])
def test_predictor_equals_the_prefill_scores(T):
    """The same GEMM as the predictor stage of spark_ffn_forward_debug: identical bits."""
    d_model, r, d_ff, k = 2304, 1152, 9216, 737
    dev, _ = make_layer(d_model, r, d_ff, T, layer=3)
    x = spark.ffn_predictor(dev["q"], dev["K1"])
    res = spark.ffn_forward_debug(dev["q"], dev["K1"], dev["K2"], dev["V"], k)
    torch.cuda.synchronize()
    assert torch.equal(x, res["x"])
