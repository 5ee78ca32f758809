"""A decoder stack of Spark FFN layers at decode T = 1 (26 Gemma-2-2B-shaped
layers, per-layer seeds, unit-gain RMSNorm with eps 1e-6 between layers).

Checked per layer with teacher forcing: the oracle runs layer l on the GPU's own
q_l, so that active-set flips cannot compound; the fp32 residual chain
h_{l+1} = h_l + out_l is checked bit for bit; q_l = bf16(RMSNorm(h_l)) against the
oracle's fp64 RMSNorm within one bf16 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
import activation_sparse_transformer_predictor_b200 as spark
from activation_sparse_transformer_predictor_b200 import synthetic

from .parity import assert_outputs_close, bf16_to_f64

pytestmark = pytest.mark.gpu


def _stack(d_model, r, d_ff, L):
    cpu = [synthetic.ffn_layer(d_model, r, d_ff, layer=l) for l in range(L)]
    dev = [(w["K1"].cuda(), w["K2"].cuda(), w["V"].cuda()) for w in cpu]
    return cpu, dev


@pytest.mark.parametrize("shape,L", [((2304, 1152, 9216, 737), 26), ((256, 128, 1024, 82), 3)])
def test_stack_teacher_forced(shape, L):
    d_model, r, d_ff, k = shape
    eps = 1e-6
    cpu, dev = _stack(d_model, r, d_ff, L)
    h0 = synthetic.residual(1, d_model)[0]
    hout, qd, od = spark.ffn_decode_stack(h0.cuda(), dev, k, eps, debug=True)
    torch.cuda.synchronize()
    assert spark.query_status() == 0
    outs = od.float().cpu().numpy()
    hs = [h0.numpy().astype(np.float32)]
    for l in range(L):
        hs.append((hs[-1] + outs[l]).astype(np.float32))
    assert np.array_equal(hout.cpu().numpy(), hs[-1])  # fp32 residual chain, bit for bit
    for l in range(L):
        ref_q = oracle.rmsnorm(hs[l].astype(np.float64), eps)
        gq = bf16_to_f64(qd[l])
        assert np.all(np.abs(gq - ref_q) <= 2.0 ** -8 * np.abs(ref_q)), l
        bits = {n: synthetic.bf16_bits(t) for n, t in cpu[l].items()}
        qb = synthetic.bf16_bits(qd[l].cpu())[None, :]
        ref = oracle.spark_ffn(qb, bits["K1"], bits["K2"], bits["V"], r, k, n_threads=8)["out"]
        assert_outputs_close(outs[l][None, :].astype(np.float64), ref)


def test_stack_matches_single_layer_calls():
    d_model, r, d_ff, k = 2304, 1152, 9216, 737
    cpu, dev = _stack(d_model, r, d_ff, 4)
    h0 = synthetic.residual(1, d_model)[0].cuda()
    hout, qd, od = spark.ffn_decode_stack(h0, dev, k, debug=True)
    # the same q through the single-layer entry point gives the same bits
    for l in range(4):
        one = spark.ffn_forward(qd[l].contiguous(), *dev[l], k)
        assert torch.equal(one, od[l])
    # in place: h_out aliasing h_in
    h = h0.clone()
    spark.ffn_decode_stack(h, dev, k, h_out=h)
    assert torch.equal(h, hout)
