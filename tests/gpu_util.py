"""Shared set-up for the GPU tests: seeded layers on the device plus their bf16 bits for the oracle."""
import numpy as np
import torch

from activation_sparse_transformer_predictor_b200 import synthetic


def widen(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def make_layer(d_model, r, d_ff, T, layer=0, base=synthetic.BASE_SEED, device="cuda"):
    w = synthetic.ffn_layer(d_model, r, d_ff, layer=layer, base=base)
    q = synthetic.tokens(T, d_model, layer=layer, base=base)
    host = {"q": q, **w}
    dev = {k: v.to(device) for k, v in host.items()}
    bits = {k: synthetic.bf16_bits(v) for k, v in host.items()}
    return dev, bits
