"""Seeded synthetic inputs shared by the CUDA path and the oracle.

This module holds no arithmetic of the method: it only draws random numbers
with a fixed recipe, so that the GPU path and the fp64 oracle see the same
bits.  Recipe (Gemma-2-2B-shaped layers stand in for trained weights, which
are not available):

* weights: ``randn`` in fp32 scaled by ``1/sqrt(fan_in)`` then rounded to
  bf16 (round-to-nearest-even by ``Tensor.to``).  fan_in is r for K1,
  d_model - r for K2 and d_ff for V (V maps the d_ff activations back to
  d_model).
* tokens q: ``randn`` fp32 -> bf16, i.e. ~N(0, 1).
* score rows: fp32 ~N(0, 1), or Student-t with 4 degrees of freedom drawn as
  Z / sqrt(W / 4) with W = -2 ln(U1 U2) ~ chi-square(4).
* attention (one decoding position): query heads, cached keys and values
  ``randn`` fp32 -> bf16, i.e. ~N(0, 1) (a random model's KV cache).
* seeds: every tensor has its own ``torch.Generator`` seeded with
  ``(base + layer) * 8 + slot`` (slot 0 = K1, 1 = K2, 2 = V, 3 = q, 4 = scores,
  5 = residual, 6 = attention keys, 7 = attention values; attention queries use slot 3).
"""
from __future__ import annotations

import math

import torch

BASE_SEED = 1234
_SLOT = {"K1": 0, "K2": 1, "V": 2, "q": 3, "scores": 4, "h": 5, "keys": 6, "values": 7}


def _gen(slot: str, layer: int = 0, base: int = BASE_SEED) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((base + layer) * 8 + _SLOT[slot])
    return g


def _randn(shape, gen) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32)


def ffn_layer(d_model: int, r: int, d_ff: int, layer: int = 0, base: int = BASE_SEED) -> dict:
    """K1 [d_ff, r], K2 [d_ff, d_model - r], V [d_ff, d_model], bf16, CPU, row-major."""
    K1 = (_randn((d_ff, r), _gen("K1", layer, base)) * (1.0 / math.sqrt(r))).to(torch.bfloat16)
    K2 = (_randn((d_ff, d_model - r), _gen("K2", layer, base)) * (1.0 / math.sqrt(d_model - r))).to(
        torch.bfloat16)
    V = (_randn((d_ff, d_model), _gen("V", layer, base)) * (1.0 / math.sqrt(d_ff))).to(torch.bfloat16)
    return {"K1": K1.contiguous(), "K2": K2.contiguous(), "V": V.contiguous()}


def tokens(T: int, d_model: int, layer: int = 0, base: int = BASE_SEED) -> torch.Tensor:
    """q [T, d_model] bf16 ~N(0, 1)."""
    return _randn((T, d_model), _gen("q", layer, base)).to(torch.bfloat16).contiguous()


def residual(T: int, d_model: int, base: int = BASE_SEED) -> torch.Tensor:
    """Initial residual stream h0 [T, d_model] fp32 ~N(0, 1) for a layer stack."""
    return _randn((T, d_model), _gen("h", 0, base)).contiguous()


def score_rows(rows: int, d: int, dist: str = "normal", base: int = BASE_SEED) -> torch.Tensor:
    """fp32 [rows, d] score rows, ~N(0,1) or Student-t(4)."""
    g = _gen("scores", 0, base)
    z = _randn((rows, d), g)
    if dist == "normal":
        return z.contiguous()
    if dist == "student_t4":
        u1 = 1.0 - torch.rand((rows, d), generator=g, dtype=torch.float64)
        u2 = 1.0 - torch.rand((rows, d), generator=g, dtype=torch.float64)
        w = -2.0 * torch.log(u1 * u2)
        return (z.double() / torch.sqrt(w / 4.0)).float().contiguous()
    raise ValueError(f"unknown distribution {dist!r}")


def attention_inputs(n_heads: int, n_kv_heads: int, n_ctx: int, d_head: int, layer: int = 0,
                     base: int = BASE_SEED) -> dict:
    """q [n_heads, d_head], K and V [n_kv_heads, n_ctx, d_head], all bf16 ~N(0, 1)."""
    q = _randn((n_heads, d_head), _gen("q", layer, base)).to(torch.bfloat16)
    K = _randn((n_kv_heads, n_ctx, d_head), _gen("keys", layer, base)).to(torch.bfloat16)
    V = _randn((n_kv_heads, n_ctx, d_head), _gen("values", layer, base)).to(torch.bfloat16)
    return {"q": q, "K": K, "V": V}


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (for the oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
