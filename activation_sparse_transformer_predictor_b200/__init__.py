"""Spark FFN with statistical top-k on NVIDIA B200 (sm_100a).

Public Python API over the C ABI of ``libspark.so`` (see ``include/spark.h``).
The method is the one of the paper-notes page "Spark Transformer: Reactivating
Sparsity in FFN and Attention", section 方法详解/关键设计 ("Spark FFN",
"Statistical Top-k"):

    x     = K1^T q[:r]
    theta = mean(x) + std(x) * Q(1 - k/d_ff)
    out   = V . (GELU(max(x - theta, 0)) (.) (K2^T q[r:]))

All tensors are CUDA tensors; work is enqueued on the current (or given)
stream.  Weights: K1 bf16 [d_ff, r], K2 bf16 [d_ff, d_model - r], V bf16
[d_ff, d_model]; tokens q bf16 [d_model] or [T, d_model].
"""
from __future__ import annotations

from . import _binding
from ._binding import SparkError

__all__ = ["ffn_forward", "ffn_forward_host", "ffn_forward_debug", "ffn_predictor", "ffn_decode_stack", "stat_topk_soft_threshold",
           "stat_topk_soft_threshold_causal", "stat_topk_huber", "stat_topk_huber_backward", "query_status", "release_workspace",
           "topk_quantile", "set_wait_limit_ns", "selftest_wait_timeout", "debug_violations", "SparkError"]


def _require(t, name, dtype, ndim=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() not in ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ffn_shapes(q, K1, K2, V):
    import torch
    for t, n in ((q, "q"), (K1, "K1"), (K2, "K2"), (V, "V")):
        _require(t, n, torch.bfloat16)
    d_ff, r = K1.shape
    T = 1 if q.dim() == 1 else q.shape[0]
    d_model = q.shape[-1]
    if K2.shape != (d_ff, d_model - r) or V.shape != (d_ff, d_model):
        raise ValueError(f"inconsistent shapes: K1 {tuple(K1.shape)}, K2 {tuple(K2.shape)}, V {tuple(V.shape)}, "
                         f"q {tuple(q.shape)}")
    return T, d_model, r, d_ff


def ffn_forward(q, K1, K2, V, k: int, out=None, stream=None):
    """Spark FFN forward; returns out (bf16, same shape as q)."""
    import torch
    T, d_model, r, d_ff = _ffn_shapes(q, K1, K2, V)
    if out is None:
        out = torch.empty_like(q)
    else:
        _require(out, "out", torch.bfloat16)
    L = _binding.lib()
    st = _binding.stream_handle(stream)
    if q.dim() == 1:
        rc = L.spark_ffn_forward(q.data_ptr(), K1.data_ptr(), K2.data_ptr(), V.data_ptr(), d_model, r, d_ff, int(k),
                                 out.data_ptr(), st)
        _binding.check("spark_ffn_forward", rc)
    else:
        rc = L.spark_ffn_forward_tokens(q.data_ptr(), K1.data_ptr(), K2.data_ptr(), V.data_ptr(), T, d_model, r,
                                        d_ff, int(k), out.data_ptr(), st)
        _binding.check("spark_ffn_forward_tokens", rc)
    return out


def ffn_forward_host(q_host, K1, K2, V, k: int, out_host=None, stream=None):
    """spark_ffn_forward_host: q_host and out_host are bf16 CPU tensors ([d_model] or [T, d_model]),
    pinned for an asynchronous call; the weights are CUDA tensors.  The output copy is enqueued on the
    stream: synchronise before reading out_host.  Returns out_host."""
    import torch
    if q_host.device.type != "cpu" or q_host.dtype != torch.bfloat16 or not q_host.is_contiguous():
        raise ValueError("ffn_forward_host: q_host must be a contiguous bf16 CPU tensor")
    d_model = q_host.shape[-1]
    T = q_host.numel() // d_model if d_model else 0
    _ffn_shapes(torch.empty(d_model, dtype=torch.bfloat16, device=K1.device), K1, K2, V)
    d_ff, r = K1.shape
    if out_host is None:
        out_host = torch.empty(tuple(q_host.shape), dtype=torch.bfloat16, pin_memory=q_host.is_pinned())
    elif out_host.device.type != "cpu" or out_host.dtype != torch.bfloat16 or out_host.shape != q_host.shape \
            or not out_host.is_contiguous():
        raise ValueError("ffn_forward_host: out_host must be a contiguous bf16 CPU tensor shaped like q_host")
    rc = _binding.lib().spark_ffn_forward_host(q_host.data_ptr(), K1.data_ptr(), K2.data_ptr(), V.data_ptr(), T,
                                               d_model, r, d_ff, int(k), out_host.data_ptr(),
                                               _binding.stream_handle(stream))
    _binding.check("spark_ffn_forward_host", rc)
    return out_host


def ffn_forward_debug(q, K1, K2, V, k: int, stream=None) -> dict:
    """Spark FFN forward that also returns x (fp32 [T, d_ff]), theta (fp32 [T]) and the
    active mask (uint8 [T, d_ff], 1 where x > theta) the kernels used."""
    import torch
    T, d_model, r, d_ff = _ffn_shapes(q, K1, K2, V)
    q2 = q.reshape(T, d_model)
    out = torch.empty_like(q2)
    x = torch.empty((T, d_ff), dtype=torch.float32, device=q.device)
    theta = torch.empty((T,), dtype=torch.float32, device=q.device)
    active = torch.empty((T, d_ff), dtype=torch.uint8, device=q.device)
    rc = _binding.lib().spark_ffn_forward_debug(q2.data_ptr(), K1.data_ptr(), K2.data_ptr(), V.data_ptr(), T,
                                                d_model, r, d_ff, int(k), out.data_ptr(), x.data_ptr(),
                                                theta.data_ptr(), active.data_ptr(), _binding.stream_handle(stream))
    _binding.check("spark_ffn_forward_debug", rc)
    return {"out": out.reshape(q.shape), "x": x, "theta": theta, "active": active}


def ffn_predictor(q, K1, out=None, stream=None):
    """The low-rank predictor alone: x = K1^T q[:r] for each token, fp32 [T, d_ff]."""
    import torch
    _require(q, "q", torch.bfloat16, ndim=(1, 2))
    _require(K1, "K1", torch.bfloat16, ndim=(2,))
    d_ff, r = K1.shape
    T = 1 if q.dim() == 1 else q.shape[0]
    d_model = q.shape[-1]
    if out is None:
        out = torch.empty((T, d_ff), dtype=torch.float32, device=q.device)
    else:
        _require(out, "out", torch.float32)
    rc = _binding.lib().spark_ffn_predictor(q.data_ptr(), K1.data_ptr(), T, d_model, r, d_ff, out.data_ptr(),
                                            _binding.stream_handle(stream))
    _binding.check("spark_ffn_predictor", rc)
    return out


def ffn_decode_stack(h, layers, k: int, eps: float = 1e-6, h_out=None, debug: bool = False, stream=None):
    """Run a stack of Spark FFN layers on one token's fp32 residual h [d_model]:
    q_l = bf16(RMSNorm(h_l)), h_{l+1} = h_l + SparkFFN_l(q_l).  `layers` is a list of
    (K1, K2, V) bf16 CUDA tensors.  Returns h_out, or (h_out, q [L, d], out [L, d]) with debug."""
    import ctypes

    import torch
    _require(h, "h", torch.float32, ndim=(1,))
    d_model = h.shape[0]
    L = len(layers)
    for i, (K1, K2, V) in enumerate(layers):
        _ffn_shapes(torch.empty(d_model, dtype=torch.bfloat16, device=h.device), K1, K2, V)
    if h_out is None:
        h_out = torch.empty_like(h)
    d_ff, r = layers[0][0].shape if L else (1, 1)
    ptrs = [(ctypes.c_void_p * max(L, 1))(*[t[j].data_ptr() for t in layers]) for j in range(3)]
    qd = od = None
    if debug:
        qd = torch.empty((L, d_model), dtype=torch.bfloat16, device=h.device)
        od = torch.empty((L, d_model), dtype=torch.bfloat16, device=h.device)
    rc = _binding.lib().spark_ffn_decode_stack(h.data_ptr(), h_out.data_ptr(), ptrs[0], ptrs[1], ptrs[2], L, d_model,
                                               r, d_ff, int(k), float(eps), _binding.ptr(qd), _binding.ptr(od),
                                               _binding.stream_handle(stream))
    _binding.check("spark_ffn_decode_stack", rc)
    return (h_out, qd, od) if debug else h_out


def stat_topk_soft_threshold(x, k: int, out=None, stream=None):
    """Row-wise statistical top-k with soft threshold on fp32 [rows, d]; out may be x."""
    import torch
    _require(x, "x", torch.float32)
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    if out is None:
        out = torch.empty_like(x)
    else:
        _require(out, "out", torch.float32)
    rc = _binding.lib().stat_topk_soft_threshold(x.data_ptr(), rows, d, int(k), out.data_ptr(),
                                                 _binding.stream_handle(stream))
    _binding.check("stat_topk_soft_threshold", rc)
    return out


def stat_topk_soft_threshold_causal(x, k: int, n_q: int | None = None, offset: int = 0, out=None, theta=None,
                                    stream=None):
    """Statistical top-k with soft threshold on causally masked fp32 rows [rows, d]: row r sees its first
    min(d, offset + r % n_q + 1) entries (n_q defaults to d: square causal scores); rows seeing at most k
    entries keep them all (theta = -inf).  Returns out, or (out, theta) when theta is a tensor to fill."""
    import torch
    _require(x, "x", torch.float32)
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    n_q = d if n_q is None else int(n_q)
    if out is None:
        out = torch.empty_like(x)
    else:
        _require(out, "out", torch.float32)
    if theta is not None:
        _require(theta, "theta", torch.float32)
    rc = _binding.lib().stat_topk_soft_threshold_causal(x.data_ptr(), rows, d, int(k), n_q, int(offset),
                                                        out.data_ptr(), _binding.ptr(theta),
                                                        _binding.stream_handle(stream))
    _binding.check("stat_topk_soft_threshold_causal", rc)
    return out if theta is None else (out, theta)


def stat_topk_huber(x, k: int, delta: float, out=None, stream=None):
    """Huber-smoothed statistical top-k on fp32 rows [rows, d]: out = rho_delta(x - theta(x))."""
    import torch
    _require(x, "x", torch.float32)
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    if out is None:
        out = torch.empty_like(x)
    else:
        _require(out, "out", torch.float32)
    rc = _binding.lib().stat_topk_huber(x.data_ptr(), rows, d, int(k), float(delta), out.data_ptr(),
                                        _binding.stream_handle(stream))
    _binding.check("stat_topk_huber", rc)
    return out


def stat_topk_huber_backward(x, grad_out, k: int, delta: float, grad_x=None, stream=None):
    """Gradient of sum(grad_out * stat_topk_huber(x)) with respect to x (fp32 [rows, d])."""
    import torch
    _require(x, "x", torch.float32)
    _require(grad_out, "grad_out", torch.float32)
    if grad_out.shape != x.shape:
        raise ValueError("stat_topk_huber_backward: x and grad_out differ in shape")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    if grad_x is None:
        grad_x = torch.empty_like(x)
    else:
        _require(grad_x, "grad_x", torch.float32)
    rc = _binding.lib().stat_topk_huber_backward(x.data_ptr(), grad_out.data_ptr(), rows, d, int(k), float(delta),
                                                 grad_x.data_ptr(), _binding.stream_handle(stream))
    _binding.check("stat_topk_huber_backward", rc)
    return grad_x


def query_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status code."""
    return int(_binding.lib().spark_query_status(_binding.stream_handle(stream)))


def debug_violations() -> int:
    """Failed bounds checks since the previous call in the current library
    (cleared by the call); -1 in the release build.  Use inside
    ``_binding.using_library(_binding.debug_lib())`` to read the checked build."""
    n = int(_binding.lib().spark_debug_violations())
    if n < -1:
        raise SparkError("spark_debug_violations", n)
    return n


def release_workspace() -> None:
    _binding.check("spark_release_workspace", _binding.lib().spark_release_workspace())


def topk_quantile(k: int, d: int) -> float:
    """Q(1 - k/d) as the library computes it (host, fp64)."""
    return float(_binding.lib().spark_topk_quantile(int(k), int(d)))


def set_wait_limit_ns(ns: int) -> None:
    _binding.check("spark_set_wait_limit_ns", _binding.lib().spark_set_wait_limit_ns(int(ns)))


def attention_decode(q, K, V, r: int, k_attn: int, scale: float | None = None, out=None, debug: bool = False,
                     stream=None):
    """Spark Attention for one decoding position (spark_attention_decode).

    q: bf16 [n_heads, d_head]; K, V: bf16 [n_kv_heads, n_ctx, d_head].  scale defaults to
    1/sqrt(d_head).  Returns out (bf16 [n_heads, d_head]), or with debug=True a dict with out,
    s (fp32 [n_heads, n_ctx]), theta (fp32 [n_heads]) and active (uint8 [n_heads, n_ctx]).
    """
    import math

    import torch
    _require(q, "q", torch.bfloat16, (2,))
    _require(K, "K", torch.bfloat16, (3,))
    _require(V, "V", torch.bfloat16, (3,))
    n_heads, d_head = q.shape
    n_kv, n_ctx, dk = K.shape
    if dk != d_head or tuple(V.shape) != tuple(K.shape):
        raise ValueError("attention_decode: q [H, d], K and V [H_kv, n_ctx, d]")
    if scale is None:
        scale = 1.0 / math.sqrt(d_head)
    if out is None:
        out = torch.empty_like(q)
    else:
        _require(out, "out", torch.bfloat16, (2,))
    st = _binding.stream_handle(stream)
    L = _binding.lib()
    if not debug:
        rc = L.spark_attention_decode(q.data_ptr(), K.data_ptr(), V.data_ptr(), n_heads, n_kv, n_ctx, d_head,
                                      int(r), int(k_attn), float(scale), out.data_ptr(), st)
        _binding.check("spark_attention_decode", rc)
        return out
    s = torch.empty((n_heads, n_ctx), dtype=torch.float32, device=q.device)
    th = torch.empty(n_heads, dtype=torch.float32, device=q.device)
    act = torch.empty((n_heads, n_ctx), dtype=torch.uint8, device=q.device)
    rc = L.spark_attention_decode_debug(q.data_ptr(), K.data_ptr(), V.data_ptr(), n_heads, n_kv, n_ctx, d_head,
                                        int(r), int(k_attn), float(scale), out.data_ptr(), s.data_ptr(),
                                        th.data_ptr(), act.data_ptr(), st)
    _binding.check("spark_attention_decode_debug", rc)
    return {"out": out, "s": s, "theta": th, "active": act}


def set_weight_overlap(enable: bool) -> None:
    """Let the single-token score kernel stream K1 behind the preceding kernel (spark_set_weight_overlap)."""
    _binding.check("spark_set_weight_overlap", _binding.lib().spark_set_weight_overlap(1 if enable else 0))


def selftest_wait_timeout(stream=None) -> int:
    """Run the bounded-wait self-test; returns the status spark_query_status reports after it."""
    st = _binding.stream_handle(stream)
    _binding.check("spark_selftest_wait_timeout", _binding.lib().spark_selftest_wait_timeout(st))
    return int(_binding.lib().spark_query_status(st))
