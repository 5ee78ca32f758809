"""fp64 CPU oracle for the Spark FFN and statistical top-k.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library never links or calls it, and it imports nothing from the product.

The arithmetic lives in ``spark_oracle.c`` (plain loops in double precision);
this module only compiles it with gcc and marshals numpy arrays through ctypes.
Source of the method: the paper-notes page "Spark Transformer: Reactivating
Sparsity in FFN and Attention", section 方法详解/关键设计 ("Spark FFN" and
"Statistical Top-k").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spark_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libspark_oracle.so")
_lock = threading.Lock()
_lib = None

GELU_TANH = 0
GELU_ERF = 1


def build(force: bool = False) -> str:
    """Compile spark_oracle.c into libspark_oracle.so (gcc, OpenMP, no FMA contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        # SPARK_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        lib = ctypes.CDLL(os.environ.get("SPARK_ORACLE_LIB") or build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_normal_upper_tail.restype = ctypes.c_double
        lib.oracle_normal_upper_tail.argtypes = [ctypes.c_double]
        lib.oracle_topk_quantile.restype = ctypes.c_double
        lib.oracle_topk_quantile.argtypes = [ctypes.c_double, ctypes.c_double]
        lib.oracle_row_stats.restype = None
        lib.oracle_row_stats.argtypes = [dp, ctypes.c_long, dp, dp]
        lib.oracle_theta.restype = ctypes.c_double
        lib.oracle_theta.argtypes = [dp, ctypes.c_long, ctypes.c_long, dp, dp]
        lib.oracle_gelu_tanh.restype = ctypes.c_double
        lib.oracle_gelu_tanh.argtypes = [ctypes.c_double]
        lib.oracle_gelu_erf.restype = ctypes.c_double
        lib.oracle_gelu_erf.argtypes = [ctypes.c_double]
        lib.oracle_stat_topk.restype = ctypes.c_int
        lib.oracle_stat_topk.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.c_int]
        lib.oracle_stat_topk_huber.restype = ctypes.c_int
        lib.oracle_stat_topk_huber.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                               ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_stat_topk_huber_backward.restype = ctypes.c_int
        lib.oracle_stat_topk_huber_backward.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_long,
                                                        ctypes.c_long, ctypes.c_long, ctypes.c_double,
                                                        ctypes.c_void_p]
        lib.oracle_stat_topk_causal.restype = ctypes.c_int
        lib.oracle_stat_topk_causal.argtypes = [ctypes.c_void_p, ctypes.c_long, ctypes.c_long, ctypes.c_long,
                                                ctypes.c_long, ctypes.c_long, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_int]
        lib.oracle_spark_ffn.restype = ctypes.c_int
        lib.oracle_spark_ffn.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_long] * 5 + [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.oracle_softplus.restype = ctypes.c_double
        lib.oracle_softplus.argtypes = [ctypes.c_double]
        lib.oracle_spark_attention.restype = ctypes.c_int
        lib.oracle_spark_attention.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_long] * 6 + [
            ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int]
        lib.oracle_rmsnorm.restype = None
        lib.oracle_rmsnorm.argtypes = [dp, ctypes.c_long, ctypes.c_double, dp]
        lib.oracle_num_threads_available.restype = ctypes.c_int
        lib.oracle_num_threads_available.argtypes = []
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().oracle_num_threads_available())


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64, one element at a time."""
    lib = _load()
    flat = np.ascontiguousarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.oracle_bf16_to_f64(int(b)) for b in flat], dtype=np.float64).reshape(bits.shape)


def topk_quantile(k: float, d: float) -> float:
    """Q(1 - k/d), the standard-normal quantile, by bisection on erfc."""
    return float(_load().oracle_topk_quantile(float(k), float(d)))


def normal_upper_tail(z: float) -> float:
    return float(_load().oracle_normal_upper_tail(float(z)))


def row_stats(x: np.ndarray) -> tuple[float, float]:
    """Population mean and std of a 1-D row (two passes, fp64)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    m = ctypes.c_double()
    s = ctypes.c_double()
    _load().oracle_row_stats(_dptr(x), x.size, ctypes.byref(m), ctypes.byref(s))
    return m.value, s.value


def theta(x: np.ndarray, k: int) -> float:
    x = np.ascontiguousarray(x, dtype=np.float64)
    return float(_load().oracle_theta(_dptr(x), x.size, int(k), None, None))


def gelu(s: float, kind: int = GELU_TANH) -> float:
    lib = _load()
    return float(lib.oracle_gelu_erf(s) if kind == GELU_ERF else lib.oracle_gelu_tanh(s))


def stat_topk(x: np.ndarray, k: int, n_threads: int = 1):
    """Statistical top-k + soft threshold on fp32 rows [rows, d].

    Returns (out fp64 [rows,d], theta [rows], mean [rows], std [rows]).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim == 1:
        x = x[None, :]
    rows, d = x.shape
    out = np.empty((rows, d), dtype=np.float64)
    th = np.empty(rows, dtype=np.float64)
    mu = np.empty(rows, dtype=np.float64)
    sd = np.empty(rows, dtype=np.float64)
    rc = _load().oracle_stat_topk(_ptr(x), rows, d, int(k), _ptr(out), _ptr(th), _ptr(mu),
                                  _ptr(sd), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_stat_topk: invalid arguments (d={d}, k={k})")
    return out, th, mu, sd


def stat_topk_huber(x: np.ndarray, k: int, delta: float):
    """Huber-smoothed statistical top-k on fp64 rows [rows, d]: out = rho_delta(x - theta(x)).
    Returns (out [rows, d], theta [rows])."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    if x.ndim == 1:
        x = x[None, :]
    rows, d = x.shape
    out = np.empty((rows, d), dtype=np.float64)
    th = np.empty(rows, dtype=np.float64)
    if _load().oracle_stat_topk_huber(_ptr(x), rows, d, int(k), float(delta), _ptr(out), _ptr(th)) != 0:
        raise ValueError(f"oracle_stat_topk_huber: invalid arguments (d={d}, k={k}, delta={delta})")
    return out, th


def stat_topk_huber_backward(x: np.ndarray, g: np.ndarray, k: int, delta: float) -> np.ndarray:
    """dL/dx of the Huber-smoothed statistical top-k for upstream gradient g (both fp64 [rows, d])."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(g, dtype=np.float64)
    if x.ndim == 1:
        x, g = x[None, :], g[None, :]
    if g.shape != x.shape:
        raise ValueError("stat_topk_huber_backward: x and g differ in shape")
    rows, d = x.shape
    dx = np.empty((rows, d), dtype=np.float64)
    if _load().oracle_stat_topk_huber_backward(_ptr(x), _ptr(g), rows, d, int(k), float(delta), _ptr(dx)) != 0:
        raise ValueError(f"oracle_stat_topk_huber_backward: invalid arguments (d={d}, k={k}, delta={delta})")
    return dx


def stat_topk_causal(x: np.ndarray, k: int, n_q: int, offset: int = 0, n_threads: int = 1):
    """Statistical top-k + soft threshold on causally masked fp32 rows [rows, d]: row i sees its
    first min(d, offset + i % n_q + 1) entries.  Returns (out fp64 [rows, d], theta [rows];
    theta = -inf on rows whose visible entries number at most k, which pass through unshifted)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim == 1:
        x = x[None, :]
    rows, d = x.shape
    out = np.empty((rows, d), dtype=np.float64)
    th = np.empty(rows, dtype=np.float64)
    rc = _load().oracle_stat_topk_causal(_ptr(x), rows, d, int(k), int(n_q), int(offset), _ptr(out), _ptr(th),
                                         int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_stat_topk_causal: invalid arguments (d={d}, k={k}, n_q={n_q}, offset={offset})")
    return out, th


def spark_ffn(q_bits, K1_bits, K2_bits, V_bits, r: int, k: int, gelu_kind: int = GELU_TANH,
              override_active=None, n_threads: int = 1):
    """Spark FFN forward on bf16 bit patterns (uint16 arrays).

    q_bits [T, d_model], K1_bits [d_ff, r], K2_bits [d_ff, d_model - r],
    V_bits [d_ff, d_model].  Returns a dict with out [T, d_model] (fp64),
    x [T, d_ff], theta/mean/std [T] and active [T, d_ff] (bool, x > theta).
    """
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    if q.ndim == 1:
        q = q[None, :]
    K1 = np.ascontiguousarray(K1_bits, dtype=np.uint16)
    K2 = np.ascontiguousarray(K2_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    T, d_model = q.shape
    d_ff = K1.shape[0]
    if K1.shape != (d_ff, r) or K2.shape != (d_ff, d_model - r) or V.shape != (d_ff, d_model):
        raise ValueError("oracle.spark_ffn: inconsistent shapes")
    ov = None
    if override_active is not None:
        ov = np.ascontiguousarray(override_active, dtype=np.uint8).reshape(T, d_ff)
    out = np.empty((T, d_model), dtype=np.float64)
    x = np.empty((T, d_ff), dtype=np.float64)
    th = np.empty(T, dtype=np.float64)
    mu = np.empty(T, dtype=np.float64)
    sd = np.empty(T, dtype=np.float64)
    act = np.empty((T, d_ff), dtype=np.uint8)
    rc = _load().oracle_spark_ffn(_ptr(q), _ptr(K1), _ptr(K2), _ptr(V), T, d_model, r, d_ff, int(k),
                                  int(gelu_kind), _ptr(ov), _ptr(out), _ptr(x), _ptr(th), _ptr(mu),
                                  _ptr(sd), _ptr(act), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_spark_ffn: invalid arguments")
    return {"out": out, "x": x, "theta": th, "mean": mu, "std": sd, "active": act.astype(bool)}


def rmsnorm(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.float64)
    y = np.empty_like(h)
    _load().oracle_rmsnorm(_dptr(h), h.size, float(eps), _dptr(y))
    return y


def softplus(a: float) -> float:
    return float(_load().oracle_softplus(float(a)))


def spark_attention(q_bits, K_bits, V_bits, r: int, k_attn: int, scale: float, override_active=None,
                    n_threads: int = 1):
    """Spark Attention for one decoding position on bf16 bit patterns (uint16 arrays).

    q_bits [n_heads, d_head]; K_bits and V_bits [n_kv_heads, n_ctx, d_head].  Returns a dict with
    out [n_heads, d_head] (fp64), s [n_heads, n_ctx] (scaled predictor scores), theta [n_heads]
    (-inf when every key is selected) and active [n_heads, n_ctx] (bool, s > theta).
    """
    q = np.ascontiguousarray(q_bits, dtype=np.uint16)
    K = np.ascontiguousarray(K_bits, dtype=np.uint16)
    V = np.ascontiguousarray(V_bits, dtype=np.uint16)
    n_heads, d_head = q.shape
    n_kv, n_ctx, dk = K.shape
    if dk != d_head or V.shape != K.shape or n_heads % n_kv != 0:
        raise ValueError("oracle.spark_attention: inconsistent shapes")
    ov = None
    if override_active is not None:
        ov = np.ascontiguousarray(override_active, dtype=np.uint8).reshape(n_heads, n_ctx)
    out = np.empty((n_heads, d_head), dtype=np.float64)
    sc = np.empty((n_heads, n_ctx), dtype=np.float64)
    th = np.empty(n_heads, dtype=np.float64)
    act = np.empty((n_heads, n_ctx), dtype=np.uint8)
    rc = _load().oracle_spark_attention(_ptr(q), _ptr(K), _ptr(V), n_heads, n_kv, n_ctx, d_head, int(r),
                                        int(k_attn), float(scale), _ptr(ov), _ptr(out), _ptr(sc), _ptr(th),
                                        _ptr(act), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_spark_attention: invalid arguments")
    return {"out": out, "s": sc, "theta": th, "active": act.astype(bool)}
