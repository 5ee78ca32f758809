"""ctypes binding of libspark.so -- argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
only checks tensor dtypes/devices/contiguity, passes raw device pointers and
the current CUDA stream through the C ABI of ``include/spark.h``, and turns
status codes into exceptions.  There is no fallback: if the library is
missing, every call raises.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libspark.so")
# the same library compiled with SPARK_DEBUG (bounds-checked kernels)
DEBUG_LIB_PATH = os.path.join(PKG, "libspark_debug.so")

SPARK_OK = 0
STATUS_NAMES = {0: "SPARK_OK", -1: "SPARK_EINVAL", -2: "SPARK_EALIGN", -3: "SPARK_ECUDA", -4: "SPARK_ENOMEM",
                -5: "SPARK_ETIMEOUT", -6: "SPARK_EDEVICE", -7: "SPARK_ESCRATCH",
                -8: "SPARK_EBOUNDS"}

# Every symbol that include/spark.h declares.
EXPORTS = ("spark_ffn_forward", "spark_ffn_forward_tokens", "spark_ffn_forward_debug", "stat_topk_soft_threshold",
           "spark_query_status", "spark_release_workspace", "spark_status_string", "spark_topk_quantile",
           "spark_set_wait_limit_ns", "spark_selftest_wait_timeout", "spark_version", "spark_ffn_forward_noalloc",
           "spark_ffn_decode_stack", "spark_set_weight_overlap", "spark_attention_decode",
           "spark_attention_decode_debug", "spark_ffn_predictor", "stat_topk_soft_threshold_causal",
           "stat_topk_huber", "stat_topk_huber_backward", "spark_debug_violations", "spark_ffn_forward_host")

_lock = threading.Lock()
_lib = None
_debug_lib = None
_override = None


class SparkError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


def _load(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m activation_sparse_transformer_predictor_b200.build`")
    L = ctypes.CDLL(path)
    vp, ci = ctypes.c_void_p, ctypes.c_int
    L.spark_ffn_forward.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, vp, vp]
    L.spark_ffn_forward_tokens.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, vp]
    L.spark_ffn_forward_host.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, vp]
    L.spark_ffn_forward_debug.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp]
    L.stat_topk_soft_threshold.argtypes = [vp, ci, ci, ci, vp, vp]
    L.spark_query_status.argtypes = [vp]
    L.spark_release_workspace.argtypes = []
    L.spark_status_string.argtypes = [ci]
    L.spark_status_string.restype = ctypes.c_char_p
    L.spark_topk_quantile.argtypes = [ci, ci]
    L.spark_topk_quantile.restype = ctypes.c_double
    L.spark_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    L.spark_set_weight_overlap.argtypes = [ci]
    L.spark_attention_decode.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, ctypes.c_float, vp, vp]
    L.spark_attention_decode_debug.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, ctypes.c_float, vp, vp, vp,
                                               vp, vp]
    L.spark_selftest_wait_timeout.argtypes = [vp]
    L.spark_version.argtypes = []
    L.spark_debug_violations.argtypes = []
    L.spark_ffn_forward_noalloc.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, vp, vp]
    L.spark_ffn_decode_stack.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ctypes.c_float, vp, vp, vp]
    L.spark_ffn_predictor.argtypes = [vp, vp, ci, ci, ci, ci, vp, vp]
    L.stat_topk_soft_threshold_causal.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp]
    L.stat_topk_huber.argtypes = [vp, ci, ci, ci, ctypes.c_float, vp, vp]
    L.stat_topk_huber_backward.argtypes = [vp, vp, ci, ci, ci, ctypes.c_float, vp, vp]
    for name in EXPORTS:
        if name not in ("spark_status_string", "spark_topk_quantile"):
            getattr(L, name).restype = ci
    return L


def lib() -> ctypes.CDLL:
    """The library every wrapper calls: libspark.so (raises if it has not been
    built), or the one installed by ``using_library``."""
    global _lib
    if _override is not None:
        return _override
    with _lock:
        if _lib is None:
            _lib = _load(LIB_PATH)
        return _lib


def debug_lib() -> ctypes.CDLL:
    """libspark_debug.so, the bounds-checked build (raises if it has not been built)."""
    global _debug_lib
    with _lock:
        if _debug_lib is None:
            _debug_lib = _load(DEBUG_LIB_PATH)
        return _debug_lib


@contextlib.contextmanager
def using_library(L: ctypes.CDLL):
    """Route every wrapper through ``L`` (e.g. ``debug_lib()``) inside the block.
    Process-wide and not thread-safe; each library keeps its own workspaces."""
    global _override
    prev, _override = _override, L
    try:
        yield L
    finally:
        _override = prev


def check(fn: str, status: int) -> None:
    if status != SPARK_OK:
        raise SparkError(fn, status)


def ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)
