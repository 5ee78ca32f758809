"""libspark.so on a machine without a GPU: it loads, exports every symbol that
include/spark.h declares, and its host-only logic (quantile, argument checks,
status strings) behaves.  No kernel is launched here."""
import ctypes
import math
import os
import re

import pytest

import oracle
from activation_sparse_transformer_predictor_b200 import _binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _binding.lib()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"SPARK_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported(L):
    declared = _declared_functions()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(_binding.EXPORTS)


def test_version_and_status_strings(L):
    assert L.spark_version() >= 100
    assert L.spark_status_string(0) == b"SPARK_OK"
    assert L.spark_status_string(-5).startswith(b"SPARK_ETIMEOUT")
    assert L.spark_status_string(123) == b"SPARK_UNKNOWN"


@pytest.mark.parametrize("d", [8, 64, 1000, 1024, 4096, 9216])
def test_host_quantile_matches_oracle(L, d):
    """The library's Q (rational guess + Newton on erfc) against the oracle's bisection."""
    for k in sorted({1, 2, 3, d // 16, d // 12, int(0.08 * d), d // 2, d - 1} - {0, d}):
        assert abs(L.spark_topk_quantile(k, d) - oracle.topk_quantile(k, d)) <= 1e-12 * max(1, abs(
            oracle.topk_quantile(k, d))), (d, k)
    assert math.isnan(L.spark_topk_quantile(0, d)) and math.isnan(L.spark_topk_quantile(d, d))


def test_argument_checks_before_any_device_work(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # never dereferenced: every case below fails validation first
    null = vp(0)
    EINVAL, EALIGN = -1, -2
    f = L.spark_ffn_forward_tokens
    assert f(null, fake, fake, fake, 1, 64, 32, 256, 20, vp(1 << 30), null) == EINVAL  # NULL q
    assert f(fake, fake, fake, fake, -1, 64, 32, 256, 20, vp(1 << 30), null) == EINVAL  # T < 0
    assert f(fake, fake, fake, fake, 0, 64, 32, 256, 20, vp(1 << 30), null) == 0  # empty batch: no-op
    assert f(fake, fake, fake, fake, 1, 64, 64, 256, 20, vp(1 << 30), null) == EINVAL  # r == d_model
    assert f(fake, fake, fake, fake, 1, 64, 0, 256, 20, vp(1 << 30), null) == EINVAL  # r == 0
    assert f(fake, fake, fake, fake, 1, 64, 32, 256, 0, vp(1 << 30), null) == EINVAL  # k == 0
    assert f(fake, fake, fake, fake, 1, 64, 32, 256, 256, vp(1 << 30), null) == EINVAL  # k == d_ff
    assert f(fake, fake, fake, fake, 1, 64, 36, 256, 20, vp(1 << 30), null) == EALIGN  # r % 8
    assert f(fake, fake, fake, fake, 1, 68, 32, 256, 20, vp(1 << 30), null) == EALIGN  # d_model % 8
    assert f(vp((1 << 20) + 2), fake, fake, fake, 1, 64, 32, 256, 20, vp(1 << 30), null) == EALIGN
    # out overlapping q
    assert f(fake, vp(1 << 24), vp(1 << 25), vp(1 << 26), 1, 64, 32, 256, 20, vp((1 << 20) + 64), null) == EINVAL
    hf = L.spark_ffn_forward_host  # host q / out: no alignment asked of them, weights as above
    assert hf(fake, fake, fake, fake, 0, 64, 32, 256, 20, vp(1 << 30), null) == 0  # empty batch: no-op
    assert hf(null, fake, fake, fake, 1, 64, 32, 256, 20, vp(1 << 30), null) == EINVAL  # NULL q_host
    assert hf(fake, fake, fake, fake, 1, 64, 32, 256, 20, null, null) == EINVAL  # NULL out_host
    assert hf(fake, null, fake, fake, 1, 64, 32, 256, 20, vp(1 << 30), null) == EINVAL  # NULL K1
    assert hf(fake, fake, fake, fake, -1, 64, 32, 256, 20, vp(1 << 30), null) == EINVAL  # T < 0
    assert hf(fake, fake, fake, fake, 1, 64, 32, 256, 256, vp(1 << 30), null) == EINVAL  # k == d_ff
    assert hf(fake, fake, fake, fake, 1, 64, 36, 256, 20, vp(1 << 30), null) == EALIGN  # r % 8
    assert hf(fake, vp((1 << 20) + 2), fake, fake, 1, 64, 32, 256, 20, vp(1 << 30), null) == EALIGN  # K1
    assert hf(fake, fake, fake, fake, 2, 64, 32, 256, 20, vp((1 << 20) + 2), null) == EINVAL  # out on q
    t = L.stat_topk_soft_threshold
    assert t(fake, 4, 100, 0, fake, null) == EINVAL
    assert t(fake, 4, 100, 100, fake, null) == EINVAL
    assert t(fake, 4, 1, 1, fake, null) == EINVAL
    assert t(null, 4, 100, 10, fake, null) == EINVAL
    assert t(fake, 0, 100, 10, fake, null) == 0  # no rows: no-op
    assert t(fake, 4, 100, 10, vp((1 << 20) + 16), null) == EINVAL  # partial overlap
    assert t(vp((1 << 20) + 2), 4, 100, 10, vp(1 << 30), null) == EALIGN  # not 4-byte aligned
    p = L.spark_ffn_predictor
    assert p(fake, fake, 0, 64, 32, 256, vp(1 << 30), null) == 0  # no tokens: no-op
    assert p(null, fake, 2, 64, 32, 256, vp(1 << 30), null) == EINVAL
    assert p(fake, fake, -1, 64, 32, 256, vp(1 << 30), null) == EINVAL
    assert p(fake, fake, 2, 64, 64, 256, vp(1 << 30), null) == EINVAL  # r == d_model
    assert p(fake, fake, 2, 64, 32, 264, vp(1 << 30), null) == EALIGN  # d_ff % 16
    assert p(fake, fake, 2, 64, 36, 256, vp(1 << 30), null) == EALIGN  # r % 8
    assert p(fake, fake, 2, 64, 32, 256, vp((1 << 30) + 4), null) == EALIGN  # x_out alignment
    assert p(fake, fake, 2, 64, 32, 256, vp((1 << 20) + 64), null) == EINVAL  # x_out overlapping q
    c = L.stat_topk_soft_threshold_causal
    assert c(fake, 0, 64, 8, 64, 0, fake, null, null) == 0  # no rows: no-op
    assert c(fake, 4, 64, 0, 64, 0, vp(1 << 30), null, null) == EINVAL  # k == 0
    assert c(fake, 4, 64, 8, 0, 0, vp(1 << 30), null, null) == EINVAL  # n_q == 0
    assert c(fake, 4, 64, 8, 64, -1, vp(1 << 30), null, null) == EINVAL  # offset < 0
    assert c(null, 4, 64, 8, 64, 0, vp(1 << 30), null, null) == EINVAL
    assert c(fake, 4, 64, 8, 64, 0, vp((1 << 20) + 16), null, null) == EINVAL  # partial overlap
    assert c(fake, 4, 64, 8, 64, 0, vp(1 << 30), vp((1 << 20) + 8), null) == EINVAL  # theta inside x
    assert c(vp((1 << 20) + 2), 4, 64, 8, 64, 0, vp(1 << 30), null, null) == EALIGN
    h = L.stat_topk_huber
    hb = L.stat_topk_huber_backward
    assert h(fake, 0, 64, 8, 0.1, fake, null) == 0  # no rows: no-op
    assert h(fake, 4, 64, 0, 0.1, vp(1 << 30), null) == EINVAL  # k == 0
    assert h(fake, 4, 64, 8, -0.1, vp(1 << 30), null) == EINVAL  # negative delta
    assert h(fake, 4, 64, 8, float("inf"), vp(1 << 30), null) == EINVAL
    assert h(fake, 4, 64, 8, 0.1, vp((1 << 20) + 16), null) == EINVAL  # partial overlap
    assert hb(fake, vp(1 << 24), 4, 64, 64, 0.1, vp(1 << 30), null) == EINVAL  # k == d
    assert hb(fake, vp(1 << 24), 4, 64, 8, 0.1, vp((1 << 24) + 16), null) == EINVAL  # grad_x inside grad_out
    assert hb(vp((1 << 20) + 2), vp(1 << 24), 4, 64, 8, 0.1, vp(1 << 30), null) == EALIGN


def test_debug_library_exports_the_same_symbols(L):
    """libspark_debug.so (SPARK_DEBUG) declares the same C ABI; the release
    library answers -1 to spark_debug_violations without touching a device."""
    D = _binding.debug_lib()
    for name in _declared_functions():
        assert hasattr(D, name), name
    assert D.spark_version() == L.spark_version()
    assert L.spark_debug_violations() == -1


def test_using_library_routes_every_wrapper_and_restores(L):
    """The binding's override (used to run the wrappers through the bounds-checked
    build) applies inside the block only, and nests."""
    D = _binding.debug_lib()
    assert _binding.lib() is L
    with _binding.using_library(D):
        assert _binding.lib() is D
        with _binding.using_library(L):
            assert _binding.lib() is L
        assert _binding.lib() is D
    assert _binding.lib() is L
    try:
        with _binding.using_library(D):
            raise KeyError("inside")
    except KeyError:
        pass
    assert _binding.lib() is L


def _strip_comments(src):
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    return re.sub(r"//[^\n]*", " ", src)


def _function_body(src, signature):
    """The text between the braces of the function whose definition starts with
    `signature` (brace matching on comment-free source)."""
    start = src.index(signature)
    i = src.index("{", start)
    depth = 0
    for j in range(i, len(src)):
        depth += {"{": 1, "}": -1}.get(src[j], 0)
        if depth == 0:
            return src[i:j + 1]
    raise AssertionError("unbalanced braces after " + signature)


ALLOCATING = re.compile(r"\b(cudaMalloc\w*|cudaHostAlloc|cudaMemPool\w*|cuMem\w*|get_buffer|get_workspace|"
                        r"ffn_forward_impl|malloc|calloc|realloc)\b|\bnew\s+[\w:]")


def test_noalloc_entry_point_names_no_allocator():
    """spark_ffn_forward_noalloc's defining property, checked on its source: its
    translation unit and the fused launcher it calls name no device, host or pool
    allocator and do not reach the workspace pool that the other entry points grow."""
    csrc = os.path.join(ROOT, "activation_sparse_transformer_predictor_b200", "csrc")
    noalloc = _strip_comments(open(os.path.join(csrc, "spark_noalloc.cu")).read())
    assert "launch_fused(" in noalloc
    assert not ALLOCATING.search(noalloc), ALLOCATING.search(noalloc).group(0)
    fused = _strip_comments(open(os.path.join(csrc, "ffn_fused.cu")).read())
    api = _strip_comments(open(os.path.join(csrc, "spark_api.cu")).read())
    body = _function_body(fused, "cudaError_t launch_fused(const FusedPlan&")
    assert "cudaLaunchKernelEx" in body
    # the host helpers it calls: the launch plan, k's quantile, the wait limit
    for name in ("plan_fused", "spark_topk_quantile", "wait_limit_ns"):
        assert name + "(" in noalloc, name
    body += _function_body(fused, "FusedPlan plan_fused(")
    body += _function_body(api, "double spark_topk_quantile(int k, int d)")
    body += _function_body(api, "double upper_tail_quantile(")
    body += _function_body(api, "unsigned long long wait_limit_ns()")
    assert not ALLOCATING.search(body), ALLOCATING.search(body).group(0)
    # the pattern does catch what it is meant to catch
    for bad in ("cudaMallocAsync(&p, n, s)", "get_buffer(pool, dev, s, n, true, &p)", "auto* p = new float[4];"):
        assert ALLOCATING.search(bad), bad
