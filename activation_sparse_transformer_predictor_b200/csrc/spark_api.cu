// spark_api.cu -- the C ABI declared in include/spark.h: argument checks,
// per-(device, stream) workspaces, the host-side quantile Q(1 - k/d), and the
// dispatch onto the kernels.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "spark.h"
#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {
namespace {

constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;  // one second
unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;

// Speculative L2 prefetch margin of the fused small-batch kernel, in units of
// the local standard deviation below the threshold.
constexpr float kSpecMargin = 0.35f;

// Single-token decode: whether the score kernel may stream K1 before the work
// ahead of it on the stream has completed (spark_set_weight_overlap).
bool g_weight_overlap = false;


struct DeviceInfo {
  bool probed = false;
  bool is_sm100 = false;
  int num_sms = 0;
  size_t smem_optin = 0;
};

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};

std::mutex g_mutex;
std::map<int, DeviceInfo> g_devices;
std::map<std::pair<int, cudaStream_t>, Workspace> g_workspaces;
// device copies of q and out for spark_ffn_forward_host, per device and stream
std::map<std::pair<int, cudaStream_t>, Workspace> g_staging;

int current_device(int* dev) {
  return cudaGetDevice(dev) == cudaSuccess ? SPARK_OK : SPARK_ECUDA;
}

int device_info(int dev, DeviceInfo* out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& di = g_devices[dev];
  if (!di.probed) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SPARK_ECUDA;
    di.is_sm100 = prop.major == 10;
    di.num_sms = prop.multiProcessorCount;
    di.smem_optin = prop.sharedMemPerBlockOptin;
    di.probed = true;
  }
  *out = di;
  return di.is_sm100 ? SPARK_OK : SPARK_EDEVICE;
}

// Returns a buffer of `pool` of at least `bytes` for (dev, stream), allocated
// or regrown on `stream` (never inside a stream capture).  With `zero_control`
// a new buffer starts with a zeroed device control block.
int get_buffer(std::map<std::pair<int, cudaStream_t>, Workspace>& pool, int dev, cudaStream_t stream, size_t bytes,
               bool zero_control, void** ptr) {
  std::lock_guard<std::mutex> lock(g_mutex);
  Workspace& ws = pool[{dev, stream}];
  if (ws.bytes >= bytes && ws.ptr != nullptr) {
    *ptr = ws.ptr;
    return SPARK_OK;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return SPARK_ECUDA;
  if (cap != cudaStreamCaptureStatusNone) return SPARK_ENOMEM;  // no growth inside a capture
  if (ws.ptr != nullptr) {
    if (cudaFreeAsync(ws.ptr, stream) != cudaSuccess) return SPARK_ECUDA;
    ws.ptr = nullptr;
    ws.bytes = 0;
  }
  size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
  void* p = nullptr;
  if (cudaMallocAsync(&p, want, stream) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ENOMEM;
  }
  if (zero_control && cudaMemsetAsync(p, 0, sizeof(DeviceControl), stream) != cudaSuccess) return SPARK_ECUDA;
  ws.ptr = p;
  ws.bytes = want;
  *ptr = p;
  return SPARK_OK;
}

// The kernels' workspace for (dev, stream): control block first, then scratch.
int get_workspace(int dev, cudaStream_t stream, size_t bytes, void** ptr) {
  return get_buffer(g_workspaces, dev, stream, bytes, true, ptr);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The device-visible address of host memory p, if p lies in a pinned buffer
// that is mapped for device `dev` (cudaHostAlloc / cudaHostRegister with
// mapping, which unified addressing implies); else nullptr.
void* mapped_host_address(const void* p, int dev) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || at.device != dev) return nullptr;
  return at.devicePointer;
}

bool overlaps(const void* a, size_t abytes, const void* b, size_t bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bbytes && b0 < a0 + abytes;
}

// Standard-normal upper-tail quantile: z with P(Z > z) = p.  First guess from
// the rational approximation of Abramowitz & Stegun, Handbook of Mathematical
// Functions, eq. 26.2.23 (|error| < 4.5e-4), then Newton steps on the C
// library's erfc: z <- z + (U(z) - p) / phi(z), U(z) = erfc(z / sqrt 2) / 2.
double upper_tail_quantile(double p) {
  if (!(p > 0.0) || !(p < 1.0)) return NAN;
  const bool upper = p <= 0.5;
  const double pp = upper ? p : 1.0 - p;
  const double t = std::sqrt(-2.0 * std::log(pp));
  double z = t - (2.515517 + 0.802853 * t + 0.010328 * t * t) /
                     (1.0 + 1.432788 * t + 0.189269 * t * t + 0.001308 * t * t * t);
  if (!upper) z = -z;
  const double inv_sqrt2 = 0.70710678118654752440;
  const double inv_sqrt2pi = 0.39894228040143267794;
  for (int it = 0; it < 6; ++it) {
    const double u = 0.5 * std::erfc(z * inv_sqrt2);
    const double phi = inv_sqrt2pi * std::exp(-0.5 * z * z);
    if (!(phi > 0.0)) break;
    const double step = (u - p) / phi;
    z += step;
    if (std::fabs(step) < 1e-16 * (1.0 + std::fabs(z))) break;
  }
  return z;
}

int check_ffn_args(const void* q, const void* K1, const void* K2, const void* V, int T, int d_model, int r,
                   int d_ff, int k, const void* out) {
  if (!q || !K1 || !K2 || !V || !out) return SPARK_EINVAL;
  if (T < 1 || d_model < 2 || !(r > 0 && r < d_model) || !(k > 0 && k < d_ff)) return SPARK_EINVAL;
  if (r % 8 != 0 || d_model % 8 != 0) return SPARK_EALIGN;
  if (!aligned16(q) || !aligned16(K1) || !aligned16(K2) || !aligned16(V) || !aligned16(out)) return SPARK_EALIGN;
  const size_t ob = static_cast<size_t>(T) * d_model * 2;
  if (overlaps(out, ob, q, ob) || overlaps(out, ob, K1, static_cast<size_t>(d_ff) * r * 2) ||
      overlaps(out, ob, K2, static_cast<size_t>(d_ff) * (d_model - r) * 2) ||
      overlaps(out, ob, V, static_cast<size_t>(d_ff) * d_model * 2))
    return SPARK_EINVAL;
  return SPARK_OK;
}

// q_fetch (single-token decode only): a device-visible address of q in mapped
// host memory, copied to q (a device buffer) by the first kernel of the call.
int ffn_forward_impl(const void* q, const void* K1, const void* K2, const void* V, int T, int d_model, int r,
                     int d_ff, int k, void* out, float* x_out, float* theta_out, unsigned char* active_out,
                     cudaStream_t stream, int never_arrive, const void* q_fetch = nullptr) {
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  const double Qd = upper_tail_quantile(static_cast<double>(k) / static_cast<double>(d_ff));
  const float Q = static_cast<float>(Qd);

  if (T >= kPrefillMinTokens && d_ff % 16 == 0) {
    void* ws = nullptr;
    const int wst = get_workspace(dev, stream, prefill_workspace_bytes(T, d_model, d_ff, di.num_sms), &ws);
    if (wst != SPARK_OK) return wst;
    PrefillArgs a;
    a.q = q;
    a.K1 = K1;
    a.K2 = K2;
    a.V = V;
    a.out = out;
    a.T = T;
    a.d_model = d_model;
    a.r = r;
    a.d_ff = d_ff;
    a.Q = Q;
    a.x_out = x_out;
    a.theta_out = theta_out;
    a.active_out = active_out;
    a.workspace = ws;
    a.wait_limit_ns = g_wait_limit_ns;
    if (launch_prefill(a, di.num_sms, stream) != cudaSuccess) {
      cudaGetLastError();
      return SPARK_ECUDA;
    }
    return SPARK_OK;
  }

  if (T == 1 && never_arrive == 0) {
    const DecodePgPlan pp = plan_decode_pg(d_model, r, d_ff, di.num_sms, di.smem_optin);
    if (pp.ok) {
      void* ws = nullptr;
      const int wst = get_workspace(dev, stream, pp.ws_bytes, &ws);
      if (wst != SPARK_OK) return wst;
      DecodePgArgs a;
      a.q = q;
      a.q_fetch = q_fetch;
      a.K1 = K1;
      a.K2 = K2;
      a.V = V;
      a.out = out;
      a.d_model = d_model;
      a.r = r;
      a.d_ff = d_ff;
      a.Q = Q;
      a.x_out = x_out;
      a.theta_out = theta_out;
      a.active_out = active_out;
      a.workspace = ws;
      a.wait_limit_ns = g_wait_limit_ns;
      a.overlap_weights = g_weight_overlap;
      if (launch_decode_pg(pp, a, stream) != cudaSuccess) {
        cudaGetLastError();
        return SPARK_ECUDA;
      }
      return SPARK_OK;
    }
  }

  // The fused kernel takes up to kFusedMaxTokens tokens per launch; fall back
  // to fewer tokens per launch when shared memory does not fit more.
  int group = T < kFusedMaxTokens ? T : kFusedMaxTokens;
  FusedPlan plan = plan_fused(group, d_model, r, d_ff, di.num_sms, di.smem_optin);
  while (!plan.ok && group > 1) {
    group = (group + 1) / 2;
    plan = plan_fused(group, d_model, r, d_ff, di.num_sms, di.smem_optin);
  }
  if (!plan.ok) return SPARK_EINVAL;  // shape not supported by this build
  void* ws = nullptr;
  const int wst = get_workspace(dev, stream, plan.ws_bytes, &ws);
  if (wst != SPARK_OK) return wst;
  const unsigned char* qb = static_cast<const unsigned char*>(q);
  unsigned char* ob = static_cast<unsigned char*>(out);
  for (int t0 = 0; t0 < T; t0 += group) {
    const int g = T - t0 < group ? T - t0 : group;
    FusedPlan pl = plan;
    if (g != group) pl = plan_fused(g, d_model, r, d_ff, di.num_sms, di.smem_optin);
    FusedArgs a;
    a.q = qb + static_cast<size_t>(t0) * d_model * 2;
    a.K1 = K1;
    a.K2 = K2;
    a.V = V;
    a.out = ob + static_cast<size_t>(t0) * d_model * 2;
    a.T = g;
    a.d_model = d_model;
    a.r = r;
    a.d_ff = d_ff;
    a.Q = Q;
    a.spec_margin = kSpecMargin;
    a.x_out = x_out ? x_out + static_cast<size_t>(t0) * d_ff : nullptr;
    a.theta_out = theta_out ? theta_out + t0 : nullptr;
    a.active_out = active_out ? active_out + static_cast<size_t>(t0) * d_ff : nullptr;
    a.workspace = ws;
    a.wait_limit_ns = g_wait_limit_ns;
    a.never_arrive = never_arrive;
    if (launch_fused(pl, a, stream) != cudaSuccess) {
      cudaGetLastError();
      return SPARK_ECUDA;
    }
  }
  return SPARK_OK;
}

}  // namespace

unsigned long long wait_limit_ns() { return g_wait_limit_ns; }

}  // namespace spark

using namespace spark;

extern "C" {

SPARK_API int spark_ffn_forward(const void* q, const void* K1, const void* K2, const void* V, int d_model, int r,
                                int d_ff, int k, void* out, spark_stream_t stream) {
  return spark_ffn_forward_tokens(q, K1, K2, V, 1, d_model, r, d_ff, k, out, stream);
}

SPARK_API int spark_ffn_forward_tokens(const void* q, const void* K1, const void* K2, const void* V, int n_tokens,
                                       int d_model, int r, int d_ff, int k, void* out, spark_stream_t stream) {
  return spark_ffn_forward_debug(q, K1, K2, V, n_tokens, d_model, r, d_ff, k, out, nullptr, nullptr, nullptr,
                                 stream);
}

SPARK_API int spark_ffn_forward_debug(const void* q, const void* K1, const void* K2, const void* V, int n_tokens,
                                      int d_model, int r, int d_ff, int k, void* out, float* x_out,
                                      float* theta_out, unsigned char* active_out, spark_stream_t stream) {
  if (n_tokens == 0) return SPARK_OK;
  const int st = check_ffn_args(q, K1, K2, V, n_tokens, d_model, r, d_ff, k, out);
  if (st != SPARK_OK) return st;
  if (x_out != nullptr && !aligned16(x_out)) return SPARK_EALIGN;
  return ffn_forward_impl(q, K1, K2, V, n_tokens, d_model, r, d_ff, k, out, x_out, theta_out, active_out,
                          reinterpret_cast<cudaStream_t>(stream), 0);
}

SPARK_API int spark_ffn_forward_host(const void* q_host, const void* K1, const void* K2, const void* V,
                                     int n_tokens, int d_model, int r, int d_ff, int k, void* out_host,
                                     spark_stream_t stream_) {
  if (n_tokens == 0) return SPARK_OK;
  // every check spark_ffn_forward_tokens makes, before anything is enqueued
  if (!q_host || !out_host || !K1 || !K2 || !V) return SPARK_EINVAL;
  if (n_tokens < 1 || d_model < 2 || !(r > 0 && r < d_model) || !(k > 0 && k < d_ff)) return SPARK_EINVAL;
  if (r % 8 != 0 || d_model % 8 != 0) return SPARK_EALIGN;
  if (!aligned16(K1) || !aligned16(K2) || !aligned16(V)) return SPARK_EALIGN;
  const size_t bytes = static_cast<size_t>(n_tokens) * d_model * 2;
  if (overlaps(q_host, bytes, out_host, bytes)) return SPARK_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int dst = device_info(dev, &di);
  if (dst != SPARK_OK) return dst;
  const size_t half = (bytes + 255) / 256 * 256;
  void* st = nullptr;
  const int wst = get_buffer(g_staging, dev, stream, 2 * half, false, &st);
  if (wst != SPARK_OK) return wst;
  void* qd = st;
  void* od = static_cast<unsigned char*>(st) + half;
  if (n_tokens == 1 && plan_decode_pg(d_model, r, d_ff, di.num_sms, di.smem_optin).ok) {
    // single-token decode from mapped pinned buffers: the first kernel reads q
    // from host memory and the last one stores out into it (no copy-engine
    // transfers between calls)
    void* qm = aligned16(q_host) ? mapped_host_address(q_host, dev) : nullptr;
    void* om = qm != nullptr ? mapped_host_address(out_host, dev) : nullptr;
    if (qm != nullptr && om != nullptr)
      return ffn_forward_impl(qd, K1, K2, V, 1, d_model, r, d_ff, k, om, nullptr, nullptr, nullptr, stream, 0, qm);
  }
  if (cudaMemcpyAsync(qd, q_host, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  const int rc = spark_ffn_forward_tokens(qd, K1, K2, V, n_tokens, d_model, r, d_ff, k, od, stream_);
  if (rc != SPARK_OK) return rc;
  if (cudaMemcpyAsync(out_host, od, bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

SPARK_API int spark_ffn_predictor(const void* q, const void* K1, int n_tokens, int d_model, int r, int d_ff,
                                  float* x_out, spark_stream_t stream_) {
  if (n_tokens == 0) return SPARK_OK;
  if (!q || !K1 || !x_out || n_tokens < 0 || d_model < 2 || !(r > 0 && r < d_model) || d_ff < 16)
    return SPARK_EINVAL;
  if (r % 8 != 0 || d_model % 8 != 0 || d_ff % 16 != 0) return SPARK_EALIGN;
  if (!aligned16(q) || !aligned16(K1) || !aligned16(x_out)) return SPARK_EALIGN;
  const size_t xb = static_cast<size_t>(n_tokens) * d_ff * 4;
  if (overlaps(x_out, xb, q, static_cast<size_t>(n_tokens) * d_model * 2) ||
      overlaps(x_out, xb, K1, static_cast<size_t>(d_ff) * r * 2))
    return SPARK_EINVAL;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  void* ws = nullptr;
  const int wst = get_workspace(dev, stream, predictor_workspace_bytes(n_tokens, d_ff), &ws);
  if (wst != SPARK_OK) return wst;
  if (launch_predictor(q, K1, n_tokens, d_model, r, d_ff, x_out, ws, g_wait_limit_ns, di.num_sms, stream) !=
      cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

SPARK_API int spark_ffn_decode_stack(const float* h_in, float* h_out, const void* const* K1s, const void* const* K2s,
                                     const void* const* Vs, int n_layers, int d_model, int r, int d_ff, int k,
                                     float eps, void* q_dbg, void* out_dbg, spark_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!h_in || !h_out || n_layers < 0 || !(eps >= 0.f)) return SPARK_EINVAL;
  if (n_layers > 0 && (!K1s || !K2s || !Vs)) return SPARK_EINVAL;
  if ((reinterpret_cast<uintptr_t>(h_in) | reinterpret_cast<uintptr_t>(h_out)) & 15u) return SPARK_EALIGN;
  const size_t hb = static_cast<size_t>(d_model) * 4;
  if (h_in != h_out && overlaps(h_in, hb, h_out, hb)) return SPARK_EINVAL;
  if (n_layers == 0) {
    if (h_in != h_out && cudaMemcpyAsync(h_out, h_in, hb, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
      return SPARK_ECUDA;
    return SPARK_OK;
  }
  for (int l = 0; l < n_layers; ++l) {
    // q_l lives in the kernel's shared memory; q_dbg stands in for q in the checks
    const int st = check_ffn_args(K1s[l], K1s[l], K2s[l], Vs[l], 1, d_model, r, d_ff, k,
                                  out_dbg ? static_cast<unsigned char*>(out_dbg) + static_cast<size_t>(l) * d_model * 2
                                          : reinterpret_cast<void*>(static_cast<uintptr_t>(16)));
    if (st != SPARK_OK) return st;
  }
  if ((q_dbg && !aligned16(q_dbg)) || (out_dbg && !aligned16(out_dbg))) return SPARK_EALIGN;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int dst = device_info(dev, &di);
  if (dst != SPARK_OK) return dst;
  const float Q = static_cast<float>(upper_tail_quantile(static_cast<double>(k) / static_cast<double>(d_ff)));
  const DecodePgPlan pp = plan_decode_pg(d_model, r, d_ff, di.num_sms, di.smem_optin);
  if (!pp.ok) return SPARK_EINVAL;  // shape not supported by the single-token kernels
  void* ws = nullptr;
  const int wst = get_workspace(dev, stream, pp.ws_bytes, &ws);
  if (wst != SPARK_OK) return wst;
  // every layer's score kernel forms q_l = bf16(RMSNorm(h_l)); its reduce
  // kernel writes h_{l+1} = h_l + bf16(out_l)
  for (int l = 0; l < n_layers; ++l) {
    DecodePgArgs a;
    a.K1 = K1s[l];
    a.K2 = K2s[l];
    a.V = Vs[l];
    a.out = out_dbg ? static_cast<unsigned char*>(out_dbg) + static_cast<size_t>(l) * d_model * 2 : nullptr;
    a.d_model = d_model;
    a.r = r;
    a.d_ff = d_ff;
    a.Q = Q;
    a.q_dbg = q_dbg ? static_cast<unsigned char*>(q_dbg) + static_cast<size_t>(l) * d_model * 2 : nullptr;
    a.workspace = ws;
    a.wait_limit_ns = g_wait_limit_ns;
    // after the first layer, the kernel ahead of each score kernel is this
    // library's own reduce kernel, which writes no weights
    a.overlap_weights = l > 0 || g_weight_overlap;
    a.h_in = l == 0 ? h_in : h_out;
    a.h_base = a.h_in;
    a.h_out = h_out;
    a.eps = eps;
    if (launch_decode_pg(pp, a, stream) != cudaSuccess) {
      cudaGetLastError();
      return SPARK_ECUDA;
    }
  }
  return SPARK_OK;
}

SPARK_API int spark_attention_decode_debug(const void* q, const void* K, const void* V, int n_heads, int n_kv_heads,
                                          int n_ctx, int d_head, int r, int k_attn, float scale, void* out,
                                          float* s_out, float* theta_out, unsigned char* active_out,
                                          spark_stream_t stream) {
  if (!q || !K || !V || !out) return SPARK_EINVAL;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0 || n_ctx < 1 || n_ctx > 65536 || k_attn < 1)
    return SPARK_EINVAL;
  if (!(r > 0 && r < d_head) || d_head > kAttnMaxDHead) return SPARK_EINVAL;
  if (!(scale > 0.f) || !std::isfinite(scale)) return SPARK_EINVAL;
  if (r % 8 != 0 || d_head % 8 != 0) return SPARK_EALIGN;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return SPARK_EALIGN;
  const size_t ob = static_cast<size_t>(n_heads) * d_head * 2;
  const size_t kvb = static_cast<size_t>(n_kv_heads) * n_ctx * d_head * 2;
  if (overlaps(out, ob, q, ob) || overlaps(out, ob, K, kvb) || overlaps(out, ob, V, kvb)) return SPARK_EINVAL;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  AttnArgs a;
  a.q = q;
  a.K = K;
  a.V = V;
  a.out = out;
  a.n_heads = n_heads;
  a.n_kv_heads = n_kv_heads;
  a.n_ctx = n_ctx;
  a.d_head = d_head;
  a.r = r;
  a.scale = scale;
  a.select_all = k_attn >= n_ctx;
  a.Q = a.select_all ? 0.f
                     : static_cast<float>(upper_tail_quantile(static_cast<double>(k_attn) / static_cast<double>(n_ctx)));
  a.s_out = s_out;
  a.theta_out = theta_out;
  a.active_out = active_out;
  if (launch_attn_decode(a, di.num_sms, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

SPARK_API int spark_attention_decode(const void* q, const void* K, const void* V, int n_heads, int n_kv_heads,
                                    int n_ctx, int d_head, int r, int k_attn, float scale, void* out,
                                    spark_stream_t stream) {
  return spark_attention_decode_debug(q, K, V, n_heads, n_kv_heads, n_ctx, d_head, r, k_attn, scale, out, nullptr,
                                      nullptr, nullptr, stream);
}

SPARK_API int stat_topk_soft_threshold(const float* x, int rows, int d, int k, float* out, spark_stream_t stream) {
  if (rows == 0) return SPARK_OK;
  if (!x || !out || rows < 0 || d < 2 || !(k > 0 && k < d)) return SPARK_EINVAL;
  const size_t bytes = static_cast<size_t>(rows) * d * sizeof(float);
  if (x != out && overlaps(x, bytes, out, bytes)) return SPARK_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 3u) return SPARK_EALIGN;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  const float Q = static_cast<float>(upper_tail_quantile(static_cast<double>(k) / static_cast<double>(d)));
  if (launch_stat_topk(x, out, rows, d, Q, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

SPARK_API int stat_topk_huber(const float* x, int rows, int d, int k, float delta, float* out, spark_stream_t stream) {
  if (rows == 0) return SPARK_OK;
  if (!x || !out || rows < 0 || d < 2 || !(k > 0 && k < d) || !(delta >= 0.f) || !std::isfinite(delta))
    return SPARK_EINVAL;
  const size_t bytes = static_cast<size_t>(rows) * d * sizeof(float);
  if (x != out && overlaps(x, bytes, out, bytes)) return SPARK_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 3u) return SPARK_EALIGN;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  const float Q = static_cast<float>(upper_tail_quantile(static_cast<double>(k) / static_cast<double>(d)));
  if (launch_stat_topk_huber(x, out, rows, d, Q, delta, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

SPARK_API int stat_topk_huber_backward(const float* x, const float* grad_out, int rows, int d, int k, float delta,
                                       float* grad_x, spark_stream_t stream) {
  if (rows == 0) return SPARK_OK;
  if (!x || !grad_out || !grad_x || rows < 0 || d < 2 || !(k > 0 && k < d) || !(delta >= 0.f) ||
      !std::isfinite(delta))
    return SPARK_EINVAL;
  const size_t bytes = static_cast<size_t>(rows) * d * sizeof(float);
  // grad_x may be x or grad_out itself (in place); any other overlap is refused
  if ((grad_x != x && overlaps(grad_x, bytes, x, bytes)) ||
      (grad_x != grad_out && overlaps(grad_x, bytes, grad_out, bytes)))
    return SPARK_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(grad_out) | reinterpret_cast<uintptr_t>(grad_x)) &
      3u)
    return SPARK_EALIGN;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  const float Q = static_cast<float>(upper_tail_quantile(static_cast<double>(k) / static_cast<double>(d)));
  if (launch_stat_topk_huber_backward(x, grad_out, grad_x, rows, d, Q, delta,
                                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

SPARK_API int stat_topk_soft_threshold_causal(const float* x, int rows, int d, int k, int n_q, int offset,
                                              float* out, float* theta_out, spark_stream_t stream) {
  if (rows == 0) return SPARK_OK;
  if (!x || !out || rows < 0 || d < 1 || k < 1 || n_q < 1 || offset < 0) return SPARK_EINVAL;
  const size_t bytes = static_cast<size_t>(rows) * d * sizeof(float);
  if (x != out && overlaps(x, bytes, out, bytes)) return SPARK_EINVAL;
  if (theta_out != nullptr && (overlaps(theta_out, static_cast<size_t>(rows) * 4, x, bytes) ||
                               overlaps(theta_out, static_cast<size_t>(rows) * 4, out, bytes)))
    return SPARK_EINVAL;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(theta_out)) & 3u)
    return SPARK_EALIGN;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  if (launch_stat_topk_causal(x, out, rows, d, k, n_q, offset, theta_out, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}

// Failed index checks counted by the kernels of the current device (bounds-check
// build; 0 in release builds), cleared with `clear`; -1 if reading them failed.
static long long bounds_violations(bool clear) {
  const unsigned counts[4] = {take_bounds_violations_decode(clear), take_bounds_violations_fused(clear),
                              take_bounds_violations_prefill(clear), take_bounds_violations_attention(clear)};
  long long total = 0;
  for (unsigned c : counts) {
    if (c == 0xffffffffu) return -1;
    total += c;
  }
  return total;
}

static int with_bounds_status(int status) {
  if (status != SPARK_OK) return status;
  const long long v = bounds_violations(false);
  return v < 0 ? SPARK_ECUDA : v > 0 ? SPARK_EBOUNDS : SPARK_OK;
}

SPARK_API int spark_query_status(spark_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  // errors recorded by spark_ffn_forward_noalloc live in its own scratch
  const int na = noalloc_take_status(dev);
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    auto it = g_workspaces.find({dev, stream});
    if (it == g_workspaces.end() || it->second.ptr == nullptr) ptr = nullptr;
    else ptr = it->second.ptr;
  }
  if (ptr == nullptr) return with_bounds_status(na);
  DeviceControl ctl;
  if (cudaMemcpy(&ctl, ptr, sizeof ctl, cudaMemcpyDeviceToHost) != cudaSuccess) return SPARK_ECUDA;
  if (ctl.status == kDevOk && ctl.abort == 0) return with_bounds_status(na);
  if (cudaMemset(ptr, 0, sizeof ctl) != cudaSuccess) return SPARK_ECUDA;  // barrier state too
  return ctl.status == kDevTimeout ? SPARK_ETIMEOUT : SPARK_ECUDA;
}

SPARK_API int spark_release_workspace(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  int prev = 0;
  cudaGetDevice(&prev);
  int rc = SPARK_OK;
  for (auto* pool : {&g_workspaces, &g_staging}) {
    for (auto& kv : *pool) {
      if (kv.second.ptr == nullptr) continue;
      cudaSetDevice(kv.first.first);
      if (cudaDeviceSynchronize() != cudaSuccess || cudaFree(kv.second.ptr) != cudaSuccess) rc = SPARK_ECUDA;
    }
    pool->clear();
  }
  cudaSetDevice(prev);
  return rc;
}

SPARK_API const char* spark_status_string(int status) {
  switch (status) {
    case SPARK_OK: return "SPARK_OK";
    case SPARK_EINVAL: return "SPARK_EINVAL: invalid argument";
    case SPARK_EALIGN: return "SPARK_EALIGN: misaligned pointer or size";
    case SPARK_ECUDA: return "SPARK_ECUDA: CUDA error";
    case SPARK_ENOMEM: return "SPARK_ENOMEM: workspace allocation failed";
    case SPARK_ETIMEOUT: return "SPARK_ETIMEOUT: device wait timed out";
    case SPARK_EDEVICE: return "SPARK_EDEVICE: device is not sm_100";
    case SPARK_ESCRATCH: return "SPARK_ESCRATCH: problem exceeds the fixed no-allocation scratch";
    case SPARK_EBOUNDS: return "SPARK_EBOUNDS: a kernel index check failed (bounds-check build)";
    default: return "SPARK_UNKNOWN";
  }
}

SPARK_API double spark_topk_quantile(int k, int d) {
  if (!(k > 0 && k < d)) return NAN;
  return upper_tail_quantile(static_cast<double>(k) / static_cast<double>(d));
}

SPARK_API int spark_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns = ns == 0 ? kDefaultWaitLimitNs : ns;
  return SPARK_OK;
}

SPARK_API int spark_set_weight_overlap(int enable) {
  g_weight_overlap = enable != 0;
  return SPARK_OK;
}

SPARK_API int spark_selftest_wait_timeout(spark_stream_t stream) {
  // A tiny valid problem whose first grid barrier waits for one arrival more
  // than there are CTAs; every CTA records the time-out and returns.
  const int d_model = 64, r = 32, d_ff = 256, k = 20;
  int dev;
  if (current_device(&dev) != SPARK_OK) return SPARK_ECUDA;
  DeviceInfo di;
  const int st = device_info(dev, &di);
  if (st != SPARK_OK) return st;
  void* buf = nullptr;
  const size_t bytes = static_cast<size_t>(d_ff) * (r + (d_model - r) + d_model) * 2 + 2 * 2 * d_model + 1024;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMallocAsync(&buf, bytes, s) != cudaSuccess) return SPARK_ENOMEM;
  cudaMemsetAsync(buf, 0, bytes, s);
  unsigned char* b = static_cast<unsigned char*>(buf);
  const void* K1 = b;
  const void* K2 = b + static_cast<size_t>(d_ff) * r * 2;
  const void* V = b + static_cast<size_t>(d_ff) * d_model * 2;
  const void* q = b + static_cast<size_t>(d_ff) * 2 * d_model * 2;
  void* out = b + static_cast<size_t>(d_ff) * 2 * d_model * 2 + 256;
  const unsigned long long saved = g_wait_limit_ns;
  g_wait_limit_ns = 20000000ull;  // 20 ms
  const int rc = ffn_forward_impl(q, K1, K2, V, 1, d_model, r, d_ff, k, out, nullptr, nullptr, nullptr, s, 1);
  g_wait_limit_ns = saved;
  cudaFreeAsync(buf, s);
  return rc;
}

SPARK_API int spark_debug_violations(void) {
#ifdef SPARK_DEBUG
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  const long long total = bounds_violations(true);
  if (total < 0) return SPARK_ECUDA;
  return total > 0x7fffffffll ? 0x7fffffff : static_cast<int>(total);
#else
  return -1;
#endif
}

SPARK_API int spark_version(void) { return 100; }

}  // extern "C"
