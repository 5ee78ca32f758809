// spark_noalloc.cu -- decode entry point that never allocates device memory.
//
// Same kernel and arithmetic as spark_ffn_forward (one token).  Its scratch --
// the device control block, the per-CTA moments and the per-CTA partial
// outputs -- lives in a fixed buffer compiled into the library instead of the
// lazily allocated per-stream workspace, so a call performs no cudaMalloc,
// cudaMallocAsync, cudaFree or allocating library call.  Callers that need this
// are those for which allocating while they run is forbidden or unsafe: the
// execute/enqueue hook of an inference-engine plugin, a runtime that plans all
// device memory up front and treats any later allocation as a failure, or code
// running where a device allocation could block on or interfere with another
// allocator.
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "spark.h"
#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {
namespace {

// The scratch buffer.  Every GPU that loads the library holds it until the
// process exits.  Host code must not use this name as a device address: the
// address comes from cudaGetSymbolAddress (below), once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SPARK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on `dev` (which must be current),
// looked up on the first call for that device and cached.
int scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (dev < 0 || dev >= kMaxDevices) return SPARK_EINVAL;
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SPARK_ECUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SPARK_OK;
}

// Device address of the scratch on `dev` if it was already looked up, else nullptr.
void* scratch_address_if_set(int dev) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  return (dev >= 0 && dev < kMaxDevices) ? g_scratch_addr[dev] : nullptr;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ranges_overlap(const void* a, size_t abytes, const void* b, size_t bbytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bbytes && b0 < a0 + abytes;
}

}  // namespace

int noalloc_take_status(int dev) {
  void* scratch = scratch_address_if_set(dev);
  if (scratch == nullptr) return SPARK_OK;
  DeviceControl ctl;
  if (cudaMemcpy(&ctl, scratch, sizeof ctl, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  if (ctl.status == kDevOk && ctl.abort == 0) return SPARK_OK;
  if (cudaMemset(scratch, 0, sizeof ctl) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return ctl.status == kDevTimeout ? SPARK_ETIMEOUT : SPARK_ECUDA;
}

}  // namespace spark

extern "C" SPARK_API int spark_ffn_forward_noalloc(const void* q, const void* K1, const void* K2, const void* V,
                                                   int d_model, int r, int d_ff, int k, void* out,
                                                   spark_stream_t stream_) {
  using namespace spark;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!q || !K1 || !K2 || !V || !out) return SPARK_EINVAL;
  if (d_model < 2 || !(r > 0 && r < d_model) || !(k > 0 && k < d_ff)) return SPARK_EINVAL;
  if (r % 8 != 0 || d_model % 8 != 0) return SPARK_EALIGN;
  if (!is_aligned16(q) || !is_aligned16(K1) || !is_aligned16(K2) || !is_aligned16(V) || !is_aligned16(out))
    return SPARK_EALIGN;
  const size_t ob = static_cast<size_t>(d_model) * 2;
  if (ranges_overlap(out, ob, q, ob) || ranges_overlap(out, ob, K1, static_cast<size_t>(d_ff) * r * 2) ||
      ranges_overlap(out, ob, K2, static_cast<size_t>(d_ff) * (d_model - r) * 2) ||
      ranges_overlap(out, ob, V, static_cast<size_t>(d_ff) * d_model * 2))
    return SPARK_EINVAL;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPARK_ECUDA;
  int major = 0, sms = 0, smem_optin = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return SPARK_ECUDA;
  if (major != 10) return SPARK_EDEVICE;

  const FusedPlan plan = plan_fused(1, d_model, r, d_ff, sms, static_cast<size_t>(smem_optin));
  if (!plan.ok) return SPARK_EINVAL;
  if (plan.ws_bytes > SPARK_NOALLOC_SCRATCH_BYTES) return SPARK_ESCRATCH;

  void* scratch = nullptr;
  const int st = scratch_address(dev, &scratch);
  if (st != SPARK_OK) return st;
  // The arrival counters and the published threshold must start at zero (the
  // last CTA of a completed launch resets them, but a launch that gave up
  // waiting leaves them set); the rest of the scratch is fully written before
  // it is read.  The first three words -- the recorded error, the abort flag
  // and where the wait gave up -- are kept, so that a time-out stays visible to
  // spark_query_status and later calls return at once until it is read.
  constexpr size_t kKeep = offsetof(DeviceControl, exit_count);
  if (cudaMemsetAsync(static_cast<unsigned char*>(scratch) + kKeep, 0, sizeof(DeviceControl) - kKeep, stream) !=
      cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  FusedArgs a;
  a.q = q;
  a.K1 = K1;
  a.K2 = K2;
  a.V = V;
  a.out = out;
  a.T = 1;
  a.d_model = d_model;
  a.r = r;
  a.d_ff = d_ff;
  a.Q = static_cast<float>(spark_topk_quantile(k, d_ff));
  a.spec_margin = 0.35f;
  a.x_out = nullptr;
  a.theta_out = nullptr;
  a.active_out = nullptr;
  a.workspace = scratch;
  a.wait_limit_ns = wait_limit_ns();
  a.never_arrive = 0;
  if (launch_fused(plan, a, stream) != cudaSuccess) {
    cudaGetLastError();
    return SPARK_ECUDA;
  }
  return SPARK_OK;
}
