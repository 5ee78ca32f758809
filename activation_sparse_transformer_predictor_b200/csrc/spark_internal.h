// spark_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace spark {

struct DeviceControl;

// ---------------------------------------------------------------- library settings
// Time limit of every device-side wait (spark_set_wait_limit_ns).
unsigned long long wait_limit_ns();

// The no-allocation entry point's fixed scratch on device `dev` (current):
// if a device error is recorded in its control block, clear the block and
// return that error (SPARK_ETIMEOUT); SPARK_OK if none, or if the entry point
// was never set up on `dev`.
int noalloc_take_status(int dev);

// ---------------------------------------------------------------- debug builds
// Failed index checks counted by each file's kernels (bounds-check build) since
// the last clearing read; 0xffffffff if the read failed; 0 without a CUDA call
// in release builds.
unsigned take_bounds_violations_decode(bool clear);
unsigned take_bounds_violations_fused(bool clear);
unsigned take_bounds_violations_prefill(bool clear);
unsigned take_bounds_violations_attention(bool clear);

// ---------------------------------------------------------------- stat top-k
cudaError_t launch_stat_topk(const float* x, float* out, int rows, int d, float Q, cudaStream_t stream);
cudaError_t launch_stat_topk_huber(const float* x, float* out, int rows, int d, float Q, float delta,
                                   cudaStream_t stream);
cudaError_t launch_stat_topk_huber_backward(const float* x, const float* g, float* gx, int rows, int d, float Q,
                                            float delta, cudaStream_t stream);
cudaError_t launch_stat_topk_causal(const float* x, float* out, int rows, int d, int k, int n_q, int offset,
                                    float* theta_out, cudaStream_t stream);

// ---------------------------------------------------------------- fused decode / small-batch FFN
constexpr int kFusedMaxTokens = 4;     // tokens per launch of the fused kernel
constexpr int kFusedMaxChunks = 8;     // 16-byte chunks per lane: r and d_model - r <= 2048
constexpr int kFusedMaxRowsPerCta = 256;

struct FusedPlan {
  int grid;          // CTAs (all co-resident; cooperative launch)
  int rows_per_cta;  // neurons owned by each CTA (multiple of 8)
  int col_width;     // output columns per CTA in the value phase (power of two, >= 8)
  int n_col_ctas;    // CTAs that own output columns
  size_t smem_bytes; // dynamic shared memory per CTA
  size_t ws_bytes;   // workspace bytes (device control block included)
  bool ok;           // false: shape does not fit the fused kernel
};

FusedPlan plan_fused(int n_tokens, int d_model, int r, int d_ff, int num_sms, size_t smem_optin);

struct FusedArgs {
  const void* q;
  const void* K1;
  const void* K2;
  const void* V;
  void* out;
  int T, d_model, r, d_ff;
  float Q;
  float spec_margin;         // > 0: speculative L2 prefetch of likely-active K2/V rows
  float* x_out;
  float* theta_out;
  unsigned char* active_out;
  void* workspace;           // FusedPlan::ws_bytes, device control block first
  unsigned long long wait_limit_ns;
  int never_arrive;          // self-test: barrier 1 can never complete
  // single-token stack mode (decode kernel only): q = bf16(RMSNorm(h_in)),
  // h_out = h_in + bf16(out); nullptr h_in = plain mode
  const float* h_in = nullptr;
  float* h_out = nullptr;
  float eps = 0.f;
  void* q_dbg = nullptr;
};

cudaError_t launch_fused(const FusedPlan& plan, const FusedArgs& args, cudaStream_t stream);

// ---------------------------------------------------------------- single-token decode: score + gather kernels
struct DecodePgPlan {
  int n_slices;           // score- and gather-kernel CTAs; slice c = neurons [c*rows_per_cta, ...)
  int rows_per_cta;       // multiple of 8
  int chunks_per_thread;  // 16-byte output chunks per gather thread (1, 2 or 4)
  int lane_chunks;        // 16-byte chunks per lane of a K1 / K2 row (5 or 8)
  int n_rctas;            // reduce-kernel CTAs (16 output columns each)
  size_t smem_p, smem_g, ws_bytes;
  bool ok;
};

DecodePgPlan plan_decode_pg(int d_model, int r, int d_ff, int num_sms, size_t smem_optin);

struct DecodePgArgs {
  const void* q = nullptr;      // bf16 [d_model] (ignored when h_in is set)
  // Device-visible address of q in mapped host memory, or nullptr: a one-CTA
  // kernel first copies it to q (then a device buffer the call may write).
  const void* q_fetch = nullptr;
  const float* h_in = nullptr;  // stack mode: q = bf16(RMSNorm(h_in)), formed by the score kernel
  const void* K1 = nullptr;
  const void* K2 = nullptr;
  const void* V = nullptr;
  void* out = nullptr;          // bf16 [d_model] (device memory or a device-visible address of mapped
                                // host memory); may be nullptr in stack mode
  int d_model = 0, r = 0, d_ff = 0;
  float Q = 0.f;
  float eps = 0.f;
  float* x_out = nullptr;
  float* theta_out = nullptr;
  unsigned char* active_out = nullptr;
  void* q_dbg = nullptr;        // bf16 [d_model]: copy of the q used
  void* workspace = nullptr;
  unsigned long long wait_limit_ns = 0;
  // Launch the score kernel programmatically behind the preceding kernel on the
  // stream: it then reads K1 before that kernel has completed.
  bool overlap_weights = false;
  // stack mode, reduce kernel: h_out = h_base + bf16(out) (h_out may equal h_base)
  const float* h_base = nullptr;
  float* h_out = nullptr;
};

cudaError_t launch_decode_pg(const DecodePgPlan& plan, const DecodePgArgs& args, cudaStream_t stream);

// ---------------------------------------------------------------- Spark Attention, one decoding position
constexpr int kAttnMaxDHead = 256;
constexpr int kAttnMaxKeysPerCta = 2048;

struct AttnArgs {
  const void* q = nullptr;  // bf16 [n_heads][d_head]
  const void* K = nullptr;  // bf16 [n_kv_heads][n_ctx][d_head]
  const void* V = nullptr;  // bf16 [n_kv_heads][n_ctx][d_head]
  void* out = nullptr;      // bf16 [n_heads][d_head]
  int n_heads = 0, n_kv_heads = 0, n_ctx = 0, d_head = 0, r = 0;
  float scale = 1.f, Q = 0.f;
  bool select_all = false;  // k_attn >= n_ctx
  float* s_out = nullptr;
  float* theta_out = nullptr;
  unsigned char* active_out = nullptr;
};

cudaError_t launch_attn_decode(const AttnArgs& args, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- batched (prefill) FFN on tcgen05
constexpr int kPrefillMinTokens = kFusedMaxTokens + 1;  // smaller batches take the fused kernel

struct PrefillArgs {
  const void* q;
  const void* K1;
  const void* K2;
  const void* V;
  void* out;
  int T, d_model, r, d_ff;
  float Q;
  float* x_out;              // optional copy of the predictor scores
  float* theta_out;
  unsigned char* active_out;
  void* workspace;           // prefill_workspace_bytes(), device control block first
  unsigned long long wait_limit_ns;
};

int prefill_splitk(int T, int d_model, int d_ff, int num_sms);
size_t predictor_workspace_bytes(int T, int d_ff);
cudaError_t launch_predictor(const void* q, const void* K1, int T, int d_model, int r, int d_ff, float* x_out,
                             void* workspace, unsigned long long wait_limit_ns, int num_sms, cudaStream_t stream);
size_t prefill_workspace_bytes(int T, int d_model, int d_ff, int num_sms);
cudaError_t launch_prefill(const PrefillArgs& args, int num_sms, cudaStream_t stream);

}  // namespace spark
