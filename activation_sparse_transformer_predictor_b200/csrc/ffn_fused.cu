// ffn_fused.cu -- Spark FFN forward for a few tokens (decode) in ONE kernel.
//
// Spark Transformer notes, 关键设计 / "Spark FFN":
//   x = K1^T q[:r];  theta = mean(x) + std(x) Q(1 - k/d_ff)  ("Statistical Top-k");
//   out = V . (GELU(max(x - theta, 0)) (.) (K2^T q[r:])), evaluated only on the
//   neurons with x > theta.
//
// Decode is bound by HBM bytes (all of K1, plus the active rows of K2 and V) and
// by the latency of the one global dependency (theta needs every score).  The
// kernel is a cooperative launch of one CTA per SM, all co-resident:
//
//  phase 1  CTA c owns neurons [c*RPC, (c+1)*RPC).  Thread 0 issues bulk
//           (TMA-engine) copies of the CTA's whole K1 slice into shared memory
//           at kernel start (8 rows per mbarrier), so all of K1 is in flight at
//           once.  Eight warps compute x for their rows (fp32 FMA, q[:r] in
//           registers) and the slice's per-token moments (count, mean, M2),
//           taken about the slice's first score.  While the other CTAs finish,
//           the CTA prefetches into L2 the K2 / V rows of neurons that its own
//           moments say are likely to pass the threshold (HBM is idle then).
//  stats    The last CTA to arrive (acquire-release counter) merges all
//           moments in a fixed order, derives theta and publishes it with one
//           release store; the others poll that word.  Every CTA therefore uses
//           the same bits of theta.
//  phase 2  Each CTA applies the soft threshold and GELU to its own neurons,
//           compacts the active ones, bulk-copies their whole K2 and V rows into
//           shared memory, computes h = g * <K2[i,:], q[r:]> and its partial
//           output sum_i h_i V[i,:] (fp32), and writes it to the workspace.
//  reduce   After a second counter, CTA c sums the partial outputs of its
//           output columns over all CTAs in a fixed order and writes bf16.
//
// No atomics touch data; the result is bit-reproducible run to run.
#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

#ifdef SPARK_DEBUG
// bounds-check violations of this file's kernels (see SPARK_CHECK)
static __device__ unsigned g_bounds_violations;
#endif


namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerStage = kWarps;  // one row per warp per stage
constexpr int kMaxColChunks = 2;       // 8-column chunks per thread in phase 2: d_model <= 4096

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared-memory carve-up; computed identically on host and device.
struct SmemLayout {
  size_t region_a;  // K1 slice (phase 1), then K2/V row batches (phase 2), then the reduce buffer
  size_t qs, xs, bars, theta, spec, uidx, ug, hs, wcnt, flags, total;
  int batch_rows;   // K2/V row pairs per phase-2 batch
  __host__ __device__ SmemLayout(int T, int d_model, int r, int rpc) {
    const int nst = rpc / kRowsPerStage;
    const size_t k1_bytes = static_cast<size_t>(nst) * kRowsPerStage * r * 2;
    const size_t row_bytes = static_cast<size_t>(d_model) * 2 * 2 - static_cast<size_t>(r) * 2;  // K2 + V row
    const size_t red_bytes = 16 * 1024;
    size_t a = k1_bytes;
    if (a < row_bytes) a = row_bytes;
    if (a < red_bytes) a = red_bytes;
    batch_rows = static_cast<int>(a / row_bytes);
    size_t off = 0;
    region_a = off;
    off += align_up(a, 128);
    qs = off;
    off += align_up(static_cast<size_t>(T) * d_model * 2, 128);
    xs = off;
    off += align_up(static_cast<size_t>(T) * rpc * 4, 16);
    bars = off;
    off += align_up(static_cast<size_t>(nst + 2) * 8, 16);
    theta = off;
    off += 16 * 4;
    spec = off;
    off += 16 * 4;
    uidx = off;
    off += align_up(static_cast<size_t>(rpc) * 4, 16);
    ug = off;
    off += align_up(static_cast<size_t>(rpc) * T * 4, 16);
    hs = off;
    off += align_up(static_cast<size_t>(rpc) * T * 4, 16);
    wcnt = off;
    off += align_up(static_cast<size_t>(kWarps + 1) * 4, 16);
    flags = off;
    off += 16;
    total = off;
  }
};

// Workspace carve-up (after the device control block).
struct WsLayout {
  size_t partials, pout, total;
  WsLayout(int T, int d_model, int grid) {
    size_t off = sizeof(DeviceControl);
    partials = off;
    off += align_up(static_cast<size_t>(T) * grid * sizeof(float2), 256);
    pout = off;
    off += align_up(static_cast<size_t>(grid) * T * d_model * 4, 256);
    total = off;
  }
};

struct KParams {
  const uint16_t* q;
  const uint16_t* K1;
  const uint16_t* K2;
  const uint16_t* V;
  uint16_t* out;
  int T, d_model, r, d2, d_ff, rpc, col_width, n_col_ctas;
  float Q;
  float spec_margin;  // > 0: prefetch rows with x > local mean + local std (Q - margin)
  float* x_out;
  float* theta_out;
  unsigned char* active_out;
  DeviceControl* ctl;
  float2* partials;  // [T][grid] (mean, M2) of each CTA's slice
  float* pout;       // [grid][T][d_model] partial outputs
  unsigned long long wait_limit_ns;
  int never_arrive;
};

__device__ __forceinline__ int rows_of_cta(int c, int rpc, int d_ff) {
  const int n0 = c * rpc;
  return max(0, min(rpc, d_ff - n0));
}

// x for token group [tg0, tg0 + TG) over this warp's rows (row = stage*8 + warp).
template <int TG>
__device__ __forceinline__ bool phase1_token_group(const KParams& p, const uint16_t* k1s, const uint16_t* qs,
                                                   float* xs, uint64_t* bars, int nr, int tg0) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nchunk = p.r / 8;
  uint4 qreg[TG][kFusedMaxChunks];
#pragma unroll
  for (int tt = 0; tt < TG; ++tt) {
#pragma unroll
    for (int m = 0; m < kFusedMaxChunks; ++m) {
      const int c = lane + 32 * m;
      if (c < nchunk && tg0 + tt < p.T)
        qreg[tt][m] = lds128(qs + static_cast<size_t>(tg0 + tt) * p.d_model + c * 8);
      else
        qreg[tt][m] = make_uint4(0, 0, 0, 0);
    }
  }
  const int nst = (nr + kRowsPerStage - 1) / kRowsPerStage;
  for (int s = 0; s < nst; ++s) {
    if (!mbar_wait_bounded(&bars[s], 0, p.wait_limit_ns, p.ctl, 10 + s)) return false;
    const int row = s * kRowsPerStage + warp;
    if (row >= nr) continue;
    const uint16_t* krow = k1s + static_cast<size_t>(row) * p.r;
    float acc[TG];
#pragma unroll
    for (int tt = 0; tt < TG; ++tt) acc[tt] = 0.f;
#pragma unroll
    for (int m = 0; m < kFusedMaxChunks; ++m) {
      const int c = lane + 32 * m;
      if (c < nchunk) {
        const uint4 kv = lds128(krow + c * 8);
#pragma unroll
        for (int tt = 0; tt < TG; ++tt) acc[tt] = dot8_bf16(kv, qreg[tt][m], acc[tt]);
      }
    }
#pragma unroll
    for (int tt = 0; tt < TG; ++tt) {
      const float v = warp_sum(acc[tt]);
      if (lane == 0 && tg0 + tt < p.T) xs[(tg0 + tt) * p.rpc + row] = v;
    }
  }
  return true;
}

template <int TG>
__global__ void __launch_bounds__(kThreads, 1) spark_ffn_fused_kernel(const KParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SmemLayout L(p.T, p.d_model, p.r, p.rpc);
  unsigned char* region_a = smem + L.region_a;
  uint16_t* k1s = reinterpret_cast<uint16_t*>(region_a);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* theta_s = reinterpret_cast<float*>(smem + L.theta);
  float* spec_s = reinterpret_cast<float*>(smem + L.spec);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  float* ug = reinterpret_cast<float*>(smem + L.ug);
  float* hs = reinterpret_cast<float*>(smem + L.hs);
  int* wcnt = reinterpret_cast<int*>(smem + L.wcnt);
  int* flags = reinterpret_cast<int*>(smem + L.flags);
  DeviceControl* ctl = p.ctl;

  const int n0 = cta * p.rpc;
  const int nr = rows_of_cta(cta, p.rpc, p.d_ff);
  const int nst = (nr + kRowsPerStage - 1) / kRowsPerStage;
  const int qbar = p.rpc / kRowsPerStage;  // bars[qbar]: q copy; bars[qbar + 1]: phase-2 batches
  const int pbar = qbar + 1;

  // A previous launch on this workspace gave up waiting: do nothing until the
  // host has read and cleared the status.
  if (ld_relaxed_gpu(&ctl->abort)) return;

  // ---------------------------------------------------------------- phase 1
  if (tid == 0) {
    for (int s = 0; s <= pbar; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    const unsigned qbytes = static_cast<unsigned>(p.T) * p.d_model * 2;
    mbar_arrive_expect_tx(&bars[qbar], qbytes);
    bulk_g2s(qs, p.q, qbytes, &bars[qbar]);
    for (int s = 0; s < nst; ++s) {
      const int rows = min(kRowsPerStage, nr - s * kRowsPerStage);
      const unsigned bytes = static_cast<unsigned>(rows) * p.r * 2;
      mbar_arrive_expect_tx(&bars[s], bytes);
      bulk_g2s(k1s + static_cast<size_t>(s) * kRowsPerStage * p.r,
               p.K1 + static_cast<size_t>(n0 + s * kRowsPerStage) * p.r, bytes, &bars[s]);
    }
  }
  __syncthreads();
  bool ok = mbar_wait_bounded(&bars[qbar], 0, p.wait_limit_ns, ctl, 9);
  for (int tg0 = 0; ok && tg0 < p.T; tg0 += TG) ok = phase1_token_group<TG>(p, k1s, qs, xs, bars, nr, tg0);
  if (!__syncthreads_and(ok)) {
    // give the copies in flight a bounded chance to land before the CTA exits
    if (tid == 0)
      for (int s = 0; s < nst; ++s) mbar_wait_bounded(&bars[s], 0, p.wait_limit_ns, ctl, 30);
    return;
  }

  // per-token moments of this CTA's slice, about its first score
  for (int t = warp; t < p.T; t += kWarps) {
    const float* xt = xs + t * p.rpc;
    const float shift = nr > 0 ? xt[0] : 0.f;
    float acc = 0.f;
    for (int i = lane; i < nr; i += 32) acc += xt[i] - shift;
    acc = __shfl_sync(0xffffffffu, warp_sum(acc), 0);
    const float mean = nr > 0 ? shift + acc / static_cast<float>(nr) : 0.f;
    float m2 = 0.f;
    for (int i = lane; i < nr; i += 32) {
      const float c = xt[i] - mean;
      m2 += c * c;
    }
    m2 = warp_sum(m2);
    if (lane == 0) {
      p.partials[static_cast<size_t>(t) * G + cta] = make_float2(mean, m2);
      const float sd = nr > 0 ? sqrtf(m2 / static_cast<float>(nr)) : 0.f;
      spec_s[t] = p.spec_margin > 0.f ? fmaf(sd, p.Q - p.spec_margin, mean) : __int_as_float(0x7f800000);
    }
    if (p.x_out != nullptr)
      for (int i = lane; i < nr; i += 32) p.x_out[static_cast<size_t>(t) * p.d_ff + n0 + i] = xt[i];
  }
  __syncthreads();

  // arrive at the statistics exchange
  if (tid == 0) {
    const unsigned old = atom_add_acq_rel_gpu(&ctl->arrive1, 1u);
    flags[0] = (old == static_cast<unsigned>(G - 1) + (p.never_arrive ? 1u : 0u)) ? 1 : 0;
  }
  // speculative L2 prefetch of likely-active K2 / V rows while the others finish
  if (p.spec_margin > 0.f) {
    for (int li = tid; li < nr; li += kThreads) {
      bool cand = false;
      for (int t = 0; t < p.T; ++t) cand |= xs[t * p.rpc + li] > spec_s[t];
      if (cand) {
        const size_t row = static_cast<size_t>(n0 + li);
        prefetch_l2_bulk(p.K2 + row * p.d2, p.d2 * 2);
        prefetch_l2_bulk(p.V + row * p.d_model, p.d_model * 2);
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- thresholds
  if (flags[0]) {
    // last arrival: merge every CTA's moments in CTA order (two passes over the
    // partials: weighted mean, then M2 = sum M2_c + n_c (mean_c - mean)^2)
    for (int t = warp; t < p.T; t += kWarps) {
      float2 pr[8];
      float nc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = lane + 32 * j;
        const bool in = c < G;
        pr[j] = in ? __ldcg(p.partials + static_cast<size_t>(t) * G + c) : make_float2(0.f, 0.f);
        nc[j] = in ? static_cast<float>(rows_of_cta(c, p.rpc, p.d_ff)) : 0.f;
      }
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) s = fmaf(nc[j], pr[j].x, s);
      s = __shfl_sync(0xffffffffu, warp_sum(s), 0);
      const float mean = s / static_cast<float>(p.d_ff);
      float m2 = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float dm = pr[j].x - mean;
        m2 += pr[j].y + nc[j] * dm * dm;
      }
      m2 = warp_sum(m2);
      if (lane == 0) theta_s[t] = fmaf(sqrtf(fmaxf(m2, 0.f) / static_cast<float>(p.d_ff)), p.Q, mean);
    }
    __syncthreads();
    if (tid == 0) {
      for (int t = 1; t < p.T; ++t) ctl->theta[t] = theta_s[t];
      if (p.theta_out != nullptr)
        for (int t = 0; t < p.T; ++t) p.theta_out[t] = theta_s[t];
      const unsigned long long word =
          (static_cast<unsigned long long>(__float_as_uint(theta_s[0])) << 32) | 1ull;
      st_release_gpu_u64(&ctl->theta_word, word);
    }
  } else if (tid == 0) {
    int good = 1;
    unsigned long long word = ld_acquire_gpu_u64(&ctl->theta_word);
    if ((word & 0xffffffffull) == 0) {
      const uint64_t t0 = global_timer_ns();
      while (((word = ld_acquire_gpu_u64(&ctl->theta_word)) & 0xffffffffull) == 0) {
        if (ld_relaxed_gpu(&ctl->abort)) { good = 0; break; }
        if (global_timer_ns() - t0 > p.wait_limit_ns) {
          record_error(ctl, kDevTimeout, 1);
          good = 0;
          break;
        }
      }
    }
    theta_s[0] = __uint_as_float(static_cast<unsigned>(word >> 32));
    for (int t = 1; t < p.T; ++t) theta_s[t] = ld_relaxed_gpu_f32(&ctl->theta[t]);
    flags[1] = good;
  }
  if (tid == 0 && flags[0]) flags[1] = 1;
  __syncthreads();
  if (!flags[1]) return;

  // ---------------------------------------------------------------- phase 2
  // soft threshold + GELU on own neurons; compact the union-active ones (ascending)
  for (int base = 0; base < p.rpc; base += kThreads) {
    const int li = base + tid;
    float g[kFusedMaxTokens];
    bool any = false;
#pragma unroll
    for (int t = 0; t < kFusedMaxTokens; ++t) {
      g[t] = 0.f;
      if (t < p.T && li < nr) {
        const float s = xs[t * p.rpc + li] - theta_s[t];
        const bool act = s > 0.f;
        if (act) g[t] = gelu_tanh(s);
        any |= act;
        if (p.active_out != nullptr) p.active_out[static_cast<size_t>(t) * p.d_ff + n0 + li] = act ? 1 : 0;
      }
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, any);
    if (lane == 0) wcnt[warp] = __popc(ballot);
    __syncthreads();
    if (tid == 0) {
      int run = base == 0 ? 0 : wcnt[kWarps];
      for (int w = 0; w < kWarps; ++w) {
        const int c = wcnt[w];
        wcnt[w] = run;
        run += c;
      }
      wcnt[kWarps] = run;
    }
    __syncthreads();
    const int pos = wcnt[warp] + __popc(ballot & ((1u << lane) - 1u));
    if (any && SPARK_CHECK(pos < nr)) {
      uidx[pos] = li;
#pragma unroll
      for (int t = 0; t < kFusedMaxTokens; ++t)
        if (t < p.T) ug[pos * p.T + t] = g[t];
    }
    __syncthreads();
  }
  const int nu = wcnt[kWarps];

  // K2 / V rows of the active neurons -> shared memory (batches), h, partial out
  const int nchunk2 = p.d2 / 8;
  const int ncc = p.d_model / 8;  // 8-column chunks of the output row
  const size_t row_bytes = static_cast<size_t>(p.d2 + p.d_model) * 2;
  float acc[kMaxColChunks][kFusedMaxTokens][8];
#pragma unroll
  for (int ci = 0; ci < kMaxColChunks; ++ci)
#pragma unroll
    for (int t = 0; t < kFusedMaxTokens; ++t)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[ci][t][j] = 0.f;

  int batch = 0;
  for (int b0 = 0; b0 < nu; b0 += L.batch_rows, ++batch) {
    const int nb = min(L.batch_rows, nu - b0);
    if (warp == 0) {
      if (lane == 0) {
        fence_proxy_async_shared();
        mbar_arrive_expect_tx(&bars[pbar], static_cast<unsigned>(nb * row_bytes));
      }
      __syncwarp();
      for (int u = lane; u < nb; u += 32) {
        // (a failed check copies the slice's first row so the byte count still
        // matches the barrier's expected transaction bytes)
        const int li = uidx[b0 + u];
        const size_t row = static_cast<size_t>(n0 + (SPARK_CHECK(li >= 0 && n0 + li < p.d_ff) ? li : 0));
        unsigned char* dst = region_a + static_cast<size_t>(u) * row_bytes;
        bulk_g2s(dst, p.K2 + row * p.d2, p.d2 * 2, &bars[pbar]);
        bulk_g2s(dst + static_cast<size_t>(p.d2) * 2, p.V + row * p.d_model, p.d_model * 2, &bars[pbar]);
      }
    }
    const bool landed = mbar_wait_bounded(&bars[pbar], batch & 1, p.wait_limit_ns, ctl, 40);
    if (!__syncthreads_and(landed)) return;
    // h = g * <K2[i,:], q[r:]>: one warp per row
    for (int u = warp; u < nb; u += kWarps) {
      const uint16_t* k2row = reinterpret_cast<const uint16_t*>(region_a + static_cast<size_t>(u) * row_bytes);
      uint4 kv[kFusedMaxChunks];
#pragma unroll
      for (int m = 0; m < kFusedMaxChunks; ++m) {
        const int c = lane + 32 * m;
        kv[m] = c < nchunk2 ? lds128(k2row + c * 8) : make_uint4(0, 0, 0, 0);
      }
      for (int t = 0; t < p.T; ++t) {
        const float g = ug[(b0 + u) * p.T + t];
        float h = 0.f;
        if (g != 0.f) {
          const uint16_t* q2 = qs + static_cast<size_t>(t) * p.d_model + p.r;
          float a = 0.f;
#pragma unroll
          for (int m = 0; m < kFusedMaxChunks; ++m) {
            const int c = lane + 32 * m;
            if (c < nchunk2) a = dot8_bf16(kv[m], lds128(q2 + c * 8), a);
          }
          h = g * warp_sum(a);
        }
        if (lane == 0) hs[(b0 + u) * p.T + t] = h;
      }
    }
    __syncthreads();
    // partial out[t, cols] += h[t][u] V[i_u, cols]
#pragma unroll
    for (int ci = 0; ci < kMaxColChunks; ++ci) {
      const int cc = tid + ci * kThreads;
      if (cc < ncc) {
        for (int u = 0; u < nb; ++u) {
          const uint4 v = lds128(region_a + static_cast<size_t>(u) * row_bytes + static_cast<size_t>(p.d2) * 2 +
                                 static_cast<size_t>(cc) * 16);
          const float2 v0 = bf16x2_to_float2(v.x), v1 = bf16x2_to_float2(v.y);
          const float2 v2 = bf16x2_to_float2(v.z), v3 = bf16x2_to_float2(v.w);
#pragma unroll
          for (int t = 0; t < kFusedMaxTokens; ++t) {
            if (t < p.T) {
              const float h = hs[(b0 + u) * p.T + t];
              acc[ci][t][0] = fmaf(h, v0.x, acc[ci][t][0]);
              acc[ci][t][1] = fmaf(h, v0.y, acc[ci][t][1]);
              acc[ci][t][2] = fmaf(h, v1.x, acc[ci][t][2]);
              acc[ci][t][3] = fmaf(h, v1.y, acc[ci][t][3]);
              acc[ci][t][4] = fmaf(h, v2.x, acc[ci][t][4]);
              acc[ci][t][5] = fmaf(h, v2.y, acc[ci][t][5]);
              acc[ci][t][6] = fmaf(h, v3.x, acc[ci][t][6]);
              acc[ci][t][7] = fmaf(h, v3.y, acc[ci][t][7]);
            }
          }
        }
      }
    }
    __syncthreads();  // batch buffers free for the next batch
  }
  // this CTA's partial output (zeros when it owns no active neuron)
#pragma unroll
  for (int ci = 0; ci < kMaxColChunks; ++ci) {
    const int cc = tid + ci * kThreads;
    if (cc < ncc) {
#pragma unroll
      for (int t = 0; t < kFusedMaxTokens; ++t) {
        if (t < p.T) {
          float4* dst = reinterpret_cast<float4*>(p.pout + (static_cast<size_t>(cta) * p.T + t) * p.d_model + cc * 8);
          __stcg(dst, make_float4(acc[ci][t][0], acc[ci][t][1], acc[ci][t][2], acc[ci][t][3]));
          __stcg(dst + 1, make_float4(acc[ci][t][4], acc[ci][t][5], acc[ci][t][6], acc[ci][t][7]));
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    atom_add_release_gpu(&ctl->arrive2, 1u);
    flags[2] = wait_count_geq(ctl, &ctl->arrive2, static_cast<unsigned>(G), p.wait_limit_ns, 2) ? 1 : 0;
  }
  __syncthreads();
  if (!flags[2]) return;

  // ---------------------------------------------------------------- reduce
  if (cta < p.n_col_ctas) {
    const int col0 = cta * p.col_width;
    const int ncol = min(p.col_width, p.d_model - col0);
    const int P = p.col_width / 4;  // float4 chunks per token (power of two, <= 256)
    const int groups = kThreads / P;
    const int ch = tid % P, grp = tid / P;
    const bool col_ok = ch * 4 < ncol;
    float4 s[kFusedMaxTokens];
#pragma unroll
    for (int t = 0; t < kFusedMaxTokens; ++t) s[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (col_ok) {
      // sources grp, grp + groups, ...: four loaded before each group of sums
      for (int src0 = grp; src0 < G; src0 += 4 * groups) {
        float4 v[4][kFusedMaxTokens];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int src = src0 + u * groups;
#pragma unroll
          for (int t = 0; t < kFusedMaxTokens; ++t)
            v[u][t] = (src < G && t < p.T)
                          ? __ldcg(reinterpret_cast<const float4*>(
                                p.pout + (static_cast<size_t>(src) * p.T + t) * p.d_model + col0 + ch * 4))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int t = 0; t < kFusedMaxTokens; ++t) {
            s[t].x += v[u][t].x;
            s[t].y += v[u][t].y;
            s[t].z += v[u][t].z;
            s[t].w += v[u][t].w;
          }
      }
    }
    float4* red = reinterpret_cast<float4*>(region_a);
    int nred;
    if (P < 32) {
      for (int off = 16; off >= P; off >>= 1) {
#pragma unroll
        for (int t = 0; t < kFusedMaxTokens; ++t) {
          s[t].x += __shfl_xor_sync(0xffffffffu, s[t].x, off);
          s[t].y += __shfl_xor_sync(0xffffffffu, s[t].y, off);
          s[t].z += __shfl_xor_sync(0xffffffffu, s[t].z, off);
          s[t].w += __shfl_xor_sync(0xffffffffu, s[t].w, off);
        }
      }
      if (lane < P)
#pragma unroll
        for (int t = 0; t < kFusedMaxTokens; ++t) red[(warp * P + lane) * kFusedMaxTokens + t] = s[t];
      nred = kWarps;
    } else {
#pragma unroll
      for (int t = 0; t < kFusedMaxTokens; ++t) red[(grp * P + ch) * kFusedMaxTokens + t] = s[t];
      nred = groups;
    }
    __syncthreads();
    for (int o = tid; o < p.T * P; o += kThreads) {
      const int t = o / P, c4 = o % P;
      if (c4 * 4 >= ncol) continue;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int w = 0; w < nred; ++w) {
        const float4 b = red[(w * P + c4) * kFusedMaxTokens + t];
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
      __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
      uint2 packed;
      packed.x = *reinterpret_cast<uint32_t*>(&lo);
      packed.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(p.out + static_cast<size_t>(t) * p.d_model + col0 + c4 * 4) = packed;
    }
  }

  // ---------------------------------------------------------------- exit
  __syncthreads();
  if (tid == 0) {
    const unsigned old = atom_add_acq_rel_gpu(&ctl->exit_count, 1u);
    if (old == static_cast<unsigned>(G - 1)) {  // last CTA out resets the counters for the next launch
      ctl->arrive1 = 0u;
      ctl->arrive2 = 0u;
      ctl->theta_word = 0ull;
      __threadfence();
      ctl->exit_count = 0u;
    }
  }
}

}  // namespace

FusedPlan plan_fused(int T, int d_model, int r, int d_ff, int num_sms, size_t smem_optin) {
  FusedPlan pl{};
  pl.ok = false;
  const int d2 = d_model - r;
  if (T < 1 || T > kFusedMaxTokens || r > 32 * 8 * kFusedMaxChunks || d2 > 32 * 8 * kFusedMaxChunks) return pl;
  if (d_model > 8 * kThreads * kMaxColChunks) return pl;
  int rpc = (d_ff + num_sms - 1) / num_sms;
  rpc = static_cast<int>(align_up(static_cast<size_t>(rpc), kRowsPerStage));
  if (rpc > kFusedMaxRowsPerCta) return pl;
  const int grid = (d_ff + rpc - 1) / rpc;
  if (grid > 256) return pl;  // moments merge reads up to 8 partials per lane
  int cw = 4;
  while ((d_model + cw - 1) / cw > grid) cw *= 2;
  if (cw / 4 > kThreads) return pl;
  const SmemLayout L(T, d_model, r, rpc);
  if (L.total > smem_optin || L.batch_rows < 1) return pl;
  const WsLayout W(T, d_model, grid);
  pl.grid = grid;
  pl.rows_per_cta = rpc;
  pl.col_width = cw;
  pl.n_col_ctas = (d_model + cw - 1) / cw;
  pl.smem_bytes = L.total;
  pl.ws_bytes = W.total;
  pl.ok = true;
  return pl;
}

cudaError_t launch_fused(const FusedPlan& pl, const FusedArgs& a, cudaStream_t stream) {
  const WsLayout W(a.T, a.d_model, pl.grid);
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  KParams p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.K1 = static_cast<const uint16_t*>(a.K1);
  p.K2 = static_cast<const uint16_t*>(a.K2);
  p.V = static_cast<const uint16_t*>(a.V);
  p.out = static_cast<uint16_t*>(a.out);
  p.T = a.T;
  p.d_model = a.d_model;
  p.r = a.r;
  p.d2 = a.d_model - a.r;
  p.d_ff = a.d_ff;
  p.rpc = pl.rows_per_cta;
  p.col_width = pl.col_width;
  p.n_col_ctas = pl.n_col_ctas;
  p.Q = a.Q;
  p.spec_margin = a.spec_margin;
  p.x_out = a.x_out;
  p.theta_out = a.theta_out;
  p.active_out = a.active_out;
  p.ctl = reinterpret_cast<DeviceControl*>(ws);
  p.partials = reinterpret_cast<float2*>(ws + W.partials);
  p.pout = reinterpret_cast<float*>(ws + W.pout);
  p.wait_limit_ns = a.wait_limit_ns;
  p.never_arrive = a.never_arrive;

  const int tmpl = a.T == 1 ? 0 : 1;
  const void* fn = tmpl == 0 ? reinterpret_cast<const void*>(&spark_ffn_fused_kernel<1>)
                             : reinterpret_cast<const void*>(&spark_ffn_fused_kernel<2>);
  // Raise the dynamic shared-memory limit once per (device, kernel) so that
  // launches inside a stream capture issue no attribute calls.
  static size_t smem_set[64][2] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem_set[dev][tmpl] < pl.smem_bytes) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.smem_bytes));
    if (e != cudaSuccess) return e;
    smem_set[dev][tmpl] = pl.smem_bytes;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.T == 1) return cudaLaunchKernelEx(&cfg, spark_ffn_fused_kernel<1>, p);
  return cudaLaunchKernelEx(&cfg, spark_ffn_fused_kernel<2>, p);
}


// ---------------------------------------------------------------- debug builds
unsigned take_bounds_violations_fused(bool clear) {
#ifdef SPARK_DEBUG
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_bounds_violations, sizeof v) != cudaSuccess ||
      (clear && cudaMemcpyToSymbol(g_bounds_violations, &zero, sizeof zero) != cudaSuccess)) {
    cudaGetLastError();
    return 0xffffffffu;
  }
  return v;
#else
  (void)clear;
  return 0;
#endif
}

}  // namespace spark
