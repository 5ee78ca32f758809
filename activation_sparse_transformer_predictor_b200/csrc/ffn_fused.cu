// ffn_fused.cu -- Spark FFN forward for a few tokens (decode) in ONE kernel.
//
// Spark Transformer notes, 关键设计 / "Spark FFN":
//   x = K1^T q[:r];  theta = mean(x) + std(x) Q(1 - k/d_ff)  ("Statistical Top-k");
//   out = V . (GELU(max(x - theta, 0)) (.) (K2^T q[r:])), evaluated only on the
//   neurons with x > theta.
//
// Decode is bound by HBM bytes: all of K1 plus the active rows of K2 and V.  The
// kernel is a cooperative launch of one CTA per SM (all co-resident) in three
// phases separated by two bounded grid barriers:
//
//  phase 1  CTA c owns neurons [c*RPC, (c+1)*RPC).  One thread issues bulk
//           (TMA-engine) copies of the CTA's whole K1 slice into shared memory at
//           kernel start (8 rows per mbarrier), so every byte of K1 is in flight
//           at once.  Eight warps compute x for their rows (fp32 FMA, q[:r] held
//           in registers), then per-token moments (count, mean, M2) of the slice.
//  barrier 1
//  phase 2a Every CTA merges all CTAs' moments in the same fixed order (so every
//           CTA derives bit-identical thresholds), applies the soft threshold and
//           GELU to its own neurons, compacts the union-active ones, and for each
//           computes h = g * <K2[i,:], q[r:]>, reading only active K2 rows.  It
//           prefetches the matching V rows into L2 and publishes (i, h) lists.
//  barrier 2
//  phase 2b CTA c owns output columns [c*CW, (c+1)*CW): it walks every published
//           (i, h) entry in ascending neuron order, reads V[i, cols] (16-byte
//           loads) and reduces in a fixed order, then writes bf16.  No split-K
//           workspace and no atomics: the result is deterministic.
#include <algorithm>

#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerStage = kWarps;  // one row per warp per stage
constexpr int kStageEntries = 1024;    // (i, h) entries staged per pass in phase 2b

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Shared-memory carve-up; computed identically on host and device.
struct SmemLayout {
  size_t region_a;  // K1 slice (phase 1), then staging + reduction (phase 2b)
  size_t qs, xs, bars, theta, ug, uidx, wcnt, prefix, flag, total;
  __host__ __device__ SmemLayout(int T, int d_model, int r, int rpc, int grid) {
    const int nst = rpc / kRowsPerStage;
    const size_t k1_bytes = static_cast<size_t>(nst) * kRowsPerStage * r * 2;
    const size_t p2b = static_cast<size_t>(kStageEntries) * 4 + static_cast<size_t>(kStageEntries) * T * 4 +
                       static_cast<size_t>(T) * kWarps * 32 * 8 * 4;
    size_t off = 0;
    region_a = off;
    off += align_up(k1_bytes > p2b ? k1_bytes : p2b, 128);
    qs = off;
    off += align_up(static_cast<size_t>(T) * d_model * 2, 128);
    xs = off;
    off += align_up(static_cast<size_t>(T) * rpc * 4, 16);
    bars = off;
    off += align_up(static_cast<size_t>(nst + 1) * 8, 16);
    theta = off;
    off += align_up(static_cast<size_t>(kFusedMaxTokens) * 4, 16);
    ug = off;
    off += align_up(static_cast<size_t>(rpc) * T * 4, 16);
    uidx = off;
    off += align_up(static_cast<size_t>(rpc) * 4, 16);
    wcnt = off;
    off += align_up(static_cast<size_t>(kWarps + 1) * 4, 16);
    prefix = off;
    off += align_up(static_cast<size_t>(grid + 1) * 4, 16);
    flag = off;
    off += 16;
    total = off;
  }
};

// Workspace carve-up (after the 64-byte device control block).
struct WsLayout {
  size_t partials, cta_count, list_idx, list_h, total;
  WsLayout(int T, int rpc, int grid) {
    size_t off = sizeof(DeviceControl);
    partials = off;
    off += align_up(static_cast<size_t>(T) * grid * sizeof(float2), 256);
    cta_count = off;
    off += align_up(static_cast<size_t>(grid) * 4, 256);
    list_idx = off;
    off += align_up(static_cast<size_t>(grid) * rpc * 4, 256);
    list_h = off;
    off += align_up(static_cast<size_t>(grid) * rpc * T * 4, 256);
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
  float* x_out;
  float* theta_out;
  unsigned char* active_out;
  DeviceControl* ctl;
  float2* partials;
  int* cta_count;
  int* list_idx;
  float* list_h;
  unsigned long long wait_limit_ns;
  int never_arrive;
};

__device__ __forceinline__ float dot8_bf16(uint4 a, uint4 b, float acc) {
  float2 a0 = bf16x2_to_float2(a.x), b0 = bf16x2_to_float2(b.x);
  acc = fmaf(a0.x, b0.x, acc);
  acc = fmaf(a0.y, b0.y, acc);
  float2 a1 = bf16x2_to_float2(a.y), b1 = bf16x2_to_float2(b.y);
  acc = fmaf(a1.x, b1.x, acc);
  acc = fmaf(a1.y, b1.y, acc);
  float2 a2 = bf16x2_to_float2(a.z), b2 = bf16x2_to_float2(b.z);
  acc = fmaf(a2.x, b2.x, acc);
  acc = fmaf(a2.y, b2.y, acc);
  float2 a3 = bf16x2_to_float2(a.w), b3 = bf16x2_to_float2(b.w);
  acc = fmaf(a3.x, b3.x, acc);
  acc = fmaf(a3.y, b3.y, acc);
  return acc;
}

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

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
  const SmemLayout L(p.T, p.d_model, p.r, p.rpc, G);
  uint16_t* k1s = reinterpret_cast<uint16_t*>(smem + L.region_a);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* theta_s = reinterpret_cast<float*>(smem + L.theta);
  float* ug = reinterpret_cast<float*>(smem + L.ug);
  int* uidx = reinterpret_cast<int*>(smem + L.uidx);
  int* wcnt = reinterpret_cast<int*>(smem + L.wcnt);
  int* prefix = reinterpret_cast<int*>(smem + L.prefix);
  int* flag = reinterpret_cast<int*>(smem + L.flag);

  const int n0 = cta * p.rpc;
  const int nr = rows_of_cta(cta, p.rpc, p.d_ff);
  const int nst = (nr + kRowsPerStage - 1) / kRowsPerStage;
  const int qbar = p.rpc / kRowsPerStage;  // last barrier slot

  // A previous launch on this workspace gave up waiting: do nothing until the
  // host has read and cleared the status.
  if (ld_relaxed_gpu(&p.ctl->abort)) return;

  // ---------------------------------------------------------------- phase 1
  if (tid == 0) {
    for (int s = 0; s <= qbar; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
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
  bool ok = mbar_wait_bounded(&bars[qbar], 0, p.wait_limit_ns, p.ctl, 9);
  for (int tg0 = 0; ok && tg0 < p.T; tg0 += TG) ok = phase1_token_group<TG>(p, k1s, qs, xs, bars, nr, tg0);
  if (!__syncthreads_and(ok)) {
    // give the copies in flight a bounded chance to land before the CTA exits
    if (tid == 0)
      for (int s = 0; s < nst; ++s) mbar_wait_bounded(&bars[s], 0, p.wait_limit_ns, p.ctl, 30);
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
    if (lane == 0) p.partials[static_cast<size_t>(t) * G + cta] = make_float2(mean, m2);
    if (p.x_out != nullptr)
      for (int i = lane; i < nr; i += 32) p.x_out[static_cast<size_t>(t) * p.d_ff + n0 + i] = xt[i];
  }

  if (!grid_barrier(p.ctl, G, p.never_arrive ? 1u : 0u, p.wait_limit_ns, 1, flag)) return;

  // ---------------------------------------------------------------- phase 2a
  // thresholds: every CTA merges all partials in the same order
  for (int t = warp; t < p.T; t += kWarps) {
    Moments m{0.f, 0.f, 0.f};
    for (int c = lane; c < G; c += 32) {
      const float2 pr = __ldcg(p.partials + static_cast<size_t>(t) * G + c);
      m = merge_moments(m, Moments{static_cast<float>(rows_of_cta(c, p.rpc, p.d_ff)), pr.x, pr.y});
    }
    m = warp_merge_moments(m);
    if (lane == 0) {
      const float sd = m.n > 0.f ? sqrtf(fmaxf(m.m2, 0.f) / m.n) : 0.f;
      const float th = fmaf(sd, p.Q, m.mean);
      theta_s[t] = th;
      if (cta == 0 && p.theta_out != nullptr) p.theta_out[t] = th;
    }
  }
  __syncthreads();

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
    if (any) {
      const int pos = wcnt[warp] + __popc(ballot & ((1u << lane) - 1u));
      uidx[pos] = li;
#pragma unroll
      for (int t = 0; t < kFusedMaxTokens; ++t)
        if (t < p.T) ug[pos * p.T + t] = g[t];
    }
    __syncthreads();
  }
  const int nu = nr > 0 ? wcnt[kWarps] : 0;

  // h = g * <K2[i,:], q[r:]> for union-active rows; V rows prefetched into L2
  {
    const int nchunk2 = p.d2 / 8;
    for (int u = warp; u < nu; u += kWarps) {
      const int row = n0 + uidx[u];
      if (lane == 0) prefetch_l2_bulk(p.V + static_cast<size_t>(row) * p.d_model, p.d_model * 2);
      const uint16_t* k2row = p.K2 + static_cast<size_t>(row) * p.d2;
      uint4 kv[kFusedMaxChunks];
#pragma unroll
      for (int m = 0; m < kFusedMaxChunks; ++m) {
        const int c = lane + 32 * m;
        kv[m] = c < nchunk2 ? ldg_nc128(k2row + c * 8) : make_uint4(0, 0, 0, 0);
      }
      for (int t = 0; t < p.T; ++t) {
        const float g = ug[u * p.T + t];
        float h = 0.f;
        if (g != 0.f) {
          const uint16_t* q2 = qs + static_cast<size_t>(t) * p.d_model + p.r;
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < kFusedMaxChunks; ++m) {
            const int c = lane + 32 * m;
            if (c < nchunk2) acc = dot8_bf16(kv[m], lds128(q2 + c * 8), acc);
          }
          h = g * warp_sum(acc);
        }
        if (lane == 0) p.list_h[(static_cast<size_t>(cta) * p.rpc + u) * p.T + t] = h;
      }
      if (lane == 0) p.list_idx[static_cast<size_t>(cta) * p.rpc + u] = row;
    }
    if (tid == 0) p.cta_count[cta] = nu;
  }

  if (!grid_barrier(p.ctl, G, 0u, p.wait_limit_ns, 2, flag)) return;

  // ---------------------------------------------------------------- phase 2b
  if (cta >= p.n_col_ctas) return;
  // exclusive prefix of the per-CTA entry counts (warp 0, fixed order)
  if (warp == 0) {
    const int per = (G + 31) / 32;
    int local[8];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = lane * per + j;
      local[j] = (j < per && c < G) ? __ldcg(p.cta_count + c) : 0;
      sum += local[j];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = lane * per + j;
      if (j < per && c < G) prefix[c] = run;
      run += local[j];
    }
    if (lane == 31) prefix[G] = incl;
  }
  __syncthreads();
  const int total = prefix[G];

  const int col0 = cta * p.col_width;
  const int ncol = min(p.col_width, p.d_model - col0);
  const int cpr_full = p.col_width / 8;  // power of two, divides kThreads
  const int cc = tid % cpr_full;
  const int estride = kThreads / cpr_full;
  const bool col_ok = cc * 8 < ncol;

  int* st_idx = reinterpret_cast<int*>(smem + L.region_a);
  float* st_h = reinterpret_cast<float*>(smem + L.region_a + static_cast<size_t>(kStageEntries) * 4);
  float* red = st_h + static_cast<size_t>(kStageEntries) * p.T;

  float acc[kFusedMaxTokens][8];
#pragma unroll
  for (int t = 0; t < kFusedMaxTokens; ++t)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[t][j] = 0.f;

  for (int e0 = 0; e0 < total; e0 += kStageEntries) {
    const int ne = min(kStageEntries, total - e0);
    __syncthreads();  // previous chunk consumed
    for (int e = tid; e < ne; e += kThreads) {
      const int ge = e0 + e;
      int lo = 0, hi = G - 1;  // last src with prefix[src] <= ge
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= ge) lo = mid; else hi = mid - 1;
      }
      const size_t slot = static_cast<size_t>(lo) * p.rpc + (ge - prefix[lo]);
      st_idx[e] = __ldcg(p.list_idx + slot);
      for (int t = 0; t < p.T; ++t) st_h[e * p.T + t] = __ldcg(p.list_h + slot * p.T + t);
    }
    __syncthreads();
    if (col_ok) {
      int e = tid / cpr_full;
      // four rows in flight per thread
      for (; e + 3 * estride < ne; e += 4 * estride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[u] = ldg_nc128(p.V + static_cast<size_t>(st_idx[e + u * estride]) * p.d_model + col0 + cc * 8);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int eu = e + u * estride;
          const float2 v0 = bf16x2_to_float2(v[u].x), v1 = bf16x2_to_float2(v[u].y);
          const float2 v2 = bf16x2_to_float2(v[u].z), v3 = bf16x2_to_float2(v[u].w);
#pragma unroll
          for (int t = 0; t < kFusedMaxTokens; ++t) {
            if (t < p.T) {
              const float h = st_h[eu * p.T + t];
              acc[t][0] = fmaf(h, v0.x, acc[t][0]);
              acc[t][1] = fmaf(h, v0.y, acc[t][1]);
              acc[t][2] = fmaf(h, v1.x, acc[t][2]);
              acc[t][3] = fmaf(h, v1.y, acc[t][3]);
              acc[t][4] = fmaf(h, v2.x, acc[t][4]);
              acc[t][5] = fmaf(h, v2.y, acc[t][5]);
              acc[t][6] = fmaf(h, v3.x, acc[t][6]);
              acc[t][7] = fmaf(h, v3.y, acc[t][7]);
            }
          }
        }
      }
      for (; e < ne; e += estride) {
        const uint4 v = ldg_nc128(p.V + static_cast<size_t>(st_idx[e]) * p.d_model + col0 + cc * 8);
        const float2 v0 = bf16x2_to_float2(v.x), v1 = bf16x2_to_float2(v.y);
        const float2 v2 = bf16x2_to_float2(v.z), v3 = bf16x2_to_float2(v.w);
#pragma unroll
        for (int t = 0; t < kFusedMaxTokens; ++t) {
          if (t < p.T) {
            const float h = st_h[e * p.T + t];
            acc[t][0] = fmaf(h, v0.x, acc[t][0]);
            acc[t][1] = fmaf(h, v0.y, acc[t][1]);
            acc[t][2] = fmaf(h, v1.x, acc[t][2]);
            acc[t][3] = fmaf(h, v1.y, acc[t][3]);
            acc[t][4] = fmaf(h, v2.x, acc[t][4]);
            acc[t][5] = fmaf(h, v2.y, acc[t][5]);
            acc[t][6] = fmaf(h, v3.x, acc[t][6]);
            acc[t][7] = fmaf(h, v3.y, acc[t][7]);
          }
        }
      }
    }
  }
  // Fixed-order reduction over the threads that share a column chunk: an xor
  // butterfly inside each warp (lanes with equal lane % cpr_full), then the 8
  // warps in order.  Addition is commutative, so every lane of a butterfly pair
  // holds the same bits.
  for (int off = 16; off >= cpr_full; off >>= 1) {
#pragma unroll
    for (int t = 0; t < kFusedMaxTokens; ++t)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[t][j] += __shfl_xor_sync(0xffffffffu, acc[t][j], off);
  }
  __syncthreads();  // staging buffers no longer read
  if (lane < cpr_full) {
#pragma unroll
    for (int t = 0; t < kFusedMaxTokens; ++t)
      if (t < p.T)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          red[((static_cast<size_t>(t) * kWarps + warp) * cpr_full + lane) * 8 + j] = acc[t][j];
  }
  __syncthreads();
  for (int o = tid; o < p.T * ncol; o += kThreads) {
    const int t = o / ncol, col = o % ncol;
    const int ch = col / 8, j = col % 8;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[((static_cast<size_t>(t) * kWarps + w) * cpr_full + ch) * 8 + j];
    const __nv_bfloat16 b = __float2bfloat16_rn(s);
    p.out[static_cast<size_t>(t) * p.d_model + col0 + col] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace

FusedPlan plan_fused(int T, int d_model, int r, int d_ff, int num_sms, size_t smem_optin) {
  FusedPlan pl{};
  pl.ok = false;
  const int d2 = d_model - r;
  if (T < 1 || T > kFusedMaxTokens || r > 32 * 8 * kFusedMaxChunks || d2 > 32 * 8 * kFusedMaxChunks) return pl;
  int rpc = (d_ff + num_sms - 1) / num_sms;
  rpc = static_cast<int>(align_up(static_cast<size_t>(rpc), kRowsPerStage));
  if (rpc > kFusedMaxRowsPerCta) return pl;
  const int grid = (d_ff + rpc - 1) / rpc;
  int cw = 16;
  while ((d_model + cw - 1) / cw > grid) cw *= 2;
  if (cw > 256) return pl;  // at most 32 column chunks: one per lane
  const SmemLayout L(T, d_model, r, rpc, grid);
  if (L.total > smem_optin) return pl;
  const WsLayout W(T, rpc, grid);
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
  const WsLayout W(a.T, pl.rows_per_cta, pl.grid);
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
  p.x_out = a.x_out;
  p.theta_out = a.theta_out;
  p.active_out = a.active_out;
  p.ctl = reinterpret_cast<DeviceControl*>(ws);
  p.partials = reinterpret_cast<float2*>(ws + W.partials);
  p.cta_count = reinterpret_cast<int*>(ws + W.cta_count);
  p.list_idx = reinterpret_cast<int*>(ws + W.list_idx);
  p.list_h = reinterpret_cast<float*>(ws + W.list_h);
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

}  // namespace spark
