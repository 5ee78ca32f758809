// stat_topk.cu -- standalone statistical top-k with soft threshold.
//
// Spark Transformer notes, 关键设计 / "Statistical Top-k": per row,
// theta = mean(x) + std(x) * Q(1 - k/d), out = max(x - theta, 0).
//
// One CTA per row.  The vectorised kernel keeps the row in registers (one HBM
// read and one HBM write per element, 8 bytes); per-thread moments are taken
// about the thread's first element (exact for constant rows, stable when
// |mean| >> std) and merged across the CTA with the pairwise (Chan) update in a
// fixed tree.  Rows that are misaligned, have d % 4 != 0 or are longer than the
// register budget take the two-pass generic kernel (12 bytes per element).
// The causal variant (below) does the same over each row's visible prefix.
#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;

// Merges the threads' moments (warp shuffles, then warp order through shared
// memory); thread 0 forms theta = mean + std * Q and every thread returns it.
// get_q() is evaluated by thread 0 after the first barrier, so it may read a Q
// that another warp left in shared memory.
template <class GetQ>
__device__ __forceinline__ float block_theta_with(Moments m, GetQ get_q, Moments* s_warp, float* s_theta) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  m = warp_merge_moments(m);
  if (lane == 0) s_warp[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    Moments a = s_warp[0];
#pragma unroll
    for (int w = 1; w < kTopkWarps; ++w) a = merge_moments(a, s_warp[w]);
    const float sd = a.n > 0.f ? sqrtf(fmaxf(a.m2, 0.f) / a.n) : 0.f;
    *s_theta = fmaf(sd, get_q(), a.mean);
  }
  __syncthreads();
  return *s_theta;
}

__device__ __forceinline__ float block_theta(Moments m, float Q, Moments* s_warp, float* s_theta) {
  return block_theta_with(m, [Q] { return Q; }, s_warp, s_theta);
}

template <int NV>
__global__ void __launch_bounds__(kTopkThreads) stat_topk_vec_kernel(const float* x, float* out, int d,
                                                                     float Q) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float s_theta;
  const size_t row = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + row * (size_t)d);
  float4* orow = reinterpret_cast<float4*>(out + row * (size_t)d);
  const int nvec = d >> 2;

  float4 v[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) v[j] = __ldcs(xr + idx);
  }
  // moments about the thread's first element
  float shift = 0.f, cnt = 0.f, acc = 0.f;
  if (threadIdx.x < nvec) shift = v[0].x;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      acc += ((v[j].x - shift) + (v[j].y - shift)) + ((v[j].z - shift) + (v[j].w - shift));
      cnt += 4.f;
    }
  }
  const float mean = cnt > 0.f ? shift + acc / cnt : 0.f;
  float m2 = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      const float a = v[j].x - mean, b = v[j].y - mean, c = v[j].z - mean, e = v[j].w - mean;
      m2 += (a * a + b * b) + (c * c + e * e);
    }
  }
  const float theta = block_theta(Moments{cnt, mean, m2}, Q, s_warp, &s_theta);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      float4 o;
      o.x = fmaxf(v[j].x - theta, 0.f);
      o.y = fmaxf(v[j].y - theta, 0.f);
      o.z = fmaxf(v[j].z - theta, 0.f);
      o.w = fmaxf(v[j].w - theta, 0.f);
      __stcs(orow + idx, o);
    }
  }
}

// Any d, any alignment: pass 1 accumulates per-thread moments (about the
// thread's first element), pass 2 re-reads x and writes the soft threshold.
__global__ void __launch_bounds__(kTopkThreads) stat_topk_generic_kernel(const float* x, float* out,
                                                                         int d, float Q) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float s_theta;
  const size_t row = blockIdx.x;
  const float* xr = x + row * (size_t)d;
  float* orow = out + row * (size_t)d;
  float shift = threadIdx.x < d ? xr[threadIdx.x] : 0.f;
  float cnt = 0.f, acc = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    acc += xr[i] - shift;
    cnt += 1.f;
  }
  const float mean = cnt > 0.f ? shift + acc / cnt : 0.f;
  float m2 = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    const float a = xr[i] - mean;
    m2 += a * a;
  }
  const float theta = block_theta(Moments{cnt, mean, m2}, Q, s_warp, &s_theta);
  for (int i = threadIdx.x; i < d; i += kTopkThreads) orow[i] = fmaxf(xr[i] - theta, 0.f);
}

// ---------------------------------------------------------------------------
// Causal mask ("Spark Attention": a token attends to at most k_attn tokens, so
// the work per query is min{k_attn, n_ctx}): row r is query r mod n_q of its
// head at position offset + r mod n_q and sees its first n = min(d, pos + 1)
// entries.  k < n: theta = mean + std * Q(1 - k/n) over those n, out =
// max(x - theta, 0); k >= n: every visible entry is kept, out = x, theta = -inf.
// Masked entries are written as 0 and never used.  Q depends on n, so each CTA
// evaluates it (double precision, Q(1 - p) = -Phi^-1(p) with CUDA's normcdfinv),
// in one thread of its last warp while the row's loads are in flight.  The vector
// kernel is held to 32 registers so that eight 256-thread CTAs share an SM (32768
// rows x 4096 on B200: 188 us at 48 registers, 165 at 40, 148 at 32).
__device__ __forceinline__ int causal_visible(int row, int d, int n_q, int offset) {
  const long long pos = static_cast<long long>(offset) + row % n_q;
  return pos + 1 < d ? static_cast<int>(pos + 1) : d;
}

__device__ __forceinline__ float causal_quantile(int k, int n) {
  return static_cast<float>(-normcdfinv(static_cast<double>(k) / static_cast<double>(n)));
}

template <int NV>
__global__ void __launch_bounds__(kTopkThreads, 8) stat_topk_causal_vec_kernel(const float* x, float* out, int d, int k,
                                                                            int n_q, int offset, float* theta_out) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float s_theta, s_q;
  const int row = blockIdx.x;
  const int n = causal_visible(row, d, n_q, offset);
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * d);
  float4* orow = reinterpret_cast<float4*>(out + static_cast<size_t>(row) * d);
  const int nvec = d >> 2;
  const int nvis = (n + 3) >> 2;  // float4 groups holding a visible entry

  float4 v[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    v[j] = idx < nvis ? __ldcs(xr + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const bool keep_all = k >= n;
  // the last warp evaluates the quantile while the row's loads are in flight
  if (!keep_all && threadIdx.x == kTopkThreads - 32) s_q = causal_quantile(k, n);
  float theta = -__int_as_float(0x7f800000);
  if (!keep_all) {
    // moments of the visible entries about the thread's first one; groups wholly
    // visible take the unmasked path, only the group holding entry n - 1 is masked
    float shift = 0.f, cnt = 0.f, acc = 0.f;
    if (threadIdx.x < nvis) shift = v[0].x;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e0 = 4 * (threadIdx.x + j * kTopkThreads);
      if (e0 + 4 <= n) {
        acc += ((v[j].x - shift) + (v[j].y - shift)) + ((v[j].z - shift) + (v[j].w - shift));
        cnt += 4.f;
      } else if (e0 < n) {
        const float e[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (e0 + u < n) {
            acc += e[u] - shift;
            cnt += 1.f;
          }
      }
    }
    const float mean = cnt > 0.f ? shift + acc / cnt : 0.f;
    float m2 = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int e0 = 4 * (threadIdx.x + j * kTopkThreads);
      if (e0 + 4 <= n) {
        const float a = v[j].x - mean, b = v[j].y - mean, c = v[j].z - mean, e = v[j].w - mean;
        m2 += (a * a + b * b) + (c * c + e * e);
      } else if (e0 < n) {
        const float e[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (e0 + u < n) {
            const float a = e[u] - mean;
            m2 += a * a;
          }
      }
    }
    // only thread 0 forms theta: the quantile is evaluated there alone
    theta = block_theta_with(Moments{cnt, mean, m2}, [] { return s_q; }, s_warp, &s_theta);
  }
  if (theta_out != nullptr && threadIdx.x == 0) theta_out[row] = theta;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      const int e0 = 4 * idx;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0 + 4 <= n) {
        o = keep_all ? v[j]
                     : make_float4(fmaxf(v[j].x - theta, 0.f), fmaxf(v[j].y - theta, 0.f),
                                   fmaxf(v[j].z - theta, 0.f), fmaxf(v[j].w - theta, 0.f));
      } else if (e0 < n) {
        const float e[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
        float r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) r[u] = e0 + u >= n ? 0.f : keep_all ? e[u] : fmaxf(e[u] - theta, 0.f);
        o = make_float4(r[0], r[1], r[2], r[3]);
      }
      __stcs(orow + idx, o);
    }
  }
}

// Any d, any alignment (two passes over the visible entries).
__global__ void __launch_bounds__(kTopkThreads) stat_topk_causal_generic_kernel(const float* x, float* out, int d,
                                                                                int k, int n_q, int offset,
                                                                                float* theta_out) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float s_theta;
  const int row = blockIdx.x;
  const int n = causal_visible(row, d, n_q, offset);
  const float* xr = x + static_cast<size_t>(row) * d;
  float* orow = out + static_cast<size_t>(row) * d;
  const bool keep_all = k >= n;
  float theta = -__int_as_float(0x7f800000);
  if (!keep_all) {
    const float shift = threadIdx.x < n ? xr[threadIdx.x] : 0.f;
    float cnt = 0.f, acc = 0.f;
    for (int i = threadIdx.x; i < n; i += kTopkThreads) {
      acc += xr[i] - shift;
      cnt += 1.f;
    }
    const float mean = cnt > 0.f ? shift + acc / cnt : 0.f;
    float m2 = 0.f;
    for (int i = threadIdx.x; i < n; i += kTopkThreads) {
      const float a = xr[i] - mean;
      m2 += a * a;
    }
    // only thread 0 forms theta: the quantile is evaluated there alone
    theta = block_theta(Moments{cnt, mean, m2}, threadIdx.x == 0 ? causal_quantile(k, n) : 0.f, s_warp, &s_theta);
  }
  if (theta_out != nullptr && threadIdx.x == 0) theta_out[row] = theta;
  for (int i = threadIdx.x; i < d; i += kTopkThreads)
    orow[i] = i >= n ? 0.f : keep_all ? xr[i] : fmaxf(xr[i] - theta, 0.f);
}

cudaError_t launch_stat_topk_causal(const float* x, float* out, int rows, int d, int k, int n_q, int offset,
                                    float* theta_out, cudaStream_t stream) {
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15u) == 0;
  const int nvec = d / 4;
  const dim3 grid(static_cast<unsigned>(rows));
  if (aligned && d % 4 == 0 && nvec <= 8 * kTopkThreads) {
    const int per_thread = (nvec + kTopkThreads - 1) / kTopkThreads;
    if (per_thread <= 1)
      stat_topk_causal_vec_kernel<1><<<grid, kTopkThreads, 0, stream>>>(x, out, d, k, n_q, offset, theta_out);
    else if (per_thread <= 2)
      stat_topk_causal_vec_kernel<2><<<grid, kTopkThreads, 0, stream>>>(x, out, d, k, n_q, offset, theta_out);
    else if (per_thread <= 4)
      stat_topk_causal_vec_kernel<4><<<grid, kTopkThreads, 0, stream>>>(x, out, d, k, n_q, offset, theta_out);
    else
      stat_topk_causal_vec_kernel<8><<<grid, kTopkThreads, 0, stream>>>(x, out, d, k, n_q, offset, theta_out);
  } else {
    stat_topk_causal_generic_kernel<<<grid, kTopkThreads, 0, stream>>>(x, out, d, k, n_q, offset, theta_out);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Huber-smoothed statistical top-k ("Statistical Top-k", Theorem 3.2: with a
// Huber smoothing the operator is continuously differentiable): the ramp
// max{z, 0} of Soft-Threshold becomes rho(z) = 0 (z <= 0), z^2 / (2 delta)
// (0 < z < delta), z - delta/2 (z >= delta), z = x - theta(x); delta = 0 gives
// the plain operator.  The backward is the vector-Jacobian product
//   dx_j = w_j - W (1/d + Q (x_j - mean) / (d std)),  w = g rho'(z),  W = sum_j w_j
// (theta depends on every x through the row's mean and std).

__device__ __forceinline__ float huber_ramp(float z, float delta, float half_inv_delta) {
  return z <= 0.f ? 0.f : z < delta ? z * z * half_inv_delta : z - 0.5f * delta;
}
__device__ __forceinline__ float huber_slope(float z, float delta, float inv_delta) {
  return z <= 0.f ? 0.f : z < delta ? z * inv_delta : 1.f;
}

// mean and population std of the row from per-thread moments (fixed merge tree).
__device__ __forceinline__ float2 block_mean_std(Moments m, Moments* s_warp, float2* s_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  m = warp_merge_moments(m);
  if (lane == 0) s_warp[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    Moments a = s_warp[0];
#pragma unroll
    for (int w = 1; w < kTopkWarps; ++w) a = merge_moments(a, s_warp[w]);
    *s_out = make_float2(a.mean, a.n > 0.f ? sqrtf(fmaxf(a.m2, 0.f) / a.n) : 0.f);
  }
  __syncthreads();
  return *s_out;
}

// sum over the block, warps in order (the same bits in every thread).
__device__ __forceinline__ float block_sum(float v, float* s_part) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  if (lane == 0) s_part[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) t += s_part[w];
  return t;
}

// Per-thread moments of the thread's elements e[0..n) (n <= N) about e[0].
template <int N>
__device__ __forceinline__ Moments thread_moments(const float (&e)[N], int n) {
  if (n == 0) return Moments{0.f, 0.f, 0.f};
  const float shift = e[0];
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (i < n) acc += e[i] - shift;
  const float mean = shift + acc / static_cast<float>(n);
  float m2 = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i)
    if (i < n) {
      const float a = e[i] - mean;
      m2 += a * a;
    }
  return Moments{static_cast<float>(n), mean, m2};
}

// Forward, row in registers (NV float4 per thread).
template <int NV>
__global__ void __launch_bounds__(kTopkThreads) stat_topk_huber_vec_kernel(const float* x, float* out, int d, float Q,
                                                                           float delta) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float2 s_ms;
  const size_t row = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + row * static_cast<size_t>(d));
  float4* orow = reinterpret_cast<float4*>(out + row * static_cast<size_t>(d));
  const int nvec = d >> 2;
  float e[4 * NV];
  int ne = 0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      const float4 v = __ldcs(xr + idx);
      e[4 * j] = v.x;
      e[4 * j + 1] = v.y;
      e[4 * j + 2] = v.z;
      e[4 * j + 3] = v.w;
      ne = 4 * j + 4;
    }
  }
  const float2 ms = block_mean_std(thread_moments(e, ne), s_warp, &s_ms);
  const float theta = fmaf(ms.y, Q, ms.x);
  const float hinv = delta > 0.f ? 0.5f / delta : 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec)
      __stcs(orow + idx, make_float4(huber_ramp(e[4 * j] - theta, delta, hinv), huber_ramp(e[4 * j + 1] - theta, delta, hinv),
                                     huber_ramp(e[4 * j + 2] - theta, delta, hinv),
                                     huber_ramp(e[4 * j + 3] - theta, delta, hinv)));
  }
}

// Forward, any d and alignment (two passes, then the output pass).
__global__ void __launch_bounds__(kTopkThreads) stat_topk_huber_generic_kernel(const float* x, float* out, int d,
                                                                               float Q, float delta) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float2 s_ms;
  const size_t row = blockIdx.x;
  const float* xr = x + row * static_cast<size_t>(d);
  float* orow = out + row * static_cast<size_t>(d);
  const float shift = threadIdx.x < d ? xr[threadIdx.x] : 0.f;
  float cnt = 0.f, acc = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    acc += xr[i] - shift;
    cnt += 1.f;
  }
  const float mean = cnt > 0.f ? shift + acc / cnt : 0.f;
  float m2 = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    const float a = xr[i] - mean;
    m2 += a * a;
  }
  const float2 ms = block_mean_std(Moments{cnt, mean, m2}, s_warp, &s_ms);
  const float theta = fmaf(ms.y, Q, ms.x);
  const float hinv = delta > 0.f ? 0.5f / delta : 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) orow[i] = huber_ramp(xr[i] - theta, delta, hinv);
}

// Backward, x and the upstream gradient in registers (NV float4 each).
template <int NV>
__global__ void __launch_bounds__(kTopkThreads) stat_topk_huber_bwd_vec_kernel(const float* x, const float* g, float* gx,
                                                                               int d, float Q, float delta) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float2 s_ms;
  __shared__ float s_part[kTopkWarps];
  const size_t row = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + row * static_cast<size_t>(d));
  const float4* gr = reinterpret_cast<const float4*>(g + row * static_cast<size_t>(d));
  float4* orow = reinterpret_cast<float4*>(gx + row * static_cast<size_t>(d));
  const int nvec = d >> 2;
  float e[4 * NV], w[4 * NV];
  int ne = 0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      const float4 v = __ldcs(xr + idx);
      const float4 u = __ldcs(gr + idx);
      e[4 * j] = v.x;
      e[4 * j + 1] = v.y;
      e[4 * j + 2] = v.z;
      e[4 * j + 3] = v.w;
      w[4 * j] = u.x;
      w[4 * j + 1] = u.y;
      w[4 * j + 2] = u.z;
      w[4 * j + 3] = u.w;
      ne = 4 * j + 4;
    }
  }
  const float2 ms = block_mean_std(thread_moments(e, ne), s_warp, &s_ms);
  const float theta = fmaf(ms.y, Q, ms.x);
  const float inv = delta > 0.f ? 1.f / delta : 0.f;
  float wsum = 0.f;
#pragma unroll
  for (int i = 0; i < 4 * NV; ++i)
    if (i < ne) {
      w[i] *= huber_slope(e[i] - theta, delta, inv);
      wsum += w[i];
    }
  const float W = block_sum(wsum, s_part);
  const float dn = static_cast<float>(d);
  const float a = W / dn;
  const float b = ms.y > 0.f ? W * Q / (dn * ms.y) : 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int idx = threadIdx.x + j * kTopkThreads;
    if (idx < nvec) {
      float r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) r[u] = w[4 * j + u] - fmaf(b, e[4 * j + u] - ms.x, a);
      __stcs(orow + idx, make_float4(r[0], r[1], r[2], r[3]));
    }
  }
}

// Backward, any d and alignment: moments, then W, then the output pass.
__global__ void __launch_bounds__(kTopkThreads) stat_topk_huber_bwd_generic_kernel(const float* x, const float* g,
                                                                                   float* gx, int d, float Q,
                                                                                   float delta) {
  __shared__ Moments s_warp[kTopkWarps];
  __shared__ float2 s_ms;
  __shared__ float s_part[kTopkWarps];
  const size_t row = blockIdx.x;
  const float* xr = x + row * static_cast<size_t>(d);
  const float* gr = g + row * static_cast<size_t>(d);
  float* orow = gx + row * static_cast<size_t>(d);
  const float shift = threadIdx.x < d ? xr[threadIdx.x] : 0.f;
  float cnt = 0.f, acc = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    acc += xr[i] - shift;
    cnt += 1.f;
  }
  const float mean = cnt > 0.f ? shift + acc / cnt : 0.f;
  float m2 = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    const float a = xr[i] - mean;
    m2 += a * a;
  }
  const float2 ms = block_mean_std(Moments{cnt, mean, m2}, s_warp, &s_ms);
  const float theta = fmaf(ms.y, Q, ms.x);
  const float inv = delta > 0.f ? 1.f / delta : 0.f;
  float wsum = 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) wsum += gr[i] * huber_slope(xr[i] - theta, delta, inv);
  const float W = block_sum(wsum, s_part);
  const float dn = static_cast<float>(d);
  const float a = W / dn;
  const float b = ms.y > 0.f ? W * Q / (dn * ms.y) : 0.f;
  for (int i = threadIdx.x; i < d; i += kTopkThreads) {
    const float xi = xr[i];
    const float wi = gr[i] * huber_slope(xi - theta, delta, inv);
    orow[i] = wi - fmaf(b, xi - ms.x, a);
  }
}

cudaError_t launch_stat_topk_huber(const float* x, float* out, int rows, int d, float Q, float delta,
                                   cudaStream_t stream) {
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15u) == 0;
  const int nvec = d / 4;
  const dim3 grid(static_cast<unsigned>(rows));
  if (aligned && d % 4 == 0 && nvec <= 4 * kTopkThreads) {
    const int per_thread = (nvec + kTopkThreads - 1) / kTopkThreads;
    if (per_thread <= 1)
      stat_topk_huber_vec_kernel<1><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q, delta);
    else if (per_thread <= 2)
      stat_topk_huber_vec_kernel<2><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q, delta);
    else
      stat_topk_huber_vec_kernel<4><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q, delta);
  } else {
    stat_topk_huber_generic_kernel<<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q, delta);
  }
  return cudaGetLastError();
}

cudaError_t launch_stat_topk_huber_backward(const float* x, const float* g, float* gx, int rows, int d, float Q,
                                            float delta, cudaStream_t stream) {
  const bool aligned =
      ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(g) | reinterpret_cast<uintptr_t>(gx)) & 15u) == 0;
  const int nvec = d / 4;
  const dim3 grid(static_cast<unsigned>(rows));
  if (aligned && d % 4 == 0 && nvec <= 4 * kTopkThreads) {
    const int per_thread = (nvec + kTopkThreads - 1) / kTopkThreads;
    if (per_thread <= 1)
      stat_topk_huber_bwd_vec_kernel<1><<<grid, kTopkThreads, 0, stream>>>(x, g, gx, d, Q, delta);
    else if (per_thread <= 2)
      stat_topk_huber_bwd_vec_kernel<2><<<grid, kTopkThreads, 0, stream>>>(x, g, gx, d, Q, delta);
    else
      stat_topk_huber_bwd_vec_kernel<4><<<grid, kTopkThreads, 0, stream>>>(x, g, gx, d, Q, delta);
  } else {
    stat_topk_huber_bwd_generic_kernel<<<grid, kTopkThreads, 0, stream>>>(x, g, gx, d, Q, delta);
  }
  return cudaGetLastError();
}

cudaError_t launch_stat_topk(const float* x, float* out, int rows, int d, float Q, cudaStream_t stream) {
  const bool aligned = ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15u) == 0;
  const int nvec = d / 4;
  const dim3 grid(static_cast<unsigned>(rows));
  if (aligned && d % 4 == 0 && nvec <= 8 * kTopkThreads) {
    const int per_thread = (nvec + kTopkThreads - 1) / kTopkThreads;
    if (per_thread <= 1)
      stat_topk_vec_kernel<1><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q);
    else if (per_thread <= 2)
      stat_topk_vec_kernel<2><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q);
    else if (per_thread <= 4)
      stat_topk_vec_kernel<4><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q);
    else
      stat_topk_vec_kernel<8><<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q);
  } else {
    stat_topk_generic_kernel<<<grid, kTopkThreads, 0, stream>>>(x, out, d, Q);
  }
  return cudaGetLastError();
}

}  // namespace spark
