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
#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;

__device__ __forceinline__ float block_theta(Moments m, float Q, Moments* s_warp, float* s_theta) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  m = warp_merge_moments(m);
  if (lane == 0) s_warp[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    Moments a = s_warp[0];
#pragma unroll
    for (int w = 1; w < kTopkWarps; ++w) a = merge_moments(a, s_warp[w]);
    const float sd = a.n > 0.f ? sqrtf(fmaxf(a.m2, 0.f) / a.n) : 0.f;
    *s_theta = fmaf(sd, Q, a.mean);
  }
  __syncthreads();
  return *s_theta;
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
