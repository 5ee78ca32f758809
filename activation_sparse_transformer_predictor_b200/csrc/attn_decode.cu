// attn_decode.cu -- Spark Attention for one decoding position.
//
// Spark Transformer notes, 关键设计 / "Spark Attention" and "Statistical Top-k":
// the key vectors are split like the FFN's K into K1 (the first r dimensions,
// the predictor) and K2 (the rest); each query attends to at most k_attn keys
// chosen by statistical top-k on the predictor scores; sigma_1 = softmax and
// sigma_2 = softplus.  For query head h and its key/value head g:
//   s_j   = scale * <K1[g][j], q[h][:r]>                         (j < n_ctx)
//   theta = mean(s) + std(s) Q(1 - k_attn / n_ctx)   (every key when k_attn >= n_ctx)
//   out[h] = sum_{s_j > theta} softmax_j(s) softplus(<K2[g][j], q[h][r:]>) V[g][j]
// with the softmax over the selected keys.
//
// One thread-block cluster per query head (CS CTAs, distributed shared memory),
// one launch, no global exchange: every dependency stays inside the cluster.
//  scores   CTA q of the cluster scores keys [q*KPC, (q+1)*KPC): per key, a group
//           of lanes reads the K1 part in 16-byte chunks (eight keys in flight
//           per lane) and reduces with shuffles.
//  stats    the CTA's (count, mean, M2, max), two passes over shared memory;
//           cluster barrier; every CTA merges the CS records in rank order, so
//           all derive the same bits of theta and of the score maximum M.
//  gather   the selected keys of the CTA: a = <K2[j], q[r:]> (one warp per key),
//           w = exp(s_j - M), f = w softplus(a); the CTA's partial numerator
//           sum f_j V[j] (thread groups over keys, fixed-order reduction) and
//           partial normaliser sum w_j.
//  reduce   cluster barrier; CTA q sums its share of the columns over the
//           cluster's CTAs in rank order, divides by the summed normaliser and
//           stores bf16.  No atomics: bit-reproducible.
#include <cstdlib>

#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {
namespace {

constexpr int kAThreads = 256;
constexpr int kAWarps = kAThreads / 32;
constexpr int kMaxDHead = 256;           // 32 chunks of 16 bytes per key row
constexpr int kKeyBatch = 8;             // key-steps in flight per lane in the score loop

struct AttnParams {
  const uint16_t* q;  // bf16 [n_heads][d_head]
  const uint16_t* K;  // bf16 [n_kv_heads][n_ctx][d_head]
  const uint16_t* V;  // bf16 [n_kv_heads][n_ctx][d_head]
  uint16_t* out;      // bf16 [n_heads][d_head]
  int n_heads, group, n_ctx, d_head, r, kpc;
  float scale, Q;
  bool select_all;    // k_attn >= n_ctx
  float* s_out;       // optional [n_heads][n_ctx]
  float* theta_out;   // optional [n_heads]
  unsigned char* active_out;  // optional [n_heads][n_ctx]
};

__device__ __forceinline__ unsigned cluster_rank_a() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_a() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ float ld_dsmem(const float* p, unsigned rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ uint4 ldg_ro(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// softplus(a) = log(1 + e^a) without overflow
__device__ __forceinline__ float softplus_f(float a) {
  return a > 0.f ? a + log1pf(__expf(-a)) : log1pf(__expf(a));
}

// Shared-memory layout (dynamic part).
struct ALayout {
  size_t qs, ss, act_i, act_f, act_w, red, part, stats, misc, total;
  __host__ __device__ ALayout(int d_head, int kpc) {
    size_t off = 0;
    qs = off;
    off += static_cast<size_t>(kMaxDHead) * 2;
    ss = off;
    off += static_cast<size_t>(kpc) * 4;
    act_i = off;
    off += static_cast<size_t>(kpc) * 4;
    act_f = off;
    off += static_cast<size_t>(kpc) * 4;
    act_w = off;
    off += static_cast<size_t>(kpc) * 4;
    red = off;  // per-group partial numerators [kAWarps][kMaxDHead]
    off += static_cast<size_t>(kAWarps) * kMaxDHead * 4;
    part = off;  // this CTA's partial numerator, read by the cluster
    off += static_cast<size_t>(kMaxDHead) * 4;
    stats = off;  // (count, mean, M2, max, normaliser), read by the cluster
    off += 32;
    misc = off;
    off += 64;
    total = off;
    (void)d_head;
  }
};

template <int CS>
__global__ void __launch_bounds__(kAThreads, 1) attn_decode_kernel(const AttnParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned rank = cluster_rank_a();
  const int h = blockIdx.x / CS;
  const int g = h / p.group;
  const ALayout L(p.d_head, p.kpc);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs);
  float* ss = reinterpret_cast<float*>(smem + L.ss);
  int* act_i = reinterpret_cast<int*>(smem + L.act_i);
  float* act_f = reinterpret_cast<float*>(smem + L.act_f);
  float* act_w = reinterpret_cast<float*>(smem + L.act_w);
  float* red = reinterpret_cast<float*>(smem + L.red);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* stats = reinterpret_cast<float*>(smem + L.stats);
  float* misc_f = reinterpret_cast<float*>(smem + L.misc);
  int* misc_i = reinterpret_cast<int*>(smem + L.misc) + 8;
  const int D = p.d_head;
  const int j0 = static_cast<int>(rank) * p.kpc;
  const int nk = max(0, min(p.kpc, p.n_ctx - j0));
  const uint16_t* Kg = p.K + static_cast<size_t>(g) * p.n_ctx * D;
  const uint16_t* Vg = p.V + static_cast<size_t>(g) * p.n_ctx * D;

  for (int ch = tid; ch < D / 8; ch += kAThreads)
    *reinterpret_cast<uint4*>(qs + ch * 8) = ldg_ro(p.q + static_cast<size_t>(h) * D + ch * 8);
  __syncthreads();

  // ---------------------------------------------------------------- scores
  // a key's K1 part is cpk 16-byte chunks, read by a group of lpk lanes; a warp
  // covers 32 / lpk keys per step and keeps kKeyBatch steps in flight
  const int cpk = p.r / 8;
  int lpk = 1;
  while (lpk < cpk) lpk <<= 1;
  const int kps = 32 / lpk;
  const int cc = lane % lpk, ko = lane / lpk;
  const bool cok = cc < cpk;
  const uint4 qv = cok ? lds128(qs + cc * 8) : make_uint4(0, 0, 0, 0);
  for (int base = warp * kps * kKeyBatch; base < nk; base += kAWarps * kps * kKeyBatch) {
    uint4 kv[kKeyBatch];
#pragma unroll
    for (int u = 0; u < kKeyBatch; ++u) {
      const int j = base + u * kps + ko;
      kv[u] = (cok && j < nk) ? ldg_ro(Kg + static_cast<size_t>(j0 + j) * D + cc * 8) : make_uint4(0, 0, 0, 0);
    }
    float sv[kKeyBatch];
#pragma unroll
    for (int u = 0; u < kKeyBatch; ++u) sv[u] = dot8_bf16(kv[u], qv, 0.f);
    for (int off = lpk / 2; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < kKeyBatch; ++u) sv[u] += __shfl_xor_sync(0xffffffffu, sv[u], off);
    if (cc == 0)
#pragma unroll
      for (int u = 0; u < kKeyBatch; ++u) {
        const int j = base + u * kps + ko;
        if (j < nk) ss[j] = sv[u] * p.scale;
      }
  }
  __syncthreads();

  // ---------------------------------------------------------------- statistics
  if (warp == 0) {
    float sum = 0.f, mx = -__int_as_float(0x7f800000);
    for (int i = lane; i < nk; i += 32) {
      sum += ss[i];
      mx = fmaxf(mx, ss[i]);
    }
    sum = __shfl_sync(0xffffffffu, warp_sum(sum), 0);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float mean = nk > 0 ? sum / static_cast<float>(nk) : 0.f;
    float m2 = 0.f;
    for (int i = lane; i < nk; i += 32) {
      const float d = ss[i] - mean;
      m2 = fmaf(d, d, m2);
    }
    m2 = warp_sum(m2);
    if (lane == 0) {
      stats[0] = static_cast<float>(nk);
      stats[1] = mean;
      stats[2] = m2;
      stats[3] = mx;
    }
  }
  cluster_sync_a();
  if (tid == 0) {
    // the cluster's records merged in rank order: the same bits in every CTA
    float n[CS], mu[CS], m2[CS];
    float N = 0.f, sx = 0.f, mx = -__int_as_float(0x7f800000);
#pragma unroll
    for (int src = 0; src < CS; ++src) {
      n[src] = ld_dsmem(stats + 0, src);
      mu[src] = ld_dsmem(stats + 1, src);
      m2[src] = ld_dsmem(stats + 2, src);
      mx = fmaxf(mx, ld_dsmem(stats + 3, src));
    }
#pragma unroll
    for (int src = 0; src < CS; ++src) {
      N += n[src];
      sx = fmaf(n[src], mu[src], sx);
    }
    const float mean = sx / fmaxf(N, 1.f);
    float M2 = 0.f;
#pragma unroll
    for (int src = 0; src < CS; ++src) {
      const float d = mu[src] - mean;
      M2 += m2[src] + n[src] * d * d;
    }
    misc_f[0] = p.select_all ? -__int_as_float(0x7f800000)
                             : fmaf(sqrtf(fmaxf(M2, 0.f) / fmaxf(N, 1.f)), p.Q, mean);
    misc_f[1] = mx;
  }
  __syncthreads();
  const float theta = misc_f[0];
  const float smax = misc_f[1];
  if (rank == 0 && tid == 0 && p.theta_out != nullptr) p.theta_out[h] = theta;
  for (int i = tid; i < nk; i += kAThreads) {
    if (p.s_out != nullptr) p.s_out[static_cast<size_t>(h) * p.n_ctx + j0 + i] = ss[i];
    if (p.active_out != nullptr) p.active_out[static_cast<size_t>(h) * p.n_ctx + j0 + i] = ss[i] > theta ? 1 : 0;
  }

  // ---------------------------------------------------------------- gather
  // the selected keys of this CTA, ascending
  if (warp == 0) {
    int cnt = 0;
    for (int base = 0; base < nk; base += 32) {
      const int i = base + lane;
      const bool act = i < nk && ss[i] > theta;
      const unsigned ball = __ballot_sync(0xffffffffu, act);
      if (act) act_i[cnt + __popc(ball & ((1u << lane) - 1u))] = i;
      cnt += __popc(ball);
    }
    if (lane == 0) misc_i[0] = cnt;
  }
  __syncthreads();
  const int nact = misc_i[0];
  // f_j = exp(s_j - M) softplus(<K2[j], q[r:]>): one warp per key, four keys'
  // loads in flight before the arithmetic
  const int cpk2 = (D - p.r) / 8;
  constexpr int kKB = 4;
  const uint4 q2 = lane < cpk2 ? lds128(qs + p.r + lane * 8) : make_uint4(0, 0, 0, 0);
  for (int jb = warp * kKB; jb < nact; jb += kAWarps * kKB) {
    uint4 kv[kKB];
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      const int jj = jb + u;
      kv[u] = (jj < nact && lane < cpk2)
                  ? ldg_ro(Kg + static_cast<size_t>(j0 + act_i[jj]) * D + p.r + lane * 8)
                  : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      const float a = warp_sum(dot8_bf16(kv[u], q2, 0.f));
      const int jj = jb + u;
      if (lane == 0 && jj < nact) {
        const float w = __expf(ss[act_i[jj]] - smax);
        act_w[jj] = w;
        act_f[jj] = w * softplus_f(a);
      }
    }
  }
  __syncthreads();
  // partial numerator: warp w sums the keys w, w + 8, ... over column chunk `lane`
  const int cpr = D / 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  constexpr int kVB = 8;
  for (int jb = warp; jb < nact; jb += kAWarps * kVB) {
    uint4 v[kVB];
#pragma unroll
    for (int u = 0; u < kVB; ++u) {
      const int jj = jb + u * kAWarps;
      v[u] = (jj < nact && lane < cpr) ? ldg_ro(Vg + static_cast<size_t>(j0 + act_i[jj]) * D + lane * 8)
                                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kVB; ++u) {
      const int jj = jb + u * kAWarps;
      if (jj < nact) {
        const float f = act_f[jj];
        const float2 v0 = bf16x2_to_float2(v[u].x), v1 = bf16x2_to_float2(v[u].y);
        const float2 v2 = bf16x2_to_float2(v[u].z), v3 = bf16x2_to_float2(v[u].w);
        acc[0] = fmaf(f, v0.x, acc[0]);
        acc[1] = fmaf(f, v0.y, acc[1]);
        acc[2] = fmaf(f, v1.x, acc[2]);
        acc[3] = fmaf(f, v1.y, acc[3]);
        acc[4] = fmaf(f, v2.x, acc[4]);
        acc[5] = fmaf(f, v2.y, acc[5]);
        acc[6] = fmaf(f, v3.x, acc[6]);
        acc[7] = fmaf(f, v3.y, acc[7]);
      }
    }
  }
  if (lane < cpr)
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp * kMaxDHead + lane * 8 + e] = acc[e];
  // partial normaliser, fixed order
  if (warp == 0) {
    float z = 0.f;
    for (int jj = lane; jj < nact; jj += 32) z += act_w[jj];
    z = warp_sum(z);
    if (lane == 0) stats[4] = z;
  }
  __syncthreads();
  for (int col = tid; col < D; col += kAThreads) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) sum += red[w * kMaxDHead + col];
    part[col] = sum;
  }

  // ---------------------------------------------------------------- reduce over the cluster
  cluster_sync_a();
  const int cw = (D + CS - 1) / CS;
  const int col = static_cast<int>(rank) * cw + tid;
  if (tid < cw && col < D) {
    float num = 0.f, z = 0.f;
#pragma unroll
    for (int src = 0; src < CS; ++src) {
      num += ld_dsmem(part + col, static_cast<unsigned>(src));
      z += ld_dsmem(stats + 4, static_cast<unsigned>(src));
    }
    const __nv_bfloat16 b = __float2bfloat16_rn(z > 0.f ? num / z : 0.f);
    p.out[static_cast<size_t>(h) * D + col] = *reinterpret_cast<const uint16_t*>(&b);
  }
  // no CTA leaves while another may still read its shared memory
  cluster_sync_a();
}

}  // namespace

cudaError_t launch_attn_decode(const AttnArgs& a, int num_sms, cudaStream_t stream) {
  // clusters of 16 CTAs (a non-portable size) when the GPU runs them, else 8
  static int cs16_ok[64] = {};  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (cs16_ok[dev] == 0) {
    e = cudaFuncSetAttribute(attn_decode_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    cs16_ok[dev] = e == cudaSuccess ? 1 : 2;
    cudaGetLastError();
  }
  int cs = (cs16_ok[dev] == 1 && a.n_ctx >= 16 * 32) ? 16 : 8;
  // SPARK_ATTN_CLUSTER=8 (test / tuning knob) forces the portable cluster size
  const char* env = std::getenv("SPARK_ATTN_CLUSTER");
  if (env != nullptr && std::atoi(env) == 8) cs = 8;
  AttnParams p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.K = static_cast<const uint16_t*>(a.K);
  p.V = static_cast<const uint16_t*>(a.V);
  p.out = static_cast<uint16_t*>(a.out);
  p.n_heads = a.n_heads;
  p.group = a.n_heads / a.n_kv_heads;
  p.n_ctx = a.n_ctx;
  p.d_head = a.d_head;
  p.r = a.r;
  p.kpc = (a.n_ctx + cs - 1) / cs;
  p.scale = a.scale;
  p.Q = a.Q;
  p.select_all = a.select_all;
  p.s_out = a.s_out;
  p.theta_out = a.theta_out;
  p.active_out = a.active_out;
  const size_t smem = ALayout(a.d_head, p.kpc).total;
  auto kern = cs == 16 ? attn_decode_kernel<16> : attn_decode_kernel<8>;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_heads * cs);
  cfg.blockDim = dim3(kAThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  (void)num_sms;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace spark
