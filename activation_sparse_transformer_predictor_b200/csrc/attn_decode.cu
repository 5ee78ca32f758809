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
//           of lanes reads the K1 part in 16-byte chunks (all of the CTA's keys
//           in flight at once, issued together with the query chunks) and
//           reduces with shuffles.
//  stats    the CTA's (count, mean, M2, max), two passes over shared memory,
//           pushed into every CTA's inbox; one cluster barrier; every thread
//           merges the CS records in rank order, so all derive the same bits of
//           theta and of the score maximum M.
//  gather   each warp takes its own blocks of 32 keys, lists their selected keys
//           and, for a batch of them at a time, loads the K2 part and the value
//           row together: a = <K2[j], q[r:]>, w = exp(s_j - M),
//           f = w softplus(a), numerator += f V[j], normaliser += w.
//  reduce   the CTA sums its warps' partials in warp order and pushes column c
//           to the inbox of CTA c / ceil(d_head / CS); one cluster barrier; each
//           CTA sums its columns over the cluster in rank order, divides by the
//           summed normaliser and stores bf16.  No atomics: bit-reproducible.
// Remote shared memory is only ever written (st.shared::cluster) and only read
// locally after a barrier; the first remote store waits on a barrier phase that
// every CTA arrived at on entry, so no CTA writes into one that has not started.
#include <cstdlib>

#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

#ifdef SPARK_DEBUG
// bounds-check violations of this file's kernels (see SPARK_CHECK)
static __device__ unsigned g_bounds_violations;
#endif

namespace {

constexpr int kAThreads = 256;
constexpr int kAWarps = kAThreads / 32;
constexpr int kMaxDHead = 256;           // 32 chunks of 16 bytes per key row
constexpr int kKeyBatch = 16;            // key-steps in flight per lane in the score loop
constexpr int kGather = 8;               // selected keys in flight per warp in the gather

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

__device__ __forceinline__ void cluster_arrive_relaxed_a() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait_a() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// store v into the same offset of CTA `rank`'s shared memory
__device__ __forceinline__ void st_dsmem(float* p, unsigned rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
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
  size_t ss, lists, red, redz, in_stats, in_part, in_z, total;
  int seg;  // list capacity of one warp: its blocks of 32 keys
  __host__ __device__ ALayout(int kpc) {
    const int blocks = (kpc + 31) / 32;
    seg = (blocks + kAWarps - 1) / kAWarps * 32;
    size_t off = 0;
    ss = off;  // the CTA's scores
    off += static_cast<size_t>(kpc) * 4;
    lists = off;  // per-warp lists of selected keys [kAWarps][seg]
    off += static_cast<size_t>(kAWarps) * seg * 4;
    red = off;  // per-warp partial numerators [kAWarps][kMaxDHead]
    off += static_cast<size_t>(kAWarps) * kMaxDHead * 4;
    redz = off;  // per-warp partial normalisers
    off += kAWarps * 4;
    in_stats = off;  // inbox: (count, mean, M2, max) of every CTA of the cluster
    off += 16 * 4 * 4;
    in_part = off;  // inbox: [CS][ceil(d_head / CS)] column partials
    off += (kMaxDHead + 16) * 4;
    in_z = off;  // inbox: every CTA's normaliser
    off += 16 * 4;
    total = off;
  }
};

// Two CTAs per SM (at most 128 registers a thread): a GPU with fewer than
// sixteen free SMs in some of its GPCs still holds one 16-CTA cluster per head
// of an 8-head call resident at once, instead of running the last one as a
// second wave.
template <int CS>
__global__ void __launch_bounds__(kAThreads, 2) attn_decode_kernel(const AttnParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  // every CTA of the cluster has started once this phase completes
  cluster_arrive_relaxed_a();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned rank = cluster_rank_a();
  const int h = blockIdx.x / CS;
  const int g = h / p.group;
  const ALayout L(p.kpc);
  float* ss = reinterpret_cast<float*>(smem + L.ss);
  int* list = reinterpret_cast<int*>(smem + L.lists) + warp * L.seg;
  float* red = reinterpret_cast<float*>(smem + L.red);
  float* redz = reinterpret_cast<float*>(smem + L.redz);
  float* in_stats = reinterpret_cast<float*>(smem + L.in_stats);
  float* in_part = reinterpret_cast<float*>(smem + L.in_part);
  float* in_z = reinterpret_cast<float*>(smem + L.in_z);
  const int D = p.d_head;
  const int j0 = static_cast<int>(rank) * p.kpc;
  const int nk = max(0, min(p.kpc, p.n_ctx - j0));
  const uint16_t* Kg = p.K + static_cast<size_t>(g) * p.n_ctx * D;
  const uint16_t* Vg = p.V + static_cast<size_t>(g) * p.n_ctx * D;
  const uint16_t* qh = p.q + static_cast<size_t>(h) * D;

  // ---------------------------------------------------------------- scores
  // a key's K1 part is cpk 16-byte chunks, read by a group of lpk lanes; a warp
  // covers 32 / lpk keys per step and keeps kKeyBatch steps in flight
  const int cpk = p.r / 8;
  int lpk = 1;
  while (lpk < cpk) lpk <<= 1;
  const int kps = 32 / lpk;
  const int cc = lane % lpk, ko = lane / lpk;
  const bool cok = cc < cpk;
  const int cpk2 = (D - p.r) / 8;
  const uint4 qv = cok ? ldg_ro(qh + cc * 8) : make_uint4(0, 0, 0, 0);
  const uint4 q2 = lane < cpk2 ? ldg_ro(qh + p.r + lane * 8) : make_uint4(0, 0, 0, 0);
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
  cluster_wait_a();

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
    m2 = __shfl_sync(0xffffffffu, warp_sum(m2), 0);
    if (lane < CS) {
      float* slot = in_stats + rank * 4;
      st_dsmem(slot + 0, lane, static_cast<float>(nk));
      st_dsmem(slot + 1, lane, mean);
      st_dsmem(slot + 2, lane, m2);
      st_dsmem(slot + 3, lane, mx);
    }
  }
  cluster_sync_a();
  // the cluster's records merged by every warp: lane l < CS holds record l and
  // xor-butterflies combine them; a butterfly adds the same pairs in every lane
  // (addition commutes), so every thread of every CTA derives the same bits of
  // theta and of the score maximum M
  float theta, smax;
  {
    const bool own = lane < CS;
    const float n = own ? in_stats[lane * 4 + 0] : 0.f;
    const float mu = own ? in_stats[lane * 4 + 1] : 0.f;
    const float m2 = own ? in_stats[lane * 4 + 2] : 0.f;
    smax = own ? in_stats[lane * 4 + 3] : -__int_as_float(0x7f800000);
    float N = n, sx = n * mu;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      N += __shfl_xor_sync(0xffffffffu, N, off);
      sx += __shfl_xor_sync(0xffffffffu, sx, off);
      smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, off));
    }
    const float mean = sx / fmaxf(N, 1.f);
    const float d = mu - mean;
    float M2 = m2 + n * d * d;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M2 += __shfl_xor_sync(0xffffffffu, M2, off);
    theta = p.select_all ? -__int_as_float(0x7f800000) : fmaf(sqrtf(fmaxf(M2, 0.f) / fmaxf(N, 1.f)), p.Q, mean);
  }
  if (rank == 0 && tid == 0 && p.theta_out != nullptr) p.theta_out[h] = theta;
  if (p.s_out != nullptr || p.active_out != nullptr)
    for (int i = tid; i < nk; i += kAThreads) {
      if (p.s_out != nullptr) p.s_out[static_cast<size_t>(h) * p.n_ctx + j0 + i] = ss[i];
      if (p.active_out != nullptr) p.active_out[static_cast<size_t>(h) * p.n_ctx + j0 + i] = ss[i] > theta ? 1 : 0;
    }

  // ---------------------------------------------------------------- gather
  // warp w lists the selected keys of its blocks w, w + 8, ... in ascending order
  int cnt = 0;
  for (int b = warp * 32; b < nk; b += kAWarps * 32) {
    const int i = b + lane;
    const bool act = i < nk && ss[i] > theta;
    const unsigned ball = __ballot_sync(0xffffffffu, act);
    const int slot = cnt + __popc(ball & ((1u << lane) - 1u));
    if (act && SPARK_CHECK(slot < L.seg)) list[slot] = i;
    cnt += __popc(ball);
  }
  __syncwarp();
  // K2 part (lanes < cpk2) and value row (lanes < cpr) of kGather keys in flight
  const int cpr = D / 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float zw = 0.f;
  for (int jb = 0; jb < cnt; jb += kGather) {
    uint4 kv[kGather], vv[kGather];
    int idx[kGather];
#pragma unroll
    for (int u = 0; u < kGather; ++u) {
      idx[u] = jb + u < cnt ? list[jb + u] : -1;
      if (idx[u] >= 0 && !SPARK_CHECK(idx[u] < nk && j0 + idx[u] < p.n_ctx)) idx[u] = -1;
      const size_t row = static_cast<size_t>(j0 + max(idx[u], 0)) * D;
      kv[u] = (idx[u] >= 0 && lane < cpk2) ? ldg_ro(Kg + row + p.r + lane * 8) : make_uint4(0, 0, 0, 0);
      vv[u] = (idx[u] >= 0 && lane < cpr) ? ldg_ro(Vg + row + lane * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kGather; ++u) {
      // every lane scales its value chunk by f: the sum is broadcast from lane 0
      const float a = __shfl_sync(0xffffffffu, warp_sum(dot8_bf16(kv[u], q2, 0.f)), 0);
      if (idx[u] >= 0) {
        const float w = __expf(ss[idx[u]] - smax);
        const float f = w * softplus_f(a);
        zw += w;
        const float2 v0 = bf16x2_to_float2(vv[u].x), v1 = bf16x2_to_float2(vv[u].y);
        const float2 v2 = bf16x2_to_float2(vv[u].z), v3 = bf16x2_to_float2(vv[u].w);
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
  if (lane == 0) redz[warp] = zw;
  __syncthreads();

  // ---------------------------------------------------------------- reduce over the cluster
  // column c goes to CTA c / cw, slot (rank, c % cw); the normaliser to every CTA
  const int cw = (D + CS - 1) / CS;
  for (int col = tid; col < D; col += kAThreads) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) sum += red[w * kMaxDHead + col];
    st_dsmem(in_part + rank * cw + col % cw, static_cast<unsigned>(col / cw), sum);
  }
  if (tid < CS) {
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < kAWarps; ++w) z += redz[w];
    st_dsmem(in_z + rank, static_cast<unsigned>(tid), z);
  }
  cluster_sync_a();
  const int col = static_cast<int>(rank) * cw + tid;
  if (tid < cw && col < D) {
    float num = 0.f, z = 0.f;
#pragma unroll
    for (int src = 0; src < CS; ++src) {
      num += in_part[src * cw + tid];
      z += in_z[src];
    }
    const __nv_bfloat16 b = __float2bfloat16_rn(z > 0.f ? num / z : 0.f);
    p.out[static_cast<size_t>(h) * D + col] = *reinterpret_cast<const uint16_t*>(&b);
  }
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
  const size_t smem = ALayout(p.kpc).total;
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


// ---------------------------------------------------------------- debug builds
unsigned take_bounds_violations_attention(bool clear) {
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
