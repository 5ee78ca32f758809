// ffn_decode_pg.cu -- Spark FFN forward for ONE token (decode) as two chained
// kernels, the score kernel P and the gather kernel G.
//
// Spark Transformer notes, 关键设计 / "Spark FFN" and "Statistical Top-k":
//   x = K1^T q[:r];  theta = mean(x) + std(x) Q(1 - k/d_ff);
//   out = V . (GELU(max(x - theta, 0)) (.) (K2^T q[r:])) over the neurons with x > theta.
//
// The one global dependency (theta needs every score) is the boundary between
// the two kernels, so neither kernel waits on another CTA's progress:
//
//  P  CTA c owns neurons [c*RPC, (c+1)*RPC).  Before anything else it bulk-copies
//     its whole K1 slice into shared memory.  Only then does it wait for the
//     work ahead of it on the stream (programmatic dependent launch): with
//     weight overlap on, P is launched while the previous call's G still runs,
//     so the K1 stream -- 80% of the layer's bytes -- overlaps the previous
//     call's tail.  After the wait: q[:r] into registers, x row by row (fp32
//     FMA), the slice's moments (mean, M2) and x to the workspace.
//  G  launched behind P (programmatic), in clusters of CS CTAs.  CTA c merges all
//     slices' moments in slice order (every CTA derives the same bits of theta),
//     compacts the active neurons of its SPC slices, reads their K2 rows
//     (a = K2.q[r:]) and V rows, and forms its partial output
//     sum_i GELU(x_i - theta) a_i V[i,:] (fp32).  The CS partials of a cluster are summed through distributed shared
//     memory in rank order; each cluster writes one partial; the last cluster to
//     arrive (one atomic counter, no waiting) sums the cluster partials in
//     cluster order and stores bf16.  Stack mode also adds the residual and forms
//     the next layer's q = bf16(RMSNorm(h)) there.  No data atomics: results are
//     bit-reproducible.
//
// Neither kernel spins on another CTA: P's only waits are on its own bulk
// copies (bounded), G's are cluster barriers, so no co-residency is assumed.
#include <map>
#include <mutex>
#include <utility>

#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {
namespace {


constexpr int kPWarps = 8;
constexpr int kPThreads = kPWarps * 32;
constexpr int kStageRows = 8;            // K1 rows per bulk copy / mbarrier
constexpr int kGWarps = 9;
constexpr int kGThreads = kGWarps * 32;  // one 16-byte output chunk per thread at d_model = 2304
constexpr int kMaxSlices = 256;          // moments merged by one warp, 8 per lane
constexpr int kMaxGChunks = 4;           // output columns per G thread in the final sum: d_model <= 9216
constexpr int kMaxClusters = 32;         // cluster partials summed by the last cluster in one batch

__host__ __device__ inline size_t pg_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct PgParams {
  const uint16_t* q;   // bf16 [d_model]
  const uint16_t* K1;  // bf16 [d_ff][r]
  const uint16_t* K2;  // bf16 [d_ff][d_model - r]
  const uint16_t* V;   // bf16 [d_ff][d_model]
  uint16_t* out;       // bf16 [d_model], may be nullptr in stack mode
  int d_model, r, d2, d_ff;
  int rpc;             // rows (neurons) per P CTA
  int rpg;             // rows per G CTA (a whole number of P slices)
  int n_slices, n_clusters;
  float Q;
  // workspace
  DeviceControl* ctl;
  float2* mom;       // [n_slices] (mean, M2) of each slice's scores
  float* xg;         // [d_ff] scores
  float* cpart;      // [n_clusters][d_model] cluster partial outputs
  unsigned* arrive;  // clusters that have written their partial (reset by the last one)
  // optional debug outputs
  float* x_out;
  float* theta_out;
  unsigned char* active_out;
  uint16_t* q_dbg;
  // stack mode (h_base != nullptr): h_out = h_base + bf16(out), q_next = bf16(RMSNorm(h_out))
  const float* h_base;
  float* h_out;
  uint16_t* q_next;
  float eps;
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Load from the shared memory of CTA `rank` of this cluster, at the offset of
// the local address `p`.
__device__ __forceinline__ float ld_dsmem_f32(const float* p, unsigned rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ unsigned ld_dsmem_u32(const unsigned* p, unsigned rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  unsigned v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ uint4 ldcg128(const void* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }

// Read-only 16-byte load (weights).  Not volatile, so that the compiler may
// hoist a row's loads ahead of the arithmetic that consumes them.
__device__ __forceinline__ uint4 ldg_ro128(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ int rows_in(int n0, int n, int d_ff) { return max(0, min(n, d_ff - n0)); }

__device__ __forceinline__ void bf16x8_to_float(uint4 w, float* f) {
  const float2 a = bf16x2_to_float2(w.x), b = bf16x2_to_float2(w.y);
  const float2 c = bf16x2_to_float2(w.z), d = bf16x2_to_float2(w.w);
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
  f[4] = c.x;
  f[5] = c.y;
  f[6] = d.x;
  f[7] = d.y;
}

// Shared-memory layout of P.
struct PLayout {
  size_t k1, qs, xs, bars, total;
  __host__ __device__ PLayout(int r, int rpc) {
    size_t off = 0;
    k1 = off;
    off += pg_align(static_cast<size_t>(rpc) * r * 2, 128);
    qs = off;
    off += pg_align(static_cast<size_t>(r) * 2, 128);
    xs = off;
    off += pg_align(static_cast<size_t>(rpc) * 4, 16);
    bars = off;
    off += pg_align(static_cast<size_t>(rpc / kStageRows) * 8, 16);
    total = off;
  }
};

// Shared-memory layout of G.
struct GLayout {
  size_t q2, mom, xs, act_i, act_h, bal_i, bal_h, part, red, misc, total;
  __host__ __device__ GLayout(int d_model, int r, int rpg, int n_slices) {
    size_t off = 0;
    q2 = off;
    off += pg_align(static_cast<size_t>(d_model - r) * 2, 128);
    mom = off;
    off += pg_align(static_cast<size_t>(n_slices) * 8, 16);
    xs = off;
    off += pg_align(static_cast<size_t>(rpg) * 4, 16);
    act_i = off;
    off += pg_align(static_cast<size_t>(rpg) * 4, 16);
    act_h = off;
    off += pg_align(static_cast<size_t>(rpg) * 4, 16);
    // a CTA's balanced share of its cluster's active rows is at most the
    // cluster's rows / CS + 1 <= rpg + 1
    bal_i = off;
    off += pg_align(static_cast<size_t>(rpg + 1) * 4, 16);
    bal_h = off;
    off += pg_align(static_cast<size_t>(rpg + 1) * 4, 16);
    part = off;
    off += pg_align(static_cast<size_t>(d_model) * 4, 16);
    red = off;
    off += 64;
    misc = off;
    off += 64;
    total = off;
  }
};

// Workspace layout (after the device control block).
struct PgWs {
  size_t mom, xg, cpart, qbuf, total;
  PgWs(int d_model, int d_ff, int n_slices, int n_clusters) {
    size_t off = sizeof(DeviceControl);
    mom = off;
    off += pg_align(static_cast<size_t>(n_slices) * 8, 256);
    xg = off;
    off += pg_align(static_cast<size_t>(d_ff) * 4, 256);
    cpart = off;
    off += pg_align(static_cast<size_t>(n_clusters) * d_model * 4, 256);
    qbuf = off;
    off += pg_align(static_cast<size_t>(d_model) * 2, 256);
    total = off;
  }
};

// ------------------------------------------------------------------------ P
// KCH: 16-byte chunks per lane of a K1 row (r <= 256 * KCH).
template <int KCH>
__global__ void __launch_bounds__(kPThreads, 1) decode_score_kernel(const PgParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const PLayout L(p.r, p.rpc);
  uint16_t* k1s = reinterpret_cast<uint16_t*>(smem + L.k1);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  const int n0 = c * p.rpc;
  const int nr = rows_in(n0, p.rpc, p.d_ff);
  const int nst = (nr + kStageRows - 1) / kStageRows;

  // The weights only: nothing that an earlier kernel on the stream may still be
  // writing is touched before griddep_wait().
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    for (int s = 0; s < nst; ++s) {
      const int rows = min(kStageRows, nr - s * kStageRows);
      const unsigned bytes = static_cast<unsigned>(rows) * p.r * 2;
      mbar_arrive_expect_tx(&bars[s], bytes);
      bulk_g2s(k1s + static_cast<size_t>(s) * kStageRows * p.r,
               p.K1 + static_cast<size_t>(n0 + s * kStageRows) * p.r, bytes, &bars[s]);
    }
  }
  griddep_wait();
  // G of this call may now be scheduled; it waits for this grid to complete.
  griddep_launch_dependents();
  const int nchunk = p.r / 8;
  for (int ch = tid; ch < nchunk; ch += kPThreads)
    *reinterpret_cast<uint4*>(qs + ch * 8) = ldcg128(p.q + ch * 8);
  __syncthreads();  // q staged; the barrier inits are visible

  // Warp w scores the stages w, w + 8, ...: the 8 rows of a stage together, so
  // that each lane runs 8 independent FMA chains; then one transposed butterfly
  // reduces the 8 row sums over the warp (9 shuffles instead of 8 x 5).
  bool ok = true;
  for (int s = warp; s < nst; s += kPWarps) {
    if (ok) ok = mbar_wait_bounded(&bars[s], 0, p.wait_limit_ns, p.ctl, 70);
    if (!ok) break;
    const uint16_t* kst = k1s + static_cast<size_t>(s) * kStageRows * p.r;
    float acc[kStageRows];
#pragma unroll
    for (int j = 0; j < kStageRows; ++j) acc[j] = 0.f;
#pragma unroll
    for (int m = 0; m < KCH; ++m) {
      const int ch = lane + 32 * m;
      if (ch < nchunk) {
        float qf[8];
        bf16x8_to_float(lds128(qs + ch * 8), qf);
        uint4 kv[kStageRows];
#pragma unroll
        for (int j = 0; j < kStageRows; ++j) kv[j] = lds128(kst + static_cast<size_t>(j) * p.r + ch * 8);
#pragma unroll
        for (int j = 0; j < kStageRows; ++j) {
          const float2 a = bf16x2_to_float2(kv[j].x), b = bf16x2_to_float2(kv[j].y);
          const float2 c2 = bf16x2_to_float2(kv[j].z), d = bf16x2_to_float2(kv[j].w);
          float t = acc[j];
          t = fmaf(a.x, qf[0], t);
          t = fmaf(a.y, qf[1], t);
          t = fmaf(b.x, qf[2], t);
          t = fmaf(b.y, qf[3], t);
          t = fmaf(c2.x, qf[4], t);
          t = fmaf(c2.y, qf[5], t);
          t = fmaf(d.x, qf[6], t);
          t = fmaf(d.y, qf[7], t);
          acc[j] = t;
        }
      }
    }
    // Transposed butterfly: after the xor-16, -8 and -4 steps lane l holds row
    // 4*b4 + 2*b3 + b2 (b = bits of l) summed over its lane group; xor-2 and
    // xor-1 finish the sum.  Rows past the end of a partial stage hold stale
    // shared memory; their sums are discarded.
    const bool hi16 = (lane & 16) != 0, hi8 = (lane & 8) != 0, hi4 = (lane & 4) != 0;
    float a4[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float send = hi16 ? acc[j] : acc[j + 4];
      const float keep = hi16 ? acc[j + 4] : acc[j];
      a4[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float a2[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float send = hi8 ? a4[j] : a4[j + 2];
      const float keep = hi8 ? a4[j + 2] : a4[j];
      a2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float a1;
    {
      const float send = hi4 ? a2[0] : a2[1];
      const float keep = hi4 ? a2[1] : a2[0];
      a1 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
    a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
    const int row = s * kStageRows + (hi16 ? 4 : 0) + (hi8 ? 2 : 0) + (hi4 ? 1 : 0);
    if ((lane & 3) == 0 && row < nr) xs[row] = a1;
  }
  if (!__syncthreads_and(ok)) {
    // a copy did not land in time (recorded); let those in flight finish before exit
    if (tid == 0)
      for (int s = 0; s < nst; ++s) mbar_wait_bounded(&bars[s], 0, p.wait_limit_ns, p.ctl, 71);
    return;
  }
  // moments of the slice, two passes over shared memory, fixed order
  if (warp == 0) {
    float sum = 0.f;
    for (int i = lane; i < nr; i += 32) sum += xs[i];
    sum = __shfl_sync(0xffffffffu, warp_sum(sum), 0);
    const float mean = nr > 0 ? sum / static_cast<float>(nr) : 0.f;
    float m2 = 0.f;
    for (int i = lane; i < nr; i += 32) {
      const float d = xs[i] - mean;
      m2 = fmaf(d, d, m2);
    }
    m2 = warp_sum(m2);
    if (lane == 0) p.mom[c] = make_float2(mean, m2);
  }
  for (int i = tid; i < nr; i += kPThreads) {
    p.xg[n0 + i] = xs[i];
    if (p.x_out != nullptr) p.x_out[n0 + i] = xs[i];
  }
  if (c == 0 && p.q_dbg != nullptr)
    for (int i = tid; i < p.d_model; i += kPThreads) p.q_dbg[i] = p.q[i];
}

// ------------------------------------------------------------------------ G
// CS: cluster size.  CPT: 16-byte output chunks per thread (d_model <= 2304 * CPT).
// KCH: 16-byte chunks per lane of a K2 row (d_model - r <= 256 * KCH).
template <int CS, int CPT, int KCH>
__global__ void __maxnreg__(168) decode_gather_kernel(const PgParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kVB = 16 / CPT;  // active rows whose V chunks are in flight at once
  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned rank = cluster_rank();
  const int cl = c / CS;
  const int D = p.d_model;
  const GLayout L(D, p.r, p.rpg, p.n_slices);
  uint16_t* q2s = reinterpret_cast<uint16_t*>(smem + L.q2);
  float2* moms = reinterpret_cast<float2*>(smem + L.mom);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  int* act_i = reinterpret_cast<int*>(smem + L.act_i);
  float* act_h = reinterpret_cast<float*>(smem + L.act_h);
  int* bal_i = reinterpret_cast<int*>(smem + L.bal_i);
  float* bal_h = reinterpret_cast<float*>(smem + L.bal_h);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* red = reinterpret_cast<float*>(smem + L.red);
  int* misc_i = reinterpret_cast<int*>(smem + L.misc);
  float* misc_f = reinterpret_cast<float*>(smem + L.misc) + 8;

  // The next call's P may now be scheduled (it streams weights, then waits for
  // this grid to complete); this grid waits for P of this call.
  griddep_launch_dependents();
  griddep_wait();

  const int n0 = c * p.rpg;
  const int nr = rows_in(n0, p.rpg, p.d_ff);
  for (int i = tid; i < p.n_slices; i += kGThreads) moms[i] = __ldcg(p.mom + i);
  for (int i = tid; i < nr; i += kGThreads) xs[i] = __ldcg(p.xg + n0 + i);
  for (int ch = tid; ch < p.d2 / 8; ch += kGThreads)
    *reinterpret_cast<uint4*>(q2s + ch * 8) = ldcg128(p.q + p.r + ch * 8);
  __syncthreads();

  // theta from the slice moments, merged in slice order (same bits in every CTA),
  // then the active neurons of this CTA's rows in ascending order
  if (warp == 0) {
    float2 h[kMaxSlices / 32];
    float nc[kMaxSlices / 32];
#pragma unroll
    for (int j = 0; j < kMaxSlices / 32; ++j) {
      const int s = lane + 32 * j;
      h[j] = s < p.n_slices ? moms[s] : make_float2(0.f, 0.f);
      nc[j] = s < p.n_slices ? static_cast<float>(rows_in(s * p.rpc, p.rpc, p.d_ff)) : 0.f;
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxSlices / 32; ++j) sum = fmaf(nc[j], h[j].x, sum);
    const float mean = __shfl_sync(0xffffffffu, warp_sum(sum), 0) / static_cast<float>(p.d_ff);
    float m2 = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxSlices / 32; ++j) {
      const float dm = h[j].x - mean;
      m2 += h[j].y + nc[j] * dm * dm;
    }
    m2 = warp_sum(m2);
    const float th =
        __shfl_sync(0xffffffffu, fmaf(sqrtf(fmaxf(m2, 0.f) / static_cast<float>(p.d_ff)), p.Q, mean), 0);
    int cnt = 0;
    for (int base = 0; base < nr; base += 32) {
      const int i = base + lane;
      const float x = i < nr ? xs[i] : 0.f;
      const bool act = i < nr && x > th;
      const unsigned ball = __ballot_sync(0xffffffffu, act);
      const int slot = cnt + __popc(ball & ((1u << lane) - 1u));
      if (act) {
        act_i[slot] = n0 + i;
        act_h[slot] = x;  // x for now; h = GELU(x - theta) a below
      }
      cnt += __popc(ball);
    }
    if (lane == 0) {
      misc_i[0] = cnt;
      misc_f[0] = th;
    }
  }
  __syncthreads();
  const float theta = misc_f[0];
  if (c == 0 && tid == 0 && p.theta_out != nullptr) p.theta_out[0] = theta;
  if (p.active_out != nullptr)
    for (int i = tid; i < nr; i += kGThreads) p.active_out[n0 + i] = xs[i] > theta ? 1 : 0;

  // Balance: the cluster's active rows, in rank order, are split into CS
  // contiguous near-equal shares, so that no CTA takes a second round of loads
  // while the others idle.  Entries come from the owners' shared memory.
  cluster_sync();
  int nact;
  {
    int pref[CS + 1];
    pref[0] = 0;
#pragma unroll
    for (int src = 0; src < CS; ++src)
      pref[src + 1] = pref[src] + static_cast<int>(ld_dsmem_u32(reinterpret_cast<const unsigned*>(misc_i), src));
    const int total = pref[CS];
    const int lo = static_cast<int>((static_cast<long long>(total) * rank) / CS);
    const int hi = static_cast<int>((static_cast<long long>(total) * (rank + 1)) / CS);
    nact = hi - lo;
    for (int j = tid; j < nact; j += kGThreads) {
      const int g = lo + j;
      int src = 0;
#pragma unroll
      for (int t = 1; t < CS; ++t) src += g >= pref[t] ? 1 : 0;
      const int li = g - pref[src];
      bal_i[j] = static_cast<int>(ld_dsmem_u32(reinterpret_cast<const unsigned*>(act_i + li), src));
      bal_h[j] = ld_dsmem_f32(act_h + li, src);
    }
  }
  __syncthreads();

  // partial output of these rows: thread t owns 16-byte chunks t, t + 288, ...
  const int nco = D / 8;
  float acc[CPT][8];
#pragma unroll
  for (int cp = 0; cp < CPT; ++cp)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[cp][e] = 0.f;
  for (int j0 = 0; j0 < nact; j0 += kVB) {
    // V chunks of up to kVB active rows in flight ...
    uint4 v[CPT][kVB];
#pragma unroll
    for (int u = 0; u < kVB; ++u)
#pragma unroll
      for (int cp = 0; cp < CPT; ++cp) {
        const int ch = tid + cp * kGThreads;
        v[cp][u] = (j0 + u < nact && ch < nco)
                       ? ldg_ro128(p.V + static_cast<size_t>(bal_i[j0 + u]) * D + ch * 8)
                       : make_uint4(0, 0, 0, 0);
      }
    if (j0 == 0) {
      // ... while the warps form h = GELU(x - theta) a, a = <K2[i,:], q[r:]>:
      // two rows per warp, all of both rows' loads issued before the arithmetic
      for (int j = warp; j < nact; j += 2 * kGWarps) {
        const int jb = j + kGWarps;
        const bool hasb = jb < nact;
        const uint16_t* ra = p.K2 + static_cast<size_t>(bal_i[j]) * p.d2;
        const uint16_t* rb = p.K2 + static_cast<size_t>(bal_i[hasb ? jb : j]) * p.d2;
        uint4 ka[KCH], kb[KCH];
#pragma unroll
        for (int m = 0; m < KCH; ++m) {
          const int ch = lane + 32 * m;
          const bool in = ch * 8 < p.d2;
          ka[m] = in ? ldg_ro128(ra + ch * 8) : make_uint4(0, 0, 0, 0);
          kb[m] = (in && hasb) ? ldg_ro128(rb + ch * 8) : make_uint4(0, 0, 0, 0);
        }
        float fa = 0.f, fb = 0.f;
#pragma unroll
        for (int m = 0; m < KCH; ++m) {
          const int ch = lane + 32 * m;
          if (ch * 8 < p.d2) {
            const uint4 qv = lds128(q2s + ch * 8);
            fa = dot8_bf16(ka[m], qv, fa);
            fb = dot8_bf16(kb[m], qv, fb);
          }
        }
        fa = warp_sum(fa);
        fb = warp_sum(fb);
        if (lane == 0) {
          bal_h[j] = gelu_tanh(bal_h[j] - theta) * fa;
          if (hasb) bal_h[jb] = gelu_tanh(bal_h[jb] - theta) * fb;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < kVB; ++u) {
      if (j0 + u < nact) {
        const float hu = bal_h[j0 + u];
#pragma unroll
        for (int cp = 0; cp < CPT; ++cp) {
          const float2 v0 = bf16x2_to_float2(v[cp][u].x), v1 = bf16x2_to_float2(v[cp][u].y);
          const float2 v2 = bf16x2_to_float2(v[cp][u].z), v3 = bf16x2_to_float2(v[cp][u].w);
          acc[cp][0] = fmaf(hu, v0.x, acc[cp][0]);
          acc[cp][1] = fmaf(hu, v0.y, acc[cp][1]);
          acc[cp][2] = fmaf(hu, v1.x, acc[cp][2]);
          acc[cp][3] = fmaf(hu, v1.y, acc[cp][3]);
          acc[cp][4] = fmaf(hu, v2.x, acc[cp][4]);
          acc[cp][5] = fmaf(hu, v2.y, acc[cp][5]);
          acc[cp][6] = fmaf(hu, v3.x, acc[cp][6]);
          acc[cp][7] = fmaf(hu, v3.y, acc[cp][7]);
        }
      }
    }
  }
#pragma unroll
  for (int cp = 0; cp < CPT; ++cp) {
    const int ch = tid + cp * kGThreads;
    if (ch < nco) {
      float4* dst = reinterpret_cast<float4*>(part + ch * 8);
      dst[0] = make_float4(acc[cp][0], acc[cp][1], acc[cp][2], acc[cp][3]);
      dst[1] = make_float4(acc[cp][4], acc[cp][5], acc[cp][6], acc[cp][7]);
    }
  }
  cluster_sync();

  // cluster partial: rank q sums columns [q*cw, (q+1)*cw) over the CS CTAs in rank order
  const int cw = (D + CS - 1) / CS;
  const int col_lo = static_cast<int>(rank) * cw;
  const int col_hi = min(col_lo + cw, D);
  for (int col = col_lo + tid; col < col_hi; col += kGThreads) {
    float v[CS];
#pragma unroll
    for (int src = 0; src < CS; ++src) v[src] = ld_dsmem_f32(part + col, static_cast<unsigned>(src));
    float s = 0.f;
#pragma unroll
    for (int src = 0; src < CS; ++src) s += v[src];
    __stcg(p.cpart + static_cast<size_t>(cl) * D + col, s);
  }
  __threadfence();
  cluster_sync();
  if (rank == 0 && tid == 0) {
    const unsigned old = atomicAdd(p.arrive, 1u);
    misc_i[1] = old == static_cast<unsigned>(p.n_clusters - 1) ? 1 : 0;
  }
  cluster_sync();
  if (tid == 0) misc_i[2] = static_cast<int>(ld_dsmem_u32(reinterpret_cast<const unsigned*>(misc_i + 1), 0u));
  __syncthreads();
  if (misc_i[2]) {
    // the last cluster: every cluster partial is written; sum them in cluster order
    __threadfence();
    float hv[kMaxGChunks];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxGChunks; ++k) {
      const int col = col_lo + tid + k * kGThreads;
      hv[k] = 0.f;
      if (col >= col_hi) continue;
      float v[kMaxClusters];
#pragma unroll
      for (int g = 0; g < kMaxClusters; ++g)
        v[g] = g < p.n_clusters ? __ldcg(p.cpart + static_cast<size_t>(g) * D + col) : 0.f;
      float s = 0.f;
#pragma unroll
      for (int g = 0; g < kMaxClusters; ++g) s += v[g];
      const __nv_bfloat16 b = __float2bfloat16_rn(s);
      if (p.out != nullptr) p.out[col] = *reinterpret_cast<const uint16_t*>(&b);
      if (p.h_base != nullptr) {
        const float hn = p.h_base[col] + __bfloat162float(b);
        p.h_out[col] = hn;
        hv[k] = hn;
        ss = fmaf(hn, hn, ss);
      }
    }
    if (p.h_base != nullptr && p.q_next != nullptr) {
      // next layer's q = bf16(h / sqrt(mean(h^2) + eps)): CTA sums, then the
      // cluster's in rank order (same bits in every rank)
      ss = warp_sum(ss);
      if (lane == 0) red[warp] = ss;
      __syncthreads();
      if (tid == 0) {
        float t = 0.f;
        for (int w = 0; w < kGWarps; ++w) t += red[w];
        misc_f[1] = t;
      }
      cluster_sync();
      float tot = 0.f;
#pragma unroll
      for (int src = 0; src < CS; ++src) tot += ld_dsmem_f32(misc_f + 1, static_cast<unsigned>(src));
      const float inv = 1.f / sqrtf(tot / static_cast<float>(D) + p.eps);
#pragma unroll
      for (int k = 0; k < kMaxGChunks; ++k) {
        const int col = col_lo + tid + k * kGThreads;
        if (col >= col_hi) continue;
        const __nv_bfloat16 b = __float2bfloat16_rn(hv[k] * inv);
        p.q_next[col] = *reinterpret_cast<const uint16_t*>(&b);
      }
    }
    if (rank == 0 && tid == 0) *p.arrive = 0u;  // for the next call on this workspace
  }
  // no CTA leaves while another may still read its shared memory
  cluster_sync();
}

// q = bf16(h / sqrt(mean(h^2) + eps)) for the first layer of a stack (one CTA).
__global__ void __launch_bounds__(1024, 1) rmsnorm_q_kernel(const float* h, uint16_t* q, int d, float eps) {
  __shared__ float red[32];
  __shared__ float inv_s;
  // The first layer's P may start streaming its weights now; it reads q only
  // after this grid has completed.
  griddep_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float ss = 0.f;
  for (int i = tid; i < d; i += blockDim.x) ss = fmaf(h[i], h[i], ss);
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x / 32); ++w) t += red[w];
    inv_s = 1.f / sqrtf(t / static_cast<float>(d) + eps);
  }
  __syncthreads();
  for (int i = tid; i < d; i += blockDim.x) {
    const __nv_bfloat16 b = __float2bfloat16_rn(h[i] * inv_s);
    q[i] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

using KernelFn = void (*)(PgParams);

KernelFn score_kernel(int kch) {
  return kch == 5 ? decode_score_kernel<5> : kch == 8 ? decode_score_kernel<8> : nullptr;
}

template <int CS, int CPT>
KernelFn gather_for_kch(int kch) {
  return kch == 5 ? decode_gather_kernel<CS, CPT, 5> : kch == 8 ? decode_gather_kernel<CS, CPT, 8> : nullptr;
}

template <int CS>
KernelFn gather_for_cpt(int cpt, int kch) {
  switch (cpt) {
    case 1: return gather_for_kch<CS, 1>(kch);
    case 2: return gather_for_kch<CS, 2>(kch);
    case 4: return gather_for_kch<CS, 4>(kch);
    default: return nullptr;
  }
}

KernelFn gather_kernel(int cs, int cpt, int kch) {
  switch (cs) {
    case 8: return gather_for_cpt<8>(cpt, kch);
    case 4: return gather_for_cpt<4>(cpt, kch);
    case 2: return gather_for_cpt<2>(cpt, kch);
    default: return nullptr;
  }
}

// cudaFuncAttributeMaxDynamicSharedMemorySize, raised once per (kernel, device).
std::mutex g_attr_mutex;
std::map<std::pair<const void*, int>, size_t> g_attr_done;

cudaError_t ensure_smem(const void* fn, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  size_t& done = g_attr_done[{fn, dev}];
  if (done >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) done = bytes;
  return e;
}

}  // namespace

DecodePgPlan plan_decode_pg(int d_model, int r, int d_ff, int num_sms, size_t smem_optin, int cluster_override) {
  DecodePgPlan pl{};
  pl.ok = false;
  const int d2 = d_model - r;
  if (d_model % 8 != 0 || r % 8 != 0 || r < 8 || d2 < 8 || num_sms < 1) return pl;
  const int lane_chunks = (max(r, d2) / 8 + 31) / 32;
  const int kch = lane_chunks <= 5 ? 5 : lane_chunks <= 8 ? 8 : 0;
  if (kch == 0) return pl;
  int rpc = (d_ff + num_sms - 1) / num_sms;
  rpc = static_cast<int>(pg_align(static_cast<size_t>(rpc), kStageRows));
  const int n_slices = (d_ff + rpc - 1) / rpc;
  if (n_slices > kMaxSlices) return pl;
  const int nco = d_model / 8;
  const int cpt_min = (nco + kGThreads - 1) / kGThreads;
  const int cpt = cpt_min <= 1 ? 1 : cpt_min <= 2 ? 2 : cpt_min <= 4 ? 4 : 0;
  if (cpt == 0) return pl;
  const int cs = cluster_override > 0 ? cluster_override : 8;
  if (cs != 8 && cs != 4 && cs != 2) return pl;
  // columns per rank in the final sum must fit kMaxGChunks per thread
  if ((((d_model + cs - 1) / cs) + kGThreads - 1) / kGThreads > kMaxGChunks) return pl;
  // two score slices per gather CTA (about 2 * 8% * rpc active rows), more if
  // needed to keep the cluster partials within one batch of the final sum
  int spc = 2;
  while ((((n_slices + spc - 1) / spc + cs - 1) / cs) > kMaxClusters) ++spc;
  const int n_g = (n_slices + spc - 1) / spc;
  const int grid_g = (n_g + cs - 1) / cs * cs;
  const size_t smem_p = PLayout(r, rpc).total;
  const size_t smem_g = GLayout(d_model, r, spc * rpc, n_slices).total;
  if (smem_p > smem_optin || smem_g > smem_optin) return pl;
  pl.n_slices = n_slices;
  pl.rows_per_cta = rpc;
  pl.slices_per_g = spc;
  pl.grid_g = grid_g;
  pl.cluster = cs;
  pl.chunks_per_thread = cpt;
  pl.lane_chunks = kch;
  pl.n_clusters = grid_g / cs;
  pl.smem_p = smem_p;
  pl.smem_g = smem_g;
  pl.ws_bytes = PgWs(d_model, d_ff, n_slices, pl.n_clusters).total;
  pl.ok = true;
  return pl;
}

void* decode_pg_qbuf(const DecodePgPlan& pl, void* workspace, int d_model, int d_ff) {
  const PgWs W(d_model, d_ff, pl.n_slices, pl.n_clusters);
  return static_cast<unsigned char*>(workspace) + W.qbuf;
}

cudaError_t launch_decode_pg(const DecodePgPlan& pl, const DecodePgArgs& a, cudaStream_t stream) {
  const PgWs W(a.d_model, a.d_ff, pl.n_slices, pl.n_clusters);
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  PgParams p;
  p.q = a.q_from_workspace ? reinterpret_cast<const uint16_t*>(ws + W.qbuf) : static_cast<const uint16_t*>(a.q);
  p.K1 = static_cast<const uint16_t*>(a.K1);
  p.K2 = static_cast<const uint16_t*>(a.K2);
  p.V = static_cast<const uint16_t*>(a.V);
  p.out = static_cast<uint16_t*>(a.out);
  p.d_model = a.d_model;
  p.r = a.r;
  p.d2 = a.d_model - a.r;
  p.d_ff = a.d_ff;
  p.rpc = pl.rows_per_cta;
  p.rpg = pl.rows_per_cta * pl.slices_per_g;
  p.n_slices = pl.n_slices;
  p.n_clusters = pl.n_clusters;
  p.Q = a.Q;
  p.ctl = reinterpret_cast<DeviceControl*>(ws);
  p.arrive = &p.ctl->pg_arrive;  // zeroed with the control block; the last cluster resets it
  p.mom = reinterpret_cast<float2*>(ws + W.mom);
  p.xg = reinterpret_cast<float*>(ws + W.xg);
  p.cpart = reinterpret_cast<float*>(ws + W.cpart);
  p.x_out = a.x_out;
  p.theta_out = a.theta_out;
  p.active_out = a.active_out;
  p.q_dbg = static_cast<uint16_t*>(a.q_dbg);
  p.h_base = a.h_base;
  p.h_out = a.h_out;
  p.q_next = a.write_q_next ? reinterpret_cast<uint16_t*>(ws + W.qbuf) : nullptr;
  p.eps = a.eps;
  p.wait_limit_ns = a.wait_limit_ns;

  const KernelFn pfn = score_kernel(pl.lane_chunks);
  const KernelFn gfn = gather_kernel(pl.cluster, pl.chunks_per_thread, pl.lane_chunks);
  if (pfn == nullptr || gfn == nullptr) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(pfn), pl.smem_p);
  if (e != cudaSuccess) return e;
  e = ensure_smem(reinterpret_cast<const void*>(gfn), pl.smem_g);
  if (e != cudaSuccess) return e;

  cudaLaunchAttribute pattr[1];
  cudaLaunchConfig_t pc = {};
  pc.gridDim = dim3(pl.n_slices);
  pc.blockDim = dim3(kPThreads);
  pc.dynamicSmemBytes = pl.smem_p;
  pc.stream = stream;
  pattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pattr[0].val.programmaticStreamSerializationAllowed = 1;
  pc.attrs = pattr;
  pc.numAttrs = a.overlap_weights ? 1 : 0;
  e = cudaLaunchKernelEx(&pc, pfn, p);
  if (e != cudaSuccess) return e;

  // G follows P programmatically: its reads of P's results come after griddepcontrol.wait
  cudaLaunchAttribute gattr[2];
  cudaLaunchConfig_t gc = {};
  gc.gridDim = dim3(pl.grid_g);
  gc.blockDim = dim3(kGThreads);
  gc.dynamicSmemBytes = pl.smem_g;
  gc.stream = stream;
  gattr[0].id = cudaLaunchAttributeClusterDimension;
  gattr[0].val.clusterDim.x = pl.cluster;
  gattr[0].val.clusterDim.y = 1;
  gattr[0].val.clusterDim.z = 1;
  gattr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  gattr[1].val.programmaticStreamSerializationAllowed = 1;
  gc.attrs = gattr;
  gc.numAttrs = 2;
  return cudaLaunchKernelEx(&gc, gfn, p);
}

cudaError_t launch_rmsnorm_q(const DecodePgPlan& pl, void* workspace, const float* h, int d_model, int d_ff,
                             float eps, cudaStream_t stream) {
  uint16_t* q = static_cast<uint16_t*>(decode_pg_qbuf(pl, workspace, d_model, d_ff));
  rmsnorm_q_kernel<<<1, 1024, 0, stream>>>(h, q, d_model, eps);
  return cudaGetLastError();
}

}  // namespace spark
