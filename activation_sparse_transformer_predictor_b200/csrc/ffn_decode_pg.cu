// ffn_decode_pg.cu -- Spark FFN forward for ONE token (decode) as three
// chained kernels: score (P), gather (G) and reduce (R).
//
// Spark Transformer notes, 关键设计 / "Spark FFN" and "Statistical Top-k":
//   x = K1^T q[:r];  theta = mean(x) + std(x) Q(1 - k/d_ff);
//   out = V . (GELU(max(x - theta, 0)) (.) (K2^T q[r:])) over the neurons with x > theta.
//
// The two global dependencies (theta needs every score; out needs every
// neuron's contribution) are kernel boundaries, so no kernel waits on another
// CTA's progress and no co-residency is assumed.  Each kernel is launched as a
// programmatic dependent of the one before it (griddepcontrol): it may start
// while its predecessor runs, and reads its predecessor's results only after
// griddepcontrol.wait.
//
//  P  CTA c owns neurons [c*RPC, (c+1)*RPC).  Before anything else it bulk-copies
//     its whole K1 slice into shared memory; only then does it wait for the work
//     ahead of it on the stream.  With weight overlap on, P is launched while
//     the previous call's kernels still run, so the K1 stream -- 80% of the
//     layer's bytes -- hides behind them.  After the wait: q (stack mode:
//     q = bf16(RMSNorm(h)), formed by every CTA), x row by row (fp32 FMA on bf16
//     operands), and the slice's moments (mean, M2); x and the moments go to
//     the workspace.
//  G  CTA c merges all slices' moments in slice order (every CTA derives the
//     same bits of theta), compacts the active neurons of slice c, reads their
//     K2 rows (a = K2.q[r:]) and V rows, and writes its fp32 partial output
//     sum_i GELU(x_i - theta) a_i V[i,:].
//  R  CTA b owns 16 output columns: it sums the partials of all slices in a
//     fixed order and stores bf16 (stack mode: h_out = h + bf16(out)).
// No atomics: results are bit-reproducible.
//
// With q and out in mapped (pinned) host memory, a one-CTA kernel F ahead of P
// copies q into the workspace (P, launched programmatically behind F, streams
// K1 meanwhile), and R stores out straight into host memory: no copy-engine
// transfer sits between two calls' kernels.
#include <map>
#include <mutex>
#include <utility>

#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

#ifdef SPARK_DEBUG
// bounds-check violations of this file's kernels (see SPARK_CHECK)
static __device__ unsigned g_bounds_violations;
#endif

namespace {

constexpr int kPWarps = 8;
constexpr int kPThreads = kPWarps * 32;
constexpr int kStageRows = 8;            // K1 rows per bulk copy / mbarrier
constexpr int kGWarps = 9;
constexpr int kGThreads = kGWarps * 32;  // one 16-byte output chunk per thread at d_model = 2304
constexpr int kMaxSlices = 256;          // moments merged by one warp, 8 per lane
constexpr int kRThreads = 128;
constexpr int kRCols = 16;               // output columns per R CTA (four float4)
constexpr int kRSubsets = kRThreads / (kRCols / 4);

__host__ __device__ inline size_t pg_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct PgParams {
  const uint16_t* q;   // bf16 [d_model] (ignored in stack mode)
  const float* h_in;   // stack mode: fp32 [d_model]; P forms q = bf16(h / rms(h))
  const uint16_t* K1;  // bf16 [d_ff][r]
  const uint16_t* K2;  // bf16 [d_ff][d_model - r]
  const uint16_t* V;   // bf16 [d_ff][d_model]
  uint16_t* out;       // bf16 [d_model], may be nullptr in stack mode
  int d_model, r, d2, d_ff;
  int rpc;             // rows (neurons) per P / G CTA
  int n_slices;        // P and G CTAs
  float Q;
  float eps;
  DeviceControl* ctl;
  float2* mom;         // [n_slices] (mean, M2) of each slice's scores
  float* xg;           // [d_ff] scores
  float* part;         // [n_slices][d_model] partial outputs
  uint16_t* qbuf;      // [d_model] the q used (written by P's CTA 0, read by G)
  float* x_out;        // optional debug outputs
  float* theta_out;
  unsigned char* active_out;
  uint16_t* q_dbg;
  const float* h_base;  // stack mode, R: h_out = h_base + bf16(out)
  float* h_out;
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// Shared-memory layout of P.
struct PLayout {
  size_t k1, qs, xs, bars, red, total;
  __host__ __device__ PLayout(int d_model, int r, int rpc) {
    size_t off = 0;
    k1 = off;
    off += pg_align(static_cast<size_t>(rpc) * r * 2, 128);
    qs = off;
    off += pg_align(static_cast<size_t>(d_model) * 2, 128);
    xs = off;
    off += pg_align(static_cast<size_t>(rpc) * 4, 16);
    bars = off;
    off += pg_align(static_cast<size_t>(rpc / kStageRows) * 8, 16);
    red = off;
    off += 64;
    total = off;
  }
};

// Shared-memory layout of G.
struct GLayout {
  size_t q2, mom, xs, act_i, act_h, misc, total;
  __host__ __device__ GLayout(int d_model, int r, int rpc, int n_slices) {
    size_t off = 0;
    q2 = off;
    off += pg_align(static_cast<size_t>(d_model - r) * 2, 128);
    mom = off;
    off += pg_align(static_cast<size_t>(n_slices) * 8, 16);
    xs = off;
    off += pg_align(static_cast<size_t>(rpc) * 4, 16);
    act_i = off;
    off += pg_align(static_cast<size_t>(rpc) * 4, 16);
    act_h = off;
    off += pg_align(static_cast<size_t>(rpc) * 4, 16);
    misc = off;
    off += 64;
    total = off;
  }
};

// Workspace layout (after the device control block).
struct PgWs {
  size_t mom, xg, part, qbuf, total;
  PgWs(int d_model, int d_ff, int n_slices) {
    size_t off = sizeof(DeviceControl);
    mom = off;
    off += pg_align(static_cast<size_t>(n_slices) * 8, 256);
    xg = off;
    off += pg_align(static_cast<size_t>(d_ff) * 4, 256);
    part = off;
    off += pg_align(static_cast<size_t>(n_slices) * d_model * 4, 256);
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
  const PLayout L(p.d_model, p.r, p.rpc);
  uint16_t* k1s = reinterpret_cast<uint16_t*>(smem + L.k1);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  float* red = reinterpret_cast<float*>(smem + L.red);
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

  // q into shared memory (stack mode: q = bf16(h / sqrt(mean(h^2) + eps)), the
  // same bits in every CTA: fixed per-thread, warp and block orders)
  const int nq = p.d_model / 8;
  if (p.h_in == nullptr) {
    for (int ch = tid; ch < nq; ch += kPThreads)
      *reinterpret_cast<uint4*>(qs + ch * 8) = ldcg128(p.q + ch * 8);
  } else {
    float ss = 0.f;
    for (int i = tid; i < p.d_model; i += kPThreads) {
      const float h = __ldcg(p.h_in + i);
      ss = fmaf(h, h, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kPWarps; ++w) t += red[w];
      red[8] = 1.f / sqrtf(t / static_cast<float>(p.d_model) + p.eps);
    }
    __syncthreads();
    const float inv = red[8];
    for (int i = tid; i < p.d_model; i += kPThreads) {
      const __nv_bfloat16 b = __float2bfloat16_rn(__ldcg(p.h_in + i) * inv);
      qs[i] = *reinterpret_cast<const uint16_t*>(&b);
    }
  }
  __syncthreads();  // q staged; the barrier inits are visible

  // Warp w scores the stages w, w + 8, ...: the 8 rows of a stage together, so
  // that each lane runs 8 independent FMA chains; then one transposed butterfly
  // reduces the 8 row sums over the warp (9 shuffles instead of 8 x 5).
  const int nchunk = p.r / 8;
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
        const uint4 qv = lds128(qs + ch * 8);
        uint4 kv[kStageRows];
#pragma unroll
        for (int j = 0; j < kStageRows; ++j) kv[j] = lds128(kst + static_cast<size_t>(j) * p.r + ch * 8);
#pragma unroll
        for (int j = 0; j < kStageRows; ++j) {
          float t = acc[j];
          t = fma_bf16x2_f32(kv[j].x, qv.x, t);
          t = fma_bf16x2_f32(kv[j].y, qv.y, t);
          t = fma_bf16x2_f32(kv[j].z, qv.z, t);
          t = fma_bf16x2_f32(kv[j].w, qv.w, t);
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
  if (c == 0)
    for (int i = tid; i < p.d_model; i += kPThreads) {
      p.qbuf[i] = qs[i];
      if (p.q_dbg != nullptr) p.q_dbg[i] = qs[i];
    }
}

// ------------------------------------------------------------------------ G
// CPT: 16-byte output chunks per thread (d_model <= 2304 * CPT).
// KCH: 16-byte chunks per lane of a K2 row (d_model - r <= 256 * KCH).
template <int CPT, int KCH>
__global__ void __maxnreg__(128) decode_gather_kernel(const PgParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kVB = 16 / CPT;  // active rows whose V chunks are in flight at once
  const int c = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int D = p.d_model;
  const GLayout L(D, p.r, p.rpc, p.n_slices);
  uint16_t* q2s = reinterpret_cast<uint16_t*>(smem + L.q2);
  float2* moms = reinterpret_cast<float2*>(smem + L.mom);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  int* act_i = reinterpret_cast<int*>(smem + L.act_i);
  float* act_h = reinterpret_cast<float*>(smem + L.act_h);
  int* misc_i = reinterpret_cast<int*>(smem + L.misc);
  float* misc_f = reinterpret_cast<float*>(smem + L.misc) + 8;

  // This grid waits for P of this call.  R of this call (and through it the next
  // call's P, whose K1 stream fills the memory queues) is released only once
  // this CTA's V-row loads are issued, below.
  griddep_wait();

  const int n0 = c * p.rpc;
  const int nr = rows_in(n0, p.rpc, p.d_ff);
  for (int i = tid; i < p.n_slices; i += kGThreads) moms[i] = __ldcg(p.mom + i);
  for (int i = tid; i < nr; i += kGThreads) xs[i] = __ldcg(p.xg + n0 + i);
  for (int ch = tid; ch < p.d2 / 8; ch += kGThreads)
    *reinterpret_cast<uint4*>(q2s + ch * 8) = ldcg128(p.qbuf + p.r + ch * 8);
  __syncthreads();

  // theta from the slice moments, merged in slice order (same bits in every CTA),
  // then the active neurons of this slice in ascending order
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
      if (act && SPARK_CHECK(slot < nr)) {
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
  const int nact = misc_i[0];
  const float theta = misc_f[0];
  // the K2 rows of the active neurons into L2 now, ahead of the next call's K1
  // stream (released below once the V loads are issued): 13.45 -> 13.32 us per
  // call with weight overlap, 15.19 -> 14.93 without
  if (tid < nact) prefetch_l2_bulk(p.K2 + static_cast<size_t>(act_i[tid]) * p.d2, static_cast<unsigned>(p.d2) * 2);
  if (nact == 0) griddep_launch_dependents();
  if (c == 0 && tid == 0 && p.theta_out != nullptr) p.theta_out[0] = theta;
  if (p.active_out != nullptr)
    for (int i = tid; i < nr; i += kGThreads) p.active_out[n0 + i] = xs[i] > theta ? 1 : 0;

  // partial output of this slice: thread t owns 16-byte chunks t, t + 288, ...
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
        v[cp][u] = (j0 + u < nact && ch < nco && SPARK_CHECK(act_i[j0 + u] < p.d_ff))
                       ? ldg_ro128(p.V + static_cast<size_t>(act_i[j0 + u]) * D + ch * 8)
                       : make_uint4(0, 0, 0, 0);
      }
    if (j0 == 0) griddep_launch_dependents();
    if (j0 == 0) {
      // ... while the warps form h = GELU(x - theta) a, a = <K2[i,:], q[r:]>:
      // two rows per warp, all of both rows' loads issued before the arithmetic
      for (int j = warp; j < nact; j += 2 * kGWarps) {
        const int jb = j + kGWarps;
        const bool hasb = jb < nact;
        if (!SPARK_CHECK(act_i[j] < p.d_ff && act_i[hasb ? jb : j] < p.d_ff)) continue;
        const uint16_t* ra = p.K2 + static_cast<size_t>(act_i[j]) * p.d2;
        const uint16_t* rb = p.K2 + static_cast<size_t>(act_i[hasb ? jb : j]) * p.d2;
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
          act_h[j] = gelu_tanh(act_h[j] - theta) * fa;
          if (hasb) act_h[jb] = gelu_tanh(act_h[jb] - theta) * fb;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < kVB; ++u) {
      if (j0 + u < nact) {
        const float hu = act_h[j0 + u];
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
  if (!SPARK_CHECK(c < p.n_slices && p.n_slices <= kMaxSlices)) return;
  float* mypart = p.part + static_cast<size_t>(c) * D;
#pragma unroll
  for (int cp = 0; cp < CPT; ++cp) {
    const int ch = tid + cp * kGThreads;
    if (ch < nco) {
      __stcg(reinterpret_cast<float4*>(mypart + ch * 8), make_float4(acc[cp][0], acc[cp][1], acc[cp][2], acc[cp][3]));
      __stcg(reinterpret_cast<float4*>(mypart + ch * 8) + 1,
             make_float4(acc[cp][4], acc[cp][5], acc[cp][6], acc[cp][7]));
    }
  }
}

// ------------------------------------------------------------------------ F
// q from host memory (a device-visible address of a mapped pinned buffer) into
// the device copy P reads.  It lets its dependent (P) launch at once, reads q,
// and writes it only after the kernel ahead of it has completed, so that F's
// completion also stands for that kernel's (the chain stays ordered).
__global__ void __launch_bounds__(256) decode_fetch_q_kernel(const uint4* src, uint4* dst, int n16) {
  griddep_launch_dependents();
  constexpr int kPer = 4;  // up to 4 x 256 chunks of 16 bytes: d_model <= 8192
  uint4 v[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < n16) v[j] = __ldcv(src + i);  // host memory: plain (coherent) loads, not the read-only path
  }
  griddep_wait();
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = threadIdx.x + j * 256;
    if (i < n16) dst[i] = v[j];
  }
}

// ------------------------------------------------------------------------ R
// CTA b owns columns [16b, 16b + 16): thread t sums the partials of slices
// t/4, t/4 + 32, ... for its float4 of columns (t % 4), then the 32 subsets are
// summed in order.  bf16 store; stack mode also h_out = h_base + bf16(out).
__global__ void __launch_bounds__(kRThreads, 8) decode_reduce_kernel(const PgParams p) {
  __shared__ float4 red[kRSubsets][kRCols / 4];
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int cq = tid % (kRCols / 4);
  const int sub = tid / (kRCols / 4);
  const int col = b * kRCols + cq * 4;
  // the next call's P may now be scheduled; this grid waits for G of this call
  griddep_launch_dependents();
  griddep_wait();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col < p.d_model) {
    constexpr int kUnroll = 8;
    for (int s0 = sub; s0 < p.n_slices; s0 += kUnroll * kRSubsets) {
      float4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int s = s0 + u * kRSubsets;
        v[u] = s < p.n_slices ? __ldcg(reinterpret_cast<const float4*>(p.part + static_cast<size_t>(s) * p.d_model + col))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        acc.x += v[u].x;
        acc.y += v[u].y;
        acc.z += v[u].z;
        acc.w += v[u].w;
      }
    }
  }
  red[sub][cq] = acc;
  __syncthreads();
  if (tid < kRCols) {
    const int o = b * kRCols + tid;
    if (o < p.d_model) {
      float sum = 0.f;
      for (int k = 0; k < kRSubsets; ++k) sum += reinterpret_cast<const float*>(&red[k][tid / 4])[tid % 4];
      const __nv_bfloat16 bb = __float2bfloat16_rn(sum);
      if (p.out != nullptr) p.out[o] = *reinterpret_cast<const uint16_t*>(&bb);
      if (p.h_base != nullptr) p.h_out[o] = p.h_base[o] + __bfloat162float(bb);
    }
  }
}

using KernelFn = void (*)(PgParams);

KernelFn score_kernel(int kch) {
  return kch == 5 ? decode_score_kernel<5> : kch == 8 ? decode_score_kernel<8> : nullptr;
}

template <int CPT>
KernelFn gather_for_kch(int kch) {
  return kch == 5 ? decode_gather_kernel<CPT, 5> : kch == 8 ? decode_gather_kernel<CPT, 8> : nullptr;
}

KernelFn gather_kernel(int cpt, int kch) {
  switch (cpt) {
    case 1: return gather_for_kch<1>(kch);
    case 2: return gather_for_kch<2>(kch);
    case 4: return gather_for_kch<4>(kch);
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

DecodePgPlan plan_decode_pg(int d_model, int r, int d_ff, int num_sms, size_t smem_optin) {
  DecodePgPlan pl{};
  pl.ok = false;
  const int d2 = d_model - r;
  if (d_model % 8 != 0 || r % 8 != 0 || r < 8 || d2 < 8 || num_sms < 1 || d_ff < 1) return pl;
  const int lane_chunks = (max(r, d2) / 8 + 31) / 32;
  const int kch = lane_chunks <= 5 ? 5 : lane_chunks <= 8 ? 8 : 0;
  if (kch == 0) return pl;
  int rpc = (d_ff + num_sms - 1) / num_sms;
  rpc = static_cast<int>(pg_align(static_cast<size_t>(rpc), kStageRows));
  if (rpc > 256) return pl;
  const int n_slices = (d_ff + rpc - 1) / rpc;
  if (n_slices > kMaxSlices) return pl;
  const int nco = d_model / 8;
  const int cpt_min = (nco + kGThreads - 1) / kGThreads;
  const int cpt = cpt_min <= 1 ? 1 : cpt_min <= 2 ? 2 : cpt_min <= 4 ? 4 : 0;
  if (cpt == 0) return pl;
  const size_t smem_p = PLayout(d_model, r, rpc).total;
  const size_t smem_g = GLayout(d_model, r, rpc, n_slices).total;
  if (smem_p > smem_optin || smem_g > smem_optin) return pl;
  pl.n_slices = n_slices;
  pl.rows_per_cta = rpc;
  pl.chunks_per_thread = cpt;
  pl.lane_chunks = kch;
  pl.n_rctas = (d_model + kRCols - 1) / kRCols;
  pl.smem_p = smem_p;
  pl.smem_g = smem_g;
  pl.ws_bytes = PgWs(d_model, d_ff, n_slices).total;
  pl.ok = true;
  return pl;
}

cudaError_t launch_decode_pg(const DecodePgPlan& pl, const DecodePgArgs& a, cudaStream_t stream) {
  const PgWs W(a.d_model, a.d_ff, pl.n_slices);
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  PgParams p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.h_in = a.h_in;
  p.K1 = static_cast<const uint16_t*>(a.K1);
  p.K2 = static_cast<const uint16_t*>(a.K2);
  p.V = static_cast<const uint16_t*>(a.V);
  p.out = static_cast<uint16_t*>(a.out);
  p.d_model = a.d_model;
  p.r = a.r;
  p.d2 = a.d_model - a.r;
  p.d_ff = a.d_ff;
  p.rpc = pl.rows_per_cta;
  p.n_slices = pl.n_slices;
  p.Q = a.Q;
  p.eps = a.eps;
  p.ctl = reinterpret_cast<DeviceControl*>(ws);
  p.mom = reinterpret_cast<float2*>(ws + W.mom);
  p.xg = reinterpret_cast<float*>(ws + W.xg);
  p.part = reinterpret_cast<float*>(ws + W.part);
  p.qbuf = reinterpret_cast<uint16_t*>(ws + W.qbuf);
  p.x_out = a.x_out;
  p.theta_out = a.theta_out;
  p.active_out = a.active_out;
  p.q_dbg = static_cast<uint16_t*>(a.q_dbg);
  p.h_base = a.h_base;
  p.h_out = a.h_out;
  p.wait_limit_ns = a.wait_limit_ns;

  const KernelFn pfn = score_kernel(pl.lane_chunks);
  const KernelFn gfn = gather_kernel(pl.chunks_per_thread, pl.lane_chunks);
  if (pfn == nullptr || gfn == nullptr) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(pfn), pl.smem_p);
  if (e != cudaSuccess) return e;
  e = ensure_smem(reinterpret_cast<const void*>(gfn), pl.smem_g);
  if (e != cudaSuccess) return e;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cfg.attrs = attr;
  if (a.q_fetch != nullptr) {
    // F: q from host memory; programmatic like P (it writes only after its wait)
    const int n16 = a.d_model / 8;
    if (a.d_model % 8 != 0 || n16 > 4 * 256 || a.h_in != nullptr) return cudaErrorInvalidValue;
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.numAttrs = a.overlap_weights ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, decode_fetch_q_kernel, static_cast<const uint4*>(a.q_fetch),
                           reinterpret_cast<uint4*>(const_cast<void*>(a.q)), n16);
    if (e != cudaSuccess) return e;
  }
  // P: programmatic only with weight overlap (it reads K1 before its wait)
  cfg.gridDim = dim3(pl.n_slices);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = pl.smem_p;
  cfg.numAttrs = a.overlap_weights ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, pfn, p);
  if (e != cudaSuccess) return e;
  // G and R follow programmatically: they read their predecessor's results only
  // after griddepcontrol.wait
  cfg.gridDim = dim3(pl.n_slices);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = pl.smem_g;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gfn, p);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(pl.n_rctas);
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, decode_reduce_kernel, p);
}


// ---------------------------------------------------------------- debug builds
unsigned take_bounds_violations_decode(bool clear) {
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
