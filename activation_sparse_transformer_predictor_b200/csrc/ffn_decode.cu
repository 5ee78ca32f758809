// ffn_decode.cu -- Spark FFN forward for ONE token (decode) with one global exchange.
//
// Spark Transformer notes, 关键设计 / "Spark FFN" and "Statistical Top-k":
//   x = K1^T q[:r];  theta = mean(x) + std(x) Q(1 - k/d_ff);
//   out = V . (GELU(max(x - theta, 0)) (.) (K2^T q[r:])) over the neurons with x > theta.
//
// One cooperative launch, one CTA per SM, nine warps.  The global dependency
// (theta needs every score) costs one exchange:
//
//  phase 1  CTA c owns neurons [c*RPC, (c+1)*RPC).  Thread 0 bulk-copies the
//           whole K1 slice into shared memory at kernel start; warps 0-7 compute
//           x row by row (fp32 FMA, q[:r] in registers) and signal each 8-row
//           stage on an mbarrier.
//  speculation (warp 8, during phase 1)  publishes the moments of its first 8
//           scores, and once half of the CTAs have done the same, estimates
//           theta from them (~0.06 std) and, for each score above
//           (estimate - 6 standard errors), bulk-copies the neuron's K2 row into
//           shared memory and prefetches its V row into L2 -- while K1 is still
//           streaming.
//  publish  each CTA writes a header (exact moments of its slice, the largest
//           score it did NOT speculate on, candidate count) and (index, x,
//           a = K2.q[r:]) for each candidate.
//  exchange after an acquire-release counter, every CTA bulk-copies all
//           headers and entries and merges the moments in CTA order (so every
//           CTA derives the same bits of theta).  If some CTA's largest
//           non-candidate score passes theta (vanishingly rare), the entries of
//           every CTA are rebuilt from K1/K2 with the same arithmetic, so the
//           result never depends on the estimate.
//  gather   CTA c owns output columns [c*CW, (c+1)*CW): for each active entry
//           (x > theta) it forms h = GELU(x - theta) * a and reads V[i, cols]
//           (mostly L2 hits); thread groups own source CTAs, then a fixed-order
//           reduction; bf16 store.  No data atomics: bit-reproducible.
#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {
namespace {

constexpr int kCompWarps = 8;
constexpr int kSpecWarp = kCompWarps;  // the speculation warp
constexpr int kWarps = kCompWarps + 1;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerStage = kCompWarps;
constexpr int kEntryBytes = 12;  // neuron index, x, a
constexpr float kSpecSd = 6.0f;  // margin of the candidate threshold, in standard errors

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct DecLayout {
  size_t region_a, cand, qs, hsm, xs, bars, cidx, red, misc, total;
  size_t hdr_off, ent_off;  // inside region_a after phase 1
  __host__ __device__ DecLayout(int d_model, int r, int rpc, int grid, int cap) {
    const int nst = rpc / kRowsPerStage;
    const size_t k1 = static_cast<size_t>(nst) * kRowsPerStage * r * 2;
    hdr_off = 0;
    ent_off = align_up(static_cast<size_t>(grid) * 16, 128);
    // room for [grid][rpc] entries: the recompute path lists every active neuron
    const size_t p2 = ent_off + align_up(static_cast<size_t>(grid) * rpc * kEntryBytes, 128);
    size_t off = 0;
    region_a = off;
    off += align_up(k1 > p2 ? k1 : p2, 128);
    cand = off;
    off += align_up(static_cast<size_t>(cap) * (d_model - r) * 2, 128);
    qs = off;
    off += align_up(static_cast<size_t>(d_model) * 2, 128);
    hsm = off;  // stack mode: the fp32 residual
    off += align_up(static_cast<size_t>(d_model) * 4, 128);
    xs = off;
    off += align_up(static_cast<size_t>(rpc) * 4, 16);
    bars = off;
    off += align_up(static_cast<size_t>(2 * nst + 3) * 8, 16);
    cidx = off;
    off += align_up(static_cast<size_t>(cap) * 4, 16);
    red = off;
    off += kWarps * 32 * 8 * 4;
    misc = off;
    off += 128;
    total = off;
  }
};

struct DecWs {
  size_t s0, hdr, ent, total;
  DecWs(int grid, int cap) {
    size_t off = sizeof(DeviceControl);
    s0 = off;
    off += align_up(static_cast<size_t>(grid) * 16, 256);
    hdr = off;
    off += align_up(static_cast<size_t>(grid) * 16, 256);
    ent = off;
    off += align_up(static_cast<size_t>(grid) * cap * kEntryBytes, 256);
    total = off;
  }
};

struct DParams {
  const uint16_t* q;
  const uint16_t* K1;
  const uint16_t* K2;
  const uint16_t* V;
  uint16_t* out;
  int d_model, r, d2, d_ff, rpc, cap, col_width, n_col_ctas;
  float Q;
  float* x_out;
  float* theta_out;
  unsigned char* active_out;
  // stack mode (h_in != nullptr): q = bf16(RMSNorm(h_in)) is formed in every
  // CTA; the column owners write h_out = h_in + bf16(out) for their columns.
  const float* h_in;
  float* h_out;
  float eps;
  uint16_t* q_dbg;        // optional: the q used (bf16 [d_model]), written by CTA 0
  DeviceControl* ctl;
  float4* s0;            // [grid] (epoch tag, n, mean, M2) of each CTA's first 8 scores
  float4* hdr;           // [grid] (mean, M2, largest non-candidate x, candidate count)
  unsigned char* ent;    // [grid][cap] (index, x, a)
  unsigned long long wait_limit_ns;
  int never_arrive;
};

__device__ __forceinline__ int rows_of(int c, int rpc, int d_ff) { return max(0, min(rpc, d_ff - c * rpc)); }

// <row, q-part> for one bf16 row of length n (multiple of 8): lane-strided
// 16-byte chunks, fp32 FMA in chunk order, then the fixed warp tree.  The same
// routine serves shared and global rows, so recomputed values carry the same bits
// as the phase-1 scores and the candidate dots.
template <bool GLOBAL>
__device__ __forceinline__ float warp_row_dot(const uint16_t* row, const uint16_t* qpart, int n) {
  const int lane = threadIdx.x & 31;
  float acc = 0.f;
#pragma unroll
  for (int m = 0; m < kFusedMaxChunks; ++m) {
    const int c = lane + 32 * m;
    if (c * 8 < n) {
      const uint4 kv = GLOBAL ? ldg_nc128(row + c * 8) : lds128(row + c * 8);
      acc = dot8_bf16(kv, lds128(qpart + c * 8), acc);
    }
  }
  return warp_sum(acc);  // lane 0 holds the sum
}

__global__ void __launch_bounds__(kThreads, 1) spark_ffn_decode_kernel(const DParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const DecLayout L(p.d_model, p.r, p.rpc, G, p.cap);
  unsigned char* region_a = smem + L.region_a;
  uint16_t* k1s = reinterpret_cast<uint16_t*>(region_a);
  uint16_t* cand = reinterpret_cast<uint16_t*>(smem + L.cand);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + L.qs);
  float* hsm = reinterpret_cast<float*>(smem + L.hsm);
  float* xs = reinterpret_cast<float*>(smem + L.xs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);
  int* cidx = reinterpret_cast<int*>(smem + L.cidx);
  float* red = reinterpret_cast<float*>(smem + L.red);
  float* misc_f = reinterpret_cast<float*>(smem + L.misc);  // [0] theta, [1] largest non-candidate x
  int* misc_i = reinterpret_cast<int*>(smem + L.misc) + 4;  // [0] ncand [1] ok [2] recompute [4..12] warp flags [20] epoch
  DeviceControl* ctl = p.ctl;

  const int n0 = cta * p.rpc;
  const int nr = rows_of(cta, p.rpc, p.d_ff);
  const int nst = (nr + kRowsPerStage - 1) / kRowsPerStage;
  const int NST = p.rpc / kRowsPerStage;
  uint64_t* k1bar = bars;         // [NST]
  uint64_t* xready = bars + NST;  // [NST]
  uint64_t* qbar = bars + 2 * NST;
  uint64_t* candbar = qbar + 1;
  uint64_t* recbar = qbar + 2;

  // ---------------------------------------------------------------- set-up + K1 copies
  // No global load precedes the copies: the launch number and the abort flag
  // are read by the speculation warp while K1 streams.
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&k1bar[s], 1);
      mbar_init(&xready[s], kCompWarps);
    }
    mbar_init(qbar, 1);
    mbar_init(candbar, 1);
    mbar_init(recbar, 1);
    fence_mbar_init();
    if (p.h_in == nullptr) {
      const unsigned qbytes = static_cast<unsigned>(p.d_model) * 2;
      mbar_arrive_expect_tx(qbar, qbytes);
      bulk_g2s(qs, p.q, qbytes, qbar);
    } else {
      // stack mode: the residual first, ahead of the K1 stream
      const unsigned hbytes = static_cast<unsigned>(p.d_model) * 4;
      mbar_arrive_expect_tx(qbar, hbytes);
      bulk_g2s(hsm, p.h_in, hbytes, qbar);
    }
    for (int s = 0; s < nst; ++s) {
      const int rows = min(kRowsPerStage, nr - s * kRowsPerStage);
      const unsigned bytes = static_cast<unsigned>(rows) * p.r * 2;
      mbar_arrive_expect_tx(&k1bar[s], bytes);
      bulk_g2s(k1s + static_cast<size_t>(s) * kRowsPerStage * p.r,
               p.K1 + static_cast<size_t>(n0 + s * kRowsPerStage) * p.r, bytes, &k1bar[s]);
    }
    misc_i[0] = 0;
    misc_i[1] = 1;
    misc_i[2] = 0;
    misc_f[1] = -__int_as_float(0x7f800000);
  }
  __syncthreads();

  if (p.h_in != nullptr) {
    // stack mode: q = bf16(h / sqrt(mean(h^2) + eps)) while K1 streams in
    const bool hok = mbar_wait_bounded(qbar, 0, p.wait_limit_ns, ctl, 8);
    float ss = 0.f;
    for (int i = tid; hok && i < p.d_model; i += kThreads) {
      const float v = hsm[i];
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kWarps; ++w) t += red[w];
      misc_f[2] = 1.f / sqrtf(t / static_cast<float>(p.d_model) + p.eps);
    }
    __syncthreads();
    const float inv = misc_f[2];
    for (int i = tid; i < p.d_model; i += kThreads) {
      const __nv_bfloat16 b = __float2bfloat16_rn(hsm[i] * inv);
      qs[i] = *reinterpret_cast<const uint16_t*>(&b);
      if (cta == 0 && p.q_dbg != nullptr) p.q_dbg[i] = qs[i];
    }
    __syncthreads();
  }

  bool ok = true;
  if (warp < kCompWarps) {
    // ------------------------------------------------------------ phase 1: x
    ok = mbar_wait_bounded(qbar, 0, p.wait_limit_ns, ctl, 9);
    const int nchunk = p.r / 8;
    uint4 qreg[kFusedMaxChunks];
#pragma unroll
    for (int m = 0; m < kFusedMaxChunks; ++m) {
      const int c = lane + 32 * m;
      qreg[m] = (ok && c < nchunk) ? lds128(qs + c * 8) : make_uint4(0, 0, 0, 0);
    }
    for (int s = 0; s < nst; ++s) {
      if (ok) ok = mbar_wait_bounded(&k1bar[s], 0, p.wait_limit_ns, ctl, 10 + s);
      const int row = s * kRowsPerStage + warp;
      if (ok && row < nr) {
        const uint16_t* krow = k1s + static_cast<size_t>(row) * p.r;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < kFusedMaxChunks; ++m) {
          const int c = lane + 32 * m;
          if (c < nchunk) acc = dot8_bf16(lds128(krow + c * 8), qreg[m], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) xs[row] = acc;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&xready[s]);
    }
  } else if (warp == kSpecWarp) {
    // ------------------------------------------------------------ speculation warp
    // Launch number (its parity selects this launch's counters) and the abort
    // flag of an earlier launch that gave up waiting.
    unsigned epoch = 0, aborted = 0;
    if (lane == 0) {
      epoch = ld_relaxed_gpu(&ctl->epoch);
      aborted = ld_relaxed_gpu(&ctl->abort);
      misc_i[20] = static_cast<int>(epoch);
      // CTA 0 clears the other parity's counters: the previous launch, which
      // used them, has completed; the next launch will use them.
      if (cta == 0) {
        ctl->dec_arrive[(epoch & 1u) ^ 1u] = 0u;
        ctl->dec_s0[(epoch & 1u) ^ 1u] = 0u;
      }
    }
    epoch = __shfl_sync(0xffffffffu, epoch, 0);
    ok = __shfl_sync(0xffffffffu, aborted, 0) == 0u;
    unsigned* s0_cnt = &ctl->dec_s0[epoch & 1u];
    if (ok) ok = mbar_wait_bounded(&xready[0], 0, p.wait_limit_ns, ctl, 50);
    // moments of the first (up to) 8 scores, about the first one, tagged with the launch epoch
    const int nf = min(kRowsPerStage, nr);
    const float x0 = nr > 0 ? xs[0] : 0.f;
    const float sum = __shfl_sync(0xffffffffu, warp_sum(lane < nf ? xs[lane] - x0 : 0.f), 0);
    const float mean_f = x0 + sum / static_cast<float>(max(nf, 1));
    const float d = lane < nf ? xs[lane] - mean_f : 0.f;
    const float m2_f = warp_sum(d * d);
    if (lane == 0) {
      __stcg(p.s0 + cta, make_float4(__uint_as_float(epoch), static_cast<float>(nf), mean_f, m2_f));
      red_add_release_gpu(s0_cnt, 1u);
      // half of the CTAs are enough for the estimate
      ok = ok && wait_count_geq(ctl, s0_cnt, static_cast<unsigned>((G + 1) / 2), p.wait_limit_ns, 51);
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    // estimate theta from every first-stage record of this launch seen so far (CTA order)
    float4 e4[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = lane + 32 * j;
      e4[j] = (ok && c < G) ? __ldcg(p.s0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      if (__float_as_uint(e4[j].x) != epoch || !(e4[j].y > 0.f)) e4[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float sn = 0.f, sx = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sn += e4[j].y;
      sx = fmaf(e4[j].y, e4[j].z, sx);
    }
    sn = __shfl_sync(0xffffffffu, warp_sum(sn), 0);
    sx = __shfl_sync(0xffffffffu, warp_sum(sx), 0);
    const float mean_e = sx / fmaxf(sn, 1.f);
    float m2 = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float dm = e4[j].z - mean_e;
      m2 += e4[j].w + e4[j].y * dm * dm;
    }
    m2 = __shfl_sync(0xffffffffu, warp_sum(m2), 0);
    const float sd_e = sqrtf(fmaxf(m2, 0.f) / fmaxf(sn, 1.f));
    const float se = sd_e * sqrtf((1.f + 0.5f * p.Q * p.Q) / fmaxf(sn, 1.f));
    // without an estimate, speculate on nothing (the exchange then recomputes everything)
    const float cthr = (ok && sn > 1.f) ? fmaf(sd_e, p.Q, mean_e) - kSpecSd * se : __int_as_float(0x7f800000);
    // candidates, stage by stage as the scores land (stages already scored go
    // at once): ascending row order, so the slots are sorted by neuron
    int ncand = 0;
    float maxnc = -__int_as_float(0x7f800000);
    for (int s = 0; ok && s < nst; ++s) {
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&xready[s], 0, p.wait_limit_ns, ctl, 52));
      if (!ok) break;
      const int li = s * kRowsPerStage + lane;
      const bool valid = lane < kRowsPerStage && li < nr;
      const float x = valid ? xs[li] : 0.f;
      const bool c = valid && x > cthr;
      const unsigned ball = __ballot_sync(0xffffffffu, c);
      const int slot = ncand + __popc(ball & ((1u << lane) - 1u));
      if (c && slot < p.cap) {
        cidx[slot] = li;
        const size_t row = static_cast<size_t>(n0 + li);
        mbar_expect_tx(candbar, static_cast<unsigned>(p.d2) * 2);
        bulk_g2s(cand + static_cast<size_t>(slot) * p.d2, p.K2 + row * p.d2, p.d2 * 2, candbar);
        prefetch_l2_bulk(p.V + row * p.d_model, p.d_model * 2);
      } else if (valid) {
        maxnc = fmaxf(maxnc, x);
      }
      ncand = min(p.cap, ncand + __popc(ball));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) maxnc = fmaxf(maxnc, __shfl_xor_sync(0xffffffffu, maxnc, off));
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(candbar);  // completes once every candidate row has landed
      misc_i[0] = ncand;
      misc_f[1] = maxnc;
    }
  }
  if (!__syncthreads_and(ok)) {
    // let the copies already issued land before the CTA exits
    if (tid == 0) {
      for (int s = 0; s < nst; ++s) mbar_wait_bounded(&k1bar[s], 0, p.wait_limit_ns, ctl, 30);
      mbar_wait_bounded(candbar, 0, p.wait_limit_ns, ctl, 31);
    }
    return;
  }

  // ---------------------------------------------------------------- publish this CTA's record
  const int ncand = misc_i[0];
  if (warp == 0) {
    // exact moments of the slice, about its first score
    const float x0 = nr > 0 ? xs[0] : 0.f;
    float acc = 0.f;
    for (int i = lane; i < nr; i += 32) acc += xs[i] - x0;
    acc = __shfl_sync(0xffffffffu, warp_sum(acc), 0);
    const float mean = nr > 0 ? x0 + acc / static_cast<float>(nr) : 0.f;
    float m2 = 0.f;
    for (int i = lane; i < nr; i += 32) {
      const float c = xs[i] - mean;
      m2 += c * c;
    }
    m2 = warp_sum(m2);
    if (lane == 0) p.hdr[cta] = make_float4(mean, m2, misc_f[1], __int_as_float(ncand));
  }
  if (p.x_out != nullptr)
    for (int i = tid; i < nr; i += kThreads) p.x_out[n0 + i] = xs[i];
  // a = <K2[i,:], q[r:]> of every candidate, from the rows already in shared memory
  if (!mbar_wait_bounded(candbar, 0, p.wait_limit_ns, ctl, 60)) ok = false;
  if (ok) {
    unsigned char* myent = p.ent + static_cast<size_t>(cta) * p.cap * kEntryBytes;
    for (int u = warp; u < ncand; u += kWarps) {
      const float a = warp_row_dot<false>(cand + static_cast<size_t>(u) * p.d2, qs + p.r, p.d2);
      if (lane == 0) {
        unsigned char* e = myent + u * kEntryBytes;
        reinterpret_cast<int*>(e)[0] = n0 + cidx[u];
        reinterpret_cast<float*>(e)[1] = xs[cidx[u]];
        reinterpret_cast<float*>(e)[2] = a;
      }
    }
  }
  if (!__syncthreads_and(ok)) return;

  // ---------------------------------------------------------------- exchange
  float4* hdr_s = reinterpret_cast<float4*>(region_a + L.hdr_off);
  unsigned char* ent_s = region_a + L.ent_off;
  if (tid == 0) {
    const unsigned epoch = static_cast<unsigned>(misc_i[20]);
    unsigned* cnt = &ctl->dec_arrive[epoch & 1u];
    red_add_release_gpu(cnt, 1u);
    misc_i[1] = wait_count_geq(ctl, cnt, static_cast<unsigned>(G) + (p.never_arrive ? 1u : 0u), p.wait_limit_ns, 1)
                    ? 1
                    : 0;
    // every CTA has read the launch number by now: advance it for the next launch
    if (misc_i[1] && cta == 0) ctl->epoch = epoch + 1u;
    if (misc_i[1]) {
      // the records were written with generic stores by other CTAs; order them
      // before this thread's async-proxy (bulk copy) reads
      asm volatile("fence.proxy.async.global;" ::: "memory");
      const unsigned hbytes = static_cast<unsigned>(G) * 16;
      const unsigned ebytes = static_cast<unsigned>(G) * p.cap * kEntryBytes;
      mbar_arrive_expect_tx(recbar, hbytes + ebytes);
      bulk_g2s(hdr_s, p.hdr, hbytes, recbar);
      constexpr unsigned kChunk = 32768;
      for (unsigned o = 0; o < ebytes; o += kChunk)
        bulk_g2s(ent_s + o, p.ent + o, ebytes - o < kChunk ? ebytes - o : kChunk, recbar);
    }
  }
  __syncthreads();
  if (!misc_i[1]) return;
  if (!__syncthreads_and(mbar_wait_bounded(recbar, 0, p.wait_limit_ns, ctl, 61))) return;

  // theta: every CTA merges all CTAs' moments in CTA order
  if (warp == 0) {
    float4 h[8];
    float n_c[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = lane + 32 * j;
      h[j] = c < G ? hdr_s[c] : make_float4(0.f, 0.f, 0.f, 0.f);
      n_c[j] = c < G ? static_cast<float>(rows_of(c, p.rpc, p.d_ff)) : 0.f;
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) s = fmaf(n_c[j], h[j].x, s);
    s = __shfl_sync(0xffffffffu, warp_sum(s), 0);
    const float mean = s / static_cast<float>(p.d_ff);
    float m2 = 0.f;
    bool miss = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float dm = h[j].x - mean;
      m2 += h[j].y + n_c[j] * dm * dm;
    }
    m2 = warp_sum(m2);
    const float th = __shfl_sync(0xffffffffu, fmaf(sqrtf(fmaxf(m2, 0.f) / static_cast<float>(p.d_ff)), p.Q, mean), 0);
    // a CTA whose largest non-candidate score passes theta needs the recompute path
#pragma unroll
    for (int j = 0; j < 8; ++j) miss |= (lane + 32 * j < G) && h[j].z > th;
    miss = __any_sync(0xffffffffu, miss);
    if (lane == 0) {
      misc_f[0] = th;
      misc_i[2] = miss ? 1 : 0;
      if (cta == 0 && p.theta_out != nullptr) p.theta_out[0] = th;
    }
  }
  __syncthreads();
  const float theta = misc_f[0];
  if (p.active_out != nullptr)
    for (int i = tid; i < nr; i += kThreads) p.active_out[n0 + i] = xs[i] > theta ? 1 : 0;

  // Entries used by the gather: (index, x, a) per source CTA in ascending neuron
  // order, `stride` slots per CTA, counts in hdr_s[c].w.  Normally these are the
  // published candidates; the recompute path rewrites them (every neuron with
  // x > theta, from K1 / K2 in global memory with the same arithmetic as phase 1
  // and the candidate dots), so both paths feed identical values to the gather.
  int stride = p.cap;
  if (misc_i[2]) {
    stride = p.rpc;
    int* wact = misc_i + 4;
    for (int c = 0; c < G; ++c) {
      const int rows = rows_of(c, p.rpc, p.d_ff);
      int cnt = 0;
      for (int base = 0; base < rows; base += kWarps) {
        const int li = base + warp;
        float x = 0.f, a = 0.f;
        bool act = false;
        if (li < rows) {
          const size_t row = static_cast<size_t>(c) * p.rpc + li;
          x = __shfl_sync(0xffffffffu, warp_row_dot<true>(p.K1 + row * p.r, qs, p.r), 0);
          if (x > theta) {
            a = warp_row_dot<true>(p.K2 + row * p.d2, qs + p.r, p.d2);
            act = true;
          }
        }
        if (lane == 0) {
          wact[warp] = act ? 1 : 0;
          red[2 * warp] = x;
          red[2 * warp + 1] = a;
        }
        __syncthreads();
        for (int w = 0; w < kWarps; ++w) {
          if (wact[w]) {
            if (tid == 0) {
              unsigned char* e = ent_s + (static_cast<size_t>(c) * stride + cnt) * kEntryBytes;
              reinterpret_cast<int*>(e)[0] = c * p.rpc + base + w;
              reinterpret_cast<float*>(e)[1] = red[2 * w];
              reinterpret_cast<float*>(e)[2] = red[2 * w + 1];
            }
            ++cnt;
          }
        }
        __syncthreads();
      }
      if (tid == 0) hdr_s[c].w = __int_as_float(cnt);
    }
    __syncthreads();
  }

  // ---------------------------------------------------------------- column gather
  // CTA c owns output columns [c*CW, (c+1)*CW).  Thread group g sums the active
  // entries of source CTAs g, g + groups, ... in ascending neuron order; then a
  // fixed-order reduction over the groups.
  if (cta < p.n_col_ctas) {
    const int col0 = cta * p.col_width;
    const int ncol = min(p.col_width, p.d_model - col0);
    const int cpr = p.col_width / 8;  // 16-byte chunks per row (power of two, <= 32)
    const int cc = tid % cpr;
    const int groups = kThreads / cpr;
    const bool col_ok = cc * 8 < ncol;
    constexpr int kBatch = 16;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    if (col_ok) {
      const uint16_t* vbase = p.V + col0 + cc * 8;
      for (int src = tid / cpr; src < G; src += groups) {
        const int cnt = __float_as_int(hdr_s[src].w);
        const unsigned char* es = ent_s + static_cast<size_t>(src) * stride * kEntryBytes;
        for (int j0 = 0; j0 < cnt; j0 += kBatch) {
          // branch-free: read kBatch entries, form every h independently, mask
          // the inactive ones, then issue all loads, then the FMAs
          float h[kBatch];
          int ix[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const int j = j0 + u;
            const unsigned char* e = es + (j < cnt ? j : 0) * kEntryBytes;
            const float sx = j < cnt ? reinterpret_cast<const float*>(e)[1] - theta : -1.f;
            const bool act = sx > 0.f;
            const float g = gelu_tanh(fmaxf(sx, 0.f)) * reinterpret_cast<const float*>(e)[2];
            // fma(-0, 0, acc) == acc exactly, so inactive slots change no bit
            h[u] = act ? g : -0.f;
            ix[u] = act ? reinterpret_cast<const int*>(e)[0] : -1;
          }
          uint4 v[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
            v[u] = ix[u] >= 0 ? ldg_nc128(vbase + static_cast<size_t>(ix[u]) * p.d_model) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const float2 v0 = bf16x2_to_float2(v[u].x), v1 = bf16x2_to_float2(v[u].y);
            const float2 v2 = bf16x2_to_float2(v[u].z), v3 = bf16x2_to_float2(v[u].w);
            acc[0] = fmaf(h[u], v0.x, acc[0]);
            acc[1] = fmaf(h[u], v0.y, acc[1]);
            acc[2] = fmaf(h[u], v1.x, acc[2]);
            acc[3] = fmaf(h[u], v1.y, acc[3]);
            acc[4] = fmaf(h[u], v2.x, acc[4]);
            acc[5] = fmaf(h[u], v2.y, acc[5]);
            acc[6] = fmaf(h[u], v3.x, acc[6]);
            acc[7] = fmaf(h[u], v3.y, acc[7]);
          }
        }
      }
    }
    // fixed-order reduction: xor butterfly over lanes with equal lane % cpr, then warps in order
    for (int off = 16; off >= cpr; off >>= 1)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    if (lane < cpr)
#pragma unroll
      for (int j = 0; j < 8; ++j) red[(warp * cpr + lane) * 8 + j] = acc[j];
    __syncthreads();
    for (int o = tid; o < ncol; o += kThreads) {
      const int ch = o / 8, j = o % 8;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += red[(w * cpr + ch) * 8 + j];
      const __nv_bfloat16 b = __float2bfloat16_rn(sum);
      if (p.out != nullptr) p.out[col0 + o] = *reinterpret_cast<const uint16_t*>(&b);
      if (p.h_in != nullptr) p.h_out[col0 + o] = hsm[col0 + o] + __bfloat162float(b);
    }
  }
  // No exit bookkeeping: the next launch counts on the other parity's counters,
  // which CTA 0 of this launch has already cleared.
}

}  // namespace

DecodePlan plan_decode(int d_model, int r, int d_ff, int num_sms, size_t smem_optin, int cap_override) {
  DecodePlan pl{};
  pl.ok = false;
  const int d2 = d_model - r;
  if (r > 32 * 8 * kFusedMaxChunks || d2 > 32 * 8 * kFusedMaxChunks) return pl;
  int rpc = (d_ff + num_sms - 1) / num_sms;
  rpc = static_cast<int>(align_up(static_cast<size_t>(rpc), kRowsPerStage));
  if (rpc > 256) return pl;
  const int grid = (d_ff + rpc - 1) / rpc;
  if (grid > 256) return pl;
  int cw = 8;
  while ((d_model + cw - 1) / cw > grid) cw *= 2;
  if (cw > 256) return pl;
  int cap = cap_override >= 0 ? cap_override : 24;
  if (cap > rpc) cap = rpc;
  cap &= ~3;  // entries of all CTAs form whole 16-byte units
  while (cap > 0 && DecLayout(d_model, r, rpc, grid, cap).total > smem_optin) cap -= 4;
  if (cap < 8 && cap_override < 0) return pl;  // too little room to speculate: use the other kernel
  if (DecLayout(d_model, r, rpc, grid, cap).total > smem_optin) return pl;
  pl.grid = grid;
  pl.rows_per_cta = rpc;
  pl.cap = cap;
  pl.col_width = cw;
  pl.n_col_ctas = (d_model + cw - 1) / cw;
  pl.smem_bytes = DecLayout(d_model, r, rpc, grid, cap).total;
  pl.ws_bytes = DecWs(grid, cap).total;
  pl.ok = true;
  return pl;
}

cudaError_t launch_decode(const DecodePlan& pl, const FusedArgs& a, cudaStream_t stream) {
  const DecWs W(pl.grid, pl.cap);
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  DParams p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.K1 = static_cast<const uint16_t*>(a.K1);
  p.K2 = static_cast<const uint16_t*>(a.K2);
  p.V = static_cast<const uint16_t*>(a.V);
  p.out = static_cast<uint16_t*>(a.out);
  p.d_model = a.d_model;
  p.r = a.r;
  p.d2 = a.d_model - a.r;
  p.d_ff = a.d_ff;
  p.rpc = pl.rows_per_cta;
  p.cap = pl.cap;
  p.col_width = pl.col_width;
  p.n_col_ctas = pl.n_col_ctas;
  p.Q = a.Q;
  p.x_out = a.x_out;
  p.theta_out = a.theta_out;
  p.active_out = a.active_out;
  p.h_in = a.h_in;
  p.h_out = a.h_out;
  p.eps = a.eps;
  p.q_dbg = static_cast<uint16_t*>(a.q_dbg);
  p.ctl = reinterpret_cast<DeviceControl*>(ws);
  p.s0 = reinterpret_cast<float4*>(ws + W.s0);
  p.hdr = reinterpret_cast<float4*>(ws + W.hdr);
  p.ent = ws + W.ent;
  p.wait_limit_ns = a.wait_limit_ns;
  p.never_arrive = a.never_arrive;
  static size_t smem_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (smem_set[dev] < pl.smem_bytes) {
    e = cudaFuncSetAttribute(spark_ffn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(pl.smem_bytes));
    if (e != cudaSuccess) return e;
    smem_set[dev] = pl.smem_bytes;
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
  return cudaLaunchKernelEx(&cfg, spark_ffn_decode_kernel, p);
}

}  // namespace spark
