// umma_gemm.cu -- batched (prefill) Spark FFN on the 5th-generation tensor cores.
//
// Spark Transformer notes, 关键设计 / "Spark FFN" and "Statistical Top-k", for T
// tokens at once:
//   GEMM 1  X = Q1 K1^T                 (predictor; x = K1^T q[:r] per token)
//           epilogue: x stored once, fp32, in 128 x 128 tiles, and the
//           per-(token, 128- or 64-neuron tile) moments of x
//   GEMM 2  A = Q2 K2^T
//           epilogue: theta per token from the tile moments, theta = mean +
//           std Q(1 - k/d_ff) (merged by the epilogue warps while the main loop
//           runs up to 64 tokens, else by theta_kernel before); then
//           h = GELU(max(x - theta, 0)) * a on x > theta, else 0, with x read
//           back from GEMM 1's tiles, split h = h_hi + h_lo into two bf16
//           matrices (h_lo = bf16(h - h_hi))
//   GEMM 3  out = H_hi V + H_lo V        (V read once per k-block for both halves)
//           epilogue: bf16 out, or fp32 split-K partials reduced in fixed order.
//
// With independent tokens the union of the per-token active sets covers almost
// every neuron once a 128-token tile is formed (1 - 0.92^128), so the masked
// products run as dense tiles.  Restricting GEMM 3 to the union's V rows -- by
// gathering them (TMA tile::gather4 over compacted positions) or by zeroing the
// other rows in shared memory before the product -- measured slower at every
// prompt length, so every row of K2 and V is read (and must be finite).  h is
// split in two bf16 parts because a single bf16 rounding of h would add ~1.7e-3
// relative error on top of the bf16 output rounding and break the 2e-3
// relative-L2 target.
//
// One kernel template serves the three GEMMs: a persistent grid (one CTA per
// SM), warp 0 = producer (TMA copies of 128B-swizzled K-major tiles, V read
// N-major; GEMM 3's h blocks by 1-D bulk copies, already in operand order),
// warp 1 = TMEM allocator and single-thread tcgen05.mma issuer (M 128, N 128 or
// 256, K 16 per instruction, fp32 accumulators in TMEM, two accumulators so
// that the epilogue of one tile overlaps the main loop of the next), the
// remaining warps = epilogue (tcgen05.ld, 32 TMEM lanes per warp).  A unit is
// 128 tokens x 128 columns, x 256 once there are enough to fill the SMs, or x 64
// for GEMMs 1 and 2 with a single band of 65-128 tokens (more CTAs streaming the
// weights).  The predictor entry point writes x row-major by TMA tensor stores.
// Every wait is bounded.
//
// Each GEMM is launched as a programmatic dependent of the kernel before it:
// barrier set-up and the TMEM allocation overlap that kernel's tail, and nothing
// touches global memory before griddepcontrol.wait (measured 42.3 -> 39.8 us per
// call at 16 tokens, 13.8 -> 12.8 us for the predictor alone at 256) -- except
// GEMM 2's producer and MMA warps, whose operands do not depend on GEMM 1: up to
// 64 tokens the two GEMMs use 72 SMs each, so GEMM 2's main loop runs beside
// GEMM 1 and only its epilogue waits (40.3 -> 37.4 us per call at 16 tokens).
// Where theta_kernel runs between them it is launched the same way and releases
// GEMM 2 at once (T = 128 47.0 -> 42.8 us, T = 256 57.1 -> 54.9); so does the
// split-K reduce behind GEMM 3 (T = 256 54.9 -> 53.3 us).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "spark_device.cuh"
#include "spark_internal.h"

namespace spark {

#ifdef SPARK_DEBUG
// bounds-check violations of this file's kernels (see SPARK_CHECK)
static __device__ unsigned g_bounds_violations;
#endif

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 64;
// warp 0: TMA producer; warp 1: TMEM owner and MMA issuer; the rest: epilogue.
// GEMM 2's gate epilogue (GELU, split, score loads: a chain of dependent
// latencies per element) runs sixteen epilogue warps, four per TMEM lane
// quarter, each on its own quarter of the unit's columns; GEMM 1's runs eight,
// two per quarter, each on half of the columns (its score stores were the
// longest phase of a one-unit launch: the predictor alone at T = 256 11.9 ->
// 10.9 us together with 128-byte store rows); GEMM 3's runs four.
__host__ __device__ constexpr int epi_warps(int epi) { return epi == 2 ? 16 : epi == 1 ? 8 : 4; }
__host__ __device__ constexpr int gemm_threads(int epi) { return 64 + 32 * epi_warps(epi); }
constexpr int kABytes = BM * BK * 2;  // 16 KB
constexpr int kBBytes = BN * BK * 2;  // 16 KB

enum Epilogue : int { kEpiPredictor = 1, kEpiGate = 2, kEpiOut = 3 };

struct GemmParams {
  int M, N, K;
  int tiles_m, tiles_n, split_k, kb_per_split, nkb, units;
  float* X;               // optional predictor scores [M][N] fp32, row-major (predictor and debug entry points)
  float4* Xt;             // predictor scores in 128 x 128 tiles: written by GEMM 1, read by GEMM 2
  int xt_tiles_n;         // 128-column tiles per 128-row band of Xt
  float2* moments;        // [M][mom_stride] (mean, M2) of each 128-neuron tile
  int mom_stride;         // neuron tiles per row of moments
  int mom_w;              // neurons per moments tile: 128, or 64 with 64-column units
  const float* theta;     // [M] thresholds from theta_kernel, or nullptr: GEMM 2's epilogue derives them
  float Q;                // standard-normal quantile Q(1 - k/d_ff) of the threshold
  float* theta_out;       // optional [M]: the thresholds GEMM 2 derived (debug entry point)
  uint16_t* h_hi;         // bf16, blocked: see h_block()
  uint16_t* h_lo;         // bf16, blocked like h_hi
  int h_kb;               // 64-neuron blocks per 128-token band of h_hi / h_lo
  unsigned char* active;  // optional [M][N]
  float* part;            // GEMM 3 split-K partials [split][M][N]
  uint16_t* out;          // GEMM 3 bf16 output [M][N] when split_k == 1
  DeviceControl* ctl;
  unsigned long long wait_limit_ns;
  int x_tma;              // predictor: X row-major through TMA stores (tensor map in the fourth map slot)
  int early_main;         // GEMM 2: producer and MMA warps start before the kernel ahead completes
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// TMA store of a shared-memory box to a tensor-map region (bulk async group)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, int c0, int c1, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(c0), "r"(c1), "r"(smem_u32(src))
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (one wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Shared-memory matrix descriptors (tcgen05 "version 1"), 128-byte swizzle.
// K-major: rows of 128 B (64 bf16 along K), 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}
// K-major without swizzle: 8-row x 16-byte core matrices, 128 B each; lbo bytes
// between the two core matrices of one K 16 step, sbo bytes between 8-row groups.
__device__ __forceinline__ uint64_t desc_kmajor_none(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// N-major: 64 bf16 along N per 128-byte row, one row per K index, 8-row atoms
// 1024 B apart along K; the two 64-wide N halves of the tile are lbo bytes apart.
__device__ __forceinline__ uint64_t desc_nmajor_sw128(uint32_t saddr, uint32_t lbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D, M = 128, N = n.
__host__ __device__ constexpr uint32_t make_idesc(bool b_nmajor, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_nmajor ? 1u : 0u) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(BM >> 4) << 24);
}

__device__ __forceinline__ uint16_t f2bf(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 b) { return *reinterpret_cast<const uint32_t*>(&b); }


// Unit order: GEMMs 1 and 2 walk the token tiles under one neuron tile, so the
// weight tile (K1 / K2 rows, read once from HBM) is shared by consecutive units
// while the small token operand stays in L2.  GEMM 3 walks the output columns
// under one token tile: its A operand (h, T x d_ff, larger than L2 at long
// prompts) is then read from HBM once, and V (d_ff x d_model) stays in L2.
template <int EPI>
__device__ __forceinline__ void decode_unit(const GemmParams& p, int unit, int& tm, int& tn, int& kb0, int& kb1) {
  const int per_split = p.tiles_m * p.tiles_n;
  const int split = unit / per_split;
  const int rem = unit % per_split;
  if (EPI == kEpiOut) {
    tm = rem / p.tiles_n;
    tn = rem % p.tiles_n;
  } else {
    tn = rem / p.tiles_m;
    tm = rem % p.tiles_m;
  }
  kb0 = split * p.kb_per_split;
  kb1 = min(p.nkb, kb0 + p.kb_per_split);
}

// Tiled score layout: the 128 x 128 tile (tm, tn) is 64 KB contiguous; inside
// it, float4 i (columns 4i..4i+3) of row `row` sits at [i][row], so that the 32
// lanes of an epilogue warp (32 consecutive rows) store or load 512 contiguous
// bytes per instruction.
__device__ __forceinline__ float4* xt_tile(const GemmParams& p, int tm, int nb) {
  return p.Xt + (static_cast<size_t>(tm) * p.xt_tiles_n + nb / BN) * (BN / 4) * BM;
}

// The gated activations h_hi / h_lo (the A operand of GEMM 3) are stored in
// blocks of 128 tokens x 64 neurons, 16 KB contiguous each, block (tm, kb) at
// (tm * h_kb + kb) * 16 KB; inside a block, 16-byte chunk c (neurons 8c..8c+7)
// of token row r sits at c * 2048 + r * 16.  That is the tensor core's K-major
// no-swizzle operand layout as it stands, so GEMM 3 fetches a block with one
// bulk copy, and the 32 lanes of a GEMM 2 epilogue warp (32 consecutive rows)
// store 512 contiguous bytes per instruction.
constexpr int kHBlockBytes = BM * BK * 2;  // 16 KB
__device__ __forceinline__ uint4* h_block(uint16_t* h, const GemmParams& p, int tm, int kb) {
  return reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(h) +
                                  (static_cast<size_t>(tm) * p.h_kb + kb) * kHBlockBytes);
}

// GEMM 2 epilogue: float4 group i of row `row` of the scores [nb, nb + 128), as
// GEMM 1 stored them (N is a multiple of 16: a group of four is wholly inside)
__device__ __forceinline__ float4 gate_x(const GemmParams& p, const float4* tile, int row, int nb, int i) {
  return nb + 4 * i < p.N && SPARK_CHECK(nb / BN < p.xt_tiles_n) ? __ldcg(tile + i * BM + row)
                                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// theta of token m from the per-(token, 128-neuron tile) moments of GEMM 1: the
// four gate epilogue warps that share TMEM lane quarter `quarter` (and so this
// row) each merge a quarter of the tiles, weighted mean first, then
// M2 = sum_j M2_j + n_j (mean_j - mean)^2; the partials are combined through
// shared memory (tred, 8 x 128 floats) in warp order, so every warp gets the
// same bits.  All four warps must call it.
__device__ __forceinline__ float gate_theta(const GemmParams& p, int m, int row, int colgrp, int quarter,
                                            float* tred) {
  const int tiles = p.mom_stride;
  const int j0 = colgrp * tiles / 4, j1 = (colgrp + 1) * tiles / 4;
  const bool ok = m < p.M;
  const float2* mr = p.moments + static_cast<size_t>(ok ? m : 0) * p.mom_stride;
  // loads in batches of 8, all of a batch in flight before its arithmetic
  constexpr int kB = 8;
  float s = 0.f;
  for (int jb = j0; jb < j1; jb += kB) {
    float2 mm[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) mm[u] = (ok && jb + u < j1) ? mr[jb + u] : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kB; ++u)
      if (jb + u < j1) s = fmaf(static_cast<float>(min(p.mom_w, p.N - (jb + u) * p.mom_w)), mm[u].x, s);
  }
  tred[colgrp * BM + row] = s;
  named_bar_sync(1 + quarter, 128);
  const float mean = (((tred[row] + tred[BM + row]) + tred[2 * BM + row]) + tred[3 * BM + row]) / static_cast<float>(p.N);
  float m2 = 0.f;
  for (int jb = j0; jb < j1; jb += kB) {
    float2 mm[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) mm[u] = (ok && jb + u < j1) ? mr[jb + u] : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kB; ++u)
      if (jb + u < j1) {
        const float d = mm[u].x - mean;
        m2 += mm[u].y + static_cast<float>(min(p.mom_w, p.N - (jb + u) * p.mom_w)) * d * d;
      }
  }
  tred[(4 + colgrp) * BM + row] = m2;
  named_bar_sync(1 + quarter, 128);
  const float M2 = ((tred[4 * BM + row] + tred[5 * BM + row]) + tred[6 * BM + row]) + tred[7 * BM + row];
  return fmaf(sqrtf(fmaxf(M2, 0.f) / static_cast<float>(p.N)), p.Q, mean);
}

// WIDE (GEMMs 1 and 2): a unit is 128 rows x 256 columns: each stage holds one
// A tile and two adjacent 128-row B tiles, and each K 16 step is one M 128 x
// N 256 instruction into 256 TMEM columns.
// A64 (GEMMs 1 and 2, at most 64 tokens): each stage holds only the 64 token
// rows that exist (an 8 KB A box) and the B tile right after it; the M 128
// instruction still reads 128 A rows, its rows 64..127 coming from the B tile's
// bytes, which only ever reach accumulator rows >= 64 -- rows no token owns,
// which the epilogue skips.  The 24 KB stages let 8 of them (128 KB of weights)
// be in flight instead of 6 (96 KB).
// NW (GEMMs 1 and 2, one 128-token band): a unit is 128 rows x 64 columns, so
// that twice as many CTAs stream the weights when there are only 72 128-column
// tiles; its scores fill half of a 128 x 128 score tile and its moments cover
// 64 neurons.
template <int EPI, bool B_NMAJOR, bool DUAL, int STAGES, bool WIDE = false, bool A64 = false, bool NW = false>
__global__ void __launch_bounds__(gemm_threads(EPI), 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                     const GemmParams p) {
  static_assert(!WIDE || B_NMAJOR == (EPI == kEpiOut), "wide GEMM 3 takes V N-major; GEMMs 1 and 2 K-major");
  static_assert(!DUAL || EPI == kEpiOut, "two A operands (h_hi, h_lo) are GEMM 3's");
  static_assert(!A64 || (EPI != kEpiOut && !WIDE), "64-row A boxes: narrow GEMMs 1 and 2 only");
  static_assert(!NW || (!WIDE && EPI != kEpiOut), "64-column units: GEMMs 1 and 2 only");
  constexpr int kBTiles = WIDE ? 2 : 1;
  constexpr int kUC = WIDE ? 2 * BN : (NW ? BN / 2 : BN);  // columns of one unit
  constexpr int kHalf = WIDE ? BN : kUC;                     // columns per B tile
  constexpr int kBB = kHalf * BK * 2;                        // bytes of one K-major B tile
  constexpr int kAB = A64 ? kABytes / 2 : kABytes;  // bytes of one stage's A box
  constexpr int kStageBytes = kAB * (DUAL ? 2 : 1) + (EPI == kEpiOut ? kBBytes : kBB) * kBTiles;
  constexpr int kAccCols = kUC;  // TMEM columns of one tile's accumulators
  constexpr int kTmemCols = 2 * kAccCols;       // double buffered
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* tred = reinterpret_cast<float*>(smem + STAGES * kStageBytes + 256);  // GEMM 2: theta partials

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  DeviceControl* ctl = p.ctl;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * epi_warps(EPI));
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above touches no global memory, so it may overlap the tail of the
  // kernel ahead of this one on the stream (a programmatic launch).  GEMM 2's
  // operands (q[r:] and K2) do not depend on GEMM 1, which lets it launch only
  // after its own wait: with early_main GEMM 2's producer and MMA warps start at
  // once and only its epilogue waits (for GEMM 1's scores and moments).
  // Otherwise everything below runs once the kernel ahead has completed and its
  // writes are visible.
  if (EPI == kEpiGate && p.early_main) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  } else {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  if (tid == 0 && ld_relaxed_gpu(&ctl->abort)) *abort_flag = 1;
  __syncthreads();

  if (*abort_flag) {
    // an earlier launch on this workspace gave up: nothing is issued
  } else if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t ph = 0;
    int issued = 0;
    bool ok = true;
    for (int unit = blockIdx.x; ok && unit < p.units; unit += gridDim.x) {
      int tm, tn, kb0, kb1;
      decode_unit<EPI>(p, unit, tm, tn, kb0, kb1);
      if (EPI == kEpiGate) {
        // the gate epilogue reads this unit's score tiles a whole main loop from
        // now: pull them into L2 (a 64 KB tile is contiguous)
#pragma unroll
        for (int h = 0; h < kBTiles; ++h) {
          const int cb = tn * kUC + h * BN;  // a 64-column unit's scores are half of a tile
          if (cb < p.N) prefetch_l2_bulk(xt_tile(p, tm, cb) + cb % BN / 4 * BM, BM * kHalf * 4);
        }
      }
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], ph ^ 1u, p.wait_limit_ns, ctl, 100) || *abort_flag) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        unsigned char* sa = smem + stage * kStageBytes;
        mbar_arrive_expect_tx(&full[stage], kStageBytes);
        unsigned char* sb = sa + kAB * (DUAL ? 2 : 1);
        if (EPI == kEpiOut) {
          // h_hi and h_lo blocks: already in the operand layout (a failed check
          // copies block (0, 0) so the byte count still matches the barrier)
          const bool hb_ok = SPARK_CHECK(tm < p.tiles_m && kb < p.h_kb);
          bulk_g2s(sa, h_block(p.h_hi, p, hb_ok ? tm : 0, hb_ok ? kb : 0), kHBlockBytes, &full[stage]);
          bulk_g2s(sa + kABytes, h_block(p.h_lo, p, hb_ok ? tm : 0, hb_ok ? kb : 0), kHBlockBytes, &full[stage]);
        } else {
          tma_load_2d(sa, &tmA, kb * BK, tm * BM, &full[stage]);
          if (DUAL) tma_load_2d(sa + kABytes, &tmA2, kb * BK, tm * BM, &full[stage]);
        }
        if (B_NMAJOR) {
          // V rows kb*64.. as 64-column boxes, 8 KB apart (two per 128 columns)
#pragma unroll
          for (int h = 0; h < 2 * kBTiles; ++h)
            tma_load_2d(sb + h * (kBBytes / 2), &tmB, tn * BN * kBTiles + h * 64, kb * BK, &full[stage]);
        } else {
#pragma unroll
          for (int h = 0; h < kBTiles; ++h)
            tma_load_2d(sb + h * kBB, &tmB, kb * BK, tn * kUC + h * BN, &full[stage]);
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          ph ^= 1u;
        }
      }
    }
    if (ok) {
      // tail: wait until the MMA warp has released every stage, so that no
      // commit arrives on a barrier after the CTA has exited
      for (int i = 0; i < STAGES; ++i) {
        if (!mbar_wait_bounded(&empty[stage], ph ^ 1u, p.wait_limit_ns, ctl, 102)) break;
        if (++stage == STAGES) {
          stage = 0;
          ph ^= 1u;
        }
      }
    } else {
      // let the copies already issued land before the CTA can exit
      int s = stage;
      uint32_t q = ph;
      for (int i = 0; i < STAGES && i < issued; ++i) {
        if (--s < 0) {
          s = STAGES - 1;
          q ^= 1u;
        }
        mbar_wait_bounded(&full[s], q, p.wait_limit_ns, ctl, 101);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    // a wide unit is one M 128 x N 256 instruction per K 16 step: its two B tiles
    // are adjacent in shared memory, 8-row atoms 1024 B apart throughout
    constexpr uint32_t idesc = make_idesc(B_NMAJOR, kUC);
    int stage = 0;
    uint32_t ph = 0;
    uint32_t uses[2] = {0u, 0u};
    int acc = 0;
    bool ok = true;
    for (int unit = blockIdx.x; ok && unit < p.units; unit += gridDim.x) {
      int tm, tn, kb0, kb1;
      decode_unit<EPI>(p, unit, tm, tn, kb0, kb1);
      if (!mbar_wait_bounded(&tempty[acc], (uses[acc] & 1u) ^ 1u, p.wait_limit_ns, ctl, 110) || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
      for (int kb = kb0; kb < kb1; ++kb) {
        const bool first = kb == kb0;
        if (!mbar_wait_bounded(&full[stage], ph, p.wait_limit_ns, ctl, 111) || *abort_flag) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * kStageBytes);
        const uint32_t sb = sa + kAB * (DUAL ? 2 : 1);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t bdesc = B_NMAJOR ? desc_nmajor_sw128(sb + k * 16 * 128, kBBytes / 2)
                                          : desc_kmajor_sw128(sb + k * 32);
          // GEMM 3's A: chunks 2k and 2k + 1 of the h block (2048 B apart), 8-row groups 128 B apart
          const uint64_t adesc = EPI == kEpiOut ? desc_kmajor_none(sa + k * 4096, 2048, 128)
                                                : desc_kmajor_sw128(sa + k * 32);
          umma_bf16(d_tmem, adesc, bdesc, idesc, (!first || k > 0) ? 1u : 0u);
          if (DUAL) umma_bf16(d_tmem, desc_kmajor_none(sa + kABytes + k * 4096, 2048, 128), bdesc, idesc, 1u);
        }
        umma_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(&tfull[acc]);
      ++uses[acc];
      acc ^= 1;
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32 quarter, 32 quarter + 32)
    const int row = quarter * 32 + lane;
    const int colgrp = (warp - 2) >> 2;  // gate epilogue: which quarter of the columns
    if (EPI == kEpiGate && p.early_main) asm volatile("griddepcontrol.wait;" ::: "memory");
    uint32_t uses[2] = {0u, 0u};
    int acc = 0;
    for (int unit = blockIdx.x; unit < p.units; unit += gridDim.x) {
      int tm, tn, kb0, kb1;
      decode_unit<EPI>(p, unit, tm, tn, kb0, kb1);
      const int m = tm * BM + row;
      const int n_base = tn * kUC;
      const bool row_ok = m < p.M;
      // GEMM 2: this warp's columns of the tile (a wide unit's half, or half of a
      // narrow unit) and this row's scores there, stored by GEMM 1, loaded while
      // the accumulator is still being formed
      constexpr int kGateCols = kUC / (epi_warps(kEpiGate) / 4);
      const int gcol = colgrp * kGateCols;                // first column within the unit
      const int gtile_nb = (n_base + gcol) / BN * BN;     // first column of its score tile
      const int gx0 = (n_base + gcol) % BN / 4;           // its first float4 group in that tile
      float4 xr[EPI == kEpiGate ? kGateCols / 4 : 1];
      float th = 0.f;
      if (EPI == kEpiGate) {
        const float4* t0 = xt_tile(p, tm, gtile_nb);
#pragma unroll
        for (int i = 0; i < kGateCols / 4; ++i) xr[i] = gate_x(p, t0, row, gtile_nb, gx0 + i);
        if (WIDE || p.theta != nullptr) {  // wide units: always several per CTA, theta_kernel ran
          th = row_ok ? p.theta[m] : 0.f;
        } else {
          // the threshold of this row, while the accumulator is still being formed
          th = gate_theta(p, m, row, colgrp, quarter, tred);
          if (p.theta_out != nullptr && colgrp == 0 && row_ok) p.theta_out[m] = th;
        }
      }
      if (!mbar_wait_bounded(&tfull[acc], uses[acc] & 1u, p.wait_limit_ns, ctl, 120) || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      float v[16];
      if (EPI == kEpiPredictor) {
        // two warps per TMEM lane quarter, each on half of the unit's columns: a
        // wide unit's 128-column tile each, else half of the unit's one moments
        // tile (the two halves' sums and M2 are combined through shared memory)
        constexpr int kEpiCols = kUC / 2;
        const int col0 = colgrp * kEpiCols;                 // first unit column of this warp
        const int tile0 = WIDE ? n_base + col0 : n_base;    // first column of its moments tile
        // staging blocks 1024-byte aligned (the TMA store reads them 128-byte swizzled)
        float4* stg = reinterpret_cast<float4*>(smem + STAGES * kStageBytes + 1024) + (warp - 2) * 256;
        float* red = reinterpret_cast<float*>(smem + STAGES * kStageBytes + 1024 + epi_warps(EPI) * 4096);
        float sum = 0.f;
#pragma unroll 1
        for (int c = col0; c < col0 + kEpiCols; c += 32) {
          float w[32];
          tmem_ld32(taddr + c, w);
          const int nc0 = n_base + c;
          if (p.X != nullptr && p.x_tma) {
            // lane l's 32 values go to row l of the warp's 32 x 32 staging block in the
            // 128-byte-swizzled order (16-byte chunk j at j ^ (l % 8)); one lane then
            // stores the block with one TMA instruction (rows >= M and columns >= N
            // are clipped by the tensor map)
            if (lane == 0) bulk_wait_read_all();  // the previous block has been read
            __syncwarp();
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8)
              stg[lane * 8 + (q8 ^ (lane & 7))] = make_float4(w[4 * q8], w[4 * q8 + 1], w[4 * q8 + 2], w[4 * q8 + 3]);
            fence_proxy_async_shared();
            __syncwarp();
            const int m0 = tm * BM + quarter * 32;
            if (lane == 0 && m0 < p.M && nc0 < p.N) tma_store_2d(&tmB2, nc0, m0, stg);
          } else if (p.X != nullptr) {
            // through shared memory: lane l's 32 values go to row l of a 32 x 32
            // staging block (16-byte chunks xor-swizzled by row), read back so that
            // one store instruction covers 4 rows x 128 contiguous bytes
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8)
              stg[lane * 8 + (q8 ^ (lane & 7))] = make_float4(w[4 * q8], w[4 * q8 + 1], w[4 * q8 + 2], w[4 * q8 + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = i * 4 + (lane >> 3), q8 = lane & 7;
              const float4 val = stg[rr * 8 + (q8 ^ (rr & 7))];
              const int mr = tm * BM + quarter * 32 + rr;
              const int nc = nc0 + 4 * q8;
              if (mr < p.M) {
                float* dst = p.X + static_cast<size_t>(mr) * p.N + nc;
                if (nc + 4 <= p.N) {
                  *reinterpret_cast<float4*>(dst) = val;
                } else {
                  if (nc < p.N) dst[0] = val.x;
                  if (nc + 1 < p.N) dst[1] = val.y;
                  if (nc + 2 < p.N) dst[2] = val.z;
                }
              }
            }
            __syncwarp();
          }
#pragma unroll
          for (int s = 0; s < 32; s += 16) {
            const float* v = w + s;
            const int n = nc0 + s;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (n + j < p.N) sum += v[j];
            if (row_ok && n < p.N && p.Xt != nullptr && SPARK_CHECK(tm < p.tiles_m && n / BN < p.xt_tiles_n)) {
              float4* xt = xt_tile(p, tm, n);
              const int g0 = n % BN / 4;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                xt[(g0 + q4) * BM + row] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            }
          }
        }
        if (p.moments != nullptr) {
          const int tw = WIDE ? BN : p.mom_w;  // columns of a moments tile
          const int cnt = tile0 < p.N ? min(tw, p.N - tile0) : 0;
          if (!WIDE) {
            red[colgrp * BM + row] = sum;
            named_bar_sync(1 + quarter, 64);
            sum = red[row] + red[BM + row];
          }
          const float mean = cnt > 0 ? sum / static_cast<float>(cnt) : 0.f;
          float m2 = 0.f;
#pragma unroll 1
          for (int c = col0; c < col0 + kEpiCols; c += 32) {
            float w[32];
            tmem_ld32(taddr + c, w);
            const int n = n_base + c;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < p.N) {
                const float d = w[j] - mean;
                m2 += d * d;
              }
          }
          if (!WIDE) {
            named_bar_sync(1 + quarter, 64);  // both halves' sums read before red is reused
            red[colgrp * BM + row] = m2;
            named_bar_sync(1 + quarter, 64);
            m2 = red[row] + red[BM + row];
            named_bar_sync(1 + quarter, 64);  // read before the next unit writes red
          }
          if (row_ok && tile0 < p.N && (WIDE || colgrp == 0))
            p.moments[static_cast<size_t>(m) * p.mom_stride + tile0 / tw] = make_float2(mean, m2);
        }
      } else if (EPI == kEpiGate) {
        {
          const int nb = n_base + gcol;
          const uint32_t ta = taddr + static_cast<uint32_t>(gcol);
#pragma unroll
          for (int c = 0; c < kGateCols; c += 16) {
            tmem_ld16(ta + c, v);  // a = K2^T q[r:]
            const int n = nb + c;
            const float x[16] = {xr[c / 4].x,     xr[c / 4].y,     xr[c / 4].z,     xr[c / 4].w,
                                 xr[c / 4 + 1].x, xr[c / 4 + 1].y, xr[c / 4 + 1].z, xr[c / 4 + 1].w,
                                 xr[c / 4 + 2].x, xr[c / 4 + 2].y, xr[c / 4 + 2].z, xr[c / 4 + 2].w,
                                 xr[c / 4 + 3].x, xr[c / 4 + 3].y, xr[c / 4 + 3].z, xr[c / 4 + 3].w};
            // rows < M are stored (rows >= M only ever reach output rows >= M,
            // whatever the block holds there); neurons in [N, next multiple of 64)
            // are stored as zeros, since GEMM 3 multiplies them with the zero rows
            // TMA fills in for V
            if (n >= (p.N + BK - 1) / BK * BK || !row_ok) continue;
            if (!SPARK_CHECK(tm < p.tiles_m && n / BK < p.h_kb)) continue;
            const bool col_ok = n < p.N;
            uint32_t hi[8], lo[8];
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              float h2[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const float sft = x[j + u] - th;
                h2[u] = col_ok && sft > 0.f ? gelu_tanh(sft) * v[j + u] : 0.f;
              }
              // h = h_hi + h_lo: round to bf16, then round the remainder (pairs packed
              // by one conversion each; element j in the low half)
              hi[j >> 1] = bf162_bits(__floats2bfloat162_rn(h2[0], h2[1]));
              const float2 hf = bf16x2_to_float2(hi[j >> 1]);
              lo[j >> 1] = bf162_bits(__floats2bfloat162_rn(h2[0] - hf.x, h2[1] - hf.y));
            }
            // N is a multiple of 16: a 16-column group is wholly inside or outside
            const int c8 = (n % BK) / 8;  // first of this group's two 16-byte chunks
            uint4* dh = h_block(p.h_hi, p, tm, n / BK);
            uint4* dl = h_block(p.h_lo, p, tm, n / BK);
            dh[c8 * BM + row] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            dh[(c8 + 1) * BM + row] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            dl[c8 * BM + row] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            dl[(c8 + 1) * BM + row] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            if (p.active != nullptr && row_ok && col_ok) {
              const size_t off = static_cast<size_t>(m) * p.N + n;
#pragma unroll
              for (int j = 0; j < 16; ++j) p.active[off + j] = x[j] - th > 0.f ? 1 : 0;
            }
          }
        }
      } else {  // kEpiOut
        const int split = unit / (p.tiles_m * p.tiles_n);
#pragma unroll 1
        for (int c = 0; c < BN * kBTiles; c += 16) {
          tmem_ld16(taddr + c, v);
          const int n = n_base + c;
          if (!row_ok) continue;
          if (p.split_k == 1) {
            uint16_t* orow = p.out + static_cast<size_t>(m) * p.N;
            if (n + 16 <= p.N) {
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                w[j] = static_cast<uint32_t>(f2bf(v[2 * j])) | (static_cast<uint32_t>(f2bf(v[2 * j + 1])) << 16);
              uint4* d = reinterpret_cast<uint4*>(orow + n);
              d[0] = make_uint4(w[0], w[1], w[2], w[3]);
              d[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
              for (int j = 0; j < 16; ++j)
                if (n + j < p.N) orow[n + j] = f2bf(v[j]);
            }
          } else {
            if (!SPARK_CHECK(split < p.split_k)) continue;
            float* prow = p.part + (static_cast<size_t>(split) * p.M + m) * p.N;
            if (n + 16 <= p.N) {
              float4* d = reinterpret_cast<float4*>(prow + n);
              d[0] = make_float4(v[0], v[1], v[2], v[3]);
              d[1] = make_float4(v[4], v[5], v[6], v[7]);
              d[2] = make_float4(v[8], v[9], v[10], v[11]);
              d[3] = make_float4(v[12], v[13], v[14], v[15]);
            } else {
              for (int j = 0; j < 16; ++j)
                if (n + j < p.N) prow[n + j] = v[j];
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      ++uses[acc];
      acc ^= 1;
    }
    if (EPI == kEpiPredictor && p.x_tma && lane == 0) bulk_wait_all();  // the TMA stores are done
  }

  // ------------------------------------------------------------ teardown
  // Warps 0 and 1 diverged (lane 0 produced / issued, lanes 1-31 came straight
  // here): reconverge them first, since __syncthreads is an aligned barrier that
  // every lane of a warp must reach together.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort_flag && lane == 0) {
      // wait (bounded) for every MMA issued so far before TMEM is released
      umma_commit(&tfull[0]);
      mbar_wait_bounded(&tfull[0], 0, p.wait_limit_ns, ctl, 130);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// theta per token from the tile moments: two passes over the partials
// (weighted mean, then M2 = sum M2_j + n_j (mean_j - mean)^2), fixed order.
__global__ void __launch_bounds__(128) theta_kernel(const float2* moments, int M, int N, int tiles_n, int mw,
                                                    float Q, float* theta, float* theta_out) {
  // launched programmatically behind GEMM 1: GEMM 2 (whose main loop needs no
  // theta) may launch at once; the moments are read after GEMM 1 has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 4 + warp;
  if (m >= M) return;
  const float2* mr = moments + static_cast<size_t>(m) * tiles_n;
  float s = 0.f;
  for (int j = lane; j < tiles_n; j += 32) {
    const float nj = static_cast<float>(min(mw, N - j * mw));
    s = fmaf(nj, mr[j].x, s);
  }
  s = __shfl_sync(0xffffffffu, warp_sum(s), 0);
  const float mean = s / static_cast<float>(N);
  float m2 = 0.f;
  for (int j = lane; j < tiles_n; j += 32) {
    const float nj = static_cast<float>(min(mw, N - j * mw));
    const float d = mr[j].x - mean;
    m2 += mr[j].y + nj * d * d;
  }
  m2 = warp_sum(m2);
  if (lane == 0) {
    const float th = fmaf(sqrtf(fmaxf(m2, 0.f) / static_cast<float>(N)), Q, mean);
    theta[m] = th;
    if (theta_out != nullptr) theta_out[m] = th;
  }
}

// out = bf16(sum over splits, in split order) of the GEMM 3 partials.
__global__ void splitk_reduce_kernel(const float* part, int splits, size_t n4, uint16_t* out) {
  // launched programmatically behind GEMM 3: resident while it finishes, reads
  // the partials once it has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float4 a = __ldcs(reinterpret_cast<const float4*>(part) + i);
    for (int s = 1; s < splits; ++s) {
      const float4 b = __ldcs(reinterpret_cast<const float4*>(part) + s * n4 + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    uint2 w;
    w.x = static_cast<uint32_t>(f2bf(a.x)) | (static_cast<uint32_t>(f2bf(a.y)) << 16);
    w.y = static_cast<uint32_t>(f2bf(a.z)) | (static_cast<uint32_t>(f2bf(a.w)) << 16);
    reinterpret_cast<uint2*>(out)[i] = w;
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows of
// `row_bytes`, box (box_inner x box_outer), 128-byte swizzle, zero fill.
bool make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [outer][inner] row-major, box (32 x 32), 128-byte swizzle: the predictor's X for TMA stores
bool make_tmap_x(CUtensorMap* tm, void* base, uint64_t inner, uint64_t outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int EPI, bool B_NMAJOR, bool DUAL, int STAGES, bool WIDE = false, bool A64 = false, bool NW = false>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b, const CUtensorMap& b2,
                        const GemmParams& p, int num_sms, cudaStream_t stream) {
  constexpr int kStageBytes = (A64 ? kABytes / 2 : kABytes) * (DUAL ? 2 : 1) + (NW ? kBBytes / 2 : kBBytes) * (WIDE ? 2 : 1);
  constexpr size_t smem = static_cast<size_t>(STAGES) * kStageBytes + 1024 + (EPI == kEpiPredictor ? 1024 : 256) +
                          (EPI == kEpiGate ? 8 * BM * 4 : 0) +
                          (EPI == kEpiPredictor ? epi_warps(EPI) * 4096 + 2 * BM * 4 : 0);
  auto kern = umma_gemm_kernel<EPI, B_NMAJOR, DUAL, STAGES, WIDE, A64, NW>;
  static int set_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (set_dev != dev) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    set_dev = dev;
  }
  const int grid = p.units < num_sms ? p.units : num_sms;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(gemm_threads(EPI));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, a2, b, b2, p);
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

size_t predictor_workspace_bytes(int, int) { return align256(sizeof(DeviceControl)); }

size_t prefill_workspace_bytes(int T, int d_model, int d_ff, int num_sms) {
  const int tiles_n = (d_ff + BN - 1) / BN;
  size_t b = align256(sizeof(DeviceControl));
  b += align256(static_cast<size_t>(T) * ((d_ff + 63) / 64) * sizeof(float2));  // moments (64-neuron tiles at most)
  b += align256(static_cast<size_t>(T) * 4);                                   // theta
  b += 2 * static_cast<size_t>((T + BM - 1) / BM) * ((d_ff + BK - 1) / BK) * BM * BK * 2;  // h_hi, h_lo
  b += static_cast<size_t>((T + BM - 1) / BM) * tiles_n * BM * BN * 4;         // tiled scores
  const int splits = prefill_splitk(T, d_model, d_ff, num_sms);
  if (splits > 1) b += align256(static_cast<size_t>(splits) * T * d_model * 4);  // partials
  return b;
}

// GEMM 3 runs 128 x 256 units (one N 256 instruction per K 16 step, both A
// halves on each V tile) once there are about a third as many of them as SMs
// (measured at the Gemma shape: better from T = 1024 on, worse at T <= 256,
// where the wide units need twice the split-K partials); below that the narrow
// 128 x 128 units.
bool prefill_gemm3_wide(int T, int d_model, int num_sms) {
  return ((T + BM - 1) / BM) * ((d_model + 2 * BN - 1) / (2 * BN)) * 3 >= num_sms;
}

int prefill_splitk(int T, int d_model, int d_ff, int num_sms) {
  const int wn = prefill_gemm3_wide(T, d_model, num_sms) ? 2 * BN : BN;
  const int tiles = ((T + BM - 1) / BM) * ((d_model + wn - 1) / wn);
  const int nkb = (d_ff + BK - 1) / BK;
  int s = 1;
  while (tiles * s * 2 <= num_sms && s * 2 <= nkb / 4) s *= 2;
  return s;
}

cudaError_t launch_prefill(const PrefillArgs& a, int num_sms, cudaStream_t stream) {
  const int T = a.T, d_model = a.d_model, r = a.r, d2 = a.d_model - a.r, d_ff = a.d_ff;
  const int tiles_n = (d_ff + BN - 1) / BN;
  unsigned char* ws = static_cast<unsigned char*>(a.workspace);
  size_t off = align256(sizeof(DeviceControl));
  float2* moments = reinterpret_cast<float2*>(ws + off);
  off += align256(static_cast<size_t>(T) * ((d_ff + 63) / 64) * sizeof(float2));
  float* theta = reinterpret_cast<float*>(ws + off);
  off += align256(static_cast<size_t>(T) * 4);
  const int h_kb = (d_ff + BK - 1) / BK;
  const size_t h_bytes = static_cast<size_t>((T + BM - 1) / BM) * h_kb * BM * BK * 2;
  uint16_t* h_hi = reinterpret_cast<uint16_t*>(ws + off);
  off += h_bytes;
  uint16_t* h_lo = reinterpret_cast<uint16_t*>(ws + off);
  off += h_bytes;
  float4* Xt = reinterpret_cast<float4*>(ws + off);
  off += static_cast<size_t>((T + BM - 1) / BM) * tiles_n * BM * BN * 4;
  const int splits = prefill_splitk(T, d_model, d_ff, num_sms);
  float* part = splits > 1 ? reinterpret_cast<float*>(ws + off) : nullptr;

  const uint16_t* q = static_cast<const uint16_t*>(a.q);
  CUtensorMap tq1, tq2, tk1, tk2, tv;
  const uint64_t qrow = static_cast<uint64_t>(d_model) * 2;
  // up to 64 tokens the token operand is fetched as 64-row boxes (A64 above)
  const bool a64 = T <= 64;
  const uint32_t qbox = a64 ? 64 : BM;
  if (!make_tmap(&tq1, q, r, T, qrow, BK, qbox) || !make_tmap(&tq2, q + r, d2, T, qrow, BK, qbox) ||
      !make_tmap(&tk1, a.K1, r, d_ff, static_cast<uint64_t>(r) * 2, BK, BN) ||
      !make_tmap(&tk2, a.K2, d2, d_ff, static_cast<uint64_t>(d2) * 2, BK, BN) ||
      !make_tmap(&tv, a.V, d_model, d_ff, static_cast<uint64_t>(d_model) * 2, 64, BK))
    return cudaErrorInvalidValue;
  // 65 to 128 tokens (one band): GEMMs 1 and 2 run 128 x 64 units (64-row weight
  // boxes), so that 144 CTAs rather than 72 stream the weights (T = 100 47.6 ->
  // 45.2 us, T = 128 49.2 -> 46.8).  Up to 64 tokens they measured no faster
  // (T = 64 43.8 -> 45.3 us: GEMM 2's epilogue warps then merge the moments of
  // twice as many tiles per CTA, in twice as many CTAs, while a shorter main loop
  // hides less of it).
  const bool nw = T > 64 && T <= BM;
  const int nw_tiles = (d_ff + 63) / 64;
  CUtensorMap tk1n, tk2n;
  if (nw && (!make_tmap(&tk1n, a.K1, r, d_ff, static_cast<uint64_t>(r) * 2, BK, 64) ||
             !make_tmap(&tk2n, a.K2, d2, d_ff, static_cast<uint64_t>(d2) * 2, BK, 64)))
    return cudaErrorInvalidValue;

  GemmParams g{};
  g.ctl = reinterpret_cast<DeviceControl*>(ws);
  g.wait_limit_ns = a.wait_limit_ns;
  g.X = a.x_out;  // row-major copy for the debug entry point
  g.Xt = Xt;      // GEMM 1 stores the scores once, tiled; GEMM 2's gate reads them back
  g.xt_tiles_n = tiles_n;
  g.moments = moments;
  g.mom_stride = nw ? nw_tiles : tiles_n;
  g.mom_w = nw ? 64 : BN;
  g.theta = nullptr;
  g.Q = a.Q;
  g.theta_out = a.theta_out;
  g.h_hi = h_hi;
  g.h_lo = h_lo;
  g.h_kb = h_kb;
  g.active = a.active_out;
  g.part = part;
  g.out = static_cast<uint16_t*>(a.out);

  // GEMM 1: X = Q1 K1^T
  g.M = T;
  g.N = d_ff;
  g.K = r;
  g.tiles_m = (T + BM - 1) / BM;
  g.tiles_n = tiles_n;
  g.nkb = (r + BK - 1) / BK;
  g.split_k = 1;
  g.kb_per_split = g.nkb;
  g.units = g.tiles_m * g.tiles_n;
  // Wide units (128 tokens x 256 neurons, 4 stages of 48 KB) carry twice the MMA
  // work per token tile loaded; they pay off once they still fill every SM.
  const int wide_units = g.tiles_m * ((d_ff + 2 * BN - 1) / (2 * BN));
  cudaError_t e;
  if (wide_units >= num_sms) {
    g.tiles_n = (d_ff + 2 * BN - 1) / (2 * BN);
    g.units = wide_units;
    e = launch_gemm<kEpiPredictor, false, false, 4, true>(tq1, tq1, tk1, tk1, g, num_sms, stream);
  } else if (nw) {
    g.tiles_n = nw_tiles;
    g.units = g.tiles_m * g.tiles_n;
    e = launch_gemm<kEpiPredictor, false, false, 8, false, false, true>(tq1, tq1, tk1n, tk1n, g, num_sms, stream);
  } else if (a64) {
    e = launch_gemm<kEpiPredictor, false, false, 8, false, true>(tq1, tq1, tk1, tk1, g, num_sms, stream);
  } else {
    e = launch_gemm<kEpiPredictor, false, false, 6>(tq1, tq1, tk1, tk1, g, num_sms, stream);
  }
  if (e != cudaSuccess) return e;
  // GEMM 2: A = Q2 K2^T; the gate h = GELU(max(x - theta, 0)) a with x as GEMM 1
  // stored it, split into h_hi + h_lo.  Wide units under the same rule as GEMM 1.
  // Up to 64 tokens the epilogue warps derive theta from the tile moments while
  // the main loop runs, which saves theta_kernel and one kernel boundary
  // (measured 47.4 -> 45.0 us per call at T = 16, 45.4 -> 44.6 at T = 64).  Every
  // CTA of a token band repeats that merge for the same rows, which at T = 256
  // (72 CTAs per band, 256 rows) cost more than it saved (+6 us), and with several
  // units per CTA it would sit between units: there theta_kernel runs first.
  const int gate_units = wide_units >= num_sms ? wide_units : g.tiles_m * (nw ? nw_tiles : tiles_n);
  if (T > 64 || wide_units >= num_sms || gate_units > num_sms) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((T + 3) / 4);
    cfg.blockDim = dim3(128);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, theta_kernel, static_cast<const float2*>(moments), T, d_ff, g.mom_stride,
                                g.mom_w, a.Q, theta, a.theta_out)) != cudaSuccess)
      return e;
    g.theta = theta;
  }
  g.early_main = 1;
  g.K = d2;
  g.nkb = (d2 + BK - 1) / BK;
  g.kb_per_split = g.nkb;
  if (wide_units >= num_sms) {
    g.tiles_n = (d_ff + 2 * BN - 1) / (2 * BN);
    g.units = wide_units;
    e = launch_gemm<kEpiGate, false, false, 4, true>(tq2, tq2, tk2, tk2, g, num_sms, stream);
  } else if (nw) {
    g.tiles_n = nw_tiles;
    g.units = g.tiles_m * g.tiles_n;
    e = launch_gemm<kEpiGate, false, false, 8, false, false, true>(tq2, tq2, tk2n, tk2n, g, num_sms, stream);
  } else {
    g.tiles_n = tiles_n;
    g.units = g.tiles_m * g.tiles_n;
    e = a64 ? launch_gemm<kEpiGate, false, false, 8, false, true>(tq2, tq2, tk2, tk2, g, num_sms, stream)
            : launch_gemm<kEpiGate, false, false, 6>(tq2, tq2, tk2, tk2, g, num_sms, stream);
  }
  if (e != cudaSuccess) return e;
  // GEMM 3: out = H_hi V + H_lo V
  g.early_main = 0;
  g.N = d_model;
  g.K = d_ff;
  const bool wide3 = prefill_gemm3_wide(T, d_model, num_sms);
  g.tiles_n = wide3 ? (d_model + 2 * BN - 1) / (2 * BN) : (d_model + BN - 1) / BN;
  g.nkb = (d_ff + BK - 1) / BK;
  g.split_k = splits;
  g.kb_per_split = (g.nkb + splits - 1) / splits;
  g.units = g.tiles_m * g.tiles_n * splits;
  // GEMM 3 takes h_hi / h_lo by bulk copies of whole blocks: no tensor maps for A
  e = wide3 ? launch_gemm<kEpiOut, true, true, 3, true>(tv, tv, tv, tv, g, num_sms, stream)
            : launch_gemm<kEpiOut, true, true, 4>(tv, tv, tv, tv, g, num_sms, stream);
  if (e != cudaSuccess) return e;
  if (splits > 1) {
    const size_t n4 = static_cast<size_t>(T) * d_model / 4;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms * 4);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, static_cast<const float*>(part), splits, n4,
                                static_cast<uint16_t*>(a.out))) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

// GEMM 1 alone (the low-rank predictor x = K1^T q[:r] for T tokens), the same
// kernel and unit choice as in launch_prefill, writing x row-major to x_out
// instead of the tiled copy GEMM 2 reads, and no tile moments (measured
// 12.8 -> 11.9 us at T = 256 together with 32-column TMEM loads).  The
// workspace holds only the control block.
cudaError_t launch_predictor(const void* q, const void* K1, int T, int d_model, int r, int d_ff, float* x_out,
                             void* workspace, unsigned long long wait_limit_ns, int num_sms, cudaStream_t stream) {
  const int tiles_n = (d_ff + BN - 1) / BN;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const bool a64 = T <= 64;
  CUtensorMap tq1, tk1;
  CUtensorMap tx;
  if (!make_tmap(&tq1, q, r, T, static_cast<uint64_t>(d_model) * 2, BK, a64 ? 64 : BM) ||
      !make_tmap(&tk1, K1, r, d_ff, static_cast<uint64_t>(r) * 2, BK, BN) || !make_tmap_x(&tx, x_out, d_ff, T))
    return cudaErrorInvalidValue;
  GemmParams g{};
  g.ctl = reinterpret_cast<DeviceControl*>(ws);
  g.wait_limit_ns = wait_limit_ns;
  g.X = x_out;
  g.x_tma = 1;
  g.Xt = nullptr;
  g.xt_tiles_n = tiles_n;
  g.moments = nullptr;  // x only
  g.mom_stride = tiles_n;
  g.mom_w = BN;
  g.M = T;
  g.N = d_ff;
  g.K = r;
  g.tiles_m = (T + BM - 1) / BM;
  g.tiles_n = tiles_n;
  g.nkb = (r + BK - 1) / BK;
  g.split_k = 1;
  g.kb_per_split = g.nkb;
  g.units = g.tiles_m * g.tiles_n;
  const int wide_units = g.tiles_m * ((d_ff + 2 * BN - 1) / (2 * BN));
  if (wide_units >= num_sms) {
    g.tiles_n = (d_ff + 2 * BN - 1) / (2 * BN);
    g.units = wide_units;
    return launch_gemm<kEpiPredictor, false, false, 4, true>(tq1, tq1, tk1, tx, g, num_sms, stream);
  }
  if (T <= BM) {
    // one token band: 128 x 64 units, 144 CTAs streaming K1 (T = 16 10.8 -> 9.9 us,
    // T = 128 11.7 -> 10.4)
    CUtensorMap tk1n;
    if (!make_tmap(&tk1n, K1, r, d_ff, static_cast<uint64_t>(r) * 2, BK, 64)) return cudaErrorInvalidValue;
    g.tiles_n = (d_ff + 63) / 64;
    g.units = g.tiles_m * g.tiles_n;
    return a64 ? launch_gemm<kEpiPredictor, false, false, 12, false, true, true>(tq1, tq1, tk1n, tx, g, num_sms, stream)
               : launch_gemm<kEpiPredictor, false, false, 8, false, false, true>(tq1, tq1, tk1n, tx, g, num_sms, stream);
  }
  if (a64) return launch_gemm<kEpiPredictor, false, false, 8, false, true>(tq1, tq1, tk1, tx, g, num_sms, stream);
  return launch_gemm<kEpiPredictor, false, false, 6>(tq1, tq1, tk1, tx, g, num_sms, stream);
}


// ---------------------------------------------------------------- debug builds
unsigned take_bounds_violations_prefill(bool clear) {
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
