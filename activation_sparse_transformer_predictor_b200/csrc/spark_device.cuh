// spark_device.cuh -- device-side building blocks shared by the Spark kernels:
// bounded waits, the grid barrier, mbarrier / bulk-copy wrappers, row-statistics
// merging and GELU.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spark {

// ----------------------------------------------------------------------------
// Device control block.  It sits at the start of every workspace, is zeroed
// when the workspace is allocated, and is read (and cleared) by
// spark_query_status.  The arrival counters are reset by the last CTA to leave
// each launch, so every launch starts from zeros.
// ----------------------------------------------------------------------------
enum DeviceError : unsigned { kDevOk = 0, kDevTimeout = 1 };

struct DeviceControl {
  unsigned int status;      // first device error recorded (0 = none)
  unsigned int abort;       // set once any CTA gave up waiting; later launches return at once
  unsigned int where;       // which wait gave up (diagnostic)
  unsigned int exit_count;  // CTAs that finished the current launch
  unsigned int arrive1;     // arrivals at the statistics exchange
  unsigned int arrive2;     // arrivals at the partial-output exchange
  unsigned int pad0[2];
  unsigned long long theta_word;  // published threshold of token 0 (high word) | flag (low word)
  float theta[8];                 // published thresholds of tokens 1..7
  unsigned int pad1[14];
};
static_assert(sizeof(DeviceControl) == 128, "DeviceControl layout");

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ float ld_relaxed_gpu_f32(const float* p) {
  float v;
  asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}

// Release-add: this CTA's earlier writes (ordered before by __syncthreads)
// become visible to whoever acquires the counter value it produced.
__device__ __forceinline__ unsigned atom_add_release_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void record_error(DeviceControl* ctl, unsigned code, unsigned where) {
  if (atomicCAS(&ctl->status, 0u, code) == 0u) ctl->where = where;
  atomicExch(&ctl->abort, 1u);
}

// Release-add without a return value: the arriving thread does not wait for
// the round trip.
__device__ __forceinline__ void red_add_release_gpu(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Thread 0: spin until *cnt >= target (acquire), with a time limit.  Returns
// false after recording kDevTimeout, or once another CTA gave up.  The abort
// flag and the clock are checked every 16 polls so that each poll is one load.
__device__ __forceinline__ bool wait_count_geq(DeviceControl* ctl, const unsigned* cnt, unsigned target,
                                               uint64_t limit_ns, unsigned where) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (unsigned it = 1;; ++it) {
    if (ld_acquire_gpu(cnt) >= target) return true;
    if ((it & 15u) == 0u) {
      if (ld_relaxed_gpu(&ctl->abort)) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        record_error(ctl, kDevTimeout, where);
        return false;
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Debug builds (compiled with SPARK_DEBUG: libspark_debug.so) check indices the
// kernels compute -- gathered neuron and key rows, active counts, partial-output
// slots, operand block numbers -- before using them.  A failed check counts into
// the word g_bounds_violations that every .cu file using SPARK_CHECK defines
// (static __device__), and the guarded access is skipped; nothing traps.
// spark_debug_violations() reads and clears the words.  Release builds compile
// SPARK_CHECK(c) to `true` without evaluating c.
// ----------------------------------------------------------------------------
__device__ __forceinline__ bool bounds_check(bool ok, unsigned* counter) {
  if (!ok) atomicAdd(counter, 1u);
  return ok;
}
#ifdef SPARK_DEBUG
#define SPARK_CHECK(cond) ::spark::bounds_check(static_cast<bool>(cond), &g_bounds_violations)
#else
#define SPARK_CHECK(cond) true
#endif

// ----------------------------------------------------------------------------
// mbarrier + bulk copy (TMA engine, 1-D form) wrappers.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait on an mbarrier phase.  Returns false (and records kDevTimeout)
// if the phase did not complete within limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, uint64_t limit_ns,
                                                  DeviceControl* ctl, unsigned where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) {
      record_error(ctl, kDevTimeout, where);
      return false;
    }
  }
  return true;
}

// Global -> shared bulk copy completing on an mbarrier.  dst, src 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Hint: pull [src, src+bytes) into L2.  src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ----------------------------------------------------------------------------
// Row statistics: (count, mean, M2) partials merged with Chan et al.'s
// pairwise update, which is exact in exact arithmetic and stable in fp32.
// ----------------------------------------------------------------------------
struct Moments {
  float n, mean, m2;
};

__device__ __forceinline__ Moments merge_moments(Moments a, Moments b) {
  const float n = a.n + b.n;
  if (n == 0.f) return a;
  const float delta = b.mean - a.mean;
  const float wb = b.n / n;
  Moments r;
  r.n = n;
  r.mean = a.mean + delta * wb;
  r.m2 = a.m2 + b.m2 + delta * delta * a.n * wb;
  return r;
}

// Fixed-shape tree over the 32 lanes (shfl_down); lane 0 holds the result.
// Deterministic: the same inputs give the same bits on every CTA.
__device__ __forceinline__ Moments warp_merge_moments(Moments m) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    Moments o;
    o.n = __shfl_down_sync(0xffffffffu, m.n, off);
    o.mean = __shfl_down_sync(0xffffffffu, m.mean, off);
    o.m2 = __shfl_down_sync(0xffffffffu, m.m2, off);
    m = merge_moments(m, o);
  }
  return m;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
  return v;
}

// GELU, tanh form, for s >= 0 (the kernels only evaluate it on s = x - theta > 0):
// 0.5 s (1 + tanh(u)) with u = sqrt(2/pi) (s + 0.044715 s^3).  Uses the identity
// 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)); for u >= 0, exp(-2u) lies in (0, 1], so
// the quotient is well conditioned.  The fast divide (<= 2 ulp for a divisor in
// [1, 2]) has no slow path; relative error of the result ~1e-6.
__device__ __forceinline__ float gelu_tanh(float s) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  const float u = k0 * fmaf(0.044715f * s, s * s, s);
  return __fdividef(s, 1.f + __expf(-2.f * u));
}

// bf16x2 packed in a 32-bit word -> two floats (exact widening).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  float2 r;
  r.x = __uint_as_float(w << 16);
  r.y = __uint_as_float(w & 0xffff0000u);
  return r;
}

// c + a.lo * b.lo + a.hi * b.hi for two bf16 pairs, with the mixed-precision
// FMA of sm_100 (bf16 operands widened exactly, one fp32 rounding per step):
// the same bits as two fmaf calls on the widened values, without the widening
// instructions.
__device__ __forceinline__ float fma_bf16x2_f32(uint32_t a, uint32_t b, float c) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(c)
      : "r"(a), "r"(b));
  return c;
}

// acc + <a, b> over 8 bf16 pairs, in a fixed order (fp32 FMA, element 0 first).
__device__ __forceinline__ float dot8_bf16(uint4 a, uint4 b, float acc) {
  acc = fma_bf16x2_f32(a.x, b.x, acc);
  acc = fma_bf16x2_f32(a.y, b.y, acc);
  acc = fma_bf16x2_f32(a.z, b.z, acc);
  acc = fma_bf16x2_f32(a.w, b.w, acc);
  return acc;
}

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

__device__ __forceinline__ uint4 ldg_nc128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// mbarrier: add expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

}  // namespace spark
