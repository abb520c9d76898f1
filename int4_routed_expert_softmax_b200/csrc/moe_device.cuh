// moe_device.cuh -- device helpers shared by the libmoe kernels (sm_100a).
//
// * Fixed-order fp32 arithmetic: every step whose result feeds an integer
//   decision (router top-k, Q8_0 codes of x and of SiLU(g)*u) is written with
//   explicit round-to-nearest intrinsics (__fmul_rn, __fadd_rn, __fmaf_rn,
//   __fdiv_rn) so the compiler cannot contract or reorder it.  The router's
//   logits and the Q8_0 codes of x follow the layer's canonical order and are
//   reproducible bit for bit by a CPU restatement; the expert sums follow the
//   kernels' own fixed order (deterministic run to run) and agree with the
//   plain definition within the layer's float tolerance.  e^x is CUDA's expf.
// * TMA bulk copies (cp.async.bulk, global -> shared, completion counted on
//   an mbarrier) and bounded mbarrier waits: a wait that runs out records an
//   error code in the workspace status word and returns false; no kernel
//   traps or spins forever.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "moe_internal.h"

namespace moe {

// ------------------------------------------------------------------ status
__device__ __forceinline__ void set_status(int32_t *status, int32_t code, int32_t detail) {
  if (status != nullptr && atomicCAS(status, 0, code) == 0) status[1] = detail;
}

// ------------------------------------------------------------------ fp32
__device__ __forceinline__ float fmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float fadd(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float ffma(float a, float b, float c) { return __fmaf_rn(a, b, c); }
__device__ __forceinline__ float fdiv(float a, float b) { return __fdiv_rn(a, b); }

// SwiGLU activation: SiLU(g) * u with SiLU(g) = g / (1 + exp(-g)).
__device__ __forceinline__ float swiglu(float g, float u) {
  const float e = expf(-g);
  const float den = fadd(1.0f, e);
  return fmul(fdiv(g, den), u);
}

// Q8_0 code of v for block scale d (d == 0 -> 0): round half to even.
__device__ __forceinline__ int q8_code(float v, float d) {
  if (d == 0.0f) return 0;
  float r = rintf(fdiv(v, d));
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return (int)r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// ------------------------------------------------------------------ int dot
// dp4a with unsigned bytes in a (offset-binary nibbles 0..15) and signed
// bytes in b (int8 activations): c + sum_i a_i * b_i.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ------------------------------------------------------------------ smem / mbarrier / TMA bulk
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the same phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `parity` to complete.  Gives up after `limit`
// SM clocks (the launch's wait limit: about a second by default, shorter when
// a caller sets one with moe_set_wait_limit), records `detail` with
// MOE_ERR_TIMEOUT in the status word and returns false.  With the default
// limit the wait uses try_wait, which may suspend the thread until the phase
// completes; with a shorter one it polls with test_wait, so that the limit,
// not the hardware's suspend time, bounds the wait.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status,
                                          int32_t detail, long long limit) {
  if (limit >= kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
      if (clock64() - t0 > limit) {
        set_status(status, MOE_ERR_TIMEOUT, detail);
        return false;
      }
    }
    return true;
  }
  const long long t0 = clock64();
  while (!mbar_test_wait(bar, parity)) {
    if (clock64() - t0 > limit) {
      set_status(status, MOE_ERR_TIMEOUT, detail);
      return false;
    }
  }
  return true;
}

// The same wait for the teardown of a role: the completion of copies or MMAs
// this CTA issued itself, which must land before the CTA exits.  Always the
// full limit (kWaitLimitCycles), whatever the launch's wait limit.
__device__ __forceinline__ bool mbar_drain(uint64_t *bar, uint32_t parity, int32_t *status,
                                           int32_t detail) {
  return mbar_wait(bar, parity, status, detail, kWaitLimitCycles);
}

// 1-D bulk copy global -> shared (this CTA), completion on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same with an L2 eviction-priority hint (streamed expert weights are read
// once per call: evict first so they do not push out the activations).
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes,
                                              uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------------ profiling
// Per-call profiling record (moe_profile_enable): for phase k, word 2k holds
// ~(earliest start) and word 2k+1 the latest end in ns of %globaltimer, both
// kept with atomicMax from a zeroed record, stamped by thread 0 of every CTA.
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void prof_start(unsigned long long *p, int k) {
  if (p != nullptr && threadIdx.x == 0) atomicMax(p + 2 * k, ~global_ns());
}
__device__ __forceinline__ void prof_end(unsigned long long *p, int k) {
  if (p != nullptr && threadIdx.x == 0) atomicMax(p + 2 * k + 1, global_ns());
}

// Named barrier among `nthreads` threads (warp multiples) with id `id` (1..15).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Arrival at named barrier `id` without waiting (the waiting side uses
// named_sync with the same thread count); prior shared-memory writes of the
// arriving threads are visible to the waiting threads once it completes.
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Programmatic dependent launch: wait for the preceding kernel's results /
// let the following kernel start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace moe
