// pa_device.cuh -- device helpers shared by the libpa kernels (sm_100a).
//
// mbarrier + bulk-async-copy (TMA, non-tensor form) wrappers, bounded waits,
// element conversion to fp32 and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

// Longest time any wait inside a kernel may spin before it gives up, sets
// PA_DEVERR_TIMEOUT and unwinds (nanoseconds of %globaltimer).  The test
// build of the decode kernel (libpa_waittest.so) sets a short one.
#ifndef PA_WAIT_LIMIT_NS
#define PA_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kWaitLimitNs = PA_WAIT_LIMIT_NS;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void raise_error(unsigned int *err, unsigned int bits) {
  if (err) atomicOr(err, bits);
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
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
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false if
// kWaitLimitNs passed first (the caller then records PA_DEVERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// Wait (each wait bounded) until the copies into the last `issued` uses of a
// ring of `stages` full barriers have landed: use i of the ring is stage
// i % stages in phase (i / stages) & 1.  A use that was only arrived on
// (aborted or skipped) completes at once.  The issuing thread calls this
// before its CTA may exit, so that a CTA unwinding early never leaves a bulk
// copy in flight into shared memory that the SM may hand to the next CTA.
// Returns false if a wait expired.
__device__ __forceinline__ bool drain_ring(uint64_t *full, uint32_t stages, uint32_t issued) {
  bool ok = true;
  const uint32_t first = issued > stages ? issued - stages : 0u;
  for (uint32_t i = first; i < issued; ++i) ok = mbar_wait(&full[i % stages], (i / stages) & 1u) && ok;
  return ok;
}

// ---- bulk async copy global -> shared (completes on an mbarrier) ------------
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gmem_src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- named barrier for a subset of warps ------------------------------------
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---- element types ----------------------------------------------------------
template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPerVec = 4;  // elements per 16-byte vector
  // 16 bytes -> kPerVec/2 float2 pairs (elements 2i, 2i+1)
  __device__ __forceinline__ static void to_f2(const uint4 &v, float2 *o) {
    o[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    o[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ __forceinline__ static float to_f(float x) { return x; }
  __device__ __forceinline__ static float from_f(float x) { return x; }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static float2 pair(uint32_t u) {
    // bfloat16 is the high half of a binary32: widening is a shift / mask.
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  __device__ __forceinline__ static void to_f2(const uint4 &v, float2 *o) {
    o[0] = pair(v.x);
    o[1] = pair(v.y);
    o[2] = pair(v.z);
    o[3] = pair(v.w);
  }
  __device__ __forceinline__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

template <>
struct Elem<__half> {
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static float2 pair(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(h);
  }
  __device__ __forceinline__ static void to_f2(const uint4 &v, float2 *o) {
    o[0] = pair(v.x);
    o[1] = pair(v.y);
    o[2] = pair(v.z);
    o[3] = pair(v.w);
  }
  __device__ __forceinline__ static float to_f(__half x) { return __half2float(x); }
  __device__ __forceinline__ static __half from_f(float x) { return __float2half_rn(x); }
};

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace pa
