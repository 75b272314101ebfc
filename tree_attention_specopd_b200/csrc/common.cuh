// Shared device helpers of the SpecOPD B200 library (sm_100a only).
//
// Status word: kernels never trap.  A device-detected error sets a bit in
// g_status (per device, one word) and the kernel writes NaN to the affected
// outputs; specopd_get_device_status() reads and clears it.  Every spin-wait
// in this library is bounded by wall time (%globaltimer) and sets
// SPECOPD_DEV_TIMEOUT when it gives up.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/specopd.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a only"
#endif

namespace specopd {

// Per-device status word (one definition: the library is a single
// translation unit, see api.cu).
__device__ unsigned int g_status = 0u;

// Upper bound of every bounded wait (ns).  Normal waits last microseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Host-driven fault injection for tests (specopd_debug_fault_injection):
// off unless a test sets it.  withhold_position >= 0 makes the E2E-TV
// scorer of that supervised position skip publishing its overlap, so the
// other positions of its branch wait for it in vain; branch_wait_ns, when
// nonzero, replaces kWaitLimitNs for those branch waits only.
struct FaultInject {
  long long withhold_position;
  unsigned long long branch_wait_ns;
};
__device__ FaultInject g_inject = {-1ll, 0ull};

__device__ __forceinline__ void set_status(unsigned bits) { atomicOr(&g_status, bits); }

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- bf16 / f32
template <typename T> struct Elt;
template <> struct Elt<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elt<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Pack two floats as bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- memory order
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acqrel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Spin (one thread) until *flag >= want or the time limit passes.
// Returns true on success; on expiry sets SPECOPD_DEV_TIMEOUT.
__device__ __forceinline__ bool wait_flag_geq(const unsigned* flag, unsigned want) {
  if (ld_acquire_gpu(flag) >= want) return true;
  const unsigned long long t0 = globaltimer_ns();
  // Short, fixed pause: the waits here last microseconds, and a growing
  // back-off would overshoot the moment the flag flips.
  while (true) {
    __nanosleep(64);
    if (ld_acquire_gpu(flag) >= want) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_status(SPECOPD_DEV_TIMEOUT);
      return false;
    }
  }
}

// Same, with an explicit limit (ns).
__device__ __forceinline__ bool wait_flag_geq_limit(const unsigned* flag, unsigned want,
                                                    unsigned long long limit_ns) {
  if (ld_acquire_gpu(flag) >= want) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire_gpu(flag) >= want) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      set_status(SPECOPD_DEV_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Same, with a suspend-time hint: the thread may sleep in the instruction
// until the phase completes or about kSuspendNs have passed, so a waiting
// warp takes no issue slots from the others.
constexpr unsigned kSuspendNs = 1000000u;
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_status(SPECOPD_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared (this CTA), completion on an mbarrier.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 eviction-priority policy (from createpolicy).
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, unsigned bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2^x with the hardware approximation (ex2.approx.ftz.f32: one MUFU op,
// relative error about 2^-22; results below 2^-126 flush to zero, which a
// softmax term that small never affects at fp32 precision).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- warp utils
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Combine two (max, sum of 2^(x - max)) pairs, -inf safe.
__device__ __forceinline__ void lse2_combine(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;  // both empty
  const float a = (m == -INFINITY) ? 0.f : s * exp2f(m - mn);
  const float b = (m2 == -INFINITY) ? 0.f : s2 * exp2f(m2 - mn);
  m = mn;
  s = a + b;
}

}  // namespace specopd
