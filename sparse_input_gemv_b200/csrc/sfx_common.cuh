// Device helpers shared by the sm_100a kernels of the activation-sparse library:
// dtype loads/conversions, inline-PTX wrappers for mbarriers and 1-D bulk
// (TMA) copies with an L2 evict-first policy, bounded waits and warp scans.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sfx.h"

namespace sfx {

// Kernel-side limit on any spin: a wait that sees no progress for this long
// gives up, raises SFX_DEV_TIMEOUT in the workspace status word and the kernel
// returns. Normal waits last microseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr unsigned long long kDrainLimitNs = 20000000ull;   // 20 ms

// ---------------------------------------------------------------- dtypes

template <typename T> struct DT;
template <> struct DT<__half> { static constexpr int id = SFX_F16; };
template <> struct DT<__nv_bfloat16> { static constexpr int id = SFX_BF16; };
template <> struct DT<float> { static constexpr int id = SFX_F32; };

__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }

// Eight 16-bit weights packed in a uint4 -> eight floats (exact conversions).
__device__ __forceinline__ void unpack8(const uint4& q, float (&w)[8], __nv_bfloat16) {
  const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w[2 * j] = __uint_as_float(u[j] << 16);
    w[2 * j + 1] = __uint_as_float(u[j] & 0xffff0000u);
  }
}
__device__ __forceinline__ void unpack8(const uint4& q, float (&w)[8], __half) {
  const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __half2 h2 = *reinterpret_cast<const __half2*>(&u[j]);
    float2 f = __half22float2(h2);
    w[2 * j] = f.x;
    w[2 * j + 1] = f.y;
  }
}

// Store one float as dtype `dt` (round to nearest even).
__device__ __forceinline__ void store_as(void* base, long long i, int dt, float v) {
  if (dt == SFX_F32) {
    reinterpret_cast<float*>(base)[i] = v;
  } else if (dt == SFX_BF16) {
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<__half*>(base)[i] = __float2half_rn(v);
  }
}

__device__ __forceinline__ float load_as_f32(const void* base, long long i, int dt) {
  if (dt == SFX_F32) return reinterpret_cast<const float*>(base)[i];
  if (dt == SFX_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

// ---------------------------------------------------------------- activations

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }
__device__ __forceinline__ float gelu_erf_f(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}
__device__ __forceinline__ float gelu_tanh_f(float v) {
  return 0.5f * v * (1.0f + tanhf(0.79788456080286536f * (v + 0.044715f * v * v * v)));
}

// ---------------------------------------------------------------- status

__device__ __forceinline__ void raise_status(unsigned* status, unsigned bits) {
  if (status) atomicOr(status, bits);
}

// Split-K arrival on a tile counter, after a CTA barrier: the release half
// publishes the CTA's partial sums (ordered before it by the barrier), the
// acquire half lets the last arriver read everyone else's. Returns the count
// before this arrival.
__device__ __forceinline__ int arrive_acq_rel(int32_t* counter) {
  int prev;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(prev) : "l"(counter) : "memory");
  return prev;
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier / bulk copy

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

// Wait for phase `parity` of `bar` to complete. Gives up after `limit_ns`
// (or at once if *abort is set by another thread) and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// L2 cache policy: weights are streamed once per call, so they are marked
// evict-first and do not push reusable data (activations, partials) out of L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> shared (async proxy), completing `bytes` of
// transaction count on `bar`. dst/src 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Asks L2 to fetch [p, p + bytes) (p 16-byte aligned, bytes a multiple of 16); a
// hint with no completion to wait for.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Programmatic dependent launch controls (no-ops without the launch attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- warp helpers

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace sfx
