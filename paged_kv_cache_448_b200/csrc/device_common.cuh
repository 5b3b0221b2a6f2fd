// device_common.cuh — small sm_100a building blocks shared by the kernels:
// shared-memory mbarriers, TMA tensor loads, number-format conversions and
// the error word the kernels report table problems through.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "decode_args.h"

namespace paged {

// Upper bound on mbarrier polls before a wait gives up and reports
// kErrWaitTimeout (each try_wait blocks for a hardware-defined slice; this
// bound is many seconds, far above any real TMA latency).
constexpr uint32_t kMaxWaitPolls = 1u << 26;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar`; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kMaxWaitPolls; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 3-D tiled TMA load global -> shared, completion counted on `bar` (bytes).
// Coordinates are innermost first. Out-of-range boxes are zero-filled.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// Same, with an L2 cache-eviction policy (e.g. evict-first for streamed data).
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t x, int32_t y, int32_t z,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar)),
      "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- formats

struct F16 {
  using T = __half;
  static constexpr int kBytes = 2;
};
struct BF16 {
  using T = __nv_bfloat16;
  static constexpr int kBytes = 2;
};
struct E4M3 {
  using T = uint8_t;
  static constexpr int kBytes = 1;
};

// Convert a 32-bit word holding two 16-bit values (low half first) to fp32.
__device__ __forceinline__ float2 cvt2(F16, uint32_t w) {
  __half2 h = *reinterpret_cast<__half2*>(&w);
  return __half22float2(h);
}
__device__ __forceinline__ float2 cvt2(BF16, uint32_t w) {
  // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits.
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// Two E4M3 codes (low byte first) -> fp32 via the exact E4M3 -> f16 conversion.
__device__ __forceinline__ float2 cvt2_e4m3(uint16_t w) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w), __NV_E4M3);
  return __half22float2(*reinterpret_cast<__half2*>(&h));
}

__device__ __forceinline__ void store_out(F16, void* base, int64_t idx, float v) {
  reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
}
__device__ __forceinline__ void store_out(BF16, void* base, int64_t idx, float v) {
  reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
}
__device__ __forceinline__ float load_in(F16, const void* base, int64_t idx) {
  return __half2float(reinterpret_cast<const __half*>(base)[idx]);
}
__device__ __forceinline__ float load_in(BF16, const void* base, int64_t idx) {
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
}

__device__ __forceinline__ void report(int32_t* err, int32_t bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace paged
