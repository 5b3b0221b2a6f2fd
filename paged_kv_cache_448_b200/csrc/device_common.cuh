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

// Default wall-clock bound of every pipeline wait (the launch passes it in
// the kernel arguments): far above any real TMA or hand-over latency, yet a
// wait that can never complete ends in about a second (the kernel then
// reports kErrWaitTimeout instead of hanging).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Plain bulk copy global -> shared (16-byte aligned addresses, size a multiple
// of 16), completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
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

// Non-blocking test of phase `parity` of `bar` (a thread polling several
// barriers uses it instead of try_wait, which may suspend the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete. Gives up (returns false) after
// limit_ns of wall time, or at once when *abort is set (another warp of the
// CTA has given up already).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          const volatile int* abort = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// True for the one load a failure-detection test asked to leave out: tile
// `tile` of the launch's first CTA (skip_tile < 0: none). The wait for that
// tile then runs out, which exercises the abort and drain path.
__device__ __forceinline__ bool skip_for_test(int32_t skip_tile, int tile) {
  return skip_tile >= 0 && tile == skip_tile && blockIdx.x == 0 && blockIdx.y == 0 &&
         blockIdx.z == 0;
}

// The same for a kernel whose CTAs take their work units in another order
// than their index: `first_unit` says whether this CTA runs the unit whose
// coordinates are all 0.
__device__ __forceinline__ bool skip_unit_for_test(int32_t skip_tile, int tile, bool first_unit) {
  return skip_tile >= 0 && tile == skip_tile && first_unit;
}

// First failure of a launch: where it happened and the state there, written
// once (words: site, then up to 7 values) to the diagnostic words.
__device__ __forceinline__ void record_failure(int32_t* diag, int32_t site, int32_t v0,
                                               int32_t v1, int32_t v2, int32_t v3, int32_t v4,
                                               int32_t v5, int32_t v6) {
  if (!diag || atomicCAS(diag, 0, site) != 0) return;
  diag[1] = v0; diag[2] = v1; diag[3] = v2; diag[4] = v3;
  diag[5] = v4; diag[6] = v5; diag[7] = v6;
}

// 4-D tiled TMA load global -> shared with an L2 cache-eviction policy,
// completion counted on `bar` in bytes. Coordinates are innermost first;
// boxes reaching outside the tensor are zero-filled there.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2, int32_t c3,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
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
