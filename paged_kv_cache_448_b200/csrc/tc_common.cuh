// tc_common.cuh — 5th-generation tensor core (tcgen05) building blocks:
// tensor-memory allocation, shared-memory matrix descriptors, the f16/bf16
// and 8-bit (E4M3 / E5M2) instruction descriptors, MMA issue and commit, tensor-memory loads/stores.
// Bit layouts follow the PTX ISA's tcgen05 description (the same encoding
// CUTLASS's sm100 UMMA descriptors use).
#pragma once

#include <stdint.h>

#include "device_common.cuh"

namespace paged {
namespace tc {

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   bits  0-13: start address >> 4      bits 16-29: leading byte offset >> 4
//   bits 32-45: stride byte offset >> 4 bits 46-47: version (1)
//   bits 61-63: layout (2 = 128-byte swizzle)
// K-major (rows of K elements, 128 bytes per row, 8-row groups 1024 bytes
// apart): lbo = 16 (unused), sbo = 1024. MN-major (rows of the K index, each
// 128 bytes of MN elements (64 16-bit or 128 8-bit ones), 8-row groups `sbo`
// apart, the next 128 bytes of MN elements `lbo` apart).
__device__ __forceinline__ uint64_t sw128_desc(const void* smem, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
  const uint64_t a = (smem_addr(smem) >> 4) & 0x3FFFu;
  return a | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with fp32 accumulation:
//   bits 4-5: D format (1 = f32)   bits 7-9 / 10-12: A / B format (0 f16, 1 bf16)
//   bit 15 / 16: A / B major (0 = K-major, 1 = MN-major)
//   bits 17-22: N >> 3             bits 24-28: M >> 4
template <bool BF, int M, int N, bool B_MN_MAJOR>
__device__ __forceinline__ constexpr uint32_t idesc_f16() {
  static_assert(M == 128 && N % 16 == 0 && N >= 16 && N <= 256, "UMMA shape");
  return (1u << 4) | ((BF ? 1u : 0u) << 7) | ((BF ? 1u : 0u) << 10) |
         ((B_MN_MAJOR ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// The same with the major-ness of A chosen as well (bit 15: A MN-major).
template <bool BF, int M, int N, bool A_MN_MAJOR, bool B_MN_MAJOR>
__device__ __forceinline__ constexpr uint32_t idesc_f16_ab() {
  return idesc_f16<BF, M, N, B_MN_MAJOR>() | ((A_MN_MAJOR ? 1u : 0u) << 15);
}

// Instruction descriptor of kind::f8f6f4 with fp32 accumulators; operand
// formats 0 = E4M3, 1 = E5M2 (bits 7-9 for A, 10-12 for B), the other fields
// as in idesc_f16.
template <int A_FMT, int B_FMT, int M, int N, bool B_MN_MAJOR>
__device__ __forceinline__ constexpr uint32_t idesc_f8() {
  static_assert(M == 128 && N % 16 == 0 && N >= 16 && N <= 256, "UMMA shape");
  static_assert((A_FMT == 0 || A_FMT == 1) && (B_FMT == 0 || B_FMT == 1), "E4M3 / E5M2");
  return (1u << 4) | (static_cast<uint32_t>(A_FMT) << 7) | (static_cast<uint32_t>(B_FMT) << 10) |
         ((B_MN_MAJOR ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// The same with the major-ness of A chosen as well (bit 15: A MN-major), for
// an A operand whose M index runs along the rows in shared memory.
template <int A_FMT, int B_FMT, int M, int N, bool A_MN_MAJOR, bool B_MN_MAJOR>
__device__ __forceinline__ constexpr uint32_t idesc_f8_ab() {
  return idesc_f8<A_FMT, B_FMT, M, N, B_MN_MAJOR>() | ((A_MN_MAJOR ? 1u : 0u) << 15);
}

// Shared-memory matrix descriptor of an operand without swizzle (layout 0):
// 8 x 16-byte core matrices, rows of one core matrix 16 bytes apart. With
// both offsets 128 bytes and 16 bytes of the MN index per row (an MN-major
// operand N = 16 of 8-bit values), the operand is simply [K rows][16 bytes].
__device__ __forceinline__ uint64_t plain_desc(const void* smem, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
  const uint64_t a = (smem_addr(smem) >> 4) & 0x3FFFu;
  return a | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// D (tensor memory) (+)= A . B, 8-bit operands (K = 32 per instruction), both
// from shared memory.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// The same with A in tensor memory (lane = row, four 8-bit K elements per
// 32-bit column, K order; 8 columns per instruction).
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// D[tmem] (+)= A[smem] . B[smem]; issued by one thread.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// D[tmem] (+)= A[tmem] . B[smem]: A (M x 16, 16-bit) read from tensor memory,
// row m in lane m, the 16 K elements packed in pairs into 8 consecutive
// 32-bit columns starting at a_tmem.
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Tensor-memory allocation of `cols` columns (a power of two >= 32) by one
// whole warp; the base address lands in *slot (shared memory).
__device__ __forceinline__ void alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(slot)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols)
               : "memory");
}

// 32 consecutive fp32 columns of this thread's lane (warp w reads lanes
// 32w..32w+31; `taddr` carries the warp's lane base).
__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 8 / 16 consecutive fp32 columns of this thread's lane; the caller waits
// (tcgen05.wait::ld) before using them.
__device__ __forceinline__ void ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void ld32u_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// The same wait with the destination registers of an unwaited load tied to
// it, so that no use of them can be scheduled before the wait.
__device__ __forceinline__ void wait_ld(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}
__device__ __forceinline__ void wait_ld(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st8u(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}

// Two 32-column loads in flight before one wait (columns taddr .. taddr+63).
__device__ __forceinline__ void ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
#define PAGED_LD32(OFF)                                                                      \
  asm volatile(                                                                              \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, " \
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "  \
      "%28, %29, %30, %31}, [%32];"                                                          \
      : "=r"(r[OFF + 0]), "=r"(r[OFF + 1]), "=r"(r[OFF + 2]), "=r"(r[OFF + 3]),              \
        "=r"(r[OFF + 4]), "=r"(r[OFF + 5]), "=r"(r[OFF + 6]), "=r"(r[OFF + 7]),              \
        "=r"(r[OFF + 8]), "=r"(r[OFF + 9]), "=r"(r[OFF + 10]), "=r"(r[OFF + 11]),            \
        "=r"(r[OFF + 12]), "=r"(r[OFF + 13]), "=r"(r[OFF + 14]), "=r"(r[OFF + 15]),          \
        "=r"(r[OFF + 16]), "=r"(r[OFF + 17]), "=r"(r[OFF + 18]), "=r"(r[OFF + 19]),          \
        "=r"(r[OFF + 20]), "=r"(r[OFF + 21]), "=r"(r[OFF + 22]), "=r"(r[OFF + 23]),          \
        "=r"(r[OFF + 24]), "=r"(r[OFF + 25]), "=r"(r[OFF + 26]), "=r"(r[OFF + 27]),          \
        "=r"(r[OFF + 28]), "=r"(r[OFF + 29]), "=r"(r[OFF + 30]), "=r"(r[OFF + 31])           \
      : "r"(taddr + OFF)                                                                     \
      : "memory");
  PAGED_LD32(0)
  PAGED_LD32(32)
#undef PAGED_LD32
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// Four values -> E4M3 hi parts and 8-bit residuals (E4M3 or E5M2), four bytes
// each in order. The values go through f16 (exact for the inputs here: bf16 /
// f16 queries times a power of two, probabilities of at most 2^8); the
// residual h - hi is exact in f16.
template <bool LO_E5M2>
__device__ __forceinline__ void split_fp8x4(float a, float b, float c, float d, uint32_t& hi,
                                            uint32_t& lo) {
  const __half2 h01 = __floats2half2_rn(a, b), h23 = __floats2half2_rn(c, d);
  const __nv_fp8x2_storage_t hi01 = __nv_cvt_halfraw2_to_fp8x2(
      *reinterpret_cast<const __half2_raw*>(&h01), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi23 = __nv_cvt_halfraw2_to_fp8x2(
      *reinterpret_cast<const __half2_raw*>(&h23), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw b01 = __nv_cvt_fp8x2_to_halfraw2(hi01, __NV_E4M3);
  const __half2_raw b23 = __nv_cvt_fp8x2_to_halfraw2(hi23, __NV_E4M3);
  const __half2 r01 = __hsub2(h01, *reinterpret_cast<const __half2*>(&b01));
  const __half2 r23 = __hsub2(h23, *reinterpret_cast<const __half2*>(&b23));
  constexpr __nv_fp8_interpretation_t LO = LO_E5M2 ? __NV_E5M2 : __NV_E4M3;
  const __nv_fp8x2_storage_t lo01 =
      __nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&r01), __NV_SATFINITE, LO);
  const __nv_fp8x2_storage_t lo23 =
      __nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&r23), __NV_SATFINITE, LO);
  hi = static_cast<uint32_t>(hi01) | (static_cast<uint32_t>(hi23) << 16);
  lo = static_cast<uint32_t>(lo01) | (static_cast<uint32_t>(lo23) << 16);
}

// 2^x by the MUFU instruction (flushes subnormal results to zero, which the
// softmax weights below 2^-126 can afford).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace tc
}  // namespace paged
