// decode_fp8_tc.cu — decode over an FP8 E4M3 cache on the 5th-generation
// tensor cores, with the tokens on the M dimension.
//
// Same operation as the decode kernel ("vLLM推理引擎架构：PagedAttention机制
// 与高吞吐推理" §2.3, with the 8-bit K/V storage of "大模型推理KV Cache内存管理
// 与PagedAttention分页显存实战", FP8 KV Cache量化): for each (sequence, kv-head)
// the G query heads of the group attend over the context through the block
// table. A cache row of head_dim 128 E4M3 codes is one 128-byte line, so a
// tile of 128 tokens, as TMA lands it (16-row boxes, 128-byte swizzle), is at
// once
//   * the K-major A operand of  S^T[t][n] = sum_d K[t][d] Q'[n][d]  (M = 128
//     tokens, K = 128 dims), and
//   * the MN-major A operand of O^T[d][n] += sum_t V[t][d] P'[n][t]  (M = 128
//     dims, K = 128 tokens),
// read by tcgen05.mma kind::f8f6f4 as stored: no code widens a cache byte.
// Q' holds per query head g an E4M3 hi row and an E4M3 lo row with
// q_g * 2^e_g = hi + lo (e_g a power of two that puts max |q_g| below 2^8,
// undone in the head's logit scale together with the kv-head's K scale), so
// S^T column g + column G + g is the head's logit; N = 16 covers G <= 8.
// P' holds per token an E4M3 hi and an E5M2 residual part of each head's
// probability (<= 2^8 under the lazily moved maximum), written by the token's
// softmax thread as one 16-byte row of an MN-major operand [tokens][16 B];
// the two O^T products (hi with E4M3, residual with E5M2) add into the same
// accumulator. V's scale multiplies the output.
//
// A CTA is one work unit (kv-head, sequence, context partition) with six
// warps:
//  * four softmax warps: thread i owns tensor-memory lane i, i.e. token i of
//    the tile in S^T and dimension i of O^T. Per tile it loads its S^T row,
//    forms the G logits (masking tokens past the context), and the CTA takes
//    each head's tile maximum (an ordered-integer warp reduction, then the
//    four warps through shared memory behind an mbarrier). The running
//    maximum moves only when a tile's maximum passes it by more than 8
//    (base 2), so probabilities stay below 2^8 and O is rarely rescaled (in
//    tensor memory, after the previous O += P V completed). Each thread keeps
//    its own partial sums; they are added across the CTA at the end;
//  * the MMA warp (one thread) owns the tensor memory: two 16-column S^T
//    buffers and 16 columns of O^T. It issues S^T of tile k+1 before
//    O^T += V^T P'^T of tile k, so S is computed under the softmax of tile k;
//  * the TMA warp (one thread) loads K and V tiles into 3-stage rings (one
//    16-row box per 16 tokens through the block table) and refills a stage
//    when the MMAs that read it completed.
// Every wait is bounded by wall time, and no barrier between the softmax
// warps is an unbounded one: their exchanges go through mbarriers. A wait
// that gives up records the failure, sets a shared abort flag that ends the
// other waits, and the roles drain their loads and MMAs before the tensor
// memory is freed; the unit then leaves zeros (or an empty partial).
#include <math_constants.h>

#include <type_traits>

#include "decode_args.h"
#include "decode_kernel.cuh"
#include "device_common.cuh"
#include "tc_common.cuh"

namespace paged {
namespace {

constexpr int kTok = 128;                // tokens per tile (M of S^T)
constexpr int kN = 16;                   // N of both products: 2G <= 16 query rows
constexpr int kStages = 3;               // K and V ring depth
constexpr int kTileBytes = kTok * 128;   // one K (or V) tile: 128 rows of 128 B
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4, kTmaWarp = 5, kThreads = 192;
constexpr uint32_t kTmemCols = 64;       // S^T x 2 (columns 0, 16), O^T (32)
constexpr uint32_t kColO = 32;
// shared memory from the 1024-aligned base
constexpr int kOffV = kStages * kTileBytes;
constexpr int kOffQ = 2 * kStages * kTileBytes;
constexpr int kOffP = kOffQ + kN * 128;            // [2 buffers][hi, lo][128 tokens][16 B]
constexpr int kPBuf = 2 * kTok * 16;
constexpr int kOffIds = kOffP + 2 * kPBuf;
constexpr float kLazy = 8.f;             // base-2 margin of the lazy maximum

// Byte offset of 16-byte chunk c of row r of a 128-byte-swizzled K-major
// operand (8-row groups of 1024 bytes).
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// Floats as integers of the same order (for an integer warp maximum).
__device__ __forceinline__ int ord_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float float_of(int i) {
  return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF);
}

template <class QF>
__device__ __forceinline__ float2 q_pair(uint32_t w) {
  if constexpr (std::is_same<QF, BF16>::value)
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  const __half2 h = *reinterpret_cast<const __half2*>(&w);
  return __half22float2(h);
}

template <class QF, int G>
__global__ void __launch_bounds__(kThreads, 2)
    paged_decode_fp8_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                               const __grid_constant__ CUtensorMap vmap) {
  static_assert(G >= 1 && 2 * G <= kN, "query group");
  constexpr int NL = G <= 4 ? 8 : 16;   // S^T / O^T columns a thread loads
  constexpr int TR = kTileRows;         // 16 tokens per TMA box
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = smem + kOffQ;
  uint8_t* sp = smem + kOffP;
  int32_t* ids = reinterpret_cast<int32_t*>(smem + kOffIds);
  auto sk = [&](int k) { return smem + (k % kStages) * kTileBytes; };
  auto sv = [&](int k) { return smem + kOffV + (k % kStages) * kTileBytes; };
  // kfull/vfull: a tile's boxes landed; kempty/vempty: the MMAs reading the
  // stage completed; s_full[b]: S^T buffer b computed; s_free[b]: the softmax
  // warps read it; p_full[b]: P' buffer b written (and O rescaled);
  // p_free[b]: O += P V that read it completed; red_bar[b]: the four warps'
  // tile maxima posted; sum_bar: their partial sums posted.
  __shared__ uint64_t kfull[kStages], kempty[kStages], vfull[kStages], vempty[kStages],
      s_full[2], s_free[2], p_full[2], p_free[2], red_bar[2], sum_bar, drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int aborted;
  __shared__ float qscale_s[G];
  __shared__ float red[2][kSoftmaxWarps][G];
  __shared__ float lsum[kSoftmaxWarps][G];

  const int kvh = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t lim = a.wait_limit_ns;
  if (tid == 0) {
    for (int r = 0; r < kStages; ++r) {
      mbar_init(&kfull[r], 1);
      mbar_init(&kempty[r], 1);
      mbar_init(&vfull[r], 1);
      mbar_init(&vempty[r], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSoftmaxWarps);
      mbar_init(&p_full[b], kSoftmaxWarps);
      mbar_init(&p_free[b], 1);
      mbar_init(&red_bar[b], kSoftmaxWarps);
    }
    mbar_init(&sum_bar, kSoftmaxWarps);
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
    aborted = 0;
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  // Everything below reads data of earlier kernels in the stream (the cache
  // rows the scatter kernel wrote): wait for them here.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (tid == 0 && part == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  const int nblk = (ctx + a.block_size - 1) / a.block_size;
  const int parts = nblk == 0 ? 1 : (nblk + a.partition_blocks - 1) / a.partition_blocks;
  if (part >= parts) return;
  const int b_begin = part * a.partition_blocks;
  const int nlocal = min(b_begin + a.partition_blocks, nblk) - b_begin;
  const int tok0 = b_begin * a.block_size;
  const int ntok = max(0, min(ctx, (b_begin + nlocal) * a.block_size) - tok0);
  const int ntiles = (ntok + kTok - 1) / kTok;

  // Block ids of this unit -> shared memory, validated once.
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
  for (int i = tid; i < nlocal; i += kThreads) {
    int32_t id = table[b_begin + i];
    if (id < 0 || id >= a.num_blocks) {
      report(a.err, kErrBadBlockId);
      id = -1;  // read as a box outside the pool: zero-filled
    }
    ids[i] = id;
  }
  // Q' -> shared memory: one warp per query head; lane l holds dims 4l..4l+3
  if (warp < kSoftmaxWarps) {
    for (int g = warp; g < G; g += kSoftmaxWarps) {
      const uint2 raw = *reinterpret_cast<const uint2*>(
          static_cast<const uint8_t*>(a.query) +
          ((static_cast<int64_t>(s) * a.num_heads + kvh * G + g) * 128 + 4 * lane) * 2);
      const float2 f0 = q_pair<QF>(raw.x), f1 = q_pair<QF>(raw.y);
      float mq = fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mq = fmaxf(mq, __shfl_xor_sync(FULL, mq, o));
      int e = 0;
      if (mq > 0.f && isfinite(mq)) {
        int k2;
        frexpf(mq, &k2);                  // mq < 2^k2
        e = min(max(8 - k2, -100), 100);  // mq * 2^e < 2^8
      }
      uint32_t hi, lo;
      tc::split_fp8x4<false>(ldexpf(f0.x, e), ldexpf(f0.y, e), ldexpf(f1.x, e), ldexpf(f1.y, e),
                             hi, lo);
      const int c = lane >> 2, b = (lane & 3) * 4;
      *reinterpret_cast<uint32_t*>(sq + sw128_off(g, c) + b) = hi;
      *reinterpret_cast<uint32_t*>(sq + sw128_off(G + g, c) + b) = lo;
      if (lane == 0) qscale_s[g] = a.scale_log2 * a.k_scale[kvh] * ldexpf(1.f, -e);
    }
    for (int i = tid; i < (kN - 2 * G) * 8; i += kSoftmaxWarps * 32)
      *reinterpret_cast<uint4*>(sq + sw128_off(2 * G + i / 8, i % 8)) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  __syncthreads();  // barrier initialisation, ids and Q' visible to every thread
  if (warp == kMmaWarp) tc::alloc(&tmem_slot, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp == kTmaWarp) {
    // ================= TMA loads (one thread) =================
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      auto issue = [&](int k, bool is_v) {
        uint8_t* dst = is_v ? sv(k) : sk(k);
        uint64_t* bar = is_v ? &vfull[k % kStages] : &kfull[k % kStages];
        const CUtensorMap* map = is_v ? &vmap : &kmap;
        const int u0 = k * kTok;
        const int nsub = (min(kTok, ntok - u0) + TR - 1) / TR;  // boxes holding context tokens
        if (!is_v && a.skip_tile >= u0 / TR && a.skip_tile < u0 / TR + nsub &&
            skip_for_test(a.skip_tile, a.skip_tile))
          return;
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nsub * TR * 128));
        for (int j = 0; j < nsub; ++j) {
          const int u = u0 + j * TR;
          const int32_t bid = ids[u / a.block_size];
          const int32_t row0 = bid >= 0 ? bid * a.block_size + u % a.block_size : -TR;
          tma_load_4d(dst + j * TR * 128, map, bar, 0, row0, kvh, 0, policy);
        }
      };
      bool ok = true;
      int k_issued = 0, v_issued = 0, k = 0;
      for (; ok && k < ntiles; ++k) {
        if (k >= kStages)
          ok = mbar_wait(&kempty[k % kStages], ((k - kStages) / kStages) & 1, lim, &aborted);
        if (!ok) break;
        issue(k, false);
        k_issued = k + 1;
        if (k >= kStages)
          ok = mbar_wait(&vempty[k % kStages], ((k - kStages) / kStages) & 1, lim, &aborted);
        if (!ok) break;
        issue(k, true);
        v_issued = k + 1;
      }
      if (!ok) {
        record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 0, k, ntiles, 0);
        aborted = 1;
        report(a.err, kErrWaitTimeout);
      }
      // every issued load lands before the CTA's shared memory goes away
      for (int j = max(0, k_issued - kStages); j < k_issued; ++j)
        mbar_wait(&kfull[j % kStages], (j / kStages) & 1, lim);
      for (int j = max(0, v_issued - kStages); j < v_issued; ++j)
        mbar_wait(&vfull[j % kStages], (j / kStages) & 1, lim);
    }
  } else if (warp == kMmaWarp) {
    // ================= MMA issue (one thread) =================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = tc::idesc_f8_ab<0, 0, kTok, kN, false, false>();
      constexpr uint32_t IDESC_O_HI = tc::idesc_f8_ab<0, 0, kTok, kN, true, true>();
      constexpr uint32_t IDESC_O_LO = tc::idesc_f8_ab<0, 1, kTok, kN, true, true>();
      // descriptors computed once; a k-step or stage offset is added to the
      // start-address field (16-byte units)
      const uint64_t qd = tc::sw128_desc(sq, 16, 1024);
      const uint64_t kd0 = tc::sw128_desc(smem, 16, 1024);
      const uint64_t vd0 = tc::sw128_desc(smem + kOffV, kTileBytes, 1024);
      const uint64_t pd0 = tc::plain_desc(sp, 128, 128);
      int k = 0;
      auto issue_s = [&](int kk_tile) {  // S^T of tile kk_tile into buffer kk_tile & 1
        if (kk_tile >= 2 &&
            !mbar_wait(&s_free[kk_tile & 1], ((kk_tile - 2) >> 1) & 1, lim, &aborted))
          return false;
        if (!mbar_wait(&kfull[kk_tile % kStages], (kk_tile / kStages) & 1, lim, &aborted))
          return false;
        tc::fence_after_sync();
        const uint64_t kd = kd0 + static_cast<uint64_t>(((kk_tile % kStages) * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 32 dims (bytes) per K step
          tc::mma_f8(tmem + (kk_tile & 1) * kN, kd + 2 * kk, qd + 2 * kk, IDESC_S, kk > 0);
        tc::commit(&s_full[kk_tile & 1]);
        tc::commit(&kempty[kk_tile % kStages]);
        return true;
      };
      bool ok = ntiles == 0 || issue_s(0);
      for (; ok && k < ntiles; ++k) {
        if (k + 1 < ntiles) ok = issue_s(k + 1);
        if (!ok) break;
        ok = mbar_wait(&vfull[k % kStages], (k / kStages) & 1, lim, &aborted) &&
             mbar_wait(&p_full[k & 1], (k >> 1) & 1, lim, &aborted);
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t vd = vd0 + static_cast<uint64_t>(((k % kStages) * kTileBytes) >> 4);
        const uint64_t ph = pd0 + static_cast<uint64_t>(((k & 1) * kPBuf) >> 4);
        const uint64_t pl = ph + static_cast<uint64_t>((kTok * 16) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTok / 32; ++kk) {  // 32 tokens per K step
          const uint64_t av = vd + static_cast<uint64_t>((kk * 32 * 128) >> 4);
          const uint64_t off = static_cast<uint64_t>((kk * 32 * 16) >> 4);
          tc::mma_f8(tmem + kColO, av, ph + off, IDESC_O_HI, k > 0 || kk > 0);
          tc::mma_f8(tmem + kColO, av, pl + off, IDESC_O_LO, true);
        }
        tc::commit(&p_free[k & 1]);
        tc::commit(&vempty[k % kStages]);
      }
      if (!ok) {
        // A wait gave up (never expected): let this CTA's MMAs finish (bounded)
        // before its tensor and shared memory go away.
        record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 1, k, ntiles, 0);
        aborted = 1;
        report(a.err, kErrWaitTimeout);
        tc::commit(&drain_bar);
        mbar_wait(&drain_bar, 0, lim);
      }
    }
  } else {
    // ================= softmax warps =================
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m[G], l[G], qs[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -CUDART_INF_F;
      l[g] = 0.f;
      qs[g] = qscale_s[g];
    }
    bool ok = true;
    int k = 0;
    for (; ok && k < ntiles; ++k) {
      ok = __all_sync(FULL, mbar_wait(&s_full[k & 1], (k >> 1) & 1, lim, &aborted));
      if (!ok) break;
      tc::fence_after_sync();
      uint32_t r[NL];
      if constexpr (NL == 8) tc::ld8_nowait(tmem + (k & 1) * kN + lane_base, r);
      else tc::ld16_nowait(tmem + (k & 1) * kN + lane_base, r);
      tc::wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[k & 1]);
      const int vk = min(kTok, ntok - k * kTok);  // context tokens in this tile
      const bool live = tid < vk;
      float x[G];
#pragma unroll
      for (int g = 0; g < G; ++g)
        x[g] = live ? (__uint_as_float(r[g]) + __uint_as_float(r[G + g])) * qs[g]
                    : -CUDART_INF_F;
      // the tile's maximum per head over the CTA
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int mx = __reduce_max_sync(FULL, ord_of(x[g]));
        if (lane == 0) red[k & 1][warp][g] = float_of(mx);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_bar[k & 1]);
      ok = __all_sync(FULL, mbar_wait(&red_bar[k & 1], (k >> 1) & 1, lim, &aborted));
      if (!ok) break;
      float alpha[G];
      bool rescale = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float tmax = red[k & 1][0][g];
#pragma unroll
        for (int w = 1; w < kSoftmaxWarps; ++w) tmax = fmaxf(tmax, red[k & 1][w][g]);
        alpha[g] = 1.f;
        if (tmax > m[g] + kLazy) {  // false while the head has seen nothing
          alpha[g] = tc::ex2(m[g] - tmax);
          m[g] = tmax;
          rescale = true;
        }
      }
      float p[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) p[g] = 0.f;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mu = m[g] == -CUDART_INF_F ? 0.f : m[g];
        p[g] = tc::ex2(x[g] - mu);
        l[g] = fmaf(l[g], alpha[g], p[g]);
      }
      // O^T may be rescaled only once O += P V of tile k-1 completed (rare:
      // the maximum moves lazily); the same for every thread of the CTA
      if (rescale && k >= 1) {
        ok = __all_sync(FULL, mbar_wait(&p_free[(k - 1) & 1], ((k - 1) >> 1) & 1, lim, &aborted));
        if (!ok) break;
        tc::fence_after_sync();
        uint32_t o[NL];
        if constexpr (NL == 8) tc::ld8_nowait(tmem + kColO + lane_base, o);
        else tc::ld16_nowait(tmem + kColO + lane_base, o);
        tc::wait_ld();
#pragma unroll
        for (int g = 0; g < G; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
        if constexpr (NL == 8) tc::st8u(tmem + kColO + lane_base, o);
        else tc::st16u(tmem + kColO + lane_base, o);
        tc::wait_st();
      }
      // P' buffer k & 1 is free once O += P V of tile k-2 completed
      if (k >= 2) {
        ok = __all_sync(FULL, mbar_wait(&p_free[k & 1], ((k - 2) >> 1) & 1, lim, &aborted));
        if (!ok) break;
      }
      uint32_t hw[4], lw[4];
      tc::split_fp8x4<true>(p[0], p[1], p[2], p[3], hw[0], lw[0]);
      if constexpr (G > 4) {
        tc::split_fp8x4<true>(p[4], p[5], p[6], p[7], hw[1], lw[1]);
      } else {
        hw[1] = lw[1] = 0u;
      }
      hw[2] = hw[3] = lw[2] = lw[3] = 0u;
      uint8_t* prow = sp + (k & 1) * kPBuf + tid * 16;
      *reinterpret_cast<uint4*>(prow) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(prow + kTok * 16) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      // V rows without context tokens (end of the unit) may hold anything,
      // even NaN codes, and 0 * NaN is NaN inside the MMA: clear them once
      // the tile's loads landed
      if (vk < kTok) {
        ok = __all_sync(FULL, mbar_wait(&vfull[k % kStages], (k / kStages) & 1, lim, &aborted));
        if (!ok) break;
        if (!live) {
          uint4* row = reinterpret_cast<uint4*>(sv(k) + tid * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[k & 1]);
    }
    if (ok && ntiles > 0)
      ok = __all_sync(FULL, mbar_wait(&p_free[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, lim,
                                      &aborted));
    // A warp that gave up says so before it posts its sums, so that the
    // others, which wait for those, see the flag.
    if (!ok && lane == 0) {
      record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 2, k, ntiles, 0);
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    // the partial sums over the CTA (every softmax warp posts its own)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float v = l[g];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
      if (lane == 0) lsum[warp][g] = v;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sum_bar);
    const bool sums = __all_sync(FULL, mbar_wait(&sum_bar, 0, lim, &aborted));
    if (!sums && lane == 0) {
      record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 3, k, ntiles, 0);
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    __syncwarp();
    ok = __all_sync(FULL, ok && sums && *static_cast<volatile int*>(&aborted) == 0);
    const bool single = parts == 1;
    const int64_t row0 = static_cast<int64_t>(s) * a.num_heads + kvh * G;
    if (!ok) {
      // The unit's result is lost: leave zeros (single pass) or an empty
      // partial that the combine kernel gives no weight, never stale data.
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if (single) store_out(QF{}, a.out, (row0 + g) * 128 + tid, 0.f);
        else if (tid == 0) a.ws_ml[(row0 + g) * a.max_parts + part] = make_float2(-CUDART_INF_F, 0.f);
      }
    } else {
      // ---- epilogue: thread i holds dimension i of every head's O
      float L[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        L[g] = 0.f;
#pragma unroll
        for (int w = 0; w < kSoftmaxWarps; ++w) L[g] += lsum[w][g];
      }
      uint32_t o[NL];
#pragma unroll
      for (int i = 0; i < NL; ++i) o[i] = 0u;
      if (ntiles > 0) {
        tc::fence_after_sync();
        if constexpr (NL == 8) tc::ld8_nowait(tmem + kColO + lane_base, o);
        else tc::ld16_nowait(tmem + kColO + lane_base, o);
        tc::wait_ld();
      }
      const float vs = a.v_scale[kvh];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float val = L[g] > 0.f ? __uint_as_float(o[g]) / L[g] * vs : 0.f;
        if (single) {
          store_out(QF{}, a.out, (row0 + g) * 128 + tid, val);
        } else {
          const int64_t pi = (row0 + g) * a.max_parts + part;
          a.ws_o[pi * 128 + tid] = val;
          if (tid == 0) a.ws_ml[pi] = make_float2(m[g], L[g]);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::dealloc(tmem, kTmemCols);
  }
}

template <class QF, int G>
cudaError_t launch_one(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t stream) {
  if (a.partition_blocks > kMaxUnitBlocks) return cudaErrorNotSupported;
  const size_t smem = 1024 + kOffIds + 4 * static_cast<size_t>(a.partition_blocks);
  auto kern = paged_decode_fp8_tc_kernel<QF, G>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(a.num_kv_heads, a.num_seqs, a.max_parts), kThreads, smem, stream,
                    a, kmap, vmap);
}

}  // namespace

cudaError_t decode_fp8_tc(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int q_dtype, int group, cudaStream_t stream) {
#define PAGED_FP8TC(QF, g) \
  if (group == g) return launch_one<QF, g>(a, kmap, vmap, stream);
  if (q_dtype == kF16) {
    PAGED_FP8TC(F16, 1) PAGED_FP8TC(F16, 2) PAGED_FP8TC(F16, 4) PAGED_FP8TC(F16, 8)
  } else if (q_dtype == kBF16) {
    PAGED_FP8TC(BF16, 1) PAGED_FP8TC(BF16, 2) PAGED_FP8TC(BF16, 4) PAGED_FP8TC(BF16, 8)
  }
#undef PAGED_FP8TC
  return cudaErrorNotSupported;
}

}  // namespace paged
