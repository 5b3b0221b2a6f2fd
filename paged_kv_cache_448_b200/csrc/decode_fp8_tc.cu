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
// A CTA is one work unit (kv-head, sequence, context partition) with nine
// warps:
//  * four softmax warps: thread i owns tensor-memory lane i, i.e. token i of
//    the tile in S^T and dimension i of O^T. Per tile it loads its S^T row,
//    forms the G logits (masking tokens past the context), and the CTA takes
//    each head's tile maximum (an ordered-integer warp reduction, then the
//    four warps through shared memory behind an mbarrier). The running
//    maximum moves only when a tile's maximum passes it by more than 8
//    (base 2), so probabilities stay below 2^8 and O is rarely rescaled (in
//    tensor memory, after the previous O += P V completed). Each thread keeps
//    its own partial sums, added over the CTA at the end;
//  * the MMA warp (one thread) owns the tensor memory: two 16-column S^T
//    buffers and 16 columns of O^T. It polls and issues whichever is ready:
//    S^T of the next tile, or O^T += V^T P'^T of the oldest tile whose P' is
//    posted;
//  * four TMA warps, two per ring: K tiles and V tiles are loaded each on its
//    own (a V stage is held until O += P V, and that must not hold back a K
//    load), and box j of a tile is issued by lane j / 2 of the ring's warp
//    j % 2, the lanes of a warp at once, so a tile's 8 boxes are all in
//    flight soon after its stage is free.
// A tile's time is the latency of that chain (loads, S, the softmax with its
// exchange, O += P V), so throughput comes from units in flight: two K and
// two V stages keep a CTA near 70 KB of shared memory, and three CTAs share
// an SM (query groups up to 4).
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
constexpr int kN = 16;                   // N of both products: hi and lo query rows, padded
constexpr int kStagesK = 2, kStagesV = 2;
constexpr int kTileBytes = kTok * 128;   // one K (or V) tile: 128 rows of 128 B
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kTmaWarp = 5;              // TMA warps 5, 6 load K tiles, 7, 8 V tiles
constexpr int kRingWarps = 2;            // TMA warps per ring
constexpr int kThreads = (kTmaWarp + 2 * kRingWarps) * 32;
constexpr uint32_t kTmemCols = 64;       // S^T x 2 (columns 0, 16), O^T (32)
constexpr uint32_t kColO = 32;
// shared memory from the 1024-aligned base
constexpr int kOffV = kStagesK * kTileBytes;
constexpr int kOffQ = (kStagesK + kStagesV) * kTileBytes;
constexpr int kOffP = kOffQ + kN * 128;  // P': [hi, lo][128 tokens][16 B]
constexpr int kPBuf = 2 * kTok * 16;
constexpr int kOffIds = kOffP + kPBuf;
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
__global__ void __launch_bounds__(kThreads, G <= 4 ? 3 : 2)
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
  auto sk = [&](int k) { return smem + (k % kStagesK) * kTileBytes; };
  auto sv = [&](int k) { return smem + kOffV + (k % kStagesV) * kTileBytes; };
  // kfull/vfull: a tile's boxes landed (one arrival per TMA warp of the
  // ring); kempty/vempty: the MMAs reading the stage completed; s_full[b]:
  // S^T buffer b computed; s_free[b]: the softmax warps read it; p_full: P'
  // written (and O rescaled); p_free: O += P V that read it completed;
  // red_bar[b]: the four warps' tile maxima posted; sum_bar: their partial
  // sums posted.
  __shared__ uint64_t kfull[kStagesK], kempty[kStagesK], vfull[kStagesV], vempty[kStagesV],
      s_full[2], s_free[2], p_full, p_free, red_bar[2], sum_bar, drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int aborted;
  __shared__ float qscale_s[G];
  __shared__ float red[2][kSoftmaxWarps][G];
  __shared__ float lsum[kSoftmaxWarps][G];

  const int kvh = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t lim = a.wait_limit_ns;
  if (tid == 0) {
    for (int r = 0; r < kStagesK; ++r) {
      mbar_init(&kfull[r], kRingWarps);
      mbar_init(&kempty[r], 1);
    }
    for (int r = 0; r < kStagesV; ++r) {
      mbar_init(&vfull[r], kRingWarps);
      mbar_init(&vempty[r], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSoftmaxWarps);
      mbar_init(&red_bar[b], kSoftmaxWarps);
    }
    mbar_init(&p_full, kSoftmaxWarps);
    mbar_init(&p_free, 1);
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

  if (warp >= kTmaWarp) {
    // ================= TMA loads: two warps per ring =================
    // Box j of a tile is issued by lane j / kRingWarps of the ring's warp
    // j % kRingWarps; each warp's lane 0 posts the bytes of its boxes.
    const int producer = warp - kTmaWarp;
    const bool is_v = producer >= kRingWarps;
    const int pr = producer % kRingWarps;
    const int NS_ = is_v ? kStagesV : kStagesK;
    uint64_t* full = is_v ? vfull : kfull;
    uint64_t* empty = is_v ? vempty : kempty;
    const CUtensorMap* map = is_v ? &vmap : &kmap;
    const uint64_t policy = l2_policy_evict_first();
    bool ok = true;
    int k = 0, issued = 0;
    for (; k < ntiles; ++k) {
      if (k >= NS_)
        ok = __all_sync(FULL, mbar_wait(&empty[k % NS_], ((k - NS_) / NS_) & 1, lim, &aborted));
      if (!ok) break;
      uint8_t* dst = is_v ? sv(k) : sk(k);
      uint64_t* bar = &full[k % NS_];
      const int u0 = k * kTok;
      const int nsub = (min(kTok, ntok - u0) + TR - 1) / TR;  // boxes holding context tokens
      issued = k + 1;
      if (!is_v && a.skip_tile >= u0 / TR && a.skip_tile < u0 / TR + nsub &&
          skip_for_test(a.skip_tile, a.skip_tile))
        continue;  // (both K warps leave it out: the tile never completes)
      const int mine = nsub > pr ? (nsub - pr + kRingWarps - 1) / kRingWarps : 0;
      if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(mine * TR * 128));
      __syncwarp();
      if (lane < mine) {
        const int j = pr + kRingWarps * lane;
        const int u = u0 + j * TR;
        const int32_t bid = ids[u / a.block_size];
        const int32_t row0 = bid >= 0 ? bid * a.block_size + u % a.block_size : -TR;
        tma_load_4d(dst + j * TR * 128, map, bar, 0, row0, kvh, 0, policy);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 0, k, ntiles, producer);
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    // every load this warp issued lands before the CTA's shared memory goes
    // away (the last use of each stage; earlier ones were consumed)
    if (lane == 0)
      for (int t = max(0, issued - NS_); t < issued; ++t)
        mbar_wait(&full[t % NS_], (t / NS_) & 1, lim);
    __syncwarp();  // whole warps reach the CTA barrier below
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
      const uint64_t ph = tc::plain_desc(sp, 128, 128);
      const uint64_t pl = ph + static_cast<uint64_t>((kTok * 16) >> 4);
      // Issue whichever is ready: S of the next tile (its S buffer read by the
      // softmax warps, its K landed) or O += P V of the oldest tile whose P
      // is posted (and V landed), so neither waits behind the other. Gives
      // up after the wait limit without progress.
      bool ok = true;
      int ns = 0, k = 0;  // next tile for S, for P V
      uint64_t t_last = global_timer_ns();
      while (k < ntiles) {
        bool progress = false;
        if (ns < ntiles && (ns < 2 || mbar_test_wait(&s_free[ns & 1], ((ns - 2) >> 1) & 1)) &&
            mbar_test_wait(&kfull[ns % kStagesK], (ns / kStagesK) & 1)) {
          tc::fence_after_sync();
          const uint64_t kd = kd0 + static_cast<uint64_t>(((ns % kStagesK) * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 32 dims (bytes) per K step
            tc::mma_f8(tmem + (ns & 1) * kN, kd + 2 * kk, qd + 2 * kk, IDESC_S, kk > 0);
          tc::commit(&s_full[ns & 1]);
          tc::commit(&kempty[ns % kStagesK]);
          ++ns;
          progress = true;
        }
        if (k < ns && mbar_test_wait(&vfull[k % kStagesV], (k / kStagesV) & 1) &&
            mbar_test_wait(&p_full, k & 1)) {
          tc::fence_after_sync();
          const uint64_t vd = vd0 + static_cast<uint64_t>(((k % kStagesV) * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTok / 32; ++kk) {  // 32 tokens per K step
            const uint64_t av = vd + static_cast<uint64_t>((kk * 32 * 128) >> 4);
            const uint64_t off = static_cast<uint64_t>((kk * 32 * 16) >> 4);
            tc::mma_f8(tmem + kColO, av, ph + off, IDESC_O_HI, k > 0 || kk > 0);
            tc::mma_f8(tmem + kColO, av, pl + off, IDESC_O_LO, true);
          }
          tc::commit(&p_free);
          tc::commit(&vempty[k % kStagesV]);
          ++k;
          progress = true;
        }
        if (progress) {
          t_last = global_timer_ns();
        } else if (aborted || global_timer_ns() - t_last > lim) {
          ok = false;
          break;
        }
      }
      if (!ok) {
        // A wait gave up (never expected): let this CTA's MMAs finish (bounded)
        // before its tensor and shared memory go away.
        record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 1, k, ntiles, ns);
        aborted = 1;
        report(a.err, kErrWaitTimeout);
        tc::commit(&drain_bar);
        mbar_wait(&drain_bar, 0, lim);
      }
    }
    __syncwarp();  // whole warps reach the CTA barrier below
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
      tc::wait_ld(r);
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
      // P' has one buffer, rewritten (and O^T rescaled) once O += P V of the
      // previous tile completed
      if (k >= 1) {
        ok = __all_sync(FULL, mbar_wait(&p_free, (k - 1) & 1, lim, &aborted));
        if (!ok) break;
      }
      if (rescale && k >= 1) {  // rare: the maximum moves lazily; the same in every thread
        tc::fence_after_sync();
        uint32_t o[NL];
        if constexpr (NL == 8) tc::ld8_nowait(tmem + kColO + lane_base, o);
        else tc::ld16_nowait(tmem + kColO + lane_base, o);
        tc::wait_ld(o);
#pragma unroll
        for (int g = 0; g < G; ++g) o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
        if constexpr (NL == 8) tc::st8u(tmem + kColO + lane_base, o);
        else tc::st16u(tmem + kColO + lane_base, o);
        tc::wait_st();
      }
      uint32_t hw[4], lw[4];
      tc::split_fp8x4<true>(p[0], p[1], p[2], p[3], hw[0], lw[0]);
      if constexpr (G > 4) {
        tc::split_fp8x4<true>(p[4], p[5], p[6], p[7], hw[1], lw[1]);
      } else {
        hw[1] = lw[1] = 0u;
      }
      hw[2] = hw[3] = lw[2] = lw[3] = 0u;
      *reinterpret_cast<uint4*>(sp + tid * 16) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sp + kTok * 16 + tid * 16) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      // V rows without context tokens (end of the unit) may hold anything,
      // even NaN codes, and 0 * NaN is NaN inside the MMA: clear them once
      // the tile's loads landed
      if (vk < kTok) {
        ok = __all_sync(FULL, mbar_wait(&vfull[k % kStagesV], (k / kStagesV) & 1, lim, &aborted));
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
      if (lane == 0) mbar_arrive(&p_full);
    }
    if (ok && ntiles > 0)
      ok = __all_sync(FULL, mbar_wait(&p_free, (ntiles - 1) & 1, lim, &aborted));
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
    // A unit whose result is lost leaves zeros (single pass) or an empty
    // partial that the combine kernel gives no weight, never stale data.
    const bool good = __all_sync(FULL, ok && sums && *static_cast<volatile int*>(&aborted) == 0);
    // ---- epilogue: thread i holds dimension i of every head's O
    uint32_t o[NL];
#pragma unroll
    for (int i = 0; i < NL; ++i) o[i] = 0u;
    if (good && ntiles > 0) {
      tc::fence_after_sync();
      if constexpr (NL == 8) tc::ld8_nowait(tmem + kColO + lane_base, o);
      else tc::ld16_nowait(tmem + kColO + lane_base, o);
      tc::wait_ld(o);
    }
    const bool single = parts == 1;
    const int64_t row0 = static_cast<int64_t>(s) * a.num_heads + kvh * G;
    const float vs = a.v_scale[kvh];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < kSoftmaxWarps; ++w) L += lsum[w][g];
      const bool has = good && L > 0.f;
      const float val = has ? __uint_as_float(o[g]) / L * vs : 0.f;
      if (single) {
        store_out(QF{}, a.out, (row0 + g) * 128 + tid, val);
      } else {
        const int64_t pi = (row0 + g) * a.max_parts + part;
        a.ws_o[pi * 128 + tid] = val;
        if (tid == 0) a.ws_ml[pi] = has ? make_float2(m[g], L) : make_float2(-CUDART_INF_F, 0.f);
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

int decode_fp8_tc_heads_per_cta(int, int) { return 1; }

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
