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
//    its own partial sums; they are added across the CTA at the end;
//  * the MMA warp (one thread) owns the tensor memory: two 16-column S^T
//    buffers and 16 columns of O^T. It issues S^T of tile k+1 before
//    O^T += V^T P'^T of tile k, so S is computed under the softmax of tile k;
//  * four TMA warps (one thread each, every fourth tile) load K and V tiles
//    into 3-stage rings (one 16-row box per 16 tokens through the block
//    table) and refill a stage when the MMAs that read it completed.
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

constexpr int kTok = 128;                // rows per tile (M of S^T): tokens x kv-heads
constexpr int kN = 16;                   // N of O^T: query heads of the CTA, padded
constexpr int kStages = 3;               // K and V ring depth
constexpr int kTileBytes = kTok * 128;   // one K (or V) tile: 128 rows of 128 B
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4, kTmaWarp = 5;  // TMA warps 5 .. 5 + kProducers - 1
constexpr int kProducers = 4;               // tile k is loaded by TMA warp k % kProducers
constexpr int kThreads = (kTmaWarp + kProducers) * 32;
// shared memory from the 1024-aligned base
constexpr int kOffV = kStages * kTileBytes;
constexpr int kOffQ = 2 * kStages * kTileBytes;
constexpr int kOffP = kOffQ + 32 * 128;            // [2 buffers][hi, lo][128 rows][16 B]
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

// H2 kv-heads per CTA (1 or 2): one TMA box carries 16 tokens of all H2
// heads, [head][16 rows][128 B], so tile row i is head (i / 16) % H2, token
// (i / (16 H2)) * 16 + i % 16 of the tile; the HG = H2 G query heads of the
// CTA are the columns, and a row uses those of its own kv-head.
template <class QF, int G, int H2>
__global__ void __launch_bounds__(kThreads, 2)
    paged_decode_fp8_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                               const __grid_constant__ CUtensorMap vmap) {
  constexpr int HG = G * H2;             // query heads of the CTA
  static_assert(G >= 1 && (H2 == 1 || H2 == 2) && 2 * HG <= 16, "query group");
  constexpr int NS = 16;                  // S^T columns: per query head hi and lo parts
  constexpr uint32_t kTmemCols = 64;      // S^T x 2 (columns 0, 16), then O^T (32)
  constexpr uint32_t kColO = 2 * NS;
  constexpr int TT = kTok / H2;           // context tokens per tile
  constexpr int TR = kTileRows;           // 16 tokens per TMA box
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
  __shared__ int last_k[kStages], last_v[kStages];  // last tile loaded into each stage
  __shared__ float qscale_s[HG];
  __shared__ float red[2][kSoftmaxWarps][HG];
  __shared__ float lsum[kSoftmaxWarps][HG];

  const int kvh = blockIdx.x * H2, s = blockIdx.y, part = blockIdx.z;  // first kv-head
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
    for (int r = 0; r < kStages; ++r) last_k[r] = last_v[r] = -1;
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
  const int ntiles = (ntok + TT - 1) / TT;

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
  // Q' -> shared memory: one warp per query head n (of kv-head kvh + n / G);
  // its hi and lo rows are 2G (n / G) + n % G and that + G; lane l holds
  // dims 4l..4l+3
  if (warp < kSoftmaxWarps) {
    for (int n = warp; n < HG; n += kSoftmaxWarps) {
      const int g = (n / G) * 2 * G + n % G;  // hi row
      const uint2 raw = *reinterpret_cast<const uint2*>(
          static_cast<const uint8_t*>(a.query) +
          ((static_cast<int64_t>(s) * a.num_heads + kvh * G + n) * 128 + 4 * lane) * 2);
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
      if (lane == 0) qscale_s[n] = a.scale_log2 * a.k_scale[kvh + n / G] * ldexpf(1.f, -e);
    }
    for (int i = tid; i < (NS - 2 * HG) * 8; i += kSoftmaxWarps * 32)
      *reinterpret_cast<uint4*>(sq + sw128_off(2 * HG + i / 8, i % 8)) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  __syncthreads();  // barrier initialisation, ids and Q' visible to every thread
  if (warp == kMmaWarp) tc::alloc(&tmem_slot, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp >= kTmaWarp) {
    // ================= TMA loads (one thread per TMA warp) =================
    // Issuing a tensor load costs its thread hundreds of cycles, and a tile is
    // 16 boxes of 2 KB: the tiles are dealt to kProducers warps so that
    // enough loads are issued per SM.
    const int producer = warp - kTmaWarp;
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      auto issue = [&](int k, bool is_v) {
        uint8_t* dst = is_v ? sv(k) : sk(k);
        uint64_t* bar = is_v ? &vfull[k % kStages] : &kfull[k % kStages];
        const CUtensorMap* map = is_v ? &vmap : &kmap;
        const int u0 = k * TT;
        const int nsub = (min(TT, ntok - u0) + TR - 1) / TR;  // boxes holding context tokens
        if (!is_v && a.skip_tile >= u0 / TR && a.skip_tile < u0 / TR + nsub &&
            skip_for_test(a.skip_tile, a.skip_tile))
          return;
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nsub * H2 * TR * 128));
        for (int j = 0; j < nsub; ++j) {
          const int u = u0 + j * TR;
          const int32_t bid = ids[u / a.block_size];
          const int32_t row0 = bid >= 0 ? bid * a.block_size + u % a.block_size : -TR;
          tma_load_4d(dst + j * H2 * TR * 128, map, bar, 0, row0, kvh, 0, policy);
        }
      };
      bool ok = true;
      int k = producer;
      for (; ok && k < ntiles; k += kProducers) {
        if (k >= kStages)
          ok = mbar_wait(&kempty[k % kStages], ((k - kStages) / kStages) & 1, lim, &aborted);
        if (!ok) break;
        issue(k, false);
        atomicMax(&last_k[k % kStages], k);
        if (k >= kStages)
          ok = mbar_wait(&vempty[k % kStages], ((k - kStages) / kStages) & 1, lim, &aborted);
        if (!ok) break;
        issue(k, true);
        atomicMax(&last_v[k % kStages], k);
      }
      if (!ok) {
        record_failure(a.diag, kSiteFp8Tile, kvh, s, part, 0, k, ntiles, 0);
        aborted = 1;
        report(a.err, kErrWaitTimeout);
      }
    }
    // Every issued load lands before the CTA's shared memory goes away: once
    // all TMA warps stopped (their loops end in bounded time), the last load
    // of each stage is waited for (earlier ones were consumed before the stage
    // was reused). The warp reconverges first: the named barrier is executed
    // by whole warps.
    __syncwarp();
    asm volatile("bar.sync 1, %0;" ::"n"(kProducers * 32) : "memory");
    if (producer == 0 && lane == 0) {
      for (int r = 0; r < kStages; ++r) {
        if (last_k[r] >= 0) mbar_wait(&kfull[r], (last_k[r] / kStages) & 1, lim);
        if (last_v[r] >= 0) mbar_wait(&vfull[r], (last_v[r] / kStages) & 1, lim);
      }
    }
    __syncwarp();  // whole warps reach the CTA barrier below
  } else if (warp == kMmaWarp) {
    // ================= MMA issue (one thread) =================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = tc::idesc_f8_ab<0, 0, kTok, NS, false, false>();
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
          tc::mma_f8(tmem + (kk_tile & 1) * NS, kd + 2 * kk, qd + 2 * kk, IDESC_S, kk > 0);
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
    __syncwarp();  // whole warps reach the CTA barrier below
  } else {
    // ================= softmax warps =================
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int h = (tid / TR) % H2;                        // this row's kv-head (of the CTA)
    const int utok = (tid / (TR * H2)) * TR + tid % TR;   // and its token in the tile
    float m[HG], l[HG], qs[HG];
#pragma unroll
    for (int n = 0; n < HG; ++n) {
      m[n] = -CUDART_INF_F;
      l[n] = 0.f;
      qs[n] = qscale_s[n];
    }
    bool ok = true;
    int k = 0;
    for (; ok && k < ntiles; ++k) {
      ok = __all_sync(FULL, mbar_wait(&s_full[k & 1], (k >> 1) & 1, lim, &aborted));
      if (!ok) break;
      tc::fence_after_sync();
      uint32_t r[NS];
      tc::ld16_nowait(tmem + (k & 1) * NS + lane_base, r);
      tc::wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[k & 1]);
      const int vk = min(TT, ntok - k * TT);  // context tokens in this tile
      const bool live = utok < vk;
      // logits (base 2) of the query heads of this row's kv-head; -inf elsewhere
      float x[HG];
#pragma unroll
      for (int n = 0; n < HG; ++n) {
        const int c = (n / G) * 2 * G + n % G;
        x[n] = live && n / G == h
                   ? (__uint_as_float(r[c]) + __uint_as_float(r[c + G])) * qs[n]
                   : -CUDART_INF_F;
      }
      // the tile's maximum per query head over the CTA
#pragma unroll
      for (int n = 0; n < HG; ++n) {
        const int mx = __reduce_max_sync(FULL, ord_of(x[n]));
        if (lane == 0) red[k & 1][warp][n] = float_of(mx);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red_bar[k & 1]);
      ok = __all_sync(FULL, mbar_wait(&red_bar[k & 1], (k >> 1) & 1, lim, &aborted));
      if (!ok) break;
      float alpha[HG];
      bool rescale = false;
#pragma unroll
      for (int n = 0; n < HG; ++n) {
        float tmax = red[k & 1][0][n];
#pragma unroll
        for (int w = 1; w < kSoftmaxWarps; ++w) tmax = fmaxf(tmax, red[k & 1][w][n]);
        alpha[n] = 1.f;
        if (tmax > m[n] + kLazy) {  // false while the head has seen nothing
          alpha[n] = tc::ex2(m[n] - tmax);
          m[n] = tmax;
          rescale = true;
        }
      }
      float p[16];
#pragma unroll
      for (int n = 0; n < 16; ++n) p[n] = 0.f;
#pragma unroll
      for (int n = 0; n < HG; ++n) {
        const float mu = m[n] == -CUDART_INF_F ? 0.f : m[n];
        p[n] = tc::ex2(x[n] - mu);
        l[n] = fmaf(l[n], alpha[n], p[n]);
      }
      // O^T may be rescaled only once O += P V of tile k-1 completed (rare:
      // the maximum moves lazily); the same for every thread of the CTA
      if (rescale && k >= 1) {
        ok = __all_sync(FULL, mbar_wait(&p_free[(k - 1) & 1], ((k - 1) >> 1) & 1, lim, &aborted));
        if (!ok) break;
        tc::fence_after_sync();
        uint32_t o[16];
        tc::ld16_nowait(tmem + kColO + lane_base, o);
        tc::wait_ld();
#pragma unroll
        for (int n = 0; n < HG; ++n) o[n] = __float_as_uint(__uint_as_float(o[n]) * alpha[n]);
        tc::st16u(tmem + kColO + lane_base, o);
        tc::wait_st();
      }
      // P' buffer k & 1 is free once O += P V of tile k-2 completed
      if (k >= 2) {
        ok = __all_sync(FULL, mbar_wait(&p_free[k & 1], ((k - 2) >> 1) & 1, lim, &aborted));
        if (!ok) break;
      }
      uint32_t hw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int q = 0; q < (HG + 3) / 4; ++q)
        tc::split_fp8x4<true>(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3], hw[q], lw[q]);
      uint8_t* prow = sp + (k & 1) * kPBuf + tid * 16;
      *reinterpret_cast<uint4*>(prow) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(prow + kTok * 16) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      // V rows without context tokens (end of the unit) may hold anything,
      // even NaN codes, and 0 * NaN is NaN inside the MMA: clear them once
      // the tile's loads landed
      if (vk < TT) {
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
    for (int n = 0; n < HG; ++n) {
      float v = l[n];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
      if (lane == 0) lsum[warp][n] = v;
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
      for (int n = 0; n < HG; ++n) {
        if (single) store_out(QF{}, a.out, (row0 + n) * 128 + tid, 0.f);
        else if (tid == 0) a.ws_ml[(row0 + n) * a.max_parts + part] = make_float2(-CUDART_INF_F, 0.f);
      }
    } else {
      // ---- epilogue: thread i holds dimension i of every query head's O
      uint32_t o[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) o[i] = 0u;
      if (ntiles > 0) {
        tc::fence_after_sync();
        tc::ld16_nowait(tmem + kColO + lane_base, o);
        tc::wait_ld();
      }
#pragma unroll
      for (int n = 0; n < HG; ++n) {
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kSoftmaxWarps; ++w) L += lsum[w][n];
        const float val = L > 0.f ? __uint_as_float(o[n]) / L * a.v_scale[kvh + n / G] : 0.f;
        if (single) {
          store_out(QF{}, a.out, (row0 + n) * 128 + tid, val);
        } else {
          const int64_t pi = (row0 + n) * a.max_parts + part;
          a.ws_o[pi * 128 + tid] = val;
          if (tid == 0) a.ws_ml[pi] = make_float2(m[n], L);
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

template <class QF, int G, int H2>
cudaError_t launch_one(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       cudaStream_t stream) {
  if (a.partition_blocks > kMaxUnitBlocks || a.num_kv_heads % H2 != 0)
    return cudaErrorNotSupported;
  const size_t smem = 1024 + kOffIds + 4 * static_cast<size_t>(a.partition_blocks);
  auto kern = paged_decode_fp8_tc_kernel<QF, G, H2>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(a.num_kv_heads / H2, a.num_seqs, a.max_parts), kThreads, smem,
                    stream, a, kmap, vmap);
}

}  // namespace

// One kv-head per CTA. (A form with two kv-heads per CTA, one 4 KB box per
// 16 tokens, is written above as H2 = 2; it is not launched: on B200 it
// ended in an unspecified launch failure on the full-size shared-prefix
// workload with units of 8 or more of its tiles, with the cause not found.)
int decode_fp8_tc_heads_per_cta(int, int) { return 1; }

cudaError_t decode_fp8_tc(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int q_dtype, int group, cudaStream_t stream) {
#define PAGED_FP8TC(QF, g) \
  if (group == g) return launch_one<QF, g, 1>(a, kmap, vmap, stream);
  if (q_dtype == kF16) {
    PAGED_FP8TC(F16, 1) PAGED_FP8TC(F16, 2) PAGED_FP8TC(F16, 4) PAGED_FP8TC(F16, 8)
  } else if (q_dtype == kBF16) {
    PAGED_FP8TC(BF16, 1) PAGED_FP8TC(BF16, 2) PAGED_FP8TC(BF16, 4) PAGED_FP8TC(BF16, 8)
  }
#undef PAGED_FP8TC
  return cudaErrorNotSupported;
}

}  // namespace paged
