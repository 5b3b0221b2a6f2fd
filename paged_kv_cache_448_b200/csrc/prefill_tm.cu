// prefill_tm.cu — the multi-token query of short chunks (draft verification,
// a few tokens per sequence) on the 5th-generation tensor cores, with the
// key tokens on the M dimension.
//
// Same operation as prefill_kernel.cu ("vLLM推理引擎架构：PagedAttention机制
// 与高吞吐推理" §2.3 with a query of several trailing tokens per sequence and
// the causal rule). The row-major tcgen05 kernel puts (query token, head)
// rows on M = 128; a chunk of 8 tokens for a group of 8 heads fills only 64
// of them, so half of every S, softmax and P V step is empty. Here the roles
// turn: a CTA owns one (sequence, kv-head, part of the key range), its R <= 64
// query rows (row r = token r / G, head r % G) are the N = 64 columns, and a
// tile of 128 key tokens, as TMA lands it (16-row boxes of one 128-byte
// segment, 128-byte swizzle, [segment][128 rows][128 B]), is at once
//   * the K-major A operand of  S^T[t][r] = sum_d K[t][d] Q[r][d]   (M = 128
//     tokens, K = head_dim 128, B = Q rows K-major), and
//   * the MN-major A operand of O^T[d][r] += sum_t V[t][d] P[r][t]  (M = 128
//     dims, K = 128 tokens, B = P^T MN-major: one 128-byte row of 64 16-bit
//     probabilities per token, 128-byte swizzled),
// on tcgen05.mma kind::f16. A bf16 P is stored as hi + lo parts (two P V
// products into the same accumulator), an f16 P as is.
// Warps, as in the E4M3 decode kernel (decode_fp8_tc.cu):
//  * four softmax warps: thread i owns tensor-memory lane i, i.e. key token i
//    of the tile in S^T and dimension i of O^T. Per tile: its S^T row (64
//    logits), the causal mask (row r sees tokens up to its position
//    ctx - q_len + r / G), then a CTA-wide vote whether any logit passes its
//    row's running maximum by more than 8 (base 2). Only then (the first tile,
//    and rarely after) the warps exchange their exact row maxima, the maxima
//    move, and O^T is rescaled in tensor memory. The exchanges go through
//    mbarriers with bounded waits. Each thread keeps its own partial sums,
//    added across the CTA at the end;
//  * the MMA warp (one thread, owns the tensor memory: two 64-column S^T
//    buffers, 64 columns of O^T) issues S^T of tile k+1 before O^T += V^T P^T
//    of tile k;
//  * the TMA warp (one thread) loads K and V tiles into 2-stage rings through
//    the block table.
// One CTA per SM (176 KB of shared memory): with few (sequence, kv-head)
// pairs the key range is cut into parts of whole tiles, merged by the
// multi-token combine kernel. Every wait is bounded by wall time; a wait that
// gives up records the failure, the roles drain their loads and MMAs before
// the tensor memory is freed, and the rows are left as zeros (or an empty
// part).
#include <math_constants.h>

#include <type_traits>

#include "consumer_mma.cuh"
#include "decode_args.h"
#include "decode_kernel.cuh"
#include "device_common.cuh"
#include "prefill_args.h"
#include "tc_common.cuh"

namespace paged {
namespace {

constexpr int kTok = 128;                 // key tokens per tile (M of S^T)
constexpr int kN = 64;                    // query rows per CTA (N of both products)
constexpr int kStages = 2;
constexpr int kSeg = kTok * 128;          // one 64-dim segment of a tile: 128 rows x 128 B
constexpr int kTile = 2 * kSeg;           // head_dim 128, 16-bit
constexpr int kSoftmaxWarps = 4, kMmaWarp = 4, kTmaWarp = 5, kThreads = 192;
constexpr uint32_t kTmemCols = 256;       // S^T x 2 (columns 0, 64), O^T (128)
constexpr uint32_t kColO = 128;
constexpr int kOffV = kStages * kTile;
constexpr int kOffQ = 2 * kStages * kTile;
constexpr int kQSeg = kN * 128;           // one segment of Q: 64 rows x 128 B
constexpr int kOffP = kOffQ + 2 * kQSeg;  // P^T hi, then lo: [128 tokens][128 B] each
constexpr int kPPart = kTok * 128;
constexpr int kSmem = kOffP + 2 * kPPart;
constexpr float kLazy = 8.f;
static_assert(kSmem + 1024 <= 227 * 1024, "shared memory of one CTA");

// Byte offset of 16-byte chunk c of row r of a 128-byte-swizzled [rows][128 B] tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ int ord_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float float_of(int i) {
  return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF);
}

// NR: query rows the softmax handles (a multiple of 8, >= rows of the launch).
template <class QF, int NR>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_tm_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap, int G) {
  static_assert(NR % 8 == 0 && NR <= kN, "query rows");
  constexpr bool BF = std::is_same<QF, BF16>::value;
  constexpr int TR = kTileRows;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sq = smem + kOffQ;
  uint8_t* sp = smem + kOffP;
  auto sk = [&](int k) { return smem + (k % kStages) * kTile; };
  auto sv = [&](int k) { return smem + kOffV + (k % kStages) * kTile; };
  // kfull/vfull, kempty/vempty: the K / V rings; s_full[b] / s_free[b]: S^T
  // buffer b computed / read; p_full: P^T of a tile written (and O rescaled);
  // p_free: O += P V of the tile done (P^T has one buffer); vote_bar[b],
  // max_bar[b]: the four warps posted their votes / row maxima; sum_bar:
  // their partial sums.
  __shared__ uint64_t kfull[kStages], kempty[kStages], vfull[kStages], vempty[kStages],
      s_full[2], s_free[2], p_full, p_free, vote_bar[2], max_bar[2], sum_bar, drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int aborted;
  __shared__ int vote[2][kSoftmaxWarps];
  __shared__ float4 red[2][NR][1];           // per row: the four warps' maxima
  __shared__ float lsum[kSoftmaxWarps][NR];

  const int part = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
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
      mbar_init(&vote_bar[b], kSoftmaxWarps);
      mbar_init(&max_bar[b], kSoftmaxWarps);
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
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int q0 = a.cu_query_lens[s];
  const int qlen = a.cu_query_lens[s + 1] - q0;
  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (tid == 0 && part == 0 && kvh == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  if (qlen <= 0) return;
  const int rows = qlen * G;   // <= NR (the launch checks max_query_len * G)
  if (qlen > ctx) {            // a query longer than its context: rows become zeros
    if (part > 0) return;
    if (tid == 0 && kvh == 0) report(a.err, kErrQueryLonger);
    for (int i = tid; i < rows * 16; i += kThreads) {
      const int r = i / 16, c = i % 16;
      reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.out) +
                               ((static_cast<int64_t>(q0 + r / G) * a.num_heads + kvh * G +
                                 r % G) * 128) * 2)[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }
  // 16-token tiles up to the last query row's position, cut into parts of
  // partition_tiles (a multiple of 8); this CTA takes part `part`
  const int ntiles16 = (ctx - 1) / TR + 1;
  const int parts = (ntiles16 + a.partition_tiles - 1) / a.partition_tiles;
  if (part >= parts) return;
  const int t16 = part * a.partition_tiles;
  const int tok_begin = t16 * TR;
  const int ntok = min(ctx, min(ntiles16, t16 + a.partition_tiles) * TR) - tok_begin;
  const int ntiles = (ntok + kTok - 1) / kTok;
  const int pos0 = ctx - qlen;  // position of query token 0

  // Q rows -> shared memory ([segment][64 rows][128 B], swizzled), zeros past the chunk
  if (warp < kSoftmaxWarps) {
    const int r = tid >> 1, sg = tid & 1;
    const uint4* q4 = reinterpret_cast<const uint4*>(
        static_cast<const uint8_t*>(a.query) +
        ((static_cast<int64_t>(q0 + r / G) * a.num_heads + kvh * G + r % G) * 128 + sg * 64) *
            2);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = r < rows ? q4[c] : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(sq + sg * kQSeg + sw128(r, c)) = v;
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (warp == kMmaWarp) tc::alloc(&tmem_slot, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp == kTmaWarp) {
    // ================= TMA loads (one thread) =================
    if (lane == 0) {
      const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
      const uint64_t policy = l2_policy_evict_first();
      int32_t bid[kTok / TR];
      auto load_ids = [&](int k) {
#pragma unroll
        for (int j = 0; j < kTok / TR; ++j) {
          const int u = k * kTok + j * TR;
          bid[j] = u < ntok ? table[(tok_begin + u) / a.block_size] : 0;
        }
      };
      auto issue = [&](int k, bool is_v) {
        uint8_t* dst = is_v ? sv(k) : sk(k);
        uint64_t* bar = is_v ? &vfull[k % kStages] : &kfull[k % kStages];
        const CUtensorMap* map = is_v ? &vmap : &kmap;
        const int u0 = k * kTok;
        const int nsub = (min(kTok, ntok - u0) + TR - 1) / TR;
        if (!is_v && a.skip_tile >= u0 / TR && a.skip_tile < u0 / TR + nsub &&
            skip_for_test(a.skip_tile, a.skip_tile))
          return;
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nsub * 2 * TR * 128));
        for (int j = 0; j < nsub; ++j) {
          int32_t b = bid[j];
          if (b < 0 || b >= a.num_blocks) {
            if (!is_v) report(a.err, kErrBadBlockId);
            b = -1;  // read as a box outside the pool: zero-filled
          }
          const int32_t row0 = b >= 0 ? b * a.block_size + (tok_begin + u0 + j * TR) % a.block_size
                                      : -TR;
#pragma unroll
          for (int sg = 0; sg < 2; ++sg)
            tma_load_4d(dst + sg * kSeg + j * TR * 128, map, bar, 0, row0, kvh, sg, policy);
        }
      };
      bool ok = true;
      int k_issued = 0, v_issued = 0, k = 0;
      for (; ok && k < ntiles; ++k) {
        load_ids(k);
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
        record_failure(a.diag, kSiteTmTile, blockIdx.x, blockIdx.y, blockIdx.z, 0, k, ntiles,
                       0);
        aborted = 1;
        report(a.err, kErrWaitTimeout);
      }
      for (int j = max(0, k_issued - kStages); j < k_issued; ++j)
        mbar_wait(&kfull[j % kStages], (j / kStages) & 1, lim);
      for (int j = max(0, v_issued - kStages); j < v_issued; ++j)
        mbar_wait(&vfull[j % kStages], (j / kStages) & 1, lim);
    }
    __syncwarp();  // whole warps reach the CTA barrier below
  } else if (warp == kMmaWarp) {
    // ================= MMA issue (one thread) =================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = tc::idesc_f16_ab<BF, kTok, kN, false, false>();
      constexpr uint32_t IDESC_O = tc::idesc_f16_ab<BF, kTok, kN, true, true>();
      const uint64_t qd = tc::sw128_desc(sq, 16, 1024);
      const uint64_t kd0 = tc::sw128_desc(smem, 16, 1024);
      const uint64_t vd0 = tc::sw128_desc(smem + kOffV, kSeg, 1024);
      const uint64_t pd = tc::sw128_desc(sp, kPPart, 1024);
      int k = 0;
      auto issue_s = [&](int t) {  // S^T of tile t into buffer t & 1
        if (t >= 2 && !mbar_wait(&s_free[t & 1], ((t - 2) >> 1) & 1, lim, &aborted)) return false;
        if (!mbar_wait(&kfull[t % kStages], (t / kStages) & 1, lim, &aborted)) return false;
        tc::fence_after_sync();
        const uint64_t kd = kd0 + static_cast<uint64_t>(((t % kStages) * kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 dims per K step: segment kk / 4
          const int off = (kk / 4) * kSeg + (kk % 4) * 32, qoff = (kk / 4) * kQSeg + (kk % 4) * 32;
          tc::mma_f16(tmem + (t & 1) * kN, kd + static_cast<uint64_t>(off >> 4),
                      qd + static_cast<uint64_t>(qoff >> 4), IDESC_S, kk > 0);
        }
        tc::commit(&s_full[t & 1]);
        tc::commit(&kempty[t % kStages]);
        return true;
      };
      bool ok = ntiles == 0 || issue_s(0);
      for (; ok && k < ntiles; ++k) {
        if (k + 1 < ntiles) ok = issue_s(k + 1);
        if (!ok) break;
        ok = mbar_wait(&vfull[k % kStages], (k / kStages) & 1, lim, &aborted) &&
             mbar_wait(&p_full, k & 1, lim, &aborted);
        if (!ok) break;
        tc::fence_after_sync();
        const uint64_t vd = vd0 + static_cast<uint64_t>(((k % kStages) * kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk) {  // 16 tokens per K step
          const uint64_t off = static_cast<uint64_t>((kk * 16 * 128) >> 4);
          tc::mma_f16(tmem + kColO, vd + off, pd + off, IDESC_O, k > 0 || kk > 0);
          if constexpr (BF)
            tc::mma_f16(tmem + kColO, vd + off, pd + static_cast<uint64_t>(kPPart >> 4) + off,
                        IDESC_O, true);
        }
        tc::commit(&p_free);
        tc::commit(&vempty[k % kStages]);
      }
      if (!ok) {
        record_failure(a.diag, kSiteTmTile, blockIdx.x, blockIdx.y, blockIdx.z, 1, k, ntiles,
                       0);
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
    const float qs = a.scale_log2;
    float m[NR], l[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      m[r] = -CUDART_INF_F;
      l[r] = 0.f;
    }
    bool ok = true;
    int k = 0, nmax = 0;  // tiles done, exact-maximum exchanges done
    for (; ok && k < ntiles; ++k) {
      ok = __all_sync(FULL, mbar_wait(&s_full[k & 1], (k >> 1) & 1, lim, &aborted));
      if (!ok) break;
      tc::fence_after_sync();
      float x[kN];
      tc::ld64(tmem + (k & 1) * kN + lane_base, x);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[k & 1]);
      // logits (base 2) with the causal mask: row r sees key positions <= pos0 + r / G
      const int tp = tok_begin + k * kTok + tid;   // this thread's key position
      const bool live = tp < tok_begin + ntok;
      bool need = false;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const bool vis = live && r < rows && tp <= pos0 + r / G;
        x[r] = vis ? x[r] * qs : -CUDART_INF_F;
        need |= x[r] > m[r] + kLazy;
      }
      // does any logit of the CTA pass its row's maximum by more than the margin?
      const bool wneed = __any_sync(FULL, need);
      if (lane == 0) vote[k & 1][warp] = wneed ? 1 : 0;
      __syncwarp();
      if (lane == 0) mbar_arrive(&vote_bar[k & 1]);
      ok = __all_sync(FULL, mbar_wait(&vote_bar[k & 1], (k >> 1) & 1, lim, &aborted));
      if (!ok) break;
      const bool any = (vote[k & 1][0] | vote[k & 1][1] | vote[k & 1][2] | vote[k & 1][3]) != 0;
      if (any) {  // the exact row maxima (the first tile; rare afterwards)
        const int b = nmax & 1;
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          const float wm = float_of(__reduce_max_sync(FULL, ord_of(x[r])));
          if (lane == (r & 31)) reinterpret_cast<float*>(&red[b][r][0])[warp] = wm;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&max_bar[b]);
        ok = __all_sync(FULL, mbar_wait(&max_bar[b], (nmax >> 1) & 1, lim, &aborted));
        if (!ok) break;
        ++nmax;
        // O^T may be rescaled only once O += P V of tile k-1 completed
        if (k >= 1) {
          ok = __all_sync(FULL, mbar_wait(&p_free, (k - 1) & 1, lim, &aborted));
          if (!ok) break;
          tc::fence_after_sync();
        }
#pragma unroll
        for (int c = 0; c < (NR + 31) / 32; ++c) {
          float o[32];
          if (k >= 1) tc::ld32(tmem + kColO + c * 32 + lane_base, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int r = c * 32 + i;
            if (r >= NR) break;
            const float4 w4 = red[b][r][0];
            const float tmax = fmaxf(fmaxf(w4.x, w4.y), fmaxf(w4.z, w4.w));
            if (tmax > m[r] + kLazy) {  // false while the row has seen nothing
              const float alpha = tc::ex2(m[r] - tmax);
              m[r] = tmax;
              l[r] *= alpha;
              o[i] *= alpha;
            }
          }
          if (k >= 1) tc::st32(tmem + kColO + c * 32 + lane_base, o);
        }
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const float mu = m[r] == -CUDART_INF_F ? 0.f : m[r];
        x[r] = tc::ex2(x[r] - mu);
        l[r] += x[r];
      }
      // P^T has one buffer: O += P V of tile k-1 must be done before it is rewritten
      if (k >= 1) {
        ok = __all_sync(FULL, mbar_wait(&p_free, (k - 1) & 1, lim, &aborted));
        if (!ok) break;
      }
      // this token's row of P^T: 64 probabilities (hi, and for bf16 the lo part)
#pragma unroll
      for (int c = 0; c < kN / 8; ++c) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = c * 8 + 2 * j;
          const float p0 = r < NR ? x[r] : 0.f, p1 = r + 1 < NR ? x[r + 1] : 0.f;
          hw[j] = pack2<BF>(p0, p1);
          if constexpr (BF)
            lw[j] = pack2<true>(p0 - __uint_as_float(hw[j] << 16),
                                p1 - __uint_as_float(hw[j] & 0xffff0000u));
        }
        *reinterpret_cast<uint4*>(sp + sw128(tid, c)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        if constexpr (BF)
          *reinterpret_cast<uint4*>(sp + kPPart + sw128(tid, c)) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      // V rows without key tokens (end of the range) may hold anything, even
      // NaN; 0 * NaN is NaN inside the MMA: clear them once the loads landed
      if (ntok - k * kTok < kTok) {
        ok = __all_sync(FULL, mbar_wait(&vfull[k % kStages], (k / kStages) & 1, lim, &aborted));
        if (!ok) break;
        if (!live) {
#pragma unroll
          for (int sg = 0; sg < 2; ++sg) {
            uint4* row = reinterpret_cast<uint4*>(sv(k) + sg * kSeg + tid * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) row[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full);
    }
    if (ok && ntiles > 0)
      ok = __all_sync(FULL, mbar_wait(&p_free, (ntiles - 1) & 1, lim, &aborted));
    if (!ok && lane == 0) {
      record_failure(a.diag, kSiteTmTile, blockIdx.x, blockIdx.y, blockIdx.z, 2, k, ntiles, 0);
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    // the partial sums over the CTA
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      float v = l[r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
      if (lane == (r & 31)) lsum[warp][r] = v;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sum_bar);
    const bool sums = __all_sync(FULL, mbar_wait(&sum_bar, 0, lim, &aborted));
    if (!sums && lane == 0) {
      record_failure(a.diag, kSiteTmTile, blockIdx.x, blockIdx.y, blockIdx.z, 3, k, ntiles, 0);
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    __syncwarp();
    ok = __all_sync(FULL, ok && sums && *static_cast<volatile int*>(&aborted) == 0);
    // ---- epilogue: thread i holds dimension i of every row's O
    const bool single = parts == 1;
    float o[kN];
    if (ok && ntiles > 0) {
      tc::fence_after_sync();
      tc::ld64(tmem + kColO + lane_base, o);
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      if (r >= rows) break;
      const int64_t row = static_cast<int64_t>(q0 + r / G) * a.num_heads + kvh * G + r % G;
      const float L = lsum[0][r] + lsum[1][r] + lsum[2][r] + lsum[3][r];
      const float val = ok && L > 0.f && ntiles > 0 ? o[r] / L : 0.f;
      if (single) {
        store_out(QF{}, a.out, row * 128 + tid, val);
      } else {
        const int64_t pi = row * a.max_parts + part;
        a.ws_o[pi * 128 + tid] = val;
        if (tid == 0) a.ws_ml[pi] = ok ? make_float2(m[r], L) : make_float2(-CUDART_INF_F, 0.f);
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

template <class QF, int NR>
cudaError_t launch_one(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       int group, int32_t max_query_len, cudaStream_t stream) {
  const size_t smem = 1024 + kSmem;
  auto kern = paged_prefill_tm_kernel<QF, NR>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(static_cast<unsigned>(a.max_parts), a.num_kv_heads, a.num_seqs),
                 kThreads, smem, stream, a, kmap, vmap, group);
  if (e != cudaSuccess || a.max_parts <= 1) return e;
  // every CTA took the whole chunk: query tiles of kN / group tokens
  return launch_prefill_combine(a, std::is_same<QF, BF16>::value ? kBF16 : kF16, 128,
                                kN / group, max_query_len, stream);
}

}  // namespace

cudaError_t launch_prefill_tm(const PrefillArgs& a, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int q_dtype, int head_dim, int group,
                              int32_t max_query_len, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(max_query_len) * group;
  if (head_dim != 128 || rows > kN || rows < 1 || a.partition_tiles % (kTok / kTileRows) != 0)
    return cudaErrorNotSupported;
#define PAGED_TM(QF)                                                                      \
  if (rows <= 16) return launch_one<QF, 16>(a, kmap, vmap, group, max_query_len, stream); \
  if (rows <= 32) return launch_one<QF, 32>(a, kmap, vmap, group, max_query_len, stream); \
  return launch_one<QF, 64>(a, kmap, vmap, group, max_query_len, stream);
  if (q_dtype == kF16) {
    PAGED_TM(F16)
  }
  if (q_dtype == kBF16) {
    PAGED_TM(BF16)
  }
#undef PAGED_TM
  return cudaErrorNotSupported;
}

}  // namespace paged
