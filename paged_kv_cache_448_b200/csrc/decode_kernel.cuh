// decode_kernel.cuh — the paged decode kernel: block-table walk, TMA staging
// of K/V tiles through per-warp shared-memory rings, merge of the per-warp
// online-softmax states, and the combine of context partitions. The
// arithmetic on a staged tile is done by a Consumer (consumer_simt.cuh:
// fp32 CUDA cores; consumer_mma.cuh: tensor cores for query groups).
//
// Follows "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.3 (PagedAttention
// Kernel): for each sequence, find the physical K/V block of each logical
// block through block_tables, compute the attention scores inside the block
// and accumulate across blocks. The logical->physical translation of
// "vLLM框架中的KV cache优化与PagedAttention机制详解" §5.1 is done once per block
// for a whole work unit (a warp reads 32 table entries per coalesced load,
// the page's "批量转换"), and tiles are requested well ahead of use (the
// page's "预取机制", §5.2: R tiles per warp in flight through TMA).
//
// Organisation (persistent CTAs, warp-specialised):
//  * scheduler warp: draws work units (sequence, kv-head, context partition)
//    from a device counter in the order the plan kernel laid out (longest
//    sequences first) and publishes each in a unit slot: its description, its
//    block ids, and a bulk copy of its query rows. It works up to US units
//    ahead, so no consumer ever waits on this bookkeeping.
//  * NC consumer warps: tile k of a unit (16 tokens; a 32-token block is two
//    tiles) belongs to warp (rot + k) mod NC. Each warp issues the TMA loads of
//    its own tiles into its own R-deep ring (one box per K tile and per V
//    tile, swizzled) — its issue cursor runs ahead into the next units while
//    its consume cursor finishes the current one — and keeps one
//    online-softmax state per unit. At the end of a unit all consumer warps
//    merge their states through shared memory, write the output row (or a
//    partial result, below) and free the unit slot.
// Every wait is bounded; a wait that gives up makes the CTA stop and report.
//
// A sequence cut into several partitions leaves one partial (m, l, o) per
// partition; the CTA that writes the last one (atomic arrival count, no
// waiting) combines them: M = max m_p, out = sum l_p 2^(m_p-M) o_p / sum l_p 2^(m_p-M).
#pragma once

#include <math_constants.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "decode_args.h"
#include "device_common.cuh"

namespace paged {

constexpr int kTileRows = 16;           // tokens per pipeline tile
constexpr int kMaxSliceEntries = 1025;  // partition slices + 1 (at most 1024 partitions)
constexpr int kMaxUnitBlocks = 1024;    // blocks of one work unit (partition_blocks bound)

#ifndef PAGED_CONSUMER_WARPS
#define PAGED_CONSUMER_WARPS 8
#endif
#ifndef PAGED_CTAS_PER_SM
#define PAGED_CTAS_PER_SM 1
#endif
#ifndef PAGED_UNIT_SLOTS
#define PAGED_UNIT_SLOTS 4
#endif

// Shared-memory geometry of one staged K (or V) tile: kTileRows token rows of
// one kv-head, RB bytes each, stored back to back; the TMA swizzles the 16-byte
// chunks inside every BOXB-byte segment (128B or 64B pattern).
template <class CF, int D_>
struct Tile {
  static constexpr int D = D_, BS = kTileRows;
  static constexpr int EB = CF::kBytes;
  static constexpr int RB = D * EB;                          // bytes per token row
  static constexpr int BOXB = box_bytes(RB);                 // bytes per box row segment
  static constexpr int NBOX = RB / BOXB;                     // segments per row
  static constexpr int SWZ = BOXB == 128 ? 0x70 : (BOXB == 64 ? 0x30 : 0);
  static constexpr int BYTES = BS * RB;
  // Byte offset of logical byte `o` of row `r`.
  static __device__ __forceinline__ uint32_t off(int r, int o) {
    const int lin = r * RB + o;
    return lin ^ ((lin >> 3) & SWZ);
  }
};

// Shared-memory plan of the kernel for one consumer type.
template <class Consumer>
struct Layout {
  using T = typename Consumer::Tile;
  static constexpr int G = Consumer::G, D = T::D;
  static constexpr int NC = PAGED_CONSUMER_WARPS;            // consumer warps
  static constexpr int CTAS = PAGED_CTAS_PER_SM;             // resident CTAs per SM
  static constexpr int THREADS = (NC + 1) * 32;              // + the scheduler warp
  static constexpr int US = PAGED_UNIT_SLOTS;                // unit slots
  static constexpr int STAGE = 2 * T::BYTES;                 // K and V tiles
  static constexpr int QBYTES = G * D * 2;                   // the unit's query rows
  static constexpr int SLOT = 64 + QBYTES + 4 * kMaxUnitBlocks;  // description, query, ids
  static constexpr int MERGE = NC * G * (D + 2) * 4;         // per-warp (m, l, acc)
  // per-CTA share of the SM's 228 KB (1 KB of each CTA's share is reserved)
  static constexpr int SMEM_MAX = CTAS == 1 ? 227 * 1024 : (228 / CTAS - 1) * 1024;
  static constexpr int FIXED = 1024 /*alignment*/ + MERGE + 16 + US * SLOT + 16 * US +
                               8 * G + 16 + 4 * kMaxSliceEntries;
  static constexpr int R_RAW = (SMEM_MAX - FIXED) / (NC * (STAGE + 8));
  static_assert(R_RAW >= 1, "no room for a ring stage per warp");
  static constexpr int R = R_RAW > 8 ? 8 : R_RAW;            // stages per warp
  // byte offsets from the 1024-aligned base
  static constexpr int OFF_MERGE = NC * R * STAGE;
  static constexpr int OFF_SLOTS = (OFF_MERGE + MERGE + 15) & ~15;
  static constexpr int OFF_BARS = OFF_SLOTS + US * SLOT;
  static constexpr int OFF_COMB = OFF_BARS + 8 * (NC * R + 2 * US);
  static constexpr int OFF_FLAG = OFF_COMB + 8 * G;
  static constexpr int OFF_SLICE = OFF_FLAG + 16;
  static constexpr int BYTES = 1024 + OFF_SLICE + 4 * kMaxSliceEntries;
  static_assert(BYTES <= SMEM_MAX, "shared memory plan");
};

// Unit slot description words.
enum : int { kUSeq = 0, kUKvh, kUPart, kUCtx, kUTiles, kURot, kUParts, kUTok0 };

__device__ __forceinline__ void consumer_sync(int threads) {
  asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}

template <class Consumer>
__global__ void __launch_bounds__(Layout<Consumer>::THREADS, Layout<Consumer>::CTAS)
    paged_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap) {
  using L = Layout<Consumer>;
  using T = typename Consumer::Tile;
  constexpr int D = T::D, G = Consumer::G, NC = L::NC, R = L::R, US = L::US;
  constexpr int STAGE = L::STAGE, TR = kTileRows;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* mbuf = reinterpret_cast<float*>(smem + L::OFF_MERGE);     // [NC][G][2]: m, l
  float* obuf = mbuf + NC * G * 2;                                 // [NC][G][D]: acc
  uint8_t* slots = smem + L::OFF_SLOTS;                            // [US][SLOT]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BARS);  // [NC][R]
  uint64_t* ufull = full + NC * R;
  uint64_t* uempty = ufull + US;
  float2* comb = reinterpret_cast<float2*>(smem + L::OFF_COMB);   // [G]: (M, 1/L)
  volatile int* flag = reinterpret_cast<int*>(smem + L::OFF_FLAG); // [0] abort, [1] last
  int* slice = reinterpret_cast<int*>(smem + L::OFF_SLICE);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NC * R; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < US; ++i) {
      mbar_init(&ufull[i], 1);
      mbar_init(&uempty[i], 1);
    }
    fence_mbar_init();
    flag[0] = 0;
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  // Everything below reads data of earlier kernels in the stream (the plan,
  // and through it the cache scatter): wait for them here.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i <= a.max_parts; i += L::THREADS) slice[i] = a.slice_start[i];
  const int total = a.counters[kCounterTotal];
  const int tpb = a.block_size / TR;  // tiles per block
  __syncthreads();

  if (warp == NC) {
    // ----------------------------------------------------------- scheduler
    uint32_t rot = 0;  // tiles published so far: rotates the first warp of each unit
    int next = lane == 0 ? atomicAdd(&a.counters[kCounterWork], 1) : 0;
    next = __shfl_sync(FULL, next, 0);
    for (uint32_t uc = 0;; ++uc) {
      const int u = next;
      const int us = uc % US;
      uint8_t* slot = slots + us * L::SLOT;
      int* info = reinterpret_cast<int*>(slot);
      int32_t* sids = reinterpret_cast<int32_t*>(slot + 64 + L::QBYTES);
      // (the scheduler only reads the abort flag; if one of its waits gives up
      // it stops, and the consumers' own bounded waits end the CTA)
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&uempty[us], ((uc / US) & 1) ^ 1, flag);
        if (!ok) record_failure(a.diag, kSiteSlotFree, blockIdx.x, static_cast<int>(uc), u, 0, 0, 0, 0);
      }
      if (!__shfl_sync(FULL, ok, 0)) break;
      if (u >= total) {
        if (lane == 0) {
          info[kUSeq] = -1;  // no more work
          mbar_arrive(&ufull[us]);
        }
        break;
      }
      int s = 0, nblk = 0, part = 0, kvh = 0;
      if (lane == 0) {
        int lo = 0, hi = a.max_parts - 1;  // partition slice: largest p with slice[p] <= u
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (slice[mid] <= u) lo = mid; else hi = mid - 1;
        }
        const int idx = u - slice[lo];
        const int j = idx / a.num_kv_heads;
        int2 e = make_int2(-1, 0);
        if (j < a.num_seqs) e = a.order[j];
        s = e.x;
        nblk = e.y;
        part = lo;
        kvh = idx % a.num_kv_heads;
        // self-check of the plan: a ticket must decode to a real unit
        const int parts_s = nblk == 0 ? 1 : (nblk + a.partition_blocks - 1) / a.partition_blocks;
        if (j >= a.num_seqs || s < 0 || s >= a.num_seqs || nblk < 0 ||
            nblk > a.max_blocks_per_seq || part >= parts_s) {
          record_failure(a.diag, kSiteBadUnit, blockIdx.x, u, total, j, s, nblk, part);
          report(a.err, kErrBadPlan);
          s = -1;
        }
        next = atomicAdd(&a.counters[kCounterWork], 1);  // fetched early, used next round
      }
      s = __shfl_sync(FULL, s, 0);
      if (s < 0) {  // stop this CTA's work: publish the end marker
        if (lane == 0) {
          info[kUSeq] = -1;
          mbar_arrive(&ufull[us]);
        }
        break;
      }
      nblk = __shfl_sync(FULL, nblk, 0);
      part = __shfl_sync(FULL, part, 0);
      kvh = __shfl_sync(FULL, kvh, 0);
      const int ctx = min(max(a.context_lens[s], 0), a.ctx_limit);
      const int parts = nblk == 0 ? 1 : (nblk + a.partition_blocks - 1) / a.partition_blocks;
      const int b_begin = part * a.partition_blocks;
      const int nlocal = min(b_begin + a.partition_blocks, nblk) - b_begin;
      const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
      for (int k = lane; k < nlocal; k += 32) {
        int32_t id = table[b_begin + k];
        if (id < 0 || id >= a.num_blocks) {
          report(a.err, kErrBadBlockId);
          id = -1;  // read as a box outside the pool: zero-filled
        }
        sids[k] = id;
      }
      // tiles holding at least one context token (a 32-token block whose
      // context ends in its first half contributes one tile, not two)
      const int tok0 = b_begin * a.block_size;
      const int ntiles = (min(ctx, (b_begin + nlocal) * a.block_size) - tok0 + TR - 1) / TR;
      if (lane == 0) {
        info[kUSeq] = s;
        info[kUKvh] = kvh;
        info[kUPart] = part;
        info[kUCtx] = ctx;
        info[kUTiles] = max(ntiles, 0);
        info[kURot] = static_cast<int>(rot % NC);
        info[kUParts] = parts;
        info[kUTok0] = tok0;
      }
      rot += max(ntiles, 0);
      __syncwarp();  // the ids and the description precede the slot's release
      if (lane == 0) {
        const uint8_t* qsrc = static_cast<const uint8_t*>(a.query) +
                              (static_cast<int64_t>(s) * a.num_heads + kvh * G) * D * 2;
        mbar_arrive_expect_tx(&ufull[us], L::QBYTES);
        bulk_load(slot + 64, qsrc, L::QBYTES, &ufull[us]);
      }
      next = __shfl_sync(FULL, next, 0);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // Every consumer warp reaches every consumer barrier: a failed wait only
  // sets the abort flag (written by consumers before barrier A, read after it),
  // and the decision to stop is taken by all warps together after barrier A.
  constexpr int CT = NC * 32;
  uint8_t* my_ring = smem + warp * R * STAGE;
  uint64_t* my_full = full + warp * R;
  const uint64_t policy = l2_policy_evict_first();
  uint32_t issued = 0, consumed = 0;       // tiles of this warp's ring
  uint32_t cunit = 0;                      // unit being consumed
  uint32_t iunit = 0;                      // unit the issue cursor is in
  int ik = -1, i_tiles = 0, i_kvh = 0;     // issue cursor: next tile (-1: unit not entered)
  const int32_t* i_ids = nullptr;
  bool no_more = false;

  // Keep up to R of this warp's tiles in flight; the cursor may run into the
  // next units, but not so far that their slots are still owned by a unit
  // this warp has not finished (those are published only after it is).
  auto issue_more = [&]() {
    while (!no_more && issued - consumed < static_cast<uint32_t>(R)) {
      if (ik < 0) {
        if (iunit >= cunit + US) break;
        if (!__all_sync(FULL, mbar_wait(&ufull[iunit % US], (iunit / US) & 1, flag))) {
          if (lane == 0) {
            flag[0] = 1;
            record_failure(a.diag, kSiteUnitAhead, blockIdx.x, warp, static_cast<int>(cunit),
                           static_cast<int>(iunit), static_cast<int>(issued),
                           static_cast<int>(consumed), 0);
          }
          no_more = true;
          break;
        }
        const uint8_t* slot = slots + (iunit % US) * L::SLOT;
        const int* inf = reinterpret_cast<const int*>(slot);
        if (inf[kUSeq] < 0) {
          no_more = true;
          break;
        }
        i_tiles = inf[kUTiles];
        i_kvh = inf[kUKvh];
        i_ids = reinterpret_cast<const int32_t*>(slot + 64 + L::QBYTES);
        ik = (warp - inf[kURot] + NC) % NC;
      }
      if (ik >= i_tiles) {
        ++iunit;
        ik = -1;
        continue;
      }
      if (lane == 0) {
        const uint32_t st = issued % R;
        const int32_t bid = i_ids[ik / tpb];
        const int32_t row0 = bid >= 0 ? bid * a.block_size + (ik % tpb) * TR : -TR;
        uint8_t* kt = my_ring + st * STAGE;
        mbar_arrive_expect_tx(&my_full[st], STAGE);
        tma_load_4d(kt, &kmap, &my_full[st], 0, 0, i_kvh, row0, policy);
        tma_load_4d(kt + T::BYTES, &vmap, &my_full[st], 0, 0, i_kvh, row0, policy);
      }
      ++issued;
      ik += NC;
    }
  };

  for (;; ++cunit) {
    const int us = cunit % US;
    const uint8_t* slot = slots + us * L::SLOT;
    const int* info = reinterpret_cast<const int*>(slot);
    const bool have_unit = __all_sync(FULL, mbar_wait(&ufull[us], (cunit / US) & 1, flag));
    if (!have_unit && lane == 0) {
      flag[0] = 1;
      record_failure(a.diag, kSiteUnit, blockIdx.x, warp, static_cast<int>(cunit),
                     static_cast<int>(iunit), static_cast<int>(issued),
                     static_cast<int>(consumed), 0);
    }
    // The end marker carries only kUSeq: the other words of its slot are stale
    // shared memory and must not be used.
    const int s = have_unit ? info[kUSeq] : -1;
    const bool real = s >= 0;
    const int kvh = real ? info[kUKvh] : 0, part = real ? info[kUPart] : 0;
    const int ctx = real ? info[kUCtx] : 0, ntiles = real ? info[kUTiles] : 0;
    const int rot = real ? info[kURot] : 0, parts = real ? info[kUParts] : 1;
    const int tok0 = real ? info[kUTok0] : 0;

    Consumer c;
    if (s >= 0) c.init(a, slot + 64, kvh, lane);
    for (int k = (warp - rot + NC) % NC; k < ntiles; k += NC) {
      issue_more();
      const uint32_t st = consumed % R;
      if (!__all_sync(FULL, mbar_wait(&my_full[st], (consumed / R) & 1, flag))) {
        if (lane == 0) {
          flag[0] = 1;
          record_failure(a.diag, kSiteTile, blockIdx.x, warp, static_cast<int>(cunit), k,
                         static_cast<int>(issued), static_cast<int>(consumed), ntiles);
        }
        break;
      }
      uint8_t* kt = my_ring + st * STAGE;
      c.block(kt, kt + T::BYTES, max(0, min(TR, ctx - (tok0 + k * TR))), lane);
      __syncwarp();
      ++consumed;
    }
    // start the next unit's loads before merging (the flag read is made
    // warp-uniform: issue_more() synchronises the whole warp)
    if (s >= 0 && !__any_sync(FULL, flag[0] != 0)) issue_more();
    consumer_sync(CT);                     // barrier A
    if (flag[0] || s < 0) break;

    c.finish(mbuf + warp * G * 2, obuf + warp * G * D, lane);
    consumer_sync(CT);

    const bool single = parts == 1;
    const float vs = a.v_scale ? a.v_scale[kvh] : 1.f;
    const int64_t row0 = static_cast<int64_t>(s) * a.num_heads + kvh * G;
    for (int idx = threadIdx.x; idx < G * D; idx += CT) {
      const int g = idx / D, d = idx % D;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < NC; ++w) M = fmaxf(M, mbuf[(w * G + g) * 2]);
      float Lsum = 0.f, o = 0.f;
#pragma unroll
      for (int w = 0; w < NC; ++w) {
        const float mw = mbuf[(w * G + g) * 2];
        const float f = mw == -CUDART_INF_F ? 0.f : exp2f(mw - M);
        Lsum += mbuf[(w * G + g) * 2 + 1] * f;
        o += obuf[(w * G + g) * D + d] * f;
      }
      o = Lsum > 0.f ? o / Lsum * vs : 0.f;
      if (single) {
        store_out(typename Consumer::QF{}, a.out, (row0 + g) * D + d, o);
      } else {
        const int64_t pi = (row0 + g) * a.max_parts + part;
        a.ws_o[pi * D + d] = o;
        if (d == 0) a.ws_ml[pi] = make_float2(M, Lsum);
      }
    }

    if (!single) {
      // The CTA that delivers the last partial of (s, kvh) combines them.
      consumer_sync(CT);
      if (threadIdx.x == 0) {
        __threadfence();
        const int prev = atomicAdd(&a.arrive[s * a.num_kv_heads + kvh], 1);
        flag[1] = prev == parts - 1;
      }
      consumer_sync(CT);
      if (flag[1]) {
        __threadfence();
        for (int g = warp; g < G; g += NC) {
          const float2* ml = a.ws_ml + (row0 + g) * a.max_parts;
          float M = -CUDART_INF_F;
          for (int q = lane; q < parts; q += 32) M = fmaxf(M, __ldcg(ml + q).x);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, o));
          float Lsum = 0.f;
          for (int q = lane; q < parts; q += 32) {
            const float2 v = __ldcg(ml + q);
            Lsum += v.x == -CUDART_INF_F ? 0.f : v.y * exp2f(v.x - M);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(FULL, Lsum, o);
          if (lane == 0) comb[g] = make_float2(M, Lsum > 0.f ? 1.f / Lsum : 0.f);
        }
        consumer_sync(CT);
        for (int idx = threadIdx.x; idx < G * D; idx += CT) {
          const int g = idx / D, d = idx % D;
          const float2* ml = a.ws_ml + (row0 + g) * a.max_parts;
          const float* op = a.ws_o + (row0 + g) * a.max_parts * D + d;
          const float M = comb[g].x;
          float acc = 0.f;
          for (int q = 0; q < parts; ++q) {
            const float2 v = __ldcg(ml + q);
            const float w = v.x == -CUDART_INF_F ? 0.f : v.y * exp2f(v.x - M);
            acc = fmaf(w, __ldcg(op + static_cast<int64_t>(q) * D), acc);
          }
          store_out(typename Consumer::QF{}, a.out, (row0 + g) * D + d, acc * comb[g].y);
        }
      }
    }
    consumer_sync(CT);  // merge buffers are reused by the next unit
    if (threadIdx.x == 0) mbar_arrive(&uempty[us]);
  }
  if (flag[0]) {
    // A wait gave up (never expected): let this warp's loads still in flight
    // land (bounded again) before the CTA's shared memory goes away.
    for (; consumed < issued; ++consumed) mbar_wait(&my_full[consumed % R], (consumed / R) & 1);
    if (threadIdx.x == 0) report(a.err, kErrWaitTimeout);
  }
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
inline cudaError_t configure_kernel(const void* kern, size_t smem) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> configured;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (std::find(configured.begin(), configured.end(), std::make_pair(kern, dev)) !=
      configured.end())
    return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e == cudaSuccess) configured.emplace_back(kern, dev);
  return e;
}

template <class Consumer>
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          cudaStream_t stream) {
  using L = Layout<Consumer>;
  if (a.max_parts + 1 > kMaxSliceEntries || a.partition_blocks > kMaxUnitBlocks ||
      a.block_size % kTileRows != 0)
    return cudaErrorNotSupported;
  auto kern = paged_decode_kernel<Consumer>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), L::BYTES);
  if (e != cudaSuccess) return e;
  const int64_t upper = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads * a.max_parts;
  const int grid = static_cast<int>(std::min<int64_t>(upper, static_cast<int64_t>(a.num_sms) *
                                                                 L::CTAS));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(L::THREADS);
  cfg.dynamicSmemBytes = L::BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, kmap, vmap);
}

}  // namespace paged
