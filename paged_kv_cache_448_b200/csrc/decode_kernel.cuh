// decode_kernel.cuh — the paged decode kernel: block-table walk, TMA staging
// of K/V tiles through per-warp shared-memory rings, and the merge of the
// per-warp online-softmax states. The arithmetic on a staged tile is done by a
// Consumer (consumer_simt.cuh: fp32 CUDA cores; consumer_mma.cuh: tensor cores
// for query groups).
//
// Follows "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.3 (PagedAttention
// Kernel): for each sequence, find the physical K/V block of each logical
// block through block_tables, compute the attention scores inside the block
// and accumulate across blocks. The logical->physical translation of
// "vLLM框架中的KV cache优化与PagedAttention机制详解" §5.1 is done once per block
// for a whole work unit (all ids of the unit in one coalesced load, the page's
// "批量转换"), and tiles are requested ahead of use (the page's "预取机制", §5.2:
// R tiles per warp in flight through TMA).
//
// Work unit = one CTA per (kv-head, sequence, context partition); several CTAs
// share an SM, so one CTA's start-up and merge overlap the others' streaming.
// Tiles are 16 tokens of one kv-head (a 32-token block is two tiles). Each of
// the NW warps owns every NW-th tile of the unit and runs its own R-deep ring:
// its lane 0 issues one 4-D TMA box for the K tile and one for the V tile
// (whole rows, segment-major, swizzled) and the warp waits on the stage's mbarrier. No
// barrier is shared between warps until the final merge. Every wait is bounded
// by wall time; a wait that gives up makes the CTA stop and report.
#pragma once

#include <math_constants.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "decode_args.h"
#include "device_common.cuh"

namespace paged {

constexpr int kTileRows = 16;         // tokens per pipeline tile
constexpr int kMaxUnitBlocks = 1024;  // blocks of one work unit (ids staged in shared memory)

// Shared-memory geometry of one staged K (or V) tile: kTileRows token rows of
// one kv-head, RB bytes each. A row longer than the swizzle span (BOXB = 128
// or 64 bytes) is split into NBOX segments, and the TMA box puts the segment
// outermost: all rows' segment 0, then all rows' segment 1. Consecutive
// tokens of one segment thus sit in consecutive BOXB-byte lines, whose 16-byte
// chunks the TMA swizzles (128B or 64B pattern), so 8 rows read at the same
// logical column fall in 8 different bank groups.
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
    const int lin = ((o / BOXB) * BS + r) * BOXB + o % BOXB;
    return lin ^ ((lin >> 3) & SWZ);
  }
};

// Per-CTA shape: NW warps whose R-deep rings take 16 KB per warp (64 KB for
// the 4-warp CTA, so that three CTAs fit on an SM; six of the 2-warp CTA).
template <class Consumer, int NW_>
struct GridCfg {
  using T = typename Consumer::Tile;
  static constexpr int G = Consumer::G, D = T::D;
  static constexpr int NW = NW_;
  static constexpr int STAGE = 2 * T::BYTES;                 // K and V tiles
  static constexpr int R_RAW = 16384 / STAGE;
  static constexpr int R = R_RAW < 1 ? 1 : (R_RAW > 8 ? 8 : R_RAW);
  static constexpr int STAGES_BYTES = NW * R * STAGE;
  static_assert(NW * G * (D + 2) * 4 <= STAGES_BYTES, "merge buffer fits in the stages");
};

template <class Consumer, int NW_>
__global__ void __launch_bounds__(NW_ * 32)
    paged_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap) {
  using C = GridCfg<Consumer, NW_>;
  using T = typename Consumer::Tile;
  constexpr int D = T::D, G = Consumer::G, NW = C::NW, R = C::R, STAGE = C::STAGE;
  constexpr int TR = kTileRows;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES_BYTES);
  int32_t* ids = reinterpret_cast<int32_t*>(bars + NW * R);
  __shared__ int aborted;

  const int kvh = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    for (int r = 0; r < R; ++r) mbar_init(&bars[warp * R + r], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    aborted = 0;
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  // Everything below reads data of earlier kernels in the stream (the cache
  // rows the scatter kernel wrote): wait for them here.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Context length, clipped to what the launch covers.
  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (threadIdx.x == 0 && part == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  const int nblk = (ctx + a.block_size - 1) / a.block_size;
  const int parts = nblk == 0 ? 1 : (nblk + a.partition_blocks - 1) / a.partition_blocks;
  if (part >= parts) return;
  const int b_begin = part * a.partition_blocks;
  const int nlocal = min(b_begin + a.partition_blocks, nblk) - b_begin;
  const int tpb = a.block_size / TR;
  const int tok0 = b_begin * a.block_size;
  // tiles holding at least one context token
  const int ntiles = max(0, (min(ctx, (b_begin + nlocal) * a.block_size) - tok0 + TR - 1) / TR);

  // Block ids of this unit -> shared memory, validated once.
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
  for (int i = threadIdx.x; i < nlocal; i += NW * 32) {
    int32_t id = table[b_begin + i];
    if (id < 0 || id >= a.num_blocks) {
      report(a.err, kErrBadBlockId);
      id = -1;  // read as a box outside the pool: zero-filled
    }
    ids[i] = id;
  }
  __syncthreads();

  const int my_count = ntiles > warp ? (ntiles - warp + NW - 1) / NW : 0;
  uint8_t* my_stages = smem + warp * R * STAGE;
  uint64_t* my_bars = bars + warp * R;
  const uint64_t policy = l2_policy_evict_first();

  auto issue = [&](int k) {  // k-th tile of this warp
    const int t = warp + k * NW;
    const int stage = k % R;
    const int32_t bid = ids[t / tpb];
    const int32_t row0 = bid >= 0 ? bid * a.block_size + (t % tpb) * TR : -TR;
    uint8_t* kt = my_stages + stage * STAGE;
    if (skip_for_test(a.skip_tile, t)) return;
    mbar_arrive_expect_tx(&my_bars[stage], STAGE);
    tma_load_4d(kt, &kmap, &my_bars[stage], 0, row0, kvh, 0, policy);
    tma_load_4d(kt + T::BYTES, &vmap, &my_bars[stage], 0, row0, kvh, 0, policy);
  };
  if (lane == 0) {
    for (int k = 0; k < min(R, my_count); ++k) issue(k);
  }

  Consumer c;
  c.init(a, static_cast<const uint8_t*>(a.query) +
                (static_cast<int64_t>(s) * a.num_heads + kvh * G) * D * 2,
         kvh, lane);
  int k = 0;
  for (; k < my_count; ++k) {
    const int stage = k % R;
    if (!__all_sync(FULL, mbar_wait(&my_bars[stage], (k / R) & 1, a.wait_limit_ns, &aborted)))
      break;
    uint8_t* kt = my_stages + stage * STAGE;
    const int t = warp + k * NW;
    c.block(kt, kt + T::BYTES, max(0, min(TR, ctx - (tok0 + t * TR))), lane);
    __syncwarp();
    if (lane == 0 && k + R < my_count) issue(k + R);
  }
  if (k < my_count) {
    // A wait gave up (never expected): record it, let this warp's loads still
    // in flight land (bounded again), and stop the CTA after the barrier.
    if (lane == 0) {
      // the record first: a warp stopped by the flag below must not take it
      record_failure(a.diag, kSiteTile, blockIdx.x, blockIdx.y, blockIdx.z, warp, k, my_count,
                     0);
      aborted = 1;
    }
    for (int kk = k; kk < min(k + R, my_count); ++kk)
      mbar_wait(&my_bars[kk % R], (kk / R) & 1, a.wait_limit_ns);
  }

  // Merge the warps through shared memory (the rings are idle: every issued
  // load has been waited for).
  __syncthreads();
  const bool single = parts == 1;
  const int64_t row0 = static_cast<int64_t>(s) * a.num_heads + kvh * G;
  if (aborted) {
    // The unit's result is lost: leave zeros (single pass) or an empty
    // partial that the combine kernel gives no weight, never stale data.
    if (threadIdx.x == 0) report(a.err, kErrWaitTimeout);
    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
      const int g = idx / D, d = idx % D;
      if (single) {
        store_out(typename Consumer::QF{}, a.out, (row0 + g) * D + d, 0.f);
      } else if (d == 0) {
        a.ws_ml[(row0 + g) * a.max_parts + part] = make_float2(-CUDART_INF_F, 0.f);
      }
    }
    return;
  }
  float* mbuf = reinterpret_cast<float*>(smem);              // [NW][G][2]: m, l
  float* obuf = mbuf + NW * G * 2;                           // [NW][G][D]: acc
  c.finish(mbuf + warp * G * 2, obuf + warp * G * D, lane);
  __syncthreads();

  const float vs = a.v_scale ? a.v_scale[kvh] : 1.f;
  for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
    const int g = idx / D, d = idx % D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mbuf[(w * G + g) * 2]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = mbuf[(w * G + g) * 2];
      const float f = mw == -CUDART_INF_F ? 0.f : exp2f(mw - M);
      L += mbuf[(w * G + g) * 2 + 1] * f;
      o += obuf[(w * G + g) * D + d] * f;
    }
    o = L > 0.f ? o / L * vs : 0.f;
    if (single) {
      store_out(typename Consumer::QF{}, a.out, (row0 + g) * D + d, o);
    } else {
      const int64_t pi = (row0 + g) * a.max_parts + part;
      a.ws_o[pi * D + d] = o;
      if (d == 0) a.ws_ml[pi] = make_float2(M, L);
    }
  }
}

// Raise a kernel's dynamic shared-memory limit (once per kernel, device and size).
inline cudaError_t configure_kernel(const void* kern, size_t smem) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void*, int>, size_t>> configured;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (auto& c : configured)
    if (c.first.first == kern && c.first.second == dev) {
      if (c.second >= smem) return cudaSuccess;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e == cudaSuccess) c.second = smem;
      return e;
    }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e == cudaSuccess) configured.push_back({{kern, dev}, smem});
  return e;
}

// Launch with programmatic dependent launch: the grid may be scheduled while
// the previous kernel of the stream finishes; it waits (griddepcontrol.wait)
// before reading anything that kernel wrote.
template <class Kernel, class... Args>
cudaError_t launch_pdl(Kernel kern, dim3 grid, int threads, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <class Consumer, int NW>
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          cudaStream_t stream) {
  using C = GridCfg<Consumer, NW>;
  if (a.partition_blocks > kMaxUnitBlocks || a.block_size % kTileRows != 0)
    return cudaErrorNotSupported;
  const size_t smem = 1024 + C::STAGES_BYTES + 8 * C::NW * C::R +
                      4 * static_cast<size_t>(a.partition_blocks);
  auto kern = paged_decode_kernel<Consumer, NW>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(a.num_kv_heads, a.num_seqs, a.max_parts), C::NW * 32, smem,
                    stream, a, kmap, vmap);
}

}  // namespace paged
