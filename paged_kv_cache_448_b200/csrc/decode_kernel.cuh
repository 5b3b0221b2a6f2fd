// decode_kernel.cuh — the paged decode kernel: block-table walk, TMA staging
// of K/V blocks through a per-warp shared-memory ring, and the merge of the
// per-warp online-softmax states. The arithmetic on a staged block is done by
// a Consumer (consumer_simt.cuh: fp32 CUDA cores; consumer_mma.cuh: tensor
// cores for query groups).
//
// Follows "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.3 (PagedAttention
// Kernel): for each sequence, find the physical K/V block of each logical
// block through block_tables, compute the attention scores inside the block
// and accumulate across blocks. The logical->physical translation of
// "vLLM框架中的KV cache优化与PagedAttention机制详解" §5.1 is done once per block
// (one table lookup per block, the page's "批量转换": all ids of a partition
// are read in one coalesced load) and blocks are requested ahead of use (the
// page's "预取机制", §5.2: here R blocks per warp in flight through TMA).
//
// Work unit = one CTA per (kv-head, sequence, context partition). Each of the
// NW warps owns every NW-th block of the partition and runs its own R-deep ring
// of stages: its lane 0 issues one TMA box load per <=128-byte column of the
// K and V tiles of a block (block_size rows of one kv-head, 128B/64B
// swizzled), and the warp waits on the stage's mbarrier. No barrier is shared
// between warps until the final merge.
#pragma once

#include <math_constants.h>

#include "decode_args.h"
#include "device_common.cuh"

namespace paged {

// Shared-memory geometry of one staged K (or V) tile: block_size rows of one
// kv-head, each row cut into NBOX boxes of BOXB bytes stored box after box,
// swizzled the way the TMA writes them (128B or 64B pattern).
template <class CF, int D_, int BS_>
struct Tile {
  static constexpr int D = D_, BS = BS_;
  static constexpr int EB = CF::kBytes;
  static constexpr int RB = D * EB;                          // bytes per token row
  static constexpr int BOXB = box_bytes(RB);
  static constexpr int NBOX = RB / BOXB;
  static constexpr int SWZ = BOXB == 128 ? 0x70 : (BOXB == 64 ? 0x30 : 0);
  static constexpr int BYTES = BS * RB;
  // Byte offset of logical byte `o` of row `r`.
  static __device__ __forceinline__ uint32_t off(int r, int o) {
    const int box = o / BOXB;
    const int lin = r * BOXB + (o % BOXB);
    return box * (BS * BOXB) + (lin ^ ((lin >> 3) & SWZ));
  }
};

template <class Consumer>
__global__ void __launch_bounds__(Consumer::NW * 32)
    paged_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap) {
  using T = typename Consumer::Tile;
  constexpr int BS = T::BS, D = T::D, G = Consumer::G, NW = Consumer::NW, R = Consumer::R;
  constexpr int STAGE = 2 * T::BYTES;
  constexpr int STAGES_BYTES = NW * R * STAGE;
  static_assert(NW * G * (D + 2) * 4 <= STAGES_BYTES, "merge buffer fits in the stages");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES_BYTES);
  int32_t* ids = reinterpret_cast<int32_t*>(bars + NW * R);

  const int kvh = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Context length, clipped to what the launch covers.
  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (threadIdx.x == 0 && part == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int parts = nblk == 0 ? 1 : (nblk + a.partition_blocks - 1) / a.partition_blocks;
  if (part >= parts) return;
  const int b_begin = part * a.partition_blocks;
  const int nlocal = min(b_begin + a.partition_blocks, nblk) - b_begin;

  // Block ids of this partition -> shared memory, validated once.
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
  for (int i = threadIdx.x; i < nlocal; i += NW * 32) {
    int32_t id = table[b_begin + i];
    if (id < 0 || id >= a.num_blocks) {
      report(a.err, kErrBadBlockId);
      id = -1;
    }
    ids[i] = id;
  }
  if (lane == 0) {
    for (int r = 0; r < R; ++r) mbar_init(&bars[warp * R + r], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  __syncthreads();

  const int my_count = nlocal > warp ? (nlocal - warp + NW - 1) / NW : 0;
  uint8_t* my_stages = smem + warp * R * STAGE;
  uint64_t* my_bars = bars + warp * R;
  const uint64_t policy = l2_policy_evict_first();

  auto issue = [&](int it) {
    const int stage = it % R;
    const int32_t id = ids[warp + it * NW];
    // An invalid id reads a box entirely outside the pool: TMA zero-fills it.
    const int32_t row0 = id >= 0 ? id * BS : -BS;
    uint8_t* kt = my_stages + stage * STAGE;
    uint8_t* vt = kt + T::BYTES;
    mbar_arrive_expect_tx(&my_bars[stage], STAGE);
#pragma unroll
    for (int b = 0; b < T::NBOX; ++b) {
      const int x = b * (T::BOXB / T::EB);
      tma_load_3d_hint(kt + b * BS * T::BOXB, &kmap, &my_bars[stage], x, kvh, row0, policy);
      tma_load_3d_hint(vt + b * BS * T::BOXB, &vmap, &my_bars[stage], x, kvh, row0, policy);
    }
  };
  if (lane == 0) {
    for (int it = 0; it < min(R, my_count); ++it) issue(it);
  }

  Consumer c;
  c.init(a, s, kvh, lane);

  bool timed_out = false;
  for (int it = 0; it < my_count; ++it) {
    const int stage = it % R;
    if (!mbar_wait(&my_bars[stage], (it / R) & 1)) {
      timed_out = true;
      break;
    }
    uint8_t* kt = my_stages + stage * STAGE;
    const int valid = min(BS, ctx - (b_begin + warp + it * NW) * BS);
    c.block(kt, kt + T::BYTES, valid, lane);
    __syncwarp();
    if (lane == 0 && it + R < my_count) issue(it + R);
  }
  if (timed_out && lane == 0) report(a.err, kErrWaitTimeout);

  // Merge the warps through shared memory (the ring is idle: every issued
  // load has been waited for).
  __syncthreads();
  float* mbuf = reinterpret_cast<float*>(smem);              // [NW][G][2]: m, l
  float* obuf = mbuf + NW * G * 2;                           // [NW][G][D]: unnormalised acc
  c.finish(mbuf + warp * G * 2, obuf + warp * G * D, lane);
  __syncthreads();

  const bool single = parts == 1;
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
    const int64_t row = static_cast<int64_t>(s) * a.num_heads + kvh * G + g;
    if (single) {
      store_out(typename Consumer::QF{}, a.out, row * D + d, o);
    } else {
      const int64_t pi = row * a.max_parts + part;
      a.ws_o[pi * D + d] = o;
      if (d == 0) a.ws_ml[pi] = make_float2(M, L);
    }
  }
}

template <class Consumer>
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          cudaStream_t stream) {
  using T = typename Consumer::Tile;
  const size_t stages = static_cast<size_t>(Consumer::NW) * Consumer::R * 2 * T::BYTES;
  const size_t smem = 1024 + stages + 8 * Consumer::NW * Consumer::R +
                      4 * static_cast<size_t>(a.partition_blocks);
  auto kern = paged_decode_kernel<Consumer>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_kv_heads, a.num_seqs, a.max_parts);
  kern<<<grid, Consumer::NW * 32, smem, stream>>>(a, kmap, vmap);
  return cudaGetLastError();
}

}  // namespace paged
