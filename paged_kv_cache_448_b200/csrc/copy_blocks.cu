// copy_blocks.cu — whole-block copies between or within caches.
//
// Two uses share this kernel:
//  * the private copy of a shared block before a write ("大模型推理KV Cache内存
//    管理与PagedAttention分页显存实战": the prefix blocks of several requests are
//    shared under a reference count; a holder that writes into one gets its own
//    copy first), source and destination in the same cache;
//  * migration of blocks between GPU memory and host memory ("Paged KVCache：
//    大模型推理显存管理优化方案" §5, Hybrid Cache; the swap space of the vLLM
//    configuration in the first page), one side a pinned host pool read or
//    written through its mapped device address.
//
// A block of one cache is contiguous ([block_size, num_kv_heads, head_dim]), so
// a copy is a straight stream of 16-byte vectors. The work is cut into 128 KB
// chunks; a CTA of 256 threads loads a whole chunk into registers (32 vectors
// a thread, all in flight at once) and then stores it, with streaming cache
// hints since neither side is re-read by this kernel. The grid strides over
// (pair, chunk) for the K cache in y = 0 and the V cache in y = 1.
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_args.h"
#include "device_common.cuh"

namespace paged {
namespace {

constexpr int kCopyThreads = 256;
// 16-byte vectors per thread (measured on B200, 2048 copy-on-write pairs of
// 128 KB blocks: 5832 / 6162 / 6291 GB/s with 8 / 16 / 32)
constexpr int kCopyVec = 32;
constexpr int64_t kCopyChunk = int64_t(kCopyThreads) * kCopyVec * 16;  // 128 KB

struct CopyArgs {
  const uint8_t* src[2];  // K, V (V may be null)
  uint8_t* dst[2];
  const int32_t* pairs;   // [num_pairs][2]: source block, destination block
  int64_t num_pairs;
  int64_t block_bytes;
  int64_t chunks_per_block;
  int64_t num_src_blocks;
  int64_t num_dst_blocks;
  int32_t* err;           // optional error word
};

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const CopyArgs a) {
  const int cache = blockIdx.y;
  const uint8_t* src = a.src[cache];
  uint8_t* dst = a.dst[cache];
  if (!src) return;
  const int64_t total = a.num_pairs * a.chunks_per_block;
  for (int64_t i = blockIdx.x; i < total; i += gridDim.x) {
    const int64_t p = i / a.chunks_per_block, c = i % a.chunks_per_block;
    const int64_t s = a.pairs[2 * p], d = a.pairs[2 * p + 1];
    if (s < 0 || s >= a.num_src_blocks || d < 0 || d >= a.num_dst_blocks) {
      if (threadIdx.x == 0 && c == 0 && cache == 0 && a.err) report(a.err, kErrBadBlockId);
      continue;
    }
    const int64_t off = c * kCopyChunk;
    const int64_t nvec = min(kCopyChunk, a.block_bytes - off) / 16;
    const uint4* sp = reinterpret_cast<const uint4*>(src + s * a.block_bytes + off);
    uint4* dp = reinterpret_cast<uint4*>(dst + d * a.block_bytes + off);
    uint4 v[kCopyVec];
#pragma unroll
    for (int k = 0; k < kCopyVec; ++k) {
      const int64_t j = threadIdx.x + k * kCopyThreads;
      if (j < nvec) v[k] = __ldcs(sp + j);
    }
#pragma unroll
    for (int k = 0; k < kCopyVec; ++k) {
      const int64_t j = threadIdx.x + k * kCopyThreads;
      if (j < nvec) __stcs(dp + j, v[k]);
    }
  }
}

}  // namespace

cudaError_t launch_copy_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                               const int32_t* pairs, int64_t num_pairs, int64_t block_bytes,
                               int64_t num_src_blocks, int64_t num_dst_blocks, int32_t* err,
                               int sm_count, cudaStream_t stream) {
  CopyArgs a{};
  a.src[0] = static_cast<const uint8_t*>(src_k);
  a.src[1] = static_cast<const uint8_t*>(src_v);
  a.dst[0] = static_cast<uint8_t*>(dst_k);
  a.dst[1] = static_cast<uint8_t*>(dst_v);
  a.pairs = pairs;
  a.num_pairs = num_pairs;
  a.block_bytes = block_bytes;
  a.chunks_per_block = (block_bytes + kCopyChunk - 1) / kCopyChunk;
  a.num_src_blocks = num_src_blocks;
  a.num_dst_blocks = num_dst_blocks;
  a.err = err;
  const int64_t total = num_pairs * a.chunks_per_block;
  // up to eight CTAs per SM (each holding a 128 KB chunk in registers),
  // striding beyond that
  const int64_t cap = static_cast<int64_t>(sm_count) * 8;
  const dim3 grid(static_cast<unsigned>(total < cap ? total : cap), src_v ? 2u : 1u);
  copy_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace paged
