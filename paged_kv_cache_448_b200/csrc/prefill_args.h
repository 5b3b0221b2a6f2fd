// prefill_args.h — host/device argument block of the multi-token query kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "decode_args.h"

namespace paged {

struct PrefillArgs {
  void* out;                     // [T, H, D] q dtype
  const void* query;             // [T, H, D] q dtype
  const int32_t* cu_query_lens;  // [S + 1]: rows of sequence s are cu[s] .. cu[s+1]-1
  const int32_t* block_tables;   // [S, max_blocks_per_seq]
  const int32_t* context_lens;   // [S], including the query tokens
  const float* k_scale;          // [Hkv] (E4M3 cache) or null
  const float* v_scale;
  int32_t* err;                  // error word
  int32_t* diag;                 // failure record
  int64_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t ctx_limit;             // min(max_context_len, max_blocks_per_seq * block_size)
  int32_t num_seqs;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t block_size;
  float scale_log2;              // softmax scale * log2(e)
  // split of the key range (1 part = no split)
  int32_t q_tiles;               // query tiles per (sequence, kv-head) in the launch
  int32_t partition_tiles;       // 16-token tiles per part (a multiple of 4)
  int32_t max_parts;
  float* ws_o;                   // [T * H][max_parts][D] partial outputs (normalised)
  float2* ws_ml;                 // [T * H][max_parts] (max, sum) in base-2 units
  int32_t skip_tile;             // failure-detection test: 16-token tile of the unit
                                 // (query tile 0, kv-head 0, sequence 0) whose loads are
                                 // left out; -1 none
  int32_t dup_rows;              // tcgen05 kernel, one row group, units of <= 64 rows:
                                 // each row repeated 64 lanes further on (set by
                                 // launch_prefill_tc)
  uint64_t wait_limit_ns;        // bound of every pipeline wait
};

// Query tokens per CTA of the mma.sync kernel (64 rows = tokens x group).
__host__ __device__ constexpr int prefill_tokens_per_cta(int group) { return 64 / group; }

// mma.sync kernel for one (q dtype, cache dtype) pair: grid of
// a.q_tiles * a.max_parts CTAs per (sequence, kv-head), then, when the key
// range is split (a.max_parts > 1), the combine kernel. cudaErrorNotSupported
// for shapes without a kernel.
cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                           int q_dtype, int cache_dtype, int head_dim, int group,
                           int32_t max_query_len, cudaStream_t stream);

// Merge of the key-range parts of a split launch (a.max_parts > 1) whose
// CTAs took qt query tokens each: one warp per (query token, head).
cudaError_t launch_prefill_combine(const PrefillArgs& a, int q_dtype, int head_dim, int qt,
                                   int32_t max_query_len, cudaStream_t stream);

// The same on the 5th-generation tensor cores (tcgen05, tensor memory); the
// tensor maps are the one-segment boxes of encode_cache_map(..., 1 segment).
// An E4M3 cache needs head_dim 128.
cudaError_t launch_prefill_tc(const PrefillArgs& a, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int q_dtype, int cache_dtype,
                              int head_dim, int group, int32_t max_query_len,
                              cudaStream_t stream);

}  // namespace paged
