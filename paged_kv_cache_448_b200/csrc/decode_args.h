// decode_args.h — host/device argument block of the decode kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace paged {

enum DType : int { kF16 = 0, kBF16 = 1, kE4M3 = 2 };

// Bits of the workspace error word.
enum : int32_t {
  kErrBadBlockId = 1,      // a block-table entry outside [0, num_blocks)
  kErrContextClipped = 2,  // a context length above what the launch covers
  kErrWaitTimeout = 4,     // a pipeline wait gave up (never expected)
  kErrBadSlot = 8,         // reshape_and_cache: a slot outside the pool
  kErrQueryLonger = 16,    // multi-token query: more query rows than context (rows are zeros)
};

// Failure sites recorded in the diagnostic words (the first word of the record).
enum : int32_t {
  kSiteTile = 4,        // decode: a tile's loads never completed
                        //   (values: kv-head, sequence, partition, warp, warp's tile, its count)
  kSitePrefill = 5,     // multi-token query on mma.sync: a tile or a stage release
                        //   (values: CTA x, y, z, warp or step, tile, tiles, 0 / 1 = producer)
  kSiteTcStep = 6,      // multi-token query on tcgen05: an MMA-warp wait
                        //   (values: the CTA's unit - query tile + q_tiles * part, kv-head,
                        //   sequence - then K steps received, V steps received, steps, groups)
  kSiteFp8Tile = 7,     // decode on tcgen05 (E4M3 cache): a role's wait
                        //   (values: kv-head, sequence, partition, role, tile, tiles)
};

// Words of the workspace header (int32): the error word and, from kWordDiag,
// the record of the first failure of a launch.
enum : int { kWordError = 0, kWordDiag = 8 };


struct DecodeArgs {
  void* out;                    // [S, H, D] q dtype
  const void* query;            // [S, H, D] q dtype
  const int32_t* block_tables;  // [S, max_blocks_per_seq]
  const int32_t* context_lens;  // [S]
  const float* k_scale;         // [Hkv] (FP8 cache) or null
  const float* v_scale;
  float* ws_o;                  // [S, H, max_parts, D] partial outputs (split mode)
  float2* ws_ml;                // [S, H, max_parts] (running max, sum) in log2 units
  int32_t* err;                 // error word (bits of the kErr* enum)
  int32_t* diag;                // header words kWordDiag..+7: first failure record
  int64_t num_blocks;
  int32_t max_blocks_per_seq;
  int32_t ctx_limit;            // min(max_context_len, max_blocks_per_seq * block_size)
  int32_t num_seqs;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t partition_blocks;     // blocks per partition (single pass: covers max context)
  int32_t max_parts;            // partitions per sequence in the launch (1 = single pass)
  float scale_log2;             // softmax scale * log2(e)
  int32_t block_size;           // tokens per cache block (a multiple of 16)
  int32_t skip_tile;            // failure-detection test: tile of CTA (0,0,0) not loaded; -1 none
  uint64_t wait_limit_ns;       // bound of every pipeline wait
};

// Per (q dtype, cache dtype) dispatchers, defined in decode_<q>_<c>.cu.
// `warps` is the CTA width (2 or 4 warps). Return cudaErrorNotSupported for a
// (head_dim, group, width) they lack.
using DecodeFn = cudaError_t (*)(const DecodeArgs&, const CUtensorMap&, const CUtensorMap&,
                                 int head_dim, int group, int warps, cudaStream_t);

cudaError_t decode_f16_f16(const DecodeArgs&, const CUtensorMap&, const CUtensorMap&, int, int,
                           int, cudaStream_t);
cudaError_t decode_bf16_bf16(const DecodeArgs&, const CUtensorMap&, const CUtensorMap&, int, int,
                             int, cudaStream_t);
cudaError_t decode_f16_e4m3(const DecodeArgs&, const CUtensorMap&, const CUtensorMap&, int, int,
                            int, cudaStream_t);
cudaError_t decode_bf16_e4m3(const DecodeArgs&, const CUtensorMap&, const CUtensorMap&, int, int,
                             int, cudaStream_t);

cudaError_t launch_reduce(const DecodeArgs& a, int q_dtype, int head_dim, cudaStream_t stream);

// Decode over an E4M3 cache with head_dim 128 on tcgen05 (tokens on M), any
// query group up to 8; cudaErrorNotSupported otherwise.
cudaError_t decode_fp8_tc(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                          int q_dtype, int group, cudaStream_t stream);
// kv-heads per CTA of that kernel (its TMA boxes span as many heads).
int decode_fp8_tc_heads_per_cta(int num_kv_heads, int group);

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache,
                                     void* value_cache, const int32_t* slot_mapping,
                                     int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int64_t num_blocks, int kv_dtype,
                                     int cache_dtype, const float* k_scale, const float* v_scale,
                                     int32_t* err, cudaStream_t stream);

cudaError_t launch_copy_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                               const int32_t* pairs, int64_t num_pairs, int64_t block_bytes,
                               int64_t num_src_blocks, int64_t num_dst_blocks, int32_t* err,
                               int sm_count, cudaStream_t stream);

// Box geometry shared by the host tensor-map encoder and the kernels: a row
// of head_dim elements is cut into segments of at most 128 bytes (the widest
// swizzled box row), all loaded by one 4-D box per tile.
__host__ __device__ constexpr int box_bytes(int row_bytes) { return row_bytes < 128 ? row_bytes : 128; }

}  // namespace paged
