// api.cu — the C ABI of libpaged's device calls: argument validation on the
// host, the launch plan (single pass or context partitions + combine), TMA
// descriptors for the cache, and the kernel launches. No device memory is
// allocated here; the caller owns every buffer.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "decode_args.h"
#include "device_common.cuh"
#include "prefill_args.h"
#include "paged.h"
#include "status.h"

namespace paged {
namespace {

constexpr size_t kHeaderBytes = 256;          // error word + padding
constexpr int32_t kMaxPartitionBlocks = 1024; // block ids staged in shared memory per CTA
constexpr int32_t kMinAutoPartition = 256;    // tokens
// Partitions of at most this many tokens run on the 2-warp CTA: six of them
// per SM overlap their start-up (table read, first loads) and the end of
// their unit better than three 4-warp CTAs (~7% on 512-token partitions of a
// 64-sequence, 8-kv-head batch); longer units keep the 4-warp CTA.
constexpr int32_t kNarrowTokens = 512;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) dev = 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over a cache viewed as [rows = num_blocks*block_size][num_kv_heads]
// [segments][segment elements] (a row of head_dim elements cut into <=128-byte
// segments): one box = 16 rows of one kv-head, whole rows, swizzled per segment,
// stored in shared memory segment-major (all rows' first segment, then the next).
pa_status encode_cache_map(CUtensorMap* map, const void* cache, int64_t num_blocks,
                           int32_t block_size, int32_t hkv, int32_t head_dim, int elem,
                           bool one_segment = false, int heads_per_box = 1) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int row_bytes = head_dim * elem;
  const int seg = box_bytes(row_bytes);
  // dims: elements of a segment, token slots, kv-heads, segments of a row.
  // The box is one kv-head x 16 slots x all segments, segment outermost.
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(seg / elem),
                        static_cast<cuuint64_t>(num_blocks) * block_size,
                        static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(row_bytes / seg)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(row_bytes) * hkv,
                           static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(seg)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(seg / elem), 16u,
                       static_cast<cuuint32_t>(heads_per_box),
                       one_segment ? 1u : static_cast<cuuint32_t>(row_bytes / seg)};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapSwizzle swz = seg == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                               : seg == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = enc(map, elem == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                   4, const_cast<void*>(cache), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return PA_OK;
}

pa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return PA_OK;
  if (e == cudaErrorNotSupported)
    return fail(PA_ERR_UNSUPPORTED, "%s: no kernel for this shape", what);
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int elem_bytes(pa_dtype t) { return t == PA_FP8_E4M3 ? 1 : 2; }

// Launch plan shared by pa_decode and the sizing queries.
struct Plan {
  int32_t partition_tokens;  // tokens per partition
  int32_t partition_blocks;
  int32_t max_parts;         // 1 = single pass
};

constexpr int32_t kMaxParts = 65535;  // partitions per sequence (grid z extent)

// fp8_tc: the E4M3 tcgen05 kernel (two CTAs per SM, two tiles of 128 tokens
// in flight in each), which runs best on few, long units: measured on B200 on
// the shared-prefix E4M3 workload (1 024 sequence x kv-head pairs of 1 100 to
// 1 500 tokens), one pass 77 us against 98 / 120 / 175 us with partitions of
// 1 024 / 512 / 256 tokens. It is cut into partitions only below one wave of
// units. The other decode kernels (three CTAs per SM) want about four waves.
Plan make_plan(int32_t num_seqs, int32_t num_kv_heads, int32_t block_size,
               int32_t max_context_len, int32_t requested, bool fp8_tc) {
  const int32_t blocks_max = std::max<int32_t>(1, (max_context_len + block_size - 1) / block_size);
  Plan p{};
  int32_t pb;
  if (requested > 0) {
    pb = (requested + block_size - 1) / block_size;
  } else {
    // Enough independent work units to keep every SM busy through the end of
    // the launch; otherwise cut the context into partitions (>= 256 tokens).
    const int64_t pairs = static_cast<int64_t>(num_seqs) * num_kv_heads;
    const int64_t want = fp8_tc ? 2LL * sm_count() : 4LL * sm_count() * 3;
    pb = blocks_max;
    if (pairs < want && static_cast<int64_t>(blocks_max) * block_size > kMinAutoPartition) {
      const int32_t min_pb = std::max(1, kMinAutoPartition / block_size);
      pb = min_pb;
      // largest power-of-two multiple of the minimum that still gives `want` units
      for (int32_t cand = min_pb; cand < blocks_max; cand *= 2) {
        const int64_t units = pairs * ((blocks_max + cand - 1) / cand);
        if (units >= want) pb = cand;
      }
    }
  }
  pb = std::min(std::max(pb, 1), std::min(blocks_max, kMaxPartitionBlocks));
  pb = std::max(pb, (blocks_max + kMaxParts - 1) / kMaxParts);
  p.partition_blocks = pb;
  p.partition_tokens = pb * block_size;
  p.max_parts = (blocks_max + pb - 1) / pb;
  return p;
}

// Workspace layout: [header 256 B: error word, failure record] then, with
// partitions: [partial (m, l), S*H*max_parts float2] [partial o, S*H*max_parts*D float].
struct Layout {
  size_t ml, o, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Layout layout_for(const Plan& p, int32_t num_seqs, int32_t num_heads, int32_t head_dim) {
  Layout l{};
  size_t at = kHeaderBytes;
  if (p.max_parts > 1) {
    const size_t rows = static_cast<size_t>(num_seqs) * num_heads * p.max_parts;
    l.ml = at;
    at = align256(at + rows * sizeof(float2));
    l.o = at;
    at += rows * head_dim * sizeof(float);
  }
  l.total = at;
  return l;
}

// The address kernels use for a buffer: device (or managed) memory as is;
// pinned host memory through its mapped device address. Pageable host memory
// has none and is rejected.
pa_status device_view(const void* p, const void** out, const char* what) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: %s is not a CUDA-visible pointer", what);
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
    *out = p;
    return PA_OK;
  }
  if (at.type == cudaMemoryTypeHost && at.devicePointer) {
    *out = at.devicePointer;
    return PA_OK;
  }
  return fail(PA_ERR_INVALID_ARG,
              "copy_blocks: %s is pageable host memory (pin it, e.g. cudaHostAlloc)", what);
}

bool shape_supported(int32_t head_dim, int32_t block_size) {
  return (head_dim == 64 || head_dim == 128) && (block_size == 16 || block_size == 32);
}

// A failure-detection test's request for the next launch on this thread
// (pa_inject_wait_timeout): the tile whose loads are left out, and the bound
// of every wait. Taken, and cleared, by the next decode or multi-token launch.
struct Injection {
  int32_t tile = -1;
  uint64_t limit_ns = 0;
};
thread_local Injection g_injection;

void take_injection(int32_t* skip_tile, uint64_t* wait_limit_ns) {
  *skip_tile = g_injection.tile;
  *wait_limit_ns = g_injection.tile >= 0 && g_injection.limit_ns > 0 ? g_injection.limit_ns
                                                                      : kWaitLimitNs;
  g_injection = Injection{};
}

}  // namespace
}  // namespace paged

using namespace paged;

extern "C" {

PA_API pa_status pa_reshape_and_cache(const void* key, const void* value, void* key_cache,
                                      void* value_cache, const int32_t* slot_mapping,
                                      int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, int64_t num_blocks, pa_dtype kv_dtype,
                                      pa_dtype cache_dtype, const float* k_scale,
                                      const float* v_scale, pa_stream_t stream) {
  clear_error();
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: negative or zero size");
  if (!shape_supported(head_dim, block_size))
    return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: head_dim %d / block_size %d unsupported",
                head_dim, block_size);
  if (kv_dtype != PA_F16 && kv_dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: new K/V must be f16 or bf16");
  if (cache_dtype != kv_dtype && cache_dtype != PA_FP8_E4M3)
    return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: cache dtype must equal kv dtype or be e4m3");
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (fp8 != (k_scale != nullptr) || fp8 != (v_scale != nullptr))
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: k_scale/v_scale required exactly for e4m3");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: null pointer");
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(key_cache, 16) ||
      !aligned(value_cache, 16) || !aligned(slot_mapping, 4) || (k_scale && !aligned(k_scale, 4)) ||
      (v_scale && !aligned(v_scale, 4)))
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: misaligned pointer");
  cudaError_t e = launch_reshape_and_cache(
      key, value, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
      block_size, num_blocks, kv_dtype, cache_dtype, k_scale, v_scale, nullptr,
      reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e, "reshape_and_cache");
}

PA_API int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_heads,
                                          int32_t num_kv_heads, int32_t head_dim,
                                          int32_t block_size, int32_t max_context_len,
                                          int32_t partition_tokens, pa_dtype cache_dtype) {
  (void)num_heads;
  if (num_seqs < 0 || num_kv_heads <= 0 || block_size <= 0 || max_context_len < 0) return 0;
  Plan p = make_plan(num_seqs, num_kv_heads, block_size, max_context_len, partition_tokens,
                     cache_dtype == PA_FP8_E4M3 && head_dim == 128);
  return p.max_parts <= 1 ? std::max(p.partition_tokens, max_context_len) : p.partition_tokens;
}

PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t block_size,
                                       int32_t max_context_len, int32_t partition_tokens,
                                       pa_dtype cache_dtype) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_context_len < 0)
    return 0;
  Plan p = make_plan(num_seqs, num_kv_heads, block_size, max_context_len, partition_tokens,
                     cache_dtype == PA_FP8_E4M3 && head_dim == 128);
  (void)num_kv_heads;
  return layout_for(p, num_seqs, num_heads, head_dim).total;
}

PA_API pa_status pa_workspace_init(void* workspace, size_t workspace_bytes, pa_stream_t stream) {
  clear_error();
  if (!workspace || workspace_bytes < kHeaderBytes || !aligned(workspace, 256))
    return fail(PA_ERR_INVALID_ARG, "workspace_init: need >= 256 bytes, 256-byte aligned");
  return cuda_status(
      cudaMemsetAsync(workspace, 0, kHeaderBytes, reinterpret_cast<cudaStream_t>(stream)),
      "workspace_init");
}

PA_API pa_status pa_inject_wait_timeout(int32_t tile, uint64_t wait_limit_ns) {
  clear_error();
  if (tile >= 0 && wait_limit_ns == 0)
    return fail(PA_ERR_INVALID_ARG, "inject_wait_timeout: wait limit must be positive");
  g_injection.tile = tile < 0 ? -1 : tile;
  g_injection.limit_ns = tile < 0 ? 0 : wait_limit_ns;
  return PA_OK;
}

PA_API pa_status pa_decode_check(void* workspace, pa_stream_t stream) {
  clear_error();
  if (!workspace) return fail(PA_ERR_INVALID_ARG, "decode_check: null workspace");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // error word (int 0) and the first failure's record (ints 8..15)
  int32_t head[16] = {};
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(head, workspace, sizeof(head), cudaMemcpyDeviceToHost);
  const int32_t word = head[kWordError];
  if (e == cudaSuccess && word != 0) e = cudaMemset(workspace, 0, 64);  // error + failure record
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode_check: %s", cudaGetErrorString(e));
  if (word & kErrWaitTimeout) {
    const int32_t* r = head + kWordDiag;
    const char* site = r[0] == kSiteTile       ? "decode tile"
                       : r[0] == kSitePrefill  ? "multi-token (mma.sync) tile"
                       : r[0] == kSiteTcStep   ? "multi-token (tcgen05) step"
                       : r[0] == kSiteFp8Tile  ? "decode (tcgen05 FP8) tile"
                                               : "unknown site";
    return fail(PA_ERR_CUDA,
                "decode: a pipeline wait timed out; first failure: site %d (%s), CTA (%d, %d, "
                "%d), values %d %d %d %d",
                r[0], site, r[1], r[2], r[3], r[4], r[5], r[6], r[7]);
  }
  if (word & (kErrBadBlockId | kErrContextClipped | kErrQueryLonger))
    return fail(PA_ERR_BAD_TABLE, "decode: %s%s%s",
                (word & kErrBadBlockId) ? "block-table entry outside the pool; " : "",
                (word & kErrContextClipped) ? "context length beyond the launch; clipped; " : "",
                (word & kErrQueryLonger) ? "query longer than its context; rows zeroed" : "");
  if (word) return fail(PA_ERR_CUDA, "decode: error word 0x%x", word);
  return PA_OK;
}

PA_API pa_status pa_decode(void* out, const void* query, const void* key_cache,
                           const void* value_cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens,
                           int32_t max_context_len, int32_t num_seqs, int32_t num_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int64_t num_blocks, float scale, pa_dtype q_dtype,
                           pa_dtype cache_dtype, const float* k_scale, const float* v_scale,
                           int32_t partition_tokens, void* workspace, size_t workspace_bytes,
                           pa_stream_t stream) {
  clear_error();
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      max_context_len < 0 || num_blocks <= 0 || partition_tokens < 0)
    return fail(PA_ERR_INVALID_ARG, "decode: negative or zero size");
  if (num_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "decode: num_heads %% num_kv_heads != 0");
  const int32_t group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PA_ERR_UNSUPPORTED, "decode: query group %d not in {1,2,4,8}", group);
  if (!shape_supported(head_dim, block_size))
    return fail(PA_ERR_UNSUPPORTED, "decode: head_dim %d / block_size %d unsupported", head_dim,
                block_size);
  if (q_dtype != PA_F16 && q_dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "decode: query must be f16 or bf16");
  if (cache_dtype != q_dtype && cache_dtype != PA_FP8_E4M3)
    return fail(PA_ERR_UNSUPPORTED, "decode: cache dtype must equal query dtype or be e4m3");
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (fp8 != (k_scale != nullptr) || fp8 != (v_scale != nullptr))
    return fail(PA_ERR_INVALID_ARG, "decode: k_scale/v_scale required exactly for e4m3");
  if (num_blocks * block_size > INT32_MAX)
    return fail(PA_ERR_UNSUPPORTED, "decode: pool rows exceed 2^31");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "decode: scale is not finite");
  if (!workspace || !aligned(workspace, 256))
    return fail(PA_ERR_INVALID_ARG, "decode: workspace missing or not 256-byte aligned");
  if (num_seqs == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "decode: null pointer");
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) ||
      !aligned(value_cache, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4) ||
      (k_scale && !aligned(k_scale, 4)) || (v_scale && !aligned(v_scale, 4)))
    return fail(PA_ERR_INVALID_ARG, "decode: misaligned pointer");

  const Plan plan = make_plan(num_seqs, num_kv_heads, block_size, max_context_len,
                              partition_tokens, fp8 && head_dim == 128);
  if (num_seqs > 65535 || plan.max_parts > kMaxParts)
    return fail(PA_ERR_UNSUPPORTED, "decode: %d sequences x %d partitions exceed the grid",
                num_seqs, plan.max_parts);
  const Layout lay = layout_for(plan, num_seqs, num_heads, head_dim);
  const size_t need = lay.total;
  if (workspace_bytes < need)
    return fail(PA_ERR_INVALID_ARG, "decode: workspace %zu bytes < %zu needed", workspace_bytes,
                need);

  const int elem = elem_bytes(cache_dtype);
  // an E4M3 cache with head_dim 128 runs on the tcgen05 kernel, whose boxes
  // span its kv-heads per CTA
  const bool fp8_tc = fp8 && head_dim == 128;
  const int box_heads = fp8_tc ? decode_fp8_tc_heads_per_cta(num_kv_heads, group) : 1;
  CUtensorMap kmap, vmap;
  pa_status st = encode_cache_map(&kmap, key_cache, num_blocks, block_size, num_kv_heads,
                                  head_dim, elem, false, box_heads);
  if (st == PA_OK)
    st = encode_cache_map(&vmap, value_cache, num_blocks, block_size, num_kv_heads, head_dim,
                          elem, false, box_heads);
  if (st != PA_OK) return st;

  DecodeArgs a{};
  a.out = out;
  a.query = query;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.err = reinterpret_cast<int32_t*>(ws) + kWordError;
  a.diag = reinterpret_cast<int32_t*>(ws) + kWordDiag;
  if (plan.max_parts > 1) {
    a.ws_ml = reinterpret_cast<float2*>(ws + lay.ml);
    a.ws_o = reinterpret_cast<float*>(ws + lay.o);
  }
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.ctx_limit = std::min<int64_t>(max_context_len,
                                  static_cast<int64_t>(max_blocks_per_seq) * block_size);
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.partition_blocks = plan.partition_blocks;
  a.max_parts = plan.max_parts;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.block_size = block_size;
  take_injection(&a.skip_tile, &a.wait_limit_ns);

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (fp8_tc) {
    // E4M3 rows of 128 bytes: the tcgen05 kernel takes the tiles as stored
    st = cuda_status(decode_fp8_tc(a, kmap, vmap, q_dtype == PA_F16 ? kF16 : kBF16, group, cs),
                     "decode");
  } else {
    DecodeFn fn = nullptr;
    if (q_dtype == PA_F16) fn = fp8 ? decode_f16_e4m3 : decode_f16_f16;
    else fn = fp8 ? decode_bf16_e4m3 : decode_bf16_bf16;
    const int warps = plan.max_parts > 1 && plan.partition_tokens <= kNarrowTokens ? 2 : 4;
    st = cuda_status(fn(a, kmap, vmap, head_dim, group, warps, cs), "decode");
  }
  if (st != PA_OK || plan.max_parts <= 1) return st;
  return cuda_status(launch_reduce(a, q_dtype, head_dim, cs), "decode combine");
}

PA_API pa_status pa_copy_blocks(const void* src_key_cache, const void* src_value_cache,
                                void* dst_key_cache, void* dst_value_cache,
                                const int32_t* block_pairs, int32_t num_pairs, int64_t block_bytes,
                                int64_t num_src_blocks, int64_t num_dst_blocks,
                                int32_t* error_word, pa_stream_t stream) {
  clear_error();
  if (num_pairs < 0 || block_bytes <= 0 || block_bytes % 16 != 0 || num_src_blocks <= 0 ||
      num_dst_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: bad sizes (block_bytes a positive multiple of 16)");
  if (!src_key_cache || !dst_key_cache || !block_pairs)
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: null pointer");
  if ((src_value_cache == nullptr) != (dst_value_cache == nullptr))
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: give both value caches or neither");
  if (!aligned(src_key_cache, 16) || !aligned(dst_key_cache, 16) ||
      !aligned(src_value_cache, 16) || !aligned(dst_value_cache, 16) || !aligned(block_pairs, 4) ||
      !aligned(error_word, 4))
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: misaligned pointer");
  if (num_pairs == 0) return PA_OK;
  const void* views[5] = {};
  const void* ptrs[5] = {src_key_cache, dst_key_cache, src_value_cache, dst_value_cache,
                         block_pairs};
  const char* names[5] = {"src_key_cache", "dst_key_cache", "src_value_cache",
                          "dst_value_cache", "block_pairs"};
  for (int i = 0; i < 5; ++i) {
    if (!ptrs[i]) continue;
    pa_status st = device_view(ptrs[i], &views[i], names[i]);
    if (st != PA_OK) return st;
  }
  int32_t* err = nullptr;
  if (error_word) {
    const void* v = nullptr;
    pa_status st = device_view(error_word, &v, "error_word");
    if (st != PA_OK) return st;
    err = const_cast<int32_t*>(static_cast<const int32_t*>(v));
  }
  cudaError_t e = launch_copy_blocks(
      views[0], views[2], const_cast<void*>(views[1]), const_cast<void*>(views[3]),
      static_cast<const int32_t*>(views[4]), num_pairs, block_bytes, num_src_blocks,
      num_dst_blocks, err, sm_count(), reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e, "copy_blocks");
}

}  // extern "C"

namespace paged {
namespace {

// Kernel choice and split of the key range for the multi-token query.
// Chunks that fill the 128 rows of a tensor-memory CTA (query tokens x heads
// of a kv-head's group) run on tcgen05 (an E4M3 cache: head_dim 128 only).
// Shorter ones (a few draft tokens) leave most of those rows empty, yet the
// tcgen05 kernel still wins while its CTAs fill a wave (two per SM) and each
// kv-head has at least 8 rows (measured on B200: 8 draft tokens x 8 heads for
// 64 sequences, 313 -> 275 us with a bf16 cache and 404 -> 259 us with E4M3,
// where the mma.sync kernel widens every code in each of its four warps);
// with fewer CTAs or rows they run on the 64-row mma.sync kernel. When the
// CTAs (query tiles x kv-heads x sequences) cannot fill a wave of the
// tcgen05 kernel, or about four waves of three mma.sync CTAs per SM, the
// tiles of each CTA are cut into parts of at least 256 tokens (16 tiles, whole
// steps of the kernel) handled by separate CTAs and merged by a combine kernel.
struct PrefillPlan {
  bool tc;                  // tcgen05 kernel (rows on M), else mma.sync
  int32_t q_tiles, partition_tiles, max_parts;
};

PrefillPlan make_prefill_plan(int32_t num_seqs, int32_t num_kv_heads, int32_t group,
                              int32_t head_dim, int32_t max_query_len, int32_t max_context_len,
                              bool fp8) {
  PrefillPlan p{};
  const int64_t rows = static_cast<int64_t>(max_query_len) * group;

  // query tokens per CTA: tcgen05 128 rows per group, two groups once the
  // chunks fill 256 rows; mma.sync 64 rows
  const int32_t qt_tc = (rows >= 256 ? 256 : 128) / group;
  const int64_t tc_ctas = static_cast<int64_t>(num_seqs) * num_kv_heads *
                          ((max_query_len + qt_tc - 1) / qt_tc);
  p.tc = (!fp8 || head_dim == 128) &&
         (rows >= 128 || (rows >= 8 && tc_ctas >= 2LL * sm_count()));
  const int32_t qt = p.tc ? qt_tc : prefill_tokens_per_cta(group);
  p.q_tiles = (max_query_len + qt - 1) / qt;
  const int32_t max_tiles = std::max<int32_t>(1, (max_context_len + 15) / 16);
  p.partition_tiles = max_tiles;
  p.max_parts = 1;
  const int64_t ctas = static_cast<int64_t>(p.q_tiles) * num_kv_heads * num_seqs;
  // CTAs wanted: tcgen05 splits below half a wave (one CTA of two groups, or
  // two of one group, per SM) up to a wave - measured on B200, 64 CTAs of
  // 4 x 128-token chunks 325 -> 247 us, while 128 CTAs of one 512-token
  // chunk lost (326 -> 354 us); mma.sync about four waves of three per SM
  const int64_t wave = (rows >= 256 ? 1LL : 2LL) * sm_count();
  const int64_t want = p.tc ? wave : 4LL * sm_count() * 3;
  if (ctas >= (p.tc ? (wave + 1) / 2 : want) || max_tiles < 32) return p;
  const int64_t by_work = (want + ctas - 1) / ctas;
  const int32_t parts = static_cast<int32_t>(std::min<int64_t>(by_work, max_tiles / 16));
  if (parts <= 1) return p;
  // whole steps of the kernel: 4 tiles (64 tokens), 8 for the tcgen05 kernel
  // with two row groups (128 tokens)
  const int32_t step_tiles = p.tc && rows >= 256 ? 8 : 4;
  int32_t pt = (max_tiles + parts - 1) / parts;
  pt = (pt + step_tiles - 1) / step_tiles * step_tiles;
  p.partition_tiles = pt;
  p.max_parts = (max_tiles + pt - 1) / pt;
  return p;
}

size_t prefill_workspace_bytes(const PrefillPlan& p, int32_t num_tokens, int32_t num_heads,
                               int32_t head_dim) {
  if (p.max_parts <= 1) return kHeaderBytes;
  const size_t rows = static_cast<size_t>(num_tokens) * num_heads * p.max_parts;
  return align256(kHeaderBytes + rows * sizeof(float2)) + rows * head_dim * sizeof(float);
}

}  // namespace
}  // namespace paged

extern "C" {

PA_API size_t pa_chunked_prefill_workspace_size(int32_t num_seqs, int32_t num_tokens,
                                                int32_t num_heads, int32_t num_kv_heads,
                                                int32_t head_dim, int32_t max_query_len,
                                                int32_t max_context_len, pa_dtype cache_dtype) {
  if (num_seqs < 0 || num_tokens < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_query_len < 0 || max_context_len < 0 || num_heads % num_kv_heads != 0 ||
      (cache_dtype != PA_F16 && cache_dtype != PA_BF16 && cache_dtype != PA_FP8_E4M3))
    return 0;
  const PrefillPlan p = make_prefill_plan(num_seqs, num_kv_heads, num_heads / num_kv_heads,
                                          head_dim, max_query_len, max_context_len,
                                          cache_dtype == PA_FP8_E4M3);
  return prefill_workspace_bytes(p, num_tokens, num_heads, head_dim);
}

PA_API pa_status pa_chunked_prefill(void* out, const void* query, const int32_t* cu_query_lens,
                                    int32_t num_tokens, int32_t max_query_len,
                                    const void* key_cache, const void* value_cache,
                                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    const int32_t* context_lens, int32_t max_context_len,
                                    int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t block_size, int64_t num_blocks,
                                    float scale, pa_dtype q_dtype, pa_dtype cache_dtype,
                                    const float* k_scale, const float* v_scale,
                                    void* workspace, size_t workspace_bytes,
                                    pa_stream_t stream) {
  clear_error();
  if (num_tokens < 0 || max_query_len < 0 || num_seqs < 0 || num_heads <= 0 ||
      num_kv_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: negative or zero size");
  if (num_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: num_heads %% num_kv_heads != 0");
  const int32_t group = num_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8)
    return fail(PA_ERR_UNSUPPORTED, "chunked_prefill: query group %d not in {1,2,4,8}", group);
  if (!shape_supported(head_dim, block_size))
    return fail(PA_ERR_UNSUPPORTED, "chunked_prefill: head_dim %d / block_size %d unsupported",
                head_dim, block_size);
  if (q_dtype != PA_F16 && q_dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "chunked_prefill: query must be f16 or bf16");
  if (cache_dtype != q_dtype && cache_dtype != PA_FP8_E4M3)
    return fail(PA_ERR_UNSUPPORTED,
                "chunked_prefill: cache dtype must equal query dtype or be e4m3");
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (fp8 != (k_scale != nullptr) || fp8 != (v_scale != nullptr))
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: k_scale/v_scale required exactly for e4m3");
  if (num_blocks * block_size > INT32_MAX)
    return fail(PA_ERR_UNSUPPORTED, "chunked_prefill: pool rows exceed 2^31");
  if (num_seqs > 65535 || num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED, "chunked_prefill: more than 65535 sequences or kv-heads");
  if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "chunked_prefill: scale is not finite");
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < kHeaderBytes)
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: workspace missing, small or misaligned");
  if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens ||
      !cu_query_lens)
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: null pointer");
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) ||
      !aligned(value_cache, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4) ||
      !aligned(cu_query_lens, 4) || (k_scale && !aligned(k_scale, 4)) ||
      (v_scale && !aligned(v_scale, 4)))
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: misaligned pointer");

  CUtensorMap kmap, vmap;
  const PrefillPlan plan =
      make_prefill_plan(num_seqs, num_kv_heads, group, head_dim, max_query_len,
                        max_context_len, fp8);
  const bool tc = plan.tc;   // the tcgen05 kernel takes one-segment boxes
  const size_t need = prefill_workspace_bytes(plan, num_tokens, num_heads, head_dim);
  if (workspace_bytes < need)
    return fail(PA_ERR_INVALID_ARG, "chunked_prefill: workspace %zu bytes < %zu needed",
                workspace_bytes, need);
  const int elem = elem_bytes(cache_dtype);
  pa_status st = encode_cache_map(&kmap, key_cache, num_blocks, block_size, num_kv_heads,
                                  head_dim, elem, tc);
  if (st == PA_OK)
    st = encode_cache_map(&vmap, value_cache, num_blocks, block_size, num_kv_heads, head_dim,
                          elem, tc);
  if (st != PA_OK) return st;
  PrefillArgs a{};
  a.out = out;
  a.query = query;
  a.cu_query_lens = cu_query_lens;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.err = reinterpret_cast<int32_t*>(workspace) + kWordError;
  a.diag = reinterpret_cast<int32_t*>(workspace) + kWordDiag;
  a.num_blocks = num_blocks;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.ctx_limit = std::min<int64_t>(max_context_len,
                                  static_cast<int64_t>(max_blocks_per_seq) * block_size);
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_tiles = plan.q_tiles;
  a.partition_tiles = plan.partition_tiles;
  a.max_parts = plan.max_parts;
  take_injection(&a.skip_tile, &a.wait_limit_ns);
  if (plan.max_parts > 1) {
    const size_t rows = static_cast<size_t>(num_tokens) * num_heads * plan.max_parts;
    a.ws_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + kHeaderBytes);
    a.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                      align256(kHeaderBytes + rows * sizeof(float2)));
  }
  const int qd = q_dtype == PA_F16 ? kF16 : kBF16;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const int cd = fp8 ? kE4M3 : qd;
  const cudaError_t e =
      tc ? launch_prefill_tc(a, kmap, vmap, qd, cd, head_dim, group, max_query_len, cs)
         : launch_prefill(a, kmap, vmap, qd, cd, head_dim, group, max_query_len, cs);
  return cuda_status(e, "chunked_prefill");
}

}  // extern "C"
