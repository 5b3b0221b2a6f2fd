/*
 * paged.h — C ABI of libpaged: paged KV-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * Sources this interface follows (web pages, cited by title and section):
 *   [P1] "vLLM框架中的KV cache优化与PagedAttention机制详解" (trdm.cn)
 *   [P2] "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" (maplevalley.com.cn)
 *   [P3] "Paged KVCache：大模型推理显存管理优化方案" (intelliparadigm.com)
 *   [P4] "大模型推理KV Cache内存管理与PagedAttention分页显存实战" (yunthe.com)
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Device pointers are plain CUDA device addresses owned by the caller; the
 *    library never allocates, frees or retains device memory. Host pointers are
 *    read (or written) only during the call.
 *  - Every device call is asynchronous on `stream` and performs no device
 *    synchronisation. Argument errors are detected on the host before any
 *    launch; the call then returns a non-zero status, launches nothing and
 *    records a message readable with pa_last_error() (thread-local).
 *  - Launch failures return PA_ERR_CUDA with the CUDA error string.
 *  - Every device pointer must be 16-byte aligned; rows of head_dim elements
 *    must be a multiple of 16 bytes (always true for the supported head_dim).
 *  - Integer tables (block tables, context lengths, slot mappings) are int32.
 *    All element offsets are formed in 64 bits, so caches larger than 2^31
 *    elements are fine.
 *  - Caches are laid out [num_blocks, block_size, num_kv_heads, head_dim]
 *    ([P2] §2.2 "Block管理器实现"; the per-head dimension is num_kv_heads,
 *    which equals num_heads for multi-head attention).
 */
#ifndef LIBPAGED_PAGED_H
#define LIBPAGED_PAGED_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same ABI as cudaStream_t; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* pa_stream_t;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, inconsistent shape */
  PA_ERR_UNSUPPORTED = 2, /* valid but not implemented: head_dim, block_size, group size, dtype pair */
  PA_ERR_OOM = 3,         /* host allocator: not enough free blocks (nothing was allocated) */
  PA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed; see pa_last_error() */
  PA_ERR_BAD_TABLE = 5    /* a block-table entry, slot or context length is out of range */
} pa_status;

typedef enum {
  PA_F16 = 0,      /* IEEE binary16 */
  PA_BF16 = 1,     /* bfloat16 */
  PA_FP8_E4M3 = 2  /* OCP FP8 E4M3 (bias 7, max finite 448, no infinities) */
} pa_dtype;

/* Thread-local description of the last failing call on this thread ("" if none). */
PA_API const char* pa_last_error(void);

/* ------------------------------------------------------------------------- */
/* reshape_and_cache: scatter one step's new K/V into the paged cache.        */
/* ------------------------------------------------------------------------- */
/*
 * For every token n in [0, num_tokens) with slot = slot_mapping[n] >= 0:
 *     blk = slot / block_size, off = slot % block_size
 *     key_cache  [blk][off][h][:] = enc(key  [n][h][:], k_scale[h])
 *     value_cache[blk][off][h][:] = enc(value[n][h][:], v_scale[h])     for all h
 * Tokens with a negative slot are skipped (padding). The slot is the physical
 * address of a token: physical block * block_size + offset inside the block,
 * the address translation of [P3] §2.3 "地址转换流程" with the page size
 * counted in tokens ([P4] "Block大小为16"), as in [P1] §5.1.
 *
 * key, value      device, [num_tokens, num_kv_heads, head_dim] of kv_dtype (F16 or BF16).
 * key_cache,      device, [num_blocks, block_size, num_kv_heads, head_dim] of cache_dtype.
 *   value_cache
 * slot_mapping    device int32 [num_tokens]; slots must be unique (caller's duty) and
 *                 < num_blocks * block_size.
 * cache_dtype     == kv_dtype: the bytes are copied unchanged.
 *                 == PA_FP8_E4M3: enc(x, s) = e4m3_rne_satfinite((float)x / s), one IEEE
 *                 fp32 division and one rounding (FP8 KV storage, [P4] "FP8 KV Cache量化").
 * k_scale,        device fp32 [num_kv_heads] (FP8 cache only; NULL otherwise).
 *   v_scale
 * Errors: PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED on the host before launch. A slot
 * outside the pool is not written (the kernel checks every slot).
 * head_dim in {64, 128}; block_size in {16, 32}.
 */
PA_API pa_status pa_reshape_and_cache(const void* key, const void* value,
                               void* key_cache, void* value_cache,
                               const int32_t* slot_mapping, int32_t num_tokens,
                               int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int64_t num_blocks,
                               pa_dtype kv_dtype, pa_dtype cache_dtype,
                               const float* k_scale, const float* v_scale,
                               pa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* decode: one query token per sequence against its paged context.            */
/* ------------------------------------------------------------------------- */
/*
 * The kernel of [P2] §2.3 "PagedAttention Kernel": for each sequence s and query
 * head h, with kvh = h / (num_heads / num_kv_heads) (contiguous query groups) and
 * n = context_lens[s]:
 *     K_s[t] = key_cache  [block_tables[s][t / block_size]][t % block_size][kvh][:]
 *     V_s[t] = value_cache[block_tables[s][t / block_size]][t % block_size][kvh][:]
 *     out[s][h][:] = sum_t softmax_t(scale * query[s][h]·K_s[t]) * V_s[t],  t < n
 * i.e. the logical->physical block translation of [P1] §5.1 followed by
 * attention accumulated across blocks. n == 0 gives an all-zero output row.
 * For an FP8 cache the stored codes are dequantised as code * k_scale[kvh]
 * (keys) and code * v_scale[kvh] (values).
 *
 * out             device [num_seqs, num_heads, head_dim] of q_dtype (written).
 * query           device [num_seqs, num_heads, head_dim] of q_dtype (F16 or BF16).
 * key_cache,      device [num_blocks, block_size, num_kv_heads, head_dim] of cache_dtype
 *   value_cache   (cache_dtype == q_dtype, or PA_FP8_E4M3).
 * block_tables    device int32 [num_seqs, max_blocks_per_seq]; entries past
 *                 ceil(n / block_size) are never read (any value, e.g. -1).
 * context_lens    device int32 [num_seqs].
 * max_context_len host int, >= every context_lens[s]; sizes the launch.
 * scale           softmax scale (e.g. 1/sqrt(head_dim)).
 * k_scale,        device fp32 [num_kv_heads] for an FP8 cache, else NULL.
 *   v_scale
 * partition_tokens 0 = choose automatically; otherwise the context is cut into
 *                 partitions of this many tokens (a multiple of block_size) that
 *                 are processed independently and combined by a second kernel.
 *                 A value >= max_context_len forces the single-pass path.
 * workspace       device scratch of at least pa_decode_workspace_size(...) bytes,
 *                 caller-owned, 256-byte aligned. Its first 256 bytes hold an error
 *                 word (see pa_decode_check); the rest holds per-partition partial
 *                 results. Two calls in flight at once must not share it.
 * Supported: head_dim in {64, 128}; block_size in {16, 32};
 *            num_heads / num_kv_heads in {1, 2, 4, 8}.
 * Run-time table errors (an entry outside [0, num_blocks), a context length above
 * max_context_len or above max_blocks_per_seq * block_size) never cause an
 * out-of-range access: the offending block reads as zeros, the context is
 * clipped, and the error word is set for pa_decode_check to report.
 */
PA_API pa_status pa_decode(void* out, const void* query,
                    const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context_len,
                    int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t block_size, int64_t num_blocks,
                    float scale, pa_dtype q_dtype, pa_dtype cache_dtype,
                    const float* k_scale, const float* v_scale,
                    int32_t partition_tokens,
                    void* workspace, size_t workspace_bytes,
                    pa_stream_t stream);

/*
 * pa_decode without a workspace argument, for callers that cannot allocate
 * device memory: a serving loop that forbids cudaMalloc once it is running
 * (cudaMalloc synchronises the device and stalls every stream), a process whose
 * device memory is already claimed by another framework's caching allocator,
 * or a host-language binding that has no device allocation API. The pages
 * describe nothing like it; it exists only for those callers.
 *
 * Same arguments, meaning and results as pa_decode, minus workspace and
 * workspace_bytes. The scratch is a 32 MiB file-scope device array inside this
 * library, held on every GPU that loads the library until the process exits.
 * The call allocates and frees nothing. Sizes whose partitioned path needs more
 * than 32 MiB (pa_decode_workspace_size > 32 MiB) return PA_ERR_UNSUPPORTED
 * without launching; use pa_decode for them.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current, and again only if the device's context
 * was replaced, e.g. after cudaDeviceReset); make that first call before any
 * stream capture. Every call shares the one array and leaves its contents
 * behind: two calls whose kernels overlap on the GPU (e.g. on two streams)
 * race on it and give wrong results, so serialise them. Nothing in it needs
 * clearing between calls: every partial result a call combines is written by
 * that call, and a work unit whose pipeline wait gave up writes an empty
 * partial (or zeros) rather than leaving another call's data to be combined.
 * Table errors and waits that gave up are made harmless as in pa_decode and
 * recorded in the array's error word: read them with pa_decode_noalloc_check.
 */
PA_API pa_status pa_decode_noalloc(void* out, const void* query,
                    const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context_len,
                    int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t block_size, int64_t num_blocks,
                    float scale, pa_dtype q_dtype, pa_dtype cache_dtype,
                    const float* k_scale, const float* v_scale,
                    int32_t partition_tokens, pa_stream_t stream);

/*
 * pa_decode_check for pa_decode_noalloc: synchronises `stream`, then reads and
 * clears the error word of this device's static scratch. Same results as
 * pa_decode_check (PA_OK, PA_ERR_BAD_TABLE, or PA_ERR_CUDA for a wait that
 * gave up, with the first failure's record in pa_last_error()). It allocates
 * nothing either. The word collects every pa_decode_noalloc call on this
 * device since the last check.
 */
PA_API pa_status pa_decode_noalloc_check(pa_stream_t stream);

/*
 * Attention of several query tokens per sequence over the paged cache
 * (chunked prefill; verification of several draft tokens). [P2] §2.3's
 * interface takes a query tensor; here it has more rows than sequences:
 * rows cu_query_lens[s] .. cu_query_lens[s+1]-1 of query are the last
 * q_len_s = cu_query_lens[s+1] - cu_query_lens[s] positions of sequence s,
 * p_i = context_lens[s] - q_len_s + i, whose keys and values are already in
 * the cache (pa_reshape_and_cache). Row i attends to the tokens t <= p_i of
 * its sequence (the causal rule of autoregressive attention), query head h
 * to kv-head h / (num_heads / num_kv_heads), with softmax scale `scale`.
 * out, query      device [num_tokens, num_heads, head_dim] of q_dtype (f16 or bf16).
 * cache_dtype     q_dtype, or PA_FP8_E4M3 with k_scale / v_scale (device float
 *                 [num_kv_heads], as written by pa_reshape_and_cache; null otherwise):
 *                 logits use scale * k_scale[kv-head], outputs are multiplied by
 *                 v_scale[kv-head].
 * cu_query_lens   device int32 [num_seqs + 1], cu[0] = 0, cu[num_seqs] = num_tokens.
 * max_query_len   host int >= every q_len_s; sizes the launch.
 * key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens,
 * max_context_len, num_blocks: as in pa_decode (context_lens include the
 * query tokens).
 * workspace       >= pa_chunked_prefill_workspace_size(...) bytes, 256-byte aligned,
 *                 zeroed once (pa_workspace_init). Launches whose CTAs cannot
 *                 fill the GPU (few sequences or kv-heads) split each key range
 *                 into parts combined by a second kernel, with partial results
 *                 here. Its error word reports, through pa_decode_check, table
 *                 entries outside the pool (read as zeros), clipped context
 *                 lengths, and a query longer than its context (bit 16; those
 *                 rows are written as zeros).
 * Supported: head_dim in {64, 128}; block_size in {16, 32}; group in {1, 2, 4, 8};
 *            at most 65535 sequences and kv-heads.
 * Errors (returned before any launch, nothing written): PA_ERR_INVALID_ARG for
 * negative sizes, num_heads % num_kv_heads != 0, a non-finite scale, null or
 * misaligned pointers (16 bytes for tensors, 4 for tables and scales), scales
 * given for a 16-bit cache or missing for E4M3, and a workspace that is
 * missing, misaligned or smaller than needed; PA_ERR_UNSUPPORTED for other
 * dtypes, head_dim, block_size or group; PA_ERR_CUDA for a failed launch.
 * Nothing to do (no sequences, tokens or query rows) returns PA_OK at once.
 */
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
                                    pa_stream_t stream);

/*
 * Bytes of workspace pa_chunked_prefill needs for these sizes and cache dtype
 * on the current device (256 when the key range is not split). Returns 0 for
 * invalid sizes.
 */
PA_API size_t pa_chunked_prefill_workspace_size(int32_t num_seqs, int32_t num_tokens,
                                                int32_t num_heads, int32_t num_kv_heads,
                                                int32_t head_dim, int32_t max_query_len,
                                                int32_t max_context_len, pa_dtype cache_dtype);

/*
 * Bytes of workspace pa_decode needs for these sizes and cache dtype on the
 * current device (the automatic partition choice depends on the device's SM
 * count and on the kernel the cache dtype and head_dim select).
 * Returns 0 for invalid sizes.
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t block_size,
                                int32_t max_context_len, int32_t partition_tokens,
                                pa_dtype cache_dtype);

/*
 * The partition length (tokens) pa_decode will use for these sizes and cache
 * dtype on the current device; a result >= max_context_len means the
 * single-pass path.
 */
PA_API int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                   int32_t head_dim, int32_t block_size,
                                   int32_t max_context_len, int32_t partition_tokens,
                                   pa_dtype cache_dtype);

/*
 * Synchronises `stream`, reads and clears the error word of `workspace`.
 * Returns PA_OK, or PA_ERR_BAD_TABLE if a previous pa_decode or
 * pa_chunked_prefill on this workspace met an out-of-range table entry or
 * context length or a query longer than its context, or PA_ERR_CUDA (a wait
 * that gave up, or a CUDA error). For a wait that gave up, pa_last_error()
 * names the first failure: its site (decode tile, multi-token tile or step,
 * FP8 decode tile), the CTA and the pipeline position where it stopped.
 */
PA_API pa_status pa_decode_check(void* workspace, pa_stream_t stream);

/*
 * Zero the error word of a fresh workspace (asynchronous on `stream`).
 * pa_decode never needs the rest of the workspace cleared.
 */
PA_API pa_status pa_workspace_init(void* workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * Test hook of the failure detection (no counterpart on the pages). Every
 * pipeline wait inside the decode and multi-token kernels is bounded by wall
 * time (1 s by default); a wait that runs out makes the kernel record the
 * failure, set the timeout bit of the error word, let its own loads and
 * tensor-core operations in flight complete, free its tensor memory and
 * return, leaving zeros (or an empty partial result) for the rows it could
 * not finish. Nothing faults, traps or hangs.
 * This call makes the NEXT pa_decode, pa_decode_noalloc or pa_chunked_prefill
 * made on the calling thread leave out the loads of one 16-token tile, `tile`
 * (counted from 0 within the key range of the launch's first work unit:
 * sequence 0, kv-head 0, first partition and query tile), and bound every wait
 * of that launch by wait_limit_ns instead. The wait for the left-out tile then
 * runs out and pa_decode_check / pa_decode_noalloc_check return PA_ERR_CUDA
 * with the failure record. The request is used up by that call; tile < 0
 * cancels a pending one. PA_ERR_INVALID_ARG if tile >= 0 and wait_limit_ns is 0.
 */
PA_API pa_status pa_inject_wait_timeout(int32_t tile, uint64_t wait_limit_ns);

/*
 * Copy whole blocks: for each pair i, block block_pairs[2i] of the source
 * caches is copied byte for byte to block block_pairs[2i+1] of the destination
 * caches (K, and V when the value caches are given). One block of one cache is
 * block_bytes contiguous bytes (block_size * num_kv_heads * head_dim * elem).
 * Two uses:
 *  - copy-on-write of a shared block (source and destination in the same
 *    cache), after pa_alloc_copy_on_write; [P4] shares prefix blocks among
 *    requests under a reference count;
 *  - migration between GPU memory and a host pool ([P3] "Paged KVCache：大模型
 *    推理显存管理优化方案" §5 Hybrid Cache: GPU memory, then CPU memory, then
 *    disk; [P4]'s swap_space): one side may be pinned host memory
 *    (cudaHostAlloc / cudaHostRegister), which the kernel reads or writes through
 *    its mapped device address. Pageable host memory is rejected.
 * src_key_cache, src_value_cache  [num_src_blocks, ...] device or pinned host
 * dst_key_cache, dst_value_cache  [num_dst_blocks, ...] device or pinned host
 *                 (value caches: both NULL to copy the key cache only)
 * block_pairs     int32 [num_pairs][2], device or pinned host; destination ids
 *                 distinct; with the same cache on both sides no destination
 *                 may also be a source (else the result is unspecified).
 * error_word      optional device int32: a pair with an id outside its pool is
 *                 skipped (nothing is read or written for it) and bit 1 is set.
 * block_bytes must be a positive multiple of 16 and every pointer 16-byte
 * aligned (4 for block_pairs / error_word). Asynchronous on `stream`.
 */
PA_API pa_status pa_copy_blocks(const void* src_key_cache, const void* src_value_cache,
                                void* dst_key_cache, void* dst_value_cache,
                                const int32_t* block_pairs, int32_t num_pairs, int64_t block_bytes,
                                int64_t num_src_blocks, int64_t num_dst_blocks,
                                int32_t* error_word, pa_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Block content hashes for prefix caching (host only).                        */
/* ------------------------------------------------------------------------- */

/* SHA-256 (FIPS 180-4) of n bytes. */
PA_API pa_status pa_sha256(const void* data, int64_t n, uint8_t out[32]);
/* Hash of one block: SHA-256 of the parent block's 32-byte hash (32 zero bytes
 * when parent is NULL: the first block of a prompt) followed by the block's
 * num_tokens token ids as little-endian int32. [P4] recognises shareable
 * prefix blocks by hash matching without naming a hash; chaining through the
 * parent makes equal hashes mean equal whole prefixes. */
PA_API pa_status pa_block_hash(const uint8_t* parent, const int32_t* tokens, int32_t num_tokens,
                               uint8_t out[32]);
/* Chained hashes of the floor(num_tokens / block_size) full blocks of a
 * prompt into hashes_out[32 * j]; a partial last block has none. */
PA_API pa_status pa_prompt_block_hashes(const int32_t* tokens, int64_t num_tokens,
                                        int32_t block_size, uint8_t* hashes_out);

/* ------------------------------------------------------------------------- */
/* Host block allocator (no device memory; produces integer tables only).      */
/* ------------------------------------------------------------------------- */
/*
 * The free list of [P2] §2.2 "Block管理器实现": allocate(n) takes the first n
 * free ids or fails with PA_ERR_OOM leaving the list untouched; free appends
 * released ids to the back. Blocks shared by several sequences (shared
 * prompt prefix) carry a reference count ([P4] "通过引用计数管理生命周期"):
 * share() adds a reference, free() drops one, and a block returns to the
 * free list when its count reaches zero.
 */
typedef struct pa_alloc pa_alloc;

/* initial_free_order: NULL for 0..num_blocks-1, else a permutation of it (e.g. a
 * seeded shuffle) that becomes the initial free list, front first. */
PA_API pa_status pa_alloc_create(int64_t num_blocks, const int32_t* initial_free_order, pa_alloc** out);
PA_API void pa_alloc_destroy(pa_alloc* a);
/* All-or-nothing: on PA_ERR_OOM nothing changes. n == 0 is a no-op. */
PA_API pa_status pa_alloc_allocate(pa_alloc* a, int32_t n, int32_t* ids_out);
/* refcount++ of an allocated block; PA_ERR_INVALID_ARG if the block is free. */
PA_API pa_status pa_alloc_share(pa_alloc* a, int32_t id);
/* refcount-- of each id, in order; all ids are validated first (an id that is
 * free or listed more often than its refcount gives PA_ERR_INVALID_ARG and
 * changes nothing). */
PA_API pa_status pa_alloc_free(pa_alloc* a, const int32_t* ids, int32_t n);
/* Before a write into block `id`: with refcount 1, *id_out = id and
 * *must_copy = 0 (write in place). With refcount > 1 (shared), a fresh block
 * is taken from the head of the free list, one reference moves to it,
 * *id_out = that block and *must_copy = 1: the caller copies the contents
 * (pa_copy_blocks) and points its table entry at *id_out. The pages share
 * blocks under a reference count ([P4]) but give no write rule; this is the
 * reading taken. PA_ERR_OOM (nothing changes) when no block is free;
 * PA_ERR_INVALID_ARG for a free or unknown id. */
PA_API pa_status pa_alloc_copy_on_write(pa_alloc* a, int32_t id, int32_t* id_out,
                                        int32_t* must_copy);
/* Prefix caching ([P4] Prefix Caching: prefix blocks are reused across
 * requests, recognised by hash matching). hashes: n 32-byte block hashes
 * (pa_prompt_block_hashes), in prompt order. Each hash that names a cached
 * block takes a reference to it (a cached block whose references were all
 * freed is taken back out of the free list); every other hash gets a fresh
 * block from the head of the free list, registered under that hash (the
 * caller then fills it). ids_out[i] is the block of hash i; *num_hits counts
 * the hashes that found a block. PA_ERR_OOM (nothing changes) when the fresh
 * blocks do not fit. A block keeps its hash after it is freed and loses it
 * when it is handed out again from the head of the free list. */
PA_API pa_status pa_alloc_acquire_prefix(pa_alloc* a, const uint8_t* hashes, int32_t n,
                                         int32_t* ids_out, int32_t* num_hits);
/* Register the hash of an allocated block that has just become full (e.g. a
 * decode step filled it), replacing any hash it had. Nothing happens when the
 * hash names a block already. PA_ERR_INVALID_ARG for a free or unknown id. */
PA_API pa_status pa_alloc_register_hash(pa_alloc* a, int32_t id, const uint8_t* hash);
/* The block registered under a hash, or -1. */
PA_API int32_t pa_alloc_lookup(const pa_alloc* a, const uint8_t* hash);
PA_API int64_t pa_alloc_num_free(const pa_alloc* a);
PA_API int64_t pa_alloc_num_blocks(const pa_alloc* a);
/* Reference count of a block (0 = free), -1 for an id out of range. */
PA_API int32_t pa_alloc_refcount(const pa_alloc* a, int32_t id);
/* Copy the free list, front first, into ids_out (capacity cap); returns the
 * number of free blocks. */
PA_API int64_t pa_alloc_free_list(const pa_alloc* a, int32_t* ids_out, int64_t cap);

/*
 * Row-major block table [num_seqs, max_blocks_per_seq] from per-sequence id
 * lists; unused entries are set to -1. PA_ERR_INVALID_ARG if a list is longer
 * than max_blocks_per_seq.
 */
PA_API pa_status pa_build_block_table(const int32_t* const* seq_block_ids,
                               const int32_t* num_blocks_per_seq, int32_t num_seqs,
                               int32_t max_blocks_per_seq, int32_t* table_out);

/*
 * slots_out[i] = block_tables[seq][pos / block_size] * block_size + pos % block_size
 * with seq = seq_ids ? seq_ids[i] : i and pos = positions[i] ([P3] §2.3 address
 * translation, page size in tokens). pos < 0 gives slot -1 (padding token).
 * PA_ERR_BAD_TABLE if pos / block_size >= max_blocks_per_seq, the table entry is
 * negative, or the slot does not fit in int32; slots_out is then unspecified.
 * All arrays are host memory.
 */
PA_API pa_status pa_build_slot_mapping(const int32_t* block_tables, int32_t num_seqs,
                                int32_t max_blocks_per_seq, const int32_t* seq_ids,
                                const int32_t* positions, int32_t num_tokens,
                                int32_t block_size, int32_t* slots_out);

#ifdef __cplusplus
}
#endif

#endif /* LIBPAGED_PAGED_H */
