// noalloc.cu — pa_decode_noalloc: decode with library-owned static scratch.
//
// pa_decode needs a caller-provided device workspace for its partitioned
// path. Some callers cannot provide one: a serving loop that forbids
// cudaMalloc after start-up (it synchronises the device and stalls other
// streams), a process whose device memory is already claimed by another
// framework's caching allocator, or a host-language binding with no device
// allocation API at all. For them the scratch lives here, in a file-scope
// __device__ array of fixed size that every GPU loading this library holds
// until the process exits. No allocation call of any kind is made.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "paged.h"
#include "status.h"

namespace paged {
namespace {

// Upper bound of the scratch a pa_decode_noalloc call may use.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB

// In host code this name is only a host-side stand-in for the device array;
// its device address comes from cudaGetSymbolAddress, per device.
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchSlot {
  void* ctx = nullptr;   // the context the address was resolved in
  void* addr = nullptr;  // device address of g_decode_scratch there
};
ScratchSlot g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_decode_scratch on the current device. Resolved once
// per device, with that device current, and again only when the device's
// current context changed (a cudaDeviceReset destroys the old context and
// with it the module holding the array).
pa_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "decode_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(PA_ERR_UNSUPPORTED, "decode_noalloc: device index %d", dev);
  auto current = [] {
    CUcontext c = nullptr;
    if (auto get = ctx_get_current()) get(&c);
    return static_cast<void*>(c);
  };
  void* ctx = current();  // null before the runtime made its context current
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch[dev];
  if (!slot.addr || !ctx || slot.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p)
      return fail(PA_ERR_CUDA, "decode_noalloc: cudaGetSymbolAddress failed: %s",
                  cudaGetErrorString(e));
    slot.addr = p;
    slot.ctx = current();  // the lookup made the device's context current
  }
  *out = slot.addr;
  return PA_OK;
}

}  // namespace
}  // namespace paged

extern "C" PA_API pa_status pa_decode_noalloc(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
    int32_t max_context_len, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int64_t num_blocks, float scale, pa_dtype q_dtype,
    pa_dtype cache_dtype, const float* k_scale, const float* v_scale, int32_t partition_tokens,
    pa_stream_t stream) {
  using namespace paged;
  clear_error();
  const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim,
                                               block_size, max_context_len, partition_tokens,
                                               cache_dtype);
  if (need == 0) return fail(PA_ERR_INVALID_ARG, "decode_noalloc: invalid sizes");
  if (need > kNoAllocScratchBytes)
    return fail(PA_ERR_UNSUPPORTED,
                "decode_noalloc: these sizes need %zu bytes of scratch but the static scratch "
                "holds %zu; use pa_decode with a caller-provided workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  pa_status st = scratch_address(&scratch);
  if (st != PA_OK) return st;
  // Every partial result the combine kernel reads is written by this call
  // (a unit whose wait gave up writes an empty partial), so nothing in the
  // scratch has to start at zero. Errors accumulate in the scratch's error
  // word until pa_decode_noalloc_check reads and clears it.
  return pa_decode(out, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                   context_lens, max_context_len, num_seqs, num_heads, num_kv_heads, head_dim,
                   block_size, num_blocks, scale, q_dtype, cache_dtype, k_scale, v_scale,
                   partition_tokens, scratch, kNoAllocScratchBytes, stream);
}

extern "C" PA_API pa_status pa_decode_noalloc_check(pa_stream_t stream) {
  using namespace paged;
  clear_error();
  void* scratch = nullptr;
  pa_status st = scratch_address(&scratch);
  if (st != PA_OK) return st;
  return pa_decode_check(scratch, stream);
}
