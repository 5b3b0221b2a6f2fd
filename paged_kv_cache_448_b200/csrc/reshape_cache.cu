// reshape_cache.cu — scatter one step's new K/V rows into the paged cache.
//
// Token n's rows key[n][h][:] / value[n][h][:] go to physical slot
// slot_mapping[n] = block * block_size + offset of the cache
// [num_blocks, block_size, num_kv_heads, head_dim] ("vLLM推理引擎架构：
// PagedAttention机制与高吞吐推理" §2.2 layout; "Paged KVCache：大模型推理显存
// 管理优化方案" §2.3 address translation, page size in tokens). For an FP8
// cache each element is divided by its kv-head's fp32 scale (one IEEE fp32
// division) and rounded once to E4M3, nearest even, saturating
// ("大模型推理KV Cache内存管理与PagedAttention分页显存实战", FP8 KV cache).
//
// One thread moves one 16-byte chunk of input (8 elements) of K and the same
// chunk of V; a warp covers two or four whole rows, so loads and stores are
// 128-bit and coalesced. Element offsets are 64-bit.
#include "decode_args.h"
#include "device_common.cuh"

namespace paged {

template <int D>
__global__ void __launch_bounds__(256)
    reshape_copy16(const uint4* __restrict__ key, const uint4* __restrict__ value,
                   uint4* __restrict__ kc, uint4* __restrict__ vc,
                   const int32_t* __restrict__ slots, int32_t num_tokens, int32_t hkv,
                   int64_t pool_slots, int32_t* err) {
  constexpr int CPR = D / 8;  // 16-byte chunks per head row
  // The next kernel may be scheduled now; one that reads the cache waits for
  // this grid's completion (griddepcontrol.wait) before it does.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_token = static_cast<int64_t>(hkv) * CPR;
  if (i >= num_tokens * per_token) return;
  const int64_t n = i / per_token, r = i % per_token;
  const int64_t slot = slots[n];
  if (slot < 0) return;
  if (slot >= pool_slots) {
    report(err, kErrBadSlot);
    return;
  }
  const int64_t dst = slot * per_token + r;
  kc[dst] = key[i];
  vc[dst] = value[i];
}

template <class KF, int D>
__global__ void __launch_bounds__(256)
    reshape_quant_e4m3(const uint4* __restrict__ key, const uint4* __restrict__ value,
                       uint2* __restrict__ kc, uint2* __restrict__ vc,
                       const int32_t* __restrict__ slots, int32_t num_tokens, int32_t hkv,
                       int64_t pool_slots, const float* __restrict__ k_scale,
                       const float* __restrict__ v_scale, int32_t* err) {
  constexpr int CPR = D / 8;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_token = static_cast<int64_t>(hkv) * CPR;
  if (i >= num_tokens * per_token) return;
  const int64_t n = i / per_token, r = i % per_token;
  const int h = static_cast<int>(r / CPR);
  const int64_t slot = slots[n];
  if (slot < 0) return;
  if (slot >= pool_slots) {
    report(err, kErrBadSlot);
    return;
  }
  auto quant = [](uint4 x, float s) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = cvt2(KF{}, w[j]);
      const float2 q = make_float2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
      const uint32_t b = __nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
      o[j / 2] |= (b & 0xffffu) << (16 * (j % 2));
    }
    return make_uint2(o[0], o[1]);
  };
  const int64_t dst = slot * per_token + r;
  kc[dst] = quant(key[i], k_scale[h]);
  vc[dst] = quant(value[i], v_scale[h]);
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache,
                                     void* value_cache, const int32_t* slot_mapping,
                                     int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t block_size, int64_t num_blocks, int kv_dtype,
                                     int cache_dtype, const float* k_scale, const float* v_scale,
                                     int32_t* err, cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int64_t threads = static_cast<int64_t>(num_tokens) * num_kv_heads * (head_dim / 8);
  const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
  const int64_t pool_slots = num_blocks * block_size;
  auto k = static_cast<const uint4*>(key);
  auto v = static_cast<const uint4*>(value);
  if (cache_dtype == kv_dtype) {
    auto kc = static_cast<uint4*>(key_cache);
    auto vc = static_cast<uint4*>(value_cache);
    if (head_dim == 64)
      reshape_copy16<64><<<grid, 256, 0, stream>>>(k, v, kc, vc, slot_mapping, num_tokens,
                                                     num_kv_heads, pool_slots, err);
    else
      reshape_copy16<128><<<grid, 256, 0, stream>>>(k, v, kc, vc, slot_mapping, num_tokens,
                                                      num_kv_heads, pool_slots, err);
  } else {
    auto kc = static_cast<uint2*>(key_cache);
    auto vc = static_cast<uint2*>(value_cache);
#define PAGED_Q(KF, d)                                                                       \
  reshape_quant_e4m3<KF, d><<<grid, 256, 0, stream>>>(k, v, kc, vc, slot_mapping, num_tokens, \
                                                      num_kv_heads, pool_slots, k_scale,     \
                                                      v_scale, err)
    if (kv_dtype == kF16 && head_dim == 64) PAGED_Q(F16, 64);
    else if (kv_dtype == kF16) PAGED_Q(F16, 128);
    else if (head_dim == 64) PAGED_Q(BF16, 64);
    else PAGED_Q(BF16, 128);
#undef PAGED_Q
  }
  return cudaGetLastError();
}

}  // namespace paged
