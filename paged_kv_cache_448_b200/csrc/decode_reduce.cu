// decode_reduce.cu — combine the per-partition partial results of a split
// decode. Partition p of a sequence left (m_p, l_p, o_p) with o_p already
// normalised by l_p (base-2 units); the exact combination is
//   M = max_p m_p,  w_p = l_p * 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p
// (the same rescaling the online softmax applies between blocks).
// Launched right behind the decode kernel (programmatic dependent launch); it
// waits for the decode grid before reading the partials.
#include <math_constants.h>

#include "decode_args.h"
#include "decode_kernel.cuh"
#include "device_common.cuh"

namespace paged {

template <class QF, int D>
__global__ void __launch_bounds__(128) paged_decode_reduce(const DecodeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.y, h = blockIdx.x * 4 + warp;
  if (h >= a.num_heads) return;
  int ctx = a.context_lens[s];
  ctx = ctx < 0 ? 0 : (ctx > a.ctx_limit ? a.ctx_limit : ctx);
  const int nblk = (ctx + a.block_size - 1) / a.block_size;
  const int parts = min((nblk + a.partition_blocks - 1) / a.partition_blocks, a.max_parts);
  if (parts <= 1) return;  // written directly by the decode kernel
  const int64_t row = static_cast<int64_t>(s) * a.num_heads + h;
  const float2* ml = a.ws_ml + row * a.max_parts;
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  float M = -CUDART_INF_F, L = 0.f;
  const float* o = a.ws_o + row * a.max_parts * D;
  // kBatch partitions at a time, all their loads issued before any is used
  // (one L2 round trip per batch, not per partition), with a running maximum
  // (the sums so far rescaled when a batch raises it). A partition that saw
  // no token (or gave up) has no weight, and its o was never written: its
  // values, whatever they are, are selected away, never multiplied.
  constexpr int kBatch = 16;
  for (int p0 = 0; p0 < parts; p0 += kBatch) {
    float2 v[kBatch];
    float ov[kBatch][PER];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int p = p0 + u;
      v[u] = make_float2(-CUDART_INF_F, 0.f);
#pragma unroll
      for (int i = 0; i < PER; ++i) ov[u][i] = 0.f;
      if (p < parts) {  // the same in every lane
        v[u] = ml[p];
#pragma unroll
        for (int i = 0; i < PER; ++i) ov[u][i] = o[p * D + lane + 32 * i];
      }
    }
    bool use[kBatch];
    float bm = M;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      use[u] = p0 + u < parts && v[u].x != -CUDART_INF_F && v[u].y > 0.f;
      if (use[u]) bm = fmaxf(bm, v[u].x);
    }
    if (bm > M) {  // the same in every lane (the loads are broadcasts)
      const float f = M == -CUDART_INF_F ? 0.f : exp2f(M - bm);
      L *= f;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] *= f;
      M = bm;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const float w = use[u] ? v[u].y * exp2f(v[u].x - M) : 0.f;
      L += w;
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = use[u] ? fmaf(w, ov[u][i], acc[i]) : acc[i];
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) store_out(QF{}, a.out, row * D + lane + 32 * i, acc[i] * inv);
}

cudaError_t launch_reduce(const DecodeArgs& a, int q_dtype, int head_dim, cudaStream_t stream) {
  const dim3 grid((a.num_heads + 3) / 4, a.num_seqs);
  if (q_dtype == kF16 && head_dim == 64)
    return launch_pdl(paged_decode_reduce<F16, 64>, grid, 128, 0, stream, a);
  if (q_dtype == kF16 && head_dim == 128)
    return launch_pdl(paged_decode_reduce<F16, 128>, grid, 128, 0, stream, a);
  if (q_dtype == kBF16 && head_dim == 64)
    return launch_pdl(paged_decode_reduce<BF16, 64>, grid, 128, 0, stream, a);
  if (q_dtype == kBF16 && head_dim == 128)
    return launch_pdl(paged_decode_reduce<BF16, 128>, grid, 128, 0, stream, a);
  return cudaErrorNotSupported;
}

}  // namespace paged
