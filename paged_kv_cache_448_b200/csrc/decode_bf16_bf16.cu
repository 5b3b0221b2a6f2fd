// Decode kernels for query dtype BF16, cache dtype BF16 (all head_dim, query groups and CTA widths).
#include "decode_dispatch.cuh"

namespace paged {
cudaError_t decode_bf16_bf16(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                        int head_dim, int group, int warps, cudaStream_t stream) {
  return dispatch_decode<BF16, BF16>(a, kmap, vmap, head_dim, group, warps, stream);
}
}  // namespace paged
