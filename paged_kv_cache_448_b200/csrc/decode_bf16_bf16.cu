// Decode kernels for query dtype BF16, cache dtype BF16 (all head_dim and query groups).
#include "decode_dispatch.cuh"

namespace paged {
cudaError_t decode_bf16_bf16(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                        int head_dim, int group, cudaStream_t stream) {
  return dispatch_decode<BF16, BF16>(a, kmap, vmap, head_dim, group, stream);
}
}  // namespace paged
