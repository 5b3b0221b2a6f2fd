// Decode kernels for query dtype F16, cache dtype F16 (all head_dim, query groups and CTA widths).
#include "decode_dispatch.cuh"

namespace paged {
cudaError_t decode_f16_f16(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                        int head_dim, int group, int warps, cudaStream_t stream) {
  return dispatch_decode<F16, F16>(a, kmap, vmap, head_dim, group, warps, stream);
}
}  // namespace paged
