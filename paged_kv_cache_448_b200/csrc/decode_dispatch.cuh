// decode_dispatch.cuh — choose the consumer and instantiate the decode kernel
// for every supported (head_dim, block_size, query group) of one dtype pair:
// query groups of 1-2 heads run on the CUDA cores, groups of 4-8 heads
// (grouped-query attention) on the tensor cores.
#pragma once

#include "consumer_mma.cuh"
#include "consumer_simt.cuh"

namespace paged {

template <class QF, class CF>
cudaError_t dispatch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int D, int BS, int G, cudaStream_t st) {
#define PAGED_CASE(d, bs, g, C) \
  if (D == d && BS == bs && G == g) return launch_decode<C<QF, CF, d, bs, g>>(a, kmap, vmap, st);
#define PAGED_CASES(d, bs)                                             \
  PAGED_CASE(d, bs, 1, SimtConsumer) PAGED_CASE(d, bs, 2, SimtConsumer) \
  PAGED_CASE(d, bs, 4, MmaConsumer) PAGED_CASE(d, bs, 8, MmaConsumer)
  PAGED_CASES(64, 16)
  PAGED_CASES(64, 32)
  PAGED_CASES(128, 16)
  PAGED_CASES(128, 32)
#undef PAGED_CASES
#undef PAGED_CASE
  return cudaErrorNotSupported;
}

}  // namespace paged
