// decode_dispatch.cuh — choose the consumer and instantiate the decode kernel
// for every supported (head_dim, query group) of one dtype pair (the block
// size is a run-time parameter of the kernel):
// query groups of 1-2 heads run on the CUDA cores, groups of 4-8 heads
// (grouped-query attention) on the tensor cores.
#pragma once

#include "consumer_mma.cuh"
#include "consumer_simt.cuh"

namespace paged {

template <class QF, class CF>
cudaError_t dispatch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int D, int G, cudaStream_t st) {
#define PAGED_CASE(d, g, C) \
  if (D == d && G == g) return launch_decode<C<QF, CF, d, g>>(a, kmap, vmap, st);
#define PAGED_CASES(d)                                               \
  PAGED_CASE(d, 1, SimtConsumer) PAGED_CASE(d, 2, SimtConsumer) \
  PAGED_CASE(d, 4, MmaConsumer) PAGED_CASE(d, 8, MmaConsumer)
  PAGED_CASES(64)
  PAGED_CASES(128)
#undef PAGED_CASES
#undef PAGED_CASE
  return cudaErrorNotSupported;
}

}  // namespace paged
