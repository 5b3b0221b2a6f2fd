// decode_dispatch.cuh — choose the consumer and instantiate the decode kernel
// for every supported (head_dim, query group) of one dtype pair (the block
// size is a run-time parameter of the kernel):
// query groups of 1-2 heads run on the CUDA cores, groups of 4-8 heads
// (grouped-query attention) on the tensor cores. Each comes in two CTA widths:
// 4 warps, and 2 warps with half the ring for short partitions (more CTAs per
// SM, so more units overlap their start-up).
#pragma once

#include "consumer_mma.cuh"
#include "consumer_simt.cuh"

namespace paged {

template <class QF, class CF>
cudaError_t dispatch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int D, int G, int warps, cudaStream_t st) {
#define PAGED_CASE(d, g, C)                                                      \
  if (D == d && G == g)                                                          \
    return warps == 2 ? launch_decode<C<QF, CF, d, g>, 2>(a, kmap, vmap, st)     \
                      : launch_decode<C<QF, CF, d, g>, 4>(a, kmap, vmap, st);
#define PAGED_CASES(d)                                               \
  PAGED_CASE(d, 1, SimtConsumer) PAGED_CASE(d, 2, SimtConsumer) \
  PAGED_CASE(d, 4, MmaConsumer) PAGED_CASE(d, 8, MmaConsumer)
  if (warps != 2 && warps != 4) return cudaErrorNotSupported;
  PAGED_CASES(64)
  PAGED_CASES(128)
#undef PAGED_CASES
#undef PAGED_CASE
  return cudaErrorNotSupported;
}

}  // namespace paged
