// decode_plan.cu — the work list of one decode launch, built on the device.
//
// A work unit is (sequence, kv-head, context partition). The plan orders the
// sequences by decreasing number of blocks (a counting sort), so units are
// handed out partition-major over that order: the first partitions of every
// sequence, then the second partitions of the sequences that have one, and so
// on — the longest remaining work is always started first, and a unit index u
// maps to (p, j, kv-head) through the prefix counts C[p] (units before
// partition slice p). It also zeroes the work counter the decode CTAs draw
// tickets from and the per-(sequence, kv-head) arrival counters of the
// partition combine. One CTA; it lets the decode grid launch right away
// (programmatic dependent launch) and only finishes once the previous kernel
// in the stream has completed, so the decode kernel, which waits for this
// grid, also sees everything that kernel wrote (the new cache rows).
#include <cub/block/block_scan.cuh>

#include "decode_args.h"
#include "device_common.cuh"

namespace paged {

constexpr int kPlanThreads = 1024;
constexpr int kMaxPlanParts = 4096;   // partitions per sequence the plan supports
// Sort keys: the partition count minus one when the context is partitioned,
// else the block count (at most 1024 blocks in single-pass mode).
constexpr int kPlanKeys = 4096;

__device__ __forceinline__ int plan_key(const PlanArgs& p, int nblk, int parts) {
  return p.max_parts > 1 ? parts - 1 : min(nblk, kPlanKeys - 1);
}

// Exclusive prefix sum, in place, of an int array in shared memory whose
// length is a multiple of kPlanThreads; every thread of the block calls it.
template <class Scan>
__device__ void block_exclusive_scan(int* v, int n, typename Scan::TempStorage& tmp, int* carry) {
  if (threadIdx.x == 0) *carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kPlanThreads) {
    const int x = v[base + threadIdx.x];
    int ex, total;
    Scan(tmp).ExclusiveSum(x, ex, total);
    const int c = *carry;
    __syncthreads();
    v[base + threadIdx.x] = c + ex;
    if (threadIdx.x == 0) *carry = c + total;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kPlanThreads) paged_decode_plan(PlanArgs p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  using Scan = cub::BlockScan<int, kPlanThreads>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int hist[kPlanKeys];
  __shared__ int pcnt[kMaxPlanParts + 1];
  __shared__ int carry;
  const int tid = threadIdx.x;
  for (int i = tid; i < kPlanKeys; i += kPlanThreads) hist[i] = 0;
  for (int i = tid; i <= p.max_parts; i += kPlanThreads) pcnt[i] = 0;
  __syncthreads();

  // sequence lengths -> (sort key, partition count) histograms
  for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
    int ctx = p.context_lens[s];
    if (ctx > p.ctx_limit || ctx < 0) {
      report(p.err, kErrContextClipped);
      ctx = ctx < 0 ? 0 : p.ctx_limit;
    }
    const int nblk = (ctx + p.block_size - 1) / p.block_size;
    const int parts = nblk == 0 ? 1 : (nblk + p.partition_blocks - 1) / p.partition_blocks;
    atomicAdd(&hist[kPlanKeys - 1 - plan_key(p, nblk, parts)], 1);  // longest first
    atomicAdd(&pcnt[parts], 1);
  }
  __syncthreads();

  // exclusive scan of the key histogram -> first slot of each key
  block_exclusive_scan<Scan>(hist, kPlanKeys, scan_tmp, &carry);
  // C[q] = units in partition slices < q; slice q holds kv-heads x #{s: parts(s) > q}.
  // ge(q) = S - #{s: parts(s) <= q}; scanned in chunks of kPlanThreads.
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base <= p.max_parts; base += kPlanThreads) {
    const int q = base + tid;
    int v = q <= p.max_parts ? pcnt[q] : 0;  // #{s: parts(s) == q}
    int incl;
    Scan(scan_tmp).InclusiveSum(v, incl);    // #{s: base <= parts(s) <= q}
    const int le = carry + incl;              // #{s: parts(s) <= q}
    __syncthreads();
    if (q <= p.max_parts) {
      pcnt[q] = p.num_seqs - le;              // ge(q) = #{s: parts(s) > q}
    }
    if (tid == kPlanThreads - 1) carry = le;
    __syncthreads();
  }
  // prefix over slices (serial over at most kMaxPlanParts small ints, by one warp)
  if (tid < 32) {
    int run = 0;
    for (int base = 0; base < p.max_parts; base += 32) {
      const int q = base + tid;
      int v = q < p.max_parts ? pcnt[q] * p.num_kv_heads : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (tid >= o) x += y;
      }
      if (q < p.max_parts) p.slice_start[q] = run + x - v;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (tid == 0) {
      p.slice_start[p.max_parts] = run;
      p.counters[kCounterTotal] = run;
      p.counters[kCounterWork] = 0;
    }
  }
  __syncthreads();

  // scatter the sequences into length order
  for (int s = tid; s < p.num_seqs; s += kPlanThreads) {
    int ctx = p.context_lens[s];
    ctx = ctx < 0 ? 0 : (ctx > p.ctx_limit ? p.ctx_limit : ctx);
    const int nblk = (ctx + p.block_size - 1) / p.block_size;
    const int parts = nblk == 0 ? 1 : (nblk + p.partition_blocks - 1) / p.partition_blocks;
    const int pos = atomicAdd(&hist[kPlanKeys - 1 - plan_key(p, nblk, parts)], 1);
    p.order[pos] = make_int2(s, nblk);
  }
  if (p.arrive) {
    const int n = p.num_seqs * p.num_kv_heads;
    for (int i = tid; i < n; i += kPlanThreads) p.arrive[i] = 0;
  }
  // Finish only after the previous kernel of the stream: the decode grid waits
  // for this one, so it then also sees that kernel's writes.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

cudaError_t launch_plan(const PlanArgs& p, cudaStream_t stream) {
  if (p.max_parts > kMaxPlanParts) return cudaErrorNotSupported;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kPlanThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, paged_decode_plan, p);
}

}  // namespace paged
