// decode_simt.cuh — paged decode attention on the CUDA cores (fp32 math).
//
// Follows "vLLM推理引擎架构：PagedAttention机制与高吞吐推理" §2.3 (PagedAttention
// Kernel): for each sequence, walk its block table, gather the K/V rows of the
// physical blocks it names, compute attention scores inside each block and
// accumulate across blocks; the logical->physical translation is the one of
// "vLLM框架中的KV cache优化与PagedAttention机制详解" §5.1, done per block (one
// table lookup per block, "批量转换") and issued ahead of use ("预取机制", §5.2).
//
// Work unit = one CTA per (kv-head, sequence, context partition). Each of the
// NW warps owns every NW-th block of the partition and runs its own R-deep ring
// of shared-memory stages: its lane 0 issues one TMA box load per 128-byte
// column of the K and V tiles of a block (block_size rows of one kv-head,
// 128B/64B swizzled) and the warp waits on the stage's mbarrier. No barrier is
// shared between warps until the final merge, so every warp's ring streams
// independently.
//
// Inside a warp, TPT lanes share one token row (TPT = 8, 16 or 32, so a lane
// holds G x D/TPT query values); a token's logit is reduced over those lanes
// with shuffles; each token group keeps its own online-softmax state (running
// max m, sum l, fp32 accumulator) in base-2 units (the softmax scale is
// pre-multiplied by log2 e), merged across groups and warps at the end.
#pragma once

#include <math_constants.h>

#include "decode_args.h"
#include "device_common.cuh"

namespace paged {

template <class QF_, class CF_, int D_, int BS_, int G_>
struct SimtCfg {
  using QF = QF_;
  using CF = CF_;
  static constexpr int D = D_, BS = BS_, G = G_;
  static constexpr int EB = CF::kBytes;
  static constexpr int RB = D * EB;                          // bytes per token row
  static constexpr int BOXB = box_bytes(RB);                 // bytes per box row
  static constexpr int NBOX = RB / BOXB;
  static constexpr int SWZ = BOXB == 128 ? 0x70 : (BOXB == 64 ? 0x30 : 0);
  static constexpr int TILE = BS * RB;                       // one K (or V) tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int TPT_RAW = G * D / 16;
  static constexpr int TPT = TPT_RAW < 8 ? 8 : (TPT_RAW > 32 ? 32 : TPT_RAW);
  static constexpr int NTG = 32 / TPT;                       // token groups per warp
  static constexpr int LB = RB / TPT;                        // bytes per lane per row
  static constexpr int U = LB < 16 ? LB : 16;                // bytes per load
  static constexpr int NU = LB / U;                          // loads per row
  static constexpr int EPU = U / EB;                         // elements per load
  static constexpr int NE = NU * EPU;                        // elements per lane
  static constexpr int ROUNDS = BS / NTG;                    // rows per group per block
  static constexpr int CH_RAW = 16 / G;
  static constexpr int CH = CH_RAW < 1 ? 1 : (CH_RAW > ROUNDS ? ROUNDS : CH_RAW);
  static_assert(ROUNDS % CH == 0, "chunking");
  static_assert(NE * TPT == D, "lane split");
  static constexpr int NW = 4;                               // warps per CTA
  static constexpr int R_RAW = 65536 / (NW * STAGE);
  static constexpr int R = R_RAW < 1 ? 1 : (R_RAW > 4 ? 4 : R_RAW);  // stages per warp
  static constexpr int STAGES_BYTES = NW * R * STAGE;
  static_assert(NW * G * (D + 2) * 4 <= STAGES_BYTES, "merge buffer fits in the stages");

  // Shared-memory byte offset of logical byte `o` of row `r` inside a tile.
  static __device__ __forceinline__ uint32_t off(int r, int o) {
    const int box = o / BOXB;
    const int lin = r * BOXB + (o % BOXB);
    return box * (BS * BOXB) + (lin ^ ((lin >> 3) & SWZ));
  }
};

// Load U bytes (U in {2,4,8,16}) from shared memory into 32-bit words.
template <int U>
__device__ __forceinline__ void lds_unit(const uint8_t* p, uint32_t (&w)[(U + 3) / 4]) {
  if constexpr (U == 16) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (U == 8) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (U == 4) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  }
}

// Convert one loaded unit to EPU fp32 values.
template <class CF, int U>
__device__ __forceinline__ void cvt_unit(const uint32_t (&w)[(U + 3) / 4], float* dst) {
  if constexpr (CF::kBytes == 2) {
#pragma unroll
    for (int i = 0; i < U / 4; ++i) {
      float2 f = cvt2(CF{}, w[i]);
      dst[2 * i] = f.x;
      dst[2 * i + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < (U + 1) / 2; ++i) {
      const uint16_t pair = static_cast<uint16_t>(w[i / 2] >> (16 * (i % 2)));
      float2 f = cvt2_e4m3(pair);
      dst[2 * i] = f.x;
      dst[2 * i + 1] = f.y;
    }
  }
}

// One row of this lane's share of a tile, as NE fp32 values.
template <class C>
__device__ __forceinline__ void load_row(const uint8_t* tile, int row, int li, float (&dst)[C::NE]) {
#pragma unroll
  for (int k = 0; k < C::NU; ++k) {
    uint32_t w[(C::U + 3) / 4];
    lds_unit<C::U>(tile + C::off(row, li * C::U + k * (C::TPT * C::U)), w);
    cvt_unit<typename C::CF, C::U>(w, dst + k * C::EPU);
  }
}

// Element index (within head_dim) of lane-local element e.
template <class C>
__device__ __forceinline__ int lane_dim(int li, int e) {
  const int k = e / C::EPU, j = e % C::EPU;
  return (li * C::U + k * (C::TPT * C::U)) / C::EB + j;
}

template <class C>
__global__ void __launch_bounds__(C::NW * 32)
    paged_decode_simt(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
  constexpr int D = C::D, BS = C::BS, G = C::G, NW = C::NW, R = C::R, TPT = C::TPT;
  constexpr int NE = C::NE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES_BYTES);
  int32_t* ids = reinterpret_cast<int32_t*>(bars + NW * R);

  const int kvh = blockIdx.x, s = blockIdx.y, part = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tg = lane / TPT, li = lane % TPT;

  // Context length, clipped to what the launch covers.
  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (threadIdx.x == 0 && part == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int parts = nblk == 0 ? 1 : (nblk + a.partition_blocks - 1) / a.partition_blocks;
  if (part >= parts) return;
  const int b_begin = part * a.partition_blocks;
  const int b_end = min(b_begin + a.partition_blocks, nblk);
  const int nlocal = b_end - b_begin;

  // Block ids of this partition -> shared memory (validated once).
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
  for (int i = threadIdx.x; i < nlocal; i += NW * 32) {
    int32_t id = table[b_begin + i];
    if (id < 0 || id >= a.num_blocks) {
      report(a.err, kErrBadBlockId);
      id = -1;
    }
    ids[i] = id;
  }
  if (lane == 0) {
    for (int r = 0; r < R; ++r) mbar_init(&bars[warp * R + r], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  __syncthreads();

  const int my_count = nlocal > warp ? (nlocal - warp + NW - 1) / NW : 0;
  uint8_t* my_stages = smem + warp * R * C::STAGE;
  uint64_t* my_bars = bars + warp * R;
  const uint64_t policy = l2_policy_evict_first();

  auto issue = [&](int it) {
    const int stage = it % R;
    const int32_t id = ids[warp + it * NW];
    // An invalid id reads a box entirely outside the pool: TMA zero-fills it.
    const int32_t row0 = id >= 0 ? id * BS : -BS;
    uint8_t* kt = my_stages + stage * C::STAGE;
    uint8_t* vt = kt + C::TILE;
    mbar_arrive_expect_tx(&my_bars[stage], C::STAGE);
#pragma unroll
    for (int b = 0; b < C::NBOX; ++b) {
      const int x = b * (C::BOXB / C::EB);
      tma_load_3d_hint(kt + b * BS * C::BOXB, &kmap, &my_bars[stage], x, kvh, row0, policy);
      tma_load_3d_hint(vt + b * BS * C::BOXB, &vmap, &my_bars[stage], x, kvh, row0, policy);
    }
  };
  if (lane == 0) {
    for (int it = 0; it < min(R, my_count); ++it) issue(it);
  }

  // Query rows of the G heads of this kv-head: this lane's NE dims, scaled.
  float qf[G][NE];
  {
    float qs = a.scale_log2;
    if (a.k_scale) qs *= a.k_scale[kvh];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int64_t qrow = (static_cast<int64_t>(s) * a.num_heads + kvh * G + g) * D;
#pragma unroll
      for (int e = 0; e < NE; ++e)
        qf[g][e] = load_in(typename C::QF{}, a.query, qrow + lane_dim<C>(li, e)) * qs;
    }
  }

  float m[G], l[G], acc[G][NE];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -CUDART_INF_F;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < NE; ++e) acc[g][e] = 0.f;
  }

  bool timed_out = false;
  for (int it = 0; it < my_count; ++it) {
    const int stage = it % R;
    if (!mbar_wait(&my_bars[stage], (it / R) & 1)) {
      timed_out = true;
      break;
    }
    const uint8_t* kt = my_stages + stage * C::STAGE;
    const uint8_t* vt = kt + C::TILE;
    const int valid = min(BS, ctx - (b_begin + warp + it * NW) * BS);

#pragma unroll
    for (int c0 = 0; c0 < C::ROUNDS; c0 += C::CH) {
      float sc[G][C::CH];
#pragma unroll
      for (int r = 0; r < C::CH; ++r) {
        const int row = (c0 + r) * C::NTG + tg;
        float kf[NE];
        load_row<C>(kt, row, li, kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < NE; ++e) d = fmaf(qf[g][e], kf[e], d);
#pragma unroll
          for (int o = 1; o < TPT; o <<= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
          sc[g][r] = row < valid ? d : -CUDART_INF_F;
        }
      }
      float p[G][C::CH];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float mb = sc[g][0];
#pragma unroll
        for (int r = 1; r < C::CH; ++r) mb = fmaxf(mb, sc[g][r]);
        const float m_new = fmaxf(m[g], mb);
        const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
        const float alpha = exp2f(m[g] - m_use);
        m[g] = m_new;
        float ps = 0.f;
#pragma unroll
        for (int r = 0; r < C::CH; ++r) {
          p[g][r] = exp2f(sc[g][r] - m_use);
          ps += p[g][r];
        }
        l[g] = l[g] * alpha + ps;
#pragma unroll
        for (int e = 0; e < NE; ++e) acc[g][e] *= alpha;
      }
#pragma unroll
      for (int r = 0; r < C::CH; ++r) {
        const int row = (c0 + r) * C::NTG + tg;
        if (row < valid) {
          float vf[NE];
          load_row<C>(vt, row, li, vf);
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[g][e] = fmaf(p[g][r], vf[e], acc[g][e]);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && it + R < my_count) issue(it + R);
  }
  if (timed_out && lane == 0) report(a.err, kErrWaitTimeout);

  // Merge the token groups of this warp (lanes li, li+TPT, ...).
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float mw = m[g];
#pragma unroll
    for (int o = TPT; o < 32; o <<= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
    const float f = mw == -CUDART_INF_F ? 0.f : exp2f(m[g] - mw);
    l[g] *= f;
#pragma unroll
    for (int e = 0; e < NE; ++e) acc[g][e] *= f;
#pragma unroll
    for (int o = TPT; o < 32; o <<= 1) {
      l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
#pragma unroll
      for (int e = 0; e < NE; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
    }
    m[g] = mw;
  }

  // Merge the warps through shared memory (the stage ring is idle now: every
  // issued load has been waited for).
  __syncthreads();
  float* mbuf = reinterpret_cast<float*>(smem);              // [NW][G][2]
  float* obuf = mbuf + NW * G * 2;                           // [NW][G][D]
  if (tg == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int e = 0; e < NE; ++e) obuf[(warp * G + g) * D + lane_dim<C>(li, e)] = acc[g][e];
      if (li == 0) {
        mbuf[(warp * G + g) * 2] = m[g];
        mbuf[(warp * G + g) * 2 + 1] = l[g];
      }
    }
  }
  __syncthreads();

  const bool single = parts == 1;
  const float vs = a.v_scale ? a.v_scale[kvh] : 1.f;
  for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
    const int g = idx / D, d = idx % D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mbuf[(w * G + g) * 2]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = mbuf[(w * G + g) * 2];
      const float f = mw == -CUDART_INF_F ? 0.f : exp2f(mw - M);
      L += mbuf[(w * G + g) * 2 + 1] * f;
      o += obuf[(w * G + g) * D + d] * f;
    }
    o = L > 0.f ? o / L * vs : 0.f;
    const int h = kvh * G + g;
    const int64_t row = static_cast<int64_t>(s) * a.num_heads + h;
    if (single) {
      store_out(typename C::QF{}, a.out, row * D + d, o);
    } else {
      const int64_t pi = row * a.max_parts + part;
      a.ws_o[pi * D + d] = o;
      if (d == 0) a.ws_ml[pi] = make_float2(M, L);
    }
  }
}

template <class QF, class CF, int D, int BS, int G>
cudaError_t launch_simt(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                        cudaStream_t stream) {
  using C = SimtCfg<QF, CF, D, BS, G>;
  const size_t smem = 1024 + C::STAGES_BYTES + 8 * C::NW * C::R +
                      4 * static_cast<size_t>(a.partition_blocks);
  auto kern = paged_decode_simt<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_kv_heads, a.num_seqs, a.max_parts);
  kern<<<grid, C::NW * 32, smem, stream>>>(a, kmap, vmap);
  return cudaGetLastError();
}

// Dispatch over (head_dim, block_size, group) for one dtype pair.
template <class QF, class CF>
cudaError_t dispatch_decode(const DecodeArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int D, int BS, int G, cudaStream_t st) {
#define PAGED_CASE(d, bs, g) \
  if (D == d && BS == bs && G == g) return launch_simt<QF, CF, d, bs, g>(a, kmap, vmap, st);
#define PAGED_CASES_G(d, bs) \
  PAGED_CASE(d, bs, 1) PAGED_CASE(d, bs, 2) PAGED_CASE(d, bs, 4) PAGED_CASE(d, bs, 8)
  PAGED_CASES_G(64, 16)
  PAGED_CASES_G(64, 32)
  PAGED_CASES_G(128, 16)
  PAGED_CASES_G(128, 32)
#undef PAGED_CASES_G
#undef PAGED_CASE
  return cudaErrorNotSupported;
}

}  // namespace paged
