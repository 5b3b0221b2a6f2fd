// consumer_simt.cuh — per-block attention arithmetic on the CUDA cores (fp32),
// used for query groups of 1 and 2 heads per kv-head, where the work per byte
// is far below what the FP32 pipes sustain.
//
// TPT lanes share one token row (TPT = 8 or 16, so a lane holds G x D/TPT
// query values); a token's logit is reduced over those lanes with shuffles;
// each of the 32/TPT token groups of a warp keeps its own online-softmax state
// (running max m, sum l, fp32 accumulator), in base-2 units (the softmax
// scale is pre-multiplied by log2 e). Per block, a group computes the logits
// of its rows, rescales its state once, then accumulates p * V.
#pragma once

#include "decode_kernel.cuh"

namespace paged {

template <class QF_, class CF_, int D_, int G_>
struct SimtConsumer {
  using QF = QF_;
  using CF = CF_;
  using Tile = paged::Tile<CF, D_>;
  static constexpr int D = D_, BS = Tile::BS, G = G_;
  static constexpr int EB = CF::kBytes, RB = Tile::RB;
  static constexpr int TPT_RAW = G * D / 16;
  static constexpr int TPT = TPT_RAW < 8 ? 8 : (TPT_RAW > 32 ? 32 : TPT_RAW);
  static constexpr int NTG = 32 / TPT;           // token groups per warp
  static constexpr int LB = RB / TPT;            // bytes per lane per row
  static constexpr int U = LB < 16 ? LB : 16;    // bytes per shared load
  static constexpr int NU = LB / U;              // loads per row
  static constexpr int EPU = U / EB;             // elements per load
  static constexpr int NE = NU * EPU;            // elements per lane
  static constexpr int ROUNDS = BS / NTG;        // rows per group per block
  static constexpr int CH_RAW = 16 / G;
  static constexpr int CH = CH_RAW < 1 ? 1 : (CH_RAW > ROUNDS ? ROUNDS : CH_RAW);
  static_assert(ROUNDS % CH == 0 && NE * TPT == D, "lane split");

  float qf[G][NE];
  float m[G], l[G], acc[G][NE];
  int tg, li;

  // Element index (within head_dim) of lane-local element e.
  static __device__ __forceinline__ int lane_dim(int li, int e) {
    const int k = e / EPU, j = e % EPU;
    return (li * U + k * (TPT * U)) / EB + j;
  }

  template <int UB>
  static __device__ __forceinline__ void lds(const uint8_t* p, uint32_t (&w)[(UB + 3) / 4]) {
    if constexpr (UB == 16) {
      const uint4 v = *reinterpret_cast<const uint4*>(p);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (UB == 8) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x; w[1] = v.y;
    } else if constexpr (UB == 4) {
      w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else {
      w[0] = *reinterpret_cast<const uint16_t*>(p);
    }
  }

  // This lane's NE values of row `row` of a staged tile, as fp32.
  __device__ __forceinline__ void load_row(const uint8_t* tile, int row, float (&dst)[NE]) const {
#pragma unroll
    for (int k = 0; k < NU; ++k) {
      uint32_t w[(U + 3) / 4];
      lds<U>(tile + Tile::off(row, li * U + k * (TPT * U)), w);
      float* o = dst + k * EPU;
      if constexpr (EB == 2) {
#pragma unroll
        for (int i = 0; i < U / 4; ++i) {
          const float2 f = cvt2(CF{}, w[i]);
          o[2 * i] = f.x;
          o[2 * i + 1] = f.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < (U + 1) / 2; ++i) {
          const float2 f = cvt2_e4m3(static_cast<uint16_t>(w[i / 2] >> (16 * (i % 2))));
          o[2 * i] = f.x;
          o[2 * i + 1] = f.y;
        }
      }
    }
  }

  // qrows: the G query rows of this kv-head ([G][D], q dtype; global or shared).
  __device__ __forceinline__ void init(const DecodeArgs& a, const void* qrows, int kvh, int lane) {
    tg = lane / TPT;
    li = lane % TPT;
    float qs = a.scale_log2;
    if (a.k_scale) qs *= a.k_scale[kvh];
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int e = 0; e < NE; ++e) qf[g][e] = load_in(QF{}, qrows, g * D + lane_dim(li, e)) * qs;
      m[g] = -CUDART_INF_F;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) acc[g][e] = 0.f;
    }
  }

  __device__ __forceinline__ void block(const uint8_t* kt, const uint8_t* vt, int valid, int) {
#pragma unroll
    for (int c0 = 0; c0 < ROUNDS; c0 += CH) {
      float sc[G][CH];
#pragma unroll
      for (int r = 0; r < CH; ++r) {
        const int row = (c0 + r) * NTG + tg;
        float kf[NE];
        load_row(kt, row, kf);
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
      float p[G][CH];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float mb = sc[g][0];
#pragma unroll
        for (int r = 1; r < CH; ++r) mb = fmaxf(mb, sc[g][r]);
        const float m_new = fmaxf(m[g], mb);
        const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
        const float alpha = exp2f(m[g] - m_use);
        m[g] = m_new;
        float ps = 0.f;
#pragma unroll
        for (int r = 0; r < CH; ++r) {
          p[g][r] = exp2f(sc[g][r] - m_use);
          ps += p[g][r];
        }
        l[g] = l[g] * alpha + ps;
#pragma unroll
        for (int e = 0; e < NE; ++e) acc[g][e] *= alpha;
      }
#pragma unroll
      for (int r = 0; r < CH; ++r) {
        const int row = (c0 + r) * NTG + tg;
        if (row < valid) {  // rows past the context may hold anything, even NaN
          float vf[NE];
          load_row(vt, row, vf);
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < NE; ++e) acc[g][e] = fmaf(p[g][r], vf[e], acc[g][e]);
        }
      }
    }
  }

  // Merge the token groups, then write this warp's (m, l) and accumulator.
  __device__ __forceinline__ void finish(float* mbuf, float* obuf, int) {
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
      if (tg == 0) {
#pragma unroll
        for (int e = 0; e < NE; ++e) obuf[g * D + lane_dim(li, e)] = acc[g][e];
        if (li == 0) {
          mbuf[g * 2] = mw;
          mbuf[g * 2 + 1] = l[g];
        }
      }
    }
  }
};

}  // namespace paged
