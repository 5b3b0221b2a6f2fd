// consumer_mma.cuh — per-block attention arithmetic on the tensor cores, for
// query groups of 4 or 8 heads per kv-head (grouped-query attention), where
// a staged block really is a small dense contraction:
//   S[g, t] = Q[g, :] . K[t, :]      and      O[g, :] += P[g, t] V[t, :]
// with g the query heads of one kv-head and t the block's tokens. Each warp
// issues mma.sync m16n8k16 with fp32 accumulators: rows 0..G-1 of the 16-row
// A operand are the group's query heads (the rest are zero), the S
// accumulators are rescaled and exponentiated in registers (online softmax,
// base 2) and reused directly as the A operand of P.V.
//
// Operands come from the swizzled stage with ldmatrix (K as B of Q.K^T;
// V transposed by ldmatrix.trans as B of P.V). For an E4M3 cache the codes
// are widened exactly to f16 in registers (every E4M3 value is an f16 value):
//  * K: each 4-byte ldmatrix element row holds dims 4c..4c+3 of a token; the
//    k-index order inside each 16-wide MMA step is permuted to match (the
//    query fragments use the same permutation, so the dot product is unchanged);
//  * V: ldmatrix.trans yields byte pairs of two tokens x two dims; a byte
//    permute splits them into an even-dim and an odd-dim n-tile, and the
//    output columns are mapped back to dims when the accumulator is stored.
// The query (bf16 or f16) of an E4M3 path is scaled by a power of two so its
// largest element sits just below 2^15 and converted to f16 (exact for every
// element within 2^29 of that maximum); the factor is undone in the fp32
// logit scale, together with the kv-head's K dequantisation scale.
#pragma once

#include <type_traits>

#include "decode_kernel.cuh"

namespace paged {

__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

__device__ __forceinline__ void ldsm_x4_trans(const void* p, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

// D[rows r] += A . B for one m16n8k16 tile whose A rows 8..15 are zero:
// only the two accumulators of row r are kept.
template <bool BF>
__device__ __forceinline__ void mma_rows0_7(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0,
                                            uint32_t b1) {
  float x2, x3;
  if constexpr (BF) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(x2), "=f"(x3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]),
          "f"(0.f), "f"(0.f));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(x2), "=f"(x3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d[0]), "f"(d[1]),
          "f"(0.f), "f"(0.f));
  }
}

// Two E4M3 codes (low byte first) -> f16x2, exactly.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  const __half2_raw h =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xffffu), __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

template <bool BF>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
  }
}

template <class QF_, class CF_, int D_, int G_>
struct MmaConsumer {
  using QF = QF_;
  using CF = CF_;
  using Tile = paged::Tile<CF, D_>;
  static constexpr int D = D_, BS = Tile::BS, G = G_;
  static constexpr bool FP8 = CF::kBytes == 1;
  static constexpr bool BF = !FP8 && std::is_same<CF, BF16>::value;  // MMA input type
  static constexpr int KS = D / 16;   // k-steps of Q.K^T (head_dim)
  static constexpr int NS = BS / 8;   // n-tiles of S (tokens)
  static constexpr int KP = BS / 16;  // k-steps of P.V (tokens)
  static constexpr int NO = D / 8;    // n-tiles of O (head_dim)
  static_assert(G <= 8 && KS % (FP8 ? 4 : 2) == 0 && NO % 2 == 0, "tile shapes");

  uint32_t qa[KS][2];  // A fragments of Q (a0, a2; a1 = a3 = 0)
  float o[NO][2];      // accumulators of row r
  float m, l, qscale;
  int r, c;

  // qrows: the G query rows of this kv-head ([G][D], q dtype; global or shared).
  __device__ __forceinline__ void init(const DecodeArgs& a, const void* qrows, int kvh, int lane) {
    r = lane >> 2;
    c = lane & 3;
    const bool live = r < G;
    const int qrow = (live ? r : 0) * D;
    qscale = a.scale_log2;
    if constexpr (!FP8) {
      const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qrows);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][0] = live ? q32[(qrow + 16 * kk + 2 * c) / 2] : 0u;
        qa[kk][1] = live ? q32[(qrow + 16 * kk + 2 * c + 8) / 2] : 0u;
      }
    } else {
      float qv[KS][4];
      float mx = 0.f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          qv[kk][j] = live ? load_in(QF{}, qrows, qrow + 16 * kk + 4 * c + j) : 0.f;
          mx = fmaxf(mx, fabsf(qv[kk][j]));
        }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      int e = 0;
      if (mx > 0.f && isfinite(mx)) {
        int k;
        frexpf(mx, &k);                    // mx < 2^k
        e = min(max(15 - k, -100), 100);   // mx * 2^e < 2^15
      }
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][0] = pack2<false>(ldexpf(qv[kk][0], e), ldexpf(qv[kk][1], e));
        qa[kk][1] = pack2<false>(ldexpf(qv[kk][2], e), ldexpf(qv[kk][3], e));
      }
      qscale *= a.k_scale[kvh] * ldexpf(1.f, -e);
    }
    m = -CUDART_INF_F;
    l = 0.f;
#pragma unroll
    for (int j = 0; j < NO; ++j) o[j][0] = o[j][1] = 0.f;
  }

  __device__ __forceinline__ void block(const uint8_t* kt, const uint8_t* vt_c, int valid,
                                        int lane) {
    uint8_t* vt = const_cast<uint8_t*>(vt_c);
    // ---- S = Q . K^T
    float sacc[NS][2];
#pragma unroll
    for (int nt = 0; nt < NS; ++nt) sacc[nt][0] = sacc[nt][1] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NS; ++nt) {
      const int row = nt * 8 + (lane & 7);
      if constexpr (!FP8) {
#pragma unroll
        for (int kk = 0; kk < KS; kk += 2) {
          uint32_t b[4];
          ldsm_x4(kt + Tile::off(row, (2 * kk + (lane >> 3)) * 16), b);
          mma_rows0_7<BF>(sacc[nt], qa[kk][0], qa[kk][1], b[0], b[1]);
          mma_rows0_7<BF>(sacc[nt], qa[kk + 1][0], qa[kk + 1][1], b[2], b[3]);
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < KS; kk += 4) {
          uint32_t b[4];
          ldsm_x4(kt + Tile::off(row, (kk + (lane >> 3)) * 16), b);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_rows0_7<false>(sacc[nt], qa[kk + j][0], qa[kk + j][1],
                               e4m3x2_to_f16x2(b[j]), e4m3x2_to_f16x2(b[j] >> 16));
        }
      }
    }
    // ---- online softmax of row r (4 lanes share a row)
    float mx = -CUDART_INF_F;
#pragma unroll
    for (int nt = 0; nt < NS; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int tok = nt * 8 + 2 * c + i;
        const float x = tok < valid ? sacc[nt][i] * qscale : -CUDART_INF_F;
        sacc[nt][i] = x;
        mx = fmaxf(mx, x);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
    const float alpha = exp2f(m - m_use);
    m = m_new;
    float ps = 0.f;
#pragma unroll
    for (int nt = 0; nt < NS; ++nt)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        sacc[nt][i] = exp2f(sacc[nt][i] - m_use);
        ps += sacc[nt][i];
      }
    l = l * alpha + ps;
#pragma unroll
    for (int j = 0; j < NO; ++j) {
      o[j][0] *= alpha;
      o[j][1] *= alpha;
    }
    // Rows past the context may hold anything (even NaN); P is 0 there, but
    // 0 * NaN is NaN inside the MMA, so clear them. The stage is refilled by
    // TMA later: order these writes before that (async proxy).
    if (valid < BS) {
      constexpr int CPR = Tile::RB / 16;
      for (int i = lane; i < (BS - valid) * CPR; i += 32)
        *reinterpret_cast<uint4*>(vt + Tile::off(valid + i / CPR, (i % CPR) * 16)) =
            make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      __syncwarp();
    }
    // ---- O += P . V
#pragma unroll
    for (int kp = 0; kp < KP; ++kp) {
      const uint32_t a0 = pack2<BF>(sacc[2 * kp][0], sacc[2 * kp][1]);
      const uint32_t a2 = pack2<BF>(sacc[2 * kp + 1][0], sacc[2 * kp + 1][1]);
      const int row = kp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      if constexpr (!FP8) {
#pragma unroll
        for (int dn = 0; dn < NO; dn += 2) {
          uint32_t b[4];
          ldsm_x4_trans(vt + Tile::off(row, (dn + (lane >> 4)) * 16), b);
          mma_rows0_7<BF>(o[dn], a0, a2, b[0], b[1]);
          mma_rows0_7<BF>(o[dn + 1], a0, a2, b[2], b[3]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < D / 16; q += 2) {
          uint32_t b[4];
          ldsm_x4_trans(vt + Tile::off(row, (q + (lane >> 4)) * 16), b);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t lo = b[2 * h], hi = b[2 * h + 1];
            // even dims of the chunk: bytes 0 and 2; odd dims: bytes 1 and 3
            mma_rows0_7<false>(o[2 * (q + h)], a0, a2,
                               e4m3x2_to_f16x2(__byte_perm(lo, 0u, 0x0020)),
                               e4m3x2_to_f16x2(__byte_perm(hi, 0u, 0x0020)));
            mma_rows0_7<false>(o[2 * (q + h) + 1], a0, a2,
                               e4m3x2_to_f16x2(__byte_perm(lo, 0u, 0x0031)),
                               e4m3x2_to_f16x2(__byte_perm(hi, 0u, 0x0031)));
          }
        }
      }
    }
  }

  // Output column of accumulator (n-tile j, element i) of this lane.
  __device__ __forceinline__ int dim_of(int j, int i) const {
    if constexpr (FP8) return 16 * (j / 2) + 4 * c + 2 * i + (j % 2);
    return 8 * j + 2 * c + i;
  }

  __device__ __forceinline__ void finish(float* mbuf, float* obuf, int) {
    float lr = l + __shfl_xor_sync(0xffffffffu, l, 1);
    lr += __shfl_xor_sync(0xffffffffu, lr, 2);
    if (r < G) {
      if (c == 0) {
        mbuf[r * 2] = m;
        mbuf[r * 2 + 1] = lr;
      }
#pragma unroll
      for (int j = 0; j < NO; ++j)
#pragma unroll
        for (int i = 0; i < 2; ++i) obuf[r * D + dim_of(j, i)] = o[j][i];
    }
  }
};

}  // namespace paged
