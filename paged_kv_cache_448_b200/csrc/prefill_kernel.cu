// prefill_kernel.cu — attention of several query tokens per sequence over the
// paged cache (chunked prefill, verification of draft tokens).
//
// The q_len_s query rows of sequence s are its last positions,
// p_i = ctx_s - q_len_s + i; row i attends to the tokens t <= p_i of the
// sequence, found through its block table ("vLLM推理引擎架构：PagedAttention
// 机制与高吞吐推理" §2.3: attention over the blocks a block table names, here
// with a query tensor of more rows than sequences, and the causal rule of
// autoregressive attention).
//
// Unlike decode this is a dense contraction: a CTA owns 64 rows, a row being
// one (query token, head of the kv-head's group), i.e. 64/G consecutive query
// tokens of one (sequence, kv-head); each of its 4 warps owns 16 rows. The
// K/V tiles of that kv-head (16 tokens, the decode kernel's TMA box and
// swizzled layout) stream through an R-stage ring shared by the CTA: one
// thread issues the TMA loads (full barriers with transaction counts), every
// warp reads every tile and releases it (empty barriers, one arrival per
// warp). Per tile a warp computes S = Q K^T (16 x 16, mma.sync m16n8k16,
// fp32 accumulators; K as the B operand by ldmatrix), masks tokens after each
// row's position, runs the online softmax in base 2 and accumulates
// O += P V with P re-packed from the S accumulators as the A operand and V
// transposed by ldmatrix.trans. Every wait is bounded by wall time.
//
// This kernel serves the shapes the tensor-memory kernel (prefill_tc.cu)
// does not take: short chunks of few sequences (with the key range split
// across CTAs and merged by paged_prefill_combine), fewer than 8 rows per
// kv-head, and E4M3 caches with head_dim 64.
#include <math_constants.h>

#include "consumer_mma.cuh"
#include "decode_args.h"
#include "decode_kernel.cuh"
#include "device_common.cuh"
#include "prefill_args.h"

namespace paged {
namespace {

#ifndef PAGED_PREFILL_TPS
#define PAGED_PREFILL_TPS 1
#endif
#ifndef PAGED_PREFILL_RS
#define PAGED_PREFILL_RS 4
#endif
constexpr int kPrefillWarps = 4;
constexpr int kPrefillRows = 16 * kPrefillWarps;  // rows (token x head) per CTA
constexpr int kPrefillTps = PAGED_PREFILL_TPS;    // 16-token tiles per softmax step
constexpr int kPrefillRs = PAGED_PREFILL_RS;      // steps in flight in the ring
constexpr int kPrefillStages = kPrefillRs * kPrefillTps;

// D[16 x 8] += A[16 x 16] . B[16 x 8] (all 16 rows live).
template <bool BF>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  if constexpr (BF) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// QF: query / output type; CF: cache type (QF, or E4M3). An E4M3 cache is
// widened exactly to f16 in registers (every E4M3 value is an f16 value) as
// in the decode kernel's tensor-core consumer: K with the k order inside each
// 16-wide MMA step permuted to match 4-byte ldmatrix rows (the query uses the
// same permutation), V split into even / odd dimensions by byte permutes; the
// query goes to f16 scaled by a power of two (undone in the logit scale with
// the kv-head's K scale), the V scale applies to the output.
template <class QF, class CF, int D, int G>
__global__ void __launch_bounds__(kPrefillWarps * 32)
    paged_prefill_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap) {
  using T = Tile<CF, D>;
  constexpr bool FP8 = CF::kBytes == 1;
  constexpr bool QBF = std::is_same<QF, BF16>::value;
  constexpr bool BF = QBF && !FP8;   // MMA operand type: bf16 (16-bit bf16 cache) or f16
  constexpr int R = kPrefillStages, NW = kPrefillWarps, TR = kTileRows;
  constexpr int QT = kPrefillRows / G;  // query tokens per CTA
  constexpr int KS = D / 16, NO = D / 8;
  constexpr int STAGE = 2 * T::BYTES;
  constexpr unsigned FULL = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + R * STAGE);
  uint64_t* empty = full + R;
  __shared__ int aborted;

  const int z = blockIdx.x % a.q_tiles, part = blockIdx.x / a.q_tiles;
  const int kvh = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int r = 0; r < R; ++r) {
      mbar_init(&full[r], 1);
      mbar_init(&empty[r], NW);
    }
    fence_mbar_init();
    aborted = 0;
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  __syncthreads();
  // Everything below reads data of earlier kernels in the stream.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int q0 = a.cu_query_lens[s];
  const int qlen = a.cu_query_lens[s + 1] - q0;
  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  const int tok0 = z * QT;
  if (tok0 >= qlen) return;  // ragged chunk lengths: nothing for this CTA
  const int ntok = min(QT, qlen - tok0);

  // rows of this lane: r_lo and r_lo + 8 of the warp's 16; row = token * G + head
  const int c = lane & 3;
  const int r_lo = warp * 16 + (lane >> 2), r_hi = r_lo + 8;
  const int tk_lo = r_lo / G, tk_hi = r_hi / G;
  const bool v_lo = tk_lo < ntok, v_hi = tk_hi < ntok;
  const int64_t row_lo = (static_cast<int64_t>(q0 + tok0 + tk_lo) * a.num_heads + kvh * G +
                          r_lo % G) * D;
  const int64_t row_hi = (static_cast<int64_t>(q0 + tok0 + tk_hi) * a.num_heads + kvh * G +
                          r_hi % G) * D;

  if (qlen > ctx) {  // a query longer than its context: rows become zeros
    if (part > 0) return;
    if (threadIdx.x == 0 && z == 0 && kvh == 0) report(a.err, kErrQueryLonger);
    uint32_t* out32 = static_cast<uint32_t*>(a.out);
    for (int j = 0; j < NO; ++j) {
      if (v_lo) out32[(row_lo + j * 8 + 2 * c) / 2] = 0u;
      if (v_hi) out32[(row_hi + j * 8 + 2 * c) / 2] = 0u;
    }
    return;
  }
  const int pos0 = ctx - qlen + tok0;       // position of the CTA's first query token
  // 16-token tiles up to the CTA's last position, cut into parts of
  // partition_tiles; this CTA takes part `part`: tiles tbase .. tbase+ntiles-1
  const int ntiles_all = (pos0 + ntok - 1) / TR + 1;
  const int parts = (ntiles_all + a.partition_tiles - 1) / a.partition_tiles;
  if (part >= parts) return;
  const int tbase = part * a.partition_tiles;
  const int ntiles = min(ntiles_all - tbase, a.partition_tiles);
  const int p_lo = v_lo ? pos0 + tk_lo : -1, p_hi = v_hi ? pos0 + tk_hi : -1;
  const int p_min = min(p_lo, p_hi);

  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
  const uint64_t policy = l2_policy_evict_last();  // the other query tiles read them too
  const bool producer = threadIdx.x == 0;
  auto issue = [&](int t, int32_t bid) {
    const int stage = t % R;
    if (bid < 0 || bid >= a.num_blocks) {
      report(a.err, kErrBadBlockId);
      bid = -1;  // read as a box outside the pool: zero-filled
    }
    const int32_t row0 = bid >= 0 ? bid * a.block_size + ((tbase + t) * TR) % a.block_size : -TR;
    uint8_t* kt = smem + stage * STAGE;
    if (skip_for_test(a.skip_tile, t)) return;
    mbar_arrive_expect_tx(&full[stage], STAGE);
    tma_load_4d(kt, &kmap, &full[stage], 0, row0, kvh, 0, policy);
    tma_load_4d(kt + T::BYTES, &vmap, &full[stage], 0, row0, kvh, 0, policy);
  };
  // The producer loads the block ids of a whole step first, then issues its
  // TMA boxes (the id loads overlap instead of preceding each box).
  auto issue_step = [&](int k) {
    int32_t bid[kPrefillTps];
#pragma unroll
    for (int j = 0; j < kPrefillTps; ++j) {
      const int tt = k * kPrefillTps + j;
      bid[j] = tt < ntiles ? table[((tbase + tt) * TR) / a.block_size] : 0;
    }
#pragma unroll
    for (int j = 0; j < kPrefillTps; ++j) {
      const int tt = k * kPrefillTps + j;
      if (tt < ntiles) issue(tt, bid[j]);
    }
  };
  const int nsteps = (ntiles + kPrefillTps - 1) / kPrefillTps;
  if (producer)
    for (int k = 0; k < min(kPrefillRs, nsteps); ++k) issue_step(k);

  // Q fragments (A operand, rows r_lo / r_hi, k-steps of 16 dims)
  uint32_t qa[KS][4];
  float qscale = a.scale_log2;
  if constexpr (!FP8) {
    const uint32_t* q32 = static_cast<const uint32_t*>(a.query);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = v_lo ? q32[(row_lo + kk * 16 + 2 * c) / 2] : 0u;
      qa[kk][1] = v_hi ? q32[(row_hi + kk * 16 + 2 * c) / 2] : 0u;
      qa[kk][2] = v_lo ? q32[(row_lo + kk * 16 + 8 + 2 * c) / 2] : 0u;
      qa[kk][3] = v_hi ? q32[(row_hi + kk * 16 + 8 + 2 * c) / 2] : 0u;
    }
  } else {
    // permuted k order: k 2c, 2c+1 <-> dims 4c, 4c+1; k 2c+8, 2c+9 <-> dims 4c+2, 4c+3
    float qv[KS][2][4];
    float mq = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        qv[kk][0][j] = v_lo ? load_in(QF{}, a.query, row_lo + 16 * kk + 4 * c + j) : 0.f;
        qv[kk][1][j] = v_hi ? load_in(QF{}, a.query, row_hi + 16 * kk + 4 * c + j) : 0.f;
        mq = fmaxf(mq, fmaxf(fabsf(qv[kk][0][j]), fabsf(qv[kk][1][j])));
      }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mq = fmaxf(mq, __shfl_xor_sync(FULL, mq, o2));
    int e = 0;
    if (mq > 0.f && isfinite(mq)) {
      int k2;
      frexpf(mq, &k2);                      // mq < 2^k2
      e = min(max(15 - k2, -100), 100);     // mq * 2^e < 2^15
    }
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = pack2<false>(ldexpf(qv[kk][0][0], e), ldexpf(qv[kk][0][1], e));
      qa[kk][1] = pack2<false>(ldexpf(qv[kk][1][0], e), ldexpf(qv[kk][1][1], e));
      qa[kk][2] = pack2<false>(ldexpf(qv[kk][0][2], e), ldexpf(qv[kk][0][3], e));
      qa[kk][3] = pack2<false>(ldexpf(qv[kk][1][2], e), ldexpf(qv[kk][1][3], e));
    }
    qscale *= a.k_scale[kvh] * ldexpf(1.f, -e);
  }
  float o[NO][4];
#pragma unroll
  for (int j = 0; j < NO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_lo = -CUDART_INF_F, m_hi = -CUDART_INF_F, l_lo = 0.f, l_hi = 0.f;

  int k = 0, t = 0;  // step, and the first tile not yet received
  bool failed = false;
  for (; k < nsteps && !failed; ++k) {
    const int t0 = k * kPrefillTps;
    // refill the stages of step k-1 with step k+RS-1 once every warp released them
    if (producer && k >= 1 && k + kPrefillRs - 1 < nsteps && !aborted) {
      bool ok = true;
      for (int j = 0; j < kPrefillTps && ok; ++j) {
        const int tp = t0 - kPrefillTps + j;
        ok = mbar_wait(&empty[tp % R], (tp / R) & 1, a.wait_limit_ns, &aborted);
      }
      if (ok) {
        issue_step(k + kPrefillRs - 1);
      } else {
        record_failure(a.diag, kSitePrefill, blockIdx.x, blockIdx.y, blockIdx.z, k, t0, ntiles,
                       1);
        aborted = 1;
      }
    }
    // ---- S = Q K^T over the step's tiles (16 tokens each)
    float sacc[kPrefillTps][2][4];
#pragma unroll
    for (int j = 0; j < kPrefillTps; ++j) {
      const int tt = t0 + j;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
        sacc[j][nt][0] = sacc[j][nt][1] = sacc[j][nt][2] = sacc[j][nt][3] = 0.f;
      if (tt >= ntiles) continue;
      if (!__all_sync(FULL, mbar_wait(&full[tt % R], (tt / R) & 1, a.wait_limit_ns, &aborted))) {
        failed = true;
        break;
      }
      t = tt + 1;
      const uint8_t* kt = smem + (tt % R) * STAGE;
      // even and odd k-steps in separate accumulators: two independent MMA
      // chains per n-tile instead of one of length KS
      float s2[2][4] = {};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int row = nt * 8 + (lane & 7);
        if constexpr (!FP8) {
#pragma unroll
          for (int kk = 0; kk < KS; kk += 2) {
            uint32_t b[4];
            ldsm_x4(kt + T::off(row, (2 * kk + (lane >> 3)) * 16), b);
            mma_16816<BF>(sacc[j][nt], qa[kk], b[0], b[1]);
            mma_16816<BF>(s2[nt], qa[kk + 1], b[2], b[3]);
          }
        } else {
          // 16 E4M3 dims per 16-byte chunk: one ldmatrix x4 covers 4 k-steps
#pragma unroll
          for (int kk = 0; kk < KS; kk += 4) {
            uint32_t b[4];
            ldsm_x4(kt + T::off(row, (kk + (lane >> 3)) * 16), b);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              mma_16816<false>((q & 1) ? s2[nt] : sacc[j][nt], qa[kk + q],
                               e4m3x2_to_f16x2(b[q]), e4m3x2_to_f16x2(b[q] >> 16));
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[j][nt][i] += s2[nt][i];
    }
    if (failed) break;
    // ---- causal mask (tokens after a row's position), scale, online softmax
    float mx_lo = -CUDART_INF_F, mx_hi = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < kPrefillTps; ++j) {
      const int tok_base = (tbase + t0 + j) * TR;
      const bool masked = tok_base + TR - 1 > p_min;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tok = tok_base + nt * 8 + 2 * c + (i & 1);
          const int p = i < 2 ? p_lo : p_hi;
          const float x = (!masked || tok <= p) ? sacc[j][nt][i] * qscale : -CUDART_INF_F;
          sacc[j][nt][i] = x;
          if (i < 2) mx_lo = fmaxf(mx_lo, x);
          else mx_hi = fmaxf(mx_hi, x);
        }
    }
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(FULL, mx_lo, 1));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(FULL, mx_lo, 2));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(FULL, mx_hi, 1));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(FULL, mx_hi, 2));
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    const float mu_lo = mn_lo == -CUDART_INF_F ? 0.f : mn_lo;
    const float mu_hi = mn_hi == -CUDART_INF_F ? 0.f : mn_hi;
    const float al_lo = exp2f(m_lo - mu_lo), al_hi = exp2f(m_hi - mu_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
    for (int j = 0; j < kPrefillTps; ++j)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sacc[j][nt][0] = exp2f(sacc[j][nt][0] - mu_lo);
        sacc[j][nt][1] = exp2f(sacc[j][nt][1] - mu_lo);
        sacc[j][nt][2] = exp2f(sacc[j][nt][2] - mu_hi);
        sacc[j][nt][3] = exp2f(sacc[j][nt][3] - mu_hi);
        ps_lo += sacc[j][nt][0] + sacc[j][nt][1];
        ps_hi += sacc[j][nt][2] + sacc[j][nt][3];
      }
    l_lo = l_lo * al_lo + ps_lo;
    l_hi = l_hi * al_hi + ps_hi;
#pragma unroll
    for (int j = 0; j < NO; ++j) {
      o[j][0] *= al_lo;
      o[j][1] *= al_lo;
      o[j][2] *= al_hi;
      o[j][3] *= al_hi;
    }
    // ---- O += P V per tile (P from the S accumulators, as the A operand)
#pragma unroll
    for (int j = 0; j < kPrefillTps; ++j) {
      const int tt = t0 + j;
      if (tt >= ntiles) break;
      uint8_t* vt = smem + (tt % R) * STAGE + T::BYTES;
      const int tok_base = (tbase + tt) * TR;
      // Rows of the tile past the context may hold anything (even NaN) and
      // 0 * NaN is NaN inside the MMA: each warp clears them in its view of
      // the stage before reading V (every warp writes the same zeros; only
      // the last tile can reach past the context and its stage is not refilled).
      if (tok_base + TR > ctx) {
        constexpr int CPR = T::RB / 16;
        const int first = max(0, ctx - tok_base);
        for (int i = lane; i < (TR - first) * CPR; i += 32)
          *reinterpret_cast<uint4*>(vt + T::off(first + i / CPR, (i % CPR) * 16)) =
              make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
      }
      // bf16 keeps only 8 significant bits, too few for rows that see a
      // handful of tokens; there P = P_hi + P_lo, both bf16, in two MMAs.
      uint32_t pa[4], pl[4];
      pa[0] = pack2<BF>(sacc[j][0][0], sacc[j][0][1]);
      pa[1] = pack2<BF>(sacc[j][0][2], sacc[j][0][3]);
      pa[2] = pack2<BF>(sacc[j][1][0], sacc[j][1][1]);
      pa[3] = pack2<BF>(sacc[j][1][2], sacc[j][1][3]);
      if constexpr (BF) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* src = sacc[j][q >> 1] + 2 * (q & 1);
          pl[q] = pack2<true>(src[0] - __uint_as_float(pa[q] << 16),
                              src[1] - __uint_as_float(pa[q] & 0xffff0000u));
        }
      }
      const int vrow = (lane & 7) + ((lane >> 3) & 1) * 8;
      if constexpr (!FP8) {
#pragma unroll
        for (int dn = 0; dn < NO; dn += 2) {
          uint32_t b[4];
          ldsm_x4_trans(vt + T::off(vrow, (dn + (lane >> 4)) * 16), b);
          mma_16816<BF>(o[dn], pa, b[0], b[1]);
          mma_16816<BF>(o[dn + 1], pa, b[2], b[3]);
          if constexpr (BF) {
            mma_16816<BF>(o[dn], pl, b[0], b[1]);
            mma_16816<BF>(o[dn + 1], pl, b[2], b[3]);
          }
        }
      } else {
        // ldmatrix.trans gives byte pairs of two tokens x two dims: a byte
        // permute splits them into an even-dim and an odd-dim n-tile
#pragma unroll
        for (int q = 0; q < D / 16; q += 2) {
          uint32_t b[4];
          ldsm_x4_trans(vt + T::off(vrow, (q + (lane >> 4)) * 16), b);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t lo = b[2 * h], hi = b[2 * h + 1];
            mma_16816<false>(o[2 * (q + h)], pa, e4m3x2_to_f16x2(__byte_perm(lo, 0u, 0x0020)),
                             e4m3x2_to_f16x2(__byte_perm(hi, 0u, 0x0020)));
            mma_16816<false>(o[2 * (q + h) + 1], pa,
                             e4m3x2_to_f16x2(__byte_perm(lo, 0u, 0x0031)),
                             e4m3x2_to_f16x2(__byte_perm(hi, 0u, 0x0031)));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[tt % R]);
    }
  }
  if (failed) {
    // A wait gave up (never expected): record it and let the loads this CTA
    // issued land (bounded) before its shared memory goes away.
    if (lane == 0) {
      // the record first: a warp stopped by the flag below must not take it
      record_failure(a.diag, kSitePrefill, blockIdx.x, blockIdx.y, blockIdx.z, warp, t, ntiles,
                     0);
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    if (producer) {
      // issued so far: steps 0 .. min(k + RS - 1, nsteps - 1) at most
      const int last = min(ntiles, (min(k + kPrefillRs - 1, nsteps - 1) + 1) * kPrefillTps);
      for (int tt = t; tt < last; ++tt) mbar_wait(&full[tt % R], (tt / R) & 1, a.wait_limit_ns);
    }
    // The rows' results are lost: leave zeros (whole key range) or an empty
    // part that the combine kernel gives no weight, never stale data.
    if (parts == 1) {
      uint32_t* out32 = static_cast<uint32_t*>(a.out);
      for (int j = 0; j < NO; ++j) {
        if (v_lo) out32[(row_lo + j * 8 + 2 * c) / 2] = 0u;
        if (v_hi) out32[(row_hi + j * 8 + 2 * c) / 2] = 0u;
      }
    } else if (c == 0) {
      const int64_t pl = (row_lo / D) * a.max_parts + part, ph = (row_hi / D) * a.max_parts + part;
      if (v_lo) a.ws_ml[pl] = make_float2(-CUDART_INF_F, 0.f);
      if (v_hi) a.ws_ml[ph] = make_float2(-CUDART_INF_F, 0.f);
    }
    return;
  }

  // ---- epilogue: out = O / l, rounded to the q dtype
  l_lo += __shfl_xor_sync(FULL, l_lo, 1);
  l_lo += __shfl_xor_sync(FULL, l_lo, 2);
  l_hi += __shfl_xor_sync(FULL, l_hi, 1);
  l_hi += __shfl_xor_sync(FULL, l_hi, 2);
  float i_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, i_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
  if constexpr (FP8) {
    const float vs = a.v_scale[kvh];
    i_lo *= vs;
    i_hi *= vs;
  }
  // pairs of adjacent output dims d, d+1 and their accumulators: 16-bit cache
  // columns 8j + 2c (+1) of n-tile j; E4M3 dims 16m + 4c + 2i (+1) of the
  // even / odd n-tiles 2m, 2m+1
  auto pair_dim = [&](int pi) { return FP8 ? 16 * (pi / 2) + 4 * c + 2 * (pi % 2) : 8 * pi + 2 * c; };
  auto pair_val = [&](int pi, int hi, float& x, float& y) {
    if constexpr (FP8) {
      x = o[2 * (pi / 2)][2 * hi + pi % 2];
      y = o[2 * (pi / 2) + 1][2 * hi + pi % 2];
    } else {
      x = o[pi][2 * hi];
      y = o[pi][2 * hi + 1];
    }
  };
  if (parts == 1) {
    uint32_t* out32 = static_cast<uint32_t*>(a.out);
#pragma unroll
    for (int pi = 0; pi < NO; ++pi) {
      float x, y;
      pair_val(pi, 0, x, y);
      if (v_lo) out32[(row_lo + pair_dim(pi)) / 2] = pack2<QBF>(x * i_lo, y * i_lo);
      pair_val(pi, 1, x, y);
      if (v_hi) out32[(row_hi + pair_dim(pi)) / 2] = pack2<QBF>(x * i_hi, y * i_hi);
    }
    return;
  }
  // a part of a split key range: (max, sum) and the output normalised by this
  // part's sum, per row (a row that sees none of this part's tokens leaves
  // max = -inf, sum = 0); the combine kernel merges the parts
  const int64_t pl = (row_lo / D) * a.max_parts + part, ph = (row_hi / D) * a.max_parts + part;
  if (v_lo && c == 0) a.ws_ml[pl] = make_float2(m_lo, l_lo);
  if (v_hi && c == 0) a.ws_ml[ph] = make_float2(m_hi, l_hi);
#pragma unroll
  for (int pi = 0; pi < NO; ++pi) {
    float x, y;
    pair_val(pi, 0, x, y);
    if (v_lo)
      *reinterpret_cast<float2*>(a.ws_o + pl * D + pair_dim(pi)) = make_float2(x * i_lo, y * i_lo);
    pair_val(pi, 1, x, y);
    if (v_hi)
      *reinterpret_cast<float2*>(a.ws_o + ph * D + pair_dim(pi)) = make_float2(x * i_hi, y * i_hi);
  }
}

// Merge the parts of a split key range: part p of row r left (m_p, l_p) and
// o_p normalised by l_p (base-2 units), so with M = max_p m_p and
// w_p = l_p 2^(m_p - M): out = sum_p w_p o_p / sum_p w_p. One warp per
// (query token, head); rows whose range was not split were written directly.
template <class QF, int D>
__global__ void __launch_bounds__(128) paged_prefill_combine(const PrefillArgs a, int qt) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x * 4 + warp, i = blockIdx.y, s = blockIdx.z;
  if (h >= a.num_heads) return;
  const int q0 = a.cu_query_lens[s], qlen = a.cu_query_lens[s + 1] - q0;
  if (i >= qlen) return;
  int ctx = a.context_lens[s];
  ctx = ctx < 0 ? 0 : (ctx > a.ctx_limit ? a.ctx_limit : ctx);
  if (qlen > ctx) return;  // rows zeroed by the main kernel
  const int tok0 = (i / qt) * qt, ntok = min(qt, qlen - tok0);
  const int pos0 = ctx - qlen + tok0;
  const int ntiles_all = (pos0 + ntok - 1) / kTileRows + 1;
  const int parts = (ntiles_all + a.partition_tiles - 1) / a.partition_tiles;
  if (parts <= 1) return;
  const int64_t row = static_cast<int64_t>(q0 + i) * a.num_heads + h;
  const float2* ml = a.ws_ml + row * a.max_parts;
  float M = -CUDART_INF_F;
  for (int p = lane; p < parts; p += 32) M = fmaxf(M, ml[p].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) acc[j] = 0.f;
  float L = 0.f;
  const float* op = a.ws_o + row * a.max_parts * D;
  for (int p = 0; p < parts; ++p) {
    const float2 v = ml[p];
    // a part that saw no token of this row (or gave up) has no weight, and
    // its o may never have been written: it is not read
    if (v.x == -CUDART_INF_F || !(v.y > 0.f)) continue;
    const float w = v.y * exp2f(v.x - M);
    L += w;
#pragma unroll
    for (int j = 0; j < PER; ++j) acc[j] = fmaf(w, op[p * D + lane + 32 * j], acc[j]);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) store_out(QF{}, a.out, row * D + lane + 32 * j, acc[j] * inv);
}

template <class QF, class CF, int D, int G>
cudaError_t launch_one(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                       int32_t max_query_len, cudaStream_t stream) {
  constexpr int QT = kPrefillRows / G;
  constexpr int STAGE = 2 * Tile<CF, D>::BYTES;
  const size_t smem = 1024 + kPrefillStages * STAGE + 16 * kPrefillStages;
  auto kern = paged_prefill_kernel<QF, CF, D, G>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  static_assert(QT == prefill_tokens_per_cta(G), "tokens per CTA");
  e = launch_pdl(kern, dim3(static_cast<unsigned>(a.q_tiles * a.max_parts), a.num_kv_heads,
                            a.num_seqs),
                 kPrefillWarps * 32, smem, stream, a, kmap, vmap);
  if (e != cudaSuccess || a.max_parts <= 1) return e;
  return launch_pdl(paged_prefill_combine<QF, D>,
                    dim3((a.num_heads + 3) / 4, static_cast<unsigned>(max_query_len), a.num_seqs),
                    128, 0, stream, a, QT);
}

}  // namespace

cudaError_t launch_prefill_combine(const PrefillArgs& a, int q_dtype, int head_dim, int qt,
                                   int32_t max_query_len, cudaStream_t stream) {
  const dim3 grid((a.num_heads + 3) / 4, static_cast<unsigned>(max_query_len), a.num_seqs);
  if (q_dtype == kF16 && head_dim == 64)
    return launch_pdl(paged_prefill_combine<F16, 64>, grid, 128, 0, stream, a, qt);
  if (q_dtype == kF16 && head_dim == 128)
    return launch_pdl(paged_prefill_combine<F16, 128>, grid, 128, 0, stream, a, qt);
  if (q_dtype == kBF16 && head_dim == 64)
    return launch_pdl(paged_prefill_combine<BF16, 64>, grid, 128, 0, stream, a, qt);
  if (q_dtype == kBF16 && head_dim == 128)
    return launch_pdl(paged_prefill_combine<BF16, 128>, grid, 128, 0, stream, a, qt);
  return cudaErrorNotSupported;
}

cudaError_t launch_prefill(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                           int q_dtype, int cache_dtype, int head_dim, int group,
                           int32_t max_query_len, cudaStream_t stream) {
#define PAGED_PREFILL(QF, CF, d, g) \
  if (head_dim == d && group == g)  \
    return launch_one<QF, CF, d, g>(a, kmap, vmap, max_query_len, stream);
#define PAGED_PREFILL_ALL(QF, CF)                                                           \
  PAGED_PREFILL(QF, CF, 64, 1) PAGED_PREFILL(QF, CF, 64, 2) PAGED_PREFILL(QF, CF, 64, 4)     \
  PAGED_PREFILL(QF, CF, 64, 8) PAGED_PREFILL(QF, CF, 128, 1) PAGED_PREFILL(QF, CF, 128, 2)   \
  PAGED_PREFILL(QF, CF, 128, 4) PAGED_PREFILL(QF, CF, 128, 8)
  const bool fp8 = cache_dtype == kE4M3;
  if (q_dtype == kF16) {
    if (fp8) {
      PAGED_PREFILL_ALL(F16, E4M3)
    } else {
      PAGED_PREFILL_ALL(F16, F16)
    }
  } else if (q_dtype == kBF16) {
    if (fp8) {
      PAGED_PREFILL_ALL(BF16, E4M3)
    } else {
      PAGED_PREFILL_ALL(BF16, BF16)
    }
  }
#undef PAGED_PREFILL_ALL
#undef PAGED_PREFILL
  return cudaErrorNotSupported;
}

}  // namespace paged
