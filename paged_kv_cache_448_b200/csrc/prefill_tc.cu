// prefill_tc.cu — the multi-token query on the 5th-generation tensor cores.
//
// Same operation as prefill_kernel.cu ("vLLM推理引擎架构：PagedAttention机制
// 与高吞吐推理" §2.3 with a query of several trailing tokens per sequence and
// the causal rule): rows cu[s] .. cu[s+1]-1 of the query are the last
// positions p_i of sequence s and see its tokens t <= p_i.
//
// A CTA holds NG row groups of 128 rows (row = one (query token, head of the
// kv-head's group); NG = 2 once the chunks fill 256 rows) and 4 NG + 3 warps.
// A step is 128 tokens with two groups (S = Q K^T with N = 128), 64 with one:
//  * softmax warps, 4 per group: one row per thread and per tensor-memory
//    lane. They write Q once into shared memory (128-byte swizzled, K-major),
//    then per step load their row of S from tensor memory (the maximum first,
//    then the probabilities), mask tokens after the row's position, and run
//    the base-2 online softmax with a lazily updated maximum (it moves only
//    when a row's maximum grows by more than 8, so probabilities stay below
//    2^8 and O in tensor memory is rarely rescaled). They store P back into
//    tensor memory over the S it came from, 32 tokens into their own 32
//    columns (f16/bf16 pairs, bf16 as hi + lo parts), and post it;
//  * the MMA warp (one thread) owns the tensor memory: per group S (two
//    64-column buffers with one group, one 128-column buffer with two) and D
//    columns of O. It polls and issues whatever is ready, per group: S of the
//    next step once K landed and the S buffer's last O += P V completed, and
//    O += P V of a step (A = P from tensor memory, V read MN-major) once the
//    group posted P and V landed. With two groups, one group's MMAs run under
//    the other's softmax;
//  * two TMA warps, one per ring, load K and V of a step into 2-stage rings
//    (16-row boxes of one 128-byte segment each, so a stage is
//    [segment][step rows][128 B]), the boxes of a step from all lanes of the
//    warp at once, and refill a stage when the MMAs that read it completed.
// Units of at most 64 rows (a few draft tokens x the query group) hold each
// row twice, in lanes r and r + 64: the two copies take the lower and upper
// 32 tokens of every step with their own maximum, sum and O, and are merged
// before the epilogue (the MMAs cost 128 rows either way; the softmax work
// per thread halves).
// The epilogue divides each row of O by its sum and stores it. When the key
// range is split (few CTAs), a CTA takes one part of its 16-token tiles and
// writes (max, sum) and its normalised O per row for the combine kernel, as
// the mma.sync kernel does.
// An E4M3 cache (head_dim 128: a 128-byte row) runs on kind::f8f6f4 with the
// cache tiles as they arrive: Q goes to shared memory as E4M3 hi + lo parts
// (q * 2^e = hi + lo, e a power of two per row that puts max |q| below 2^8,
// undone in the row's logit scale with the kv-head's K scale), so S takes two
// 8-bit MMAs per K step; P (<= 2^8 under the lazy maximum) goes to tensor
// memory as an E4M3 hi part and an E5M2 residual, so O += P V takes two
// 8-bit MMAs with V read MN-major; the V scale applies in the epilogue.
// Every wait is bounded by wall time. A wait that gives up sets a shared
// abort flag that ends the other roles' waits; the MMA warp lets its issued
// MMAs and the TMA warp its issued loads complete (bounded) before the
// tensor memory is freed, and the failure is recorded in the error word.
#include <math_constants.h>

#include <type_traits>

#include "consumer_mma.cuh"
#include "decode_args.h"
#include "decode_kernel.cuh"
#include "device_common.cuh"
#include "prefill_args.h"
#include "tc_common.cuh"

namespace paged {
namespace {

constexpr int kTcRows = 128;       // M: rows of one row group (one MMA)
constexpr uint32_t kTmemGroup = 256;  // tensor-memory columns per row group: S, then O
constexpr uint32_t kTmemO = 128;      // column of O within the group

// NG row groups of 128 rows share each K/V step (NG = 2: 256 rows, eight
// softmax warps, and two independent MMA streams per step). With one group a
// step is 64 tokens and S has two buffers (S of step k+1 is computed under
// the softmax of step k); with two groups a step is 128 tokens (S = Q K^T
// with N = 128, which keeps the tensor core ahead of its shared-memory
// operand reads) and each group has one S buffer: the other group's work
// fills the tensor core while a group's softmax runs.
template <class QF, class CF, int D, int G, int NG>
struct TcCfg {
  static constexpr int NT = NG == 2 ? 128 : 64;      // tokens per step
  static constexpr int SB = NG == 2 ? 1 : 2;         // S buffers per group
  static constexpr int H = NT / 64;                  // 64-token halves of a step
  static constexpr bool FP8 = CF::kBytes == 1;
  static constexpr bool BF = std::is_same<QF, BF16>::value;
  static constexpr int NSEG = D * CF::kBytes / 128;  // 128-byte segments of a cache row
  static_assert(NSEG >= 1, "rows of at least 128 bytes");
  static constexpr int ROWS = NG * kTcRows;
  static constexpr int QT = ROWS / G;               // query tokens per CTA
  // Q of one group: NSEG segments (16-bit), or the E4M3 hi and lo parts
  static constexpr int QPART = kTcRows * 128;
  static constexpr int QG_BYTES = (FP8 ? 2 : NSEG) * QPART;
  static constexpr int KV_SEG = NT * 128;           // one segment of K or V in a stage
  static constexpr int KV_BYTES = NSEG * KV_SEG;    // one stage of K (or V)
  // ring depths (K, needed first by S, and V); deeper rings (4 for 16-bit
  // caches, 6 for E4M3, with two row groups) measured no faster
  static constexpr int KR = 2, VR = 2;
  static constexpr int OFF_K = NG * QG_BYTES;                   // K ring
  static constexpr int OFF_V = OFF_K + KR * KV_BYTES;           // V ring
  static constexpr int BYTES = OFF_V + VR * KV_BYTES;
  static constexpr uint32_t TMEM_COLS = NG * kTmemGroup;
  static constexpr uint32_t IDESC_S = FP8 ? tc::idesc_f8<0, 0, kTcRows, NT, false>()
                                           : tc::idesc_f16<BF, kTcRows, NT, false>();
  static constexpr uint32_t IDESC_PV = FP8 ? tc::idesc_f8<0, 0, kTcRows, D, true>()
                                            : tc::idesc_f16<BF, kTcRows, D, true>();
  static constexpr uint32_t IDESC_PV_LO = tc::idesc_f8<1, 0, kTcRows, D, true>();  // E5M2 P
  static_assert(SB * NT <= static_cast<int>(kTmemO), "S buffers below O");
  static_assert(BYTES + 1024 <= 227 * 1024, "shared memory of one CTA");
};

// 32 consecutive fp32 columns of this thread's lane into v[0..31], without
// waiting (tcgen05.wait::ld follows, then tie16 on the registers).
__device__ __forceinline__ void ld32f_nowait(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
        "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]),
        "=f"(v[14]), "=f"(v[15]), "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]),
        "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]), "=f"(v[24]), "=f"(v[25]),
        "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]), "=f"(v[30]), "=f"(v[31])
      : "r"(taddr)
      : "memory");
}

// An empty statement that takes and gives back 16 registers: placed after a
// wait for tensor-memory loads, it keeps every use of the loaded values after
// the wait.
__device__ __forceinline__ void tie16(float* v) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]));
}

// 16-byte chunk `c` of row `r` of a 128-byte-swizzled [rows][128 B] tile.
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_pair(bool bf, float lo, float hi) {
  return bf ? pack2<true>(lo, hi) : pack2<false>(lo, hi);
}

// Two 16-bit query values (low half first) as floats.
template <class QF>
__device__ __forceinline__ float2 unpack_q(uint32_t w) {
  if constexpr (std::is_same<QF, BF16>::value)
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  const __half2 h = *reinterpret_cast<const __half2*>(&w);
  return __half22float2(h);
}

constexpr int kOrderSeqs = 256;  // launches of up to this many sequences are reordered

// The sequence of rank `rank` when the sequences are ordered by context length,
// longest first (ties by index): sequence i has rank #{j : len_j > len_i} +
// #{j < i : len_j == len_i}, a permutation for any lengths. Launches of more
// than kOrderSeqs sequences keep their order (rank = sequence). Every thread of
// the CTA calls it (two barriers).
__device__ __forceinline__ int sequence_of_rank(const int32_t* context_lens, int n, int rank,
                                                int32_t* lens, int* pick) {
  if (n > kOrderSeqs) return rank;
  for (int i = threadIdx.x; i < n; i += blockDim.x) lens[i] = context_lens[i];
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int32_t li = lens[i];
    int r = 0;
#pragma unroll 4
    for (int j = 0; j < n; ++j) {
      const int32_t lj = lens[j];
      r += (lj > li) | ((lj == li) & (j < i));
    }
    if (r == rank) *pick = i;
  }
  __syncthreads();
  return *pick;
}

template <class QF, class CF, int D, int G, int NG>
__global__ void __launch_bounds__(NG * kTcRows + 96, NG == 1 ? 2 : 1)
    paged_prefill_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap) {
  using C = TcCfg<QF, CF, D, G, NG>;
  constexpr bool BF = C::BF, FP8 = C::FP8;
  constexpr int NSEG = C::NSEG, QT = C::QT, KR = C::KR, VR = C::VR, NT = C::NT, TR = kTileRows;
  constexpr int SB = C::SB, H = C::H;
  constexpr int kMma = NG * kTcRows / 32;   // warp issuing the MMAs (owns the tensor memory)
  constexpr int kLoader = kMma + 1;         // warps issuing the TMA loads: K, then V

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  auto sq = [&](int g) { return smem + g * C::QG_BYTES; };
  auto sk = [&](int k) { return smem + C::OFF_K + (k % KR) * C::KV_BYTES; };
  auto sv = [&](int k) { return smem + C::OFF_V + (k % VR) * C::KV_BYTES; };
  // K / V rings: *full when a stage's boxes landed, *empty when the MMAs that
  // read it completed (both groups). Per group g: s_bar[g][b] S buffer b
  // computed; p_bar[g][b] the group's softmax warps wrote P of a step of parity
  // b (and rescaled O); pv_bar[g][b] O += P V of such a step done.
  __shared__ uint64_t kfull[KR], kempty[KR], vfull[VR], vempty[VR], s_bar[NG][2], p_bar[NG][2],
      pv_bar[NG][2], drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int aborted;
  __shared__ int32_t order_lens[kOrderSeqs];
  __shared__ int order_pick;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t lim = a.wait_limit_ns;
  if (tid == 0) {
    for (int r = 0; r < KR; ++r) {
      mbar_init(&kfull[r], 1);
      mbar_init(&kempty[r], 1);
    }
    for (int r = 0; r < VR; ++r) {
      mbar_init(&vfull[r], 1);
      mbar_init(&vempty[r], 1);
    }
    for (int g = 0; g < NG; ++g)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&s_bar[g][b], 1);
        mbar_init(&p_bar[g][b], kTcRows / 32);
        mbar_init(&pv_bar[g][b], 1);
      }
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
    aborted = 0;
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // This CTA's unit. CTAs are dispatched in the order of their linear index,
  // and the units' work differs with the context length, so the launch takes
  // the sequences longest context first and, within one, its last query tile
  // (the most keys) first: list scheduling with the longest jobs first keeps
  // the last wave short.
  const int per_seq = static_cast<int>(gridDim.x * gridDim.y);
  const int64_t lin = blockIdx.x + static_cast<int64_t>(gridDim.x) *
                                       (blockIdx.y + static_cast<int64_t>(gridDim.y) * blockIdx.z);
  const int rank = static_cast<int>(lin / per_seq), in_seq = static_cast<int>(lin % per_seq);
  const int kvh = in_seq / static_cast<int>(gridDim.x), xi = in_seq % static_cast<int>(gridDim.x);
  const int z = a.q_tiles - 1 - xi % a.q_tiles, part = xi / a.q_tiles;
  const int s = sequence_of_rank(a.context_lens, a.num_seqs, rank, order_lens, &order_pick);
  const bool first_unit = z == 0 && part == 0 && kvh == 0 && s == 0;

  const int q0 = a.cu_query_lens[s];
  const int qlen = a.cu_query_lens[s + 1] - q0;
  int ctx = a.context_lens[s];
  if (ctx > a.ctx_limit || ctx < 0) {
    if (tid == 0 && z == 0 && kvh == 0) report(a.err, kErrContextClipped);
    ctx = ctx < 0 ? 0 : a.ctx_limit;
  }
  const int tok0 = z * QT;
  if (tok0 >= qlen) return;  // ragged chunk lengths: nothing for this CTA
  const int ntok = min(QT, qlen - tok0);
  // One row group whose units hold at most 64 rows (short chunks, a few draft
  // tokens): lanes 64..127 repeat rows 0..63, and the two copies of a row take
  // the lower and the upper 32 tokens of every step, each with its own
  // maximum, sum and O (rows of one MMA), merged at the end like two parts of
  // a split key range. The tensor work is the same (the MMA has 128 rows
  // either way); each softmax thread handles half as many tokens.
  const bool dup = NG == 1 && a.dup_rows != 0;
  const int half = dup ? tid / 64 : 0;  // softmax threads: which copy
  // softmax threads: row srow of the unit = token srow / G, head srow % G
  const int srow = dup ? (tid & 63) : tid;
  const int tok = srow / G;
  const bool valid = warp < kMma && tok < ntok;
  const bool out_row = valid && half == 0;  // the copy that writes the row's result
  const int64_t row_off =
      (static_cast<int64_t>(q0 + tok0 + tok) * a.num_heads + kvh * G + srow % G) * D;
  if (qlen > ctx) {  // a query longer than its context: rows become zeros
    if (part > 0) return;
    if (tid == 0 && z == 0 && kvh == 0) report(a.err, kErrQueryLonger);
    if (out_row) {
      uint4* o4 = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.out) + row_off * 2);
      for (int c = 0; c < D / 8; ++c) o4[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    return;
  }
  const int pos0 = ctx - qlen + tok0;
  const int p_max = pos0 + ntok - 1;
  // 16-token tiles holding tokens 0..p_max, cut into parts of partition_tiles
  // (a multiple of the NT / 16 tiles of a step); this CTA takes part `part`: tiles
  // tbase .. tend-1, steps kbase .. kbase+nsteps-1
  const int ntiles_all = p_max / TR + 1;
  const int parts = (ntiles_all + a.partition_tiles - 1) / a.partition_tiles;
  if (part >= parts) return;
  const int tbase = part * a.partition_tiles;
  const int tend = min(ntiles_all, tbase + a.partition_tiles);
  const int kbase = tbase / (NT / TR);
  const int nsteps = (tend - tbase + NT / TR - 1) / (NT / TR);

  __syncthreads();  // barrier initialisation visible to every thread
  if (warp == kMma) tc::alloc(&tmem_slot, C::TMEM_COLS);
  float qscale = a.scale_log2;  // logit scale of this thread's row (base 2)
  if (warp < kMma) {
    // Q rows -> shared memory (per group, 128-byte swizzle, K-major), zeros past the chunk
    const int g = tid / kTcRows, rr = tid % kTcRows;
    const uint4* q4 = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.query) +
                                                     row_off * 2);
    if constexpr (!FP8) {
#pragma unroll
      for (int sg = 0; sg < NSEG; ++sg)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = valid ? q4[sg * 8 + c] : make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(sq(g) + sg * C::QPART + sw128(rr, c)) = v;
        }
    } else {
      // row maximum, then q * 2^e = hi + lo (E4M3 each), 16 dims per 16-byte chunk
      float mq = 0.f;
      if (valid) {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 v = q4[c];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = unpack_q<QF>(w[j]);
            mq = fmaxf(mq, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        }
      }
      int e = 0;
      if (mq > 0.f && isfinite(mq)) {
        int k2;
        frexpf(mq, &k2);                  // mq < 2^k2
        e = min(max(8 - k2, -100), 100);  // mq * 2^e < 2^8
      }
      qscale *= a.k_scale[kvh] * ldexpf(1.f, -e);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t hw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u};
        if (valid) {
          const uint4 v0 = q4[2 * c], v1 = q4[2 * c + 1];
          const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f0 = unpack_q<QF>(w[2 * j]), f1 = unpack_q<QF>(w[2 * j + 1]);
            tc::split_fp8x4<false>(ldexpf(f0.x, e), ldexpf(f0.y, e), ldexpf(f1.x, e),
                               ldexpf(f1.y, e), hw[j], lw[j]);
          }
        }
        *reinterpret_cast<uint4*>(sq(g) + sw128(rr, c)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(sq(g) + C::QPART + sw128(rr, c)) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
    }
    fence_proxy_async_smem();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;

  if (warp >= kLoader) {
    // ================= TMA loads: a K warp and a V warp =================
    // Each ring has a warp of its own, so a V stage (held until O += P V)
    // never holds back a K load. The boxes of a step (16 rows of one 128-byte
    // segment each) leave from all lanes of the warp at once, lane b issuing
    // box b; each lane reads its block id one step ahead.
    constexpr int BOXES = (NT / TR) * NSEG;
    static_assert(BOXES <= 32, "one box per lane");
    const bool is_v = warp == kLoader + 1;
    const int R = is_v ? VR : KR;
    uint64_t* full = is_v ? vfull : kfull;
    uint64_t* empty = is_v ? vempty : kempty;
    const CUtensorMap* map = is_v ? &vmap : &kmap;
    const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks_per_seq;
    const uint64_t policy = l2_policy_evict_last();  // other query tiles read them too
    const int bj = lane / NSEG, bsg = lane % NSEG;   // this lane's 16-row tile and segment
    auto load_id = [&](int k) {
      const int t = (kbase + k) * (NT / TR) + bj;
      return lane < BOXES && k < nsteps && t < tend ? table[(t * TR) / a.block_size] : 0;
    };
    bool ok = true;
    int issued = 0;
    int32_t bid = load_id(0);
    for (int k = 0; k < nsteps; ++k) {
      const int32_t nbid = load_id(k + 1);  // in flight during the wait below
      if (k >= R)
        ok = __all_sync(0xffffffffu, mbar_wait(&empty[k % R], ((k - R) / R) & 1, lim, &aborted));
      if (!ok) break;
      issued = k + 1;
      const int t_begin = (kbase + k) * (NT / TR), t_end = min(tend, t_begin + NT / TR);
      if (!is_v && a.skip_tile >= t_begin - tbase && a.skip_tile < t_end - tbase &&
          skip_unit_for_test(a.skip_tile, a.skip_tile, first_unit)) {
        bid = nbid;
        continue;  // (the K warp leaves it out: the step never completes)
      }
      uint64_t* bar = &full[k % R];
      if (lane == 0)
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(NSEG * (t_end - t_begin) * TR * 128));
      __syncwarp();
      const int t = t_begin + bj;
      if (lane < BOXES && t < t_end) {
        int32_t b = bid;
        if (b < 0 || b >= a.num_blocks) {
          if (!is_v) report(a.err, kErrBadBlockId);
          b = -1;  // read as a box outside the pool: zero-filled
        }
        const int32_t row0 = b >= 0 ? b * a.block_size + (t * TR) % a.block_size : -TR;
        uint8_t* dst = (is_v ? sv(k) : sk(k)) + bsg * C::KV_SEG + bj * TR * 128;
        tma_load_4d(dst, map, bar, 0, row0, kvh, bsg, policy);
      }
      __syncwarp();
      bid = nbid;
    }
    if (!ok && lane == 0) {
      aborted = 1;
      report(a.err, kErrWaitTimeout);
    }
    // before the CTA's shared memory goes away every issued load must have
    // landed (the last use of each stage; earlier ones completed already)
    if (lane == 0)
      for (int j = max(0, issued - R); j < issued; ++j) mbar_wait(&full[j % R], (j / R) & 1, lim);
    __syncwarp();  // whole warps reach the CTA barrier below
  } else if (warp == kMma) {
    // ================= MMA issue (one thread) =================
    if (lane == 0) {
      // descriptors computed once; a k-step or stage offset is added to the
      // start-address field (bits 0-13, in 16-byte units)
      uint64_t qd[NG];
      for (int g = 0; g < NG; ++g) qd[g] = tc::sw128_desc(sq(g), 16, 1024);
      const uint64_t kd0 = tc::sw128_desc(sk(0), 16, 1024);
      const uint64_t vd0 = tc::sw128_desc(sv(0), NT * 128, 1024);
      // S = Q K^T of step k for group g (K landed, the S buffer free)
      auto issue_s = [&](int g, int k) {
        const uint32_t t_s = tmem + g * kTmemGroup + (SB == 2 ? (k & 1) * NT : 0);
        const uint64_t kd = kd0 + static_cast<uint64_t>(((k % KR) * C::KV_BYTES) >> 4);
        if constexpr (!FP8) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int sg = kk / 4, off = (kk % 4) * 32;
            tc::mma_f16(t_s, qd[g] + static_cast<uint64_t>((sg * C::QPART + off) >> 4),
                        kd + static_cast<uint64_t>((sg * C::KV_SEG + off) >> 4), C::IDESC_S,
                        kk > 0);
          }
        } else {
          // Q hi, then Q lo, each 4 K steps of 32 dims (32 bytes) along the row
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int part = kk / 4, off = (kk % 4) * 32;
            tc::mma_f8(t_s, qd[g] + static_cast<uint64_t>((part * C::QPART + off) >> 4),
                       kd + static_cast<uint64_t>(off >> 4), C::IDESC_S, kk > 0);
          }
        }
        tc::commit(&s_bar[g][k & 1]);
      };
      // O += P V of step j for group g (P posted, V landed). P of step j lies
      // over its S: per 32 tokens (quarter qq) the 16-bit pairs (or E4M3
      // codes) from column 32 qq, the bf16 (or E5M2) residual 16 (8) columns
      // further; 8 columns per k-step
      auto issue_pv = [&](int g, int j) {
        const uint32_t t_grp = tmem + g * kTmemGroup;
        const uint32_t t_p = t_grp + (SB == 2 ? (j & 1) * NT : 0);
        const uint32_t t_o = t_grp + kTmemO;
        const uint64_t vd = vd0 + static_cast<uint64_t>(((j % VR) * C::KV_BYTES) >> 4);
        if constexpr (!FP8) {
#pragma unroll
          for (int kk = 0; kk < NT / 16; ++kk) {
            const uint32_t col = (kk / 2) * 32 + (kk % 2) * 8;
            const uint64_t bv = vd + static_cast<uint64_t>((kk * 16 * 128) >> 4);
            tc::mma_f16_ts(t_o, t_p + col, bv, C::IDESC_PV, j > 0 || kk > 0);
            if constexpr (BF) tc::mma_f16_ts(t_o, t_p + col + 16, bv, C::IDESC_PV, true);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < NT / 32; ++kk) {  // 32 tokens per k-step
            const uint32_t col = kk * 32;
            const uint64_t bv = vd + static_cast<uint64_t>((kk * 32 * 128) >> 4);
            tc::mma_f8_ts(t_o, t_p + col, bv, C::IDESC_PV, j > 0 || kk > 0);
            tc::mma_f8_ts(t_o, t_p + col + 8, bv, C::IDESC_PV_LO, true);
          }
        }
        tc::commit(&pv_bar[g][j & 1]);
      };
      // A K stage is released once every group's S of its step was issued, a
      // V stage once every group's O += P V (a commit completes when all of
      // the thread's earlier MMAs have).
      int k_rel = 0, v_rel = 0;  // K / V stages released so far (steps)
      bool ok = true;
      if constexpr (NG == 2) {
        // Two groups, one S buffer each: a group's chain is softmax, O += P V,
        // its next S (once O += P V, which read P over S, completed). The
        // MMAs go in a fixed order per step: O += P V of group 0, its next S,
        // then the same for group 1, so that the groups' tensor work
        // alternates and a group's next S follows its O += P V at once. (Issued
        // greedily, whatever was ready first, the groups drifted into each
        // other: a group's O += P V queued behind the other's work.)
        ok = mbar_wait(&kfull[0], 0, lim, &aborted);
        if (ok) {
          tc::fence_after_sync();
          issue_s(0, 0);
          issue_s(1, 0);
          tc::commit(&kempty[0]);
          k_rel = 1;
        }
        for (int k = 0; ok && k < nsteps; ++k) {
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            ok = (g > 0 || mbar_wait(&vfull[k % VR], (k / VR) & 1, lim, &aborted)) &&
                 mbar_wait(&p_bar[g][k & 1], (k >> 1) & 1, lim, &aborted);
            if (!ok) break;
            tc::fence_after_sync();
            issue_pv(g, k);
            if (g == NG - 1) {
              tc::commit(&vempty[k % VR]);
              v_rel = k + 1;
            }
            if (k + 1 < nsteps) {
              ok = mbar_wait(&pv_bar[g][k & 1], (k >> 1) & 1, lim, &aborted) &&
                   mbar_wait(&kfull[(k + 1) % KR], ((k + 1) / KR) & 1, lim, &aborted);
              if (!ok) break;
              tc::fence_after_sync();
              issue_s(g, k + 1);
              if (g == NG - 1) {
                tc::commit(&kempty[(k + 1) % KR]);
                k_rel = k + 2;
              }
            }
          }
        }
      } else {
        // One group, two S buffers: the thread polls and issues whatever is
        // ready. ns = next step whose S is issued, np = next step whose
        // O += P V is issued:
        //  * S(k): K of step k landed and the S buffer is free, i.e. O += P V
        //    of step k - 2 (which read the P written over that S) completed;
        //  * O += P V (k): S(k) issued, P of step k posted, V landed.
        // Gives up after the wait limit without progress.
        int ns = 0, np = 0;
        uint64_t t_last = global_timer_ns();
        while (np < nsteps) {
          bool progress = false;
          if (np < ns && mbar_test_wait(&p_bar[0][np & 1], (np >> 1) & 1) &&
              mbar_test_wait(&vfull[np % VR], (np / VR) & 1)) {
            tc::fence_after_sync();
            issue_pv(0, np);
            tc::commit(&vempty[np % VR]);
            v_rel = ++np;
            progress = true;
          }
          if (ns < nsteps &&
              (ns < SB || mbar_test_wait(&pv_bar[0][(ns - SB) & 1], ((ns - SB) >> 1) & 1)) &&
              mbar_test_wait(&kfull[ns % KR], (ns / KR) & 1)) {
            tc::fence_after_sync();
            issue_s(0, ns);
            tc::commit(&kempty[ns % KR]);
            k_rel = ++ns;
            progress = true;
          }
          if (progress) {
            t_last = global_timer_ns();
          } else if (aborted || global_timer_ns() - t_last > lim) {
            ok = false;
            break;
          }
        }
      }
      if (!ok) {
        // A wait gave up (never expected): let this CTA's MMAs finish (bounded)
        // before its tensor and shared memory go away.
        record_failure(a.diag, kSiteTcStep, z + a.q_tiles * part, kvh, s, k_rel, v_rel, nsteps,
                       NG);
        aborted = 1;
        report(a.err, kErrWaitTimeout);
        tc::commit(&drain_bar);
        mbar_wait(&drain_bar, 0, lim);
      }
    }
    __syncwarp();  // whole warps reach the CTA barrier below
  } else {
    // ================= softmax warps: one row per thread =================
    const int g = warp / 4;                      // row group
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t t_grp = tmem + g * kTmemGroup;
    const uint32_t t_o = t_grp + kTmemO + lane_base;
    const int rr = tid % kTcRows;                // row within the group = tensor-memory lane
    const int p_row = valid ? pos0 + tok : -1;
    const int kv_valid = min(ctx, tend * TR);    // tokens with loaded, real rows
    float m_used = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int k = 0; ok && k < nsteps; ++k) {
      ok = mbar_wait(&s_bar[g][k & 1], (k >> 1) & 1, lim, &aborted);
      if (!ok) break;
      tc::fence_after_sync();
      const uint32_t t_s = t_grp + (SB == 2 ? (k & 1) * NT : 0) + lane_base;
      const int tk0 = (kbase + k) * NT;
      // With a 16-bit cache and two groups the row's 128 logits are held at
      // once (read in one go: the loads issued together, one wait); with one
      // group, or an E4M3 cache, 64 at a time (measured on B200 with the
      // fixed MMA order, chunked prefill: bf16 687 against 657 TFLOP/s held
      // and not; E4M3 733 against 781, its softmax needing more registers)
      constexpr bool kHoldAll = NG == 2 && !FP8;
      float x[kHoldAll ? 128 : 64];
      float mraw = -CUDART_INF_F;
      // this row's logits of 64-token half h, masked after the row's position
      // (the causal rule) only where the half reaches past it
      auto load_half = [&](int h) {
        tc::ld64(t_s + h * 64, *reinterpret_cast<float(*)[64]>(x));
        const int t0 = tk0 + h * 64;
        if (t0 + 63 > p_row) {
#pragma unroll
          for (int i = 0; i < 64; ++i) x[i] = t0 + i <= p_row ? x[i] : -CUDART_INF_F;
        }
      };
      // maximum of 64 raw logits (the scale is positive): 8 partial chains
      auto half_max = [&]() {
        float m8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) m8[j] = x[j];
#pragma unroll
        for (int i = 8; i < 64; ++i) m8[i & 7] = fmaxf(m8[i & 7], x[i]);
        return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                     fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      };
      if constexpr (kHoldAll) {
#pragma unroll
        for (int q = 0; q < 4; ++q) ld32f_nowait(t_s + 32 * q, x + 32 * q);
        tc::wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) tie16(x + 32 * q), tie16(x + 32 * q + 16);
        // masked after the row's position (the causal rule) only where a
        // 32-token quarter reaches past it
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t0 = tk0 + 32 * q;
          if (t0 + 31 > p_row) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              x[32 * q + i] = t0 + i <= p_row ? x[32 * q + i] : -CUDART_INF_F;
          }
        }
        // row maximum of the raw logits (the scale is positive): 8 partial chains
        float m8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) m8[j] = x[j];
#pragma unroll
        for (int i = 8; i < 128; ++i) m8[i & 7] = fmaxf(m8[i & 7], x[i]);
        mraw = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                     fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      } else if (dup) {
        // this copy's 32 tokens of the step, masked after the row's position
        tc::ld32(t_s + 32 * half, *reinterpret_cast<float(*)[32]>(x));
        const int t0 = tk0 + 32 * half;
        if (t0 + 31 > p_row) {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = t0 + i <= p_row ? x[i] : -CUDART_INF_F;
        }
        float m8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) m8[j] = x[j];
#pragma unroll
        for (int i = 8; i < 32; ++i) m8[i & 7] = fmaxf(m8[i & 7], x[i]);
        mraw = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                     fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      } else {
        // the row maximum of the step: with two halves the upper one is read
        // first for its maximum alone and read again after the lower one
        if constexpr (H == 2) {
          load_half(1);
          mraw = half_max();
        }
        load_half(0);
        mraw = fmaxf(mraw, half_max());
      }
      const float mx = mraw * qscale;
      const bool rescale = mx > m_used + 8.f;   // false while the row sees nothing
      const float alpha = rescale ? tc::ex2(m_used - mx) : 1.f;
      if (rescale) m_used = mx;
      const float mu = m_used == -CUDART_INF_F ? 0.f : m_used;
      // P -> tensor memory over the S it came from, 32 probabilities at a time:
      // quarter qq of the step (tokens 32 qq ..) goes to its own 32 S columns,
      // from column 32 qq: 16-bit pairs (16 columns; for bf16 the residual
      // P - bf16(P) in the next 16), or E4M3 codes (8 columns, the E5M2
      // residual in the next 8). A quarter's writes touch no S column still
      // to be read.
      float lsum = 0.f;
      auto emit32 = [&](float* v, int h, int q) {
        float s8[8] = {};  // p = 2^(s * scale - m), summed in 8 partial chains
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = tc::ex2(fmaf(v[i], qscale, -mu));
          s8[i & 7] += v[i];
        }
        lsum += ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
        const uint32_t t_p = t_s + 32 * (2 * h + q);
        if constexpr (FP8) {
          uint32_t w[8], wl[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            tc::split_fp8x4<true>(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], w[i], wl[i]);
          tc::st8u(t_p, w);
          tc::st8u(t_p + 8, wl);
        } else {
          uint32_t w[16], wl[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            w[i] = pack_pair(BF, v[2 * i], v[2 * i + 1]);
            if constexpr (BF)
              wl[i] = pack2<true>(v[2 * i] - __uint_as_float(w[i] << 16),
                                  v[2 * i + 1] - __uint_as_float(w[i] & 0xffff0000u));
          }
          tc::st16u(t_p, w);
          if constexpr (BF) tc::st16u(t_p + 16, wl);
        }
      };
      if constexpr (kHoldAll) {
#pragma unroll
        for (int q = 0; q < 4; ++q) emit32(x + 32 * q, q / 2, q % 2);
      } else if (dup) {
        // this copy's quarter of P, and zeros where the other copy's tokens
        // go (those are the other lane's, P of this lane has no weight there)
        emit32(x, 0, half);
        const uint32_t t_z = t_s + 32 * (1 - half);
        if constexpr (FP8) {
          const uint32_t zw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          tc::st8u(t_z, zw);
          tc::st8u(t_z + 8, zw);
        } else {
          uint32_t zw[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) zw[i] = 0u;
          tc::st16u(t_z, zw);
          if constexpr (BF) tc::st16u(t_z + 16, zw);
        }
      } else {
        emit32(x, 0, 0);
        emit32(x + 32, 0, 1);
      }
      if constexpr (H == 2 && !kHoldAll) {
        // the upper half again (E4M3 cache), a quarter at a time (measured on
        // B200: 701 against 670 TFLOP/s for the whole half in one read)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float y[32];
          tc::ld32(t_s + 64 + 32 * q, y);
          const int t0 = tk0 + 64 + 32 * q;
          if (t0 + 31 > p_row) {
#pragma unroll
            for (int i = 0; i < 32; ++i) y[i] = t0 + i <= p_row ? y[i] : -CUDART_INF_F;
          }
          emit32(y, 1, q);
        }
      }
      l = l * alpha + lsum;
      // O is rescaled (rare: the maximum moves lazily) after P is written, when
      // fewer registers are live, and before P is posted; only once O += P V
      // of step k-1 completed. With one S buffer it has: S of this step was
      // issued after it.
      if (k >= 1 && rescale) {
        if constexpr (SB == 2) {
          ok = mbar_wait(&pv_bar[g][(k - 1) & 1], ((k - 1) >> 1) & 1, lim, &aborted);
          if (!ok) break;
          tc::fence_after_sync();
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tc::ld32(t_o + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tc::st32(t_o + c * 32, o);
        }
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      // V rows without real data in this step (past the context, or tiles not
      // loaded) may hold anything, even NaN, and 0 * NaN is NaN inside the MMA;
      // every group's warps clear them (the same zeros) before their P is posted
      const int vrows = max(0, min(NT, kv_valid - tk0));
      if (vrows < NT) {
        uint8_t* vs = sv(k);
        ok = mbar_wait(&vfull[k % VR], (k / VR) & 1, lim, &aborted);  // the TMA writes come first
        if (!ok) break;
        for (int i = rr; i < (NT - vrows) * NSEG * 8; i += kTcRows) {
          const int r = vrows + i / (NSEG * 8), sg = (i / 8) % NSEG, c = i % 8;
          *reinterpret_cast<uint4*>(vs + sg * C::KV_SEG + r * 128 + c * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_bar[g][k & 1]);
    }
    if (ok)
      ok = mbar_wait(&pv_bar[g][(nsteps - 1) & 1], ((nsteps - 1) >> 1) & 1, lim, &aborted);
    // two copies of a row: the upper copy hands (maximum, sum, O) to the lower
    // through shared memory (Q's space, whose last reader, the last S, has
    // completed), column-major so that a warp's accesses are conflict-free;
    // every softmax thread reaches the barrier, also after a wait gave up
    float fa = 1.f, fb = 0.f;  // weights of this lane's O and of the other copy's
    const float* so = reinterpret_cast<const float*>(sq(0));
    if constexpr (NG == 1) {
      __shared__ float2 dup_ml[64];
      static_assert(64 * D * 4 <= C::QG_BYTES, "O of 64 rows fits in Q's space");
      float* sow = reinterpret_cast<float*>(sq(0));
      if (dup) {
        ok = __all_sync(0xffffffffu, ok);
        if (half == 1) {
          if (ok) {
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              float o[32];
              tc::ld32(t_o + c * 32, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) sow[(c * 32 + i) * 64 + srow] = o[i];
            }
          }
          dup_ml[srow] = ok ? make_float2(m_used, l) : make_float2(-CUDART_INF_F, -1.f);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (half == 0) {
          const float2 t = dup_ml[srow];
          if (t.y < 0.f) {
            ok = false;  // the other copy gave up: the row's result is lost
          } else if (ok && t.y > 0.f) {
            const float mm = fmaxf(m_used, t.x);
            fa = m_used == -CUDART_INF_F ? 0.f : tc::ex2(m_used - mm);
            fb = tc::ex2(t.x - mm);
            l = l * fa + t.y * fb;
            m_used = mm;
          }
        }
        ok = __all_sync(0xffffffffu, ok);
      }
    }
    if (!ok) {
      // The row's result is lost: leave zeros (whole key range) or an empty
      // part that the combine kernel gives no weight, never stale data.
      aborted = 1;
      if (out_row) {
        if (parts == 1) {
          uint4* o4 = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.out) + row_off * 2);
          for (int c = 0; c < D / 8; ++c) o4[c] = make_uint4(0u, 0u, 0u, 0u);
        } else {
          a.ws_ml[(row_off / D) * a.max_parts + part] = make_float2(-CUDART_INF_F, 0.f);
        }
      }
    } else {
      // ---- epilogue: out = O / l, rounded to the q dtype; or, for a part of
      // a split key range, (max, sum) and O / l in fp32 for the combine
      // kernel (a row that sees none of the part's tokens leaves -inf, 0, 0)
      tc::fence_after_sync();
      const float inv = (l > 0.f ? 1.f / l : 0.f) * (FP8 ? a.v_scale[kvh] : 1.f);
      if (parts == 1) {
        uint4* o4 = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.out) + row_off * 2);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tc::ld32(t_o + c * 32, o);
          if (dup && fb != 0.f) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = o[i] * fa + so[(c * 32 + i) * 64 + srow] * fb;
          }
          if (out_row) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              o4[c * 4 + q] = make_uint4(pack_pair(BF, o[8 * q] * inv, o[8 * q + 1] * inv),
                                         pack_pair(BF, o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                         pack_pair(BF, o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                         pack_pair(BF, o[8 * q + 6] * inv, o[8 * q + 7] * inv));
          }
        }
      } else {
        const int64_t prow = (row_off / D) * a.max_parts + part;
        if (out_row) a.ws_ml[prow] = make_float2(m_used, l);
        float4* w4 = reinterpret_cast<float4*>(a.ws_o + prow * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tc::ld32(t_o + c * 32, o);
          if (dup && fb != 0.f) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = o[i] * fa + so[(c * 32 + i) * 64 + srow] * fb;
          }
          if (out_row) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              w4[c * 8 + q] = make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv,
                                          o[4 * q + 3] * inv);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMma) {
    tc::fence_after_sync();
    tc::dealloc(tmem, C::TMEM_COLS);
  }
}

template <class QF, class CF, int D, int G, int NG>
cudaError_t launch_tc(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                      int32_t max_query_len, cudaStream_t stream) {
  using C = TcCfg<QF, CF, D, G, NG>;
  // shared memory keeps the tensor memory of the CTAs on one SM within 512
  // columns: one CTA of two groups, or at most two CTAs of one (>= 80 KB each)
  const size_t smem = std::max<size_t>(1024 + C::BYTES, NG == 2 ? 120 * 1024 : 80 * 1024);
  auto kern = paged_prefill_tc_kernel<QF, CF, D, G, NG>;
  cudaError_t e = configure_kernel(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  if (a.q_tiles != (max_query_len + C::QT - 1) / C::QT) return cudaErrorInvalidValue;
  if (a.max_parts > 1 && a.partition_tiles % (C::NT / kTileRows) != 0) return cudaErrorInvalidValue;
  PrefillArgs b = a;
  b.dup_rows = NG == 1 && static_cast<int64_t>(max_query_len) * G <= kTcRows / 2 ? 1 : 0;
  e = launch_pdl(kern, dim3(static_cast<unsigned>(a.q_tiles * a.max_parts), a.num_kv_heads,
                            a.num_seqs),
                 NG * kTcRows + 96, smem, stream, b, kmap, vmap);
  if (e != cudaSuccess || a.max_parts <= 1) return e;
  return launch_prefill_combine(a, std::is_same<QF, BF16>::value ? kBF16 : kF16, D, C::QT,
                                max_query_len, stream);
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, const CUtensorMap& kmap,
                              const CUtensorMap& vmap, int q_dtype, int cache_dtype,
                              int head_dim, int group, int32_t max_query_len,
                              cudaStream_t stream) {
  // two row groups (256 rows) when the chunks fill them
  const bool two = static_cast<int64_t>(max_query_len) * group >= 2 * kTcRows;
#define PAGED_TC(QF, CF, d, g)                                                          \
  if (head_dim == d && group == g)                                                      \
    return two ? launch_tc<QF, CF, d, g, 2>(a, kmap, vmap, max_query_len, stream)      \
               : launch_tc<QF, CF, d, g, 1>(a, kmap, vmap, max_query_len, stream);
#define PAGED_TC_ALL(QF)                                                              \
  PAGED_TC(QF, QF, 64, 1) PAGED_TC(QF, QF, 64, 2) PAGED_TC(QF, QF, 64, 4)             \
  PAGED_TC(QF, QF, 64, 8) PAGED_TC(QF, QF, 128, 1) PAGED_TC(QF, QF, 128, 2)           \
  PAGED_TC(QF, QF, 128, 4) PAGED_TC(QF, QF, 128, 8)
#define PAGED_TC_FP8(QF)                                                              \
  PAGED_TC(QF, E4M3, 128, 1) PAGED_TC(QF, E4M3, 128, 2) PAGED_TC(QF, E4M3, 128, 4)    \
  PAGED_TC(QF, E4M3, 128, 8)
  const bool fp8 = cache_dtype == kE4M3;
  if (q_dtype == kF16) {
    if (fp8) {
      PAGED_TC_FP8(F16)
    } else {
      PAGED_TC_ALL(F16)
    }
  } else if (q_dtype == kBF16) {
    if (fp8) {
      PAGED_TC_FP8(BF16)
    } else {
      PAGED_TC_ALL(BF16)
    }
  }
#undef PAGED_TC_FP8
#undef PAGED_TC_ALL
#undef PAGED_TC
  return cudaErrorNotSupported;
}

}  // namespace paged
