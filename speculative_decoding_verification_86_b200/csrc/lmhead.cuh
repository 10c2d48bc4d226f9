// The target's LM head with the verification's row statistics in its epilogue.
//
// The drafter shares the target's frozen output head ("Speculative decoding
// becomes standard: DSpark and multi-token drafters", section "What DSpark
// adds"), so every verified row -- target position j, or drafter position j --
// has logits l = h W^T with the same W [V, H].  Verification needs of most rows
// only their softmax statistics and one logit (the drafted token's), so the
// GEMM's epilogue reduces each accumulator tile straight into the statistics
// records the accept chain merges; of all the logits only the position-0 rows
// reach HBM (the rows most requests sample from).  The statistics run in
// prefix order: position 0's rows of every request first, then, once position
// 0 is decided, the other rows of the requests that accepted it.  The other
// rows a request samples from (a later rejected pair, or the bonus row) are
// produced as logits by the same kernel in its row-writing mode, after the
// chain decided.
//
// Kernel: one CTA per SM, persistent over work units (128 rows x a run of
// 128 x 256 tiles along the vocabulary), or -- the CTA-pair form -- clusters of
// two CTAs sharing 256 x 256 tiles (see LmGeo).  Warp roles:
//   warp 0     TMA producer: A (hidden rows, 128 x 64 bf16) and B (W rows,
//              256 x 64 bf16, or this CTA's 128 of them in a pair) tiles,
//              128-byte swizzle, 4-stage ring (6 stages in a pair);
//   warp 1     TMEM owner (512 columns: two 128 x 256 fp32 accumulators) and
//              MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//              M = 128 (256 for a pair, issued by rank 0), N = 256, K = 16 per
//              instruction, one thread;
//   warps 2-9  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 and one
//              half of the tile's columns (warps 2-5 the first 128, warps 6-9
//              the last 128), so two threads share each row of the tile; each
//              walks its 128 columns in batches of 16 (tcgen05.ld
//              32x32b.x16) while the MMA warp fills the other accumulator.  At
//              the end of a work unit the two halves' statistics are merged
//              through shared memory (the merge k_lm_combine applies across
//              parts) and one record per row is written.
// Every wait on an mbarrier is bounded in time; a wait that runs out raises
// the CTA's abort flag and the error word, drains what this CTA issued, frees
// TMEM and returns.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "stats.cuh"

namespace sv {

constexpr int kLmBM = 128;  // rows per tile (UMMA M)
constexpr int kLmBN = 256;  // vocabulary columns per tile (UMMA N)
constexpr int kLmBK = 64;   // hidden elements per stage: one 128-byte swizzle row of bf16
constexpr int kLmUK = 16;   // K of one kind::f16 instruction
constexpr uint32_t kLmABytes = kLmBM * kLmBK * 2;  // 16 KB: this CTA's 128 rows
constexpr int kLmEpiWarps = 8;                   // two per TMEM lane quarter
constexpr int kLmHalfN = kLmBN / 2;              // columns of a tile per epilogue warp
constexpr int kLmThreads = 32 * (2 + kLmEpiWarps);
constexpr uint32_t kLmTmemCols = 2 * kLmBN;
// A work unit covers `part_tiles` N tiles (a power of two up to kLmSegTiles);
// the statistics records of a unit ("parts") then tile the fp32 statistics
// segment exactly.
constexpr int kLmSegTiles = SegGeo<false>::kSeg / kLmBN;  // 64 tiles per statistics segment
static_assert(SegGeo<false>::kSeg % kLmBN == 0, "tiles divide the fp32 statistics segment");
constexpr size_t kLmBarrierBytes = 256;

// One row's statistics over the columns of one epilogue warp, handed to the
// warp holding the other half of the row (shared memory, one per TMEM lane).
struct LmXchg {
  double s;
  float K, mraw, er, om;
  float best;
  int best_idx;
  int bad, gbad;
};
constexpr size_t kLmXchgBytes = sizeof(LmXchg) * kLmBM;

// Geometry of the kernel with CG CTAs per MMA (1, or 2 for a CTA pair running
// tcgen05.mma.cta_group::2 on a 256 x 256 tile: each CTA holds its 128 rows of
// A and half of the 256 W rows, and gets its 128 rows of the accumulator).
template <int CG>
struct LmGeo {
  static constexpr int kRowsPerUnit = kLmBM * CG;              // M tile of one MMA
  static constexpr int kBRows = kLmBN / CG;                    // W rows per CTA and stage
  static constexpr uint32_t kBBytes = kBRows * kLmBK * 2;      // 32 KB or 16 KB
  static constexpr uint32_t kStageBytes = kLmABytes + kBBytes;  // 48 KB or 32 KB
  static constexpr int kStages = CG == 1 ? 4 : 6;
  static constexpr uint32_t kTxBytes = kStageBytes * CG;       // bytes the MMA CTA waits for
  static constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + kLmBarrierBytes + kLmXchgBytes;
};
constexpr int kLmMaxStages = 6;
constexpr unsigned long long kLmWaitNs = 2000000000ull;  // 2 s: legitimate waits are microseconds

constexpr int kLmModeStats = 0;  // epilogue -> statistics partial records + token logits
constexpr int kLmModeRows = 1;   // epilogue -> fp32 logits of listed rows

// Statistics of one row over one part (the columns of one work unit): the
// fields of a segment record before the parts are merged.
struct alignas(16) LmPart {
  float K;     // stochastic: integer exponent frame (-inf: nothing finite)
  float mraw;  // raw maximum
  float er;    // stochastic: sum e |a_then|
  float w;     // stochastic: om; greedy: lowest arg-max (int bits)
  double s;    // stochastic: sum of 2^(l c - K) terms
  int bad;     // NaN or +inf seen
  int pad;
};
static_assert(sizeof(LmPart) == 32, "part record layout");

struct LmParams {
  int mode;
  int H;
  int64_t V;
  int rows0, rows1;       // rows of A matrix 0 (target) and 1 (drafter); with rows_dev: rows0 = max rows
  const int* rows_dev;    // the row count of matrix 0 on the device (nullptr: rows0)
  // statistics mode: which rows the matrices hold.  pos0: matrix 0 holds the
  // target rows (i, 0) and matrix 1 the drafter rows (i, 0), i < B; row_map:
  // matrix 0 row r is batch row row_map[r] (target rows [B, k+1] then drafter
  // rows [B, k] numbered together); neither: the whole [B, k+1] and [B, k].
  int pos0;
  const int* row_map;
  // statistics mode
  int B, k;
  const int32_t* tokens;  // [B, k]
  const float* temp;      // [B] or nullptr (1.0)
  LmPart* parts;          // [rows0 + rows1, n_parts]
  int n_parts;
  int part_tiles;         // N tiles per work unit (both modes)
  float* tok_logits;      // [B, k, 2] (target, drafter)
  // rows mode (and, in statistics mode, the position-0 rows when `out` is set)
  const int64_t* dst;     // per row: element offset of its logits in `out` (-1: skip); nullptr: row * V
  float* out;             // statistics mode: the row buffer [B, k+1, V] then [B, k, V], or nullptr
  unsigned* error;        // bit 1: a wait timed out
};

// ------------------------------------------------------------ PTX helpers --
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long lm_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete.  Gives up (false) when another
// role raised *abort, or after kLmWaitNs, raising *abort and the error word.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned* error) {
  if (mbar_test(bar, parity)) return true;
  const unsigned long long t0 = lm_now();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (lm_now() - t0 > kLmWaitNs) {
        *abort = 1;
        atomicOr(error, 1u);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_prefetch(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 2-D tiled TMA load (no multicast): box at (x = hidden offset, y = row).
__device__ __forceinline__ void tma_load(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: 8-row groups 1024 bytes apart (stride byte offset), the
// leading byte offset unused for swizzled K-major layouts, descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128 per CTA of the group.
template <int CG>
__device__ __forceinline__ constexpr uint32_t lm_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(kLmBN >> 3) << 17) |
         (static_cast<uint32_t>((kLmBM * CG) >> 4) << 24);
}
template <int CG>
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate) {
  if constexpr (CG == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(lm_idesc<1>()), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(lm_idesc<2>()), "r"(accumulate)
        : "memory");
  }
}
// Arrive on `bar` (in every CTA of the group) once every tcgen05 operation
// this thread issued has completed.
template <int CG>
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  if constexpr (CG == 1) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
  } else {
    const uint16_t mask = 0x3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(smem_addr(bar)),
        "h"(mask)
        : "memory");
  }
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------- CTA pair helpers --
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}
// Every thread of both CTAs (the non-.aligned form: warps may arrive diverged).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// 2-D tiled TMA load of this CTA's half of a pair's operands, completing on
// the MMA CTA's barrier (a shared::cluster address); no multicast.
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster,
                                              int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

// ---------------------------------------------------------- work division --
template <int CG>
struct LmWork {
  int mt0, n_mt, n_nt, pt, n_parts, units, n_kb, first, stride;
  __device__ LmWork(int rows0, int rows1, int64_t V, int H, int part_tiles) {
    constexpr int R = LmGeo<CG>::kRowsPerUnit;
    mt0 = (rows0 + R - 1) / R;
    n_mt = mt0 + (rows1 + R - 1) / R;
    n_nt = static_cast<int>((V + kLmBN - 1) / kLmBN);
    pt = part_tiles;
    n_parts = (n_nt + pt - 1) / pt;
    units = n_mt * n_parts;
    n_kb = (H + kLmBK - 1) / kLmBK;
    first = static_cast<int>(blockIdx.x) / CG;  // the CTAs of a group take the same units
    stride = static_cast<int>(gridDim.x) / CG;
  }
  // unit u: M tile u % n_mt, part u / n_mt (the CTAs at work at one time share W columns)
  __device__ int mt(int u) const { return u % n_mt; }
  __device__ int part(int u) const { return u / n_mt; }
  __device__ int nt_lo(int u) const { return part(u) * pt; }
  __device__ int nt_hi(int u) const { return min(nt_lo(u) + pt, n_nt); }
};

struct LmShared {
  uint64_t full[kLmMaxStages];
  uint64_t empty[kLmMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t xfull[4];   // per lane quarter: the second half's statistics are in LmXchg
  uint64_t xempty[4];  // per lane quarter: the first half has read them
  uint64_t drain;
  uint32_t tmem;
  int abort;
  int rows0;
};
static_assert(sizeof(LmShared) <= kLmBarrierBytes, "barrier block");

// ---------------------------------------------------------------- epilogue --
// Per-thread row state of the statistics mode.
struct LmRowState {
  bool valid = false;
  bool greedy = false;
  bool draft = false;
  int i = 0, j = 0;
  int64_t g = 0;  // batch row: target rows [B, k+1], then drafter rows [B, k]
  int64_t tok = -1;
  float cc = 1.0f;
  SoftAcc acc;
  float best = -INFINITY;
  int best_idx = INT_MAX;
  int gbad = 0;
};

// The batch row held by TMEM lane `r_in_unit` of M tile mt (matrix 0 holds
// rows0 rows, matrix 1 p.rows1): its request i, position j, whether it is the
// drafter's, and its index g among the target rows [B, k+1] then the drafter
// rows [B, k]; false past the end of its matrix.
__device__ __forceinline__ bool lm_row_of(const LmParams& p, int rows0, int mt, int mt0,
                                          int rows_per_unit, int r_in_unit, LmRowState& st) {
  const bool m1 = mt >= mt0;
  const int r = (m1 ? mt - mt0 : mt) * rows_per_unit + r_in_unit;
  if (r >= (m1 ? p.rows1 : rows0)) return false;
  const int64_t nt = static_cast<int64_t>(p.B) * (p.k + 1);
  if (p.pos0) {
    st.draft = m1;
    st.i = r;
    st.j = 0;
    st.g = m1 ? nt + static_cast<int64_t>(r) * p.k : static_cast<int64_t>(r) * (p.k + 1);
    return true;
  }
  const int64_t g = p.row_map ? __ldg(p.row_map + r) : (m1 ? nt + r : r);
  st.g = g;
  st.draft = g >= nt;
  if (st.draft) {
    st.i = static_cast<int>((g - nt) / p.k);
    st.j = static_cast<int>(g - nt - static_cast<int64_t>(st.i) * p.k);
  } else {
    st.i = static_cast<int>(g / (p.k + 1));
    st.j = static_cast<int>(g - static_cast<int64_t>(st.i) * (p.k + 1));
  }
  return true;
}

__device__ __forceinline__ void lm_row_init(const LmParams& p, int rows0, int mt, int mt0,
                                            int rows_per_unit, int r_in_unit, LmRowState& st) {
  st = LmRowState();
  if (!lm_row_of(p, rows0, mt, mt0, rows_per_unit, r_in_unit, st)) return;
  st.valid = true;
  if (st.j < p.k) st.tok = __ldg(p.tokens + static_cast<int64_t>(st.i) * p.k + st.j);
  float T = p.temp ? __ldg(p.temp + st.i) : 1.0f;
  if (!temperature_valid(T)) T = 1.0f;  // the chain reports the request; any record will do
  st.greedy = T == 0.0f;
  if (!st.greedy) st.cc = static_cast<float>(1.4426950408889634 / static_cast<double>(T));
}

// 16 consecutive logits of the thread's row, starting at column `col`.
__device__ __forceinline__ void lm_consume_stats(const LmParams& p, LmRowState& st,
                                                 const uint32_t (&r)[16], int64_t col) {
  const int64_t nvalid = p.V - col;  // >= 1
  if (st.tok >= col && st.tok < col + 16) {
    float x = 0.0f;
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (col + q == st.tok) x = __uint_as_float(r[q]);
    p.tok_logits[(static_cast<int64_t>(st.i) * p.k + st.j) * 2 + (st.draft ? 1 : 0)] = x;
  }
  if (st.greedy) {
    float bm = -INFINITY;
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (q < nvalid) bm = fmax_nan(bm, __uint_as_float(r[q]));
    if (isnan(bm)) st.gbad = 1;
    if (bm > st.best || st.best_idx == INT_MAX) {
      int first = INT_MAX;
#pragma unroll
      for (int q = 15; q >= 0; --q)
        if (q < nvalid && __uint_as_float(r[q]) == bm) first = static_cast<int>(col) + q;
      if (first != INT_MAX) {
        st.best = bm;
        st.best_idx = first;
      }
    }
    return;
  }
  uint4 v[kBatchVecs];
  if (nvalid >= 16) {  // every batch but the vocabulary's ragged end
#pragma unroll
    for (int u = 0; u < kBatchVecs; ++u) v[u] = make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
  } else {
#pragma unroll
    for (int u = 0; u < kBatchVecs; ++u) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = (4 * u + e) < nvalid ? r[4 * u + e] : 0xff800000u;
      v[u] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  soft_batch<false>(st.acc, v, st.cc);
}

__device__ __forceinline__ void lm_write_part(const LmParams& p, const LmRowState& st, int part) {
  const int64_t g = st.g;
  LmPart o;
  if (st.greedy) {
    o.K = 0.0f;
    o.mraw = st.best;
    o.er = 0.0f;
    o.w = __int_as_float(st.best_idx == INT_MAX ? -1 : st.best_idx);
    o.s = 0.0;
    o.bad = st.gbad;
  } else {
    o.K = st.acc.K;
    o.mraw = st.acc.mraw;
    o.er = st.acc.er;
    o.w = st.acc.om;
    o.s = st.acc.s;
    o.bad = st.acc.bad;
  }
  o.pad = 0;
  p.parts[g * p.n_parts + part] = o;
}

__device__ __forceinline__ void lm_consume_rows(const LmParams& p, int64_t dst,
                                                const uint32_t (&r)[16], int64_t col) {
  float* o = p.out + dst + col;
  if (col + 16 <= p.V) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      reinterpret_cast<uint4*>(o)[u] = make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
  } else {
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (col + q < p.V) o[q] = __uint_as_float(r[q]);
  }
}

// ------------------------------------------------------------------ roles --
// With a CTA pair (CG = 2) both CTAs load their halves; the MMA CTA (rank 0)
// arms its full barrier for both halves' bytes, and the loads complete there.
template <int CG>
__device__ __forceinline__ void lm_producer(const LmParams& p, const LmWork<CG>& w, LmShared& sh,
                                            uint8_t* stages, const CUtensorMap* ma0,
                                            const CUtensorMap* ma1, const CUtensorMap* mw,
                                            uint32_t rank) {
  using G = LmGeo<CG>;
  uint32_t g = 0;
  bool ok = true;
  for (int u = w.first; ok && u < w.units; u += w.stride) {
    const int mt = w.mt(u);
    const CUtensorMap* ma = mt < w.mt0 ? ma0 : ma1;
    const int arow = (mt < w.mt0 ? mt : mt - w.mt0) * G::kRowsPerUnit + static_cast<int>(rank) * kLmBM;
    for (int nt = w.nt_lo(u); ok && nt < w.nt_hi(u); ++nt) {
      const int brow = nt * kLmBN + static_cast<int>(rank) * G::kBRows;
      for (int kb = 0; kb < w.n_kb; ++kb, ++g) {
        const int s = static_cast<int>(g % G::kStages);
        const uint32_t ph = (g / G::kStages) & 1u;
        if (!mbar_wait(&sh.empty[s], ph ^ 1u, &sh.abort, p.error)) {
          ok = false;
          break;
        }
        uint8_t* a = stages + static_cast<size_t>(s) * G::kStageBytes;
        if constexpr (CG == 1) {
          mbar_expect_tx(&sh.full[s], G::kTxBytes);
          tma_load(a, ma, &sh.full[s], kb * kLmBK, arow);
          tma_load(a + kLmABytes, mw, &sh.full[s], kb * kLmBK, brow);
        } else {
          if (rank == 0) mbar_expect_tx(&sh.full[s], G::kTxBytes);
          const uint32_t bar = peer_addr(&sh.full[s], 0);
          tma_load_pair(a, ma, bar, kb * kLmBK, arow);
          tma_load_pair(a + kLmABytes, mw, bar, kb * kLmBK, brow);
        }
      }
    }
  }
  if (!ok) {
    if constexpr (CG == 1) {
      // drain: the loads this thread issued land before the CTA's memory goes away
      for (uint32_t q = g > G::kStages ? g - G::kStages : 0; q < g; ++q) {
        volatile int no_abort = 0;
        mbar_wait(&sh.full[q % G::kStages], (q / G::kStages) & 1u, &no_abort, p.error);
      }
    } else {
      // this CTA's loads complete on the other CTA's barrier: give them time to land
      const unsigned long long t0 = lm_now();
      while (lm_now() - t0 < 200000ull) __nanosleep(1000);
    }
  }
}

template <int CG>
__device__ __forceinline__ void lm_mma(const LmParams& p, const LmWork<CG>& w, LmShared& sh,
                                       uint8_t* stages) {
  using G = LmGeo<CG>;
  uint32_t g = 0, t = 0;
  bool ok = true;
  for (int u = w.first; ok && u < w.units; u += w.stride) {
    for (int nt = w.nt_lo(u); ok && nt < w.nt_hi(u); ++nt, ++t) {
      const uint32_t a = t & 1u;
      if (!mbar_wait(&sh.tempty[a], ((t >> 1) & 1u) ^ 1u, &sh.abort, p.error)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = sh.tmem + a * kLmBN;
      for (int kb = 0; kb < w.n_kb; ++kb, ++g) {
        const int s = static_cast<int>(g % G::kStages);
        if (!mbar_wait(&sh.full[s], (g / G::kStages) & 1u, &sh.abort, p.error)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_addr(stages + static_cast<size_t>(s) * G::kStageBytes);
        const uint64_t adesc = sw128_desc(sa);
        const uint64_t bdesc = sw128_desc(sa + kLmABytes);
#pragma unroll
        for (int kk = 0; kk < kLmBK / kLmUK; ++kk) {
          // advance along K inside the swizzled 128-byte rows: 32 bytes per step
          umma_bf16<CG>(d, adesc + 2 * kk, bdesc + 2 * kk, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit<CG>(&sh.empty[s]);  // the stage is free once these MMAs have read it
      }
      if (ok) umma_commit<CG>(&sh.tfull[a]);
    }
  }
  if (!ok) {  // every MMA issued so far completes before TMEM is released
    umma_commit<CG>(&sh.drain);
    volatile int no_abort = 0;
    mbar_wait(&sh.drain, 0, &no_abort, p.error);
  }
}

// Fold the other column half's statistics of the same row into `st`: the
// greedy maximum with the lowest column among equal values, and the stochastic
// sums rebased to the larger frame and added -- the merge k_lm_combine applies
// across parts, so the record is what two separate part records would combine to.
__device__ __forceinline__ void lm_merge_half(LmRowState& st, const LmXchg& o) {
  if (st.greedy) {
    st.gbad |= o.gbad;
    if (o.best_idx != INT_MAX &&
        (st.best_idx == INT_MAX || o.best > st.best || (o.best == st.best && o.best_idx < st.best_idx))) {
      st.best = o.best;
      st.best_idx = o.best_idx;
    }
    return;
  }
  SoftAcc& a = st.acc;
  const float K = fmaxf(a.K, o.K);
  const int bad = a.bad | o.bad;
  double s = 0.0;
  float er = 0.0f, om = 0.0f;
  if (!bad && K > -INFINITY) {
    if (a.K > -INFINITY) {
      const double f = pow2_exact(a.K - K);
      const float ff = static_cast<float>(f);
      s += a.s * f;
      er += a.er * ff;
      om += (a.om + (K - a.K) * static_cast<float>(a.s)) * ff;
    }
    if (o.K > -INFINITY) {
      const double f = pow2_exact(o.K - K);
      const float ff = static_cast<float>(f);
      s += o.s * f;
      er += o.er * ff;
      om += (o.om + (K - o.K) * static_cast<float>(o.s)) * ff;
    }
  }
  a.K = K;
  a.mraw = fmax_nan(a.mraw, o.mraw);
  a.bad = bad;
  a.s = s;
  a.er = er;
  a.om = om;
}

template <int CG>
__device__ __forceinline__ void lm_epilogue(const LmParams& p, const LmWork<CG>& w, LmShared& sh,
                                            LmXchg* xchg, uint32_t rank) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3;       // TMEM lanes this warp may read
  const int half = (warp - 2) >> 2;   // columns [half * 128, half * 128 + 128) of every tile
  const int r_in_unit = static_cast<int>(rank) * kLmBM + quarter * 32 + lane;
  constexpr int R = LmGeo<CG>::kRowsPerUnit;
  LmXchg& xc = xchg[quarter * 32 + lane];
  uint32_t t = 0, n_unit = 0;
  for (int u = w.first; u < w.units; u += w.stride, ++n_unit) {
    const int mt = w.mt(u);
    LmRowState st;
    int64_t dst = -1;
    if (p.mode == kLmModeStats) {
      lm_row_init(p, sh.rows0, mt, w.mt0, R, r_in_unit, st);
      // Position 0 is the row a request samples from most often (a rejection
      // there, or the bonus row when nothing is verified): write its logits
      // now, so the row-writing pass only needs the rows of later positions.
      if (p.out && st.valid && st.j == 0) dst = st.g * p.V;
    } else {
      const int r = mt * R + r_in_unit;
      if (r < sh.rows0) dst = p.dst ? __ldg(p.dst + r) : static_cast<int64_t>(r) * p.V;
    }
    for (int nt = w.nt_lo(u); nt < w.nt_hi(u); ++nt, ++t) {
      const uint32_t a = t & 1u;
      // every lane waits (bounded), then the warp votes: it leaves together,
      // and stays converged for the .sync.aligned TMEM loads
      const bool ready = mbar_wait(&sh.tfull[a], (t >> 1) & 1u, &sh.abort, p.error);
      if (!__all_sync(0xffffffffu, ready)) return;
      tc_fence_after();
      const uint32_t taddr = sh.tmem + (static_cast<uint32_t>(quarter * 32) << 16) + a * kLmBN;
#pragma unroll 1
      for (int c = half * kLmHalfN; c < (half + 1) * kLmHalfN; c += 32) {
        uint32_t v0[16], v1[16];
        tmem_ld16(taddr + c, v0);
        tmem_ld16(taddr + c + 16, v1);
        tmem_ld_wait();
        const int64_t col = static_cast<int64_t>(nt) * kLmBN + c;
        if (col < p.V) {
          if (p.mode == kLmModeStats) {
            if (st.valid) lm_consume_stats(p, st, v0, col);
            if (dst >= 0) lm_consume_rows(p, dst, v0, col);
          } else if (dst >= 0) {
            lm_consume_rows(p, dst, v0, col);
          }
        }
        if (col + 16 < p.V) {
          if (p.mode == kLmModeStats) {
            if (st.valid) lm_consume_stats(p, st, v1, col + 16);
            if (dst >= 0) lm_consume_rows(p, dst, v1, col + 16);
          } else if (dst >= 0) {
            lm_consume_rows(p, dst, v1, col + 16);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (CG == 1) mbar_arrive(&sh.tempty[a]);
        else mbar_arrive_cluster(peer_addr(&sh.tempty[a], 0));  // the MMA CTA's barrier
      }
    }
    if (p.mode != kLmModeStats) continue;
    // The second half hands its statistics over (once the first half has read
    // the previous unit's); the first half merges them and writes the record.
    const uint32_t par = n_unit & 1u;
    if (half == 1) {
      const bool free = mbar_wait(&sh.xempty[quarter], par ^ 1u, &sh.abort, p.error);
      if (!__all_sync(0xffffffffu, free)) return;
      xc.s = st.acc.s;
      xc.K = st.acc.K;
      xc.mraw = st.acc.mraw;
      xc.er = st.acc.er;
      xc.om = st.acc.om;
      xc.bad = st.acc.bad;
      xc.best = st.best;
      xc.best_idx = st.best_idx;
      xc.gbad = st.gbad;
      mbar_arrive(&sh.xfull[quarter]);
    } else {
      const bool full = mbar_wait(&sh.xfull[quarter], par, &sh.abort, p.error);
      if (!__all_sync(0xffffffffu, full)) return;
      const LmXchg o = xc;
      mbar_arrive(&sh.xempty[quarter]);
      if (st.valid) {
        lm_merge_half(st, o);
        lm_write_part(p, st, w.part(u));
      }
    }
  }
}

// CG = 1: one CTA per SM.  CG = 2: launched in clusters of two CTAs (a pair on
// one TPC); rank 0 issues the MMAs of the pair's 256 x 256 tiles.
template <int CG>
__global__ void __launch_bounds__(kLmThreads, 1)
    k_lmhead(const __grid_constant__ CUtensorMap ma0, const __grid_constant__ CUtensorMap ma1,
             const __grid_constant__ CUtensorMap mw, LmParams p) {
  using G = LmGeo<CG>;
  extern __shared__ uint8_t lm_smem[];
  const uint32_t pad = (1024u - (smem_addr(lm_smem) & 1023u)) & 1023u;
  uint8_t* stages = lm_smem + pad;  // 1024-byte aligned: the swizzle atoms of every stage
  LmShared& sh = *reinterpret_cast<LmShared*>(stages + G::kStages * G::kStageBytes);
  LmXchg* xchg = reinterpret_cast<LmXchg*>(stages + G::kStages * G::kStageBytes + kLmBarrierBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 1 ? 0u : cluster_rank();
  if (threadIdx.x == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tempty[a], kLmEpiWarps * CG);  // one arrival per epilogue warp of the group
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&sh.xfull[q], 32);
      mbar_init(&sh.xempty[q], 32);
    }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    int rows0 = p.rows0;
    if (p.rows_dev) rows0 = max(0, min(__ldcg(p.rows_dev), p.rows0));
    sh.rows0 = rows0;
    mbar_init_fence();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&ma0);
    tma_prefetch(&ma1);
    tma_prefetch(&mw);
  }
  if (warp == 1) {
    if constexpr (CG == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_addr(&sh.tmem)),
                   "r"(kLmTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_addr(&sh.tmem)),
                   "r"(kLmTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  if constexpr (CG == 1) __syncthreads();
  else cluster_sync_all();  // barriers of both CTAs initialised before either signals the other
  tc_fence_after();
  const LmWork<CG> w(sh.rows0, p.mode == kLmModeStats ? p.rows1 : 0, p.V, p.H, p.part_tiles);
  if (warp == 0) {
    if (lane == 0) lm_producer<CG>(p, w, sh, stages, &ma0, &ma1, &mw, rank);
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) lm_mma<CG>(p, w, sh, stages);
  } else {
    lm_epilogue<CG>(p, w, sh, xchg, rank);
  }
  tc_fence_before();
  if constexpr (CG == 1) __syncthreads();
  else cluster_sync_all();  // no CTA leaves while the other may still signal it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (CG == 1) {
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(sh.tmem),
                   "r"(kLmTmemCols)
                   : "memory");
    } else {
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(sh.tmem),
                   "r"(kLmTmemCols)
                   : "memory");
    }
  }
}

// ------------------------------------------------------------ side kernels --
// Merge the parts of every (request, row slot, statistics segment) into the
// segment record the accept chain reads (the same merge as across a CTA's
// threads: rebase to the largest frame, then add).
// slot_sel: 0 every row, 1 the position-0 rows (slots 0 and k + 1) only, 2 the
// others only (a pass that computed some of the rows leaves the rest alone).
__global__ void k_lm_combine(RunParams p, const LmPart* parts, int n_parts, int parts_per_seg,
                             int rows0, int slot_sel) {
  const int rows = 2 * p.k + 1;
  const int64_t n = static_cast<int64_t>(p.B) * rows * p.n_segs;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int seg = static_cast<int>(e % p.n_segs);
    const int64_t rs = e / p.n_segs;
    const int i = static_cast<int>(rs / rows);
    const int slot = static_cast<int>(rs - static_cast<int64_t>(i) * rows);
    const bool pos0 = slot == 0 || slot == p.k + 1;
    if ((slot_sel == 1 && !pos0) || (slot_sel == 2 && pos0)) continue;
    const int64_t g = slot <= p.k ? static_cast<int64_t>(i) * (p.k + 1) + slot
                                  : rows0 + static_cast<int64_t>(i) * p.k + (slot - p.k - 1);
    float T = p.temp ? __ldg(p.temp + i) : 1.0f;
    if (!temperature_valid(T)) T = 1.0f;
    const int q0 = seg * parts_per_seg, q1 = min(q0 + parts_per_seg, n_parts);
    const LmPart* src = parts + g * n_parts;
    ChunkMeta r;
    if (T == 0.0f) {
      float best = -INFINITY;
      int arg = INT_MAX, bad = 0;
      for (int q = q0; q < q1; ++q) {
        const LmPart c = src[q];
        bad |= c.bad;
        const int a = __float_as_int(c.w);
        if (a >= 0 && (c.mraw > best || (c.mraw == best && a < arg))) {
          best = c.mraw;
          arg = a;
        }
      }
      r.K = 0.0f;
      r.mraw = bad ? __int_as_float(0x7fc00000) : best;
      r.err = 0.0f;
      r.arg = arg == INT_MAX ? -1 : arg;
      p.meta[e] = r;
      continue;
    }
    float K = -INFINITY, mraw = -INFINITY;
    int bad = 0;
    for (int q = q0; q < q1; ++q) {
      const LmPart c = src[q];
      bad |= c.bad;
      K = fmaxf(K, c.K);
      mraw = fmax_nan(mraw, c.mraw);
    }
    double s = 0.0;
    float er = 0.0f, om = 0.0f;
    if (!bad && K > -INFINITY) {
      for (int q = q0; q < q1; ++q) {
        const LmPart c = src[q];
        if (!(c.K > -INFINITY)) continue;
        const double f = pow2_exact(c.K - K);
        const float ff = static_cast<float>(f);
        s += c.s * f;
        er += c.er * ff;
        om += (c.w + (K - c.K) * static_cast<float>(c.s)) * ff;
      }
    }
    if (bad || isnan(mraw) || mraw == INFINITY) {
      r.K = __int_as_float(0x7fc00000);
      p.ssum[e] = __longlong_as_double(0x7ff8000000000000LL);
    } else {
      r.K = K;
      p.ssum[e] = K == -INFINITY ? 0.0 : s;
    }
    r.mraw = mraw;
    r.err = er;
    r.arg = __float_as_int(om);
    p.meta[e] = r;
  }
}

// The prefix-ordered LM head, first decision: position 0 of every request,
// from the statistics of its two position-0 rows (their fp32 logits are
// written, so a decision inside its bound is settled exactly here).  A request
// that accepts position 0 lists the rest of its rows -- target rows 1..L, and
// drafter rows 1..L-1 for a sampled request -- as batch rows (target rows
// [B, k+1], then drafter rows [B, k]) for the second statistics pass.
// state[i]: 0 finished, 1 continues, 2 a sample job was written.
__global__ void __launch_bounds__(kThreads) k_lm_decide0(RunParams p, int* state, int* count,
                                                         int* src) {
  __shared__ DecideShared dsh;
  const int i = blockIdx.x;
  if (threadIdx.x == 0) p.fallback[i] = 0;
  sync_compute();
  const ReqInfo ri = request_info(p, i);
  decide_position<false>(p, i, ri, 0, dsh);
  if (threadIdx.x == 0) {
    const int st = dsh.state;
    state[i] = st;
    if (st == 1) {
      const int L = ri.L;
      const int n = ri.greedy ? L : 2 * L - 1;
      const int at = atomicAdd(count, n);
      const int nt = p.B * (p.k + 1);
      int q = at;
      for (int j = 1; j <= L; ++j) src[q++] = i * (p.k + 1) + j;
      if (!ri.greedy)
        for (int j = 1; j < L; ++j) src[q++] = nt + i * p.k + j;
    }
  }
}

// Second decision: the chains of the requests that accepted position 0,
// walked from position 1 (a decision inside its bound marks the request for a
// whole redo: those rows' logits were never written).
__global__ void __launch_bounds__(kThreads) k_lm_decide_rest(RunParams p, const int* state) {
  __shared__ DecideShared dsh;
  const int i = blockIdx.x;
  if (__ldcg(state + i) != 1) return;
  decide_request<false>(p, i, request_info(p, i), dsh, 1);
}

// After the chain: the rows each request samples from (the rejected pair, or
// the bonus row), listed for the row-writing GEMM -- except position-0 rows,
// which the statistics pass has written already.  src: the hidden row (target
// rows first, then the drafter's, as the statistics pass numbers them); dst:
// the element offset of the row's logits in the row buffer, laid out as
// [B, k+1, V] target rows followed by [B, k, V] drafter rows.
__global__ void k_lm_rowlist(RunParams p, int* count, int* src, int64_t* dst) {
  const int rows0 = p.B * (p.k + 1);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.B; i += gridDim.x * blockDim.x) {
    if (__ldcg(p.fallback + i)) continue;
    const int kind = __ldcg(&p.jobs[i].kind);
    if (kind == kJobNone) continue;
    const int j = __ldcg(&p.jobs[i].row);
    if (j == 0) continue;  // written by the statistics pass
    const int n = kind == kJobResidual ? 2 : 1;
    const int at = atomicAdd(count, n);
    const int rt = i * (p.k + 1) + j;
    src[at] = rt;
    dst[at] = static_cast<int64_t>(rt) * p.V;
    if (n == 2) {
      const int rd = i * p.k + j;
      src[at + 1] = rows0 + rd;
      dst[at + 1] = (static_cast<int64_t>(rows0) + rd) * p.V;
    }
  }
}

// Copy the listed hidden rows (H bf16, 16-byte vectors) into one compact matrix.
__global__ void k_lm_gather(const int* count, const int* src, const uint4* hid_t, const uint4* hid_d,
                            int rows0, int H, int max_rows, uint4* out) {
  const int n = min(max(__ldcg(count), 0), max_rows);
  const int hv = H / 8;
  const int64_t total = static_cast<int64_t>(n) * hv;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(e / hv), c = static_cast<int>(e % hv);
    const int s = __ldcg(src + r);
    const uint4* from = s < rows0 ? hid_t + static_cast<int64_t>(s) * hv
                                  : hid_d + static_cast<int64_t>(s - rows0) * hv;
    out[e] = __ldg(from + c);
  }
}

}  // namespace sv
