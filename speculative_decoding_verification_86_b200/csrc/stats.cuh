// Pass 1: per-chunk row statistics, then (in the last CTA of each request)
// the accept chain.
//
// Stochastic rows (T > 0): the softmax normaliser of p = softmax(l / T) is
// accumulated as Z = sum_t 2^(l_t c - K) with c = fp32(log2 e / T) and K the
// exponent of the chunk's largest logit.  Each chunk reads its logits once
// (128-bit streaming loads), takes the NaN-propagating max, then sums
// ex2.approx terms pairwise in fp32 and across threads in fp64, and also sums
// e_t * |a_t| (a_t the rounded exponent), which bounds the argument-rounding
// error.  Greedy rows (T = 0) only keep the max and its lowest index.
//
// The request's last-arriving CTA merges the chunk records in chunk order and
// walks the chain ("Speculative decoding becomes standard: DSpark and
// multi-token drafters", section "Why draft-and-verify does not change the
// output"): accept drafted token x_j iff u * q(x_j) < p(x_j); the first
// rejection ends the chain.  p(x)/q(x) comes with a certified relative error
// bound; a draw inside that bound is settled by recomputing both row sums in
// fp64 at the true temperature, so every decision equals the fp64 rule.
#pragma once
#include "common.cuh"
#include "philox.cuh"
#include "stage.cuh"

namespace sv {

// ---------------------------------------------------------------------------
// Streaming statistics of one row segment.
//
// A segment is kThreads x kSegVecsPerThread 16-byte vectors (32768 bf16 or
// 16384 fp32 logits); thread t owns vectors t, t + 256, ... so every load
// instruction of a warp covers 512 contiguous bytes.  The vectors arrive in
// batches of kBatchVecs, the next batch's loads issued before the current one
// is reduced.  Each thread keeps its own exponent reference K_t: an integer,
// raised to ceil(max * c) whenever a batch brings a larger logit, so the
// rescaling of its running sums is an exact power of two and no block-wide
// maximum is needed before the exponentials.  One barrier per segment merges
// the threads.
// ---------------------------------------------------------------------------
constexpr int kSegVecsPerThread = 16;
constexpr int kBatchVecs = 4;
constexpr int kBatches = kSegVecsPerThread / kBatchVecs;
// Small dense batches use short segments of one batch step (8192 bf16 or 4096
// fp32 logits): four times the items, each a quarter as long.
constexpr int kShortSegBatches = 1;

template <bool BF16>
struct SegGeo {
  static constexpr int kPerVec = BF16 ? 8 : 4;
  static constexpr int kSegVecs = kThreads * kSegVecsPerThread;   // 4096 vectors
  static constexpr int kSeg = kSegVecs * kPerVec;                 // logits per segment
  static constexpr int kBatchElems = kBatchVecs * kPerVec;        // per thread per batch
  static constexpr int kSumLevels = BF16 ? 6 : 5;                 // pairwise depth of a batch sum (8 vectors)
};

template <bool BF16>
__device__ __forceinline__ void load_batch(const uint4* rv, int64_t nvec, int64_t seg0, int b,
                                           uint4 (&v)[kBatchVecs]) {
#pragma unroll
  for (int u = 0; u < kBatchVecs; ++u) {
    const int64_t idx = seg0 + static_cast<int64_t>(b * kBatchVecs + u) * kThreads + threadIdx.x;
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
}

// NaN-propagating maximum of one batch.
template <bool BF16>
__device__ __forceinline__ float batch_max(const uint4 (&v)[kBatchVecs]) {
  if constexpr (BF16) {
    uint32_t m2 = hmax2_nan(v[0].x, v[0].y);
    m2 = hmax2_nan(m2, v[0].z);
    m2 = hmax2_nan(m2, v[0].w);
#pragma unroll
    for (int u = 1; u < kBatchVecs; ++u) {
      m2 = hmax2_nan(m2, v[u].x);
      m2 = hmax2_nan(m2, v[u].y);
      m2 = hmax2_nan(m2, v[u].z);
      m2 = hmax2_nan(m2, v[u].w);
    }
    return fmax_nan(bf16_lo(m2), bf16_hi(m2));
  } else {
    float m = fmax_nan(__uint_as_float(v[0].x), __uint_as_float(v[0].y));
    m = fmax_nan(m, __uint_as_float(v[0].z));
    m = fmax_nan(m, __uint_as_float(v[0].w));
#pragma unroll
    for (int u = 1; u < kBatchVecs; ++u) {
      m = fmax_nan(m, __uint_as_float(v[u].x));
      m = fmax_nan(m, __uint_as_float(v[u].y));
      m = fmax_nan(m, __uint_as_float(v[u].z));
      m = fmax_nan(m, __uint_as_float(v[u].w));
    }
    return m;
  }
}

// Exact 2^d for an integer-valued d <= 0 (0 below the double range).
__device__ __forceinline__ double pow2_exact(float d) {
  return d < -1074.0f ? 0.0 : ldexp(1.0, static_cast<int>(d));
}

struct StatsShared {
  float K[kWarps];
  double s[kWarps];
  float er[kWarps];
  float om[kWarps];
  float mraw[kWarps];
  int bad[kWarps];
  int arg[kWarps];
  int flag;
};

// Running softmax statistics of one thread, in the thread's frame K (integer).
//   s  = sum of e_t = 2^(fl(l_t c - K)),
//   er = sum of e_t |a_t| with a_t the rounded exponent at the time the term
//        was computed (bounds the exponent rounding, relative per term),
//   om = sum of e_t (K - K_then): how far the term's own frame lay below K.
struct SoftAcc {
  float K = -INFINITY;
  double s = 0.0;
  float er = 0.0f;
  float om = 0.0f;
  float mraw = -INFINITY;
  int bad = 0;

  __device__ __forceinline__ void rebase(float Knew) {  // Knew > K
    if (K == -INFINITY) {
      s = 0.0;
      er = 0.0f;
      om = 0.0f;
    } else {
      const double f = pow2_exact(K - Knew);
      const float ff = static_cast<float>(f);
      om = (om + (Knew - K) * static_cast<float>(s)) * ff;
      s *= f;
      er *= ff;
    }
    K = Knew;
  }
};

// One batch of NV vectors of a thread's logits into its running statistics,
// given the batch's maximum bm (batch_max_n).  Logits are taken in pairs (the
// two halves of a bf16x2 word, or two fp32 words) so the exponent arguments,
// the bound terms and the sums use packed fp32x2 instructions; every lane is
// rounded as the scalar operation would be.  The argument is formed negated,
// n = K - l c = -(l c - K) (the same rounding, negated), clamped at 1024 so
// masked (-inf) logits give e = 0 and a finite bound term.  The batch sum is a
// balanced pairwise tree: across the batch's vectors, then across the pairs of
// a vector, then the two lanes (depth log2(NV) + log2(pairs) + 1, at most
// SegGeo::kSumLevels).
template <bool BF16, int NV>
__device__ __forceinline__ float batch_max_n(const uint4 (&v)[NV]) {
  static_assert(NV == 4 || NV == 8, "batch of 4 or 8 vectors");
  if constexpr (BF16) {
    uint32_t m[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u) m[u] = hmax2_nan(hmax2_nan(v[u].x, v[u].y), hmax2_nan(v[u].z, v[u].w));
#pragma unroll
    for (int w = 1; w < NV; w *= 2)
#pragma unroll
      for (int u = 0; u + w < NV; u += 2 * w) m[u] = hmax2_nan(m[u], m[u + w]);
    return fmax_nan(bf16_lo(m[0]), bf16_hi(m[0]));
  } else {
    float m[NV];
#pragma unroll
    for (int u = 0; u < NV; ++u)
      m[u] = fmax_nan(fmax_nan(__uint_as_float(v[u].x), __uint_as_float(v[u].y)),
                      fmax_nan(__uint_as_float(v[u].z), __uint_as_float(v[u].w)));
#pragma unroll
    for (int w = 1; w < NV; w *= 2)
#pragma unroll
      for (int u = 0; u + w < NV; u += 2 * w) m[u] = fmax_nan(m[u], m[u + w]);
    return m[0];
  }
}

template <bool BF16, int NV>
__device__ __forceinline__ void soft_terms(SoftAcc& acc, const uint4 (&v)[NV], float cc, float bm) {
  acc.mraw = fmax_nan(acc.mraw, bm);
  if (isnan(bm) || bm == INFINITY) acc.bad = 1;
  const float Kb = ceilf(bm * cc);
  if (Kb > acc.K) acc.rebase(Kb);
  if (!(acc.K > -INFINITY) || acc.K == INFINITY) return;  // nothing finite yet, or +inf seen
  const float2 ncc = make_float2(-cc, -cc);
  const float2 K2 = make_float2(acc.K, acc.K);
  float2 er2 = make_float2(acc.er, 0.0f);
  constexpr int kPairs = BF16 ? 4 : 2;  // logit pairs per 16-byte vector
  float2 ps[NV][kPairs];
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const uint32_t wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
    for (int q = 0; q < kPairs; ++q) {
      float2 x;
      if constexpr (BF16) {
        x = make_float2(bf16_lo(wd[q]), bf16_hi(wd[q]));
      } else {
        x = make_float2(__uint_as_float(wd[2 * q]), __uint_as_float(wd[2 * q + 1]));
      }
      float2 n = ffma2(x, ncc, K2);  // K - l c >= 0
      n.x = fminf(n.x, 1024.0f);
      n.y = fminf(n.y, 1024.0f);
      const float2 e = make_float2(ex2_approx(-n.x), ex2_approx(-n.y));
      er2 = ffma2(e, n, er2);
      ps[u][q] = e;
    }
  }
  // across vectors
#pragma unroll
  for (int w = 1; w < NV; w *= 2)
#pragma unroll
    for (int u = 0; u + w < NV; u += 2 * w)
#pragma unroll
      for (int q = 0; q < kPairs; ++q) ps[u][q] = fadd2(ps[u][q], ps[u + w][q]);
  float2 t;
  if constexpr (BF16) {
    t = fadd2(fadd2(ps[0][0], ps[0][1]), fadd2(ps[0][2], ps[0][3]));
  } else {
    t = fadd2(ps[0][0], ps[0][1]);
  }
  acc.er = er2.x + er2.y;
  acc.s += static_cast<double>(t.x + t.y);
}

template <bool BF16>
__device__ __forceinline__ void soft_batch(SoftAcc& acc, const uint4 (&v)[kBatchVecs], float cc) {
  soft_terms<BF16, kBatchVecs>(acc, v, cc, batch_max_n<BF16, kBatchVecs>(v));
}

// Merge `acc` of all threads of the CTA into one record (called by every thread).
__device__ __forceinline__ void soft_merge_block(SoftAcc acc, StatsShared& sh, ChunkMeta* meta_out,
                                                 double* sum_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int level = 0; level < 2; ++level) {
    int bad = __any_sync(0xffffffffu, acc.bad);
    float Kw = acc.K;
#pragma unroll
    for (int off = 16; off; off >>= 1) Kw = fmaxf(Kw, __shfl_xor_sync(0xffffffffu, Kw, off));
    double s = 0.0;
    float er = 0.0f, om = 0.0f;
    if (!bad && acc.K > -INFINITY) {
      const double f = pow2_exact(acc.K - Kw);
      const float ff = static_cast<float>(f);
      s = acc.s * f;
      er = acc.er * ff;
      om = (acc.om + (Kw - acc.K) * static_cast<float>(acc.s)) * ff;
    }
    s = warp_sum_d(s);
    er = warp_sum_f(er);
    om = warp_sum_f(om);
    const float mraw = warp_max_nan(acc.mraw);
    if (level == 0) {
      if (lane == 0) {
        sh.K[warp] = Kw;
        sh.s[warp] = s;
        sh.er[warp] = er;
        sh.om[warp] = om;
        sh.mraw[warp] = mraw;
        sh.bad[warp] = bad;
      }
      sync_compute();
      if (warp != 0) return;
      const bool have = lane < kWarps;
      acc.K = have ? sh.K[lane] : -INFINITY;
      acc.s = have ? sh.s[lane] : 0.0;
      acc.er = have ? sh.er[lane] : 0.0f;
      acc.om = have ? sh.om[lane] : 0.0f;
      acc.mraw = have ? sh.mraw[lane] : -INFINITY;
      acc.bad = have ? sh.bad[lane] : 0;
    } else if (lane == 0) {
      ChunkMeta r;
      if (bad || isnan(mraw) || mraw == INFINITY) {
        r.K = __int_as_float(0x7fc00000);  // NaN marks a row the chain must not use
        *sum_out = __longlong_as_double(0x7ff8000000000000LL);
      } else {
        r.K = Kw;  // -inf if the segment held only masked logits
        *sum_out = Kw == -INFINITY ? 0.0 : s;
      }
      r.mraw = mraw;
      r.err = er;
      r.arg = __float_as_int(om);
      *meta_out = r;
    }
  }
}

template <bool BF16>
__device__ __forceinline__ void stochastic_segment(const void* row, int64_t V, int seg, float cc,
                                                   ChunkMeta* meta_out, double* sum_out,
                                                   StatsShared& sh) {
  using G = SegGeo<BF16>;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t nvec = V / G::kPerVec;
  const int64_t seg0 = static_cast<int64_t>(seg) * G::kSegVecs;
  SoftAcc acc;
  // batches of two load steps (8 vectors), as in the staged pass, so both
  // passes round the same sums in the same order
  static_assert(kBatches == 4, "two batches of two steps");
  uint4 v[2 * kBatchVecs], w[2 * kBatchVecs];
  uint4 (&v0)[kBatchVecs] = *reinterpret_cast<uint4 (*)[kBatchVecs]>(&v[0]);
  uint4 (&v1)[kBatchVecs] = *reinterpret_cast<uint4 (*)[kBatchVecs]>(&v[kBatchVecs]);
  uint4 (&w0)[kBatchVecs] = *reinterpret_cast<uint4 (*)[kBatchVecs]>(&w[0]);
  uint4 (&w1)[kBatchVecs] = *reinterpret_cast<uint4 (*)[kBatchVecs]>(&w[kBatchVecs]);
  load_batch<BF16>(rv, nvec, seg0, 0, v0);
  load_batch<BF16>(rv, nvec, seg0, 1, v1);
  load_batch<BF16>(rv, nvec, seg0, 2, w0);
  load_batch<BF16>(rv, nvec, seg0, 3, w1);
  soft_terms<BF16, 2 * kBatchVecs>(acc, v, cc, batch_max_n<BF16, 2 * kBatchVecs>(v));
  soft_terms<BF16, 2 * kBatchVecs>(acc, w, cc, batch_max_n<BF16, 2 * kBatchVecs>(w));
  soft_merge_block(acc, sh, meta_out, sum_out);
}

// The segment passes fed by per-thread asynchronous staging (stage.cuh):
// batch b of the segment is staging step b, three steps in flight.  Thread t
// gets the same vectors as from load_batch.
static_assert(kBatchVecs == kStepVecs, "a staging step is one batch");

// FULL: the whole segment lies inside the row (every segment but a row's
// last), so no vector needs a range check.
template <bool FULL = false>
__device__ __forceinline__ void stage_segment_batch(Stager& sg, const uint4* rv, int64_t nvec,
                                                    int64_t seg0, int b) {
#pragma unroll
  for (int u = 0; u < kBatchVecs; ++u) {
    const int64_t idx = seg0 + static_cast<int64_t>(b * kBatchVecs + u) * kThreads + threadIdx.x;
    if constexpr (FULL) {
      cp_async16(sg.slot(b, u), rv + idx, true);
    } else {
      const bool valid = idx < nvec;
      cp_async16(sg.slot(b, u), valid ? rv + idx : rv, valid);
    }
  }
  cp_async_commit();
  ++sg.issued;
}

template <bool BF16, bool FULL = false>
__device__ __forceinline__ void staged_batch(Stager& sg, int64_t nvec, int64_t seg0, int b,
                                             uint4 (&v)[kBatchVecs]) {
  cp_async_wait(sg.issued - b - 1);
#pragma unroll
  for (int u = 0; u < kBatchVecs; ++u) {
    if constexpr (FULL) {
      v[u] = *sg.slot(b, u);
    } else {
      const int64_t idx = seg0 + static_cast<int64_t>(b * kBatchVecs + u) * kThreads + threadIdx.x;
      v[u] = idx < nvec ? *sg.slot(b, u) : neg_inf_vec<BF16>();
    }
  }
}

// NB: batches per segment -- kBatches for the standard 64 KB segment, fewer
// for the short segments small batches use (more CTAs per row, shorter items).
template <bool BF16, bool FULL, int NB = kBatches>
__device__ __forceinline__ void stochastic_segment_pass(const uint4* rv, int64_t nvec, int64_t seg0,
                                                        float cc, SoftAcc& acc, uint4* stage_buf) {
  Stager sg{stage_buf};
#pragma unroll
  for (int b = 0; b < kStageSlots && b < NB; ++b) stage_segment_batch<FULL>(sg, rv, nvec, seg0, b);
  if constexpr (NB % 2 == 0) {
    // two staging steps per batch (64 bf16 / 32 fp32 logits a thread): half
    // the per-batch work (maximum, frame check, fp64 accumulation)
#pragma unroll (FULL ? NB / 2 : 1)
    for (int b = 0; b < NB; b += 2) {
      uint4 v[2 * kBatchVecs];
      uint4 (&v0)[kBatchVecs] = *reinterpret_cast<uint4 (*)[kBatchVecs]>(&v[0]);
      uint4 (&v1)[kBatchVecs] = *reinterpret_cast<uint4 (*)[kBatchVecs]>(&v[kBatchVecs]);
      staged_batch<BF16, FULL>(sg, nvec, seg0, b, v0);
      staged_batch<BF16, FULL>(sg, nvec, seg0, b + 1, v1);
      const float bm = batch_max_n<BF16, 2 * kBatchVecs>(v);  // every staged value is in registers
      // refill both steps' slots
      if (b + kStageSlots < NB) stage_segment_batch<FULL>(sg, rv, nvec, seg0, b + kStageSlots);
      if (b + 1 + kStageSlots < NB) stage_segment_batch<FULL>(sg, rv, nvec, seg0, b + 1 + kStageSlots);
      soft_terms<BF16, 2 * kBatchVecs>(acc, v, cc, bm);
    }
  } else {
    // full segments: unrolled, so slots and wait counts are compile-time constants
#pragma unroll (FULL ? NB : 1)
    for (int b = 0; b < NB; ++b) {
      uint4 v[kBatchVecs];
      staged_batch<BF16, FULL>(sg, nvec, seg0, b, v);
      soft_batch<BF16>(acc, v, cc);
      // refill this step's slot once its values have been used
      if (b + kStageSlots < NB) stage_segment_batch<FULL>(sg, rv, nvec, seg0, b + kStageSlots);
    }
  }
}

template <bool BF16, int NB = kBatches>
__device__ __forceinline__ void stochastic_segment_staged(const void* row, int64_t V, int seg, float cc,
                                                          ChunkMeta* meta_out, double* sum_out,
                                                          StatsShared& sh, uint4* stage_buf) {
  using G = SegGeo<BF16>;
  constexpr int64_t kVecs = static_cast<int64_t>(kThreads) * kBatchVecs * NB;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t nvec = V / G::kPerVec;
  const int64_t seg0 = static_cast<int64_t>(seg) * kVecs;
  SoftAcc acc;
  if (seg0 + kVecs <= nvec) stochastic_segment_pass<BF16, true, NB>(rv, nvec, seg0, cc, acc, stage_buf);
  else stochastic_segment_pass<BF16, false, NB>(rv, nvec, seg0, cc, acc, stage_buf);
  soft_merge_block(acc, sh, meta_out, sum_out);
}

// Max and lowest arg-max of one segment of a greedy row: each thread keeps its
// running maximum and the lowest index attaining it (batches arrive in index
// order per thread), then the CTA reduces (larger value wins, ties go to the
// lower index).
template <bool BF16>
struct GreedyScan {
  float best = -INFINITY;
  int64_t best_idx = INT64_MAX;
  int bad = 0;

  __device__ __forceinline__ void scan(const uint4 (&v)[kBatchVecs], int64_t seg0, int b) {
    using G = SegGeo<BF16>;
    const float bm = batch_max<BF16>(v);
    if (isnan(bm)) bad = 1;
    if (!(bm > best) && best_idx != INT64_MAX) return;  // earlier batches hold lower indices
    if (!(bm >= best)) return;
    // first element of this batch equal to its max, in index order
    int64_t first = INT64_MAX;
#pragma unroll
    for (int u = kBatchVecs - 1; u >= 0; --u) {
      float x[G::kPerVec];
      unpack<BF16>(v[u], x);
#pragma unroll
      for (int q = G::kPerVec - 1; q >= 0; --q) {
        if (x[q] == bm)
          first = (seg0 + static_cast<int64_t>(b * kBatchVecs + u) * kThreads + threadIdx.x) *
                      G::kPerVec + q;
      }
    }
    best = bm;
    best_idx = first;
  }

  __device__ __forceinline__ void finish(ChunkMeta* meta_out, StatsShared& sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int idx = best_idx == INT64_MAX ? INT_MAX : static_cast<int>(best_idx);
    for (int level = 0; level < 2; ++level) {
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
        if (ob > best || (ob == best && oi < idx)) {
          best = ob;
          idx = oi;
        }
      }
      bad = __any_sync(0xffffffffu, bad);
      if (level == 0) {
        if (lane == 0) {
          sh.mraw[warp] = best;
          sh.arg[warp] = idx;
          sh.bad[warp] = bad;
        }
        sync_compute();
        if (warp != 0) return;
        best = lane < kWarps ? sh.mraw[lane] : -INFINITY;
        idx = lane < kWarps ? sh.arg[lane] : INT_MAX;
        bad = lane < kWarps ? sh.bad[lane] : 0;
      } else if (lane == 0) {
        ChunkMeta r;
        r.K = 0.0f;
        r.mraw = bad ? __int_as_float(0x7fc00000) : best;
        r.err = 0.0f;
        r.arg = idx == INT_MAX ? -1 : idx;
        *meta_out = r;
      }
    }
  }
};

template <bool BF16>
__device__ __forceinline__ void greedy_segment(const void* row, int64_t V, int seg,
                                               ChunkMeta* meta_out, StatsShared& sh) {
  using G = SegGeo<BF16>;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t nvec = V / G::kPerVec;
  const int64_t seg0 = static_cast<int64_t>(seg) * G::kSegVecs;
  GreedyScan<BF16> g;
  uint4 va[kBatchVecs], vb[kBatchVecs];
  load_batch<BF16>(rv, nvec, seg0, 0, va);
#pragma unroll
  for (int b = 0; b < kBatches; b += 2) {
    if (b + 1 < kBatches) load_batch<BF16>(rv, nvec, seg0, b + 1, vb);
    g.scan(va, seg0, b);
    if (b + 2 < kBatches) load_batch<BF16>(rv, nvec, seg0, b + 2, va);
    if (b + 1 < kBatches) g.scan(vb, seg0, b + 1);
  }
  g.finish(meta_out, sh);
}

template <bool BF16, bool FULL, int NB = kBatches>
__device__ __forceinline__ void greedy_segment_pass(const uint4* rv, int64_t nvec, int64_t seg0,
                                                    GreedyScan<BF16>& g, uint4* stage_buf) {
  Stager sg{stage_buf};
#pragma unroll
  for (int b = 0; b < kStageSlots && b < NB; ++b) stage_segment_batch<FULL>(sg, rv, nvec, seg0, b);
#pragma unroll 1
  for (int b = 0; b < NB; ++b) {
    uint4 v[kBatchVecs];
    staged_batch<BF16, FULL>(sg, nvec, seg0, b, v);
    g.scan(v, seg0, b);
    if (b + kStageSlots < NB) stage_segment_batch<FULL>(sg, rv, nvec, seg0, b + kStageSlots);
  }
}

template <bool BF16, int NB = kBatches>
__device__ __forceinline__ void greedy_segment_staged(const void* row, int64_t V, int seg,
                                                      ChunkMeta* meta_out, StatsShared& sh,
                                                      uint4* stage_buf) {
  using G = SegGeo<BF16>;
  constexpr int64_t kVecs = static_cast<int64_t>(kThreads) * kBatchVecs * NB;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t nvec = V / G::kPerVec;
  const int64_t seg0 = static_cast<int64_t>(seg) * kVecs;
  GreedyScan<BF16> g;
  if (seg0 + kVecs <= nvec) greedy_segment_pass<BF16, true, NB>(rv, nvec, seg0, g, stage_buf);
  else greedy_segment_pass<BF16, false, NB>(rv, nvec, seg0, g, stage_buf);
  g.finish(meta_out, sh);
}

// ---------------------------------------------------------------------------
// A whole row in one pass: its segments' staging steps form one pipeline, so
// the first steps of segment s+1 are in flight while segment s is finished and
// its record written -- the copies never drain between segments.  The records
// are those of the per-segment passes (the same vectors per thread, merged the
// same way).  GREEDY selects the arg-max scan instead of the softmax sums.
// ---------------------------------------------------------------------------
template <bool FULL>
__device__ __forceinline__ void stage_row_step(Stager& sg, const uint4* rv, int64_t nvec, int g) {
  const int seg = g / kBatches, b = g % kBatches;
  const int64_t base = static_cast<int64_t>(seg) * SegGeo<true>::kSegVecs + threadIdx.x;
#pragma unroll
  for (int u = 0; u < kBatchVecs; ++u) {
    const int64_t idx = base + static_cast<int64_t>(b * kBatchVecs + u) * kThreads;
    const bool valid = FULL || idx < nvec;
    cp_async16(sg.slot(g, u), valid ? rv + idx : rv, valid);
  }
  cp_async_commit();
  ++sg.issued;
}
static_assert(SegGeo<true>::kSegVecs == SegGeo<false>::kSegVecs, "segments hold the same vector count");

template <bool BF16, bool GREEDY>
__device__ void stats_row_staged(const void* row, int64_t V, int n_segs, float cc, ChunkMeta* meta,
                                 double* ssum, StatsShared& sh, uint4* stage_buf) {
  using G = SegGeo<BF16>;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t nvec = V / G::kPerVec;
  const int n_steps = n_segs * kBatches;
  // steps of segments wholly inside the row need no range checks
  const int full_steps = static_cast<int>(nvec / G::kSegVecs) * kBatches;
  Stager sg{stage_buf};
  for (int g = 0; g < kStageSlots && g < n_steps; ++g) {
    if (g < full_steps) stage_row_step<true>(sg, rv, nvec, g);
    else stage_row_step<false>(sg, rv, nvec, g);
  }
#pragma unroll 1
  for (int seg = 0; seg < n_segs; ++seg) {
    const int64_t seg0 = static_cast<int64_t>(seg) * G::kSegVecs;
    const bool full = (seg + 1) * kBatches <= full_steps;
    SoftAcc acc;
    GreedyScan<BF16> gs;
    // greedy: one step per batch; stochastic: two (as in the segment pass)
    constexpr int kSteps = GREEDY ? 1 : 2;
    static_assert(kBatches % kSteps == 0, "steps per batch divide a segment");
#pragma unroll 1
    for (int b = 0; b < kBatches; b += kSteps) {
      uint4 v[kSteps * kBatchVecs];
#pragma unroll
      for (int h = 0; h < kSteps; ++h) {
        const int g = seg * kBatches + b + h;
        cp_async_wait(sg.issued - g - 1);
#pragma unroll
        for (int u = 0; u < kBatchVecs; ++u) {
          const int64_t idx = seg0 + static_cast<int64_t>((b + h) * kBatchVecs + u) * kThreads + threadIdx.x;
          v[h * kBatchVecs + u] = (full || idx < nvec) ? *sg.slot(g, u) : neg_inf_vec<BF16>();
        }
      }
      float bm = 0.0f;
      if constexpr (GREEDY) gs.scan(v, seg0, b);
      else bm = batch_max_n<BF16, kSteps * kBatchVecs>(v);  // every staged value is in registers
      // refill the steps' slots once their values are in registers
#pragma unroll
      for (int h = 0; h < kSteps; ++h) {
        const int gn = seg * kBatches + b + h + kStageSlots;
        if (gn < n_steps) {
          if (gn < full_steps) stage_row_step<true>(sg, rv, nvec, gn);
          else stage_row_step<false>(sg, rv, nvec, gn);
        }
      }
      if constexpr (!GREEDY) soft_terms<BF16, kSteps * kBatchVecs>(acc, v, cc, bm);
    }
    if constexpr (GREEDY) gs.finish(meta + seg, sh);
    else soft_merge_block(acc, sh, meta + seg, ssum + seg);
    sync_compute();  // sh is reused by the next segment's merge
  }
}

// ---------------------------------------------------------------------------
// Merged row records, built by the deciding CTA in shared memory.
// ---------------------------------------------------------------------------
struct RowMerged {
  double Z;      // sum of 2^(fl(l c - K_then)) 2^(K_then - K) over the row (fp32 terms)
  double ER;     // sum of e |a_then| in the row's frame: exponent-rounding weight
  double EA;     // sum of e |a| with a measured from K: Z times minus the mean exponent
  float K;       // exponent reference of the row (integer)
  float mraw;    // raw max
  int arg;       // greedy: lowest arg-max
  int bad;       // NaN / +inf / all -inf
  double invZ;   // 1 / Z, and ER / Z, EA / Z (stochastic rows that are not bad)
  double erz, eaz;
};

// Constants of a request's temperature for the fp32 path and its bounds.
struct TempConsts {
  double T;         // temperature
  double c_exact;   // log2(e) / T in fp64
  double eta;       // |relative error| of cc
  double kappa;     // ln2 (2^-24 + eta): bound per unit |exponent argument|
  double eps_base;  // ex2 error + pairwise-sum rounding + slack
  float cc;         // fp32 log2(e) / T used by the fp32 path
};

struct DecideShared {
  RowMerged rows[kMaxRows];
  double red[kWarps];
  // chain state (written by thread 0)
  int state;        // 0 continue, 1 stop
  int need_exact;   // position whose accept test needs the fp64 row sums, or -1
  double exact_Za, exact_Zb;
  // dense order: every position's accept test, evaluated at once
  int dec[kMaxK];   // 1 accept, 0 reject, -1 inside the bound, 2 bad token, 3 non-finite rows
  double pa[kMaxK], qb[kMaxK];
  double u2[kMaxK + 1];  // the sample's draw of each position where the chain may end
  // prefix order: position j's inputs, loaded while the rows are merged
  int xj;
  float la, lb;
  double u;
  TempConsts tc;
};

// A lane's first segment record of a row (segment = lane), loaded ahead of
// the merge so a warp merging several rows waits for one round trip.
struct SegRec {
  float4 m;
  double s;
};
__device__ __forceinline__ SegRec load_seg_rec(const RunParams& p, int i, int slot) {
  const int lane = threadIdx.x & 31;
  const int64_t base = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_segs;
  SegRec r{make_float4(-INFINITY, -INFINITY, 0.0f, 0.0f), 0.0};
  if (lane < p.n_segs) {
    r.m = __ldcg(reinterpret_cast<const float4*>(p.meta + base + lane));
    r.s = __ldcg(p.ssum + base + lane);
  }
  return r;
}

// Merge the segment records of stochastic row `slot` with one warp.  Lane l
// holds the record of segment l (`first`, loaded by load_seg_rec) and loads
// those of segments l + 32, ... itself.
__device__ __forceinline__ void merge_stochastic_row(const RunParams& p, int i, int slot,
                                                     RowMerged& out, const SegRec& first) {
  const int lane = threadIdx.x & 31;
  const int64_t base = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_segs;
  const float4 m0 = first.m;
  const double s0 = first.s;
  float K = m0.x, mraw = m0.y;
  int bad = (isnan(m0.x) || m0.x == INFINITY) ? 1 : 0;
  for (int c = lane + 32; c < p.n_segs; c += 32) {
    const float4 m4 = __ldcg(reinterpret_cast<const float4*>(p.meta + base + c));
    if (isnan(m4.x) || m4.x == INFINITY) bad = 1;
    K = fmaxf(K, m4.x);
    mraw = fmax_nan(mraw, m4.y);
  }
  K = warp_max_nan(K);
  mraw = warp_max_nan(mraw);
  bad = __any_sync(0xffffffffu, bad);
  if (!(K > -INFINITY)) bad = 1;
  double Z = 0.0, ER = 0.0, EA = 0.0;
  if (!bad) {
    for (int c = lane; c < p.n_segs; c += 32) {
      const float4 m4 = c == lane ? m0 : __ldcg(reinterpret_cast<const float4*>(p.meta + base + c));
      if (m4.x == -INFINITY) continue;
      const double sc = c == lane ? s0 : __ldcg(p.ssum + base + c);
      const double d = static_cast<double>(K) - static_cast<double>(m4.x);  // integer >= 0
      const double f = pow2_exact(static_cast<float>(-d));
      Z += sc * f;
      ER += static_cast<double>(m4.z) * f;
      // |a| from K = |a_then| + (K_then's distance below K): the rounding weight,
      // plus the offsets recorded inside the segment, plus the segment's own offset.
      EA += (static_cast<double>(m4.z) + static_cast<double>(m4.w) +
             d * sc) * f;
    }
  }
  Z = warp_sum_d(Z);
  ER = warp_sum_d(ER);
  EA = warp_sum_d(EA);
  if (!(Z > 0.0) || isinf(Z) || isnan(Z)) bad = 1;
  if (lane == 0) {
    out.Z = Z;
    out.ER = ER;
    out.EA = EA;
    out.K = K;
    out.mraw = mraw;
    out.arg = -1;
    out.bad = bad;
    // the decision's divisions, done here while the other row merges
    const double inv = bad ? 0.0 : 1.0 / Z;
    out.invZ = inv;
    out.erz = ER * inv;
    out.eaz = EA * inv;
  }
}

__device__ __forceinline__ void merge_stochastic_row(const RunParams& p, int i, int slot,
                                                     RowMerged& out) {
  merge_stochastic_row(p, i, slot, out, load_seg_rec(p, i, slot));
}

__device__ __forceinline__ void merge_greedy_row(const RunParams& p, int i, int slot,
                                                 RowMerged& out) {
  const int lane = threadIdx.x & 31;
  const int64_t base = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_segs;
  float best = -INFINITY;
  int arg = INT_MAX;
  int bad = 0;
  for (int c = lane; c < p.n_segs; c += 32) {
    const float4 m4 = __ldcg(reinterpret_cast<const float4*>(p.meta + base + c));
    const float m = m4.y;
    const int a = __float_as_int(m4.w);
    if (isnan(m)) bad = 1;
    if (m > best || (m == best && a < arg)) {
      best = m;
      arg = a;
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, off);
    const int oa = __shfl_xor_sync(0xffffffffu, arg, off);
    if (ob > best || (ob == best && oa < arg)) {
      best = ob;
      arg = oa;
    }
  }
  bad = __any_sync(0xffffffffu, bad);
  if (isinf(best)) bad = 1;  // +inf, or -inf everywhere
  if (lane == 0) {
    out.Z = 0.0;
    out.ER = 0.0;
    out.EA = 0.0;
    out.K = 0.0f;
    out.mraw = best;
    out.arg = arg;
    out.bad = bad;
  }
}

// Exact fp64 normaliser sum_t exp(l_t / T - m) at the true temperature, over
// the whole block (slow path of an accept decision that fell inside its bound).
__device__ double exact_row_sum(const void* row, int64_t V, bool bf16, double T, double m,
                                double* red) {
  double s = 0.0;
  for (int64_t t = threadIdx.x; t < V; t += kThreads) {
    s += exp(static_cast<double>(load_logit(row, t, bf16)) / T - m);
  }
  return block_sum_d(s, red);
}

__device__ __forceinline__ double draw(const RunParams& p, int i, int j, int d) {
  if (p.uniforms) return __ldg(p.uniforms + (static_cast<int64_t>(i) * (p.k + 1) + j) * 2 + d);
  return draw_uniform(p.seed, p.req_off + static_cast<uint32_t>(i), static_cast<uint32_t>(j),
                      static_cast<uint32_t>(d), p.step);
}

constexpr double kU24 = 0x1p-24;
constexpr double kLn2 = 0.69314718055994530942;


template <bool BF16>
__device__ __forceinline__ TempConsts temp_consts(const RunParams& p, float Tf) {
  TempConsts t;
  t.T = static_cast<double>(Tf);
  t.cc = static_cast<float>(1.4426950408889634 / t.T);
  t.c_exact = 1.4426950408889634 / t.T;
  t.eta = fabs((t.c_exact - static_cast<double>(t.cc)) / static_cast<double>(t.cc));
  t.kappa = kLn2 * (kU24 + t.eta) * 1.0001;
  t.eps_base = static_cast<double>(p.eps_ex2) + SegGeo<BF16>::kSumLevels * kU24 + 1e-14;
  return t;
}

// Relative error bound of a row's fp32 normaliser Z~: one ex2 error per term,
// the pairwise rounding of the batch sums, and the exponent rounding (weighted
// by sum e|a|).  Rounding log2(e)/T to fp32 (relative eta) reshapes p itself:
// log p/p~ moves by at most ln2 * eta * |a_x - mean(a)|; that part is added
// where p(x) is formed.
__device__ __forceinline__ double row_dZ(const TempConsts& t, const RowMerged& r) {
  return t.eps_base + kLn2 * kU24 * 1.0002 * r.erz;
}

// Accept test of position j from the fp32 statistics of target row ra and
// draft row rb, given the drafted token's logits la, lb and the draw u:
// 1 accept, 0 reject, -1 inside the bound.  Also returns p~(x), q~(x).
// (Thread-local; any one thread may call it.)
template <bool BF16>
__device__ __forceinline__ int accept_eval(float la, float lb, double u, const RowMerged& ra,
                                          const RowMerged& rb, const TempConsts& t, double& pa,
                                          double& qb) {
  const double arg_a = static_cast<double>(la) * t.cc - static_cast<double>(ra.K);
  const double arg_b = static_cast<double>(lb) * t.cc - static_cast<double>(rb.K);
  pa = (la == -INFINITY) ? 0.0 : exp2(arg_a) * ra.invZ;
  qb = (lb == -INFINITY) ? 0.0 : exp2(arg_b) * rb.invZ;
  if (qb == 0.0) return pa > 0.0 ? 1 : 0;
  const double dp = row_dZ(t, ra) + kLn2 * t.eta * (fabs(arg_a + ra.eaz) + 1e-3);
  const double dq = row_dZ(t, rb) + kLn2 * t.eta * (fabs(arg_b + rb.eaz) + 1e-3);
  const double delta = (dp + dq) * 1.01 + 1e-13;
  // u against rho = p/q, compared as u q against p (q > 0)
  const double uq = u * qb;
  if (uq < pa * (1.0 - delta)) return 1;
  if (uq >= pa * (1.0 + delta)) return 0;
  return -1;
}

// The drafted token's logits at position j (target, draft): from the cache
// the statistics items (or the vocabulary-parallel gather) filled, else from
// the rows.
template <bool BF16>
__device__ __forceinline__ float2 token_logits(const RunParams& p, int i, int j, int xj) {
  const int64_t tl = (static_cast<int64_t>(i) * p.k + j) * 2;
  const float* cache = p.tok_logits ? p.tok_logits : p.tok_cache;
  if (cache) return make_float2(__ldcg(cache + tl), __ldcg(cache + tl + 1));
  return make_float2(load_logit(target_row(p, i, j, BF16), xj, BF16),
                     load_logit(draft_row(p, i, j, BF16), xj, BF16));
}

// Slow path of an accept decision inside its bound: both normalisers in fp64
// at the true temperature (all threads of the block).  Returns the exact
// decision in *accept (thread 0) and p(x), q(x).
template <bool BF16>
__device__ void accept_exact(const RunParams& p, int i, int j, int xj, const RowMerged& ra,
                             const RowMerged& rb, const TempConsts& t, double* red, bool& accept,
                             double& pa, double& qb) {
  const double ma = static_cast<double>(ra.mraw) / t.T;
  const double mb = static_cast<double>(rb.mraw) / t.T;
  const double Za = exact_row_sum(target_row(p, i, j, BF16), p.V, BF16, t.T, ma, red);
  sync_compute();
  const double Zb = exact_row_sum(draft_row(p, i, j, BF16), p.V, BF16, t.T, mb, red);
  if (threadIdx.x == 0) {
    const double la = load_logit(target_row(p, i, j, BF16), xj, BF16);
    const double lb = load_logit(draft_row(p, i, j, BF16), xj, BF16);
    pa = exp(la / t.T - ma) / Za;
    qb = exp(lb / t.T - mb) / Zb;
    const double u = draw(p, i, j, 0);
    atomicAdd(&p.counters->accept_slow, 1u);
    accept = u * qb < pa;
  }
}

// The job that samples position n of request i: the residual of row pair n
// (n < L) or the bonus row L; u2 is the sample's draw, draw(p, i, n, 1).
// (Thread 0.)
template <bool BF16>
__device__ void write_job(const RunParams& p, int i, int n, int L, const RowMerged& ra,
                          const RowMerged* rb, const TempConsts& t, double u2) {
  Job jb;
  jb.n = n;
  jb.pad0 = 0;
  jb.cc = t.cc;
  jb.kappa = static_cast<float>(t.kappa);
  jb.eta_ln2 = kLn2 * t.eta;
  jb.T = t.T;
  jb.u2 = u2;
  jb.row = n;
  jb.Ka = ra.K;
  jb.mraw_a = ra.mraw;
  if (n < L) {
    jb.kind = kJobResidual;
    jb.Kb = rb->K;
    jb.mraw_b = rb->mraw;
    jb.A = static_cast<float>(ra.invZ);
    jb.Bq = static_cast<float>(rb->invZ);
    // Sampling is scale free, so the weights may be compared with
    // (1 + alpha) max(0, p - q), alpha the relative error of the target's
    // fp32 1/Za (its normaliser's bound plus the rounding to fp32).  The
    // common factor then cancels from every target term, and what is left of
    // it is gamma = beta - alpha, the error of the ratio of the two
    // normalisers, which scales the draft terms only.  Per term: the ex2 error,
    // the scaled product's rounding and (target) the difference's rounding,
    // and |mean exponent| of the temperature-rounding term (the frame adds its
    // offset, the term its |a|); the draft terms also carry |gamma|.
    const double gamma = (kU24 + row_dZ(t, ra)) + (kU24 + row_dZ(t, *rb));
    jb.eps0a = static_cast<double>(p.eps_ex2) + 2 * kU24 + kLn2 * t.eta * ra.eaz * 1.0001;
    jb.eps0b = static_cast<double>(p.eps_ex2) + kU24 + kLn2 * t.eta * rb->eaz * 1.0001 + gamma * 1.0001;
    // Bracket of rho = Z_a / Z_b in the refinement's frames (each row relative
    // to its own max at the true temperature): the fp32 sums' bounds, the
    // reshaping by the rounded temperature factor, and a factor 3 of margin.
    const double rho = (ra.Z * rb->invZ) *
        exp2((static_cast<double>(ra.K) - static_cast<double>(rb->K)) -
             (static_cast<double>(ra.mraw) - static_cast<double>(rb->mraw)) * t.c_exact);
    const double band = 3.0 * (row_dZ(t, ra) + row_dZ(t, *rb) +
        kLn2 * t.eta * (fabs(static_cast<double>(ra.mraw) - static_cast<double>(rb->mraw)) * t.c_exact +
                        ra.eaz + rb->eaz + 1.0)) + 1e-12;
    jb.rho_lo = rho * (1.0 - band);
    jb.rho_hi = rho * (1.0 + band);
  } else {
    jb.kind = kJobBonus;
    jb.Kb = 0.0f;
    jb.mraw_b = 0.0f;
    jb.A = 1.0f;
    jb.Bq = 0.0f;
    jb.eps0a = static_cast<double>(p.eps_ex2) + 2 * kU24 + 1e-14;
    jb.eps0b = 0.0;
    jb.rho_lo = 0.0;
    jb.rho_hi = 0.0;
  }
  p.jobs[i] = jb;
}

// All outputs of request i at their "nothing decided" values (every thread).
__device__ __forceinline__ void write_defaults(const RunParams& p, int i) {
  const int k = p.k;
  int32_t* tok = p.out_tok + static_cast<int64_t>(i) * (k + 1);
  for (int j = threadIdx.x; j <= k; j += kThreads) tok[j] = -1;
  for (int j = threadIdx.x; j < k; j += kThreads) {
    if (p.out_p) p.out_p[static_cast<int64_t>(i) * k + j] = -1.0f;
    if (p.out_q) p.out_q[static_cast<int64_t>(i) * k + j] = -1.0f;
  }
}

// Request i failed with `status` (thread 0): outputs back to -1, n = -1.
__device__ __forceinline__ void fail_request(const RunParams& p, int i, uint32_t status) {
  const int k = p.k;
  int32_t* tok = p.out_tok + static_cast<int64_t>(i) * (k + 1);
  for (int jj = 0; jj <= k; ++jj) tok[jj] = -1;
  for (int jj = 0; jj < k; ++jj) {
    if (p.out_p) p.out_p[static_cast<int64_t>(i) * k + jj] = -1.0f;
    if (p.out_q) p.out_q[static_cast<int64_t>(i) * k + jj] = -1.0f;
  }
  p.out_acc[i] = -1;
  if (p.out_status) p.out_status[i] = status;
  p.jobs[i].kind = kJobNone;
}

// Resolve request i from position j0 on, once the statistics of its rows from
// j0 on are in (dense order: j0 = 0, every verified position's rows were read;
// the prefix order's dense tail: positions before j0 were accepted one at a
// time and their outputs are written).  Leaves p.jobs[i] describing the sample
// still to draw (kind kJobNone when the request is finished).
template <bool BF16>
__device__ void decide_request(const RunParams& p, int i, const ReqInfo& ri, DecideShared& sh,
                               int j0 = 0) {
  const int tid = threadIdx.x, warp = tid >> 5;
  const int k = p.k, L = ri.L;
  int32_t* tok = p.out_tok + static_cast<int64_t>(i) * (k + 1);
  float* op = p.out_p ? p.out_p + static_cast<int64_t>(i) * k : nullptr;
  float* oq = p.out_q ? p.out_q + static_cast<int64_t>(i) * k : nullptr;
  const int32_t* x = p.tokens + static_cast<int64_t>(i) * k;

  if (tid == 0) sh.state = 0;  // 2 once a sample job is written (read by the caller after a barrier)
  if (j0 == 0) write_defaults(p, i);
  if (ri.bad_T) {
    sync_compute();
    if (tid == 0) fail_request(p, i, kDevBadTemperature);
    return;
  }

  // Merge the rows the chain can read: target rows j0..L, draft rows j0..L-1.
  // A warp merging two rows loads both rows' records first.
  const int span = L - j0;
  const int nrows = ri.greedy ? span + 1 : 2 * span + 1;
  auto slot_of = [&](int r) { return r <= span ? j0 + r : (k + 1) + j0 + (r - (span + 1)); };
  if (ri.greedy) {
    for (int r = warp; r < nrows; r += kWarps) merge_greedy_row(p, i, slot_of(r), sh.rows[slot_of(r)]);
  } else {
    const int r0 = warp, r1 = warp + kWarps;
    SegRec f0{}, f1{};
    if (r0 < nrows) f0 = load_seg_rec(p, i, slot_of(r0));
    if (r1 < nrows) f1 = load_seg_rec(p, i, slot_of(r1));
    if (r0 < nrows) merge_stochastic_row(p, i, slot_of(r0), sh.rows[slot_of(r0)], f0);
    if (r1 < nrows) merge_stochastic_row(p, i, slot_of(r1), sh.rows[slot_of(r1)], f1);
    for (int r = warp + 2 * kWarps; r < nrows; r += kWarps)
      merge_stochastic_row(p, i, slot_of(r), sh.rows[slot_of(r)]);
  }
  sync_compute();

  if (ri.greedy) {
    if (tid == 0) {
      uint32_t status = 0;
      int n = L;
      for (int j = j0; j < L; ++j) {
        const int xj = __ldg(x + j);
        if (xj < 0 || static_cast<int64_t>(xj) >= p.V) { status = kDevBadToken; break; }
        if (sh.rows[j].bad) { status = kDevNonfinite; break; }
        const int a = sh.rows[j].arg;
        if (xj == a) { tok[j] = xj; continue; }
        tok[j] = a;
        n = j;
        break;
      }
      if (!status && n == L) {
        if (sh.rows[L].bad) status = kDevNonfinite;
        else tok[L] = sh.rows[L].arg;
      }
      if (status) {
        fail_request(p, i, status);
      } else {
        p.out_acc[i] = n;
        if (p.out_status) p.out_status[i] = 0;
        p.jobs[i].kind = kJobNone;
      }
    }
    return;
  }

  // Stochastic chain.  Thread j evaluates position j's accept test (all at
  // once: each waits on its own token logits); then the walk takes them in
  // order until the first rejection, the whole block settling a test inside
  // its bound in fp64 before the walk goes on.
  const TempConsts t = temp_consts<BF16>(p, ri.T);
  if (tid < span) {
    const int j = j0 + tid;
    const float* cache = p.tok_logits ? p.tok_logits : p.tok_cache;
    const int64_t tl = (static_cast<int64_t>(i) * k + j) * 2;
    float2 l = make_float2(0.0f, 0.0f);
    if (cache) l = make_float2(__ldcg(cache + tl), __ldcg(cache + tl + 1));  // with the token's load
    const int xj = __ldg(x + j);
    const RowMerged& ra = sh.rows[j];
    const RowMerged& rb = sh.rows[k + 1 + j];
    double pa = 0.0, qb = 0.0;
    int d;
    if (xj < 0 || static_cast<int64_t>(xj) >= p.V) {
      d = 2;
    } else if (ra.bad || rb.bad) {
      d = 3;
    } else {
      if (!cache) l = token_logits<BF16>(p, i, j, xj);
      d = accept_eval<BF16>(l.x, l.y, draw(p, i, j, 0), ra, rb, t, pa, qb);
    }
    sh.dec[j] = d;
    sh.pa[j] = pa;
    sh.qb[j] = qb;
  } else if (tid >= 32 && tid - 32 <= span) {
    const int j = j0 + tid - 32;
    sh.u2[j] = draw(p, i, j, 1);  // the sample's draw, wherever the chain ends
  }
  sync_compute();
  int n = L;
  uint32_t status = 0;
  for (int j = j0; j < L; ++j) {
    if (sh.dec[j] == -1) {
      if (p.fallback) {
        // the fp64 row sums need every rank's logits: the request is redone whole
        if (tid == 0) {
          for (int jj = j0; jj <= j; ++jj) {
            if (op) op[jj] = static_cast<float>(sh.pa[jj]);
            if (oq) oq[jj] = static_cast<float>(sh.qb[jj]);
          }
          p.fallback[i] = 1;
          p.jobs[i].kind = kJobNone;
        }
        return;
      }
      bool accept = false;
      double pa = 0.0, qb = 0.0;
      accept_exact<BF16>(p, i, j, __ldg(x + j), sh.rows[j], sh.rows[k + 1 + j], t, sh.red, accept, pa, qb);
      if (tid == 0) {
        sh.dec[j] = accept ? 1 : 0;
        sh.pa[j] = pa;
        sh.qb[j] = qb;
      }
      sync_compute();
    }
    const int d = sh.dec[j];
    if (d == 2 || d == 3) {
      status = d == 2 ? kDevBadToken : kDevNonfinite;
      break;
    }
    if (tid == 0) {
      if (op) op[j] = static_cast<float>(sh.pa[j]);
      if (oq) oq[j] = static_cast<float>(sh.qb[j]);
      if (d == 1) tok[j] = __ldg(x + j);
    }
    if (d != 1) {
      n = j;
      break;
    }
  }

  if (tid == 0) {
    if (!status && n == L && sh.rows[L].bad) status = kDevNonfinite;
    if (status) {
      fail_request(p, i, status);
      return;
    }
    p.out_acc[i] = n;
    if (p.out_status) p.out_status[i] = 0;
    write_job<BF16>(p, i, n, L, sh.rows[n], n < L ? &sh.rows[k + 1 + n] : nullptr, t, sh.u2[n]);
    sh.state = 2;
  }
}

// Prefix order: resolve position j of request i once its rows (target j, and
// draft j for a sampled position before L) are in.  Outcome in sh.state:
//   0 finished (outputs final, no job), 1 rows of position j+1 needed,
//   2 a sample job was written (p.jobs[i]).
template <bool BF16>
__device__ void decide_position(const RunParams& p, int i, const ReqInfo& ri, int j,
                                DecideShared& sh) {
  const int tid = threadIdx.x, warp = tid >> 5;
  const int k = p.k, L = ri.L;
  int32_t* tok = p.out_tok + static_cast<int64_t>(i) * (k + 1);
  float* op = p.out_p ? p.out_p + static_cast<int64_t>(i) * k : nullptr;
  float* oq = p.out_q ? p.out_q + static_cast<int64_t>(i) * k : nullptr;
  const int32_t* x = p.tokens + static_cast<int64_t>(i) * k;
  if (j == 0) write_defaults(p, i);
  if (ri.bad_T) {
    sync_compute();
    if (tid == 0) {
      fail_request(p, i, kDevBadTemperature);
      sh.state = 0;
    }
    sync_compute();
    return;
  }
  const bool pair = !ri.greedy && j < L;
  if (warp == 0) {
    if (ri.greedy) merge_greedy_row(p, i, j, sh.rows[0]);
    else merge_stochastic_row(p, i, j, sh.rows[0]);
  } else if (warp == 1 && pair) {
    merge_stochastic_row(p, i, k + 1 + j, sh.rows[1]);
  } else if (warp == 2) {
    // the position's other inputs, loaded while the rows are merged
    const int lane = tid & 31;
    if (lane == 0 && j < L) {
      const float* cache = p.tok_logits ? p.tok_logits : p.tok_cache;
      const int64_t tl = (static_cast<int64_t>(i) * k + j) * 2;
      if (pair && cache) {  // issued together with the token's load
        sh.la = __ldcg(cache + tl);
        sh.lb = __ldcg(cache + tl + 1);
      }
      const int xj = __ldg(x + j);
      sh.xj = xj;
      if (pair && !cache && xj >= 0 && static_cast<int64_t>(xj) < p.V) {
        const float2 l = token_logits<BF16>(p, i, j, xj);
        sh.la = l.x;
        sh.lb = l.y;
      }
    } else if (lane == 1 && pair) {
      sh.u = draw(p, i, j, 0);
    } else if (lane == 2 && !ri.greedy) {
      sh.u2[0] = draw(p, i, j, 1);
    } else if (lane == 3) {
      sh.tc = temp_consts<BF16>(p, ri.T);
    }
  }
  sync_compute();
  const RowMerged& ra = sh.rows[0];
  const RowMerged& rb = sh.rows[1];
  const TempConsts t = sh.tc;
  if (tid == 0) {
    sh.need_exact = -1;
    sh.state = 0;
    uint32_t status = 0;
    if (j == L) {  // the bonus row
      if (ra.bad) status = kDevNonfinite;
      else if (ri.greedy) tok[L] = ra.arg;
      if (!status) {
        p.out_acc[i] = L;
        if (p.out_status) p.out_status[i] = 0;
        if (ri.greedy) {
          p.jobs[i].kind = kJobNone;
        } else {
          write_job<BF16>(p, i, L, L, ra, nullptr, t, sh.u2[0]);
          sh.state = 2;
        }
      }
    } else {
      const int xj = sh.xj;
      if (xj < 0 || static_cast<int64_t>(xj) >= p.V) {
        status = kDevBadToken;
      } else if (ra.bad || (pair && rb.bad)) {
        status = kDevNonfinite;
      } else if (ri.greedy) {
        if (xj == ra.arg) {
          tok[j] = xj;
          sh.state = 1;
        } else {
          tok[j] = ra.arg;
          p.out_acc[i] = j;
          if (p.out_status) p.out_status[i] = 0;
          p.jobs[i].kind = kJobNone;
        }
      } else {
        double pa, qb;
        const int decision = accept_eval<BF16>(sh.la, sh.lb, sh.u, ra, rb, t, pa, qb);
        if (op) op[j] = static_cast<float>(pa);
        if (oq) oq[j] = static_cast<float>(qb);
        if (decision < 0) sh.need_exact = 1;
        else if (decision == 1) {
          tok[j] = xj;
          sh.state = 1;
        } else {
          p.out_acc[i] = j;
          if (p.out_status) p.out_status[i] = 0;
          write_job<BF16>(p, i, j, L, ra, &rb, t, sh.u2[0]);
          sh.state = 2;
        }
      }
    }
    if (status) fail_request(p, i, status);
  }
  sync_compute();
  if (sh.need_exact > 0) {
    bool accept = false;
    double pa = 0.0, qb = 0.0;
    const int xj = __ldg(x + j);
    accept_exact<BF16>(p, i, j, xj, ra, rb, t, sh.red, accept, pa, qb);
    if (tid == 0) {
      if (op) op[j] = static_cast<float>(pa);
      if (oq) oq[j] = static_cast<float>(qb);
      if (accept) {
        tok[j] = xj;
        sh.state = 1;
      } else {
        p.out_acc[i] = j;
        if (p.out_status) p.out_status[i] = 0;
        write_job<BF16>(p, i, j, L, ra, &rb, t, sh.u2[0]);
        sh.state = 2;
      }
    }
  }
  sync_compute();
}

// ---------------------------------------------------------------------------
// The kernel: one CTA per (request, row slot, segment).  The grid covers the
// first launch_rows slots of each request (all 2k + 1 when it is 0; k + 1,
// the target rows, for a greedy-only run); records keep the stride of 2k + 1
// slots per request either way.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_stats(RunParams p) {
  __shared__ StatsShared sh;
  __shared__ DecideShared dsh;
  const int rows_per_req = 2 * p.k + 1;
  const int launched = p.launch_rows > 0 ? p.launch_rows : rows_per_req;
  const int64_t b = blockIdx.x;
  const int seg = static_cast<int>(b % p.n_segs);
  const int64_t slot_launched = b / p.n_segs;
  const int i = static_cast<int>(slot_launched / launched);
  const int slot = static_cast<int>(slot_launched - static_cast<int64_t>(i) * launched);
  const int64_t slot_global = static_cast<int64_t>(i) * rows_per_req + slot;
  if (b == 0 && threadIdx.x == 0) *p.counters_next = Counters{};

  const ReqInfo ri = request_info(p, i);
  const bool is_draft = slot > p.k;
  const int j = is_draft ? slot - (p.k + 1) : slot;
  bool needed;
  if (ri.bad_T) needed = (slot == 0 && seg == 0);
  else if (ri.greedy) needed = !is_draft && j <= ri.L;
  else needed = is_draft ? (j < ri.L) : (j <= ri.L);
  if (!needed) return;

  if (!ri.bad_T) {
    const int64_t rec = slot_global * p.n_segs + seg;
    const void* row = is_draft ? draft_row(p, i, j, BF16) : target_row(p, i, j, BF16);
    if (ri.greedy) {
      greedy_segment<BF16>(row, p.V, seg, p.meta + rec, sh);
    } else {
      const float cc = static_cast<float>(1.4426950408889634 / static_cast<double>(ri.T));
      stochastic_segment<BF16>(row, p.V, seg, cc, p.meta + rec, p.ssum + rec, sh);
    }
  }
  if (!arrive_last(p.arrive_stats + i, static_cast<unsigned>(stats_expected(ri, p.n_segs)),
                   &sh.flag))
    return;
  __threadfence();
  decide_request<BF16>(p, i, ri, dsh);
}

}  // namespace sv
