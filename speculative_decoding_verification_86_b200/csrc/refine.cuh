// Pass 3 (only for samples the fp32 filter could not certify): the sample is
// recomputed in fp64 exactly as the rule defines it -- p_t = exp(l_t/T - m_p)
// / Z_p, q_t likewise, residual weight max(0, p_t - q_t) (or the target
// weight exp(l_t/T - m_p) for a bonus token, or when the residual mass is
// under the 1e-12 floor), inverse CDF in index order with the smallest-index
// rule and the largest-positive-index fallback.
//
// Work items are (queued request, sub-chunk of 4096 bf16 / 2048 fp32 logits:
// one batch of the chunk layout); together they make one fp64 pass over the
// row pair.  The exact normalisers Z_a, Z_b are only known once every
// chunk is done, but the residual's support {t : p_t > q_t} = {alpha_t > rho
// beta_t} (alpha = exp(a/T - m_a), beta likewise, rho = Z_a / Z_b) can be
// settled early: the fp32 pass bounds rho in [rho_lo, rho_hi], so a chunk adds
// alpha and beta of every logit with alpha > rho_hi beta to its support sums
// and only counts the few with rho_lo beta <= alpha <= rho_hi beta.  The
// request's last CTA then has each chunk's residual mass as A_c/Z_a - B_c/Z_b,
// recomputes outright the rare chunks holding unsettled logits (or all of
// them if rho missed its bracket), prefixes the masses block-wide and scans the
// one chunk holding u * total.  Weights are exp2_fast (fp64.cuh) of
// l * (log2(e)/T) - m * log2(e).
#pragma once
#include "common.cuh"
#include "fp64.cuh"
#include "stats.cuh"

namespace sv {

struct RefineShared {
  double tab[kExp2Table];
  double d[kWarps];
  int i[kWarps];
  int flag;
  int cstar;
  int redo_all;
  int use_part, ppart;  // final rescan narrowed to part ppart of the sub-chunk
  double pbase;
  int use_resid;
  int found;
  double base, target, Za, Zb;
};

struct RefineRow {
  double s, ma2, mb2;  // log2(e)/T and the row maxima times it (exponents in base 2)
};

__device__ __forceinline__ RefineRow refine_row(const Job& jb) {
  RefineRow r;
  r.s = kLog2E / jb.T;
  r.ma2 = static_cast<double>(jb.mraw_a) * r.s;
  r.mb2 = static_cast<double>(jb.mraw_b) * r.s;
  return r;
}

constexpr int kSubsPerChunk = kBatchesPerChunk;  // a sub-chunk is one batch of a chunk
constexpr int kSubVecs = kVecsPerBatch * kThreads;  // 512 contiguous vectors
constexpr int kSubPartVecs = kSubVecs / kWarps;     // 64: one warp's part of a sub-chunk

// Sub-chunk (c, bt), part layout: warp w holds the sub-chunk's vectors
// 64 w .. 64 w + 63, lane l the two vectors 64 w + l and 64 w + 32 + l, so a
// warp's sums cover one contiguous eighth of the sub-chunk.
template <bool BF16>
__device__ __forceinline__ void load_sub_parts(const void* row, int64_t V, int c, int bt,
                                               uint4 (&v)[kVecsPerBatch]) {
  using G = Geo<BF16>;
  const int64_t nvec = V / G::kPerVec;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t base = static_cast<int64_t>(c) * G::kChunkVecs + static_cast<int64_t>(bt) * kSubVecs +
                       (threadIdx.x >> 5) * kSubPartVecs + (threadIdx.x & 31);
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = base + u * 32;
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
}
static_assert(kVecsPerBatch * 32 == kSubPartVecs, "a warp's two loads cover its part");

// One pass over sub-chunk (c, bt): alpha/beta sums and, for residual jobs, the
// support sums A, B and the count of unsettled logits (alpha > 0 only: where
// alpha = 0, p_t = 0 and the weight is 0 whatever rho is).
template <bool BF16>
__device__ __forceinline__ void refine_sub_pass(const RunParams& p, int i, const Job& jb,
                                                const RefineRow& rr, int c, int bt, bool residual,
                                                const double* tab, double& za, double& zb,
                                                double& A, double& Bm, int& unc) {
  using G = Geo<BF16>;
  const void* ra = target_row(p, i, jb.row, BF16);
  const void* rb = residual ? draft_row(p, i, jb.row, BF16) : nullptr;
  uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
  load_sub_parts<BF16>(ra, p.V, c, bt, va);
  if (residual) load_sub_parts<BF16>(rb, p.V, c, bt, vb);
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    float xa[G::kPerVec], xb[G::kPerVec];
    unpack<BF16>(va[u], xa);
    if (residual) unpack<BF16>(vb[u], xb);
#pragma unroll
    for (int q = 0; q < G::kPerVec; ++q) {
      const double al = exp_weight(xa[q], rr.s, rr.ma2, tab);
      za += al;
      if (residual) {
        const double be = exp_weight(xb[q], rr.s, rr.mb2, tab);
        zb += be;
        if (al > be * jb.rho_hi) {
          A += al;
          Bm += be;
        } else if (al > 0.0 && al >= be * jb.rho_lo) {
          ++unc;
        }
      }
    }
  }
}

// Exact weight of the logit at chunk offset (bt, u, q) of the contiguous layout.
template <bool BF16>
__device__ __forceinline__ double exact_weight(float a, float b, bool use_resid,
                                               const RefineRow& rr, double iza, double izb,
                                               const double* tab) {
  const double pe = exp_weight(a, rr.s, rr.ma2, tab);
  if (!use_resid) return pe;
  const double r = pe * iza - exp_weight(b, rr.s, rr.mb2, tab) * izb;
  return r > 0.0 ? r : 0.0;
}

// Exact residual mass of sub-chunk (c, bt), block-reduced in a fixed order.
template <bool BF16>
__device__ double exact_sub_mass(const RunParams& p, int i, const Job& jb, const RefineRow& rr,
                                 int c, int bt, double iza, double izb, RefineShared& sh) {
  using G = Geo<BF16>;
  uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
  load_batch_coalesced<BF16>(target_row(p, i, jb.row, BF16), p.V, c, bt, va);
  load_batch_coalesced<BF16>(draft_row(p, i, jb.row, BF16), p.V, c, bt, vb);
  double m = 0.0;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    float xa[G::kPerVec], xb[G::kPerVec];
    unpack<BF16>(va[u], xa);
    unpack<BF16>(vb[u], xb);
#pragma unroll
    for (int q = 0; q < G::kPerVec; ++q) m += exact_weight<BF16>(xa[q], xb[q], true, rr, iza, izb, sh.tab);
  }
  sync_compute();
  return block_sum_d(m, sh.d);
}

// Sub-chunk (c, bt) is the contiguous logit range [c*kChunk + bt*4096 (bf16),
// +4096); in index order thread t holds its kVecsPerBatch vectors t*2, t*2+1.
template <bool BF16>
__device__ __forceinline__ int load_sub_contiguous(const void* row, int64_t V, int c, int bt,
                                                   uint4 (&v)[kVecsPerBatch]) {
  using G = Geo<BF16>;
  const int64_t nvec = V / G::kPerVec;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t base = static_cast<int64_t>(c) * G::kChunkVecs +
                       static_cast<int64_t>(bt) * (kVecsPerBatch * kThreads) +
                       threadIdx.x * kVecsPerBatch;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = base + u;
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
  return bt * G::kBatchElems * kThreads + threadIdx.x * G::kBatchElems;  // offset in the chunk
}

// One fp64 work item: sub-chunk `sub` of refinement slot `slot`.  Returns true
// in the CTA that completes the slot (all its sub-chunks are in).
template <bool BF16>
__device__ void refine_item(const RunParams& p, int slot, int sub, RefineShared& sh) {
  const int n_subs = p.n_chunks * kSubsPerChunk;
  const int i = __ldcg(p.refine_list + slot);
  const Job jb = load_job(p.jobs + i);
  const RefineRow rr = refine_row(jb);
  const bool residual = jb.kind == kJobResidual;
  double za = 0.0, zb = 0.0, A = 0.0, Bm = 0.0;
  int unc = 0;
  refine_sub_pass<BF16>(p, i, jb, rr, sub / kSubsPerChunk, sub % kSubsPerChunk, residual, sh.tab,
                        za, zb, A, Bm, unc);
  if (p.rmp) {  // the part sums, for a rescan of one part in the end
    const double zw = warp_sum_d(za), aw = warp_sum_d(A), bw = warp_sum_d(Bm);
    if ((threadIdx.x & 31) == 0)
      p.rmp[(static_cast<int64_t>(slot) * n_subs + sub) * kWarps + (threadIdx.x >> 5)] = make_double4(zw, aw, bw, 0.0);
  }
  za = block_sum_d(za, sh.d);
  zb = block_sum_d(zb, sh.d);
  A = block_sum_d(A, sh.d);
  Bm = block_sum_d(Bm, sh.d);
  unc = sync_compute_or(unc);
  const int64_t rec0 = static_cast<int64_t>(slot) * n_subs;
  if (threadIdx.x == 0) {
    p.rz[rec0 + sub] = make_double2(za, zb);
    p.rm[rec0 + sub] = make_double2(A, Bm);
    p.runc[rec0 + sub] = unc;
  }
}

// The last CTA of refinement slot `slot`: exact sub-chunk masses, the token.
template <bool BF16>
__device__ void refine_finalize(const RunParams& p, int slot, RefineShared& sh) {
  using G = Geo<BF16>;
  const int n_subs = p.n_chunks * kSubsPerChunk;
  const int i = __ldcg(p.refine_list + slot);
  const Job jb = load_job(p.jobs + i);
  const RefineRow rr = refine_row(jb);
  const bool residual = jb.kind == kJobResidual;
  const int64_t rec0 = static_cast<int64_t>(slot) * n_subs;
  // thread t owns sub-chunks 4t .. 4t+3
  double zav[4], zbv[4], pz[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ss = 4 * threadIdx.x + q;
    const double2 z = ss < n_subs ? __ldcg(p.rz + rec0 + ss) : make_double2(0.0, 0.0);
    zav[q] = z.x;
    zbv[q] = z.y;
  }
  const double Za = chunk_prefix(zav, pz, sh.d);
  const double Zb = chunk_prefix(zbv, pz, sh.d);
  const double iza = 1.0 / Za, izb = residual ? 1.0 / Zb : 0.0;
  const double rho = residual ? Za / Zb : 0.0;
  const bool redo_all = residual && !(rho >= jb.rho_lo && rho <= jb.rho_hi);
  double mv[4];
  int flagged = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ss = 4 * threadIdx.x + q;
    mv[q] = 0.0;
    if (ss < n_subs) {
      if (residual) {
        const double2 ab = __ldcg(p.rm + rec0 + ss);
        const double r = ab.x * iza - ab.y * izb;
        mv[q] = r > 0.0 ? r : 0.0;
        if (redo_all || __ldcg(p.runc + rec0 + ss)) flagged |= 1 << q;
      } else {
        mv[q] = zav[q];
      }
    }
  }
  // sub-chunks whose support was not settled: recompute outright (rare).  A
  // vocabulary shard holds only its own sub-chunks: the request is redone whole.
  const bool sharded = p.c_hi > 0;
  if (sharded && !p.rows_whole) {
    if (sync_compute_or(flagged)) {
      if (threadIdx.x == 0) p.shard_tok[i] = -1;
      sync_compute();
      return;
    }
  } else if (sync_compute_or(flagged)) {
#pragma unroll 1
    for (int ss = 0; ss < n_subs; ++ss) {
      const int owner = ss / 4;
      if (threadIdx.x == owner) sh.found = (flagged >> (ss % 4)) & 1;
      sync_compute();
      if (sh.found) {
        if (threadIdx.x == 0) atomicAdd(&p.counters->chunks_redone, 1u);
        const double m = exact_sub_mass<BF16>(p, i, jb, rr, ss / kSubsPerChunk,
                                              ss % kSubsPerChunk, iza, izb, sh);
        if (threadIdx.x == owner) mv[ss % 4] = m;
      }
      sync_compute();
    }
  }
  double pm[4];
  const double R = chunk_prefix(mv, pm, sh.d);
  const bool use_resid = residual && R >= 1e-12;
  if (!use_resid && residual) {  // floor: target weights exp(a/T - m_a)
#pragma unroll
    for (int q = 0; q < 4; ++q) mv[q] = zav[q];
    chunk_prefix(mv, pm, sh.d);
  }
  const double W = use_resid ? R : Za;
  const double target = jb.u2 * W;
  if (threadIdx.x == 0) {
    sh.cstar = -1;
    sh.found = -1;
  }
  sync_compute();
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ss = 4 * threadIdx.x + q;
    if (ss < n_subs && pm[q] <= target && pm[q] + mv[q] > target) {
      sh.cstar = ss;
      sh.base = pm[q];
    }
  }
  sync_compute();
  bool fallback = false;
  if (sh.cstar < 0) {
    // rounding left no cell above target: the last sub-chunk with positive weight
    int last = -1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int ss = 4 * threadIdx.x + q;
      if (ss < n_subs && mv[q] > 0.0) last = ss;
    }
    last = -block_min_i(last >= 0 ? -last : 1, sh.i);
    if (threadIdx.x == 0) sh.cstar = last >= 0 ? last : -1;
    sync_compute();
    fallback = true;
  }
  const int sstar = sh.cstar;
  if (sharded && sstar >= 0 &&
      (sstar / kSubsPerChunk < p.c_lo || sstar / kSubsPerChunk >= p.c_hi)) {
    if (threadIdx.x == 0) p.shard_tok[i] = -2;  // another rank holds the sub-chunk
    sync_compute();
    return;
  }
  int token = -1;
  // With settled support the part sums narrow the draw to one eighth of the
  // sub-chunk, and only that part is rescanned.
  bool by_part = false;
  if (sstar >= 0 && p.rmp && !fallback && !sharded) {
    if (threadIdx.x == sstar / 4) sh.use_part = !((flagged >> (sstar % 4)) & 1);
    sync_compute();
    if (sh.use_part) {
      if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        double m = 0.0;
        if (lane < kWarps) {
          const double2* r = reinterpret_cast<const double2*>(p.rmp + (rec0 + sstar) * kWarps + lane);
          const double2 r0 = __ldcg(r), r1 = __ldcg(r + 1);  // (alpha, A), (B, -)
          m = use_resid ? fmax(r0.y * iza - r1.x * izb, 0.0) : r0.x;
        }
        double incl = m;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        const double pre = incl - m;
        if (lane == 0) sh.ppart = -1;
        __syncwarp();
        if (lane < kWarps && sh.base + pre <= target && sh.base + pre + m > target) {
          sh.ppart = lane;
          sh.pbase = sh.base + pre;
        }
      }
      sync_compute();
      const int pp = sh.ppart;
      if (pp >= 0) {
        constexpr int kPartLogits = kSubPartVecs * G::kPerVec;  // 512 bf16 / 256 fp32
        constexpr int kPer = kPartLogits / kThreads;           // logits per thread
        static_assert(kPer * kThreads == kPartLogits, "a part spreads evenly over the block");
        const int c = sstar / kSubsPerChunk, bt = sstar % kSubsPerChunk;
        const int off0 = bt * (kSubVecs * G::kPerVec) + pp * kPartLogits + threadIdx.x * kPer;  // in the chunk
        const void* ra = target_row(p, i, jb.row, BF16);
        const void* rb = use_resid ? draft_row(p, i, jb.row, BF16) : nullptr;
        double w[kPer];
        double tsum = 0.0;
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
          const int64_t t = static_cast<int64_t>(c) * G::kChunk + off0 + e;
          w[e] = 0.0;
          if (t < p.V) {
            const float a = load_logit(ra, t, BF16);
            const float b = use_resid ? load_logit(rb, t, BF16) : 0.0f;
            w[e] = exact_weight<BF16>(a, b, use_resid, rr, iza, izb, sh.tab);
          }
          tsum += w[e];
        }
        double all;
        const double pre = block_exclusive_scan_d(tsum, sh.d, all);
        if (threadIdx.x == 0) sh.found = -1;
        sync_compute();
        const double start = sh.pbase + pre;
        if (start <= target && start + tsum > target) {
          double run = start;
#pragma unroll
          for (int e = 0; e < kPer; ++e) {
            run += w[e];
            if (run > target) {
              sh.found = off0 + e;
              break;
            }
          }
        }
        sync_compute();
        if (sh.found >= 0) {
          token = static_cast<int>(static_cast<int64_t>(c) * G::kChunk + sh.found);
          by_part = true;
        }
      }
    }
  }
  if (sstar >= 0 && !by_part) {
    const int c = sstar / kSubsPerChunk, bt = sstar % kSubsPerChunk;
    const void* ra = target_row(p, i, jb.row, BF16);
    const void* rb = use_resid ? draft_row(p, i, jb.row, BF16) : nullptr;
    uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
    const int off = load_sub_contiguous<BF16>(ra, p.V, c, bt, va);
    if (use_resid) load_sub_contiguous<BF16>(rb, p.V, c, bt, vb);
    double wv[G::kBatchElems];
    double tsum = 0.0;
    int last_pos = -1;
#pragma unroll
    for (int u = 0; u < kVecsPerBatch; ++u) {
      float xa[G::kPerVec], xb[G::kPerVec];
      unpack<BF16>(va[u], xa);
      if (use_resid) unpack<BF16>(vb[u], xb);
#pragma unroll
      for (int q = 0; q < G::kPerVec; ++q) {
        const double wt = exact_weight<BF16>(xa[q], use_resid ? xb[q] : 0.0f, use_resid, rr,
                                             iza, izb, sh.tab);
        wv[u * G::kPerVec + q] = wt;
        tsum += wt;
        if (wt > 0.0) last_pos = off + u * G::kPerVec + q;
      }
    }
    int found = -1;
    if (!fallback) {
      double all;
      const double pre = block_exclusive_scan_d(tsum, sh.d, all);
      const double start = sh.base + pre;
      if (start <= target && start + tsum > target) {
        double run = start;
#pragma unroll
        for (int e = 0; e < G::kBatchElems; ++e) {
          run += wv[e];
          if (run > target && sh.found < 0) sh.found = off + e;
        }
      }
      sync_compute();
      found = sh.found;
    }
    if (found < 0) {
      // fallback, or the sub-chunk's scanned total fell a rounding short of
      // target: the last logit of the sub-chunk with positive weight
      int neg = last_pos >= 0 ? -last_pos : INT_MAX;
      neg = block_min_i(neg, sh.i);
      found = neg == INT_MAX ? -1 : -neg;
    }
    token = found >= 0 ? static_cast<int>(static_cast<int64_t>(c) * G::kChunk + found) : -1;
  }
  if (threadIdx.x == 0 && sharded) {
    p.shard_tok[i] = token >= 0 ? token : -1;
  } else if (threadIdx.x == 0) {
    p.out_tok[static_cast<int64_t>(i) * (p.k + 1) + jb.n] = token;
    if (token < 0) {
      p.out_acc[i] = -1;
      if (p.out_status) p.out_status[i] |= kDevInternal;
    }
  }
  sync_compute();
}

}  // namespace sv
