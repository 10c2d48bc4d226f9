// Pass 2: the one sample each stochastic request still needs -- from the
// residual distribution norm(max(0, p - q)) of the rejected row pair, or from the
// target's bonus row when the whole block survived ("Speculative decoding
// becomes standard: DSpark and multi-token drafters", section "Why
// draft-and-verify does not change the output").
//
// Inverse-CDF sampling in index order: the token is the smallest t whose
// running weight exceeds u * (total weight).  The row pair is streamed in
// chunks (an engine item each; a segment of kChunksPerSeg chunks per CTA in
// the vocabulary-parallel kernels), warp w of the CTA streaming part w of the
// chunk, a contiguous eighth; every part's weight mass is summed in fp32 (fp64
// accumulation) together with a certified bound on its error.  The request's
// last CTA prefixes the part masses block-wide, rescans the one part holding
// u * total (one vector per thread) and checks that the chosen cell's edges
// sit farther from u * total than the bound on the error of
// (prefix - u * total): each term's bound counts 1 - u times before the cell
// and u times after it.  When they do not, the request is queued for the fp64
// refinement (refine.cuh), which recomputes the weights exactly as the fp64
// rule defines them.
#pragma once
#include "common.cuh"
#include "stage.cuh"
#include "stats.cuh"

namespace sv {

// Weight of one logit pair and its error bound (fp32 path), in a frame:
//   residual: w = max(0, p~ - q~) with p~ = 2^(a c - Fa) * Aeff, Aeff = 2^(Fa - Ka) / Za;
//   bonus:    w = 2^(a c - Fa) * Aeff, Aeff = 2^(Fa - Ka)  (unnormalised; sampling is scale free).
// Fa, Fb are integer frames at or above the logits they serve (a batch's own
// maximum), so the exponent argument, and with it its rounding, stays small.
// Bound per term: p~ (epsa + kappa |xa|) + q~ (epsb + kappa |xb|) where eps
// carries the ex2 error, the products' rounding and the frame's share of the
// temperature-rounding term; the error of the normalisers' ratio, the one part
// of their errors that does not cancel from a scale-free sample, rides on the
// draft terms (epsb).
struct WeightCtx {
  float cc, Fa, Fb, Aeff, Beff, kappa, epsa, epsb;
  bool residual;
};

__device__ __forceinline__ void weight_and_bound(const WeightCtx& w, float a, float b, float& wt,
                                                 float& bd) {
  const float xa = fmaxf(fmaf(a, w.cc, -w.Fa), -1024.0f);
  const float pa = ex2_approx(xa) * w.Aeff;
  if (!w.residual) {
    wt = pa;
    bd = pa * fmaf(w.kappa, -xa, w.epsa);
    return;
  }
  const float xb = fmaxf(fmaf(b, w.cc, -w.Fb), -1024.0f);
  const float qb = ex2_approx(xb) * w.Beff;
  wt = fmaxf(pa - qb, 0.0f);
  // Only cells where p >= q is possible can carry weight (errors are < 1e-4).
  const bool near = pa * 1.0001f >= qb;
  bd = near ? fmaf(pa, fmaf(w.kappa, -xa, w.epsa), qb * fmaf(w.kappa, -xb, w.epsb)) : 0.0f;
}

// 2^d for an integer d in [-126, 0], exactly.
__device__ __forceinline__ float pow2i(int d) { return __int_as_float((127 + d) << 23); }

// Frame of a set of logits whose maximum is `m`: the integer ceil(m c) (capped
// at the row's frame K), the matching scale 2^(F - K) * zinv and the bound's
// constant eps0 + eta_ln2 (K - F).  All-masked sets (or ones 2^-126 below the
// row's maximum) get scale 0: their weights are below 2^-126 of the maximum's.
__device__ __forceinline__ void make_frame(float m, float cc, float K, float zinv, float eps0,
                                           float eta_ln2, float& F, float& scale, float& eps) {
  F = fminf(ceilf(m * cc), K);
  const float d = F - K;  // <= 0, integer; -inf if all masked
  if (!(d >= -126.0f)) {
    scale = 0.0f;
    eps = 0.0f;
    F = K;
    return;
  }
  scale = zinv * pow2i(static_cast<int>(d));
  eps = fmaf(eta_ln2, -d, eps0);
}

struct JobF32 {  // the job's constants in the precision the fp32 pass uses
  float cc, Ka, Kb, A, Bq, kappa, eps0a, eps0b, eta_ln2;
  bool residual;
};

__device__ __forceinline__ JobF32 job_f32(const Job& jb) {
  JobF32 j;
  j.cc = jb.cc;
  j.Ka = jb.Ka;
  j.Kb = jb.Kb;
  j.A = jb.A;
  j.Bq = jb.Bq;
  j.kappa = jb.kappa;
  j.eps0a = static_cast<float>(jb.eps0a) * 1.0001f;
  j.eps0b = static_cast<float>(jb.eps0b) * 1.0001f;
  j.eta_ln2 = static_cast<float>(jb.eta_ln2) * 1.001f;
  j.residual = jb.kind == kJobResidual;
  return j;
}

__device__ __forceinline__ WeightCtx weight_ctx(const JobF32& j, float ma, float mb) {
  WeightCtx w;
  w.cc = j.cc;
  w.kappa = j.kappa;
  w.residual = j.residual;
  make_frame(ma, j.cc, j.Ka, j.A, j.eps0a, j.eta_ln2, w.Fa, w.Aeff, w.epsa);
  if (j.residual) make_frame(mb, j.cc, j.Kb, j.Bq, j.eps0b, j.eta_ln2, w.Fb, w.Beff, w.epsb);
  else { w.Fb = 0.0f; w.Beff = 0.0f; w.epsb = 0.0f; }
  return w;
}

// The weights and bounds of two logit pairs at once with packed fp32x2
// instructions.  Every weight is bit-identical to weight_and_bound's: the
// exponent argument is formed negated (F - x c, the same rounding), the draft
// term is carried negated (-q~), so p~ - q~ is one packed add.  The bound uses
// the same terms; its "near" test is taken on the exact value of
// 1.0001 p~ - q~, an equally valid criterion.
struct WeightCtx2 {
  float2 ncc, Fa, Fb, Aeff, nBeff, kappa, nkappa, epsa, nepsb;
  bool residual;
};

__device__ __forceinline__ WeightCtx2 pack_ctx(const WeightCtx& w) {
  WeightCtx2 v;
  v.ncc = make_float2(-w.cc, -w.cc);
  v.Fa = make_float2(w.Fa, w.Fa);
  v.Fb = make_float2(w.Fb, w.Fb);
  v.Aeff = make_float2(w.Aeff, w.Aeff);
  v.nBeff = make_float2(-w.Beff, -w.Beff);
  v.kappa = make_float2(w.kappa, w.kappa);
  v.nkappa = make_float2(-w.kappa, -w.kappa);
  v.epsa = make_float2(w.epsa, w.epsa);
  v.nepsb = make_float2(-w.epsb, -w.epsb);
  v.residual = w.residual;
  return v;
}

__device__ __forceinline__ void weight_and_bound2(const WeightCtx2& w, float2 a, float2 b,
                                                  float2& wt, float2& bd) {
  float2 na = ffma2(a, w.ncc, w.Fa);  // -(a c - Fa)
  na.x = fminf(na.x, 1024.0f);
  na.y = fminf(na.y, 1024.0f);
  const float2 pa = fmul2(make_float2(ex2_approx(-na.x), ex2_approx(-na.y)), w.Aeff);
  const float2 ta = ffma2(w.kappa, na, w.epsa);  // epsa + kappa |xa|
  if (!w.residual) {
    wt = pa;
    bd = fmul2(pa, ta);
    return;
  }
  float2 nb = ffma2(b, w.ncc, w.Fb);
  nb.x = fminf(nb.x, 1024.0f);
  nb.y = fminf(nb.y, 1024.0f);
  const float2 nqb = fmul2(make_float2(ex2_approx(-nb.x), ex2_approx(-nb.y)), w.nBeff);  // -q~
  const float2 diff = fadd2(pa, nqb);
  wt = make_float2(fmaxf(diff.x, 0.0f), fmaxf(diff.y, 0.0f));
  const float2 near = ffma2(pa, make_float2(1.0001f, 1.0001f), nqb);
  const float2 ntb = ffma2(w.nkappa, nb, w.nepsb);  // -(epsb + kappa |xb|)
  const float2 full = ffma2(pa, ta, fmul2(nqb, ntb));
  bd = make_float2(near.x >= 0.0f ? full.x : 0.0f, near.y >= 0.0f ? full.y : 0.0f);
}

// Weights of one batch (kBatchElems logits per thread), reduced two ways:
// `sum` is their pairwise fp32 sum (the mass pass), `exact` the fp64 sum of the
// same fp32 weights (the rescans); `bound` sums their error bounds in fp32.
// The pairwise tree has depth log2(kBatchElems) = Geo::kSumLevels.
template <bool BF16, bool EXACT>
__device__ __forceinline__ void batch_weights(const JobF32& j, const uint4 (&va)[kVecsPerBatch],
                                              const uint4 (&vb)[kVecsPerBatch], float& sum,
                                              double& exact, float& bound) {
  constexpr int kPairs = BF16 ? 4 : 2;  // logit pairs per vector
  const WeightCtx2 w = pack_ctx(weight_ctx(j, vec_max<BF16>(va), j.residual ? vec_max<BF16>(vb) : 0.0f));
  float2 bd_sum = make_float2(0.0f, 0.0f);
  float2 vs[kVecsPerBatch];
  double ex = 0.0;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const uint32_t wa[4] = {va[u].x, va[u].y, va[u].z, va[u].w};
    const uint32_t wb[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
    float2 wt[kPairs];
#pragma unroll
    for (int q = 0; q < kPairs; ++q) {
      float2 xa, xb;
      if constexpr (BF16) {
        xa = make_float2(bf16_lo(wa[q]), bf16_hi(wa[q]));
        xb = make_float2(bf16_lo(wb[q]), bf16_hi(wb[q]));
      } else {
        xa = make_float2(__uint_as_float(wa[2 * q]), __uint_as_float(wa[2 * q + 1]));
        xb = make_float2(__uint_as_float(wb[2 * q]), __uint_as_float(wb[2 * q + 1]));
      }
      float2 bd;
      weight_and_bound2(w, xa, xb, wt[q], bd);
      bd_sum = fadd2(bd_sum, bd);
      if (EXACT) ex += static_cast<double>(wt[q].x) + static_cast<double>(wt[q].y);
    }
    if constexpr (BF16) {
      vs[u] = fadd2(fadd2(wt[0], wt[1]), fadd2(wt[2], wt[3]));
    } else {
      vs[u] = fadd2(wt[0], wt[1]);
    }
  }
  const float2 t = fadd2(vs[0], vs[1]);
  sum = t.x + t.y;
  exact = ex;
  bound = bd_sum.x + bd_sum.y;
}

constexpr int kChunksPerSeg = SegGeo<true>::kSegVecs / Geo<true>::kChunkVecs;  // 2
static_assert(SegGeo<false>::kSegVecs / Geo<false>::kChunkVecs == kChunksPerSeg, "geometry");

// Mass record of part (c, this warp) of request i (lane 0 of the warp that
// streamed it): the bound was accumulated in fp32 per batch (inflated for its
// own rounding), plus the pairwise rounding of the fp32 batch sums.
template <bool BF16>
__device__ __forceinline__ void write_part(const RunParams& p, int i, int c, double m, double bb) {
  SampleChunk r;
  r.mass = m;
  r.bound = bb * 1.001 + Geo<BF16>::kSumLevels * kU24 * m;
  p.smass[(static_cast<int64_t>(i) * p.n_chunks + c) * kSampleParts + (threadIdx.x >> 5)] = r;
}

struct SampleShared {
  double d[kWarps];
  int flag;
  // locate
  int pstar;          // the part holding u * total, or -1
  double base;        // weight before part pstar
  double base_bound;  // bound before part pstar
  double pstar_bound; // the mass record's bound of part pstar
  double after_bound; // bound of the parts after pstar
  int found;          // index of the crossing inside part pstar, or -1
  int refine_slot;    // locate's outcome: -1 certain, else the refinement slot
  double lo_gap, hi_gap;
  double lo_bound, hi_bound;  // rescan bounds of part pstar's cells before / through the crossing
};

// One CTA per (request, segment of kChunksPerSeg chunks), the next batch's
// vectors in flight while the current one is reduced; each warp writes the
// records of its parts.
template <bool BF16>
__device__ __forceinline__ void segment_masses(const RunParams& p, int i, const Job& jb, int seg,
                                               SampleShared& sh) {
  const int lane = threadIdx.x & 31;
  const JobF32 j = job_f32(jb);
  const void* ra = target_row(p, i, jb.row, BF16);
  const void* rb = j.residual ? draft_row(p, i, jb.row, BF16) : nullptr;
  constexpr int kSteps = kChunksPerSeg * kBatchesPerChunk;
  const int c0 = seg * kChunksPerSeg;
  uint4 va[kVecsPerBatch], vb[kVecsPerBatch], na[kVecsPerBatch], nb[kVecsPerBatch];
  load_batch_parts<BF16>(ra, p.V, c0, 0, va);
  if (j.residual) load_batch_parts<BF16>(rb, p.V, c0, 0, vb);
  double cmass = 0.0, cbound = 0.0;
#pragma unroll 1
  for (int s = 0; s < kSteps; ++s) {
    if (s + 1 < kSteps) {
      const int c = c0 + (s + 1) / kBatchesPerChunk, b = (s + 1) % kBatchesPerChunk;
      load_batch_parts<BF16>(ra, p.V, c, b, na);
      if (j.residual) load_batch_parts<BF16>(rb, p.V, c, b, nb);
    }
    float sum, bound;
    double unused;
    batch_weights<BF16, false>(j, va, vb, sum, unused, bound);
    cmass += static_cast<double>(sum);
    cbound += static_cast<double>(bound);
    if ((s + 1) % kBatchesPerChunk == 0) {
      const double m = warp_sum_d(cmass);
      const double bb = warp_sum_d(cbound);
      const int c = c0 + s / kBatchesPerChunk;
      if (lane == 0 && c < p.n_chunks) write_part<BF16>(p, i, c, m, bb);
      cmass = 0.0;
      cbound = 0.0;
    }
#pragma unroll
    for (int u = 0; u < kVecsPerBatch; ++u) {
      va[u] = na[u];
      if (j.residual) vb[u] = nb[u];
    }
  }
}

// The same masses fed by per-thread asynchronous staging: step s (chunk
// c0 + s / 4, batch s % 4) stages the target's two vectors in slots 0-1 and
// the draft's in slots 2-3 (bonus jobs: the target's only).
static_assert(2 * kVecsPerBatch == kStepVecs, "a staging step is one batch of both rows");

// FULL: the item's chunks lie inside the row, so no range checks.
template <bool BF16, bool FULL>
__device__ __forceinline__ void stage_sample_step(Stager& sg, const void* ra, const void* rb,
                                                  int64_t nvec, int c0, int s) {
  const int c = c0 + s / kBatchesPerChunk, b = s % kBatchesPerChunk;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = part_vec_index<BF16>(c, b, u);
    const bool valid = FULL || idx < nvec;
    cp_async16(sg.slot(s, u), static_cast<const uint4*>(ra) + (valid ? idx : 0), valid);
    if (rb) cp_async16(sg.slot(s, kVecsPerBatch + u), static_cast<const uint4*>(rb) + (valid ? idx : 0), valid);
  }
  cp_async_commit();
  ++sg.issued;
}

// The streaming part of chunk_masses_staged over NC chunks from c0 (FULL: no
// range checks).
template <bool BF16, bool FULL, int NC>
__device__ __forceinline__ void chunk_masses_pass(const RunParams& p, int i, const JobF32& j,
                                                  const void* ra, const void* rb, int64_t nvec, int c0,
                                                  uint4* stage_buf) {
  const int lane = threadIdx.x & 31;
  constexpr int kSteps = NC * kBatchesPerChunk;
  Stager sg{stage_buf};
#pragma unroll
  for (int st = 0; st < kStageSlots && st < kSteps; ++st) stage_sample_step<BF16, FULL>(sg, ra, rb, nvec, c0, st);
  double cmass = 0.0, cbound = 0.0;
#pragma unroll 1
  for (int st = 0; st < kSteps; ++st) {
    cp_async_wait(sg.issued - st - 1);
    const int c = c0 + st / kBatchesPerChunk, b = st % kBatchesPerChunk;
    uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
#pragma unroll
    for (int u = 0; u < kVecsPerBatch; ++u) {
      const bool valid = FULL || part_vec_index<BF16>(c, b, u) < nvec;
      va[u] = valid ? *sg.slot(st, u) : neg_inf_vec<BF16>();
      vb[u] = rb ? (valid ? *sg.slot(st, kVecsPerBatch + u) : neg_inf_vec<BF16>()) : va[u];
    }
    float sum, bound;
    double unused;
    batch_weights<BF16, false>(j, va, vb, sum, unused, bound);
    cmass += static_cast<double>(sum);
    cbound += static_cast<double>(bound);
    if (st + kStageSlots < kSteps) stage_sample_step<BF16, FULL>(sg, ra, rb, nvec, c0, st + kStageSlots);
    if ((st + 1) % kBatchesPerChunk == 0) {
      const double m = warp_sum_d(cmass);
      const double bb = warp_sum_d(cbound);
      if (lane == 0 && c < p.n_chunks) write_part<BF16>(p, i, c, m, bb);
      cmass = 0.0;
      cbound = 0.0;
    }
  }
}

// The masses of the parts of NC chunks from c0 (one engine item), fed by the
// staging.
template <bool BF16, int NC>
__device__ __forceinline__ void chunk_masses_staged(const RunParams& p, int i, const Job& jb, int c0,
                                                    uint4* stage_buf) {
  static_assert(NC >= 1 && NC <= kChunksPerSeg, "chunks per item");
  using G = Geo<BF16>;
  const JobF32 j = job_f32(jb);
  const void* ra = target_row(p, i, jb.row, BF16);
  const void* rb = j.residual ? draft_row(p, i, jb.row, BF16) : nullptr;
  const int64_t nvec = p.V / G::kPerVec;
  if ((static_cast<int64_t>(c0) + NC) * G::kChunkVecs <= nvec)
    chunk_masses_pass<BF16, true, NC>(p, i, j, ra, rb, nvec, c0, stage_buf);
  else
    chunk_masses_pass<BF16, false, NC>(p, i, j, ra, rb, nvec, c0, stage_buf);
}

// The mass record of one part (`part` = chunk * kSampleParts + warp index)
// computed by a whole CTA, for small batches whose chunk items would leave
// most of the grid idle: thread t takes vector t of the part in each row.
template <bool BF16>
__device__ __forceinline__ void part_mass_item(const RunParams& p, int i, const Job& jb, int part,
                                               SampleShared& sh) {
  using G = Geo<BF16>;
  const JobF32 j = job_f32(jb);
  const uint4* ra = static_cast<const uint4*>(target_row(p, i, jb.row, BF16));
  const uint4* rb = j.residual ? static_cast<const uint4*>(draft_row(p, i, jb.row, BF16)) : nullptr;
  const int64_t nvec = p.V / G::kPerVec;
  const int64_t vi = static_cast<int64_t>(part) * G::kPartVecs + threadIdx.x;
  uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    va[u] = neg_inf_vec<BF16>();
    vb[u] = neg_inf_vec<BF16>();
  }
  if (vi < nvec) {
    va[0] = ld_stream(ra + vi);
    vb[0] = rb ? ld_stream(rb + vi) : va[0];
  }
  float sum, bound;
  double unused;
  batch_weights<BF16, false>(j, va, vb, sum, unused, bound);
  const double m = block_sum_d(static_cast<double>(sum), sh.d);
  const double bb = block_sum_d(static_cast<double>(bound), sh.d);
  if (threadIdx.x == 0) {
    SampleChunk r;
    r.mass = m;
    r.bound = bb * 1.001 + Geo<BF16>::kSumLevels * kU24 * m;
    p.smass[static_cast<int64_t>(i) * p.n_chunks * kSampleParts + part] = r;
  }
}

constexpr int kPartsPerThread = 8;  // records per thread in the locate prefix
static_assert(kMaxChunksPerRow / kBatchesPerChunk * kSampleParts <= kPartsPerThread * kThreads,
              "the locate prefix covers every part of the longest row");

// Last CTA of request i: find the token or queue the request for refinement.
template <bool BF16>
__device__ void locate_sample(const RunParams& p, int i, const Job& jb, SampleShared& sh) {
  using G = Geo<BF16>;
  const int tid = threadIdx.x;
  const int n_parts = p.n_chunks * kSampleParts;
  const SampleChunk* sc = p.smass + static_cast<int64_t>(i) * n_parts;
  // 1. block-wide prefix of the part masses and bounds (thread t: parts
  //    8t .. 8t+7)
  double m[kPartsPerThread], b[kPartsPerThread];
  double mloc = 0.0, bloc = 0.0;
#pragma unroll
  for (int q = 0; q < kPartsPerThread; ++q) {
    const int c = kPartsPerThread * tid + q;
    if (c < n_parts) {
      const double2 r = __ldcg(reinterpret_cast<const double2*>(sc + c));
      m[q] = r.x;
      b[q] = r.y;
    } else {
      m[q] = 0.0;
      b[q] = 0.0;
    }
    mloc += m[q];
    bloc += b[q];
  }
  if (tid == 0) sh.pstar = -1;
  double total, tball;
  const double mbase = block_exclusive_scan_d(mloc, sh.d, total);
  sync_compute();
  const double bbase = block_exclusive_scan_d(bloc, sh.d, tball);
  const double tb = tball + 1e-15 * total;
  const double target = jb.u2 * total;
  double pmq = mbase, pbq = bbase;  // prefixes before part q
#pragma unroll
  for (int q = 0; q < kPartsPerThread; ++q) {
    const int c = kPartsPerThread * tid + q;
    if (c < n_parts && pmq <= target && pmq + m[q] > target) {
      sh.pstar = c;
      sh.base = pmq;
      sh.base_bound = pbq + 1e-15 * pmq;
      sh.pstar_bound = b[q];
      sh.after_bound = fmax(0.0, tb - pbq - b[q]) + 1e-12 * tb;
    }
    pmq += m[q];
    pbq += b[q];
  }
  sync_compute();
  int pstar = sh.pstar;
  // residual mass must clear the 1e-12 floor with certainty
  if (jb.kind == kJobResidual && !(total - tb > 1e-12 * (1.0 + 1e-9))) pstar = -1;
  // vocabulary-parallel: only the rank holding part pstar's chunk rescans it
  const bool sharded = p.c_hi > 0;
  const int cstar = pstar / kSampleParts;
  if (sharded && pstar >= 0 && (cstar < p.c_lo || cstar >= p.c_hi)) {
    if (tid == 0) {
      p.shard_tok[i] = -2;
      sh.refine_slot = -1;
    }
    sync_compute();
    return;
  }
  bool certain = false;
  int token = -1;
  if (pstar >= 0) {
    // 2. rescan part pstar in index order (thread t: vector t of the part):
    //    exact fp64 sums of the fp32 weights and their bounds
    const JobF32 j = job_f32(jb);
    const uint4* ra = static_cast<const uint4*>(target_row(p, i, jb.row, BF16));
    const uint4* rb = j.residual ? static_cast<const uint4*>(draft_row(p, i, jb.row, BF16)) : nullptr;
    const int64_t nvec = p.V / G::kPerVec;
    const int64_t vi = static_cast<int64_t>(pstar) * G::kPartVecs + tid;
    const uint4 va = vi < nvec ? ld_stream(ra + vi) : neg_inf_vec<BF16>();
    const uint4 vb = rb ? (vi < nvec ? ld_stream(rb + vi) : neg_inf_vec<BF16>()) : va;
    uint4 fa[kVecsPerBatch], fb[kVecsPerBatch];  // the frames: this vector's own maxima
#pragma unroll
    for (int u = 0; u < kVecsPerBatch; ++u) {
      fa[u] = va;
      fb[u] = vb;
    }
    const WeightCtx w = weight_ctx(j, vec_max<BF16>(fa), j.residual ? vec_max<BF16>(fb) : 0.0f);
    float xa[G::kPerVec], xb[G::kPerVec];
    unpack<BF16>(va, xa);
    unpack<BF16>(vb, xb);
    double tsum = 0.0, tbound = 0.0;
#pragma unroll
    for (int q = 0; q < G::kPerVec; ++q) {
      float wt, bq;
      weight_and_bound(w, xa[q], j.residual ? xb[q] : 0.0f, wt, bq);
      tsum += static_cast<double>(wt);
      tbound += static_cast<double>(bq);
    }
    double all, allb;
    const double pre = block_exclusive_scan_d(tsum, sh.d, all);
    sync_compute();
    const double preb = block_exclusive_scan_d(tbound, sh.d, allb);
    const double start = sh.base + pre;
    if (tid == 0) sh.found = -1;
    sync_compute();
    if (start <= target && start + tsum > target) {
      // the one thread holding the crossing walks its logits again (same values)
      double run = start, runb = preb * 1.001;
      for (int q = 0; q < G::kPerVec; ++q) {
        float wt, bq;
        weight_and_bound(w, xa[q], j.residual ? xb[q] : 0.0f, wt, bq);
        const double before = run, before_b = runb;
        run += static_cast<double>(wt);
        runb += static_cast<double>(bq) * 1.001;
        if (run > target) {
          sh.found = tid * G::kPerVec + q;
          sh.lo_gap = target - before;
          sh.hi_gap = run - target;
          sh.lo_bound = before_b;
          sh.hi_bound = runb;
          break;
        }
      }
    }
    sync_compute();
    if (tid == 0 && sh.found >= 0) {
      // The gaps are u W - S(<x) and S(<=x) - u W.  A term's error enters the
      // prefix S with weight 1 and the target u W with weight u, so the
      // parts before pstar count (1 - u) times, those after it u times.
      // Part pstar's record enters the total (u times); its cells are
      // recomputed by the rescan, whose own bounds enter the prefix.
      const double u = jb.u2;
      const double common = (1.0 - u) * sh.base_bound + u * (sh.after_bound + sh.pstar_bound) +
                            1e-14 * total;
      certain = sh.lo_gap > common + sh.lo_bound && sh.hi_gap > common + sh.hi_bound;
      token = static_cast<int>(static_cast<int64_t>(pstar) * G::kPart + sh.found);
    }
  }
  if (tid == 0) {
    if (sharded) {
      // the fp64 refinement would need every rank's logits: redo the request whole
      p.shard_tok[i] = certain ? token : -1;
      if (certain) atomicAdd(&p.counters->sample_fast, 1u);
      sh.refine_slot = -1;
    } else if (certain) {
      p.out_tok[static_cast<int64_t>(i) * (p.k + 1) + jb.n] = token;
      atomicAdd(&p.counters->sample_fast, 1u);
      sh.refine_slot = -1;
    } else {
      const unsigned slot = atomicAdd(&p.counters->refine_count, 1u);
      p.refine_list[slot] = i;
      sh.refine_slot = static_cast<int>(slot);
    }
  }
  sync_compute();
}

}  // namespace sv
