// Pass 2: the one sample each stochastic request still needs -- from the
// residual distribution norm(max(0, p - q)) of the rejected row pair, or from the
// target's bonus row when the whole block survived ("Speculative decoding
// becomes standard: DSpark and multi-token drafters", section "Why
// draft-and-verify does not change the output").
//
// Inverse-CDF sampling in index order: the token is the smallest t whose
// running weight exceeds u * (total weight).  One CTA per (request, segment of
// kChunksPerSeg chunks) computes each chunk's weight mass in fp32 (fp64
// accumulation) together with a certified bound on its error; the request's
// last CTA prefixes the chunk masses block-wide, rescans the one chunk holding
// u * total and checks that the chosen cell's edges sit farther from u * total
// than the accumulated bound.  When they do not, the request is queued for the
// fp64 refinement (refine.cuh), which recomputes the weights exactly as the
// fp64 rule defines them.
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
// carries the ex2 error, the products' rounding, the normaliser's bound and the
// frame's share of the temperature-rounding term.
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

struct SampleShared {
  double d[kWarps];
  double cm[kChunksPerSeg][kWarps];   // per chunk masses of each warp
  double cb[kChunksPerSeg][kWarps];   // ... and bounds
  int flag;
  // locate
  int cstar;
  double base;        // weight before chunk cstar
  double base_bound;  // bound before chunk cstar
  int found;          // local index of the crossing in cstar, or -1
  int refine_slot;    // locate's outcome: -1 certain, else the refinement slot
  double lo_gap, hi_gap, cell_bound;
};

// One CTA per (request, segment of kChunksPerSeg chunks), coalesced loads, the
// next batch's vectors in flight while the current one is reduced.
template <bool BF16>
__device__ __forceinline__ void segment_masses(const RunParams& p, int i, const Job& jb, int seg,
                                               SampleShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const JobF32 j = job_f32(jb);
  const void* ra = target_row(p, i, jb.row, BF16);
  const void* rb = j.residual ? draft_row(p, i, jb.row, BF16) : nullptr;
  constexpr int kSteps = kChunksPerSeg * kBatchesPerChunk;
  const int c0 = seg * kChunksPerSeg;
  uint4 va[kVecsPerBatch], vb[kVecsPerBatch], na[kVecsPerBatch], nb[kVecsPerBatch];
  load_batch_coalesced<BF16>(ra, p.V, c0, 0, va);
  if (j.residual) load_batch_coalesced<BF16>(rb, p.V, c0, 0, vb);
  double cmass = 0.0, cbound = 0.0;
#pragma unroll 1
  for (int s = 0; s < kSteps; ++s) {
    if (s + 1 < kSteps) {
      const int c = c0 + (s + 1) / kBatchesPerChunk, b = (s + 1) % kBatchesPerChunk;
      load_batch_coalesced<BF16>(ra, p.V, c, b, na);
      if (j.residual) load_batch_coalesced<BF16>(rb, p.V, c, b, nb);
    }
    float sum, bound;
    double unused;
    batch_weights<BF16, false>(j, va, vb, sum, unused, bound);
    cmass += static_cast<double>(sum);
    cbound += static_cast<double>(bound);
    if ((s + 1) % kBatchesPerChunk == 0) {
      const double m = warp_sum_d(cmass);
      const double bb = warp_sum_d(cbound);
      if (lane == 0) {
        sh.cm[s / kBatchesPerChunk][warp] = m;
        sh.cb[s / kBatchesPerChunk][warp] = bb;
      }
      cmass = 0.0;
      cbound = 0.0;
    }
#pragma unroll
    for (int u = 0; u < kVecsPerBatch; ++u) {
      va[u] = na[u];
      if (j.residual) vb[u] = nb[u];
    }
  }
  sync_compute();
  if (threadIdx.x < kChunksPerSeg) {
    const int b = threadIdx.x;
    const int c = c0 + b;
    if (c < p.n_chunks) {
      double m = 0.0, bb = 0.0;
      for (int w2 = 0; w2 < kWarps; ++w2) {
        m += sh.cm[b][w2];
        bb += sh.cb[b][w2];
      }
      SampleChunk r;
      r.mass = m;
      // the bound was accumulated in fp32 per batch (inflate for its own
      // rounding), plus the pairwise rounding of the fp32 batch sums
      r.bound = bb * 1.001 + Geo<BF16>::kSumLevels * kU24 * m;
      p.smass[static_cast<int64_t>(i) * p.n_chunks + c] = r;
    }
  }
}

// The same masses fed by per-thread asynchronous staging: step s of the
// segment (chunk c0 + s / 4, batch s % 4) stages the target's two vectors in
// slots 0-1 and the draft's in slots 2-3 (bonus jobs: the target's only).
static_assert(2 * kVecsPerBatch == kStepVecs, "a staging step is one batch of both rows");

// FULL: the segment's two chunks lie inside the row, so no range checks.
template <bool BF16, bool FULL>
__device__ __forceinline__ void stage_sample_step(Stager& sg, const void* ra, const void* rb,
                                                  int64_t nvec, int c0, int s) {
  using G = Geo<BF16>;
  const int c = c0 + s / kBatchesPerChunk, b = s % kBatchesPerChunk;
  const int64_t base = static_cast<int64_t>(c) * G::kChunkVecs + threadIdx.x;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = base + static_cast<int64_t>(b * kVecsPerBatch + u) * kThreads;
    const bool valid = FULL || idx < nvec;
    cp_async16(sg.slot(s, u), static_cast<const uint4*>(ra) + (valid ? idx : 0), valid);
    if (rb) cp_async16(sg.slot(s, kVecsPerBatch + u), static_cast<const uint4*>(rb) + (valid ? idx : 0), valid);
  }
  cp_async_commit();
  ++sg.issued;
}

// The streaming part of segment_masses_staged (FULL: no range checks).
template <bool BF16, bool FULL>
__device__ __forceinline__ void segment_masses_pass(const JobF32& j, const void* ra, const void* rb,
                                                    int64_t nvec, int c0, SampleShared& sh,
                                                    uint4* stage_buf) {
  using G = Geo<BF16>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kSteps = kChunksPerSeg * kBatchesPerChunk;
  Stager sg{stage_buf};
#pragma unroll
  for (int st = 0; st < kStageSlots; ++st) stage_sample_step<BF16, FULL>(sg, ra, rb, nvec, c0, st);
  double cmass = 0.0, cbound = 0.0;
#pragma unroll 1
  for (int st = 0; st < kSteps; ++st) {
    cp_async_wait(sg.issued - st - 1);
    const int c = c0 + st / kBatchesPerChunk, b = st % kBatchesPerChunk;
    const int64_t base = static_cast<int64_t>(c) * G::kChunkVecs + threadIdx.x;
    uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
#pragma unroll
    for (int u = 0; u < kVecsPerBatch; ++u) {
      const bool valid = FULL || base + static_cast<int64_t>(b * kVecsPerBatch + u) * kThreads < nvec;
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
      if (lane == 0) {
        sh.cm[st / kBatchesPerChunk][warp] = m;
        sh.cb[st / kBatchesPerChunk][warp] = bb;
      }
      cmass = 0.0;
      cbound = 0.0;
    }
  }
}

template <bool BF16>
__device__ __forceinline__ void segment_masses_staged(const RunParams& p, int i, const Job& jb, int seg,
                                                      SampleShared& sh, uint4* stage_buf) {
  using G = Geo<BF16>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const JobF32 j = job_f32(jb);
  const void* ra = target_row(p, i, jb.row, BF16);
  const void* rb = j.residual ? draft_row(p, i, jb.row, BF16) : nullptr;
  const int64_t nvec = p.V / G::kPerVec;
  constexpr int kSteps = kChunksPerSeg * kBatchesPerChunk;
  const int c0 = seg * kChunksPerSeg;
  if ((static_cast<int64_t>(c0) + kChunksPerSeg) * G::kChunkVecs <= nvec)
    segment_masses_pass<BF16, true>(j, ra, rb, nvec, c0, sh, stage_buf);
  else
    segment_masses_pass<BF16, false>(j, ra, rb, nvec, c0, sh, stage_buf);
  sync_compute();
  if (threadIdx.x < kChunksPerSeg) {
    const int bc = threadIdx.x;
    const int c = c0 + bc;
    if (c < p.n_chunks) {
      double m = 0.0, bb = 0.0;
      for (int w2 = 0; w2 < kWarps; ++w2) {
        m += sh.cm[bc][w2];
        bb += sh.cb[bc][w2];
      }
      SampleChunk r;
      r.mass = m;
      r.bound = bb * 1.001 + Geo<BF16>::kSumLevels * kU24 * m;
      p.smass[static_cast<int64_t>(i) * p.n_chunks + c] = r;
    }
  }
}

// Last CTA of request i: find the token or queue the request for refinement.
template <bool BF16>
__device__ void locate_sample(const RunParams& p, int i, const Job& jb, SampleShared& sh) {
  using G = Geo<BF16>;
  const int tid = threadIdx.x;
  const SampleChunk* sc = p.smass + static_cast<int64_t>(i) * p.n_chunks;
  // 1. block-wide prefix of the chunk masses and bounds (thread t: chunks 4t..4t+3)
  double m[4], b[4], pm[4], pb[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = 4 * tid + q;
    if (c < p.n_chunks) {
      const double2 r = __ldcg(reinterpret_cast<const double2*>(sc + c));
      m[q] = r.x;
      b[q] = r.y;
    } else {
      m[q] = 0.0;
      b[q] = 0.0;
    }
  }
  if (tid == 0) sh.cstar = -1;
  const double total = chunk_prefix(m, pm, sh.d);
  sync_compute();
  const double tb = chunk_prefix(b, pb, sh.d) + 1e-15 * total;
  const double target = jb.u2 * total;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c = 4 * tid + q;
    if (c < p.n_chunks && pm[q] <= target && pm[q] + m[q] > target) {
      sh.cstar = c;
      sh.base = pm[q];
      sh.base_bound = pb[q] + 1e-15 * pm[q];
    }
  }
  sync_compute();
  int cstar = sh.cstar;
  // residual mass must clear the 1e-12 floor with certainty
  if (jb.kind == kJobResidual && !(total - tb > 1e-12 * (1.0 + 1e-9))) cstar = -1;
  // vocabulary-parallel: only the rank holding chunk cstar rescans it
  const bool sharded = p.c_hi > 0;
  if (sharded && cstar >= 0 && (cstar < p.c_lo || cstar >= p.c_hi)) {
    if (tid == 0) {
      p.shard_tok[i] = -2;
      sh.refine_slot = -1;
    }
    sync_compute();
    return;
  }
  bool certain = false;
  int token = -1;
  if (cstar >= 0) {
    // 2. rescan chunk cstar in index order (contiguous runs per thread): exact
    //    fp64 sums of the fp32 weights and their bounds
    const JobF32 j = job_f32(jb);
    const void* ra = target_row(p, i, jb.row, BF16);
    const void* rb = j.residual ? draft_row(p, i, jb.row, BF16) : nullptr;
    double tsum = 0.0, tbound = 0.0;
#pragma unroll 1
    for (int bt = 0; bt < kBatchesPerChunk; ++bt) {
      uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
      load_batch_contiguous<BF16>(ra, p.V, cstar, bt, va);
      if (j.residual) load_batch_contiguous<BF16>(rb, p.V, cstar, bt, vb);
      else for (int u = 0; u < kVecsPerBatch; ++u) vb[u] = va[u];
      float s, bd;
      double ex;
      batch_weights<BF16, true>(j, va, vb, s, ex, bd);
      tsum += ex;
      tbound += static_cast<double>(bd);
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
      double run = start, runb = sh.base_bound + preb * 1.001;
      bool done = false;
      for (int bt = 0; bt < kBatchesPerChunk && !done; ++bt) {
        uint4 va[kVecsPerBatch], vb[kVecsPerBatch];
        const int off = load_batch_contiguous<BF16>(ra, p.V, cstar, bt, va);
        if (j.residual) load_batch_contiguous<BF16>(rb, p.V, cstar, bt, vb);
        else for (int u = 0; u < kVecsPerBatch; ++u) vb[u] = va[u];
        const WeightCtx w = weight_ctx(j, vec_max<BF16>(va), j.residual ? vec_max<BF16>(vb) : 0.0f);
        for (int u = 0; u < kVecsPerBatch && !done; ++u) {
          float xa[G::kPerVec], xb[G::kPerVec];
          unpack<BF16>(va[u], xa);
          if (j.residual) unpack<BF16>(vb[u], xb);
          for (int q = 0; q < G::kPerVec; ++q) {
            float wt, bq;
            weight_and_bound(w, xa[q], j.residual ? xb[q] : 0.0f, wt, bq);
            const double before = run;
            run += static_cast<double>(wt);
            runb += static_cast<double>(bq) * 1.001;
            if (run > target) {
              sh.found = off + u * G::kPerVec + q;
              sh.lo_gap = target - before;
              sh.hi_gap = run - target;
              sh.cell_bound = runb;
              done = true;
              break;
            }
          }
        }
      }
    }
    sync_compute();
    if (tid == 0 && sh.found >= 0) {
      const double slack = jb.u2 * tb + 1e-14 * total;
      const double need = sh.cell_bound + slack;
      certain = sh.lo_gap > need && sh.hi_gap > need;
      token = static_cast<int>(static_cast<int64_t>(cstar) * G::kChunk + sh.found);
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
