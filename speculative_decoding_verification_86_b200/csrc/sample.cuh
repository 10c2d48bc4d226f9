// Pass 2: the one sample each stochastic request still needs -- from the
// corrected residual norm(max(0, p - q)) of the rejected row pair, or from the
// target's bonus row when the whole block survived ("Speculative decoding
// becomes standard: DSpark and multi-token drafters", section "Why
// draft-and-verify does not change the output").
//
// Inverse-CDF sampling in index order: the token is the smallest t whose
// running weight exceeds u * (total weight).  One CTA per (request, chunk)
// computes the chunk's weight mass in fp32 (fp64 accumulation) together with
// a certified bound on its error; the request's last CTA prefixes the chunk
// masses, rescans the one chunk holding u * total and checks that the chosen
// cell's edges sit farther from u * total than the accumulated bound.  When
// they do not, the request is queued for the fp64 refinement (refine.cuh),
// which recomputes the weights exactly as the fp64 rule defines them.
#pragma once
#include "common.cuh"
#include "stats.cuh"

namespace sv {

// Weight of one logit pair and its error bound (fp32 path).
//   residual: w = max(0, p~ - q~) with p~ = 2^(a c - Ka) / Za, q~ likewise;
//   bonus:    w = 2^(a c - Ka)  (unnormalised; sampling is scale free).
struct WeightCtx {
  float cc, Ka, Kb, A, Bq, kappa, eps0a, eps0b;
  bool residual;
};

__device__ __forceinline__ void weight_and_bound(const WeightCtx& w, float a, float b, float& wt,
                                                 float& bd) {
  const float xa = fmaxf(fmaf(a, w.cc, -w.Ka), -1024.0f);
  const float pa = ex2_approx(xa) * w.A;
  if (!w.residual) {
    wt = pa;
    bd = pa * fmaf(w.kappa, fabsf(xa), w.eps0a);
    return;
  }
  const float xb = fmaxf(fmaf(b, w.cc, -w.Kb), -1024.0f);
  const float qb = ex2_approx(xb) * w.Bq;
  wt = fmaxf(pa - qb, 0.0f);
  // Only cells where p >= q is possible can carry weight (errors are < 1e-4).
  const bool near = pa * 1.0001f >= qb;
  bd = near ? fmaf(pa, fmaf(w.kappa, fabsf(xa), w.eps0a), qb * fmaf(w.kappa, fabsf(xb), w.eps0b))
            : 0.0f;
}

__device__ __forceinline__ WeightCtx weight_ctx(const Job& jb) {
  WeightCtx w;
  w.cc = jb.cc;
  w.Ka = jb.Ka;
  w.Kb = jb.Kb;
  w.A = jb.A;
  w.Bq = jb.Bq;
  w.kappa = jb.kappa;
  w.eps0a = static_cast<float>(jb.eps0a);
  w.eps0b = static_cast<float>(jb.eps0b);
  w.residual = jb.kind == kJobResidual;
  return w;
}

struct SampleShared {
  double d[kWarps];
  float f[kWarps];
  int flag;
  // locate
  int cstar;
  double base;        // weight before chunk cstar
  double base_bound;  // bound before chunk cstar (incl. accumulation slack)
  double total;       // total weight
  double total_bound;
  int found;          // local index of the crossing in cstar, or -1
  double lo_gap, hi_gap, cell_bound;
};

// Chunk-ordered vectors again: thread t holds vectors t, t + 256, ... so the
// loads coalesce, exactly as in the statistics pass.
template <bool BF16>
__device__ __forceinline__ void chunk_mass(const RunParams& p, int i, const Job& jb, int c,
                                           SampleShared& sh) {
  using G = Geo<BF16>;
  const WeightCtx w = weight_ctx(jb);
  uint4 va[kUnroll], vb[kUnroll];
  load_chunk<BF16>(target_row(p, i, jb.row, BF16), p.V, c, va);
  if (w.residual) load_chunk<BF16>(draft_row(p, i, jb.row, BF16), p.V, c, vb);
  float vsum[kUnroll];
  float bound = 0.0f;
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    float xa[G::kPerVec], xb[G::kPerVec], wt[G::kPerVec];
    unpack<BF16>(va[u], xa);
    if (w.residual) unpack<BF16>(vb[u], xb);
#pragma unroll
    for (int q = 0; q < G::kPerVec; ++q) {
      float bd;
      weight_and_bound(w, xa[q], w.residual ? xb[q] : 0.0f, wt[q], bd);
      bound += bd;
    }
    if constexpr (BF16) {
      vsum[u] = ((wt[0] + wt[1]) + (wt[2] + wt[3])) + ((wt[4] + wt[5]) + (wt[6] + wt[7]));
    } else {
      vsum[u] = (wt[0] + wt[1]) + (wt[2] + wt[3]);
    }
  }
  const float tsum = (vsum[0] + vsum[1]) + (vsum[2] + vsum[3]);
  const double mass = block_sum_d(static_cast<double>(tsum), sh.d);
  // bound accumulated in fp32: inflate for its own rounding
  const double bsum = static_cast<double>(block_sum_f(bound, sh.f)) * 1.001;
  if (threadIdx.x == 0) {
    SampleChunk r;
    r.mass = mass;
    // pairwise-sum rounding of the fp32 groups
    r.bound = bsum + (G::kSumLevels + 1) * kU24 * mass;
    p.smass[static_cast<int64_t>(i) * p.n_chunks + c] = r;
  }
}

// Last CTA of request i: find the token or queue the request for refinement.
template <bool BF16>
__device__ void locate_sample(const RunParams& p, int i, const Job& jb, SampleShared& sh) {
  using G = Geo<BF16>;
  const int tid = threadIdx.x;
  const SampleChunk* sc = p.smass + static_cast<int64_t>(i) * p.n_chunks;
  if (tid == 0) {
    double total = 0.0, tb = 0.0;
    for (int c = 0; c < p.n_chunks; ++c) {
      const double2 r = __ldcg(reinterpret_cast<const double2*>(sc + c));
      total += r.x;
      tb += r.y;
    }
    tb += 1e-15 * total;
    const double target = jb.u2 * total;
    double run = 0.0, runb = 0.0;
    int cstar = -1;
    for (int c = 0; c < p.n_chunks; ++c) {
      const double2 r = __ldcg(reinterpret_cast<const double2*>(sc + c));
      if (run + r.x > target) {
        cstar = c;
        break;
      }
      run += r.x;
      runb += r.y;
    }
    sh.cstar = cstar;
    sh.base = run;
    sh.base_bound = runb + 1e-15 * run;
    sh.total = total;
    sh.total_bound = tb;
    sh.found = -1;
    // residual mass must clear the 1e-12 floor with certainty
    if (jb.kind == kJobResidual && !(total - tb > 1e-12 * (1.0 + 1e-9))) sh.cstar = -1;
  }
  __syncthreads();
  const int cstar = sh.cstar;
  bool certain = false;
  int token = -1;
  if (cstar >= 0) {
    // Rescan chunk cstar with contiguous per-thread segments (index order).
    const WeightCtx w = weight_ctx(jb);
    const int64_t chunk0 = static_cast<int64_t>(cstar) * G::kChunk;
    const int64_t seg0 = chunk0 + static_cast<int64_t>(tid) * G::kPerThread;
    const void* ra = target_row(p, i, jb.row, BF16);
    const void* rb = w.residual ? draft_row(p, i, jb.row, BF16) : nullptr;
    float wt[G::kPerThread], bd[G::kPerThread];
    double tsum = 0.0, tbound = 0.0;
#pragma unroll 4
    for (int e = 0; e < G::kPerThread; ++e) {
      const int64_t t = seg0 + e;
      if (t < p.V) {
        const float a = load_logit(ra, t, BF16);
        const float b = w.residual ? load_logit(rb, t, BF16) : 0.0f;
        weight_and_bound(w, a, b, wt[e], bd[e]);
      } else {
        wt[e] = 0.0f;
        bd[e] = 0.0f;
      }
      tsum += static_cast<double>(wt[e]);
      tbound += static_cast<double>(bd[e]);
    }
    double all, allb;
    const double pre = block_exclusive_scan_d(tsum, sh.d, all);
    __syncthreads();
    const double preb = block_exclusive_scan_d(tbound, sh.d, allb);
    const double target = jb.u2 * sh.total;
    const double start = sh.base + pre;
    if (start <= target && start + tsum > target) {
      double run = start, runb = sh.base_bound + preb;
      for (int e = 0; e < G::kPerThread; ++e) {
        const double before = run;
        run += static_cast<double>(wt[e]);
        runb += static_cast<double>(bd[e]);
        if (run > target) {
          sh.found = static_cast<int>(seg0 - chunk0) + e;
          sh.lo_gap = target - before;
          sh.hi_gap = run - target;
          sh.cell_bound = runb;
          break;
        }
      }
    }
    __syncthreads();
    if (tid == 0 && sh.found >= 0) {
      const double slack = jb.u2 * sh.total_bound + 1e-14 * sh.total;
      const double need = sh.cell_bound + slack;
      certain = sh.lo_gap > need && sh.hi_gap > need;
      token = static_cast<int>(chunk0 + sh.found);
    }
  }
  if (tid == 0) {
    if (certain) {
      p.out_tok[static_cast<int64_t>(i) * (p.k + 1) + jb.n] = token;
      atomicAdd(&p.counters->sample_fast, 1u);
    } else {
      const unsigned slot = atomicAdd(&p.counters->refine_count, 1u);
      p.refine_list[slot] = i;
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_sample(RunParams p) {
  __shared__ SampleShared sh;
  const int64_t b = blockIdx.x;
  const int i = static_cast<int>(b / p.n_chunks);
  const int c = static_cast<int>(b % p.n_chunks);
  const Job jb = p.jobs[i];
  if (jb.kind == kJobNone) return;
  chunk_mass<BF16>(p, i, jb, c, sh);
  if (!arrive_last(p.arrive_sample + i, static_cast<unsigned>(p.n_chunks), &sh.flag)) return;
  __threadfence();
  locate_sample<BF16>(p, i, jb, sh);
}

}  // namespace sv
