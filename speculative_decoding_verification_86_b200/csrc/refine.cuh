// Pass 3 (only for samples the fp32 filter could not certify): the sample is
// recomputed in fp64 exactly as the rule defines it -- p_t = exp(l_t/T - m_p)
// / Z_p, q_t likewise, residual weight max(0, p_t - q_t) (or the target
// weight exp(l_t/T - m_p) for a bonus token, or when the residual mass is
// under the 1e-12 floor), inverse CDF in index order with the smallest-index
// rule and the largest-positive-index fallback.
//
// Two launches, each a grid-stride loop over (queued request, chunk):
//   k_refine_z    : fp64 normalisers of the row pair, merged in chunk order;
//   k_refine_pick : fp64 chunk masses, then the last CTA of the request
//                   prefixes them and scans the one chunk holding u * total.
// Both read the queue length written by the sampling pass and exit at once
// when nothing was queued.
#pragma once
#include "common.cuh"
#include "stats.cuh"

namespace sv {

struct RefineShared {
  double d[kWarps];
  int i[kWarps];
  int flag;
  int cstar;
  double base, total, target;
  int use_resid;
  int found;
};

__device__ __forceinline__ double exact_weight_p(const void* ra, int64_t t, bool bf16, double T,
                                                 double ma) {
  return exp(static_cast<double>(load_logit(ra, t, bf16)) / T - ma);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_refine_z(RunParams p) {
  __shared__ RefineShared sh;
  using G = Geo<BF16>;
  const unsigned count = __ldcg(&p.counters->refine_count);
  const int64_t work = static_cast<int64_t>(count) * p.n_chunks;
  for (int64_t wi = blockIdx.x; wi < work; wi += gridDim.x) {
    const int slot = static_cast<int>(wi / p.n_chunks);
    const int c = static_cast<int>(wi % p.n_chunks);
    const int i = __ldcg(p.refine_list + slot);
    const Job jb = p.jobs[i];
    const double T = jb.T;
    const double ma = static_cast<double>(jb.mraw_a) / T;
    const double mb = static_cast<double>(jb.mraw_b) / T;
    const void* ra = target_row(p, i, jb.row, BF16);
    const void* rb = jb.kind == kJobResidual ? draft_row(p, i, jb.row, BF16) : nullptr;
    const int64_t t0 = static_cast<int64_t>(c) * G::kChunk;
    const int64_t t1 = min(p.V, t0 + G::kChunk);
    double za = 0.0, zb = 0.0;
    for (int64_t t = t0 + threadIdx.x; t < t1; t += kThreads) {
      za += exact_weight_p(ra, t, BF16, T, ma);
      if (rb) zb += exact_weight_p(rb, t, BF16, T, mb);
    }
    za = block_sum_d(za, sh.d);
    __syncthreads();
    zb = block_sum_d(zb, sh.d);
    if (threadIdx.x == 0) p.rz[static_cast<int64_t>(slot) * p.n_chunks + c] = make_double2(za, zb);
    if (arrive_last(p.arrive_r1 + slot, static_cast<unsigned>(p.n_chunks), &sh.flag)) {
      __threadfence();
      if (threadIdx.x == 0) {
        double A = 0.0, Bz = 0.0;
        for (int cc = 0; cc < p.n_chunks; ++cc) {
          const double2 r = __ldcg(p.rz + static_cast<int64_t>(slot) * p.n_chunks + cc);
          A += r.x;
          Bz += r.y;
        }
        p.rZ[slot] = make_double2(A, Bz);
      }
    }
    __syncthreads();
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_refine_pick(RunParams p) {
  __shared__ RefineShared sh;
  using G = Geo<BF16>;
  const unsigned count = __ldcg(&p.counters->refine_count);
  const int64_t work = static_cast<int64_t>(count) * p.n_chunks;
  for (int64_t wi = blockIdx.x; wi < work; wi += gridDim.x) {
    const int slot = static_cast<int>(wi / p.n_chunks);
    const int c = static_cast<int>(wi % p.n_chunks);
    const int i = __ldcg(p.refine_list + slot);
    const Job jb = p.jobs[i];
    const bool residual = jb.kind == kJobResidual;
    const double T = jb.T;
    const double ma = static_cast<double>(jb.mraw_a) / T;
    const double mb = static_cast<double>(jb.mraw_b) / T;
    const double2 Z = __ldcg(p.rZ + slot);
    const void* ra = target_row(p, i, jb.row, BF16);
    const void* rb = residual ? draft_row(p, i, jb.row, BF16) : nullptr;
    const int64_t t0 = static_cast<int64_t>(c) * G::kChunk;
    const int64_t t1 = min(p.V, t0 + G::kChunk);
    double mr = 0.0, mp = 0.0;
    for (int64_t t = t0 + threadIdx.x; t < t1; t += kThreads) {
      const double pe = exact_weight_p(ra, t, BF16, T, ma);
      mp += pe;
      if (rb) {
        const double r = pe / Z.x - exact_weight_p(rb, t, BF16, T, mb) / Z.y;
        mr += r > 0.0 ? r : 0.0;
      }
    }
    mr = block_sum_d(mr, sh.d);
    __syncthreads();
    mp = block_sum_d(mp, sh.d);
    if (threadIdx.x == 0) p.rm[static_cast<int64_t>(slot) * p.n_chunks + c] = make_double2(mr, mp);
    if (!arrive_last(p.arrive_r2 + slot, static_cast<unsigned>(p.n_chunks), &sh.flag)) continue;
    __threadfence();

    // ---- last CTA of this request: locate the token in fp64 ----
    const double2* rm = p.rm + static_cast<int64_t>(slot) * p.n_chunks;
    if (threadIdx.x == 0) {
      double R = 0.0, P = 0.0;
      for (int cc = 0; cc < p.n_chunks; ++cc) {
        const double2 r = __ldcg(rm + cc);
        R += r.x;
        P += r.y;
      }
      const int use_resid = residual && R >= 1e-12;
      const double W = use_resid ? R : P;
      const double target = jb.u2 * W;
      double run = 0.0;
      int cstar = -1;
      for (int cc = 0; cc < p.n_chunks; ++cc) {
        const double2 r = __ldcg(rm + cc);
        const double m = use_resid ? r.x : r.y;
        if (run + m > target) {
          cstar = cc;
          break;
        }
        run += m;
      }
      sh.use_resid = use_resid;
      sh.cstar = cstar;
      sh.base = run;
      sh.target = target;
      sh.found = -1;
      if (cstar < 0) {
        // rounding left no cell above target: the last chunk with positive weight
        for (int cc = p.n_chunks - 1; cc >= 0; --cc) {
          const double2 r = __ldcg(rm + cc);
          if ((use_resid ? r.x : r.y) > 0.0) {
            sh.cstar = cc;
            break;
          }
        }
        sh.found = -2;  // marks the fallback
      }
    }
    __syncthreads();
    const int cstar = sh.cstar;
    const bool fallback = sh.found == -2;
    const bool use_resid = sh.use_resid != 0;
    int token = -1;
    if (cstar >= 0) {
      const int64_t chunk0 = static_cast<int64_t>(cstar) * G::kChunk;
      const int64_t seg0 = chunk0 + static_cast<int64_t>(threadIdx.x) * G::kPerThread;
      double wv[G::kPerThread];
      double tsum = 0.0;
      int last_pos = -1;
      for (int e = 0; e < G::kPerThread; ++e) {
        const int64_t t = seg0 + e;
        double wt = 0.0;
        if (t < p.V) {
          const double pe = exact_weight_p(ra, t, BF16, T, ma);
          if (use_resid) {
            const double r = pe / Z.x - exact_weight_p(rb, t, BF16, T, mb) / Z.y;
            wt = r > 0.0 ? r : 0.0;
          } else {
            wt = pe;
          }
        }
        wv[e] = wt;
        tsum += wt;
        if (wt > 0.0) last_pos = static_cast<int>(t - chunk0);
      }
      if (fallback) {
        // largest index with positive weight in this chunk
        int neg = last_pos >= 0 ? -last_pos : INT_MAX;
        neg = block_min_i(neg, sh.i);
        token = neg == INT_MAX ? -1 : static_cast<int>(chunk0 - neg);
      } else {
        double all;
        const double pre = block_exclusive_scan_d(tsum, sh.d, all);
        const double start = sh.base + pre;
        const double target = sh.target;
        if (start <= target && start + tsum > target) {
          double run = start;
          for (int e = 0; e < G::kPerThread; ++e) {
            run += wv[e];
            if (run > target) {
              sh.found = static_cast<int>(seg0 - chunk0) + e;
              break;
            }
          }
        }
        __syncthreads();
        token = sh.found >= 0 ? static_cast<int>(chunk0 + sh.found) : -1;
      }
    }
    if (threadIdx.x == 0) {
      p.out_tok[static_cast<int64_t>(i) * (p.k + 1) + jb.n] = token;
      if (token < 0) {
        p.out_acc[i] = -1;
        if (p.out_status) p.out_status[i] |= kDevInternal;
      }
    }
    __syncthreads();
  }
}

}  // namespace sv
