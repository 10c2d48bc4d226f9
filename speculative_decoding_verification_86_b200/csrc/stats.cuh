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

namespace sv {

// ---------------------------------------------------------------------------
// Chunk statistics of one row.
// ---------------------------------------------------------------------------
template <bool BF16>
__device__ __forceinline__ void load_chunk(const void* row, int64_t V, int c,
                                           uint4 (&v)[kUnroll]) {
  using G = Geo<BF16>;
  const int64_t nvec = V / G::kPerVec;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t base = static_cast<int64_t>(c) * G::kChunkVecs + threadIdx.x;
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int64_t idx = base + u * kThreads;
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
}

template <bool BF16>
__device__ __forceinline__ float chunk_local_max(const uint4 (&v)[kUnroll]) {
  if constexpr (BF16) {
    uint32_t m2 = v[0].x;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      m2 = hmax2_nan(m2, v[u].x);
      m2 = hmax2_nan(m2, v[u].y);
      m2 = hmax2_nan(m2, v[u].z);
      m2 = hmax2_nan(m2, v[u].w);
    }
    return fmax_nan(bf16_lo(m2), bf16_hi(m2));
  } else {
    float m = __uint_as_float(v[0].x);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      m = fmax_nan(m, __uint_as_float(v[u].x));
      m = fmax_nan(m, __uint_as_float(v[u].y));
      m = fmax_nan(m, __uint_as_float(v[u].z));
      m = fmax_nan(m, __uint_as_float(v[u].w));
    }
    return m;
  }
}

struct StatsShared {
  float f[kWarps];
  double d[kWarps];
  int i[kWarps];
  int flag;
};

// Softmax statistics of chunk c of a stochastic row.
template <bool BF16>
__device__ __forceinline__ void stochastic_chunk(const void* row, int64_t V, int c, float cc,
                                                 ChunkMeta* meta_out, double* sum_out,
                                                 StatsShared& sh) {
  using G = Geo<BF16>;
  uint4 v[kUnroll];
  load_chunk<BF16>(row, V, c, v);
  const float m = block_max_nan(chunk_local_max<BF16>(v), sh.f);
  // NaN or +inf anywhere in the chunk, or nothing but -inf: no exponentials.
  if (!(m > -INFINITY) || isinf(m) || isnan(m)) {
    if (threadIdx.x == 0) {
      ChunkMeta r;
      r.K = (isnan(m) || m > 0.0f) ? (isnan(m) ? m : INFINITY) : -INFINITY;
      r.mraw = m;
      r.err = 0.0f;
      r.arg = 0;
      *meta_out = r;
      *sum_out = (isnan(m) || m > 0.0f) ? __longlong_as_double(0x7ff8000000000000LL) : 0.0;
    }
    return;
  }
  const float K = m * cc;
  float vsum[kUnroll];
  float err = 0.0f;
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    float x[G::kPerVec];
    unpack<BF16>(v[u], x);
    float e[G::kPerVec];
#pragma unroll
    for (int q = 0; q < G::kPerVec; ++q) {
      const float a = fmaxf(fmaf(x[q], cc, -K), -1024.0f);
      e[q] = ex2_approx(a);
      err = fmaf(e[q], fabsf(a), err);
    }
    if constexpr (BF16) {
      vsum[u] = ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
    } else {
      vsum[u] = (e[0] + e[1]) + (e[2] + e[3]);
    }
  }
  const float tsum = (vsum[0] + vsum[1]) + (vsum[2] + vsum[3]);
  const double s = block_sum_d(static_cast<double>(tsum), sh.d);
  const float errs = block_sum_f(err, sh.f);
  if (threadIdx.x == 0) {
    ChunkMeta r;
    r.K = K;
    r.mraw = m;
    r.err = errs;
    r.arg = 0;
    *meta_out = r;
    *sum_out = s;
  }
}

// Max and lowest arg-max of chunk c of a greedy row.
template <bool BF16>
__device__ __forceinline__ void greedy_chunk(const void* row, int64_t V, int c, ChunkMeta* meta_out,
                                             StatsShared& sh) {
  using G = Geo<BF16>;
  uint4 v[kUnroll];
  load_chunk<BF16>(row, V, c, v);
  const float m = block_max_nan(chunk_local_max<BF16>(v), sh.f);
  int first = INT_MAX;
  const int64_t chunk0 = static_cast<int64_t>(c) * G::kChunk;
#pragma unroll
  for (int u = kUnroll - 1; u >= 0; --u) {  // later vectors first, so the lowest index wins
    float x[G::kPerVec];
    unpack<BF16>(v[u], x);
#pragma unroll
    for (int q = G::kPerVec - 1; q >= 0; --q) {
      if (x[q] == m) first = (u * kThreads + threadIdx.x) * G::kPerVec + q;
    }
  }
  first = block_min_i(first, sh.i);
  if (threadIdx.x == 0) {
    ChunkMeta r;
    r.K = 0.0f;
    r.mraw = m;
    r.err = 0.0f;
    r.arg = first == INT_MAX ? -1 : static_cast<int>(chunk0 + first);
    *meta_out = r;
  }
}

// ---------------------------------------------------------------------------
// Merged row records, built by the deciding CTA in shared memory.
// ---------------------------------------------------------------------------
struct RowMerged {
  double Z;      // sum of 2^(l c - K) over the row (fp32 terms)
  double E;      // bound on sum e |a| in the row's frame
  float K;       // exponent reference (max over chunks)
  float mraw;    // raw max
  int arg;       // greedy: lowest arg-max
  int bad;       // NaN / +inf / all -inf
};

struct DecideShared {
  RowMerged rows[kMaxRows];
  double red[kWarps];
  // chain state (written by thread 0)
  int state;        // 0 continue, 1 stop
  int need_exact;   // position whose accept test needs the fp64 row sums, or -1
  double exact_Za, exact_Zb;
};

// Merge the chunk records of stochastic row `slot` with one warp.
__device__ __forceinline__ void merge_stochastic_row(const RunParams& p, int i, int slot,
                                                     RowMerged& out) {
  const int lane = threadIdx.x & 31;
  const int64_t base = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_chunks;
  float K = -INFINITY, mraw = -INFINITY;
  int bad = 0;
  for (int c = lane; c < p.n_chunks; c += 32) {
    const float4 m4 = __ldcg(reinterpret_cast<const float4*>(p.meta + base + c));
    const float Kc = m4.x;
    if (isnan(Kc) || Kc == INFINITY) bad = 1;
    K = fmaxf(K, Kc);
    mraw = fmax_nan(mraw, m4.y);
  }
  K = warp_max_nan(K);
  mraw = warp_max_nan(mraw);
  bad = __any_sync(0xffffffffu, bad);
  if (!(K > -INFINITY)) bad = 1;
  double Z = 0.0, E = 0.0;
  if (!bad) {
    for (int c = lane; c < p.n_chunks; c += 32) {
      const float4 m4 = __ldcg(reinterpret_cast<const float4*>(p.meta + base + c));
      if (m4.x == -INFINITY) continue;
      const double s = __ldcg(p.ssum + base + c);
      const double d = static_cast<double>(m4.x) - static_cast<double>(K);  // <= 0, exact
      const double f = exp2(d);
      Z += s * f;
      // |a| measured against K_c; against K it grows by at most (K - K_c) per unit mass.
      E += (static_cast<double>(m4.z) + (-d) * s) * f;
    }
  }
  Z = warp_sum_d(Z);
  E = warp_sum_d(E);
  if (!(Z > 0.0) || isinf(Z) || isnan(Z)) bad = 1;
  if (lane == 0) {
    out.Z = Z;
    out.E = E;
    out.K = K;
    out.mraw = mraw;
    out.arg = -1;
    out.bad = bad;
  }
}

__device__ __forceinline__ void merge_greedy_row(const RunParams& p, int i, int slot,
                                                 RowMerged& out) {
  const int lane = threadIdx.x & 31;
  const int64_t base = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_chunks;
  float best = -INFINITY;
  int arg = INT_MAX;
  int bad = 0;
  for (int c = lane; c < p.n_chunks; c += 32) {
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
    out.E = 0.0;
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

// Resolve request i after all its chunk statistics are in.
template <bool BF16>
__device__ void decide_request(const RunParams& p, int i, const ReqInfo& ri, DecideShared& sh) {
  const int tid = threadIdx.x, warp = tid >> 5;
  const int k = p.k, L = ri.L;
  int32_t* tok = p.out_tok + static_cast<int64_t>(i) * (k + 1);
  float* op = p.out_p ? p.out_p + static_cast<int64_t>(i) * k : nullptr;
  float* oq = p.out_q ? p.out_q + static_cast<int64_t>(i) * k : nullptr;
  const int32_t* x = p.tokens + static_cast<int64_t>(i) * k;
  Job* job = p.jobs + i;

  // Defaults: nothing accepted yet, every slot -1.
  for (int j = tid; j <= k; j += kThreads) tok[j] = -1;
  for (int j = tid; j < k; j += kThreads) {
    if (op) op[j] = -1.0f;
    if (oq) oq[j] = -1.0f;
  }

  if (ri.bad_T) {
    if (tid == 0) {
      p.out_acc[i] = -1;
      if (p.out_status) p.out_status[i] = kDevBadTemperature;
      job->kind = kJobNone;
    }
    return;
  }

  // Merge the rows the chain can read: target rows 0..L, draft rows 0..L-1.
  const int nrows = ri.greedy ? L + 1 : 2 * L + 1;
  for (int r = warp; r < nrows; r += kWarps) {
    const int slot = r <= L ? r : (k + 1) + (r - (L + 1));
    const int dst = r <= L ? r : (k + 1) + (r - (L + 1));
    if (ri.greedy) merge_greedy_row(p, i, slot, sh.rows[dst]);
    else merge_stochastic_row(p, i, slot, sh.rows[dst]);
  }
  __syncthreads();

  if (ri.greedy) {
    if (tid == 0) {
      uint32_t status = 0;
      int n = L;
      for (int j = 0; j < L; ++j) {
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
        for (int j = 0; j <= k; ++j) tok[j] = -1;
      }
      p.out_acc[i] = status ? -1 : n;
      if (p.out_status) p.out_status[i] = status;
      job->kind = kJobNone;
    }
    return;
  }

  // Stochastic chain.
  const double T = static_cast<double>(ri.T);
  const float cc = static_cast<float>(1.4426950408889634 / T);
  const double c_exact = 1.4426950408889634 / T;
  const double eta = fabs((c_exact - static_cast<double>(cc)) / static_cast<double>(cc));
  const double kappa = kLn2 * (kU24 + eta) * 1.0001;
  const double eps_base = static_cast<double>(p.eps_ex2) + (Geo<BF16>::kSumLevels + 1) * kU24 + 1e-14;

  // thread 0 carries the chain; other threads join the fp64 slow path.
  int n = L;
  uint32_t status = 0;
  int j = 0;
  for (; j < L; ++j) {
    if (tid == 0) {
      sh.state = 0;
      sh.need_exact = -1;
      const int xj = __ldg(x + j);
      const RowMerged& ra = sh.rows[j];
      const RowMerged& rb = sh.rows[k + 1 + j];
      if (xj < 0 || static_cast<int64_t>(xj) >= p.V) {
        status = kDevBadToken;
        sh.state = 1;
      } else if (ra.bad || rb.bad) {
        status = kDevNonfinite;
        sh.state = 1;
      } else {
        const float la = load_logit(target_row(p, i, j, BF16), xj, BF16);
        const float lb = load_logit(draft_row(p, i, j, BF16), xj, BF16);
        const double arg_a = static_cast<double>(la) * cc - static_cast<double>(ra.K);
        const double arg_b = static_cast<double>(lb) * cc - static_cast<double>(rb.K);
        const double pa = (la == -INFINITY) ? 0.0 : exp2(arg_a) / ra.Z;
        const double qb = (lb == -INFINITY) ? 0.0 : exp2(arg_b) / rb.Z;
        const double u = draw(p, i, j, 0);
        int decision;  // 1 accept, 0 reject, -1 inside the error bound
        if (qb == 0.0) {
          decision = pa > 0.0 ? 1 : 0;
        } else {
          const double dp = eps_base + kappa * ra.E / ra.Z + kLn2 * eta * fabs(arg_a);
          const double dq = eps_base + kappa * rb.E / rb.Z + kLn2 * eta * fabs(arg_b);
          const double delta = (dp + dq) * 1.01;
          const double rho = pa / qb;
          if (u < rho * (1.0 - delta)) decision = 1;
          else if (u >= rho * (1.0 + delta)) decision = 0;
          else decision = -1;
        }
        if (op) op[j] = static_cast<float>(pa);
        if (oq) oq[j] = static_cast<float>(qb);
        if (decision < 0) {
          sh.need_exact = j;
        } else if (decision == 1) {
          tok[j] = xj;
        } else {
          n = j;
          sh.state = 1;
        }
      }
    }
    __syncthreads();
    if (sh.need_exact >= 0) {
      // fp64 at the true temperature: recompute both normalisers exactly.
      const RowMerged& ra = sh.rows[j];
      const RowMerged& rb = sh.rows[k + 1 + j];
      const double ma = static_cast<double>(ra.mraw) / T;
      const double mb = static_cast<double>(rb.mraw) / T;
      const double Za = exact_row_sum(target_row(p, i, j, BF16), p.V, BF16, T, ma, sh.red);
      const double Zb = exact_row_sum(draft_row(p, i, j, BF16), p.V, BF16, T, mb, sh.red);
      if (tid == 0) {
        const int xj = __ldg(x + j);
        const double la = load_logit(target_row(p, i, j, BF16), xj, BF16);
        const double lb = load_logit(draft_row(p, i, j, BF16), xj, BF16);
        const double pa = exp(la / T - ma) / Za;
        const double qb = exp(lb / T - mb) / Zb;
        const double u = draw(p, i, j, 0);
        if (op) op[j] = static_cast<float>(pa);
        if (oq) oq[j] = static_cast<float>(qb);
        atomicAdd(&p.counters->accept_slow, 1u);
        if (u * qb < pa) {
          tok[j] = xj;
        } else {
          n = j;
          sh.state = 1;
        }
        sh.need_exact = -1;
      }
      __syncthreads();
    }
    const int stop = sh.state;
    __syncthreads();
    if (stop) break;
  }

  if (tid == 0) {
    if (!status && n == L && sh.rows[L].bad) status = kDevNonfinite;
    if (status) {
      for (int jj = 0; jj <= k; ++jj) tok[jj] = -1;
      if (op) for (int jj = 0; jj < k; ++jj) op[jj] = -1.0f;
      if (oq) for (int jj = 0; jj < k; ++jj) oq[jj] = -1.0f;
      p.out_acc[i] = -1;
      if (p.out_status) p.out_status[i] = status;
      job->kind = kJobNone;
      return;
    }
    p.out_acc[i] = n;
    if (p.out_status) p.out_status[i] = 0;
    Job jb;
    jb.n = n;
    jb.pad0 = 0;
    jb.cc = cc;
    jb.kappa = static_cast<float>(kappa);
    jb.T = T;
    jb.u2 = draw(p, i, n, 1);
    const RowMerged& ra = sh.rows[n];
    jb.row = n;
    jb.Ka = ra.K;
    jb.mraw_a = ra.mraw;
    if (n < L) {
      const RowMerged& rb = sh.rows[k + 1 + n];
      jb.kind = kJobResidual;
      jb.Kb = rb.K;
      jb.mraw_b = rb.mraw;
      jb.A = static_cast<float>(1.0 / ra.Z);
      jb.Bq = static_cast<float>(1.0 / rb.Z);
      // per-term constant: ex2 error, rounding of 1/Z and of the products,
      // the normaliser's own bound (incl. the temperature-rounding term).
      jb.eps0a = eps_base + 3 * kU24 + kappa * ra.E / ra.Z;
      jb.eps0b = eps_base + 3 * kU24 + kappa * rb.E / rb.Z;
    } else {
      jb.kind = kJobBonus;
      jb.Kb = 0.0f;
      jb.mraw_b = 0.0f;
      jb.A = 1.0f;
      jb.Bq = 0.0f;
      jb.eps0a = static_cast<double>(p.eps_ex2) + 2 * kU24 + 1e-14;
      jb.eps0b = 0.0;
    }
    *job = jb;
  }
}

// ---------------------------------------------------------------------------
// The kernel: one CTA per (request, row slot, chunk).
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_stats(RunParams p) {
  __shared__ StatsShared sh;
  __shared__ DecideShared dsh;
  const int rows_per_req = 2 * p.k + 1;
  const int64_t b = blockIdx.x;
  const int c = static_cast<int>(b % p.n_chunks);
  const int64_t slot_global = b / p.n_chunks;
  const int i = static_cast<int>(slot_global / rows_per_req);
  const int slot = static_cast<int>(slot_global - static_cast<int64_t>(i) * rows_per_req);
  if (b == 0 && threadIdx.x == 0) *p.counters_next = Counters{0u, 0u, 0u, 0u};

  const ReqInfo ri = request_info(p, i);
  const bool is_draft = slot > p.k;
  const int j = is_draft ? slot - (p.k + 1) : slot;
  bool needed;
  if (ri.bad_T) needed = (slot == 0 && c == 0);
  else if (ri.greedy) needed = !is_draft && j <= ri.L;
  else needed = is_draft ? (j < ri.L) : (j <= ri.L);
  if (!needed) return;

  if (!ri.bad_T) {
    const int64_t rec = slot_global * p.n_chunks + c;
    const void* row = is_draft ? draft_row(p, i, j, BF16) : target_row(p, i, j, BF16);
    if (ri.greedy) {
      greedy_chunk<BF16>(row, p.V, c, p.meta + rec, sh);
    } else {
      const float cc = static_cast<float>(1.4426950408889634 / static_cast<double>(ri.T));
      stochastic_chunk<BF16>(row, p.V, c, cc, p.meta + rec, p.ssum + rec, sh);
    }
  }
  if (!arrive_last(p.arrive_stats + i, static_cast<unsigned>(stats_expected(ri, p.n_chunks)),
                   &sh.flag))
    return;
  decide_request<BF16>(p, i, ri, dsh);
}

}  // namespace sv
