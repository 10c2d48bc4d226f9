// Confidence head ("Speculative decoding becomes standard: DSpark and
// multi-token drafters", section "What DSpark adds"): s_j = sigmoid(w . h_j + b)
// is the head's estimate that drafted position j passes verification when all
// positions before it have passed.  The chance
// that the first j positions all survive is the prefix product; the request's
// budget is the number of leading positions whose prefix product stays at or
// above the threshold.
//
// The same section ties how much is verified to the load of the batch.  With a
// batch-wide budget N > 0, the positions left by the per-request rule (and by
// verify_len) are candidates, and only the N with the largest prefix survival
// are verified -- ties to the lower request, then the lower position.  The
// prefix product never grows along a request, so the kept positions of each
// request are a leading run and its verified length is their count.
//
// One CTA per request, one warp per position: the bf16 x bf16 products are
// exact in fp32 and are summed in fp64, so every decision is made on an fp64
// prefix product.  With a batch budget the last CTA to finish selects: a
// radix select (8 passes of 8 bits over the fp64 bit patterns, which order
// like the non-negative values) finds the N-th largest survival t and how many
// of the candidates equal to t are kept; a scan over the requests in index
// order hands those ties out.
#pragma once
#include "common.cuh"

namespace sv {

// The batch-wide selection, run by the CTA that completes the last request's
// budget.  Reads the prefix products and per-request limits every CTA
// published, writes out_len.  Batches of up to `cache` candidate slots are
// first copied to shared memory (one pass of independent loads), so the eight
// radix passes and the final count run on shared memory; larger batches stream
// the candidates from L2 in every pass.
constexpr int kSelCache = 4096;        // candidate cache of the standalone k_conf
constexpr int kSelCacheEngine = 1024;  // ... of the verification engine (shared memory is the ring's)
constexpr unsigned long long kNoKey = ~0ull;  // not a candidate (valid keys are <= bits of 1.0)
static_assert(kThreads == 256, "one radix bin per thread");

struct ConfSelectShared {
  unsigned hist[256];
  double sh_d[kWarps];
  unsigned long long key;
  long long rank;
};

__device__ void conf_select(const ConfParams& cp, ConfSelectShared& ss, unsigned long long* s_keys,
                            int cache) {
  unsigned* hist = ss.hist;
  double* sh_d = ss.sh_d;
  unsigned long long& s_key = ss.key;
  long long& s_rank = ss.rank;
  const int B = cp.B, kb = cp.kb;
  const long long n = static_cast<long long>(B) * kb;
  const bool cached = n <= cache;
  auto load_key = [&](long long e) -> unsigned long long {
    const int i = static_cast<int>(e / kb), j = static_cast<int>(e - static_cast<long long>(i) * kb);
    if (j >= __ldcg(cp.cap + i)) return kNoKey;
    return static_cast<unsigned long long>(__double_as_longlong(__ldcg(cp.prefix + e)));
  };
  if (cached) {
    for (long long e = threadIdx.x; e < n; e += kThreads) s_keys[e] = load_key(e);
  }
  double m_local = 0.0;
  for (int i = threadIdx.x; i < B; i += kThreads) m_local += __ldcg(cp.cap + i);
  const long long M = static_cast<long long>(block_sum_d(m_local, sh_d));  // (also a barrier)
  if (cp.total >= M) {
    for (int i = threadIdx.x; i < B; i += kThreads) cp.out_len[i] = __ldcg(cp.cap + i);
    return;
  }
  auto key_at = [&](long long e) -> unsigned long long { return cached ? s_keys[e] : load_key(e); };

  // t = the total-th largest candidate key (rank 1 = the largest).
  if (threadIdx.x == 0) {
    s_key = 0ull;
    s_rank = cp.total;
  }
  for (int shift = 56; shift >= 0; shift -= 8) {
    hist[threadIdx.x] = 0u;  // kThreads == 256 bins
    sync_compute();
    const unsigned long long want = s_key;
    const long long rank = s_rank;
    const unsigned long long hi_mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
    for (long long e = threadIdx.x; e < n; e += kThreads) {
      const unsigned long long key = key_at(e);
      if (key != kNoKey && (key & hi_mask) == want) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    sync_compute();
    // thread t looks after digit 255 - t: the keys above it are the exclusive
    // prefix in that order; exactly one digit holds the rank
    const int digit = 255 - static_cast<int>(threadIdx.x);
    const unsigned c = hist[digit];
    double tot;
    const long long above =
        static_cast<long long>(block_exclusive_scan_d(static_cast<double>(c), sh_d, tot));
    sync_compute();  // every thread has read s_key and s_rank
    if (c > 0 && above < rank && above + static_cast<long long>(c) >= rank) {
      s_rank = rank - above;  // rank among the keys with this digit
      s_key = want | (static_cast<unsigned long long>(digit) << shift);
    }
    sync_compute();
  }
  const unsigned long long t = s_key;
  const long long take_eq = s_rank;  // how many candidates equal to t are kept
  double carry = 0.0;
  for (int base = 0; base < B; base += kThreads) {
    const int i = base + threadIdx.x;
    int gt = 0, eq = 0;
    if (i < B) {
      for (int j = 0; j < kb; ++j) {
        const unsigned long long key = key_at(static_cast<long long>(i) * kb + j);
        if (key == kNoKey) break;  // candidates are a leading run of the request
        gt += key > t;
        eq += key == t;
      }
    }
    double tot;
    const double before = carry + block_exclusive_scan_d(static_cast<double>(eq), sh_d, tot);
    if (i < B) {
      const long long left = take_eq - static_cast<long long>(before);
      const long long take = left <= 0 ? 0 : (left < eq ? left : eq);
      cp.out_len[i] = gt + static_cast<int>(take);
    }
    carry += tot;
    sync_compute();
  }
}

// Per-request part, one CTA (kThreads compute threads) per request: s_j for
// each position (one warp per position, fp64 dot), then the prefix product,
// the budget and, with a batch budget, the published prefix and limit.
__device__ void conf_request(const ConfParams& cp, int i, double* s_surv) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = warp; j < cp.kb; j += kWarps) {
    const uint16_t* h = cp.hidden + (static_cast<int64_t>(i) * cp.kb + j) * cp.H;
    double z = 0.0;
    for (int c = lane; c < cp.H; c += 32) {
      const float wf = __uint_as_float(static_cast<uint32_t>(__ldg(cp.w + c)) << 16);
      const float hf = __uint_as_float(static_cast<uint32_t>(__ldg(h + c)) << 16);
      z += static_cast<double>(wf * hf);
    }
    z = warp_sum_d(z);
    if (lane == 0) s_surv[j] = 1.0 / (1.0 + exp(-(z + static_cast<double>(cp.bias))));
  }
  sync_compute();
  if (threadIdx.x == 0) {
    double prefix = 1.0;
    int budget = 0;
    bool counting = true;
    for (int j = 0; j < cp.kb; ++j) {
      prefix *= s_surv[j];
      if (counting && prefix >= static_cast<double>(cp.threshold)) ++budget;
      else counting = false;
      if (cp.out_survival) cp.out_survival[static_cast<int64_t>(i) * cp.kb + j] = static_cast<float>(s_surv[j]);
      if (cp.total > 0) cp.prefix[static_cast<int64_t>(i) * cp.kb + j] = prefix;
    }
    if (cp.k >= 0) {
      int L = cp.vlen ? cp.vlen[i] : cp.k;
      L = L < 0 ? 0 : (L > cp.k ? cp.k : L);
      budget = budget < L ? budget : L;
    }
    if (cp.total > 0) cp.cap[i] = budget;
    else cp.out_len[i] = budget;
  }
  sync_compute();
}

__global__ void __launch_bounds__(kThreads) k_conf(ConfParams cp) {
  __shared__ double s_surv[kMaxK];
  __shared__ int s_last;
  __shared__ ConfSelectShared ss;
  __shared__ unsigned long long s_keys[kSelCache];
  conf_request(cp, blockIdx.x, s_surv);
  if (cp.total <= 0) return;
  if (!arrive_last(cp.arrive, static_cast<unsigned>(cp.B), &s_last)) return;
  conf_select(cp, ss, s_keys, kSelCache);
}

}  // namespace sv
