// The verification engine: one persistent kernel that drives every request of
// the batch through its passes with a device-side work queue.
//
// Work items (32-bit payloads):
//   STATS  (request, row slot, segment)  softmax / arg-max statistics of one row segment
//   SAMPLE (request, chunk)              residual / bonus masses of one chunk
//   REFINE (refinement slot, sub-chunk)  fp64 recomputation of one sub-chunk
// The CTA completing the last item of a task decides what follows and
// enqueues it: the chain decision after STATS (then the next position's rows,
// the sample, or nothing), the inverse-CDF locate after SAMPLE (then nothing
// or the fp64 refinement), the fp64 token after REFINE.  Requests advance
// independently.
//
// Two orders of the statistics ("Speculative decoding becomes standard: DSpark
// and multi-token drafters", section "Why draft-and-verify does not change the
// output": the block ends at its first rejected position):
//   dense  : every verified position's rows are statistics items from the start
//            and the chain is walked once they are all in;
//   prefix : a request's position j+1 rows are read only after position j was
//            accepted.  The outputs are identical; prefix reads fewer bytes.
//
// The first tickets (0 .. n_init-1) are implicit: the confidence head of every
// request when it runs in this launch, then the rows of position 0 (prefix)
// or of every position (dense), decoded from the ticket number.  Items the
// run generates go to one queue per class, served after the implicit tickets
// in the order: statistics of a later position, sample chunks, refinement
// sub-chunks.  (One FIFO for all of them kept chain items waiting behind sample
// items, and a request's chain of positions is the run's critical path.)  The
// slots carry the run's epoch in their upper 32 bits so a slot left by an
// earlier run is never taken for a new item.  A CTA waiting for work sleeps
// between polls and gives up after a bounded number of polls (setting the
// queue error), as does the whole kernel once every request is finished.
// The last CTA to leave resets the queue counters for the next run.
#pragma once
#include "common.cuh"
#include "conf.cuh"
#include "refine.cuh"
#include "sample.cuh"
#include "stats.cuh"

namespace sv {

constexpr uint32_t kItemStats = 0u, kItemSample = 1u, kItemRefine = 2u, kItemConf = 3u;
constexpr uint32_t kItemExit = 0xFFFFFFFFu;
constexpr int kRowSeg = 0xFF;  // segment field of a STATS item that covers its whole row
constexpr unsigned kSpinLimit = 1u << 24;  // polls of a queue slot before giving up (seconds)
constexpr int kEngineMinBlocks = 4;  // 64 registers: four CTAs per SM (measured best)
// Small, latency-bound batches run an instance with two CTAs per SM (128
// registers: no spills on the serial decision paths; measured faster there than
// three CTAs per SM at 80 registers, which in turn beat four at 64).
constexpr int kEngineMinBlocksSmall = 2;
// candidate keys of the batch-wide selection held in the staging buffer
constexpr int kConfKeysInStage = 4096;
static_assert(kMaxK * sizeof(double) + sizeof(ConfSelectShared) + kConfKeysInStage * sizeof(unsigned long long) <=
                  kStageBytes,
              "the confidence head's scratch fits the staging buffer");

__device__ __forceinline__ uint32_t item_stats(int i, int slot, int seg) {
  return (kItemStats << 30) | (static_cast<uint32_t>(i) << 14) |
         (static_cast<uint32_t>(slot) << 8) | static_cast<uint32_t>(seg);
}
__device__ __forceinline__ uint32_t item_sample(int i, int seg) {
  return (kItemSample << 30) | (static_cast<uint32_t>(i) << 14) | static_cast<uint32_t>(seg);
}
__device__ __forceinline__ uint32_t item_refine(int slot, int sub) {
  return (kItemRefine << 30) | (static_cast<uint32_t>(slot) << 14) | static_cast<uint32_t>(sub);
}
__device__ __forceinline__ uint32_t item_conf(int i) {
  return (kItemConf << 30) | (static_cast<uint32_t>(i) << 14);
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* a) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* a) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long* a, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(a), "l"(v) : "memory");
}

// Rows of position j that a task reads: 2 (target and draft) for a sampled
// position before L, else 1 (greedy position or the bonus row).
__device__ __forceinline__ int task_rows(const ReqInfo& ri, int j) {
  return (!ri.greedy && j < ri.L) ? 2 : 1;
}
// Rows of the prefix order's dense tail from position d <= L: target rows
// d..L and, for a sampled request, draft rows d..L-1.
__device__ __forceinline__ int tail_rows(const ReqInfo& ri, int d) {
  return ri.greedy ? ri.L - d + 1 : 2 * (ri.L - d) + 1;
}

// The implicit item of ticket h < n_init.
__device__ __forceinline__ uint32_t implicit_item(const RunParams& p, unsigned h) {
  if (h < p.n_conf) return item_conf(static_cast<int>(h));
  h -= p.n_conf;
  if (p.mode == kModeDense && p.whole_rows) {  // a request's 2k + 1 whole rows
    const unsigned per_req = static_cast<unsigned>(2 * p.k + 1);
    return item_stats(static_cast<int>(h / per_req), static_cast<int>(h % per_req), kRowSeg);
  }
  if (p.mode == kModeDense) {
    const unsigned per_req = static_cast<unsigned>(2 * p.k + 1) * p.n_segs;
    const unsigned i = h / per_req, r = h % per_req;
    return item_stats(static_cast<int>(i), static_cast<int>(r / p.n_segs), static_cast<int>(r % p.n_segs));
  }
  const unsigned per_req = 2u * p.n_segs;
  const unsigned i = h / per_req, r = h % per_req;
  const int slot = (r / p.n_segs) == 0 ? 0 : p.k + 1;  // target row 0, draft row 0
  return item_stats(static_cast<int>(i), slot, static_cast<int>(r % p.n_segs));
}

// Queue classes, in the order idle CTAs serve them once the implicit tickets
// are gone: a later position's statistics first (they extend the longest
// chains), then sample segments, then refinement sub-chunks.
constexpr int kClassStats = 0, kClassSample = 1, kClassRefine = 2;
static_assert(kClassRefine < kQClasses, "queue classes");
// Sample items cover this many chunks of the row pair (shorter items keep the
// sample step, which ends a request's chain, short), or a single part of a
// chunk when the batch is small enough for every part to get its own CTA.
constexpr int kSampleChunksPerItem = 1;
__host__ __device__ __forceinline__ int sample_items_of(int n_chunks, bool parts) {
  return parts ? n_chunks * kSampleParts : (n_chunks + kSampleChunksPerItem - 1) / kSampleChunksPerItem;
}
__device__ __forceinline__ int sample_items(const RunParams& p) {
  return sample_items_of(p.n_chunks, p.sample_parts != 0);
}

__device__ __forceinline__ int ld_volatile_s32(const unsigned* a) {
  int v;
  asm volatile("ld.volatile.global.s32 %0, [%1];" : "=r"(v) : "l"(a));
  return v;
}

// Thread 0: the item behind ticket d of class c, once its producer wrote the
// slot (it reserved the slot before publishing the count the claim came from,
// so the wait is short); kItemExit if the wait gives up.
__device__ uint32_t claim_slot(const RunParams& p, int c, unsigned d) {
  const unsigned long long* slot = p.q_slots + p.q_off[c] + d;
  for (unsigned spin = 0;; ++spin) {
    const unsigned long long v = ld_acquire_u64(slot);
    if (static_cast<unsigned>(v >> 32) == p.q_epoch) return static_cast<uint32_t>(v);
    if (spin >= kSpinLimit) {
      atomicOr(&p.counters->queue_error, 1u);
      return kItemExit;
    }
    __nanosleep(64);
  }
}

// Thread 0: the next item (or kItemExit).  Implicit tickets first (one atomic
// add each; `implicit_left` turns false at the first ticket past them), then
// the classes in order: a CTA claims an item of class c by taking one unit of
// its published count (giving it back if there was none) and then a ticket of
// the class, so it never holds a ticket whose item was not yet produced.
__device__ uint32_t fetch_item(const RunParams& p, bool& implicit_left) {
  if (implicit_left) {
    const unsigned h = atomicAdd(p.q_ctl + kQHead, 1u);
    if (h < p.n_init) return implicit_item(p, h);
    implicit_left = false;
  }
  for (unsigned spin = 0;; ++spin) {
#pragma unroll 1
    for (int c = 0; c < kQClasses; ++c) {
      unsigned* avail = p.q_ctl + kQAvail0 + c;
      if (ld_volatile_s32(avail) <= 0) continue;
      if (static_cast<int>(atomicSub(avail, 1u)) <= 0) {
        atomicAdd(avail, 1u);
        continue;
      }
      return claim_slot(p, c, atomicAdd(p.q_ctl + kQClaim0 + c, 1u));
    }
    if (ld_acquire_u32(p.q_ctl + kQDone) >= static_cast<unsigned>(p.B)) return kItemExit;
    if (spin >= kSpinLimit || ld_volatile_s32(&p.counters->queue_error) != 0) {
      atomicOr(&p.counters->queue_error, 1u);
      return kItemExit;
    }
    __nanosleep(spin < 32 ? 64 : 512);
  }
}

// Enqueue n items of class c whose payloads gen(q) (q < n) produces (all
// threads call): reserve slots, write them, then publish the count.
template <typename Gen>
__device__ __forceinline__ void enqueue(const RunParams& p, int c, int n, Gen gen, unsigned* s_base) {
  if (threadIdx.x == 0) *s_base = atomicAdd(p.q_ctl + kQTail0 + c, static_cast<unsigned>(n));
  __syncthreads();
  const unsigned base = *s_base;
  for (int q = threadIdx.x; q < n; q += kThreads) {
    const unsigned d = base + static_cast<unsigned>(q);
    if (d < p.q_cap[c]) {
      st_release_u64(p.q_slots + p.q_off[c] + d, (static_cast<unsigned long long>(p.q_epoch) << 32) | gen(q));
    } else {
      atomicOr(&p.counters->queue_error, 2u);
    }
  }
  // The count needs no ordering against the slots: a claim waits for its
  // slot's epoch tag anyway.
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned fits = base >= p.q_cap[c] ? 0u : min(static_cast<unsigned>(n), p.q_cap[c] - base);
    atomicAdd(p.q_ctl + kQAvail0 + c, fits);
  }
}

__device__ __forceinline__ void finish_request(const RunParams& p) {
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(p.q_ctl + kQDone, 1u);
  }
}

template <bool BF16>
__device__ void enqueue_sample(const RunParams& p, int i, unsigned* s_base) {
  enqueue(p, kClassSample, sample_items(p), [&](int q) { return item_sample(i, q); }, s_base);
}

// Wait (thread 0) until the confidence head run in this launch has published
// every budget; false if the wait gave up.
__device__ __forceinline__ bool wait_conf(const RunParams& p) {
  if (p.n_conf == 0) return true;
  for (unsigned w = 0;; ++w) {
    if (ld_acquire_u32(p.q_ctl + kQConfDone) == p.q_epoch) return true;
    if (w >= kSpinLimit) {
      atomicOr(&p.counters->queue_error, 4u);
      return false;
    }
    __nanosleep(w < 32 ? 64 : 256);
  }
}

// STATS item: one segment of one row of request i; the last segment of the
// task decides.
//
// When the confidence head runs in the same launch (prefix order), the rows of
// position 0 are read before its budgets are known: their plan follows
// verify_len alone (Lcap), reading the drafter's row 0 whenever a sampled
// request may verify a position, and the decision waits for the budgets.  A
// later position exists only after a decision, so its plan already has them.
template <bool BF16>
__device__ void engine_stats(const RunParams& p, int i, int slot, int seg, StatsShared& st,
                             DecideShared& dec, unsigned* s_base, uint4* stage_buf) {
  const bool is_draft = slot > p.k;
  const int j = is_draft ? slot - (p.k + 1) : slot;
  const bool early = p.n_conf > 0 && j == 0;  // planned before the head's budgets
  const ReqInfo ri = request_info(p, i, !early);
  bool needed, pass;
  unsigned expected;
  if (early) {
    // the plan cannot tell yet whether the head leaves a request without
    // drafter logits any position to verify: its target row is read
    const bool target_only = ri.greedy || ri.no_draft;
    if (ri.invalid_T) needed = (slot == 0 && seg == 0);
    else needed = !is_draft || (!target_only && ri.Lcap > 0);
    pass = !ri.invalid_T;
    expected = ri.invalid_T ? 1u
                            : static_cast<unsigned>(((!target_only && ri.Lcap > 0) ? 2 : 1) * p.n_segs);
  } else {
    if (ri.bad_T) needed = (slot == 0 && seg == 0);
    else if (ri.greedy) needed = !is_draft && j <= ri.L;
    else needed = is_draft ? (j < ri.L) : (j <= ri.L);
    pass = !ri.bad_T;
    if (ri.bad_T) expected = 1u;
    else if (p.mode == kModeDense) expected = static_cast<unsigned>(stats_expected(ri, p.n_segs));
    else if (j >= p.tail_from) expected = static_cast<unsigned>(tail_rows(ri, p.tail_from) * p.n_segs);
    else expected = static_cast<unsigned>(task_rows(ri, j) * p.n_segs);
  }
  // a whole-row item (dense order) stands for all of the row's segment items
  const bool whole = seg == kRowSeg;
  if (whole && ri.bad_T) needed = slot == 0;
  if (!needed) return;
  // a whole row arrives for its n_segs segments (a failed request's one item for one)
  const unsigned weight = (whole && pass) ? static_cast<unsigned>(p.n_segs) : 1u;
  // the drafted token, loaded now (its logit is cached once the segment is in)
  const bool cache_tok = pass && !ri.greedy && j < p.k;
  int xj = -1;
  if (cache_tok && threadIdx.x == 0) xj = __ldg(p.tokens + static_cast<int64_t>(i) * p.k + j);
  if (pass) {
    const int64_t rec0 = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_segs;
    const void* row = is_draft ? draft_row(p, i, j, BF16) : target_row(p, i, j, BF16);
    const float cc = ri.greedy ? 0.0f : static_cast<float>(1.4426950408889634 / static_cast<double>(ri.T));
    if (whole) {
      if (ri.greedy) stats_row_staged<BF16, true>(row, p.V, p.n_segs, cc, p.meta + rec0, nullptr, st, stage_buf);
      else stats_row_staged<BF16, false>(row, p.V, p.n_segs, cc, p.meta + rec0, p.ssum + rec0, st, stage_buf);
    } else if (p.short_segs) {
      if (ri.greedy) greedy_segment_staged<BF16, kShortSegBatches>(row, p.V, seg, p.meta + rec0 + seg, st, stage_buf);
      else stochastic_segment_staged<BF16, kShortSegBatches>(row, p.V, seg, cc, p.meta + rec0 + seg,
                                                             p.ssum + rec0 + seg, st, stage_buf);
    } else if (ri.greedy) {
      greedy_segment_staged<BF16>(row, p.V, seg, p.meta + rec0 + seg, st, stage_buf);
    } else {
      stochastic_segment_staged<BF16>(row, p.V, seg, cc, p.meta + rec0 + seg, p.ssum + rec0 + seg, st, stage_buf);
    }
    // The item holding the drafted token's logit leaves it for the decision
    // (published by the arrival below), which then reads a small array
    // instead of the row.
    if (cache_tok && threadIdx.x == 0) {
      const int64_t lo = whole ? 0 : static_cast<int64_t>(seg) * p.seg_len;
      const int64_t hi = whole ? p.V : min(p.V, lo + p.seg_len);
      if (xj >= lo && xj < hi)
        p.tok_cache[(static_cast<int64_t>(i) * p.k + j) * 2 + (is_draft ? 1 : 0)] = load_logit(row, xj, BF16);
    }
  }
  if (!arrive_last(p.arrive_stats + i, expected, &st.flag, weight)) return;
  if (early) {
    if (threadIdx.x == 0) st.flag = wait_conf(p) ? 1 : 0;
    __syncthreads();
    if (!st.flag) return;  // the head never finished: the run reports the queue error
  }
  if (p.mode == kModeDense || j >= p.tail_from) {
    decide_request<BF16>(p, i, ri, dec, p.mode == kModeDense ? 0 : p.tail_from);
    __syncthreads();
    if (dec.state == 2) enqueue_sample<BF16>(p, i, s_base);
    else finish_request(p);
    return;
  }
  const ReqInfo rc = early ? request_info(p, i, true) : ri;
  decide_position<BF16>(p, i, rc, j, dec);
  const int next = dec.state;
  if (next == 1) {
    const int jn = j + 1;
    const int ns = p.n_segs;
    if (jn >= p.tail_from) {
      // the rest of the request at once: target rows jn..L, then draft rows jn..L-1
      const int nt = rc.L - jn + 1;
      enqueue(p, kClassStats, tail_rows(rc, jn) * ns, [&](int q) {
        const int r = q / ns;
        return item_stats(i, r < nt ? jn + r : p.k + 1 + jn + (r - nt), q % ns);
      }, s_base);
    } else {
      const int rows = task_rows(rc, jn);
      enqueue(p, kClassStats, rows * ns, [&](int q) {
        return item_stats(i, (q / ns) == 0 ? jn : p.k + 1 + jn, q % ns);
      }, s_base);
    }
  } else if (next == 2) {
    enqueue_sample<BF16>(p, i, s_base);
  } else {
    finish_request(p);
  }
}

// CONF item: the confidence head of request i.  The CTA completing the last
// request runs the batch-wide selection (if any) and publishes the budgets.
// Its scratch is the staging buffer, idle between streaming passes.
__device__ void engine_conf(const RunParams& p, int i, int* flag, uint4* stage_buf) {
  double* s_surv = reinterpret_cast<double*>(stage_buf);
  ConfSelectShared* ss = reinterpret_cast<ConfSelectShared*>(s_surv + kMaxK);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(ss + 1);
  conf_request(p.cp, i, s_surv);
  if (!arrive_last(p.cp.arrive, static_cast<unsigned>(p.B), flag)) return;
  if (p.cp.total > 0) conf_select(p.cp, *ss, keys, kConfKeysInStage);
  sync_compute();
  if (threadIdx.x == 0) {
    __threadfence();
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.q_ctl + kQConfDone), "r"(p.q_epoch) : "memory");
  }
}

template <bool BF16>
__device__ void engine_sample(const RunParams& p, int i, int part, SampleShared& sa,
                              unsigned* s_base, uint4* stage_buf) {
  const Job jb = load_job(p.jobs + i);
  if (p.sample_parts) part_mass_item<BF16>(p, i, jb, part, sa);
  else chunk_masses_staged<BF16, kSampleChunksPerItem>(p, i, jb, part * kSampleChunksPerItem, stage_buf);
  if (!arrive_last(p.arrive_sample + i, static_cast<unsigned>(sample_items(p)), &sa.flag)) return;
  locate_sample<BF16>(p, i, jb, sa);
  const int slot = sa.refine_slot;
  if (slot < 0) {
    finish_request(p);
    return;
  }
  const int n_subs = p.n_chunks * kSubsPerChunk;
  enqueue(p, kClassRefine, n_subs, [&](int q) { return item_refine(slot, q); }, s_base);
}

template <bool BF16>
__device__ void engine_refine(const RunParams& p, int slot, int sub, RefineShared& rf) {
  refine_item<BF16>(p, slot, sub, rf);
  if (!arrive_last(p.arrive_r1 + slot, static_cast<unsigned>(p.n_chunks * kSubsPerChunk), &rf.flag)) return;
  refine_finalize<BF16>(p, slot, rf);
  finish_request(p);
}

template <bool BF16, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) k_engine(RunParams p) {
  extern __shared__ __align__(16) uint4 stage_buf[];  // kStageBytes, per-thread staging
  __shared__ StatsShared st;
  __shared__ DecideShared dec;
  __shared__ SampleShared sa;
  __shared__ RefineShared rf;
  __shared__ uint32_t s_item;
  __shared__ unsigned s_base;
  exp2_table_init(rf.tab);
  bool implicit_left = true;  // thread 0: implicit tickets may remain
#pragma unroll 1
  for (;;) {
    if (threadIdx.x == 0) s_item = fetch_item(p, implicit_left);
    __syncthreads();
    const uint32_t it = s_item;
    if (it == kItemExit) break;
    const int a = static_cast<int>((it >> 14) & 0xFFFFu);
    const int b = static_cast<int>(it & 0x3FFFu);
    switch (it >> 30) {
      case kItemStats: engine_stats<BF16>(p, a, b >> 8, b & 0xFF, st, dec, &s_base, stage_buf); break;
      case kItemSample: engine_sample<BF16>(p, a, b, sa, &s_base, stage_buf); break;
      case kItemRefine: engine_refine<BF16>(p, a, b, rf); break;
      default: engine_conf(p, a, &st.flag, stage_buf); break;
    }
    __syncthreads();
  }
  // The last CTA to leave resets the queue for the next run and clears the
  // next run's diagnostic counters.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.q_ctl + kQExits, 1u) == gridDim.x - 1) {
      p.q_ctl[kQHead] = 0u;
      p.q_ctl[kQDone] = 0u;
      p.q_ctl[kQExits] = 0u;
      for (int c = 0; c < kQClasses; ++c) {
        p.q_ctl[kQTail0 + c] = 0u;
        p.q_ctl[kQClaim0 + c] = 0u;
        p.q_ctl[kQAvail0 + c] = 0u;
      }
      *p.counters_next = Counters{};
      __threadfence();
    }
  }
}

}  // namespace sv
