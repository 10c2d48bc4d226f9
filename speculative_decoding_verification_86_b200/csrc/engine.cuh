// The verification engine: one persistent kernel that drives every request of
// the batch through its passes with a device-side work queue.
//
// Work items (32-bit payloads, ticketed by one atomic counter):
//   STATS  (request, row slot, segment)  softmax / arg-max statistics of one row segment
//   SAMPLE (request, segment)            residual / bonus masses of one segment
//   REFINE (refinement slot, sub-chunk)  fp64 recomputation of one sub-chunk
// The CTA completing the last item of a task decides what follows and
// enqueues it: the chain decision after STATS (then the next position's rows,
// the sample, or nothing), the inverse-CDF locate after SAMPLE (then nothing
// or the fp64 refinement), the fp64 token after REFINE.  Requests advance
// independently; new items join the one FIFO behind those already queued.
//
// Two orders of the statistics ("Speculative decoding becomes standard: DSpark
// and multi-token drafters", section "Why draft-and-verify does not change the
// output": the block ends at its first rejected position):
//   dense  : every verified position's rows are statistics items from the start
//            and the chain is walked once they are all in;
//   prefix : a request's position j+1 rows are read only after position j was
//            accepted.  The outputs are identical; prefix reads fewer bytes.
//
// The first tickets (0 .. n_init-1) are implicit: the rows of position 0 (prefix)
// or of every position (dense), decoded from the ticket number.  Later tickets
// index the queue, whose slots carry the run's epoch in their upper 32 bits so
// a slot left by an earlier run is never taken for a new item.  A CTA waiting
// for a slot sleeps between polls and gives up after a bounded time (setting
// the queue error), as does the whole kernel once every request is finished.
// The last CTA to leave resets the queue counters for the next run.
#pragma once
#include "common.cuh"
#include "refine.cuh"
#include "sample.cuh"
#include "stats.cuh"

namespace sv {

constexpr uint32_t kItemStats = 0u, kItemSample = 1u, kItemRefine = 2u;
constexpr uint32_t kItemExit = 0xFFFFFFFFu;
constexpr unsigned kSpinLimit = 1u << 24;  // polls of a queue slot before giving up (seconds)
constexpr int kEngineMinBlocks = 4;  // 64 registers: four CTAs per SM (measured best)

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

// The implicit item of ticket h < n_init.
__device__ __forceinline__ uint32_t implicit_item(const RunParams& p, unsigned h) {
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

// Thread 0: the next item (or kItemExit).
__device__ uint32_t fetch_item(const RunParams& p) {
  const unsigned h = atomicAdd(p.q_ctl + kQHead, 1u);
  if (h < p.n_init) return implicit_item(p, h);
  const unsigned d = h - p.n_init;
  for (unsigned spin = 0;; ++spin) {
    if (d < p.q_capacity) {
      const unsigned long long v = ld_acquire_u64(p.q_slots + d);
      if (static_cast<unsigned>(v >> 32) == p.q_epoch) return static_cast<uint32_t>(v);
    }
    if (ld_acquire_u32(p.q_ctl + kQDone) >= static_cast<unsigned>(p.B)) return kItemExit;
    if (spin >= kSpinLimit) {
      atomicOr(&p.counters->queue_error, 1u);
      return kItemExit;
    }
    __nanosleep(spin < 32 ? 64 : 512);
  }
}

// Enqueue n items whose payloads gen(q) (q < n) produces (all threads call).
template <typename Gen>
__device__ __forceinline__ void enqueue(const RunParams& p, int n, Gen gen, unsigned* s_base) {
  if (threadIdx.x == 0) *s_base = atomicAdd(p.q_ctl + kQTail, static_cast<unsigned>(n));
  __syncthreads();
  const unsigned base = *s_base;
  for (int q = threadIdx.x; q < n; q += kThreads) {
    const unsigned d = base + static_cast<unsigned>(q);
    if (d < p.q_capacity) {
      st_release_u64(p.q_slots + d, (static_cast<unsigned long long>(p.q_epoch) << 32) | gen(q));
    } else {
      atomicOr(&p.counters->queue_error, 2u);
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void finish_request(const RunParams& p) {
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(p.q_ctl + kQDone, 1u);
  }
}

template <bool BF16>
__device__ void enqueue_sample(const RunParams& p, int i, unsigned* s_base) {
  enqueue(p, p.n_segs, [&](int q) { return item_sample(i, q); }, s_base);
}

// STATS item: one segment of one row of request i; the last segment of the
// task decides.
template <bool BF16>
__device__ void engine_stats(const RunParams& p, int i, int slot, int seg, StatsShared& st,
                             DecideShared& dec, unsigned* s_base, uint4* stage_buf) {
  const ReqInfo ri = request_info(p, i);
  const bool is_draft = slot > p.k;
  const int j = is_draft ? slot - (p.k + 1) : slot;
  bool needed;
  if (ri.bad_T) needed = (slot == 0 && seg == 0);
  else if (ri.greedy) needed = !is_draft && j <= ri.L;
  else needed = is_draft ? (j < ri.L) : (j <= ri.L);
  if (!needed) return;
  if (!ri.bad_T) {
    const int64_t rec = (static_cast<int64_t>(i) * (2 * p.k + 1) + slot) * p.n_segs + seg;
    const void* row = is_draft ? draft_row(p, i, j, BF16) : target_row(p, i, j, BF16);
    if (ri.greedy) {
      greedy_segment_staged<BF16>(row, p.V, seg, p.meta + rec, st, stage_buf);
    } else {
      const float cc = static_cast<float>(1.4426950408889634 / static_cast<double>(ri.T));
      stochastic_segment_staged<BF16>(row, p.V, seg, cc, p.meta + rec, p.ssum + rec, st, stage_buf);
    }
  }
  unsigned expected;
  if (ri.bad_T) expected = 1u;
  else if (p.mode == kModeDense) expected = static_cast<unsigned>(stats_expected(ri, p.n_segs));
  else expected = static_cast<unsigned>(task_rows(ri, j) * p.n_segs);
  if (!arrive_last(p.arrive_stats + i, expected, &st.flag)) return;
  __threadfence();
  if (p.mode == kModeDense) {
    decide_request<BF16>(p, i, ri, dec);
    __syncthreads();
    if (__ldcg(&p.jobs[i].kind) != kJobNone) enqueue_sample<BF16>(p, i, s_base);
    else finish_request(p);
    return;
  }
  decide_position<BF16>(p, i, ri, j, dec);
  const int next = dec.state;
  if (next == 1) {
    const int jn = j + 1;
    const int rows = task_rows(ri, jn);
    const int ns = p.n_segs;
    enqueue(p, rows * ns, [&](int q) {
      return item_stats(i, (q / ns) == 0 ? jn : p.k + 1 + jn, q % ns);
    }, s_base);
  } else if (next == 2) {
    enqueue_sample<BF16>(p, i, s_base);
  } else {
    finish_request(p);
  }
}

template <bool BF16>
__device__ void engine_sample(const RunParams& p, int i, int seg, SampleShared& sa,
                              unsigned* s_base, uint4* stage_buf) {
  const Job jb = load_job(p.jobs + i);
  segment_masses_staged<BF16>(p, i, jb, seg, sa, stage_buf);
  if (!arrive_last(p.arrive_sample + i, static_cast<unsigned>(p.n_segs), &sa.flag)) return;
  __threadfence();
  locate_sample<BF16>(p, i, jb, sa);
  const int slot = sa.refine_slot;
  if (slot < 0) {
    finish_request(p);
    return;
  }
  const int n_subs = p.n_chunks * kSubsPerChunk;
  enqueue(p, n_subs, [&](int q) { return item_refine(slot, q); }, s_base);
}

template <bool BF16>
__device__ void engine_refine(const RunParams& p, int slot, int sub, RefineShared& rf) {
  refine_item<BF16>(p, slot, sub, rf);
  if (!arrive_last(p.arrive_r1 + slot, static_cast<unsigned>(p.n_chunks * kSubsPerChunk), &rf.flag)) return;
  __threadfence();
  refine_finalize<BF16>(p, slot, rf);
  finish_request(p);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads, kEngineMinBlocks) k_engine(RunParams p) {
  extern __shared__ __align__(16) uint4 stage_buf[];  // kStageBytes, per-thread staging
  __shared__ StatsShared st;
  __shared__ DecideShared dec;
  __shared__ SampleShared sa;
  __shared__ RefineShared rf;
  __shared__ uint32_t s_item;
  __shared__ unsigned s_base;
  exp2_table_init(rf.tab);
#pragma unroll 1
  for (;;) {
    if (threadIdx.x == 0) s_item = fetch_item(p);
    __syncthreads();
    const uint32_t it = s_item;
    if (it == kItemExit) break;
    const int a = static_cast<int>((it >> 14) & 0xFFFFu);
    const int b = static_cast<int>(it & 0x3FFFu);
    switch (it >> 30) {
      case kItemStats: engine_stats<BF16>(p, a, b >> 8, b & 0xFF, st, dec, &s_base, stage_buf); break;
      case kItemSample: engine_sample<BF16>(p, a, b, sa, &s_base, stage_buf); break;
      default: engine_refine<BF16>(p, a, b, rf); break;
    }
    __syncthreads();
  }
  // The last CTA to leave resets the queue for the next run and clears the
  // next run's diagnostic counters.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.q_ctl + kQExits, 1u) == gridDim.x - 1) {
      p.q_ctl[kQHead] = 0u;
      p.q_ctl[kQTail] = 0u;
      p.q_ctl[kQDone] = 0u;
      p.q_ctl[kQExits] = 0u;
      *p.counters_next = Counters{};
      __threadfence();
    }
  }
}

}  // namespace sv
