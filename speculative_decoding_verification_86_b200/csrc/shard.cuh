// Vocabulary-parallel verification: the target's and the drafter's logits are
// split by vocabulary over n ranks (a tensor-parallel LM head), rank r holding
// tokens [v_lo(r), v_hi(r)) of every row.  The rule is the same as the whole-
// vocabulary one ("Speculative decoding becomes standard: DSpark and
// multi-token drafters", section "Why draft-and-verify does not change the
// output"); only the data movement differs:
//
//   1. stats   every rank reduces its own segments of every verified row and
//              reads the drafted tokens' logits it holds -> exchange block 1;
//   2. decide  blocks 1 of all ranks (all-gathered) give every row's segment
//              records in global order, so every rank walks every chain and
//              gets the same decisions; each rank then computes the residual /
//              bonus masses of its own chunks -> exchange block 2;
//   3. locate  blocks 2 (all-gathered) give every chunk mass; the rank holding
//              the chunk the draw falls in rescans it and certifies the token;
//              the others answer "not here" -> an element-wise max over ranks.
//
// Shards are whole statistics segments, so the merged records are exactly the
// whole-vocabulary run's: every decision, probability and token is identical.
// A sample the fp32 filter cannot certify goes to the fp64 refinement, also
// split by vocabulary (4. refine: every rank's fp64 partial sums over its own
// sub-chunks -> exchange block 3; the rank holding the drawn sub-chunk scans
// it).  The rare cases that need rows of other ranks -- an accept draw inside
// its certified bound, a refinement whose support is not settled -- flag the
// request, which is redone whole after its rows are gathered.
#pragma once
#include "common.cuh"
#include "refine.cuh"
#include "sample.cuh"
#include "stats.cuh"

namespace sv {

constexpr int kMaxShards = 16;

// One (request, row slot, segment) record of exchange block 1.  32 bytes and
// 16-byte aligned, so the meta part can be moved as one 16-byte vector.
struct alignas(16) ShardRec {
  ChunkMeta meta;
  double sum;
  double pad;
};
static_assert(sizeof(ShardRec) == 32 && alignof(ShardRec) == 16, "exchange record layout");

struct ShardBounds {
  int n;                       // ranks
  int seg_lo[kMaxShards + 1];  // rank r holds segments [seg_lo[r], seg_lo[r+1])
  int nls_max;                 // the widest rank's segment count (block stride)
};

// Phase 1: one CTA per (request, row slot, local segment); rows not needed by
// the dense chain are skipped (their records are never read).
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_shard_stats(RunParams p, int s_lo, int nls,
                                                          ShardRec* out) {
  __shared__ StatsShared sh;
  const int rows = 2 * p.k + 1;
  const int64_t b = blockIdx.x;
  const int ls = static_cast<int>(b % nls);
  const int64_t rs = b / nls;
  const int i = static_cast<int>(rs / rows);
  const int slot = static_cast<int>(rs - static_cast<int64_t>(i) * rows);
  const ReqInfo ri = request_info(p, i);
  const bool is_draft = slot > p.k;
  const int j = is_draft ? slot - (p.k + 1) : slot;
  bool needed;
  if (ri.bad_T) needed = false;
  else if (ri.greedy) needed = !is_draft && j <= ri.L;
  else needed = is_draft ? (j < ri.L) : (j <= ri.L);
  if (!needed) return;
  ShardRec* r = out + rs * nls + ls;
  const void* row = is_draft ? draft_row(p, i, j, BF16) : target_row(p, i, j, BF16);
  const int seg = s_lo + ls;
  if (ri.greedy) {
    greedy_segment<BF16>(row, p.V, seg, &r->meta, sh);
  } else {
    const float cc = static_cast<float>(1.4426950408889634 / static_cast<double>(ri.T));
    stochastic_segment<BF16>(row, p.V, seg, cc, &r->meta, &r->sum, sh);
  }
}

// Phase 1: the drafted tokens' logits this rank holds ([B, k, 2]: target,
// draft); entries of tokens held elsewhere are written as 0 and never read.
template <bool BF16>
__global__ void k_shard_token_logits(RunParams p, float* out) {
  const int64_t n = static_cast<int64_t>(p.B) * p.k;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / p.k), j = static_cast<int>(e % p.k);
    const int64_t x = __ldg(p.tokens + e);
    float a = 0.0f, d = 0.0f;
    if (x >= p.v_lo && x < p.v_lo + p.row_stride) {
      a = load_logit(target_row(p, i, j, BF16), x, BF16);
      if (p.draft) d = load_logit(draft_row(p, i, j, BF16), x, BF16);
    }
    out[2 * e] = a;
    out[2 * e + 1] = d;
  }
}

// Phase 2: scatter every rank's block 1 into the whole-row record layout and
// pick each drafted token's logits from the rank holding the token.
__global__ void k_shard_gather_stats(RunParams p, ShardBounds sb, const char* blocks,
                                     size_t block_bytes, size_t tok_off, int64_t seg_len) {
  const int rows = 2 * p.k + 1;
  const int64_t nrec = static_cast<int64_t>(p.B) * rows * p.n_segs;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < nrec;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int seg = static_cast<int>(e % p.n_segs);
    const int64_t rs = e / p.n_segs;
    int r = 0;
    while (r + 1 < sb.n && seg >= sb.seg_lo[r + 1]) ++r;
    const int nls = sb.seg_lo[r + 1] - sb.seg_lo[r];
    const ShardRec* src = reinterpret_cast<const ShardRec*>(blocks + r * block_bytes) +
                          (rs * nls + (seg - sb.seg_lo[r]));
    const float4 m = __ldcg(reinterpret_cast<const float4*>(&src->meta));
    reinterpret_cast<float4*>(p.meta)[e] = m;
    p.ssum[e] = __ldcg(&src->sum);
  }
  const int64_t ntok = static_cast<int64_t>(p.B) * p.k;
  float* tl = const_cast<float*>(p.tok_logits);
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < ntok;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t x = __ldg(p.tokens + e);
    if (x < 0 || x >= p.V) {  // the chain reports the bad token; any value will do
      tl[2 * e] = 0.0f;
      tl[2 * e + 1] = 0.0f;
      continue;
    }
    const int seg = static_cast<int>(x / seg_len);
    int r = 0;
    while (r + 1 < sb.n && seg >= sb.seg_lo[r + 1]) ++r;
    const float* src = reinterpret_cast<const float*>(blocks + r * block_bytes + tok_off);
    tl[2 * e] = __ldcg(src + 2 * e);
    tl[2 * e + 1] = __ldcg(src + 2 * e + 1);
  }
}

// Phase 2: every chain, replicated on every rank (dense order).
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_shard_decide(RunParams p) {
  __shared__ DecideShared dsh;
  const int i = blockIdx.x;
  if (threadIdx.x == 0) p.fallback[i] = 0;
  sync_compute();
  decide_request<BF16>(p, i, request_info(p, i), dsh);
}

// Phase 2: residual / bonus masses of this rank's segments (two chunks each),
// one CTA per (request, local segment), written to the workspace.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_shard_masses(RunParams p, int s_lo, int nls) {
  __shared__ SampleShared sa;
  const int i = static_cast<int>(blockIdx.x / nls);
  const int ls = static_cast<int>(blockIdx.x % nls);
  const Job jb = load_job(p.jobs + i);
  if (jb.kind == kJobNone || __ldcg(p.fallback + i)) return;
  segment_masses<BF16>(p, i, jb, s_lo + ls, sa);
}

// Phase 2 / 3: this rank's part masses to exchange block 2
// ([B, nlc_max * kSampleParts]), and back from every rank's block into the
// whole-row layout.
__global__ void k_shard_pack_masses(RunParams p, int c_lo, int nlc, int nlc_max, SampleChunk* out) {
  const int64_t per_req = static_cast<int64_t>(nlc_max) * kSampleParts;
  const int64_t n = static_cast<int64_t>(p.B) * per_req;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / per_req);
    const int64_t lp = e % per_req;  // local part
    SampleChunk r{0.0, 0.0};
    if (lp < static_cast<int64_t>(nlc) * kSampleParts)
      r = p.smass[(static_cast<int64_t>(i) * p.n_chunks + c_lo) * kSampleParts + lp];
    out[e] = r;
  }
}

__global__ void k_shard_unpack_masses(RunParams p, ShardBounds sb, const SampleChunk* blocks,
                                      int nlc_max) {
  const int64_t per_row = static_cast<int64_t>(p.n_chunks) * kSampleParts;
  const int64_t n = static_cast<int64_t>(p.B) * per_row;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / per_row);
    const int64_t part = e % per_row;
    const int c = static_cast<int>(part / kSampleParts);
    const int seg = c / kChunksPerSeg;
    int r = 0;
    while (r + 1 < sb.n && seg >= sb.seg_lo[r + 1]) ++r;
    const int64_t lp = part - static_cast<int64_t>(sb.seg_lo[r]) * kChunksPerSeg * kSampleParts;
    const SampleChunk* src = blocks + (static_cast<int64_t>(r) * p.B + i) * nlc_max * kSampleParts + lp;
    p.smass[e] = SampleChunk{__ldcg(&src->mass), __ldcg(&src->bound)};
  }
}

// Phase 3: locate where the draw falls; the rank holding that chunk rescans it.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_shard_locate(RunParams p) {
  __shared__ SampleShared sa;
  const int i = blockIdx.x;
  const Job jb = load_job(p.jobs + i);
  if (jb.kind == kJobNone || __ldcg(p.fallback + i)) {
    if (threadIdx.x == 0) p.shard_tok[i] = -2;
    return;
  }
  locate_sample<BF16>(p, i, jb, sa);
}

// Request states after each phase (p.fallback): 0 done or in progress, 1 redo
// whole, 2 the sample needs the fp64 refinement.
constexpr int32_t kShardRedo = 1, kShardRefine = 2;

// Phase 3: the token agreed by the ranks (element-wise max of their answers:
// the token, -1 = not certified, -2 = not here).
__global__ void k_shard_finish(RunParams p, const int32_t* tok_max) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.B; i += gridDim.x * blockDim.x) {
    if (p.fallback[i]) continue;
    const int kind = __ldcg(&p.jobs[i].kind);
    if (kind == kJobNone) continue;
    const int32_t t = tok_max[i];
    if (t >= 0) {
      p.out_tok[static_cast<int64_t>(i) * (p.k + 1) + __ldcg(&p.jobs[i].n)] = t;
    } else {
      p.fallback[i] = kShardRefine;
      p.refine_list[i] = i;  // refinement slot = request index
    }
  }
}

// Phase 4: fp64 partial sums of this rank's sub-chunks for the requests whose
// sample needs the refinement (refinement slot = request index).
struct alignas(16) RefRec {
  double2 z;  // alpha, beta sums
  double2 m;  // support masses A, B
  int unc;    // logits of unsettled support
  int pad[3];
};
static_assert(sizeof(RefRec) == 48, "exchange record layout");

// Grid-stride over the B x nsub (request, sub-chunk) items: most requests need
// no refinement, so a small grid skips their items instead of launching a CTA
// for each.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_shard_refine_partials(RunParams p, int sub_lo, int nsub) {
  __shared__ RefineShared rf;
  bool table = false;
  const int64_t n = static_cast<int64_t>(p.B) * nsub;
  for (int64_t b = blockIdx.x; b < n; b += gridDim.x) {
    const int i = static_cast<int>(b / nsub);
    const int ls = static_cast<int>(b % nsub);
    if (__ldcg(p.fallback + i) != kShardRefine) continue;  // (uniform over the CTA)
    if (!table) {
      exp2_table_init(rf.tab);
      table = true;
    }
    refine_item<BF16>(p, i, sub_lo + ls, rf);
    sync_compute();  // rf is reused by the next item
  }
}

__global__ void k_shard_pack_refine(RunParams p, int sub_lo, int nsub, int nsub_max, RefRec* out) {
  const int n_subs = p.n_chunks * kSubsPerChunk;
  const int64_t n = static_cast<int64_t>(p.B) * nsub_max;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / nsub_max), ls = static_cast<int>(e % nsub_max);
    RefRec r{};
    if (ls < nsub && p.fallback[i] == kShardRefine) {
      const int64_t g = static_cast<int64_t>(i) * n_subs + sub_lo + ls;
      r.z = p.rz[g];
      r.m = p.rm[g];
      r.unc = p.runc[g];
    }
    out[e] = r;
  }
}

__global__ void k_shard_unpack_refine(RunParams p, ShardBounds sb, const RefRec* blocks, int nsub_max) {
  const int n_subs = p.n_chunks * kSubsPerChunk;
  const int64_t n = static_cast<int64_t>(p.B) * n_subs;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / n_subs), ss = static_cast<int>(e % n_subs);
    if (p.fallback[i] != kShardRefine) continue;
    const int seg = ss / (kSubsPerChunk * kChunksPerSeg);
    int r = 0;
    while (r + 1 < sb.n && seg >= sb.seg_lo[r + 1]) ++r;
    const int ls = ss - sb.seg_lo[r] * kChunksPerSeg * kSubsPerChunk;
    const RefRec* src = blocks + (static_cast<int64_t>(r) * p.B + i) * nsub_max + ls;
    p.rz[e] = make_double2(__ldcg(&src->z.x), __ldcg(&src->z.y));
    p.rm[e] = make_double2(__ldcg(&src->m.x), __ldcg(&src->m.y));
    p.runc[e] = __ldcg(&src->unc);
  }
}

// Phase 4: exact token of each refined request; the rank holding the drawn
// sub-chunk scans it (votes as in phase 3, -1 = redo the request whole).
template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_shard_refine_locate(RunParams p) {
  __shared__ RefineShared rf;
  const int i = blockIdx.x;
  if (__ldcg(p.fallback + i) != kShardRefine) {  // (uniform over the CTA)
    if (threadIdx.x == 0) p.shard_tok[i] = -2;
    return;
  }
  exp2_table_init(rf.tab);
  refine_finalize<BF16>(p, i, rf);
}

__global__ void k_shard_refine_finish(RunParams p, const int32_t* tok_max) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.B; i += gridDim.x * blockDim.x) {
    if (p.fallback[i] != kShardRefine) continue;
    const int32_t t = tok_max[i];
    if (t >= 0) {
      p.out_tok[static_cast<int64_t>(i) * (p.k + 1) + __ldcg(&p.jobs[i].n)] = t;
      p.fallback[i] = 0;
    } else {
      p.fallback[i] = kShardRedo;
    }
  }
}

}  // namespace sv
