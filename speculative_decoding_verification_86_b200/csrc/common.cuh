// Shared definitions of the verification kernels: launch geometry, workspace
// records, run parameters and small device helpers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace sv {

// ---------------------------------------------------------------- geometry --
// A "chunk" is the unit of the sampling passes: kThreads threads x
// kBatchesPerChunk batches x kVecsPerBatch 16-byte vectors, i.e. 16384 bf16
// or 8192 fp32 logits of one row.  Chunk masses are what the inverse CDF
// prefixes before it rescans one chunk.
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kVecsPerBatch = 2;
constexpr int kBatchesPerChunk = 4;
constexpr int kMaxK = 16;
constexpr int kMaxRows = 2 * kMaxK + 1;  // k+1 target rows + k draft rows

template <bool BF16>
struct Geo {
  static constexpr int kPerVec = BF16 ? 8 : 4;                                  // logits per vector
  static constexpr int kChunkVecs = kThreads * kVecsPerBatch * kBatchesPerChunk; // 2048 vectors
  static constexpr int kChunk = kChunkVecs * kPerVec;                            // logits per chunk
  static constexpr int kBatchElems = kVecsPerBatch * kPerVec;                    // per thread and batch
  static constexpr int kPerThread = kBatchElems * kBatchesPerChunk;              // per thread and chunk
  static constexpr int kSumLevels = BF16 ? 4 : 3;                                // pairwise depth of a batch sum
  static constexpr int kPartVecs = kChunkVecs / kWarps;                          // 256 vectors: one warp's part
  static constexpr int kPart = kPartVecs * kPerVec;                              // logits per part
};
// The sampling passes split a chunk into kWarps contiguous parts, warp w of
// the CTA streaming part w, and keep one mass record per part, so the inverse
// CDF rescans a single part (one vector per thread) in the end.
constexpr int kSampleParts = kWarps;

constexpr int kChunkBf16 = Geo<true>::kChunk;   // 16384
constexpr int kChunkF32 = Geo<false>::kChunk;   // 8192
constexpr int kMaxChunksPerRow = 1024;  // block-wide prefixes cover 4 records per thread

// ------------------------------------------------------------ status bits --
constexpr uint32_t kDevBadToken = 1u;
constexpr uint32_t kDevNonfinite = 2u;
constexpr uint32_t kDevBadTemperature = 4u;
constexpr uint32_t kDevInternal = 16u;

// ------------------------------------------------------- workspace records --
// Statistics of one segment of one row.
//   stochastic row: K = integer exponent reference (NaN if the segment holds
//                   NaN or +inf, -inf if it holds only masked logits),
//                   mraw = NaN-propagating max of the raw logits,
//                   err = sum_t e_t |a_t| (a_t the rounded exponent in the frame
//                   it was computed in: bounds the exponent rounding),
//                   arg = bits of sum_t e_t (K - K_t) (frame offsets, fp32);
//                   the sum of e_t = 2^(l_t c - K) is stored separately in fp64.
//   greedy row:     mraw = NaN-propagating max (NaN if any logit is NaN),
//                   arg = lowest index attaining it.
struct ChunkMeta {
  float K;
  float mraw;
  float err;
  int arg;
};

// What is left to do for a request after its accept chain has been resolved.
constexpr int kJobNone = 0;
constexpr int kJobResidual = 1;  // sample norm(max(0, p - q)) of row pair `row`
constexpr int kJobBonus = 2;     // sample p of target row `row`

struct Job {
  int kind;
  int row;
  int n;        // accepted count = index of the token to write
  int pad0;
  float cc;     // fp32 log2(e) / T used by the fp32 path
  float Ka;     // exponent reference of the target row
  float Kb;     // exponent reference of the draft row
  float A;      // fp32 1 / Za   (1 for bonus jobs)
  float Bq;     // fp32 1 / Zb
  float kappa;  // ln2 * (2^-24 + |eta|): relative error per unit |argument| in a frame
  float mraw_a; // raw max of the target row (fp64 refinement)
  float mraw_b; // raw max of the draft row
  double eps0a; // argument-independent relative error bound of p terms
  double eps0b; // ... of q terms
  double u2;    // the sample's uniform draw
  double T;     // temperature
  double eta_ln2; // ln2 * |relative error of fp32 log2(e)/T|
  double rho_lo;  // refinement: Z_a / Z_b (max-relative frames) lies in [rho_lo, rho_hi]
  double rho_hi;
};

static_assert(sizeof(Job) % 8 == 0 && alignof(Job) == 8, "Job is read as 64-bit words");

// A job is written by the CTA that decides and read by others after they
// acquired the queue slot that announced it.  Jobs of neighbouring requests
// share cache lines, so a plain (L1-cached) load could return a line this SM
// cached earlier for a neighbour; read from L2 instead.
__device__ __forceinline__ Job load_job(const Job* src) {
  Job j;
  const unsigned long long* s = reinterpret_cast<const unsigned long long*>(src);
  unsigned long long* d = reinterpret_cast<unsigned long long*>(&j);
#pragma unroll
  for (int q = 0; q < static_cast<int>(sizeof(Job) / 8); ++q) d[q] = __ldcg(s + q);
  return j;
}

struct SampleChunk {
  double mass;   // sum of fp32 weights over a part of a chunk (fp64 accumulation of pairwise groups)
  double bound;  // certified bound on |mass - exact mass|
};

struct Counters {
  unsigned refine_count;   // samples queued for fp64 refinement
  unsigned accept_slow;    // accept decisions resolved in fp64
  unsigned sample_fast;    // samples certified by the fp32 filter
  unsigned chunks_redone;  // refinement chunks recomputed outright (support unsettled)
  unsigned queue_error;    // engine: bits of the waits that gave up (see engine.cuh), 2 the queue overflowed
  unsigned wait_fail;      // engine: the first wait that gave up: site << 28 | CTA << 16 | stage (low 16 bits)
  unsigned pad[2];
};

// Engine: orders of the statistics pass, and the queue's control words.
constexpr int kModeDense = 0;
constexpr int kModePrefix = 1;
// head: implicit tickets handed out; done: requests finished; exits: CTAs that
// left; conf_done: the epoch of the run whose confidence budgets are
// published.  Generated items sit in one queue per class (statistics of a
// later position, sample segments, refinement sub-chunks), each with its own
// reserved (tail), claimed (claim) and published-but-unclaimed (avail, signed)
// counts.
constexpr int kQClasses = 3;
constexpr int kQHead = 0, kQDone = 1, kQExits = 2, kQConfDone = 3, kQTail0 = 4,
              kQClaim0 = kQTail0 + kQClasses, kQAvail0 = kQClaim0 + kQClasses, kQWords = 16;
static_assert(kQAvail0 + kQClasses <= kQWords, "queue control words");

// -------------------------------------------------------------- run params --
struct ConfParams {
  const uint16_t* hidden;  // [B, kb, H] bf16 bits
  const uint16_t* w;       // [H]
  float bias;
  float threshold;
  int B;
  int kb;
  int H;
  int k;                   // verify_len cap applies when >= 0 (clamp to [0, k])
  const int32_t* vlen;     // [B] or nullptr (=> k)
  long long total;         // batch-wide verify budget; <= 0: none
  double* prefix;          // [B, kb] workspace: prefix survival (total > 0)
  int32_t* cap;            // [B] workspace: per-request limit before the batch budget
  unsigned* arrive;        // arrival counter (self-resetting)
  int32_t* out_len;        // [B]
  float* out_survival;     // [B, kb] or nullptr
};

struct RunParams {
  const void* target;      // [B, k+1, V]
  const void* draft;       // [B, k, V] or nullptr
  const int32_t* tokens;   // [B, k]
  const int32_t* vlen;     // [B] or nullptr
  const float* temp;       // [B] or nullptr
  const int32_t* conf_len; // [B] confidence budget or nullptr
  const double* uniforms;  // [B, k+1, 2] test override or nullptr
  int B;
  int k;
  int64_t V;               // vocabulary size (token indices are global)
  int64_t row_stride;      // logits per row in the buffers: V, or a shard's width
  int64_t v_lo;            // first token the buffers hold (0, or a shard's start)
  int n_chunks;            // 8192 / 4096-logit chunks (sampling and refinement passes)
  int n_segs;              // 32768 / 16384-logit segments (statistics pass)
  uint64_t seed;
  uint32_t step;
  uint32_t req_off;
  int force_greedy;        // every request at T = 0 (spec_verify_greedy)
  int launch_rows;         // k_stats: row slots per request in its grid (0: all 2k + 1)
  float eps_ex2;           // certified relative error of ex2.approx.ftz.f32

  int32_t* out_acc;
  int32_t* out_tok;
  float* out_p;
  float* out_q;
  uint32_t* out_status;

  ChunkMeta* meta;         // [B, 2k+1, n_chunks]
  double* ssum;            // [B, 2k+1, n_chunks]
  unsigned* arrive_stats;  // [B]
  unsigned* arrive_sample; // [B]
  Job* jobs;               // [B]
  SampleChunk* smass;      // [B, n_chunks, kSampleParts] part masses
  int* refine_list;        // [B]
  unsigned* arrive_r1;     // [B]
  double2* rz;             // [B, 4 n_chunks] fp64 normaliser partials per sub-chunk
  double2* rm;             // [B, 4 n_chunks] fp64 support masses (target, draft)
  int* runc;               // [B, 4 n_chunks] sub-chunks holding unsettled logits
  double4* rmp;            // [B, 4 n_chunks, kWarps] per-part (alpha, A, B) sums, or nullptr
  Counters* counters;      // this run's counters
  Counters* counters_next; // the other run's counters, reset here

  // vocabulary-parallel runs (nullptr / 0 otherwise)
  const float* tok_logits; // [B, k, 2]: target and draft logit of each drafted token
  float* tok_cache;        // engine: the same, left by the statistics items (else nullptr)
  int32_t* fallback;       // [B]: set when a decision needs rows held by other ranks
  int32_t* shard_tok;      // [B]: located token, -1 to redo the request whole, -2 not here
  int c_lo, c_hi;          // chunks whose logits the buffers hold (c_hi = 0: all)
  int rows_whole;          // the protocol runs as one shard over complete rows in memory

  // engine
  int mode;                        // kModeDense / kModePrefix
  int whole_rows;                  // dense order: a statistics item is a whole row (else a segment)
  int tail_from;                   // prefix order: positions >= this (>= 1) are read together, once
                                   // the position before it accepted (k + 1: one at a time)
  int sample_parts;                // a sample item is one part of a chunk (small batches), else a chunk
  int short_segs;                  // statistics segments of one batch step (small dense batches)
  int seg_len;                     // logits per statistics segment
  unsigned long long* q_slots;     // queue: (epoch << 32) | payload
  unsigned q_capacity;
  unsigned q_off[kQClasses];       // each class's region of q_slots
  unsigned q_cap[kQClasses];
  unsigned q_epoch;                // this run's epoch, never 0
  unsigned* q_ctl;                 // the queue's control words (kQ*)
  unsigned n_init;                 // implicit initial tickets
  unsigned n_conf;                 // of which the confidence head's (one per request, or 0)
  ConfParams cp;                   // the confidence head run inside the engine (n_conf > 0)
};


// ------------------------------------------------------------ device utils --
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Barrier over the kThreads threads of a CTA (named barrier 1, so that code
// shared by several kernels never depends on which barrier the caller uses).
__device__ __forceinline__ void sync_compute() {
  asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}
// The same barrier, returning whether any compute thread passed x != 0.
__device__ __forceinline__ int sync_compute_or(int x) {
  int r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\tsetp.ne.s32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, %2, pi;\n\tselp.s32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(x), "n"(kThreads)
      : "memory");
  return r;
}

// Packed fp32 pairs (sm_100): two independent round-to-nearest operations per
// instruction, each rounded exactly as its scalar counterpart.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(a)),
        "l"(reinterpret_cast<const unsigned long long&>(b)),
        "l"(reinterpret_cast<const unsigned long long&>(c)));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(a)),
        "l"(reinterpret_cast<const unsigned long long&>(b)));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(a)),
        "l"(reinterpret_cast<const unsigned long long&>(b)));
  return d;
}

__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ uint32_t hmax2_nan(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float load_logit(const void* row, int64_t t, bool bf16) {
  if (bf16) {
    const uint16_t b = __ldg(reinterpret_cast<const unsigned short*>(row) + t);
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
  return __ldg(reinterpret_cast<const float*>(row) + t);
}

// Unpack the logits of one 16-byte vector (8 bf16 or 4 fp32) into floats.
template <bool BF16>
__device__ __forceinline__ void unpack(const uint4& v, float (&x)[Geo<BF16>::kPerVec]) {
  if constexpr (BF16) {
    x[0] = bf16_lo(v.x); x[1] = bf16_hi(v.x);
    x[2] = bf16_lo(v.y); x[3] = bf16_hi(v.y);
    x[4] = bf16_lo(v.z); x[5] = bf16_hi(v.z);
    x[6] = bf16_lo(v.w); x[7] = bf16_hi(v.w);
  } else {
    x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z); x[3] = __uint_as_float(v.w);
  }
}

// NaN-propagating maximum of kUnroll vectors.
template <bool BF16>
__device__ __forceinline__ float vec_max(const uint4 (&v)[kVecsPerBatch]) {
  if constexpr (BF16) {
    uint32_t m2 = hmax2_nan(v[0].x, v[0].y);
    m2 = hmax2_nan(m2, v[0].z);
    m2 = hmax2_nan(m2, v[0].w);
#pragma unroll
    for (int u = 1; u < kVecsPerBatch; ++u) {
      m2 = hmax2_nan(m2, v[u].x);
      m2 = hmax2_nan(m2, v[u].y);
      m2 = hmax2_nan(m2, v[u].z);
      m2 = hmax2_nan(m2, v[u].w);
    }
    return fmax_nan(bf16_lo(m2), bf16_hi(m2));
  } else {
    float m = fmax_nan(__uint_as_float(v[0].x), __uint_as_float(v[0].y));
    m = fmax_nan(m, __uint_as_float(v[0].z));
    m = fmax_nan(m, __uint_as_float(v[0].w));
#pragma unroll
    for (int u = 1; u < kVecsPerBatch; ++u) {
      m = fmax_nan(m, __uint_as_float(v[u].x));
      m = fmax_nan(m, __uint_as_float(v[u].y));
      m = fmax_nan(m, __uint_as_float(v[u].z));
      m = fmax_nan(m, __uint_as_float(v[u].w));
    }
    return m;
  }
}

template <bool BF16>
__device__ __forceinline__ uint4 neg_inf_vec() {
  const uint32_t w = BF16 ? 0xFF80FF80u : 0xFF800000u;
  return make_uint4(w, w, w, w);
}

// Batch b of chunk c of a row, coalesced layout: thread t holds vectors
// t + (b * kVecsPerBatch + u) * kThreads of the chunk, so each load
// instruction of a warp covers 512 contiguous bytes.  Vectors past the row end
// read as -inf (weight 0).
template <bool BF16>
__device__ __forceinline__ void load_batch_coalesced(const void* row, int64_t V, int c, int b,
                                                     uint4 (&v)[kVecsPerBatch]) {
  using G = Geo<BF16>;
  const int64_t nvec = V / G::kPerVec;
  const uint4* rv = static_cast<const uint4*>(row);
  const int64_t base = static_cast<int64_t>(c) * G::kChunkVecs + threadIdx.x;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = base + static_cast<int64_t>(b * kVecsPerBatch + u) * kThreads;
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
}

// Batch b of chunk c, part layout: warp w streams part w (vectors
// w * kPartVecs .. of the chunk), lane l holding vectors
// l + (b * kVecsPerBatch + u) * 32 of it, so each load instruction of a warp
// covers 512 contiguous bytes and a warp's sums cover one contiguous range.
// Vectors past the row end read as -inf (weight 0).
template <bool BF16>
__device__ __forceinline__ int64_t part_vec_index(int c, int b, int u) {
  using G = Geo<BF16>;
  return static_cast<int64_t>(c) * G::kChunkVecs + (threadIdx.x >> 5) * G::kPartVecs + (threadIdx.x & 31) +
         (b * kVecsPerBatch + u) * 32;
}
template <bool BF16>
__device__ __forceinline__ void load_batch_parts(const void* row, int64_t V, int c, int b,
                                                 uint4 (&v)[kVecsPerBatch]) {
  using G = Geo<BF16>;
  const int64_t nvec = V / G::kPerVec;
  const uint4* rv = static_cast<const uint4*>(row);
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = part_vec_index<BF16>(c, b, u);
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
}

// Batch b of chunk c, contiguous layout: thread t holds the kPerThread logits
// starting at chunk offset t * kPerThread, batch b being its b-th run of
// kBatchElems -- index order, for scans.  Returns the chunk offset of the batch.
template <bool BF16>
__device__ __forceinline__ int load_batch_contiguous(const void* row, int64_t V, int c, int b,
                                                     uint4 (&v)[kVecsPerBatch]) {
  using G = Geo<BF16>;
  const int64_t nvec = V / G::kPerVec;
  const uint4* rv = static_cast<const uint4*>(row);
  const int off = threadIdx.x * G::kPerThread + b * G::kBatchElems;
  const int64_t base = (static_cast<int64_t>(c) * G::kChunk + off) / G::kPerVec;
#pragma unroll
  for (int u = 0; u < kVecsPerBatch; ++u) {
    const int64_t idx = base + u;
    v[u] = idx < nvec ? ld_stream(rv + idx) : neg_inf_vec<BF16>();
  }
  return off;
}

__device__ __forceinline__ bool temperature_valid(float T) {
  return (T >= 0.0f) && !isinf(T) && !(T > 0.0f && T < 0x1p-100f);
}

// Row pointers, indexed by global token index: element t of the returned row
// is token t.  A vocabulary shard holds tokens [v_lo, v_lo + row_stride), and
// only those are ever read through its rows.
__device__ __forceinline__ const void* row_at(const void* base, int64_t row, const RunParams& p,
                                              bool bf16) {
  const int64_t es = bf16 ? 2 : 4;
  const uintptr_t a = reinterpret_cast<uintptr_t>(base) +
                      static_cast<uintptr_t>((row * p.row_stride - p.v_lo) * es);
  return reinterpret_cast<const void*>(a);
}
__device__ __forceinline__ const void* target_row(const RunParams& p, int i, int j, bool bf16) {
  return row_at(p.target, static_cast<int64_t>(i) * (p.k + 1) + j, p, bf16);
}
__device__ __forceinline__ const void* draft_row(const RunParams& p, int i, int j, bool bf16) {
  return row_at(p.draft, static_cast<int64_t>(i) * p.k + j, p, bf16);
}

struct ReqInfo {
  int L;          // verified positions
  int Lcap;       // verify_len clamped to [0, k]: L before the confidence head's budget
  float T;        // temperature
  bool greedy;
  bool bad_T;     // the request fails: invalid temperature, or sampled positions without drafter logits
  bool invalid_T; // the temperature alone is invalid
  bool no_draft;  // sampled request and no drafter logits in the call
};

// with_conf: apply the confidence head's budget (conf_len, once published);
// without it L = Lcap, which is what the plan of reads is built on.
__device__ __forceinline__ ReqInfo request_info(const RunParams& p, int i, bool with_conf = true) {
  ReqInfo r;
  int L = p.vlen ? __ldg(p.vlen + i) : p.k;
  L = max(0, min(L, p.k));
  r.Lcap = L;
  if (p.conf_len && with_conf) L = min(L, __ldcg(p.conf_len + i));
  r.L = L;
  r.T = p.force_greedy ? 0.0f : (p.temp ? __ldg(p.temp + i) : 1.0f);
  r.invalid_T = !temperature_valid(r.T);
  r.greedy = !r.invalid_T && r.T == 0.0f;
  r.no_draft = !r.invalid_T && !r.greedy && p.draft == nullptr;
  // a sampled request that verifies any position needs the drafter's logits
  r.bad_T = r.invalid_T || (r.no_draft && r.L > 0);
  return r;
}

// Number of (row, segment) CTAs the statistics pass runs for request i.
__device__ __forceinline__ int stats_expected(const ReqInfo& r, int n_segs) {
  if (r.bad_T) return 1;
  if (r.greedy) return (r.L + 1) * n_segs;
  return (2 * r.L + 1) * n_segs;
}

// ------------------------------------------------------- block reductions --
// All reductions combine in a fixed order, so results never depend on timing.
__device__ __forceinline__ float warp_max_nan(float x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x = fmax_nan(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ int warp_min_i(int x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

// Block-wide reductions over kThreads threads; `sh` holds kWarps scratch slots.
// Every thread receives the result.  Caller must not reuse `sh` before a barrier.
__device__ __forceinline__ float block_max_nan(float x, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  x = warp_max_nan(x);
  sync_compute();
  if (lane == 0) sh[warp] = x;
  sync_compute();
  float y = lane < kWarps ? sh[lane] : -INFINITY;
  return warp_max_nan(y);
}

__device__ __forceinline__ double block_sum_d(double x, double* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  x = warp_sum_d(x);
  sync_compute();
  if (lane == 0) sh[warp] = x;
  sync_compute();
  double y = lane < kWarps ? sh[lane] : 0.0;
  return warp_sum_d(y);
}

__device__ __forceinline__ float block_sum_f(float x, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  x = warp_sum_f(x);
  sync_compute();
  if (lane == 0) sh[warp] = x;
  sync_compute();
  float y = lane < kWarps ? sh[lane] : 0.0f;
  return warp_sum_f(y);
}

__device__ __forceinline__ int block_min_i(int x, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  x = warp_min_i(x);
  sync_compute();
  if (lane == 0) sh[warp] = x;
  sync_compute();
  int y = lane < kWarps ? sh[lane] : INT_MAX;
  return warp_min_i(y);
}

// Inclusive scan of one double per thread across the block, in thread order.
// Returns the exclusive prefix; `total` receives the block sum.
__device__ __forceinline__ double block_exclusive_scan_d(double x, double* sh, double& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  sync_compute();
  if (lane == 31) sh[warp] = incl;
  sync_compute();
  double warp_base = 0.0, all = 0.0;
  for (int w = 0; w < kWarps; ++w) {
    const double s = sh[w];
    if (w < warp) warp_base += s;
    all += s;
  }
  total = all;
  return warp_base + incl - x;
}

// Block-wide exclusive prefix of per-chunk values v[c], c < n (n <= 4 *
// kThreads): thread t owns chunks 4t .. 4t+3.  Fills pre[4] (prefix before each
// owned chunk) and returns the total.
__device__ __forceinline__ double chunk_prefix(const double (&v)[4], double (&pre)[4], double* sh) {
  const double local = (v[0] + v[1]) + (v[2] + v[3]);
  double total;
  const double base = block_exclusive_scan_d(local, sh, total);
  pre[0] = base;
  pre[1] = base + v[0];
  pre[2] = pre[1] + v[1];
  pre[3] = pre[2] + v[2];
  return total;
}

// Arrival of `weight` units on a per-request counter: returns true in exactly
// one CTA, the one completing `expected` units, and resets the counter for its
// next use.  Thread 0's add is a release and acquire at GPU scope after a CTA
// barrier, so everything the arriving CTAs wrote before the call is visible to
// every thread of the last arriver once the call returns.  The reset reaches
// the next use's arrivals through the release that announces their items (the
// queue's slot stores) or through the end of the launch.
__device__ __forceinline__ bool arrive_last(unsigned* counter, unsigned expected, int* sh_flag,
                                            unsigned weight = 1u) {
  sync_compute();
  if (threadIdx.x == 0) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;"
                 : "=r"(old) : "l"(counter), "r"(weight) : "memory");
    const bool last = (old + weight == expected);
    if (last) *counter = 0u;
    *sh_flag = last ? 1 : 0;
  }
  sync_compute();
  return *sh_flag != 0;
}

}  // namespace sv
