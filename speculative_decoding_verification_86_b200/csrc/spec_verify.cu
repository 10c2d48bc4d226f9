// Host side of the C ABI declared in include/spec_verify.h: argument checks,
// the context's device workspace, and the launches: one persistent k_engine
// (engine.cuh) per run -- the confidence head included in the prefix order,
// k_conf before it in the dense order.  Every launch goes to the caller's
// stream; nothing here synchronises except the host-buffer entry point, the
// diagnostics and the timing read-out.
#include "spec_verify.h"

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "conf.cuh"
#include "engine.cuh"
#include "shard.cuh"
#include "philox.cuh"
#include "refine.cuh"
#include "sample.cuh"
#include "stats.cuh"

namespace {

// Bound on the relative error of ex2.approx.ftz.f32 over the arguments the
// kernels pass (finite, <= 0, results above the fp32 subnormal range).  The
// maximum over every fp32 argument in [-126, 0], measured on B200 by
// spec_verify_selfcheck_ex2, is 1.4396e-7; the GPU tests re-measure it and
// require it to stay at or below this bound.
constexpr float kEpsEx2 = 1.5e-7f;

// timing classes: the verification kernel, the LM head's statistics and
// row-writing GEMMs, the confidence head
constexpr int kClassStats = 0, kClassLmStats = 1, kClassLmRows = 2, kClassConf = 3;
constexpr int kTimingClasses = 4;
constexpr int kMaxTimed = 4096;
// Automatic prefix tail: batches whose row segments make at most this many
// waves of the engine's grid read their requests' later positions together.
constexpr int64_t kTailWaves = 16;

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = (prev == dev) || (cudaSetDevice(dev) == cudaSuccess);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

// ---------------------------------------------------------------------------
// Scratch of spec_verify_greedy_noalloc.  Callers that may not allocate device
// memory get their working space from this fixed array instead of a context:
// every GPU that loads the library holds it (about 0.6 MB) until the process
// exits.  The statistics kernel writes one 16-byte record per (request, row,
// segment), a segment being 32768 bf16 or 16384 fp32 logits, and indexes the
// records with a stride of 2k + 1 rows per request.  Limits: B <= 256, k <= 8,
// and B * (2k + 1) * ceil(V / segment) <= 256 * 17 * 8 records, i.e.
// V <= 262144 for bf16 and V <= 131072 for fp32 at the largest B and k.
// ---------------------------------------------------------------------------
namespace {
constexpr int kNoAllocMaxBatch = 256;
constexpr int kNoAllocMaxK = 8;
constexpr size_t kNoAllocMaxRecords = size_t(kNoAllocMaxBatch) * (2 * kNoAllocMaxK + 1) * 8;
constexpr size_t kNoAllocMetaOff = 0;
constexpr size_t kNoAllocJobsOff = kNoAllocMetaOff + kNoAllocMaxRecords * sizeof(sv::ChunkMeta);
constexpr size_t kNoAllocArriveOff = kNoAllocJobsOff + size_t(kNoAllocMaxBatch) * sizeof(sv::Job);
constexpr size_t kNoAllocCountersOff = kNoAllocArriveOff + size_t(kNoAllocMaxBatch) * sizeof(unsigned);
constexpr size_t kNoAllocBytes = kNoAllocCountersOff + 2 * sizeof(sv::Counters);
static_assert(kNoAllocJobsOff % 16 == 0 && kNoAllocArriveOff % 16 == 0 &&
                  kNoAllocCountersOff % 16 == 0,
              "scratch records must stay 16-byte aligned");
constexpr int kNoAllocMaxDevices = 64;

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};
}  // namespace

static __device__ __align__(256) unsigned char g_greedy_scratch[kNoAllocBytes];

namespace {
// Device address of g_greedy_scratch on the current device.  In host code the
// array's name only stands in for the symbol; the kernels must be given the
// address the runtime reports, looked up once per device.
spec_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SPEC_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SPEC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_greedy_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return SPEC_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return SPEC_OK;
}
}  // namespace

struct spec_verify_ctx {
  int device = 0;
  int max_batch = 0;
  int max_k = 0;
  int64_t max_vocab = 0;
  int max_chunks = 0;
  int num_sms = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;

  sv::ChunkMeta* meta = nullptr;
  double* ssum = nullptr;
  unsigned* arrive_stats = nullptr;
  unsigned* arrive_sample = nullptr;
  unsigned* arrive_r1 = nullptr;
  sv::Job* jobs = nullptr;
  sv::SampleChunk* smass = nullptr;
  int* refine_list = nullptr;
  double2* rz = nullptr;
  double2* rm = nullptr;
  int* runc = nullptr;
  double4* rmp = nullptr;
  sv::Counters* counters = nullptr;  // [2], alternating between runs
  int32_t* conf_len = nullptr;
  float* tok_logits = nullptr;    // [max_batch, max_k, 2] drafted tokens' logits
  int32_t* fallback = nullptr;    // [max_batch]
  double* conf_prefix = nullptr;  // [max_batch, kMaxK]
  int32_t* conf_cap = nullptr;    // [max_batch]
  unsigned* conf_arrive = nullptr;
  unsigned long long* q_slots = nullptr;
  unsigned q_capacity = 0;
  unsigned* q_ctl = nullptr;
  int engine_grid = 0;        // CTAs of the k_engine instance for large batches
  int engine_grid_small = 0;  // ... and of the one for small dense batches
  int mode = SPEC_MODE_AUTO;  // as set by spec_verify_set_mode
  int tail_from = 0;          // as set by spec_verify_set_prefix_tail (0: automatic)
  unsigned run_id = 0;

  unsigned timing_mask = 0;  // bit c set: bracket launches of class c with events
  std::vector<cudaEvent_t> ev_start[kTimingClasses], ev_stop[kTimingClasses];
  int n_timed[kTimingClasses] = {0, 0, 0, 0};

  void* stage = nullptr;
  size_t stage_bytes = 0;
};

namespace {

// Maximum relative error of ex2.approx.ftz.f32 against fp64 exp2 over every
// fp32 value in [lo, hi]; the result (a non-negative double) is kept as its
// bit pattern so atomicMax on the integer orders it correctly.
__global__ void k_selfcheck_ex2(uint32_t first_bits, uint64_t count, unsigned long long* out) {
  double worst = 0.0;
  for (uint64_t n = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; n < count;
       n += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const float x = __uint_as_float(first_bits + static_cast<uint32_t>(n));
    const double ref = exp2(static_cast<double>(x));
    if (ref < 0x1p-126) continue;  // results in the flushed range carry absolute error only
    const double err = fabs(static_cast<double>(sv::ex2_approx(x)) - ref) / ref;
    worst = fmax(worst, err);
  }
  for (int off = 16; off; off >>= 1) worst = fmax(worst, __shfl_xor_sync(0xffffffffu, worst, off));
  if ((threadIdx.x & 31) == 0) atomicMax(out, static_cast<unsigned long long>(__double_as_longlong(worst)));
}

spec_status carve(spec_verify_ctx* c) {
  const size_t rows = static_cast<size_t>(c->max_batch) * (2 * c->max_k + 1);
  const size_t recs = rows * c->max_chunks;
  const size_t per_req_chunks = static_cast<size_t>(c->max_batch) * c->max_chunks;
  const size_t per_req_subs = per_req_chunks * sv::kBatchesPerChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t o_meta = take(recs * sizeof(sv::ChunkMeta));
  const size_t o_ssum = take(recs * sizeof(double));
  const size_t o_arr = take(3 * static_cast<size_t>(c->max_batch) * sizeof(unsigned));
  const size_t o_jobs = take(static_cast<size_t>(c->max_batch) * sizeof(sv::Job));
  const size_t o_smass = take(per_req_chunks * sv::kSampleParts * sizeof(sv::SampleChunk));
  const size_t o_rlist = take(static_cast<size_t>(c->max_batch) * sizeof(int));
  const size_t o_rz = take(per_req_subs * sizeof(double2));
  const size_t o_rm = take(per_req_subs * sizeof(double2));
  const size_t o_runc = take(per_req_subs * sizeof(int));
  const size_t o_rmp = take(per_req_subs * sv::kWarps * sizeof(double4));
  const size_t o_cnt = take(2 * sizeof(sv::Counters));
  const size_t o_conf = take(static_cast<size_t>(c->max_batch) * sizeof(int32_t));
  const size_t o_tokl = take(static_cast<size_t>(c->max_batch) * c->max_k * 2 * sizeof(float));
  const size_t o_fall = take(static_cast<size_t>(c->max_batch) * sizeof(int32_t));
  const size_t o_cpre = take(static_cast<size_t>(c->max_batch) * sv::kMaxK * sizeof(double));
  const size_t o_ccap = take(static_cast<size_t>(c->max_batch) * sizeof(int32_t));
  const size_t o_carr = take(sizeof(unsigned));
  // queue: every row segment, sample segment and refinement sub-chunk of a
  // batch, plus one exit ticket per CTA
  const size_t max_segs = static_cast<size_t>((c->max_vocab + sv::SegGeo<false>::kSeg - 1) /
                                              sv::SegGeo<false>::kSeg);
  const size_t max_subs = static_cast<size_t>(c->max_chunks) * sv::kBatchesPerChunk;
  const size_t cap = static_cast<size_t>(c->max_batch) *
                         ((2 * c->max_k + 1) * max_segs + c->max_chunks * sv::kSampleParts + max_subs) + 8192;
  if (cap > 0xFFFFFFF0ull) return SPEC_ERR_INVALID_ARG;
  c->q_capacity = static_cast<unsigned>(cap);
  const size_t o_qs = take(cap * sizeof(unsigned long long));
  const size_t o_qc = take(sv::kQWords * sizeof(unsigned));
  if (cudaMalloc(&c->ws, off) != cudaSuccess) {
    cudaGetLastError();
    return SPEC_ERR_NOMEM;
  }
  c->ws_bytes = off;
  char* b = static_cast<char*>(c->ws);
  c->meta = reinterpret_cast<sv::ChunkMeta*>(b + o_meta);
  c->ssum = reinterpret_cast<double*>(b + o_ssum);
  unsigned* arr = reinterpret_cast<unsigned*>(b + o_arr);
  c->arrive_stats = arr;
  c->arrive_sample = arr + c->max_batch;
  c->arrive_r1 = arr + 2 * c->max_batch;
  c->jobs = reinterpret_cast<sv::Job*>(b + o_jobs);
  c->smass = reinterpret_cast<sv::SampleChunk*>(b + o_smass);
  c->refine_list = reinterpret_cast<int*>(b + o_rlist);
  c->rz = reinterpret_cast<double2*>(b + o_rz);
  c->rm = reinterpret_cast<double2*>(b + o_rm);
  c->runc = reinterpret_cast<int*>(b + o_runc);
  c->rmp = reinterpret_cast<double4*>(b + o_rmp);
  c->counters = reinterpret_cast<sv::Counters*>(b + o_cnt);
  c->conf_len = reinterpret_cast<int32_t*>(b + o_conf);
  c->tok_logits = reinterpret_cast<float*>(b + o_tokl);
  c->fallback = reinterpret_cast<int32_t*>(b + o_fall);
  c->conf_prefix = reinterpret_cast<double*>(b + o_cpre);
  c->conf_cap = reinterpret_cast<int32_t*>(b + o_ccap);
  c->conf_arrive = reinterpret_cast<unsigned*>(b + o_carr);
  c->q_slots = reinterpret_cast<unsigned long long*>(b + o_qs);
  c->q_ctl = reinterpret_cast<unsigned*>(b + o_qc);
  if (cudaMemset(c->ws, 0, off) != cudaSuccess) return SPEC_ERR_CUDA;
  return SPEC_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

void timing_mark(spec_verify_ctx* c, int cls, bool start, cudaStream_t s) {
  if (!(c->timing_mask & (1u << cls))) return;
  int n = c->n_timed[cls];
  if (n >= kMaxTimed) return;
  std::vector<cudaEvent_t>& v = start ? c->ev_start[cls] : c->ev_stop[cls];
  while (static_cast<int>(v.size()) <= n) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    v.push_back(e);
  }
  cudaEventRecord(v[n], s);
  if (!start) c->n_timed[cls] = n + 1;
}

spec_status check_conf(const spec_verify_ctx* c, const spec_conf_args* conf) {
  if (!conf) return SPEC_OK;
  if (!conf->hidden || !conf->w) return SPEC_ERR_INVALID_ARG;
  if (conf->kb < 1 || conf->kb > sv::kMaxK || conf->H < 1 || conf->H > 65536)
    return SPEC_ERR_INVALID_ARG;
  if (!aligned(conf->hidden, 2) || !aligned(conf->w, 2)) return SPEC_ERR_UNSUPPORTED;
  (void)c;
  return SPEC_OK;
}

// k_conf: per-request budgets, capped by verify_len when k >= 0, then the
// batch-wide budget when conf->total_budget > 0.
spec_status launch_conf(spec_verify_ctx* c, const spec_conf_args* conf, int B, int k,
                        const int32_t* vlen, int32_t* out_len, float* out_surv, cudaStream_t s) {
  sv::ConfParams cp;
  cp.hidden = static_cast<const uint16_t*>(conf->hidden);
  cp.w = static_cast<const uint16_t*>(conf->w);
  cp.bias = conf->bias;
  cp.threshold = conf->threshold;
  cp.B = B;
  cp.kb = conf->kb;
  cp.H = conf->H;
  cp.k = k;
  cp.vlen = vlen;
  cp.total = conf->total_budget > 0 ? conf->total_budget : 0;
  cp.prefix = c->conf_prefix;
  cp.cap = c->conf_cap;
  cp.arrive = c->conf_arrive;
  cp.out_len = out_len;
  cp.out_survival = out_surv;
  timing_mark(c, kClassConf, true, s);
  sv::k_conf<<<B, sv::kThreads, 0, s>>>(cp);
  timing_mark(c, kClassConf, false, s);
  return SPEC_OK;
}

spec_status run_impl(spec_verify_ctx* c, const void* target, const void* draft, spec_dtype dtype,
                     const int32_t* tokens, const int32_t* vlen, const float* temp,
                     const spec_conf_args* conf, int B, int k, int64_t V, uint64_t seed,
                     uint32_t step, uint32_t req_off, const double* uniforms, bool force_greedy,
                     int32_t* out_acc, int32_t* out_tok, float* out_p, float* out_q,
                     uint32_t* out_status, cudaStream_t s) {
  if (!c) return SPEC_ERR_INVALID_ARG;
  if (B < 0 || B > c->max_batch || k < 0 || k > c->max_k || V < 1 || V > c->max_vocab)
    return SPEC_ERR_INVALID_ARG;
  if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_ERR_INVALID_ARG;
  if (B == 0) return SPEC_OK;
  if (!target || !out_acc || !out_tok || (k > 0 && !tokens)) return SPEC_ERR_INVALID_ARG;
  if (!force_greedy && !draft && !temp && k > 0) return SPEC_ERR_INVALID_ARG;
  if (spec_status st = check_conf(c, conf); st != SPEC_OK) return st;
  const bool bf16 = dtype == SPEC_BF16;
  const int64_t esize = bf16 ? 2 : 4;
  if ((V * esize) % 16 != 0) return SPEC_ERR_UNSUPPORTED;
  if (!aligned(target, 16) || (draft && !aligned(draft, 16))) return SPEC_ERR_UNSUPPORTED;
  if ((tokens && !aligned(tokens, 4)) || (vlen && !aligned(vlen, 4)) || (temp && !aligned(temp, 4)) ||
      !aligned(out_acc, 4) || !aligned(out_tok, 4) || (out_p && !aligned(out_p, 4)) ||
      (out_q && !aligned(out_q, 4)) || (out_status && !aligned(out_status, 4)) ||
      (uniforms && !aligned(uniforms, 8)))
    return SPEC_ERR_UNSUPPORTED;

  DeviceGuard g(c->device);
  if (!g.ok) return SPEC_ERR_CUDA;

  const int chunk = bf16 ? sv::kChunkBf16 : sv::kChunkF32;
  const int n_chunks = static_cast<int>((V + chunk - 1) / chunk);
  const int segl = bf16 ? sv::SegGeo<true>::kSeg : sv::SegGeo<false>::kSeg;
  int n_segs = static_cast<int>((V + segl - 1) / segl);

  sv::RunParams p{};
  p.target = target;
  p.draft = force_greedy ? nullptr : draft;
  p.tokens = tokens;
  p.vlen = vlen;
  p.temp = force_greedy ? nullptr : temp;
  p.conf_len = nullptr;
  p.uniforms = uniforms;
  p.B = B;
  p.k = k;
  p.V = V;
  p.row_stride = V;
  p.v_lo = 0;
  p.tok_logits = nullptr;
  p.tok_cache = c->tok_logits;  // the engine's statistics items leave the drafted tokens' logits here
  p.fallback = nullptr;
  p.shard_tok = nullptr;
  p.c_lo = 0;
  p.c_hi = 0;
  p.n_chunks = n_chunks;
  p.n_segs = n_segs;
  p.seed = seed;
  p.step = step;
  p.req_off = req_off;
  p.force_greedy = force_greedy ? 1 : 0;
  p.eps_ex2 = kEpsEx2;
  p.out_acc = out_acc;
  p.out_tok = out_tok;
  p.out_p = out_p;
  p.out_q = out_q;
  p.out_status = out_status;
  p.meta = c->meta;
  p.ssum = c->ssum;
  p.arrive_stats = c->arrive_stats;
  p.arrive_sample = c->arrive_sample;
  p.jobs = c->jobs;
  p.smass = c->smass;
  p.refine_list = c->refine_list;
  p.arrive_r1 = c->arrive_r1;
  p.rz = c->rz;
  p.rm = c->rm;
  p.runc = c->runc;
  p.rmp = c->rmp;
  if (++c->run_id == 0) c->run_id = 1;
  p.counters = c->counters + (c->run_id & 1u);
  p.counters_next = c->counters + ((c->run_id + 1u) & 1u);

  cudaGetLastError();  // clear stale errors so the check below is ours
  // Order of the statistics.  Automatic: the prefix order saves reads when the
  // batch's rows compete for the grid; when every row the batch may verify
  // fits in one wave of the grid, reading them all at once costs no extra time
  // and removes the waits between positions, so the dense order is faster.
  int mode = c->mode;
  if (mode == SPEC_MODE_AUTO)
    mode = static_cast<int64_t>(B) * (2 * k + 1) * n_segs <= c->engine_grid ? SPEC_MODE_DENSE
                                                                           : SPEC_MODE_PREFIX;
  p.mode = (force_greedy || mode == SPEC_MODE_PREFIX) ? sv::kModePrefix : sv::kModeDense;
  {
    // Prefix order's dense tail.  Automatic: from position 2 when the batch's
    // rows, in segments, make at most kTailWaves waves of the grid (the grid
    // then idles while long chains walk their positions one at a time), else
    // none (every extra row read competes with other requests' rows).
    int tail = c->tail_from;
    if (tail == 0) {
      const int64_t rows = static_cast<int64_t>(B) * (p.draft ? 2 * k + 1 : k + 1);
      tail = rows * n_segs <= kTailWaves * static_cast<int64_t>(c->engine_grid) ? 2 : k + 1;
    }
    p.tail_from = std::min(tail, k + 1);
  }
  // Dense order: a statistics item is a whole row when the batch has at least
  // as many rows as the grid has CTAs (one staging pipeline per row, no drain
  // between its segments), else a segment (small batches: every segment of
  // every row in flight at once) -- a short one when even those all fit.
  p.whole_rows = (p.mode == sv::kModeDense &&
                  static_cast<int64_t>(B) * (2 * k + 1) >= c->engine_grid) ? 1 : 0;
  p.seg_len = segl;
  if (p.mode == sv::kModeDense && !p.whole_rows) {
    const int sl = segl / sv::kBatches * sv::kShortSegBatches;
    const int ns = static_cast<int>((V + sl - 1) / sl);
    if (static_cast<int64_t>(B) * (2 * k + 1) * ns <= c->engine_grid && ns <= c->max_chunks) {
      p.short_segs = 1;
      p.seg_len = sl;
      n_segs = ns;
      p.n_segs = ns;
    }
  }
  if (conf && p.mode == sv::kModePrefix) {
    // the confidence head runs inside the verification launch, as its first B
    // items (the prefix order reads position 0 before the budgets are needed)
    sv::ConfParams& cp = p.cp;
    cp.hidden = static_cast<const uint16_t*>(conf->hidden);
    cp.w = static_cast<const uint16_t*>(conf->w);
    cp.bias = conf->bias;
    cp.threshold = conf->threshold;
    cp.B = B;
    cp.kb = conf->kb;
    cp.H = conf->H;
    cp.k = k;
    cp.vlen = vlen;
    cp.total = conf->total_budget > 0 ? conf->total_budget : 0;
    cp.prefix = c->conf_prefix;
    cp.cap = c->conf_cap;
    cp.arrive = c->conf_arrive;
    cp.out_len = c->conf_len;
    cp.out_survival = nullptr;
    p.conf_len = c->conf_len;
    p.n_conf = static_cast<unsigned>(B);
  } else if (conf) {
    // the dense order plans every row from the budgets: the head runs first,
    // as its own launch (inside the launch, with the statistics items waiting
    // for it, measured 5-10 us slower)
    launch_conf(c, conf, B, k, vlen, c->conf_len, nullptr, s);
    p.conf_len = c->conf_len;
  }
  p.q_slots = c->q_slots;
  p.q_capacity = c->q_capacity;
  p.q_ctl = c->q_ctl;
  {
    // class regions: every later position's rows, every sample item and every
    // refinement sub-chunk of the batch (each generated at most once)
    // small batches: one sample item per part of a chunk when the parts of
    // every request fit two waves of the grid (usually only some requests sample)
    p.sample_parts = static_cast<int64_t>(B) * n_chunks * sv::kSampleParts <= 2ll * c->engine_grid ? 1 : 0;
    const uint64_t caps[sv::kQClasses] = {
        static_cast<uint64_t>(B) * (2 * k + 1) * n_segs,
        static_cast<uint64_t>(B) * sv::sample_items_of(n_chunks, p.sample_parts != 0),
        static_cast<uint64_t>(B) * n_chunks * sv::kSubsPerChunk};
    uint64_t off = 0;
    for (int q = 0; q < sv::kQClasses; ++q) {
      p.q_off[q] = static_cast<unsigned>(off);
      p.q_cap[q] = static_cast<unsigned>(caps[q]);
      off += caps[q];
    }
    if (off > c->q_capacity) return SPEC_ERR_INVALID_ARG;
  }
  p.q_epoch = c->run_id;  // >= 1: slots left by earlier runs carry older epochs
  // implicit tickets: the confidence head's items, then the statistics items
  // of every row (dense) or of position 0's rows (prefix)
  const uint64_t per_req = p.mode == sv::kModePrefix ? 2ull * n_segs
                           : (p.whole_rows ? static_cast<uint64_t>(2 * k + 1)
                                           : static_cast<uint64_t>(2 * k + 1) * n_segs);
  const uint64_t n_init = static_cast<uint64_t>(p.n_conf) + static_cast<uint64_t>(B) * per_req;
  if (n_init > 0xFFFF0000ull) return SPEC_ERR_INVALID_ARG;
  p.n_init = static_cast<unsigned>(n_init);
  timing_mark(c, kClassStats, true, s);
  // a small dense batch (its items within two waves of that instance's grid)
  // is latency bound: the instance with more registers per thread
  const bool small = p.mode == sv::kModeDense && !p.whole_rows &&
                     static_cast<int64_t>(B) * (2 * k + 1) * p.n_segs <= 2ll * c->engine_grid_small;
  if (small) {
    if (bf16) sv::k_engine<true, sv::kEngineMinBlocksSmall><<<c->engine_grid_small, sv::kThreads, sv::kStageBytes, s>>>(p);
    else sv::k_engine<false, sv::kEngineMinBlocksSmall><<<c->engine_grid_small, sv::kThreads, sv::kStageBytes, s>>>(p);
  } else {
    if (bf16) sv::k_engine<true, sv::kEngineMinBlocks><<<c->engine_grid, sv::kThreads, sv::kStageBytes, s>>>(p);
    else sv::k_engine<false, sv::kEngineMinBlocks><<<c->engine_grid, sv::kThreads, sv::kStageBytes, s>>>(p);
  }
  timing_mark(c, kClassStats, false, s);
  if (cudaGetLastError() != cudaSuccess) return SPEC_ERR_CUDA;
  return SPEC_OK;
}


// ---------------------------------------------------- vocabulary-parallel --
// Shards are whole statistics segments, split as evenly as the segment count
// allows; the exchange blocks have the widest rank's size on every rank.
spec_status shard_geometry(int64_t V, bool bf16, int n_shards, sv::ShardBounds* sb,
                           int64_t* seg_len_out) {
  const int64_t segl = bf16 ? sv::SegGeo<true>::kSeg : sv::SegGeo<false>::kSeg;
  if (V < 1 || n_shards < 1 || n_shards > sv::kMaxShards) return SPEC_ERR_INVALID_ARG;
  const int64_t n_segs = (V + segl - 1) / segl;
  if (n_segs < n_shards) return SPEC_ERR_INVALID_ARG;
  sb->n = n_shards;
  sb->nls_max = 0;
  for (int r = 0; r <= n_shards; ++r) sb->seg_lo[r] = static_cast<int>(n_segs * r / n_shards);
  for (int r = 0; r < n_shards; ++r) sb->nls_max = std::max(sb->nls_max, sb->seg_lo[r + 1] - sb->seg_lo[r]);
  *seg_len_out = segl;
  return SPEC_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct ShardSizes {
  size_t rec_bytes, tok_off, block1, block2, block3;
  int nlc_max, nsub_max;
};

ShardSizes shard_sizes(int B, int k, const sv::ShardBounds& sb) {
  ShardSizes z;
  z.rec_bytes = static_cast<size_t>(B) * (2 * k + 1) * sb.nls_max * sizeof(sv::ShardRec);
  z.tok_off = align256(z.rec_bytes);
  z.block1 = z.tok_off + align256(static_cast<size_t>(B) * k * 2 * sizeof(float));
  z.nlc_max = sb.nls_max * sv::kChunksPerSeg;
  z.block2 = static_cast<size_t>(B) * z.nlc_max * sv::kSampleParts * sizeof(sv::SampleChunk);
  z.nsub_max = z.nlc_max * sv::kSubsPerChunk;
  z.block3 = static_cast<size_t>(B) * z.nsub_max * sizeof(sv::RefRec);
  return z;
}

// Common checks and parameters of the per-rank phases: the rank's logits are
// [B, k+1, width] / [B, k, width] for tokens [v_lo, v_lo + width).
spec_status shard_params(spec_verify_ctx* c, int rank, int n_shards, const void* target,
                         const void* draft, spec_dtype dtype, const int32_t* tokens,
                         const int32_t* vlen, const float* temp, const spec_conf_args* conf,
                         int B, int k, int64_t V, sv::RunParams* pp, sv::ShardBounds* sb,
                         int64_t* seg_len) {
  if (!c || B < 1 || B > c->max_batch || k < 0 || k > c->max_k || V < 1 || V > c->max_vocab)
    return SPEC_ERR_INVALID_ARG;
  if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_ERR_INVALID_ARG;
  const bool bf16 = dtype == SPEC_BF16;
  if (spec_status st = shard_geometry(V, bf16, n_shards, sb, seg_len); st != SPEC_OK) return st;
  if (rank < 0 || rank >= n_shards) return SPEC_ERR_INVALID_ARG;
  if (!target || (k > 0 && !tokens)) return SPEC_ERR_INVALID_ARG;
  if (spec_status st = check_conf(c, conf); st != SPEC_OK) return st;
  const int64_t esize = bf16 ? 2 : 4;
  if ((V * esize) % 16 != 0) return SPEC_ERR_UNSUPPORTED;
  if (!aligned(target, 16) || (draft && !aligned(draft, 16))) return SPEC_ERR_UNSUPPORTED;
  const int64_t v_lo = std::min<int64_t>(static_cast<int64_t>(sb->seg_lo[rank]) * *seg_len, V);
  const int64_t v_hi = std::min<int64_t>(static_cast<int64_t>(sb->seg_lo[rank + 1]) * *seg_len, V);
  sv::RunParams p{};
  p.target = target;
  p.draft = draft;
  p.tokens = tokens;
  p.vlen = vlen;
  p.temp = temp;
  p.conf_len = conf ? c->conf_len : nullptr;
  p.B = B;
  p.k = k;
  p.V = V;
  p.row_stride = v_hi - v_lo;
  p.v_lo = v_lo;
  const int chunk = bf16 ? sv::kChunkBf16 : sv::kChunkF32;
  p.n_chunks = static_cast<int>((V + chunk - 1) / chunk);
  p.n_segs = sb->seg_lo[n_shards];
  p.c_lo = sb->seg_lo[rank] * sv::kChunksPerSeg;
  p.c_hi = std::min(sb->seg_lo[rank + 1] * sv::kChunksPerSeg, p.n_chunks);
  p.eps_ex2 = kEpsEx2;
  p.meta = c->meta;
  p.ssum = c->ssum;
  p.jobs = c->jobs;
  p.smass = c->smass;
  p.tok_logits = c->tok_logits;
  p.fallback = c->fallback;
  p.refine_list = c->refine_list;
  p.rz = c->rz;
  p.rm = c->rm;
  p.runc = c->runc;
  p.counters = c->counters + (c->run_id & 1u);
  p.counters_next = c->counters + ((c->run_id + 1u) & 1u);
  *pp = p;
  return SPEC_OK;
}

int grid_for(int64_t n) { return static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096)); }

// The draws of a run (spec_verify_draws).
__global__ void k_draws(uint64_t seed, uint32_t step, uint32_t req_off, int B, int k, double* out) {
  const int64_t n = static_cast<int64_t>(B) * (k + 1) * 2;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / 2;
    const int d = static_cast<int>(e % 2);
    const int i = static_cast<int>(r / (k + 1)), j = static_cast<int>(r % (k + 1));
    out[e] = sv::draw_uniform(seed, req_off + static_cast<uint32_t>(i), static_cast<uint32_t>(j),
                              static_cast<uint32_t>(d), step);
  }
}

// Grid of the refinement partials: grid-strides over B x nsub items, eight CTAs per SM.
int refine_grid(const spec_verify_ctx* c, int B, int nsub) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(B) * nsub,
                                                                  8LL * c->num_sms)));
}
}  // namespace

extern "C" {

const char* spec_status_string(spec_status s) {
  switch (s) {
    case SPEC_OK: return "ok";
    case SPEC_ERR_INVALID_ARG: return "invalid argument";
    case SPEC_ERR_UNSUPPORTED: return "unsupported layout, alignment or size";
    case SPEC_ERR_CUDA: return "CUDA runtime error";
    case SPEC_ERR_NOMEM: return "out of memory";
    case SPEC_ERR_DEVICE_STATUS: return "a request failed on the device (see out_status)";
    case SPEC_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

spec_status spec_verify_init(spec_verify_ctx** out, int device, int max_batch, int max_k,
                             int64_t max_vocab) {
  if (!out) return SPEC_ERR_INVALID_ARG;
  *out = nullptr;
  if (max_batch < 1 || max_batch > 65535 || max_k < 0 || max_k > sv::kMaxK || max_vocab < 1 ||
      max_vocab > static_cast<int64_t>(sv::kMaxChunksPerRow) * (sv::kChunkF32 / sv::kBatchesPerChunk))
    return SPEC_ERR_INVALID_ARG;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess) {
    cudaGetLastError();
    return SPEC_ERR_CUDA;
  }
  if (device < 0 || device >= ndev) return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(device);
  if (!g.ok) return SPEC_ERR_CUDA;
  spec_verify_ctx* c = new (std::nothrow) spec_verify_ctx();
  if (!c) return SPEC_ERR_NOMEM;
  c->device = device;
  c->max_batch = max_batch;
  c->max_k = max_k;
  c->max_vocab = max_vocab;
  c->max_chunks = static_cast<int>((max_vocab + sv::kChunkF32 - 1) / sv::kChunkF32);
  if (cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
    delete c;
    return SPEC_ERR_CUDA;
  }
  const spec_status st = carve(c);
  if (st != SPEC_OK) {
    if (c->ws) cudaFree(c->ws);
    delete c;
    return st;
  }
  // one grid per instance: as many CTAs as are resident at once
  auto grid_of = [&](auto kb, auto kf, int* grid) {
    int occ_a = 0, occ_b = 0;
    if (cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sv::kStageBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(sv::kStageBytes)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_a, kb, sv::kThreads, sv::kStageBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_b, kf, sv::kThreads, sv::kStageBytes) != cudaSuccess)
      return false;
    *grid = c->num_sms * std::max(1, std::min(occ_a, occ_b));
    return true;
  };
  if (!grid_of(sv::k_engine<true, sv::kEngineMinBlocks>, sv::k_engine<false, sv::kEngineMinBlocks>, &c->engine_grid) ||
      !grid_of(sv::k_engine<true, sv::kEngineMinBlocksSmall>, sv::k_engine<false, sv::kEngineMinBlocksSmall>,
               &c->engine_grid_small)) {
    cudaFree(c->ws);
    delete c;
    return SPEC_ERR_CUDA;
  }
  *out = c;
  return SPEC_OK;
}

spec_status spec_verify_destroy(spec_verify_ctx* c) {
  if (!c) return SPEC_OK;
  DeviceGuard g(c->device);
  cudaDeviceSynchronize();
  for (int k = 0; k < kTimingClasses; ++k) {
    for (cudaEvent_t e : c->ev_start[k]) cudaEventDestroy(e);
    for (cudaEvent_t e : c->ev_stop[k]) cudaEventDestroy(e);
  }
  if (c->ws) cudaFree(c->ws);
  if (c->stage) cudaFree(c->stage);
  delete c;
  return SPEC_OK;
}

spec_status spec_verify_run(spec_verify_ctx* ctx, const void* target_logits,
                            const void* draft_logits, spec_dtype dtype,
                            const int32_t* draft_tokens, const int32_t* verify_len,
                            const float* temperature, const spec_conf_args* conf, int B, int k,
                            int64_t V, uint64_t seed, uint32_t step, uint32_t request_offset,
                            int32_t* out_accepted, int32_t* out_tokens, float* out_p,
                            float* out_q, uint32_t* out_status, cudaStream_t stream) {
  return run_impl(ctx, target_logits, draft_logits, dtype, draft_tokens, verify_len, temperature,
                  conf, B, k, V, seed, step, request_offset, nullptr, false, out_accepted,
                  out_tokens, out_p, out_q, out_status, stream);
}

spec_status spec_verify_run_with_uniforms(
    spec_verify_ctx* ctx, const void* target_logits, const void* draft_logits, spec_dtype dtype,
    const int32_t* draft_tokens, const int32_t* verify_len, const float* temperature,
    const spec_conf_args* conf, int B, int k, int64_t V, const double* uniforms,
    int32_t* out_accepted, int32_t* out_tokens, float* out_p, float* out_q,
    uint32_t* out_status, cudaStream_t stream) {
  if (!uniforms && B > 0) return SPEC_ERR_INVALID_ARG;
  return run_impl(ctx, target_logits, draft_logits, dtype, draft_tokens, verify_len, temperature,
                  conf, B, k, V, 0, 0, 0, uniforms, false, out_accepted, out_tokens, out_p,
                  out_q, out_status, stream);
}

spec_status spec_verify_greedy(spec_verify_ctx* ctx, const void* target_logits, spec_dtype dtype,
                               const int32_t* draft_tokens, const int32_t* verify_len, int B,
                               int k, int64_t V, int32_t* out_accepted, int32_t* out_tokens,
                               uint32_t* out_status, cudaStream_t stream) {
  return run_impl(ctx, target_logits, nullptr, dtype, draft_tokens, verify_len, nullptr, nullptr,
                  B, k, V, 0, 0, 0, nullptr, true, out_accepted, out_tokens, nullptr, nullptr,
                  out_status, stream);
}

spec_status spec_conf_budget(spec_verify_ctx* ctx, const void* hidden, const void* w, float bias,
                             int B, int kb, int H, float threshold, int32_t* out_len,
                             float* out_survival, cudaStream_t stream) {
  if (!ctx || B < 0 || B > ctx->max_batch) return SPEC_ERR_INVALID_ARG;
  if (B == 0) return SPEC_OK;
  if (!out_len) return SPEC_ERR_INVALID_ARG;
  spec_conf_args conf{hidden, w, bias, kb, H, threshold, 0};
  if (spec_status st = check_conf(ctx, &conf); st != SPEC_OK) return st;
  if (!aligned(out_len, 4) || (out_survival && !aligned(out_survival, 4)))
    return SPEC_ERR_UNSUPPORTED;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  launch_conf(ctx, &conf, B, -1, nullptr, out_len, out_survival, stream);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_verify_lengths(spec_verify_ctx* ctx, const spec_conf_args* conf,
                                const int32_t* verify_len, int B, int k, int32_t* out_len,
                                float* out_survival, cudaStream_t stream) {
  if (!ctx || !conf || B < 0 || B > ctx->max_batch || k < 0 || k > ctx->max_k)
    return SPEC_ERR_INVALID_ARG;
  if (B == 0) return SPEC_OK;
  if (!out_len) return SPEC_ERR_INVALID_ARG;
  if (spec_status st = check_conf(ctx, conf); st != SPEC_OK) return st;
  if (!aligned(out_len, 4) || (out_survival && !aligned(out_survival, 4)) ||
      (verify_len && !aligned(verify_len, 4)))
    return SPEC_ERR_UNSUPPORTED;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  launch_conf(ctx, conf, B, k, verify_len, out_len, out_survival, stream);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_verify_run_host(spec_verify_ctx* ctx, const void* target_logits,
                                 const void* draft_logits, spec_dtype dtype,
                                 const int32_t* draft_tokens, const int32_t* verify_len,
                                 const float* temperature, const spec_conf_args* conf, int B,
                                 int k, int64_t V, uint64_t seed, uint32_t step,
                                 uint32_t request_offset, int32_t* out_accepted,
                                 int32_t* out_tokens, float* out_p, float* out_q,
                                 uint32_t* out_status, cudaStream_t stream) {
  if (!ctx) return SPEC_ERR_INVALID_ARG;
  if (B < 0 || B > ctx->max_batch || k < 0 || k > ctx->max_k || V < 1 || V > ctx->max_vocab)
    return SPEC_ERR_INVALID_ARG;
  if (B == 0) return SPEC_OK;
  if (!target_logits || !out_accepted || !out_tokens || (k > 0 && !draft_tokens))
    return SPEC_ERR_INVALID_ARG;
  if (spec_status st = check_conf(ctx, conf); st != SPEC_OK) return st;
  const size_t es = dtype == SPEC_BF16 ? 2 : 4;
  const size_t nB = static_cast<size_t>(B);
  const size_t sz_t = nB * (k + 1) * V * es, sz_d = draft_logits ? nB * k * V * es : 0;
  const size_t sz_x = nB * k * 4, sz_l = verify_len ? nB * 4 : 0, sz_T = temperature ? nB * 4 : 0;
  const size_t sz_h = conf ? nB * conf->kb * conf->H * 2 : 0, sz_w = conf ? conf->H * 2 : 0;
  const size_t sz_acc = nB * 4, sz_tok = nB * (k + 1) * 4, sz_pq = nB * k * 4, sz_st = nB * 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t o_t = take(sz_t), o_d = take(sz_d), o_x = take(sz_x), o_l = take(sz_l),
               o_T = take(sz_T), o_h = take(sz_h), o_w = take(sz_w), o_acc = take(sz_acc),
               o_tok = take(sz_tok), o_p = take(out_p ? sz_pq : 0), o_q = take(out_q ? sz_pq : 0),
               o_st = take(sz_st);
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  if (off > ctx->stage_bytes) {
    if (ctx->stage) {
      cudaStreamSynchronize(stream);
      cudaFree(ctx->stage);
      ctx->stage = nullptr;
      ctx->stage_bytes = 0;
    }
    if (cudaMalloc(&ctx->stage, off) != cudaSuccess) {
      cudaGetLastError();
      return SPEC_ERR_NOMEM;
    }
    ctx->stage_bytes = off;
  }
  char* S = static_cast<char*>(ctx->stage);
  auto h2d = [&](size_t o, const void* src, size_t n) {
    return n == 0 || cudaMemcpyAsync(S + o, src, n, cudaMemcpyHostToDevice, stream) == cudaSuccess;
  };
  if (!h2d(o_t, target_logits, sz_t) || !h2d(o_d, draft_logits, sz_d) ||
      !h2d(o_x, draft_tokens, sz_x) || !h2d(o_l, verify_len, sz_l) ||
      !h2d(o_T, temperature, sz_T) || (conf && (!h2d(o_h, conf->hidden, sz_h) || !h2d(o_w, conf->w, sz_w))))
    return SPEC_ERR_CUDA;
  spec_conf_args dconf{};
  if (conf) {
    dconf = *conf;
    dconf.hidden = S + o_h;
    dconf.w = S + o_w;
  }
  spec_status st = run_impl(ctx, S + o_t, draft_logits ? S + o_d : nullptr, dtype,
                            k > 0 ? reinterpret_cast<int32_t*>(S + o_x) : nullptr,
                            verify_len ? reinterpret_cast<int32_t*>(S + o_l) : nullptr,
                            temperature ? reinterpret_cast<float*>(S + o_T) : nullptr,
                            conf ? &dconf : nullptr, B, k, V, seed, step, request_offset, nullptr,
                            false, reinterpret_cast<int32_t*>(S + o_acc),
                            reinterpret_cast<int32_t*>(S + o_tok),
                            out_p ? reinterpret_cast<float*>(S + o_p) : nullptr,
                            out_q ? reinterpret_cast<float*>(S + o_q) : nullptr,
                            reinterpret_cast<uint32_t*>(S + o_st), stream);
  if (st != SPEC_OK) return st;
  std::vector<uint32_t> status_host(out_status ? 0 : nB);
  uint32_t* st_dst = out_status ? out_status : status_host.data();
  auto d2h = [&](void* dst, size_t o, size_t n) {
    return n == 0 || cudaMemcpyAsync(dst, S + o, n, cudaMemcpyDeviceToHost, stream) == cudaSuccess;
  };
  if (!d2h(out_accepted, o_acc, sz_acc) || !d2h(out_tokens, o_tok, sz_tok) ||
      (out_p && !d2h(out_p, o_p, sz_pq)) || (out_q && !d2h(out_q, o_q, sz_pq)) ||
      !d2h(st_dst, o_st, sz_st))
    return SPEC_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SPEC_ERR_CUDA;
  for (size_t i = 0; i < nB; ++i)
    if (st_dst[i] != 0) return SPEC_ERR_DEVICE_STATUS;
  return SPEC_OK;
}

spec_status spec_verify_selfcheck_ex2(int device, float lo, float hi, double* max_rel_err) {
  if (!max_rel_err || !(lo <= hi) || hi > 0.0f || !(lo >= -126.0f)) return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(device);
  if (!g.ok) return SPEC_ERR_CUDA;
  // negative fp32 values: larger magnitude <=> larger bit pattern
  uint32_t bhi, blo;
  std::memcpy(&bhi, &hi, 4);
  std::memcpy(&blo, &lo, 4);
  if (hi == 0.0f) bhi = 0x80000000u;
  const uint32_t first = bhi, last = blo;
  const uint64_t count = static_cast<uint64_t>(last) - first + 1;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, sizeof *d) != cudaSuccess) return SPEC_ERR_NOMEM;
  cudaMemset(d, 0, sizeof *d);
  k_selfcheck_ex2<<<1184, 256>>>(first, count, d);
  unsigned long long h = 0;
  const bool ok = cudaGetLastError() == cudaSuccess &&
                  cudaMemcpy(&h, d, sizeof h, cudaMemcpyDeviceToHost) == cudaSuccess;
  cudaFree(d);
  if (!ok) return SPEC_ERR_CUDA;
  double v;
  std::memcpy(&v, &h, 8);
  *max_rel_err = v;
  return SPEC_OK;
}

double spec_verify_ex2_error_bound(void) { return static_cast<double>(kEpsEx2); }

spec_status spec_verify_greedy_noalloc(const void* target_logits, spec_dtype dtype,
                                       const int32_t* draft_tokens, const int32_t* verify_len,
                                       int B, int k, int64_t V, int32_t* out_accepted,
                                       int32_t* out_tokens, uint32_t* out_status,
                                       cudaStream_t stream) {
  if (B < 0 || B > kNoAllocMaxBatch || k < 0 || k > kNoAllocMaxK || V < 1)
    return SPEC_ERR_INVALID_ARG;
  if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_ERR_INVALID_ARG;
  const bool bf16 = dtype == SPEC_BF16;
  const int segl = bf16 ? sv::SegGeo<true>::kSeg : sv::SegGeo<false>::kSeg;
  const int64_t n_segs = (V + segl - 1) / segl;  // statistics records per row
  if (static_cast<size_t>(B) * (2 * k + 1) * static_cast<size_t>(n_segs) > kNoAllocMaxRecords)
    return SPEC_ERR_INVALID_ARG;
  if (B == 0) return SPEC_OK;
  if (!target_logits || !out_accepted || !out_tokens || (k > 0 && !draft_tokens))
    return SPEC_ERR_INVALID_ARG;
  if ((V * (bf16 ? 2 : 4)) % 16 != 0 || !aligned(target_logits, 16)) return SPEC_ERR_UNSUPPORTED;
  if ((draft_tokens && !aligned(draft_tokens, 4)) || (verify_len && !aligned(verify_len, 4)) ||
      !aligned(out_accepted, 4) || !aligned(out_tokens, 4) ||
      (out_status && !aligned(out_status, 4)))
    return SPEC_ERR_UNSUPPORTED;
  void* base = nullptr;
  if (spec_status st = noalloc_scratch(&base); st != SPEC_OK) return st;
  char* b = static_cast<char*>(base);

  sv::RunParams p{};
  p.target = target_logits;
  p.tokens = draft_tokens;
  p.vlen = verify_len;
  p.B = B;
  p.k = k;
  p.V = V;
  p.row_stride = V;
  p.n_chunks = static_cast<int>((V + (bf16 ? sv::kChunkBf16 : sv::kChunkF32) - 1) /
                                (bf16 ? sv::kChunkBf16 : sv::kChunkF32));
  p.n_segs = static_cast<int>(n_segs);
  p.force_greedy = 1;
  p.eps_ex2 = kEpsEx2;
  p.out_acc = out_accepted;
  p.out_tok = out_tokens;
  p.out_status = out_status;
  p.meta = reinterpret_cast<sv::ChunkMeta*>(b + kNoAllocMetaOff);
  p.jobs = reinterpret_cast<sv::Job*>(b + kNoAllocJobsOff);
  p.arrive_stats = reinterpret_cast<unsigned*>(b + kNoAllocArriveOff);
  p.counters = reinterpret_cast<sv::Counters*>(b + kNoAllocCountersOff);
  p.counters_next = p.counters + 1;

  cudaGetLastError();
  // The arrival counters must start at zero; the array keeps whatever the
  // previous call (or an interrupted one) left there.
  if (cudaMemsetAsync(p.arrive_stats, 0, static_cast<size_t>(B) * sizeof(unsigned), stream) !=
      cudaSuccess)
    return SPEC_ERR_CUDA;
  // greedy reads target rows only: one CTA per (request, target row, segment)
  p.launch_rows = k + 1;
  const int64_t ctas = static_cast<int64_t>(B) * (k + 1) * n_segs;
  if (bf16) sv::k_stats<true><<<static_cast<unsigned>(ctas), sv::kThreads, 0, stream>>>(p);
  else sv::k_stats<false><<<static_cast<unsigned>(ctas), sv::kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_verify_draws(spec_verify_ctx* ctx, uint64_t seed, uint32_t step,
                              uint32_t request_offset, int B, int k, double* out,
                              cudaStream_t stream) {
  if (!ctx || !out || B < 1 || k < 0 || k > sv::kMaxK) return SPEC_ERR_INVALID_ARG;
  if (!aligned(out, 8)) return SPEC_ERR_UNSUPPORTED;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  k_draws<<<grid_for(static_cast<int64_t>(B) * (k + 1) * 2), 256, 0, stream>>>(seed, step,
                                                                              request_offset, B, k, out);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_verify_set_mode(spec_verify_ctx* ctx, int mode) {
  if (!ctx || (mode != SPEC_MODE_DENSE && mode != SPEC_MODE_PREFIX && mode != SPEC_MODE_AUTO))
    return SPEC_ERR_INVALID_ARG;
  ctx->mode = mode;
  return SPEC_OK;
}

spec_status spec_verify_set_prefix_tail(spec_verify_ctx* ctx, int position) {
  if (!ctx || position < 0 || position > sv::kMaxK + 1) return SPEC_ERR_INVALID_ARG;
  ctx->tail_from = position;
  return SPEC_OK;
}

spec_status spec_verify_timing_enable(spec_verify_ctx* ctx, int class_mask) {
  if (!ctx || class_mask < 0 || class_mask >= (1 << kTimingClasses)) return SPEC_ERR_INVALID_ARG;
  ctx->timing_mask = static_cast<unsigned>(class_mask);
  for (int k = 0; k < kTimingClasses; ++k) ctx->n_timed[k] = 0;
  return SPEC_OK;
}

spec_status spec_verify_timing_read(spec_verify_ctx* ctx, int which, int* launches,
                                    double* total_ms) {
  if (!ctx || which < 0 || which >= kTimingClasses || !launches || !total_ms)
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  double tot = 0.0;
  const int n = ctx->n_timed[which];
  for (int r = 0; r < n; ++r) {
    if (cudaEventSynchronize(ctx->ev_stop[which][r]) != cudaSuccess) return SPEC_ERR_CUDA;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, ctx->ev_start[which][r], ctx->ev_stop[which][r]) != cudaSuccess)
      return SPEC_ERR_CUDA;
    tot += ms;
  }
  *launches = n;
  *total_ms = tot;
  return SPEC_OK;
}

spec_status spec_verify_last_counters(spec_verify_ctx* ctx, cudaStream_t stream, uint32_t out[6]) {
  if (!ctx || !out) return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SPEC_ERR_CUDA;
  sv::Counters h{};
  if (cudaMemcpy(&h, ctx->counters + (ctx->run_id & 1u), sizeof h, cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return SPEC_ERR_CUDA;
  out[0] = h.accept_slow;
  out[1] = h.refine_count;
  out[2] = h.sample_fast;
  out[3] = h.chunks_redone;
  out[4] = h.queue_error;
  out[5] = h.wait_fail;
  return SPEC_OK;
}


spec_status spec_shard_layout(int B, int k, int64_t V, spec_dtype dtype, int n_shards,
                              int64_t* bounds, size_t* block1_bytes, size_t* block2_bytes,
                              size_t* block3_bytes) {
  if (B < 1 || k < 0 || (dtype != SPEC_F32 && dtype != SPEC_BF16)) return SPEC_ERR_INVALID_ARG;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_geometry(V, dtype == SPEC_BF16, n_shards, &sb, &segl); st != SPEC_OK)
    return st;
  const ShardSizes z = shard_sizes(B, k, sb);
  if (bounds)
    for (int r = 0; r <= n_shards; ++r) bounds[r] = std::min<int64_t>(sb.seg_lo[r] * segl, V);
  if (block1_bytes) *block1_bytes = z.block1;
  if (block2_bytes) *block2_bytes = z.block2;
  if (block3_bytes) *block3_bytes = z.block3;
  return SPEC_OK;
}

spec_status spec_shard_stats(spec_verify_ctx* ctx, int rank, int n_shards, const void* target_shard,
                             const void* draft_shard, spec_dtype dtype, const int32_t* draft_tokens,
                             const int32_t* verify_len, const float* temperature,
                             const spec_conf_args* conf, int B, int k, int64_t V, void* block1,
                             cudaStream_t stream) {
  sv::RunParams p;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_params(ctx, rank, n_shards, target_shard, draft_shard, dtype,
                                    draft_tokens, verify_len, temperature, conf, B, k, V, &p, &sb,
                                    &segl);
      st != SPEC_OK)
    return st;
  if (!block1 || !aligned(block1, 256)) return SPEC_ERR_UNSUPPORTED;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  if (conf) launch_conf(ctx, conf, B, k, verify_len, ctx->conf_len, nullptr, stream);
  const ShardSizes z = shard_sizes(B, k, sb);
  const int nls = sb.seg_lo[rank + 1] - sb.seg_lo[rank];
  const int64_t ctas = static_cast<int64_t>(B) * (2 * k + 1) * nls;
  auto* recs = static_cast<sv::ShardRec*>(block1);
  const bool bf16 = dtype == SPEC_BF16;
  if (ctas > 0) {
    if (bf16) sv::k_shard_stats<true><<<static_cast<unsigned>(ctas), sv::kThreads, 0, stream>>>(p, sb.seg_lo[rank], nls, recs);
    else sv::k_shard_stats<false><<<static_cast<unsigned>(ctas), sv::kThreads, 0, stream>>>(p, sb.seg_lo[rank], nls, recs);
  }
  if (k > 0) {
    float* tl = reinterpret_cast<float*>(static_cast<char*>(block1) + z.tok_off);
    const int grid = grid_for(static_cast<int64_t>(B) * k);
    if (bf16) sv::k_shard_token_logits<true><<<grid, 256, 0, stream>>>(p, tl);
    else sv::k_shard_token_logits<false><<<grid, 256, 0, stream>>>(p, tl);
  }
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_shard_decide(spec_verify_ctx* ctx, int rank, int n_shards, const void* blocks1,
                              const void* target_shard, const void* draft_shard, spec_dtype dtype,
                              const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* temperature, const spec_conf_args* conf, int B, int k,
                              int64_t V, uint64_t seed, uint32_t step, uint32_t request_offset,
                              int32_t* out_accepted, int32_t* out_tokens, float* out_p,
                              float* out_q, uint32_t* out_status, void* block2,
                              cudaStream_t stream) {
  sv::RunParams p;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_params(ctx, rank, n_shards, target_shard, draft_shard, dtype,
                                    draft_tokens, verify_len, temperature, conf, B, k, V, &p, &sb,
                                    &segl);
      st != SPEC_OK)
    return st;
  if (!blocks1 || !block2 || !out_accepted || !out_tokens || !aligned(blocks1, 256) ||
      !aligned(block2, 16))
    return SPEC_ERR_INVALID_ARG;
  const int rows = 2 * k + 1;
  if (static_cast<int64_t>(B) * rows * p.n_segs >
      static_cast<int64_t>(ctx->max_batch) * (2 * ctx->max_k + 1) * ctx->max_chunks)
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  p.seed = seed;
  p.step = step;
  p.req_off = request_offset;
  p.out_acc = out_accepted;
  p.out_tok = out_tokens;
  p.out_p = out_p;
  p.out_q = out_q;
  p.out_status = out_status;
  const ShardSizes z = shard_sizes(B, k, sb);
  const bool bf16 = dtype == SPEC_BF16;
  sv::k_shard_gather_stats<<<grid_for(static_cast<int64_t>(B) * rows * p.n_segs), 256, 0, stream>>>(
      p, sb, static_cast<const char*>(blocks1), z.block1, z.tok_off, segl);
  if (bf16) sv::k_shard_decide<true><<<B, sv::kThreads, 0, stream>>>(p);
  else sv::k_shard_decide<false><<<B, sv::kThreads, 0, stream>>>(p);
  const int nls = sb.seg_lo[rank + 1] - sb.seg_lo[rank];
  if (nls > 0) {
    if (bf16) sv::k_shard_masses<true><<<B * nls, sv::kThreads, 0, stream>>>(p, sb.seg_lo[rank], nls);
    else sv::k_shard_masses<false><<<B * nls, sv::kThreads, 0, stream>>>(p, sb.seg_lo[rank], nls);
  }
  sv::k_shard_pack_masses<<<grid_for(static_cast<int64_t>(B) * z.nlc_max * sv::kSampleParts), 256, 0, stream>>>(
      p, p.c_lo, p.c_hi - p.c_lo, z.nlc_max, static_cast<sv::SampleChunk*>(block2));
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_shard_locate(spec_verify_ctx* ctx, int rank, int n_shards, const void* blocks2,
                              const void* target_shard, const void* draft_shard, spec_dtype dtype,
                              const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* temperature, const spec_conf_args* conf, int B, int k,
                              int64_t V, int32_t* out_token_votes, cudaStream_t stream) {
  sv::RunParams p;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_params(ctx, rank, n_shards, target_shard, draft_shard, dtype,
                                    draft_tokens, verify_len, temperature, conf, B, k, V, &p, &sb,
                                    &segl);
      st != SPEC_OK)
    return st;
  if (!blocks2 || !out_token_votes || !aligned(blocks2, 16) || !aligned(out_token_votes, 4))
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  const ShardSizes z = shard_sizes(B, k, sb);
  p.shard_tok = out_token_votes;
  sv::k_shard_unpack_masses<<<grid_for(static_cast<int64_t>(B) * p.n_chunks * sv::kSampleParts), 256, 0, stream>>>(
      p, sb, static_cast<const sv::SampleChunk*>(blocks2), z.nlc_max);
  if (dtype == SPEC_BF16) sv::k_shard_locate<true><<<B, sv::kThreads, 0, stream>>>(p);
  else sv::k_shard_locate<false><<<B, sv::kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_shard_finish(spec_verify_ctx* ctx, const int32_t* token_votes_max, int B, int k,
                              int32_t* out_tokens, int32_t* out_redo, cudaStream_t stream) {
  if (!ctx || B < 1 || B > ctx->max_batch || k < 0 || k > ctx->max_k || !token_votes_max ||
      !out_tokens || !out_redo)
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  sv::RunParams p{};
  p.B = B;
  p.k = k;
  p.jobs = ctx->jobs;
  p.fallback = ctx->fallback;
  p.refine_list = ctx->refine_list;
  p.out_tok = out_tokens;
  sv::k_shard_finish<<<grid_for(B), 256, 0, stream>>>(p, token_votes_max);
  if (cudaMemcpyAsync(out_redo, ctx->fallback, static_cast<size_t>(B) * sizeof(int32_t),
                      cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return SPEC_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_shard_refine_partials(spec_verify_ctx* ctx, int rank, int n_shards,
                                       const void* target_shard, const void* draft_shard,
                                       spec_dtype dtype, const int32_t* draft_tokens,
                                       const int32_t* verify_len, const float* temperature,
                                       const spec_conf_args* conf, int B, int k, int64_t V,
                                       void* block3, cudaStream_t stream) {
  sv::RunParams p;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_params(ctx, rank, n_shards, target_shard, draft_shard, dtype,
                                    draft_tokens, verify_len, temperature, conf, B, k, V, &p, &sb,
                                    &segl);
      st != SPEC_OK)
    return st;
  if (!block3 || !aligned(block3, 16)) return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  const ShardSizes z = shard_sizes(B, k, sb);
  const int sub_lo = p.c_lo * sv::kSubsPerChunk;
  const int nsub = (p.c_hi - p.c_lo) * sv::kSubsPerChunk;
  if (nsub > 0) {
    const int grid = refine_grid(ctx, B, nsub);
    if (dtype == SPEC_BF16) sv::k_shard_refine_partials<true><<<grid, sv::kThreads, 0, stream>>>(p, sub_lo, nsub);
    else sv::k_shard_refine_partials<false><<<grid, sv::kThreads, 0, stream>>>(p, sub_lo, nsub);
  }
  sv::k_shard_pack_refine<<<grid_for(static_cast<int64_t>(B) * z.nsub_max), 256, 0, stream>>>(
      p, sub_lo, nsub, z.nsub_max, static_cast<sv::RefRec*>(block3));
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_shard_refine_locate(spec_verify_ctx* ctx, int rank, int n_shards,
                                     const void* blocks3, const void* target_shard,
                                     const void* draft_shard, spec_dtype dtype,
                                     const int32_t* draft_tokens, const int32_t* verify_len,
                                     const float* temperature, const spec_conf_args* conf, int B,
                                     int k, int64_t V, int32_t* token_votes, cudaStream_t stream) {
  sv::RunParams p;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_params(ctx, rank, n_shards, target_shard, draft_shard, dtype,
                                    draft_tokens, verify_len, temperature, conf, B, k, V, &p, &sb,
                                    &segl);
      st != SPEC_OK)
    return st;
  if (!blocks3 || !token_votes || !aligned(blocks3, 16) || !aligned(token_votes, 4))
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  const ShardSizes z = shard_sizes(B, k, sb);
  p.shard_tok = token_votes;
  sv::k_shard_unpack_refine<<<grid_for(static_cast<int64_t>(B) * p.n_chunks * sv::kSubsPerChunk), 256, 0, stream>>>(
      p, sb, static_cast<const sv::RefRec*>(blocks3), z.nsub_max);
  if (dtype == SPEC_BF16) sv::k_shard_refine_locate<true><<<B, sv::kThreads, 0, stream>>>(p);
  else sv::k_shard_refine_locate<false><<<B, sv::kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status spec_shard_refine_finish(spec_verify_ctx* ctx, const int32_t* token_votes_max, int B,
                                     int k, int32_t* out_tokens, int32_t* out_redo,
                                     cudaStream_t stream) {
  if (!ctx || B < 1 || B > ctx->max_batch || k < 0 || k > ctx->max_k || !token_votes_max ||
      !out_tokens || !out_redo)
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  sv::RunParams p{};
  p.B = B;
  p.k = k;
  p.jobs = ctx->jobs;
  p.fallback = ctx->fallback;
  p.out_tok = out_tokens;
  sv::k_shard_refine_finish<<<grid_for(B), 256, 0, stream>>>(p, token_votes_max);
  if (cudaMemcpyAsync(out_redo, ctx->fallback, static_cast<size_t>(B) * sizeof(int32_t),
                      cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return SPEC_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}
}  // extern "C"

#include "lmhead_host.cuh"
