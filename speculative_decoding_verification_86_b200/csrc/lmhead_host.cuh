// Host side of the LM-head entry points (included at the end of
// spec_verify.cu, whose argument checks and launch helpers it uses): the
// context's buffers, the TMA tensor maps, and the launch sequence of the fused
// verification -- statistics GEMM, part merge, accept chain, sampled rows,
// then the vocabulary-parallel protocol's sample and refinement phases run
// with a single shard.
#include <cudaTypedefs.h>

#include "lmhead.cuh"

struct spec_lmhead_ctx {
  spec_verify_ctx* vctx = nullptr;
  int max_hidden = 0;
  int max_rows = 0;  // max_batch * (2 max_k + 1)
  int max_parts = 0;
  void* ws = nullptr;
  sv::LmPart* parts = nullptr;  // [max_rows, max_parts]
  float* rows = nullptr;        // [max_rows, max_vocab] fp32: logits of the sampled rows
  uint4* hc = nullptr;          // [max_rows, max_hidden] bf16: their hidden states
  int* src = nullptr;           // [max_rows]
  int64_t* dst = nullptr;       // [max_rows]
  int* count = nullptr;
  int* rest_count = nullptr;  // rows of the second statistics pass (prefix-ordered verify)
  int* state = nullptr;       // [max_batch]: each request's state after its position 0
  int32_t* votes = nullptr;     // [max_batch]
  unsigned* error = nullptr;
  int cta_pairs = 2;            // spec_lmhead_set_cta_pairs: 0 never, 1 always, 2 row GEMM only
};

namespace {
// CTAs per MMA of the statistics GEMM and of the row-writing GEMM.
int stats_cta_group(const spec_lmhead_ctx* lm) { return lm->cta_pairs == 1 ? 2 : 1; }
int rows_cta_group(const spec_lmhead_ctx* lm) { return lm->cta_pairs >= 1 ? 2 : 1; }
}  // namespace

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cudaGetLastError();
  });
  return fn;
}

// Row-major bf16 matrix [rows, H] as 2-D tiles of box_rows x 64 (128 bytes,
// the 128-byte swizzle); out-of-range rows and columns read as zero.  Rows are
// row_stride elements apart (0: H; a multiple of 8, so 16-byte aligned).
bool bf16_tile_map(CUtensorMap* m, const void* base, int64_t rows, int H, int box_rows,
                   int64_t row_stride = 0) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc || rows < 1) return false;
  if (row_stride == 0) row_stride = H;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(sv::kLmBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int lm_tiles(int64_t V) { return static_cast<int>((V + sv::kLmBN - 1) / sv::kLmBN); }
int lm_parts(int64_t V, int part_tiles) { return (lm_tiles(V) + part_tiles - 1) / part_tiles; }

// Smallest statistics part the kernel is given (largest record count).
constexpr int kLmMinPartTiles = 2;

// Work-unit width of the statistics GEMM: the largest of 16, 8, 4, 2 tiles
// whose unit count comes within 2% of filling its last wave as well as the
// best of them (a wider unit writes fewer records).
int lm_stats_part_tiles(int n_mt, int64_t V, int grid) {
  double best = 0.0;
  double eff[4];
  const int cand[4] = {16, 8, 4, kLmMinPartTiles};
  for (int q = 0; q < 4; ++q) {
    const int64_t units = static_cast<int64_t>(n_mt) * lm_parts(V, cand[q]);
    const int64_t waves = (units + grid - 1) / grid;
    eff[q] = static_cast<double>(units) / static_cast<double>(waves * grid);
    best = std::max(best, eff[q]);
  }
  for (int q = 0; q < 4; ++q)
    if (eff[q] >= best - 0.02) return cand[q];
  return kLmMinPartTiles;
}

// M tiles of the GEMM over rows0 (+ rows1) rows with `cg` CTAs per MMA.
int lm_mtiles(int rows0, int rows1, int cg) {
  const int r = sv::kLmBM * cg;
  return (rows0 + r - 1) / r + (rows1 + r - 1) / r;
}

// Launch k_lmhead over n_mt M tiles x the vocabulary in units of p.part_tiles
// tiles: one CTA per SM, or clusters of two CTAs (one pair per TPC).
spec_status lm_launch(const spec_lmhead_ctx* lm, int cg, const CUtensorMap& ma0,
                      const CUtensorMap& ma1, const void* head, int H, int64_t V,
                      const sv::LmParams& p, int n_mt, int cls, cudaStream_t stream) {
  CUtensorMap mw;
  if (!bf16_tile_map(&mw, head, V, H, sv::kLmBN / cg)) return SPEC_ERR_UNSUPPORTED;
  const int64_t units = static_cast<int64_t>(n_mt) * lm_parts(V, p.part_tiles);
  const int groups = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>(units, lm->vctx->num_sms / cg)));
  timing_mark(lm->vctx, cls, true, stream);
  if (cg == 1) {
    sv::k_lmhead<1><<<groups, sv::kLmThreads, sv::LmGeo<1>::kSmemBytes, stream>>>(ma0, ma1, mw, p);
  } else {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * groups);
    cfg.blockDim = dim3(sv::kLmThreads);
    cfg.dynamicSmemBytes = sv::LmGeo<2>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, sv::k_lmhead<2>, ma0, ma1, mw, p) != cudaSuccess) {
      timing_mark(lm->vctx, cls, false, stream);
      return SPEC_ERR_CUDA;
    }
  }
  timing_mark(lm->vctx, cls, false, stream);
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

spec_status lm_check(const spec_lmhead_ctx* lm, int H, int64_t V, const void* head) {
  if (!lm || !head || H < 8 || H > lm->max_hidden || V < 1 || V > lm->vctx->max_vocab)
    return SPEC_ERR_INVALID_ARG;
  if (H % 8 != 0 || V % 4 != 0 || !aligned(head, 16)) return SPEC_ERR_UNSUPPORTED;
  return SPEC_OK;
}

}  // namespace

extern "C" {

spec_status spec_lmhead_init(spec_lmhead_ctx** out, spec_verify_ctx* vctx, int max_hidden) {
  if (!out) return SPEC_ERR_INVALID_ARG;
  *out = nullptr;
  if (!vctx || max_hidden < 8 || max_hidden > 65536 || max_hidden % 8 != 0)
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(vctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  if (!tensor_map_encoder()) return SPEC_ERR_UNSUPPORTED;
  auto* lm = new (std::nothrow) spec_lmhead_ctx();
  if (!lm) return SPEC_ERR_NOMEM;
  lm->vctx = vctx;
  lm->max_hidden = max_hidden;
  lm->max_rows = vctx->max_batch * (2 * vctx->max_k + 1);
  lm->max_parts = lm_parts(vctx->max_vocab, kLmMinPartTiles);
  const size_t R = static_cast<size_t>(lm->max_rows);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t o_parts = take(R * lm->max_parts * sizeof(sv::LmPart));
  const size_t o_rows = take(R * static_cast<size_t>(vctx->max_vocab) * sizeof(float));
  const size_t o_hc = take(R * static_cast<size_t>(max_hidden) * 2);
  const size_t o_src = take(R * sizeof(int));
  const size_t o_dst = take(R * sizeof(int64_t));
  const size_t o_cnt = take(sizeof(int));
  const size_t o_rcnt = take(sizeof(int));
  const size_t o_state = take(static_cast<size_t>(vctx->max_batch) * sizeof(int));
  const size_t o_votes = take(static_cast<size_t>(vctx->max_batch) * sizeof(int32_t));
  const size_t o_err = take(sizeof(unsigned));
  if (cudaMalloc(&lm->ws, off) != cudaSuccess) {
    cudaGetLastError();
    delete lm;
    return SPEC_ERR_NOMEM;
  }
  char* b = static_cast<char*>(lm->ws);
  lm->parts = reinterpret_cast<sv::LmPart*>(b + o_parts);
  lm->rows = reinterpret_cast<float*>(b + o_rows);
  lm->hc = reinterpret_cast<uint4*>(b + o_hc);
  lm->src = reinterpret_cast<int*>(b + o_src);
  lm->dst = reinterpret_cast<int64_t*>(b + o_dst);
  lm->count = reinterpret_cast<int*>(b + o_cnt);
  lm->rest_count = reinterpret_cast<int*>(b + o_rcnt);
  lm->state = reinterpret_cast<int*>(b + o_state);
  lm->votes = reinterpret_cast<int32_t*>(b + o_votes);
  lm->error = reinterpret_cast<unsigned*>(b + o_err);
  if (cudaMemset(lm->ws, 0, off) != cudaSuccess ||
      cudaFuncSetAttribute(sv::k_lmhead<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sv::LmGeo<1>::kSmemBytes)) != cudaSuccess ||
      cudaFuncSetAttribute(sv::k_lmhead<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sv::LmGeo<2>::kSmemBytes)) != cudaSuccess) {
    cudaFree(lm->ws);
    delete lm;
    return SPEC_ERR_CUDA;
  }
  *out = lm;
  return SPEC_OK;
}

spec_status spec_lmhead_destroy(spec_lmhead_ctx* lm) {
  if (!lm) return SPEC_OK;
  DeviceGuard g(lm->vctx->device);
  cudaDeviceSynchronize();
  cudaFree(lm->ws);
  delete lm;
  return SPEC_OK;
}

spec_status spec_lmhead_set_cta_pairs(spec_lmhead_ctx* lm, int pairs) {
  if (!lm || pairs < 0 || pairs > 2) return SPEC_ERR_INVALID_ARG;
  lm->cta_pairs = pairs;
  return SPEC_OK;
}

spec_status spec_lmhead_errors(spec_lmhead_ctx* lm, uint32_t* out) {
  if (!lm || !out) return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(lm->vctx->device);
  if (cudaDeviceSynchronize() != cudaSuccess) return SPEC_ERR_CUDA;
  unsigned h = 0;
  if (cudaMemcpy(&h, lm->error, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return SPEC_ERR_CUDA;
  *out = h;
  return SPEC_OK;
}

spec_status spec_lmhead_logits(spec_lmhead_ctx* lm, const void* hidden, int rows, const void* head,
                               int H, int64_t V, float* out_logits, cudaStream_t stream) {
  if (spec_status st = lm_check(lm, H, V, head); st != SPEC_OK) return st;
  if (rows < 1 || !hidden || !out_logits) return SPEC_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(out_logits, 16)) return SPEC_ERR_UNSUPPORTED;
  DeviceGuard g(lm->vctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  CUtensorMap ma;
  if (!bf16_tile_map(&ma, hidden, rows, H, sv::kLmBM)) return SPEC_ERR_UNSUPPORTED;
  sv::LmParams p{};
  p.mode = sv::kLmModeRows;
  p.H = H;
  p.V = V;
  p.rows0 = rows;
  p.out = out_logits;
  p.error = lm->error;
  p.part_tiles = 1;  // no records: single-tile units balance the waves best
  const int cg = rows_cta_group(lm);
  return lm_launch(lm, cg, ma, ma, head, H, V, p, lm_mtiles(rows, 0, cg), kClassLmRows, stream);
}

spec_status spec_lmhead_verify(spec_lmhead_ctx* lm, const void* hidden_target,
                               const void* hidden_draft, const void* head, int H,
                               const int32_t* draft_tokens, const int32_t* verify_len,
                               const float* temperature, const spec_conf_args* conf, int B, int k,
                               int64_t V, uint64_t seed, uint32_t step, uint32_t request_offset,
                               int32_t* out_accepted, int32_t* out_tokens, float* out_p,
                               float* out_q, uint32_t* out_status, int32_t* out_redo,
                               cudaStream_t stream) {
  if (spec_status st = lm_check(lm, H, V, head); st != SPEC_OK) return st;
  spec_verify_ctx* ctx = lm->vctx;
  if (B < 1 || B > ctx->max_batch || k < 0 || k > ctx->max_k || !hidden_target || !out_accepted ||
      !out_tokens || !out_redo || (k > 0 && !draft_tokens))
    return SPEC_ERR_INVALID_ARG;
  if (!aligned(hidden_target, 16) || (hidden_draft && !aligned(hidden_draft, 16)))
    return SPEC_ERR_UNSUPPORTED;
  const int rows0 = B * (k + 1), rows1 = hidden_draft ? B * k : 0;
  float* rows_t = lm->rows;
  float* rows_d = lm->rows + static_cast<int64_t>(rows0) * V;
  sv::RunParams p;
  sv::ShardBounds sb;
  int64_t segl = 0;
  if (spec_status st = shard_params(ctx, 0, 1, rows_t, hidden_draft ? rows_d : nullptr, SPEC_F32,
                                    draft_tokens, verify_len, temperature, conf, B, k, V, &p, &sb,
                                    &segl);
      st != SPEC_OK)
    return st;
  const int rows = 2 * k + 1;
  if (static_cast<int64_t>(B) * rows * p.n_segs >
      static_cast<int64_t>(ctx->max_batch) * (2 * ctx->max_k + 1) * ctx->max_chunks)
    return SPEC_ERR_INVALID_ARG;
  DeviceGuard g(ctx->device);
  if (!g.ok) return SPEC_ERR_CUDA;
  cudaGetLastError();
  CUtensorMap mc;  // the gathered hidden rows
  if (!bf16_tile_map(&mc, lm->hc, static_cast<int64_t>(B) * rows, H, sv::kLmBM))
    return SPEC_ERR_UNSUPPORTED;
  p.rows_whole = 1;  // sampled rows are materialised in full before the sample phases
  p.seed = seed;
  p.step = step;
  p.req_off = request_offset;
  p.out_acc = out_accepted;
  p.out_tok = out_tokens;
  p.out_p = out_p;
  p.out_q = out_q;
  p.out_status = out_status;
  const int cg1 = stats_cta_group(lm), cg2 = rows_cta_group(lm);
  if (conf) launch_conf(ctx, conf, B, k, verify_len, ctx->conf_len, nullptr, stream);
  if (k > 0 && cudaMemsetAsync(ctx->tok_logits, 0, static_cast<size_t>(B) * k * 2 * sizeof(float),
                               stream) != cudaSuccess)
    return SPEC_ERR_CUDA;
  if (cudaMemsetAsync(lm->count, 0, sizeof(int), stream) != cudaSuccess ||
      cudaMemsetAsync(lm->rest_count, 0, sizeof(int), stream) != cudaSuccess)
    return SPEC_ERR_CUDA;

  // Prefix order, as in the verification of logits: position 0 first, then
  // the other rows of the requests that accepted it (most requests stop at
  // position 0, so most rows are never computed).
  //
  // 1. position 0 of every request: the statistics of its two rows, read in
  //    place (rows (k+1) H and k H elements apart); their logits are written
  sv::LmParams lp{};
  lp.mode = sv::kLmModeStats;
  lp.H = H;
  lp.V = V;
  lp.B = B;
  lp.k = k;
  lp.tokens = draft_tokens;
  lp.temp = temperature;
  lp.parts = lm->parts;
  lp.tok_logits = ctx->tok_logits;
  lp.error = lm->error;
  {
    const int r1 = (rows1 > 0 && k > 0) ? B : 0;
    CUtensorMap mp0, mp1;
    if (!bf16_tile_map(&mp0, hidden_target, B, H, sv::kLmBM, static_cast<int64_t>(k + 1) * H) ||
        (r1 > 0 && !bf16_tile_map(&mp1, hidden_draft, B, H, sv::kLmBM, static_cast<int64_t>(k) * H)))
      return SPEC_ERR_UNSUPPORTED;
    if (r1 == 0) mp1 = mp0;
    const int n_mt = lm_mtiles(B, r1, cg1);
    const int part_tiles = lm_stats_part_tiles(n_mt, V, ctx->num_sms / cg1);
    const int n_parts = lm_parts(V, part_tiles);
    lp.rows0 = B;
    lp.rows1 = r1;
    lp.pos0 = 1;
    lp.n_parts = n_parts;
    lp.part_tiles = part_tiles;
    lp.out = lm->rows;  // position-0 rows: the rows most requests sample from
    if (spec_status st = lm_launch(lm, cg1, mp0, mp1, head, H, V, lp, n_mt, kClassLmStats, stream);
        st != SPEC_OK)
      return st;
    sv::k_lm_combine<<<grid_for(static_cast<int64_t>(B) * rows * p.n_segs), 256, 0, stream>>>(
        p, lm->parts, n_parts, sv::kLmSegTiles / part_tiles, rows0, 1);
  }
  sv::k_lm_decide0<<<B, sv::kThreads, 0, stream>>>(p, lm->state, lm->rest_count, lm->src);

  // 2. the other rows of the requests that accepted position 0: gathered, then
  //    one statistics pass over them (its row count is on the device), and
  //    their chains walked from position 1
  if (k > 0) {
    const int max_rest = B * 2 * k;
    sv::k_lm_gather<<<grid_for(static_cast<int64_t>(max_rest) * (H / 8)), 256, 0, stream>>>(
        lm->rest_count, lm->src, static_cast<const uint4*>(hidden_target),
        static_cast<const uint4*>(hidden_draft ? hidden_draft : hidden_target), rows0, H, max_rest,
        lm->hc);
    const int n_mt = lm_mtiles(max_rest, 0, cg1);
    const int part_tiles = lm_stats_part_tiles(n_mt, V, ctx->num_sms / cg1);
    const int n_parts = lm_parts(V, part_tiles);
    sv::LmParams lq = lp;
    lq.rows0 = max_rest;
    lq.rows1 = 0;
    lq.rows_dev = lm->rest_count;
    lq.pos0 = 0;
    lq.row_map = lm->src;
    lq.n_parts = n_parts;
    lq.part_tiles = part_tiles;
    lq.out = nullptr;  // no position-0 rows in this pass
    if (spec_status st = lm_launch(lm, cg1, mc, mc, head, H, V, lq, n_mt, kClassLmStats, stream);
        st != SPEC_OK)
      return st;
    sv::k_lm_combine<<<grid_for(static_cast<int64_t>(B) * rows * p.n_segs), 256, 0, stream>>>(
        p, lm->parts, n_parts, sv::kLmSegTiles / part_tiles, rows0, 2);
    sv::k_lm_decide_rest<<<B, sv::kThreads, 0, stream>>>(p, lm->state);
  }

  // 3. logits of the rows each request samples from
  sv::k_lm_rowlist<<<grid_for(B), 256, 0, stream>>>(p, lm->count, lm->src, lm->dst);
  sv::k_lm_gather<<<grid_for(static_cast<int64_t>(2) * B * (H / 8)), 256, 0, stream>>>(
      lm->count, lm->src, static_cast<const uint4*>(hidden_target),
      static_cast<const uint4*>(hidden_draft ? hidden_draft : hidden_target), rows0, H, B * rows,
      lm->hc);
  sv::LmParams lr{};
  lr.mode = sv::kLmModeRows;
  lr.H = H;
  lr.V = V;
  lr.rows0 = 2 * B;  // at most a row pair per request
  lr.rows_dev = lm->count;
  lr.dst = lm->dst;
  lr.out = lm->rows;
  lr.error = lm->error;
  lr.part_tiles = 1;
  if (spec_status st = lm_launch(lm, cg2, mc, mc, head, H, V, lr, lm_mtiles(2 * B, 0, cg2),
                                 kClassLmRows, stream);
      st != SPEC_OK)
    return st;

  // 4. sample: chunk masses, locate and certify, fp64 refinement where needed
  sv::k_shard_masses<false><<<B * p.n_segs, sv::kThreads, 0, stream>>>(p, 0, p.n_segs);
  p.shard_tok = lm->votes;
  sv::k_shard_locate<false><<<B, sv::kThreads, 0, stream>>>(p);
  sv::k_shard_finish<<<grid_for(B), 256, 0, stream>>>(p, lm->votes);
  const int nsub = p.n_chunks * sv::kSubsPerChunk;
  sv::k_shard_refine_partials<false><<<refine_grid(ctx, B, nsub), sv::kThreads, 0, stream>>>(p, 0, nsub);
  sv::k_shard_refine_locate<false><<<B, sv::kThreads, 0, stream>>>(p);
  sv::k_shard_refine_finish<<<grid_for(B), 256, 0, stream>>>(p, lm->votes);
  if (cudaMemcpyAsync(out_redo, ctx->fallback, static_cast<size_t>(B) * sizeof(int32_t),
                      cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return SPEC_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SPEC_OK : SPEC_ERR_CUDA;
}

}  // extern "C"
