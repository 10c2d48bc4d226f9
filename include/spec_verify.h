/*
 * spec_verify.h -- C ABI of the B200 (sm_100a) speculative-decoding
 * verification library (libspecverify.so).
 *
 * What the library computes.  A drafter proposes a block of k tokens per
 * request; the target model has scored the whole block in one pass and its
 * logits are given for the k drafted positions plus one bonus position.
 * Verification walks each request's block left to right
 * ("Speculative decoding becomes standard: DSpark and multi-token drafters",
 * section "Why draft-and-verify does not change the output"):
 *   - stochastic (T > 0): accept drafted token x with probability
 *     min(1, p(x)/q(x)), p = softmax(target/T), q = softmax(draft/T); at the
 *     first rejection emit a sample from the residual
 *     norm(max(0, p - q)) and drop the rest of the block; if every verified
 *     position is accepted emit a bonus token drawn from the target's next row;
 *   - greedy (T == 0): keep x while it is the target's argmax (lowest index on
 *     ties); at the first disagreement emit the argmax; if all agree emit the
 *     argmax of the next row.
 * The confidence head (same page, section "What DSpark adds") maps each
 * position's hidden state to s_j = sigmoid(w . h_j + b), the estimated chance
 * that position j passes once all earlier positions have; the prefix product of these
 * probabilities, compared with a threshold, truncates the verified length.
 *
 * Readings where the pages are silent (all shared with the CPU oracle):
 *   accept iff u * q(x) < p(x) with u uniform on [0, 1) (53 bits); inverse-CDF
 *   sampling picks the smallest index whose running sum exceeds u * total
 *   (index order), falling back to the largest index with positive weight; a
 *   residual with total mass below 1e-12 is replaced by p; random draws are
 *   Philox4x32-10 with key = (seed low, seed high) and counter =
 *   (2 * position + draw, request_offset + request, step, 0), draw 0 for the
 *   accept test and draw 1 for the residual/bonus sample.  -inf logits mask a
 *   token; NaN or +inf in a row the chain reads, a row whose max is -inf, or a
 *   drafted token outside [0, V) fails that request.  Errors are found in
 *   chain order: rows and tokens past the first rejection are never judged.
 *
 * Conventions for every entry point:
 *   - Array arguments are DEVICE pointers on the context's device unless the
 *     entry point says "host".  Logit rows are contiguous ([B, rows, V]
 *     row-major); base pointers of logits must be 16-byte aligned and
 *     V * sizeof(element) a multiple of 16 bytes, else SPEC_ERR_UNSUPPORTED.
 *     Integer and fp32 side arrays must be 4-byte aligned.
 *   - The caller owns every input/output buffer and the stream.  The context
 *     owns its device workspace (allocated by spec_verify_init, freed by
 *     spec_verify_destroy).  One context per concurrently used stream.
 *   - Calls are asynchronous on `stream` (no host synchronisation) except the
 *     "_host" entry point.  The return value covers argument validation and
 *     launch errors only; per-request failures found on the device are
 *     reported through out_status (bits below) and out_accepted = -1.
 *   - Outputs are a pure function of (inputs, seed, step, request_offset):
 *     every reduction merges in a fixed order.
 */
#ifndef SPEC_VERIFY_H
#define SPEC_VERIFY_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPEC_OK = 0,
    SPEC_ERR_INVALID_ARG = 1,   /* bad size, NULL where required, ctx too small */
    SPEC_ERR_UNSUPPORTED = 2,   /* alignment / dtype / size the kernels do not take */
    SPEC_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    SPEC_ERR_NOMEM = 4,         /* device or host allocation failed */
    SPEC_ERR_DEVICE_STATUS = 5, /* (host entry point) a request failed on the device */
    SPEC_ERR_TIMEOUT = 6        /* reserved: a bounded device wait gave up */
} spec_status;

typedef enum { SPEC_F32 = 0, SPEC_BF16 = 1 } spec_dtype;

/* Order in which the statistics pass reads a request's rows.  All give the
 * same outputs, bit for bit:
 *   SPEC_MODE_PREFIX: position j+1's rows are read only once position j was
 *     accepted (the block ends at its first rejected position), so rows past
 *     the first rejection are never touched -- up to the dense tail
 *     (spec_verify_set_prefix_tail): from that position on, a request's
 *     remaining rows are read together;
 *   SPEC_MODE_DENSE: every verified position's target and draft rows are
 *     reduced, then the chain is walked;
 *   SPEC_MODE_AUTO (default): dense when the B * (2k + 1) rows, cut into
 *     segments of 32768 bf16 or 16384 fp32 logits, make at most one segment
 *     per CTA of the kernel's grid (the extra rows then cost no time and the
 *     waits between positions go), prefix otherwise.  spec_verify_greedy
 *     always uses the prefix order. */
typedef enum { SPEC_MODE_DENSE = 0, SPEC_MODE_PREFIX = 1, SPEC_MODE_AUTO = 2 } spec_mode;

/* Per-request device status bits (out_status[i]); 0 means success. */
#define SPEC_DEV_BAD_TOKEN 1u       /* a drafted token the chain reached is outside [0, V) */
#define SPEC_DEV_NONFINITE 2u       /* NaN/+inf in a row the chain read, or a row of all -inf */
#define SPEC_DEV_BAD_TEMPERATURE 4u /* temperature negative, NaN, inf, in (0, 2^-100), or
                                       T > 0 with L_i > 0 but no draft logits */
#define SPEC_DEV_INTERNAL 16u       /* internal consistency check failed (should not occur) */

typedef struct spec_verify_ctx spec_verify_ctx;

/* Confidence-head arguments ("What DSpark adds"): survival s_j =
 * sigmoid(w . hidden[i, j, :] + bias) for j < kb; the budget of request i is the
 * number of leading positions whose prefix product P_ij = prod_{j'<=j} s_ij' >=
 * threshold.
 * total_budget > 0 adds the batch-wide, load-aware limit (same section: how much
 * is verified follows the predicted survival and the load): of the positions
 * left by verify_len and the threshold, only the total_budget ones with the
 * largest P_ij are verified, ties going to the lower request index and then to
 * the lower position; P_ij never grows with j, so each request keeps a leading
 * run.  sum_i L_i = min(total_budget, positions left).  <= 0: no such limit. */
typedef struct {
    const void* hidden; /* device, [B, kb, H] bf16 drafter hidden states */
    const void* w;      /* device, [H] bf16 projection */
    float bias;
    int kb;             /* positions scored by the head (1..16) */
    int H;              /* hidden width (1..65536) */
    float threshold;
    int64_t total_budget; /* batch-wide verify budget (positions); <= 0: none */
} spec_conf_args;

/* Create a context on `device` with workspace for batches up to max_batch
 * (<= 65535) requests, blocks up to max_k drafted tokens (max_k <= 16) and vocabularies
 * up to max_vocab (<= 2097152).  The current device is restored on return. */
spec_status spec_verify_init(spec_verify_ctx** ctx, int device, int max_batch, int max_k,
                             int64_t max_vocab);

/* Free the context and its workspace (synchronises its device first). NULL is a no-op. */
spec_status spec_verify_destroy(spec_verify_ctx* ctx);

/* Select the statistics order for later runs on this context (spec_mode). */
spec_status spec_verify_set_mode(spec_verify_ctx* ctx, int mode);

/* Prefix order's dense tail, for later runs on this context: once a request
 * has accepted positions 0 .. position-1, the rows of all its remaining
 * positions (target rows position..L, draft rows position..L-1) are read at
 * once and its chain is walked from there, as in the dense order.  A request
 * that accepts many positions then waits on fewer dependent statistics passes;
 * the price is reading the rows of that tail past its first rejection.  The
 * outputs do not depend on it.  `position` in [1, 17]; a value above the run's
 * k reads every position separately; 0 (the default) chooses per run: 2 when
 * the batch's rows (2k + 1 per request, k + 1 without draft logits), cut into
 * segments of 32768 bf16 or 16384 fp32 logits, make at most 16 waves of the
 * kernel's grid, else no tail.  SPEC_ERR_INVALID_ARG for a NULL context or a
 * position outside [0, 17]. */
spec_status spec_verify_set_prefix_tail(spec_verify_ctx* ctx, int position);

/* Stochastic/mixed verification of B requests.
 *   target_logits [B, k+1, V]: row j scores drafted position j; row k is the bonus row.
 *   draft_logits  [B, k, V] (same dtype), or NULL when every temperature is 0.
 *   draft_tokens  [B, k] int32.
 *   verify_len    [B] int32 positions to verify per request (clamped to [0, k]), or NULL => k.
 *   temperature   [B] fp32 per request (0 => greedy), or NULL => 1.0 for all.
 *   conf          NULL, or a confidence head; then L_i = min(verify_len_i, budget_i),
 *                 further limited by conf->total_budget (see spec_verify_lengths).
 *   seed, step, request_offset select the random draws (see counter layout above).
 * Outputs:
 *   out_accepted [B] int32: n_i = accepted drafted tokens (-1 if the request failed).
 *   out_tokens   [B, k+1] int32: x_0..x_{n-1}, then the correction or bonus token
 *                at index n; -1 after it.
 *   out_p, out_q [B, k] fp32 or NULL: p_j(x_j), q_j(x_j) for the positions the
 *                chain evaluated (j <= n_i, j < L_i, T_i > 0); -1 elsewhere.
 *   out_status   [B] uint32 or NULL: SPEC_DEV_* bits.
 * Limits: 1 <= V <= max_vocab, 0 <= k <= max_k, 0 <= B <= max_batch (B == 0 is a no-op). */
spec_status spec_verify_run(spec_verify_ctx* ctx, const void* target_logits,
                            const void* draft_logits, spec_dtype dtype,
                            const int32_t* draft_tokens, const int32_t* verify_len,
                            const float* temperature, const spec_conf_args* conf, int B, int k,
                            int64_t V, uint64_t seed, uint32_t step, uint32_t request_offset,
                            int32_t* out_accepted, int32_t* out_tokens, float* out_p,
                            float* out_q, uint32_t* out_status, cudaStream_t stream);

/* Test hook: spec_verify_run with the random draws replaced by `uniforms`
 * (device, [B, k+1, 2] fp64; entry [i, j, d] is draw d of position j), so that
 * tests can put draws exactly on decision boundaries. */
spec_status spec_verify_run_with_uniforms(
    spec_verify_ctx* ctx, const void* target_logits, const void* draft_logits, spec_dtype dtype,
    const int32_t* draft_tokens, const int32_t* verify_len, const float* temperature,
    const spec_conf_args* conf, int B, int k, int64_t V, const double* uniforms,
    int32_t* out_accepted, int32_t* out_tokens, float* out_p, float* out_q,
    uint32_t* out_status, cudaStream_t stream);

/* Test hook: the random draws spec_verify_run makes, written to `out`
 * (device, [B, k+1, 2] fp64; entry [i, j, d] = U(seed, request_offset + i,
 * position j, draw d, step)), so tests can compare the device generator with
 * an independent one.  Asynchronous on `stream`. */
spec_status spec_verify_draws(spec_verify_ctx* ctx, uint64_t seed, uint32_t step,
                              uint32_t request_offset, int B, int k, double* out,
                              cudaStream_t stream);

/* Greedy (temperature 0) verification: target_logits [B, k+1, V], draft_tokens
 * [B, k]; no draft logits are read.  Outputs as in spec_verify_run. */
spec_status spec_verify_greedy(spec_verify_ctx* ctx, const void* target_logits, spec_dtype dtype,
                               const int32_t* draft_tokens, const int32_t* verify_len, int B,
                               int k, int64_t V, int32_t* out_accepted, int32_t* out_tokens,
                               uint32_t* out_status, cudaStream_t stream);

/* Greedy verification that allocates nothing.  The verification rule has no
 * counterpart for this entry point on the source pages: it exists for callers
 * that must not allocate device memory -- serving engines that reserve almost
 * all free GPU memory for their KV cache up front, plugin hosts that only lend
 * a stream and buffers, or latency-critical paths that cannot afford
 * cudaMalloc's implicit synchronisation.  It computes exactly what
 * spec_verify_greedy computes, with the same arguments minus the context; the
 * current device is used.
 * Working space: a fixed array inside the library (about 0.6 MB per GPU that
 * loads it, kept until the process exits), holding one 16-byte statistics
 * record per (request, row slot, segment).  Limits: 0 <= B <= 256, 0 <= k <= 8,
 * and B * (2k + 1) * ceil(V / segment) <= 34816, with segment = 32768 (bf16) or
 * 16384 (fp32) logits -- V up to 262144 (bf16) / 131072 (fp32) at B = 256, k = 8.
 * Larger calls return SPEC_ERR_INVALID_ARG without launching anything.
 * No cudaMalloc/cudaFree is made.  The first call on a device looks up the
 * array's device address (once per device; make that first call before any
 * stream capture).  Every call zeroes the array's arrival counters on `stream`
 * before launching; all calls share the one array, so calls that overlap on the
 * GPU (other streams, other host threads) race and must be serialised by the
 * caller. */
spec_status spec_verify_greedy_noalloc(const void* target_logits, spec_dtype dtype,
                                       const int32_t* draft_tokens, const int32_t* verify_len,
                                       int B, int k, int64_t V, int32_t* out_accepted,
                                       int32_t* out_tokens, uint32_t* out_status,
                                       cudaStream_t stream);

/* Confidence-head budget alone ("What DSpark adds"): hidden [B, kb, H] bf16,
 * w [H] bf16 -> out_len [B] int32 (leading positions with prefix survival >=
 * threshold) and optionally out_survival [B, kb] fp32 (per-position sigmoid). */
spec_status spec_conf_budget(spec_verify_ctx* ctx, const void* hidden, const void* w,
                             float bias, int B, int kb, int H, float threshold,
                             int32_t* out_len, float* out_survival, cudaStream_t stream);

/* Verified lengths alone, as spec_verify_run would use them: L_i = verify_len_i
 * (NULL => k) clamped to [0, k], limited by the confidence head's per-request
 * budget and then by conf->total_budget (see spec_conf_args).  A serving loop
 * calls this before the target's forward pass to decide how many positions of
 * each request to score.  out_len [B] int32; out_survival [B, kb] fp32 or NULL.
 * Limits: 0 <= B <= max_batch, 0 <= k <= max_k; `conf` is required. */
spec_status spec_verify_lengths(spec_verify_ctx* ctx, const spec_conf_args* conf,
                                const int32_t* verify_len, int B, int k, int32_t* out_len,
                                float* out_survival, cudaStream_t stream);

/* ---- Vocabulary-parallel verification (the LM heads split by vocabulary) ----
 * Rank r of n_shards holds the logits of tokens [bounds[r], bounds[r+1]) of
 * every row: target [B, k+1, w] and draft [B, k, w], w = bounds[r+1] -
 * bounds[r] (whole 32768-logit bf16 / 16384-logit fp32 segments, split as
 * evenly as their count allows; 1 <= n_shards <= 16 and n_shards <= the
 * segment count).  Same rule, readings and random draws as spec_verify_run
 * (dense statistics order); the caller moves the small exchange blocks:
 *   1. spec_shard_stats  -> this rank's block 1 (block1_bytes, 256-byte aligned);
 *      all-gather the blocks of ranks 0..n-1 into one contiguous buffer;
 *   2. spec_shard_decide(all blocks 1) -> outputs of every request (identical on
 *      every rank) except the sample token, and this rank's block 2;
 *      all-gather blocks 2;
 *   3. spec_shard_locate(all blocks 2) -> token_votes [B] int32 (device): the
 *      token, -1 (redo), or -2 (not this rank); element-wise MAX over ranks;
 *   4. spec_shard_finish(max votes) -> writes the certified sample tokens into
 *      out_tokens and out_redo [B] int32: 2 marks a sample the fp32 filter
 *      could not certify, 1 a request whose accept draw fell inside its
 *      certified bound.
 *   5. only if some out_redo == 2: spec_shard_refine_partials -> block 3
 *      (fp64 partial sums of this rank's sub-chunks); all-gather;
 *      spec_shard_refine_locate(all blocks 3) -> votes; MAX over ranks;
 *      spec_shard_refine_finish(max votes) -> the exact tokens, and out_redo
 *      with 1 left only where the refinement itself needed other ranks' rows.
 *   6. redo every request with out_redo == 1 whole: spec_verify_run on its
 *      gathered rows (B = 1, request_offset = request_offset + i) gives
 *      exactly the single-rank result.
 * All four calls of one verification use the same context, stream, arguments
 * and outputs.  Merged statistics are the whole-vocabulary run's record for
 * record, so decisions, probabilities and tokens equal spec_verify_run's. */
spec_status spec_shard_layout(int B, int k, int64_t V, spec_dtype dtype, int n_shards,
                              int64_t* bounds /* host [n_shards + 1] or NULL */,
                              size_t* block1_bytes, size_t* block2_bytes, size_t* block3_bytes);
spec_status spec_shard_stats(spec_verify_ctx* ctx, int rank, int n_shards, const void* target_shard,
                             const void* draft_shard, spec_dtype dtype, const int32_t* draft_tokens,
                             const int32_t* verify_len, const float* temperature,
                             const spec_conf_args* conf, int B, int k, int64_t V, void* block1,
                             cudaStream_t stream);
spec_status spec_shard_decide(spec_verify_ctx* ctx, int rank, int n_shards, const void* blocks1,
                              const void* target_shard, const void* draft_shard, spec_dtype dtype,
                              const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* temperature, const spec_conf_args* conf, int B, int k,
                              int64_t V, uint64_t seed, uint32_t step, uint32_t request_offset,
                              int32_t* out_accepted, int32_t* out_tokens, float* out_p,
                              float* out_q, uint32_t* out_status, void* block2,
                              cudaStream_t stream);
spec_status spec_shard_locate(spec_verify_ctx* ctx, int rank, int n_shards, const void* blocks2,
                              const void* target_shard, const void* draft_shard, spec_dtype dtype,
                              const int32_t* draft_tokens, const int32_t* verify_len,
                              const float* temperature, const spec_conf_args* conf, int B, int k,
                              int64_t V, int32_t* token_votes, cudaStream_t stream);
spec_status spec_shard_finish(spec_verify_ctx* ctx, const int32_t* token_votes_max, int B, int k,
                              int32_t* out_tokens, int32_t* out_redo, cudaStream_t stream);
spec_status spec_shard_refine_partials(spec_verify_ctx* ctx, int rank, int n_shards,
                                       const void* target_shard, const void* draft_shard,
                                       spec_dtype dtype, const int32_t* draft_tokens,
                                       const int32_t* verify_len, const float* temperature,
                                       const spec_conf_args* conf, int B, int k, int64_t V,
                                       void* block3, cudaStream_t stream);
spec_status spec_shard_refine_locate(spec_verify_ctx* ctx, int rank, int n_shards,
                                     const void* blocks3, const void* target_shard,
                                     const void* draft_shard, spec_dtype dtype,
                                     const int32_t* draft_tokens, const int32_t* verify_len,
                                     const float* temperature, const spec_conf_args* conf, int B,
                                     int k, int64_t V, int32_t* token_votes, cudaStream_t stream);
spec_status spec_shard_refine_finish(spec_verify_ctx* ctx, const int32_t* token_votes_max, int B,
                                     int k, int32_t* out_tokens, int32_t* out_redo,
                                     cudaStream_t stream);

/* spec_verify_run on HOST buffers: copies the inputs (pinned or pageable host
 * memory) to device staging owned by the context, verifies, copies the outputs
 * back and synchronises `stream`.  Staging grows on demand and is freed with the
 * context.  Returns SPEC_ERR_DEVICE_STATUS if any request failed (outputs are
 * still written).  `conf` points at HOST buffers too. */
spec_status spec_verify_run_host(spec_verify_ctx* ctx, const void* target_logits,
                                 const void* draft_logits, spec_dtype dtype,
                                 const int32_t* draft_tokens, const int32_t* verify_len,
                                 const float* temperature, const spec_conf_args* conf, int B,
                                 int k, int64_t V, uint64_t seed, uint32_t step,
                                 uint32_t request_offset, int32_t* out_accepted,
                                 int32_t* out_tokens, float* out_p, float* out_q,
                                 uint32_t* out_status, cudaStream_t stream);

/* Per-kernel timing: launches of the kernel classes selected by `class_mask`
 * (bit c selects class c: 0 = the verification engine (statistics, chain,
 * sampling and fp64 refinement in one launch), 1 = the LM head's statistics
 * GEMM, 2 = the LM head's row-writing GEMM, 3 = confidence head; 0 turns
 * timing off) are
 * bracketed by CUDA events on the caller's stream.  spec_verify_timing_read
 * synchronises on those events and returns, for class `which`, the number of
 * launches and their total milliseconds since timing was last enabled (enabling
 * resets).  At most 4096 launches per class are recorded. */
spec_status spec_verify_timing_enable(spec_verify_ctx* ctx, int class_mask);
spec_status spec_verify_timing_read(spec_verify_ctx* ctx, int which, int* launches,
                                    double* total_ms);

/* Diagnostics of the last completed run (synchronises the stream first):
 * out[0] = accept decisions settled by the fp64 path, out[1] = samples refined
 * in fp64, out[2] = samples certified by the fp32 filter, out[3] = chunks the
 * fp64 refinement recomputed outright, out[4] = engine error bits (0 on a good
 * run; bit 1 the work queue overflowed, any other bit a bounded wait of the
 * engine gave up -- the run's outputs are then not to be used), out[5] = where
 * the first such wait gave up (0 if none): site << 28 | CTA << 16 | its stage
 * or item count, the site being 1 + the index of its error bit.  `out` holds
 * 6 values. */
spec_status spec_verify_last_counters(spec_verify_ctx* ctx, cudaStream_t stream,
                                      uint32_t out[6]);

/* Self-check of the one hardware constant the fp32 filter relies on: the
 * maximum relative error of the ex2.approx.ftz.f32 instruction against fp64
 * exp2, over every fp32 argument in [lo, hi] (-126 <= lo <= hi <= 0), measured
 * on `device` (synchronous).  spec_verify_ex2_error_bound() returns the bound
 * the kernels assume; the measured maximum must not exceed it. */
spec_status spec_verify_selfcheck_ex2(int device, float lo, float hi, double* max_rel_err);
double spec_verify_ex2_error_bound(void);

/* ---------------------------------------------------------------------------
 * LM head with verification fused into its epilogue.
 *
 * The drafter shares the target's frozen output head ("Speculative decoding
 * becomes standard: DSpark and multi-token drafters", section "What DSpark
 * adds"), so the logits of every verified row are l = h W^T with one bf16
 * matrix W [V, H]: target rows from the target's last hidden states, drafter
 * rows from the drafter's.  These entry points take the hidden states instead
 * of logits.  The GEMM runs on the tensor cores (tcgen05, bf16 operands, fp32
 * accumulation); the logits are the fp32 accumulator values.
 *
 * spec_lmhead_verify computes exactly what spec_verify_run (dtype SPEC_F32)
 * computes on the logits [B, k+1, V] = hidden_target W^T and [B, k, V] =
 * hidden_draft W^T, without computing or writing most of those logits.  In
 * prefix order: the GEMM over position 0's two rows of every request, whose
 * epilogue reduces each accumulator tile to the row statistics, picks the
 * drafted tokens' logits and writes these rows (the rows a request samples
 * from most often); the decision of position 0; then the GEMM over the other
 * rows of the requests that accepted it, and their chains.  A last pass writes
 * the other rows a request samples from (the rejected pair, or the bonus row)
 * as fp32 logits, and the sample is drawn from them with the
 * vocabulary-parallel protocol's phases run as a single shard.  Outputs and
 * random draws are those of spec_verify_run.
 * --------------------------------------------------------------------------- */
typedef struct spec_lmhead_ctx spec_lmhead_ctx;

/* Create the LM-head workspace for verification context `vctx` (which must
 * outlive it and is used by it: one stream at a time for both).  Sizes follow
 * vctx's max_batch, max_k and max_vocab, and max_hidden (a multiple of 8, at
 * most 65536): about max_batch * (2 max_k + 1) * (4 max_vocab + 2 max_hidden)
 * bytes of device memory. */
spec_status spec_lmhead_init(spec_lmhead_ctx** ctx, spec_verify_ctx* vctx, int max_hidden);
spec_status spec_lmhead_destroy(spec_lmhead_ctx* ctx);

/* logits [rows, V] fp32 (row-major, caller-owned, 16-byte aligned) =
 * hidden [rows, H] bf16 (row-major, 16-byte aligned) x head [V, H] bf16
 * (row-major, 16-byte aligned)^T.  H a multiple of 8 (<= max_hidden), V a
 * multiple of 4 (<= max_vocab).  Asynchronous on `stream`. */
spec_status spec_lmhead_logits(spec_lmhead_ctx* ctx, const void* hidden, int rows,
                               const void* head, int H, int64_t V, float* out_logits,
                               cudaStream_t stream);

/* Fused verification.  hidden_target [B, k+1, H] bf16 and hidden_draft
 * [B, k, H] bf16 (NULL iff no sampled request verifies a position) are the
 * last hidden states of the two models, head [V, H] bf16 the shared output
 * head; every other argument and output is that of spec_verify_run.
 * out_redo [B] (device) receives 0 for every request whose outputs are final,
 * or 1 for a request whose decision needs rows this pass did not produce (an
 * accept draw inside its certified fp32 bound, or a refined sample whose
 * support stayed unsettled -- about one in 10^5 decisions): its outputs are to
 * be recomputed, e.g. spec_lmhead_logits of its rows then spec_verify_run with
 * request_offset + i.  Asynchronous on `stream`. */
spec_status spec_lmhead_verify(spec_lmhead_ctx* ctx, const void* hidden_target,
                               const void* hidden_draft, const void* head, int H,
                               const int32_t* draft_tokens, const int32_t* verify_len,
                               const float* temperature, const spec_conf_args* conf, int B, int k,
                               int64_t V, uint64_t seed, uint32_t step, uint32_t request_offset,
                               int32_t* out_accepted, int32_t* out_tokens, float* out_p,
                               float* out_q, uint32_t* out_status, int32_t* out_redo,
                               cudaStream_t stream);

/* Tile configuration of the LM-head GEMMs.  One CTA per SM with 128 x 256
 * tiles (tcgen05.mma.cta_group::1), or clusters of two CTAs sharing 256 x 256
 * tiles (tcgen05.mma.cta_group::2: each CTA loads its 128 rows and half of the
 * tile's W rows, a third fewer bytes per flop).  pairs = 0: one CTA per tile
 * everywhere; 1: CTA pairs everywhere; 2 (default): CTA pairs for the
 * row-writing GEMM only (measured faster there; the statistics GEMM is not).
 * Results are identical in every configuration. */
spec_status spec_lmhead_set_cta_pairs(spec_lmhead_ctx* ctx, int pairs);

/* Error word of the LM-head kernels since the context was created
 * (synchronises the device): bit 0 set = a wait inside a GEMM timed out and
 * that launch's outputs are not to be used. */
spec_status spec_lmhead_errors(spec_lmhead_ctx* ctx, uint32_t* out);

const char* spec_status_string(spec_status s);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_VERIFY_H */
