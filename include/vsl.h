/*
 * vsl.h - C ABI of libvsl: vocab-sliced logits and the per-row sampler on one
 * NVIDIA B200 (sm_100a).
 *
 * The two calls mirror the hot path of batch-sharded sampling as described in
 * "Qwen4Exp batch-sharded sampling: inside vLLM PR #61018" (orcarouter.ai blog):
 *
 *   - vsl_logits_local: the rank-local vocab-slice projection with no gather
 *     (section "why three lines were the whole job": the model's
 *     compute_logits_local returns logits_processor(lm_head, hidden_states,
 *     skip_gather=True), i.e. only the rank's own vocab shard; section
 *     "batch-sharded sampling in one paragraph": each rank computes only its
 *     own slice of the vocabulary projection).  On one GPU the S slices are
 *     kept as an input / output layout; nothing is gathered or exchanged.
 *   - vsl_sample: the sampler's per-request work over batch x (spec+1) x
 *     vocab logits (same page, section "batch-sharded sampling in one
 *     paragraph": top-k and top-p per request, logprobs under a non-negative
 *     max_logprobs), with temperature and a Philox4x32-keyed Gumbel-max draw.
 *
 * Conventions for every call:
 *   - The caller owns every buffer.  "device" pointers are CUDA device
 *     memory of the current device; "host" arrays are ordinary host memory
 *     read during the call only.  The library never allocates device
 *     memory and never synchronises the stream.  Per device the library
 *     keeps its kernels' launch attributes, the SM count and the largest
 *     cluster the device schedules (read once, on the first call made with
 *     that device current), and vsl_sample keeps one side stream and two
 *     events (created on the first call that runs its kernels side by side,
 *     kept for the process); the side-by-side launches of one device are
 *     serialised by a lock, and they can be captured into a CUDA graph (the
 *     side stream joins the capture through the events).
 *   - stream is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; host-side argument errors are returned before
 *     anything is enqueued, launch errors as VSL_ERR_CUDA.
 *   - Row r of the logits is the concatenation of its S slices: the token
 *     with index j in slice s has global id s * V_s + j.
 */
#ifndef VSL_H
#define VSL_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VSL_API __attribute__((visibility("default")))
#else
#define VSL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VSL_OK = 0,
  VSL_ERR_INVALID_ARG = 1,          /* null pointer, non-positive size, out-of-range value */
  VSL_ERR_ALIGNMENT = 2,            /* pointer or row pitch not 16-byte aligned            */
  VSL_ERR_UNSUPPORTED = 3,          /* size beyond the library's limits (see below)        */
  VSL_ERR_WORKSPACE_TOO_SMALL = 4,  /* workspace_bytes below vsl_sample_workspace_bytes()  */
  VSL_ERR_CUDA = 5,                 /* a CUDA runtime / driver call failed                 */
  VSL_ERR_DEVICE_TIMEOUT = 6        /* a kernel gave up a bounded wait (reported later by
                                       vsl_device_error)                                    */
} vsl_status;

/* Limits of the library. */
#define VSL_MAX_SLICES 16       /* S <= 16                                  */
#define VSL_MAX_LOGPROBS 20     /* 0 <= n_logprobs <= 20 (and <= S * V_s)   */
#define VSL_MAX_SPEC 64         /* speculative tokens per request in vsl_verify_drafts */

/* Row flags written by vsl_sample (bit set = the row was not sampled).  A
 * flagged row gets token -1, logprob NaN, top-n ids -1 and top-n logprobs NaN;
 * other rows are unaffected. */
#define VSL_ROW_NONFINITE        (1u << 0)  /* a logit is NaN or +inf                   */
#define VSL_ROW_ALL_NEG_INF      (1u << 1)  /* every logit is -inf                      */
#define VSL_ROW_BAD_TEMPERATURE  (1u << 2)  /* temperature < 0, NaN or inf              */
#define VSL_ROW_BAD_TOP_P        (1u << 3)  /* top_p <= 0 or NaN                        */
#define VSL_ROW_BAD_TOP_K        (1u << 4)  /* top_k < 0                                */
#define VSL_ROW_SCALE_OVERFLOW   (1u << 5)  /* some finite logit / temperature overflows */

/* Per-row sampling parameters (20 bytes, device memory, one entry per row;
 * a request's (spec + 1) rows normally repeat its entry with consecutive
 * positions).
 *   temperature : 0 = greedy (argmax of the raw logits, lowest id on ties;
 *                 top_k and top_p are then ignored); otherwise > 0 and finite.
 *                 Sampling uses x = fl(logit / temperature) in float32.
 *   top_k       : 0 or >= S * V_s = off; otherwise keep every token whose x is
 *                 >= the top_k-th largest x (ties at the boundary kept).
 *   top_p       : >= 1 = off; otherwise in (0, 1): over the top-k survivors,
 *                 with probabilities renormalised over them, keep a token iff
 *                 the probability mass of strictly larger x is < top_p.
 *   request_id, position : Philox counter words of the draw.
 * The draw is token = argmax over kept i of x_i - log(-log(u_i)), lowest id on
 * exact ties, with u_i = ((w >> 9) + 0.5) * 2^-23 and w the word (i mod 4) of
 * Philox4x32-10(counter = {i / 4, position, request_id, 0},
 *               key = {seed & 0xffffffff, seed >> 32}). */
typedef struct {
  float temperature;
  int32_t top_k;
  float top_p;
  uint32_t request_id;
  uint32_t position;
} vsl_row_params;

/* vsl_logits_local - logits_s[r][j] = sum_h hidden[r][h] * W_s[j][h] for every
 * slice s, bf16 inputs, fp32 accumulation and output, no gather.
 *   hidden_bf16   : device, [R][H] bf16 row-major, 16-byte aligned.
 *   w_slices_bf16 : host array of S device pointers, slice s = [V_s][H] bf16
 *                   row-major (nn.Linear out x in), each 16-byte aligned.
 *   logits_slices : host array of S device pointers, slice s = [R][V_s] fp32
 *                   row-major, each 16-byte aligned; fully overwritten.
 *   R >= 1, H >= 8 with H % 8 == 0 (16-byte rows), 1 <= S <= VSL_MAX_SLICES,
 *   V_s >= 1 with V_s % 4 == 0.
 * Errors: VSL_ERR_INVALID_ARG (null / sizes), VSL_ERR_ALIGNMENT,
 *         VSL_ERR_CUDA (tensor-map encode or launch failure). */
VSL_API vsl_status vsl_logits_local(const void* hidden_bf16, const void* const* w_slices_bf16,
                            float* const* logits_slices, int32_t R, int32_t H, int32_t S,
                            int32_t V_s, void* stream);

/* Tile statistics of the logits (optional; source: "Qwen4Exp batch-sharded
 * sampling: inside vLLM PR #61018" (orcarouter.ai blog), section
 * "batch-sharded sampling in one paragraph": the sampler's top-k / top-p and
 * logprobs need, per row, the softmax statistics and the top candidates of
 * the whole vocabulary; produced tile by tile where the projection writes the
 * logits, they let vsl_sample read only the tiles that can hold a row's
 * candidates).  For row r, slice s and block b of 128 ids (B = ceil(V_s / 128)
 * blocks per slice) the record at float offset ((r * S + s) * B + b) * 8 of a
 * device fp32 array of vsl_tile_stats_floats(R, S, V_s) floats (32-byte
 * aligned, rows contiguous) holds:
 *   [0..3] the largest logit of each 32-id quarter of the block (ids
 *          s * V_s + 128 b + 32 q + [0, 32) below (s + 1) * V_s; -inf for a
 *          quarter with no id; unspecified for a quarter holding a NaN)
 *   [4]    sum over the block of exp(l - c), c the block's largest logit when
 *          finite, else 0 (float32 with a fast exp; NaN if a logit is NaN,
 *          +inf if one is +inf)
 *   [5]    the block's smallest finite logit (+inf if none)
 *   [6]    the block's smallest |l| over logits that are neither 0 nor NaN
 *          (+inf if none; an infinite logit counts as +inf)
 *   [7]    0
 * vsl_tile_stats_floats returns 0 for non-positive sizes. */
VSL_API size_t vsl_tile_stats_floats(int32_t R, int32_t S, int32_t V_s);

/* vsl_logits_local_ex - vsl_logits_local that also writes the tile
 * statistics of the logits it produces from the same accumulators (tile_stats
 * may be NULL: vsl_logits_local).  Extra error: VSL_ERR_ALIGNMENT for a
 * tile_stats not 32-byte aligned. */
VSL_API vsl_status vsl_logits_local_ex(const void* hidden_bf16, const void* const* w_slices_bf16,
                                       float* const* logits_slices, int32_t R, int32_t H, int32_t S,
                                       int32_t V_s, float* tile_stats, void* stream);

/* vsl_tile_stats - the tile statistics of logits already in device memory
 * (logits_slices as for vsl_sample; one read of every logit).
 * Errors: VSL_ERR_INVALID_ARG, VSL_ERR_ALIGNMENT (slices not 16-byte or
 * tile_stats not 32-byte aligned, V_s % 4 != 0), VSL_ERR_UNSUPPORTED,
 * VSL_ERR_CUDA. */
VSL_API vsl_status vsl_tile_stats(const float* const* logits_slices, int32_t R, int32_t S, int32_t V_s,
                                  float* tile_stats, void* stream);

/* Bytes of device workspace vsl_sample needs for these sizes (0 if none). */
VSL_API size_t vsl_sample_workspace_bytes(int32_t R, int32_t S, int32_t V_s, int32_t n_logprobs);

/* Number of kernels one vsl_sample call with these sizes launches on the
 * current device (2 for a large batch, R above the SM count: the streaming
 * kernel, then the cluster kernel on the rows it leaves; 3 for a small one:
 * the cluster kernel beside the streaming kernel, which runs on a side stream,
 * then a pass over the rows the streaming kernel could not hold), or -1 for
 * sizes vsl_sample rejects.  Host only; no device work. */
VSL_API int32_t vsl_sample_launches(int32_t R, int32_t S, int32_t V_s);

/* The launches of one vsl_sample call, as plain data (host only, no device
 * work; vsl_sample makes the same choices on the current device):
 *   launches       : 2 (serial) or 3 (side by side)
 *   side_by_side   : 1 when R is at most the SM count: the streaming kernel
 *                    then splits rows, and the cluster kernel takes the rows
 *                    it leaves beside it
 *   stream_cluster : CTAs per row of the streaming kernel (1, 2, 4 or 8: the
 *                    most for which R times it fits two CTAs per SM)
 *   stream_part    : logits per streaming CTA;  stream_grid = R * stream_cluster
 *   cluster, part  : CTAs per row (cluster size) and logits per CTA of the
 *                    cluster kernel
 *   others_grid    : its grid beside the streaming kernel (R * cluster; 0 when
 *                    serial)
 *   deferred_grid  : the grid of its pass over the rows the streaming kernel
 *                    marked: min(R, 2 * sms / cluster) clusters
 * sms is the device's SM count and max_cluster the largest cluster size it
 * schedules for the cluster kernel (a power of two).  The plan is that of a
 * call without tile statistics; with them (S * B <= 4096) the streaming
 * kernel runs one CTA per row (stream_cluster 1, stream_part S * V_s,
 * stream_grid R), the rest unchanged.  Returns VSL_OK,
 * VSL_ERR_INVALID_ARG (null out, non-positive sizes), VSL_ERR_ALIGNMENT
 * (V_s % 4 != 0) or VSL_ERR_UNSUPPORTED (a vocabulary beyond the limits). */
typedef struct {
  int32_t launches;
  int32_t side_by_side;
  int32_t stream_cluster;
  int32_t stream_part;
  int32_t stream_grid;
  int32_t cluster;
  int32_t part;
  int32_t others_grid;
  int32_t deferred_grid;
} vsl_sample_plan;
VSL_API vsl_status vsl_sample_plan_for(int32_t R, int32_t S, int32_t V_s, int32_t sms, int32_t max_cluster,
                                       vsl_sample_plan* out);

/* vsl_sample - per-row temperature, top-k, top-p, Gumbel-max draw and top-n
 * raw logprobs.
 *   logits_slices : host array of S device pointers, slice s = [R][V_s] fp32
 *                   row-major, each 16-byte aligned (read only).
 *   params_dev    : device, R entries.
 *   seed          : 64-bit Philox key.
 *   n_logprobs    : 0 <= n <= VSL_MAX_LOGPROBS and n <= S * V_s.
 *   token_ids     : device int32 [R]          (output)
 *   token_logprob : device fp32 [R]           (output) raw log-softmax of the token
 *   topn_ids      : device int32 [R][n]       (output; may be NULL when n == 0)
 *   topn_logprob  : device fp32 [R][n]        (output; may be NULL when n == 0)
 *                   the n largest raw logits' ids and log-softmax values,
 *                   descending, lower id first on ties
 *   row_flags     : device uint32 [R]         (output) VSL_ROW_* bits, 0 = sampled
 *   workspace     : device, workspace_bytes >= vsl_sample_workspace_bytes()
 *                   (may be NULL when that is 0)
 * Logprobs are of the raw (unscaled) logits over the full vocabulary.
 * Errors: VSL_ERR_INVALID_ARG, VSL_ERR_ALIGNMENT, VSL_ERR_UNSUPPORTED,
 *         VSL_ERR_WORKSPACE_TOO_SMALL, VSL_ERR_CUDA. */
VSL_API vsl_status vsl_sample(const float* const* logits_slices, int32_t R, int32_t S, int32_t V_s,
                      const vsl_row_params* params_dev, uint64_t seed, int32_t n_logprobs,
                      int32_t* token_ids, float* token_logprob, int32_t* topn_ids,
                      float* topn_logprob, uint32_t* row_flags, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Optional outputs of vsl_sample_ex (every pointer may be NULL: not written).
 *   kept_theta : device fp32 [R][2], 8-byte aligned.  Row r gets
 *                (theta_k, theta_p), the two thresholds on x = fl(logit / T)
 *                the draw used: theta_k the top_k-th largest x (counted with
 *                multiplicity), theta_p the smallest x the top-p rule keeps
 *                among the top-k survivors; -inf for a rule that is off (top_k
 *                0 or >= S * V_s, top_p >= 1) and NaN for a greedy or a
 *                flagged row.  The kept set the token is drawn from is exactly
 *                { i : x_i finite and x_i >= max(theta_k, theta_p) }.
 *   processed_logprob      : device fp32 [R]: the token's log-probability under
 *                the distribution it was drawn from (after temperature, top-k
 *                and top-p): log q_i = (x_i - m) - log sum_{j in K} exp(x_j - m),
 *                K the kept set above, m = max_K x; 0 for a greedy row, NaN for
 *                a flagged row.  Needs kept_theta.
 *   processed_topn_ids     : device int32 [R][n_logprobs] (with processed_logprob,
 *   processed_topn_logprob : device fp32 [R][n_logprobs]   when n_logprobs > 0):
 *                the n_logprobs largest log q (largest x of K, lower id first on
 *                equal x) and their values, then -1 / -inf once K is exhausted
 *                (a greedy row: its token with 0).  Computed by one more pass
 *                over the logits after the draw.
 *   tile_stats : (input) device, the tile statistics of exactly these logits
 *                (vsl_logits_local_ex or vsl_tile_stats), 32-byte aligned.
 *                Rows that are greedy or have 0 < top_k <= 1024 then read the
 *                records and only the 32-id quarters whose largest x can reach
 *                their top max(n_logprobs, top_k) (greedy: max(n_logprobs, 1))
 *                instead of the whole row: the R-th largest block maximum t0
 *                is at most the row's R-th largest logit, so every candidate
 *                lies in a quarter whose largest x is >= fl(t0 / T).  Token
 *                ids, top-n ids, flags and kept_theta equal those of the call
 *                without them; the raw logprobs take the row's log-sum-exp
 *                from the records' sums (float32).  Ignored for top-k-off
 *                rows and when S * B exceeds 4096 blocks.
 * Source: "Qwen4Exp batch-sharded sampling: inside vLLM PR #61018"
 * (orcarouter.ai blog), section "batch-sharded sampling in one paragraph": the
 * sampler's top-k and top-p work per request, logprobs through max_logprobs. */
typedef struct {
  float* kept_theta;
  float* processed_logprob;
  int32_t* processed_topn_ids;
  float* processed_topn_logprob;
  const float* tile_stats;
} vsl_sample_extras;

/* vsl_sample_ex - vsl_sample with optional outputs (extras may be NULL, which
 * is vsl_sample).  Same arguments, ownership and errors as vsl_sample, plus
 * VSL_ERR_ALIGNMENT for a kept_theta that is not 8-byte aligned or a
 * tile_stats that is not 32-byte aligned, and
 * VSL_ERR_INVALID_ARG for processed outputs without kept_theta or without
 * their top-n buffers when n_logprobs > 0. */
VSL_API vsl_status vsl_sample_ex(const float* const* logits_slices, int32_t R, int32_t S, int32_t V_s,
                         const vsl_row_params* params_dev, uint64_t seed, int32_t n_logprobs,
                         int32_t* token_ids, float* token_logprob, int32_t* topn_ids,
                         float* topn_logprob, uint32_t* row_flags, void* workspace,
                         size_t workspace_bytes, const vsl_sample_extras* extras, void* stream);

/* vsl_verify_drafts - speculative verification of deterministic draft tokens
 * over the rows one vsl_sample call drew.  Source: "Qwen4Exp batch-sharded
 * sampling: inside vLLM PR #61018" (orcarouter.ai blog): the sampler's
 * batch x (speculative tokens + 1) x vocab rows and sharded draft logits left
 * for later (section "batch-sharded sampling in one paragraph"), acceptance
 * length (section "the 1.5 % estimate").
 * Request q owns rows q * (spec + 1) + j, j = 0 .. spec, row j holding the
 * target's draw t_j for position j (vsl_sample's token, -1 if flagged); its
 * drafts d_0 .. d_{spec-1} are single tokens (a point-mass draft).  Draft j is
 * accepted while t_j == d_j and t_j >= 0; with a accepted the request emits
 * d_0 .. d_{a-1}, then t_a (the correction, or the bonus token when a ==
 * spec), then -1.  With vsl_sample's draw keyed by (seed, request, position,
 * token) this is the rejection rule for a point-mass draft: d_j is accepted
 * with probability p(d_j), p the distribution the row samples from, and a
 * rejected position emits a token distributed as p without d_j.
 *   token_ids     : device int32 [requests * (spec + 1)]  (vsl_sample's output)
 *   token_logprob : device fp32 [requests * (spec + 1)]   (optional, NULL together with out_logprob)
 *   draft_ids     : device int32 [requests][spec]         (may be NULL when spec == 0)
 *   out_ids       : device int32 [requests][spec + 1]     (output) the emitted tokens, then -1
 *   out_logprob   : device fp32 [requests][spec + 1]      (optional output) each emitted
 *                   token's row logprob, NaN after the emitted tokens
 *   accepted      : device int32 [requests]               (output) a, 0 <= a <= spec
 *   1 <= requests, 0 <= spec <= VSL_MAX_SPEC.
 * Errors: VSL_ERR_INVALID_ARG (null pointers, sizes, only one of the two
 *         logprob pointers), VSL_ERR_UNSUPPORTED, VSL_ERR_CUDA. */
VSL_API vsl_status vsl_verify_drafts(const int32_t* token_ids, const float* token_logprob,
                                     const int32_t* draft_ids, int32_t requests, int32_t spec,
                                     int32_t* out_ids, float* out_logprob, int32_t* accepted, void* stream);

/* Reads and clears the device error word the kernels set when a bounded wait
 * gives up (a bug, never expected).  Synchronises the current device.
 * Returns VSL_OK, VSL_ERR_DEVICE_TIMEOUT (with *code_out = the site bits) or
 * VSL_ERR_CUDA. code_out may be NULL. */
VSL_API vsl_status vsl_device_error(uint32_t* code_out);

/* Static, human-readable name of a status code. */
VSL_API const char* vsl_status_string(vsl_status status);

/* Library version string. */
VSL_API const char* vsl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSL_H */
