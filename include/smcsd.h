/*
 * smcsd.h -- C ABI of libsmcsd.so: the per-round scoring / resampling hot path
 * shared by SMC speculative decoding, standard speculative-decoding
 * verification and Gumbel-top-k drafting, for NVIDIA B200 (sm_100a).
 *
 * Sources (gist.science summaries; each entry point cites its passage):
 *   [SMC-SD]  "Faster LLM Inference via Sequential Monte Carlo", section 2
 *             (Methodology: particles, scoring, importance weights,
 *             evict/duplicate resampling, bonus token, KV page metadata copy)
 *             and section 1 (standard SD and its rejection step).
 *   [METASD]  METASD (multi-drafter speculative decoding), section 2
 *             (Block Divergence reward built on total-variation distance,
 *             drafter selection by a UCB bandit).
 *   [STAND]   STAND (stochastic adaptive n-gram drafting), Methodology items
 *             1 (top-10 logit n-gram store) and 2 (Gumbel-Top-K sampling).
 *
 * Conventions for every entry point
 *   - Pointers marked "device" are caller-owned CUDA device pointers; the
 *     library never allocates, frees or keeps them.  Logit rows are
 *     row-major with the vocabulary contiguous; `ld` is the element distance
 *     between consecutive rows (ld >= V), so a slice of a wider buffer works.
 *   - `stream` is a cudaStream_t passed as void*; all work is enqueued on it
 *     and the call returns without synchronising.
 *   - Arguments are checked on the host before anything is enqueued; a bad
 *     argument returns SD_ERR_INVALID_ARG and enqueues nothing.  A launch
 *     failure returns SD_ERR_CUDA.  Sizes beyond what a kernel supports
 *     return SD_ERR_UNSUPPORTED.
 *   - Faults found on the device (bad token ids, NaN / +inf / all -inf rows,
 *     page ids out of range, an internal wait that ran out) never trap: they
 *     OR bits into *dev_err (device, may be NULL) and mark the affected
 *     outputs (NaN for reals, -1 for ids).  Read *dev_err after the stream
 *     has been synchronised; the library never clears it.
 *   - Randomness is counter-based Philox4x32-10: results are a pure function
 *     of (inputs, seed, round) and reruns are bit-identical.  Counter layout:
 *     key = seed; counter = (c0, row id, round mod 2^32,
 *     stream tag + 16 * ((round >> 32) mod 2^28)); per-vocabulary-entry noise
 *     uses c0 = entry / 4 and output word entry % 4; per-row draws use
 *     c0 = 0, word 0.  Uniform u = ((w >> 9) + 1/2) * 2^-23; Gumbel
 *     g = -log(-log u).
 *   - No C++ exception crosses this boundary.
 */
#ifndef SMCSD_H_
#define SMCSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SMCSD_API __attribute__((visibility("default")))
#else
#define SMCSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sd_status {
  SD_OK = 0,
  SD_ERR_INVALID_ARG = 1,
  SD_ERR_CUDA = 2,
  SD_ERR_UNSUPPORTED = 3
} sd_status;

typedef enum sd_dtype { SD_F32 = 0, SD_BF16 = 1 } sd_dtype;

/* Bits of the device error word. */
#define SD_DEV_TOKEN_OOB 1u      /* a draft token id outside [0, V)            */
#define SD_DEV_NONFINITE 2u      /* a row with NaN / +inf, or all -inf         */
#define SD_DEV_ZERO_RESIDUAL 4u  /* verify: rejection with max(p - q, 0) == 0  */
#define SD_DEV_PAGE_OOB 8u       /* page id outside [0, num_pages) and != -1   */
#define SD_DEV_ANCESTOR_OOB 16u  /* ancestor index outside [0, N)              */
#define SD_DEV_TIMEOUT 32u       /* an internal bounded wait gave up           */
#define SD_DEV_ARM_OOB 64u       /* bandit: an arm index outside [-1, M)       */
#define SD_DEV_TABLE_FULL 128u   /* n-gram store: no free slot for a new key   */
/* With SD_DEV_TIMEOUT, smcsd_score also sets one of bits 8..15 naming the
 * wait that gave up (diagnostic only; outputs of that call are invalid). */
#define SD_DEV_WAIT_SITE_MASK 0xFF00u

/* Reward of the drafter-selection bandit (sd_metasd_ucb). */
#define SD_REWARD_BD 0 /* Block Divergence: 1 - mean TV over the K drafted positions */
#define SD_REWARD_BE 1 /* Block Efficiency: accepted tokens / K                     */

/* Philox stream tags. */
#define SD_STREAM_BONUS 1u
#define SD_STREAM_ACCEPT 2u
#define SD_STREAM_RESIDUAL 3u
#define SD_STREAM_RESAMPLE 4u
#define SD_STREAM_TOPK_DENSE 5u
#define SD_STREAM_TOPK_SPARSE 6u
#define SD_STREAM_DRAFT 8u
#define SD_STREAM_BONUS_BLOCK 9u
#define SD_STREAM_DRAFT_BLOCK 10u
#define SD_STREAM_TOPK_BLOCK 11u
#define SD_STREAM_RESIDUAL_BLOCK 12u

/*
 * smcsd_score -- scoring step of one SMC-SD round ([SMC-SD] section 2, scoring
 * and resampling steps; bonus token; [METASD] section 2 for TV).
 *
 * For B sequences x N particles x (K+1) positions, with p = softmax(zT/tau),
 * q = softmax(zD/tau) per row (the same tau divides both):
 *   lse       of every target and draft row;
 *   log-probs lp = log p(x_{k+1}), lq = log q(x_{k+1}) at rows k < K;
 *   logw[b,n] = logw_prev[b,n] + phi[b,n] + sum_{k<K} (lp - lq)
 *                                                         (importance weight);
 *   tv[b,n,k] = 1/2 sum_v |p_v - q_v| at all K+1 rows    (block divergence);
 *   bonus[b,n] = a sample of softmax(zT[b,n,K,:]/tau) by an exact two-level
 *                Gumbel-max over blocks of 128 entries: block
 *                j* = argmax_j (log sum_{v in j} e^{z_v/tau} + G_j), G from
 *                stream 9, then v* = argmax_{v in j*} (z_v/tau + g_v), g from
 *                stream 1 (both: row id b*N+n, counter entry j or v; ties to
 *                the lower index).  V <= 128: plain Gumbel-max on stream 1.
 *                                                        (bonus token)
 *
 * zT, zD        device, [B, N, K+1, V] at row stride ld, dtype dt (fp32 or
 *               bf16).  Both tensors have K+1 rows per particle.
 * draft_tokens  device int32 [B, N, K]: token x_{k+1} scored at row k.
 * tau           > 0, finite.
 * logw_prev     device fp64 [B, N] or NULL (NULL = 0, i.e. after resampling).
 * log_potential device fp64 [B, N] or NULL (NULL = 0): phi, a per-particle
 *               log-potential multiplied into the target (reward-weighted or
 *               constrained targets, [SMC-SD] section 5: the target becomes
 *               p(x) * exp(phi(x)), so the importance weight gains phi).
 *               -inf marks a particle the constraint rules out (weight 0).
 * logw_out      device fp64 [B, N]                       (required)
 * bonus_out     device int32 [B, N]                      (required)
 * tv_out        device fp32 [B, N, K+1]                  (or NULL)
 * tokens_out    device int32 [B, N, K+1]: x_1..x_K, bonus (or NULL)
 * lse_out       device fp64 [B, N, K+1, 2]: (lse target, lse draft) (or NULL)
 * lp_out        device fp64 [B, N, K, 2]: (lp, lq)       (or NULL)
 * Requirements: B >= 0 (0 = no-op), N >= 1, K >= 0, 1 <= V <= 262144,
 *   ld >= V; B*N*(K+1) < 2^31.
 * Faults: token id outside [0, V) -> SD_DEV_TOKEN_OOB, that particle's lp/lq
 *   and logw are NaN.  Non-finite row -> SD_DEV_NONFINITE, its lse / tv / lp
 *   NaN, logw NaN, bonus -1 if it is the bonus row.
 */
SMCSD_API sd_status smcsd_score(const void* zT, const void* zD, sd_dtype dt, int B, int N, int K, int V,
                      int64_t ld, const int32_t* draft_tokens, float tau, uint64_t seed,
                      uint64_t round, const double* logw_prev, const double* log_potential,
                      double* logw_out, int32_t* bonus_out, float* tv_out, int32_t* tokens_out,
                      double* lse_out, double* lp_out, uint32_t* dev_err, void* stream);

/*
 * smcsd_resample -- weight normalisation, ESS and systematic resampling
 * ([SMC-SD] section 2: evict low-weight particles, duplicate high-weight ones;
 * the scheme is systematic and runs every round).
 *   W[b,j]   = exp(logw_j - max) / sum_m exp(logw_m - max)       (fp64)
 *   ess[b]   = 1 / sum_j W_j^2
 *   anc[b,i] = min{ j : W_0 + ... + W_j > (i + u0)/N }, clamped to N-1,
 *              u0 = uniform of stream 4, row id b.
 * logw      device fp64 [B, N]; w_out device fp64 [B, N] (or NULL);
 * ess_out   device fp64 [B] (or NULL); ancestors_out device int32 [B, N].
 * Requirements: B >= 0, 1 <= N <= 8192.
 * Faults: a sequence with NaN / +inf weights, or all -inf -> SD_DEV_NONFINITE,
 *   W and ess NaN, identity ancestors.
 */
SMCSD_API sd_status smcsd_resample(const double* logw, int B, int N, uint64_t seed, uint64_t round,
                         double* w_out, double* ess_out, int32_t* ancestors_out,
                         uint32_t* dev_err, void* stream);

/*
 * smcsd_resample_adaptive -- smcsd_resample run only where the weights have
 * degenerated: sequence b is resampled iff ess[b] < ess_frac * N (strict).
 * This is the ESS-triggered resampling of standard SMC, which [SMC-SD]
 * section 5 lists among the extensions of the every-round scheme of
 * section 2.  A sequence that is not resampled keeps its particles
 * (identity ancestors) and carries its log-weights into the next round.
 *   W, ess         as smcsd_resample (always written when requested);
 *   anc[b,:]       systematic ancestors if resampled, else 0..N-1;
 *   resampled[b]   1 if resampled, else 0;
 *   logw_next[b,:] 0 if resampled, else logw[b,:] (the next round's
 *                  logw_prev for smcsd_score).
 * ess_frac       >= 0 and not NaN; +inf resamples every sequence (= smcsd_resample),
 *                0 none.  Typical: 0.5.
 * resampled_out  device int32 [B] or NULL; logw_next device fp64 [B, N] or
 *                NULL (may equal logw: each entry is read before it is written
 *                by the same thread).
 * Requirements and faults: as smcsd_resample; a faulty sequence is never
 *   resampled (resampled 0, logw_next = logw).
 */
SMCSD_API sd_status smcsd_resample_adaptive(const double* logw, int B, int N, double ess_frac,
                                  uint64_t seed, uint64_t round, double* w_out, double* ess_out,
                                  int32_t* ancestors_out, int32_t* resampled_out,
                                  double* logw_next, uint32_t* dev_err, void* stream);

/*
 * kv_pagetable_remap -- KV cache update after resampling by page-pointer /
 * metadata copy instead of KV tensor copy ([SMC-SD] section 2, KV cache
 * management).
 *   pt_out[b,i,:]  = pt_in[b, anc[b,i], :]
 *   tok_out[b,i,:] = tok_in[b, anc[b,i], :]            (if tok_in != NULL)
 *   refcnt[p]      = #{ (b,i,s) : pt_out[b,i,s] == p }  (if page_refcnt != NULL;
 *                    the call zeroes it first)
 * pt_in, pt_out  device int32 [B, N, P]; must not alias.  -1 = empty slot.
 * ancestors      device int32 [B, N].
 * tok_in/tok_out device int32 [B, N, T] (both or neither; must not overlap); T >= 0.
 * page_refcnt    device int32 [num_pages] or NULL.
 * Overlapping pt_in / pt_out or tok_in / tok_out ranges -> SD_ERR_INVALID_ARG.
 * Faults: ancestor outside [0, N) -> SD_DEV_ANCESTOR_OOB, that particle's
 *   rows are filled with -1.  Page id outside [0, num_pages) other than -1
 *   -> SD_DEV_PAGE_OOB, copied but not counted.
 */
SMCSD_API sd_status kv_pagetable_remap(const int32_t* pt_in, const int32_t* ancestors, int B, int N, int P,
                             int32_t* pt_out, const int32_t* tok_in, int T, int32_t* tok_out,
                             int32_t* page_refcnt, int num_pages, uint32_t* dev_err,
                             void* stream);

/*
 * sd_verify_reject -- standard speculative-decoding verification, N = 1
 * ([SMC-SD] section 1 and [METASD] section 1: the first rejection discards the
 * rest; textbook rule below), with per-position TV ([METASD] section 2).
 *   for k < K: accept x_{k+1} iff u_k * q(x) < p(x), u_k from stream 2,
 *     row id b*(K+1)+k;  at the first reject j the emitted token is
 *     argmax_{v : r_v > 0} (log r_v + g_v), r = max(p_j - q_j, 0), g from
 *     stream 3 with row id b*(K+1)+j;  if all K are accepted the bonus token
 *     is argmax_v (zT[b,K,v]/tau + g_v), stream 1, row id b.
 * zT  device [B, K+1, V], zD device [B, K, V], row stride ld, dtype dt.
 * draft_tokens  device int32 [B, K].
 * accepted_len  device int32 [B]: j (or K).
 * out_tokens    device int32 [B, K+1]: accepted drafts, then the drawn token,
 *               then -1 padding.
 * tv_out        device fp32 [B, K] or NULL.
 * Requirements: B >= 0, K >= 1, 1 <= V <= 262144, ld >= V.
 * Faults: a draft id outside [0, V) is rejected (SD_DEV_TOKEN_OOB); a
 *   non-finite row reached by the sequence stops it there without a token
 *   (SD_DEV_NONFINITE); an all-zero residual falls back to sampling p
 *   (SD_DEV_ZERO_RESIDUAL).
 */
SMCSD_API sd_status sd_verify_reject(const void* zT, const void* zD, sd_dtype dt, int B, int K, int V,
                           int64_t ld, const int32_t* draft_tokens, float tau, uint64_t seed,
                           uint64_t round, int32_t* accepted_len, int32_t* out_tokens,
                           float* tv_out, uint32_t* dev_err, void* stream);

/*
 * gumbel_topk -- k tokens per row without replacement by Gumbel-top-k
 * ([STAND] Methodology item 2), drawn top-down over blocks of 128 entries
 * (s = z/tau, row id = row):
 *   M_j = log sum_{v in j} e^{s_v} + G_j, G from stream 11 (counter entry j);
 *   the k largest M_j are kept (ties to the lower j);
 *   in a kept block, h_v = s_v + g_v (g from stream 5, counter entry v),
 *   Z_j = max h, and S_v = -log(e^{-M_j} - e^{-Z_j} + e^{-h_v}) (Gumbels
 *   conditioned on the block's maximum M_j);
 *   output the k largest S_v, descending, ties to the lower v.
 * The law is that of one independent Gumbel per entry (k draws without
 * replacement from softmax(s)); with V <= 128 the order is that of s_v + g_v.
 * z          device [rows, V] at row stride ld, dtype dt.
 * idx_out    device int32 [rows, k] (required).
 * score_out  device fp32 [rows, k]: S_v (or NULL).
 * logp_out   device fp32 [rows, k]: s_v - logsumexp(s) (or NULL).
 * Requirements: rows >= 0, 1 <= k <= 16, k <= V <= 262144, ld >= V.
 * Faults: rows with NaN / +inf or all -inf -> SD_DEV_NONFINITE, ids -1;
 *   ranks with no finite entry left are -1.
 */
SMCSD_API sd_status gumbel_topk(const void* z, sd_dtype dt, int rows, int V, int64_t ld, int k, float tau,
                      uint64_t seed, uint64_t round, int32_t* idx_out, float* score_out,
                      float* logp_out, uint32_t* dev_err, void* stream);

/*
 * gumbel_topk_sparse -- the same draw over stored top-L (index, probability)
 * rows of a logit n-gram store ([STAND] Methodology items 1-2): s_l =
 * log(prob_l)/tau (prob 0 = unstored = never drawn), g from stream 6 with row
 * id = row at stored position l; ties to the lower l; outputs the stored
 * global ids.
 * idx   device int32 [rows, L];  prob device fp32 [rows, L];
 * idx_out device int32 [rows, k].
 * Requirements: rows >= 0, 1 <= L <= 16, 1 <= k <= L.
 * Faults: NaN / negative / infinite probability -> SD_DEV_NONFINITE, ids -1.
 */
SMCSD_API sd_status gumbel_topk_sparse(const int32_t* idx, const float* prob, int rows, int L, int k,
                             float tau, uint64_t seed, uint64_t round, int32_t* idx_out,
                             uint32_t* dev_err, void* stream);

/*
 * sd_draft_sample -- the draft step's sampling: one token per draft row drawn
 * from the drafter's own distribution ([SMC-SD] section 2: the draft model
 * extends each particle by K tokens, one position at a time; [STAND]
 * Methodology item 1: stochastic drafting samples the distribution instead of
 * taking its argmax).  Exact two-level Gumbel-max over blocks of 128 entries:
 *   block j*  = argmax_j (log sum_{v in j} e^{zD[r,v]/tau} + G_j), G from
 *               stream 10;
 *   tokens[r] = argmax_{v in j*} (zD[r, v] / tau + g_v), g from stream 8
 *               (both: row id row0 + r, counter entry j or v, ties to the
 *               lower index; V <= 128: plain Gumbel-max on stream 8);
 *   logq[r]   = zD[r, tokens[r]] / tau - logsumexp_v(zD[r, v] / tau),
 * the log q_D(x) an SMC-SD importance weight uses.  One call per draft
 * position: rows are all particles of all sequences at that position.
 * zD          device [rows, V] at row stride ld, dtype dt.
 * row0        row id of the first row (the noise of row r uses row0 + r;
 *             row0 + rows <= 2^32).
 * tokens_out  device int32 [rows]                           (required)
 * logq_out    device fp32 [rows]                            (or NULL)
 * Requirements: rows >= 0, V >= 1, ld >= V, tau > 0 finite.
 * Faults: rows with NaN / +inf or all -inf -> SD_DEV_NONFINITE, token -1,
 *   logq NaN.
 */
SMCSD_API sd_status sd_draft_sample(const void* zD, sd_dtype dt, int rows, int V, int64_t ld,
                                    float tau, uint64_t seed, uint64_t round, uint32_t row0,
                                    int32_t* tokens_out, float* logq_out, uint32_t* dev_err,
                                    void* stream);

/*
 * sd_metasd_ucb -- one round of drafter selection for B sequences, each with
 * its own M-armed bandit ([METASD] section 2: a multi-armed bandit picks the
 * drafter of each round; its reward is the Block Divergence, built on the TV
 * distance between drafter and target, or the Block Efficiency, the
 * accepted-token count; MetaSD-UCB is an upper-confidence-bound rule).  The
 * page gives no formula; the rule here is UCB1 with rewards in [0, 1]:
 *   reward  BD = 1 - (1/K) sum_{k<K} tv[b, k]   (fp64, summed in k order)
 *           BE = accepted_len[b] / K
 *   update  pulls[b, a] += 1, sums[b, a] += reward, a = arm_in[b]
 *           (nothing when arm_in[b] == -1: no arm used yet)
 *   choose  arm_out[b] = the lowest arm never pulled, else
 *           argmax_i sums/pulls + sqrt(c * ln(t) / pulls), t = sum_i pulls,
 *           ties to the lowest i.  c = 2 is the textbook UCB1 bonus.
 * tv            device fp32 [B, ld_tv], ld_tv >= K (the per-position TV of
 *               sd_verify_reject); needed for BD, ignored for BE.
 * accepted_len  device int32 [B]; needed for BE, ignored for BD.
 * arm_in        device int32 [B]: the arm each sequence used this round, or -1.
 * pulls, sums   device int32 / fp64 [B, M]: the bandit state, caller-owned,
 *               zero to start, updated in place.
 * arm_out       device int32 [B] (may alias arm_in: each thread reads its own
 *               entry first).
 * reward_out    device fp64 [B] or NULL: the reward credited (NaN if none).
 * Requirements: B >= 0, K >= 1, 1 <= M <= 4096, 0 <= c < inf,
 *   reward_kind SD_REWARD_BD or SD_REWARD_BE.
 * Faults: arm_in outside [-1, M) -> SD_DEV_ARM_OOB, no update; a NaN TV or an
 *   accepted length outside [0, K] -> SD_DEV_NONFINITE, no update.  The
 *   next arm is chosen in both cases.
 */
SMCSD_API sd_status sd_metasd_ucb(const float* tv, int64_t ld_tv, const int32_t* accepted_len,
                                  const int32_t* arm_in, int B, int K, int M, int reward_kind,
                                  double c, int32_t* pulls, double* sums, int32_t* arm_out,
                                  double* reward_out, uint32_t* dev_err, void* stream);

/*
 * Logit n-gram store ([STAND] Methodology item 1): per observed n-gram, the
 * next-token distribution reduced to its k most likely (index, probability)
 * pairs; a repeated n-gram merges the stored and the new row by a weighted
 * average (an unstored index counts as probability 0) and cuts the result
 * back to the k largest, so each n-gram costs fixed memory.  Rows feed
 * gumbel_topk_sparse (stochastic drafting, item 2).  Readings of the page:
 *   - an observation is softmax(z / tau) at one position; its k largest
 *     entries (ties to the lower index; -inf entries are not stored) keep
 *     their probabilities under the full softmax, rounded to fp32;
 *   - the average weighs by occurrence count c:
 *       p_new(v) = (c * p_old(v) + p_obs(v)) / (c + 1)
 *     in fp64 with each operation rounded once, then rounded to fp32; the k
 *     largest results (ties to the lower index) are stored in that order,
 *     unused entries as (-1, 0); the count becomes c + 1;
 *   - observations of one n-gram within a call apply in their batch order.
 * The table is one caller-owned device buffer of ngram_table_bytes(C, k)
 * bytes, 16-byte aligned, zeroed by ngram_table_clear before first use:
 *   keys u64 [C] | counts i32 [C] | idx i32 [C][k] | prob f32 [C][k];
 * capacity C a power of two in [32, 2^40]; 1 <= k <= 16.  A key is the exact
 * n-gram (1 <= n <= 3 token ids in [0, 2^20)); slots are found by linear
 * probing from a hash of the key.  Nothing is ever deleted.  Which slot a new
 * n-gram takes depends on the order in which concurrent claims land, so the
 * buffer's bytes may differ between runs; every lookup result does not.
 */
/* Bytes of a table of C slots with k entries each (0 if C or k is invalid). */
SMCSD_API size_t ngram_table_bytes(int64_t capacity, int k);
/* Bytes of the workspace ngram_store_update needs for U observations (0 if
 * U is outside [0, 16384]). */
SMCSD_API size_t ngram_workspace_bytes(int U);
/* Zeroes the table (every slot empty).  Enqueued on stream. */
SMCSD_API sd_status ngram_table_clear(void* table, int64_t capacity, int k, void* stream);

/*
 * ngram_observe_topk -- the observation rows: for u < U, with r = row_ids[u]
 * (or u when row_ids is NULL),
 *   idx_out[u, :]  = the k largest entries of z[r, :] (ties to the lower
 *                    index; finite entries only; -1 past them),
 *   prob_out[u, :] = exp(z[r, v] / tau - logsumexp_w(z[r, w] / tau)) (0 past
 *                    them), fp32.
 * z         device [rows, V] at row stride ld, dtype dt.
 * row_ids   device int32 [U] or NULL (then U <= rows).
 * idx_out   device int32 [U, k];  prob_out device fp32 [U, k].
 * Requirements: rows, U >= 0; V >= 1; ld >= V; 1 <= k <= 16; tau > 0 finite.
 * Faults: a row with NaN / +inf or all -inf -> SD_DEV_NONFINITE, ids -1,
 *   prob NaN; a row id outside [0, rows) -> SD_DEV_TOKEN_OOB, same outputs.
 */
SMCSD_API sd_status ngram_observe_topk(const void* z, sd_dtype dt, int rows, int V, int64_t ld,
                                       const int32_t* row_ids, int U, int k, float tau,
                                       int32_t* idx_out, float* prob_out, uint32_t* dev_err,
                                       void* stream);

/*
 * ngram_store_update -- merges U observations into the table, in batch order
 * for equal n-grams.
 * ctx        device int32 [U, n]: the n-gram preceding each observation.
 * idx, prob  device int32 / fp32 [U, k]: observation rows (ngram_observe_topk
 *            output; -1 entries are empty).
 * workspace  device, >= ngram_workspace_bytes(U) bytes, 4-byte aligned,
 *            caller-owned scratch (no initial contents needed); calls that
 *            share a workspace or a table must not overlap on the GPU.
 * Requirements: 1 <= n <= 3; 0 <= U <= 16384 (more -> SD_ERR_UNSUPPORTED).
 * Faults: a context id outside [0, 2^20) -> SD_DEV_TOKEN_OOB, that
 *   observation skipped; a row with a NaN / infinite / negative probability
 *   or a repeated index -> SD_DEV_NONFINITE, skipped; no free slot for a new
 *   n-gram -> SD_DEV_TABLE_FULL, its observations skipped.
 */
SMCSD_API sd_status ngram_store_update(void* table, int64_t capacity, int k, const int32_t* ctx,
                                       int n, const int32_t* idx, const float* prob, int U,
                                       void* workspace, size_t workspace_bytes, uint32_t* dev_err,
                                       void* stream);

/*
 * ngram_store_update_noalloc -- ngram_store_update without a caller
 * workspace: the library's own fixed device array (room for 16384
 * observations) serves as the workspace, and the call allocates nothing.
 * The paper has no counterpart; it exists for callers that may not allocate
 * device memory.  Nothing in the array must start at zero.  Every call
 * shares the one array, so calls that overlap on the GPU (other streams,
 * other host threads) race on it: keep them ordered.
 * Arguments, requirements and faults as ngram_store_update; U > 16384 ->
 * SD_ERR_UNSUPPORTED.
 */
SMCSD_API sd_status ngram_store_update_noalloc(void* table, int64_t capacity, int k,
                                               const int32_t* ctx, int n, const int32_t* idx,
                                               const float* prob, int U, uint32_t* dev_err,
                                               void* stream);

/*
 * ngram_store_lookup -- the stored rows of Q n-grams.
 * ctx        device int32 [Q, n].
 * idx_out    device int32 [Q, k] (-1 where absent); prob_out device fp32
 *            [Q, k] (0 where absent): ready for gumbel_topk_sparse (L = k).
 * count_out  device int32 [Q] or NULL: observations merged (0 if absent).
 * Faults: a context id outside [0, 2^20) -> SD_DEV_TOKEN_OOB, reported absent.
 */
SMCSD_API sd_status ngram_store_lookup(const void* table, int64_t capacity, int k,
                                       const int32_t* ctx, int n, int Q, int32_t* idx_out,
                                       float* prob_out, int32_t* count_out, uint32_t* dev_err,
                                       void* stream);

/* Human-readable name of a status code (static storage). */
SMCSD_API const char* sd_status_string(sd_status s);

/* Library ABI version (major * 100 + minor). */
SMCSD_API int sd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SMCSD_H_ */
