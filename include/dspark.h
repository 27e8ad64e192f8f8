/*
 * dspark.h -- C ABI of the DSpark per-step speculative-decoding hot path
 * (B200 / sm_100a).
 *
 * Three calls make one decode step, in this order on one stream:
 *   1. dspark_draft_markov       the semi-autoregressive Markov-head draft
 *   2. dspark_confidence_prefix  the confidence-scheduled prefix cut (or
 *      dspark_confidence_prefix_async: against a verify budget decided two
 *      steps earlier, with a staircase or piecewise-linear cost table)
 *   3. dspark_verify             the lossless rejection-sampling verify
 * and one offline call calibrates the confidence head that step 2 reads:
 *   dspark_sts_fit               per-position temperatures fitted on a
 *                                calibration set (sequential temperature
 *                                scaling) and the calibration error
 *
 * Sources (page title, section):
 *   yage.ai "DSpark speculative decoding hardware scheduling": the
 *     first-order Markov head paragraph (p(x_k|x_{k-1}) =
 *     softmax(base_logit_k + transition_bias(x_{k-1}, x_k)), the bias read
 *     from a V x V low-rank matrix with the previous token); the rejection
 *     sampling paragraph (the draft must give the exact single-step
 *     p_d(x_k)); the SPS(B) scheduler paragraph (rank every draft token of
 *     the batch by calibrated survival, add the most probable first, stop
 *     before the throughput curve turns down; STS on an offline set); the
 *     engineering paragraph (a staircase throughput curve; the budget from
 *     the confidences of two steps back, the selection from the current
 *     ones); the variable-length verify paragraph (verify rows flattened
 *     into one tensor, no padding).
 *   freeaitool.com "DeepSeek DSpark complete guide": 3.1 (Markov head,
 *     rank 256), 4.1 (confidence c_k, sequential temperature scaling),
 *     4.2 (greedy ordering with early stop against a profiled curve).
 *   legalagi.cn "读懂 DSpark": 三 (keep the longest accepted prefix;
 *     lossless), 五 (early stop keeps the scheduler lossless).
 * The accept / residual / bonus rule is textbook speculative sampling
 * (Leviathan et al. 2023; Chen et al. 2023).
 *
 * Conventions shared by every call
 *   - Every pointer argument is DEVICE memory owned by the caller, unless
 *     stated otherwise.  The library allocates nothing and keeps no state
 *     between calls.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on it: no host
 *     synchronisation, fixed launch shapes for fixed sizes.  The calls that
 *     take a workspace can be captured in a CUDA graph (the benchmark
 *     replays whole steps that way).
 *   - Argument errors (NULL required pointers, bad sizes, misaligned
 *     pointers, too small workspace) are reported synchronously by the
 *     return value, before anything is enqueued.
 *   - Data errors found on the device (a token id outside [0,V), a verify
 *     length outside [0,K], a target row outside the buffer, a
 *     non-positive or non-finite 1/T, a non-finite partition sum, a cost
 *     table that is not ascending) set bits in a status word kept at the
 *     start of the call's workspace; each call clears that word first.
 *     Read it with dspark_get_device_status (synchronises the stream).
 *     The kernels clamp offending values so every access stays in bounds.
 *   - Layouts are row-major and contiguous.  V, r, B, K are counts.
 *     Uniforms are fp32 in [0, 1).  Sampling is by inverse CDF: the
 *     smallest index whose running probability exceeds u.
 *   - All base / target logits are fp32; U and W are bf16 (tensor-core
 *     path for B > 16) or fp32 (CUDA-core path); arithmetic is fp32 with
 *     fp32 accumulation, partition sums and CDF scans in fp64.
 *   - Alignment: base_logits, target_logits, U, W and the workspace must
 *     be 16-byte aligned (256 for the workspace); V % 4 == 0; r % 8 == 0.
 */
#ifndef DSPARK_H_
#define DSPARK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSPARK_OK = 0,
    DSPARK_ERR_INVALID_ARG = 1,  /* bad argument, reported before any launch */
    DSPARK_ERR_CUDA = 2,         /* a CUDA runtime call failed */
    DSPARK_ERR_TIMEOUT = 3,      /* a bounded device-side wait gave up */
    DSPARK_ERR_UNSUPPORTED = 4,  /* sizes outside what this library supports */
    DSPARK_ERR_DEVICE_DATA = 5,  /* device found bad data (see status flags) */
    DSPARK_ERR_WORKSPACE = 6     /* workspace missing, misaligned or too small */
} dspark_status;

typedef enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 } dspark_dtype;

/* Device status flag bits (dspark_get_device_flags). */
#define DSPARK_FLAG_BAD_TOKEN   0x01u /* token id outside [0, V) */
#define DSPARK_FLAG_BAD_LENGTH  0x02u /* verify_len outside [0,K] or row outside target */
#define DSPARK_FLAG_NONFINITE   0x04u /* non-finite or zero partition sum */
#define DSPARK_FLAG_BAD_TEMP    0x08u /* inv_temp <= 0 or non-finite */
#define DSPARK_FLAG_TIMEOUT     0x10u /* a bounded device wait gave up */
#define DSPARK_FLAG_BAD_TABLE   0x20u /* cost table not ascending or cost <= 0 */

/* ---------------------------------------------------------------------- */
/* 1. Markov-head draft                                                    */
/* ---------------------------------------------------------------------- */

/* Workspace bytes dspark_draft_markov needs for these sizes. */
size_t dspark_draft_workspace_size(int V, int r, int B, int K);

/*
 * For every request b and position k = 1..K, sequentially in k:
 *   x_0       = prev_token[b]
 *   l_v       = (base_logits[b,k,v] + U[x_{k-1}] . W[v]) * inv_temp[b]
 *   p(.)      = softmax(l)
 *   x_k       = inverse-CDF draw from p with u_draft[b,k]
 * (yage.ai, Markov-head paragraph; freeaitool 3.1).  The bias term is
 * left out when x_{k-1} < 0 (only possible at k = 1).
 *
 * Inputs
 *   base_logits [B,K,V] fp32   base logits from the parallel backbone
 *   U, W        [V,r]          low-rank transition factors, uw_dtype
 *   prev_token  [B] int32      last committed token (<0: no bias at k=1)
 *   inv_temp    [B] fp32 or NULL (NULL: 1)
 *   u_draft     [B,K] fp32 uniforms
 * Outputs
 *   tokens   [B,K] int32   x_k
 *   p_tok    [B,K] fp32    p_d(x_k), the exact draft probability of x_k
 *   lse      [B,K] fp32    log sum_v exp(l_v)
 *   ref_max  [B,K] fp32    M: the reference maximum of the un-tempered
 *                          logits (base + bias) used by the sampler
 *   ref_sum  [B,K] fp32    Z = sum_v exp((base_v + bias_v - M) * inv_temp);
 *                          p_d(v) = exp((base_v + bias_v - M)*inv_temp) / Z.
 *                          dspark_verify needs ref_max / ref_sum to rebuild
 *                          the draft row at a rejected position exactly.
 *   draft_logits [B,K,V] fp32 or NULL: the tempered logits l, if wanted.
 *   draft_bias   [B,K,V] fp32 or NULL: the transition bias U[x_{k-1}] . W[v]
 *                of every drafted position.  Passing it on to
 *                dspark_verify lets the verify rebuild the draft row at a
 *                rejected position without another pass over W (worth it
 *                for small B; for large B the re-projection is cheaper
 *                than writing B*K*V floats).
 */
dspark_status dspark_draft_markov(
    const float *base_logits, const void *U, const void *W, dspark_dtype uw_dtype,
    int V, int r, int B, int K,
    const int32_t *prev_token, const float *inv_temp, const float *u_draft,
    int32_t *tokens, float *p_tok, float *lse, float *ref_max, float *ref_sum,
    float *draft_logits, float *draft_bias, void *workspace, size_t ws_bytes,
    void *stream);

/* ---------------------------------------------------------------------- */
/* 1b. Sequential temperature scaling of the confidence head (offline)     */
/* ---------------------------------------------------------------------- */

/* Largest K dspark_sts_fit takes. */
#define DSPARK_STS_MAX_K 32

/* Workspace bytes dspark_sts_fit needs (0 for sizes it does not take). */
size_t dspark_sts_workspace_size(long long N, int K);

/*
 * Fits the per-position temperatures T_k that dspark_confidence_prefix
 * divides the head's scores by (freeaitool 4.1: the head's raw scores are
 * over-confident and are calibrated after training, position by position
 * from left to right; yage.ai scheduler paragraph: on an offline set, so
 * that the probabilities match the observed acceptance rates).
 *
 * Calibration set: N sequences with head scores z[n, k] and the accepted
 * prefix length n_accepted[n] of a full-block verify (what dspark_verify
 * writes).  Position k (0-based) of sequence n is observed when
 * n_accepted[n] >= k and accepted when n_accepted[n] > k.  T_k minimises
 * the Bernoulli negative log-likelihood of the observed labels under
 * c = 1 / (1 + exp(-z / T_k)).  Search, the same for every position:
 * theta = 1/T in [1/20, 1/0.05]; the likelihood's derivative in theta at
 * both bounds (a sign that puts the minimiser on a bound settles it), then
 * from theta = 1 Newton steps on the derivative kept inside a bracket of
 * theta (its geometric midpoint when a step leaves it), until a step moves
 * theta by at most 1e-13 relative or after 40 steps.  A position nobody
 * reached, or with only z = 0, gets T = 1.  Sums are fp64 in a fixed
 * order (run-to-run identical).
 *
 * ece[0], ece[1]: expected calibration error before (every T = 1) and
 * after the fit: observed pairs pooled into 15 equal-width bins of c,
 * sum over bins of |accepted count - sum of c| / number of pairs.
 *
 * Inputs   z [N,K] fp32 (non-finite scores are left out and flagged),
 *          n_accepted [N] int32 in [0,K] (clamped and flagged otherwise)
 * Outputs  temps [K] fp32, ece [2] fp32, passes [1] int32 or NULL: the
 *          passes over the data the fit made (derivative evaluations of
 *          the longest search, plus two for the ECE)
 * Errors   K > DSPARK_STS_MAX_K: DSPARK_ERR_UNSUPPORTED.  At most 2 + 40
 *          derivative passes (a pass with nothing left to search returns
 *          at once), 89 launches, no host sync.
 */
dspark_status dspark_sts_fit(const float *z, const int32_t *n_accepted, long long N, int K,
                             float *temps, float *ece, int32_t *passes, void *workspace,
                             size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* 1c. RNN sequential head                                                 */
/* ---------------------------------------------------------------------- */

size_t dspark_draft_rnn_workspace_size(int V, int r, int B, int K);

/*
 * The draft with the optional RNN head in place of the Markov head
 * (freeaitool.com "DeepSeek DSpark complete guide" 3.1: the sequential head
 * is the Markov head by default, or an RNN head that keeps a recurrent state
 * to capture longer dependencies; the page gives no formula, the one below
 * is this library's reading):
 *     s_{-1} = h0[b] (zeros if h0 is NULL),  x_{-1} = prev_token[b]
 *     s_k    = tanh(R s_{k-1} + U[x_{k-1}])     (no U term when x < 0)
 *     p(x_k | x_<k) = softmax((base_logits[b,k,:] + s_k . W^T) * inv_temp[b])
 * sampled by inverse CDF with u_draft[b,k] exactly as dspark_draft_markov
 * (same outputs: tokens, p_tok, lse, ref_max, ref_sum).  p_d stays one
 * exact softmax per position, as the rejection-sampling verify needs.
 *
 * Inputs beyond dspark_draft_markov's
 *   R [r, r] bf16, row-major, (R s)_i = sum_j R[i, j] s_j
 *   h0 [B, r] fp32 or NULL: the state before position 1
 * Outputs beyond dspark_draft_markov's
 *   states [B, K, r] fp32 or NULL: s_k of every position (the caller keeps
 *       the one after the last accepted token for the next step)
 *   draft_bias [B, K, V] fp32 or NULL: s_k . W^T.  The verify of an RNN
 *       draft needs it (pass it to dspark_verify): the verify's own
 *       re-projection of a rejected row is the Markov lookup.
 * Sizes: bf16 only, r a multiple of 64 up to 256, V >= 128; any B.  The
 * state is fp32; the projection multiplies W by its bf16 high and low parts
 * (about 2^-17 relative).  Errors as for dspark_draft_markov.
 */
dspark_status dspark_draft_rnn(
    const float *base_logits, const void *U, const void *W, const void *R,
    dspark_dtype uw_dtype, int V, int r, int B, int K, const int32_t *prev_token,
    const float *h0, const float *inv_temp, const float *u_draft, int32_t *tokens,
    float *p_tok, float *lse, float *ref_max, float *ref_sum, float *states,
    float *draft_logits, float *draft_bias, void *workspace, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* 2. Confidence-scheduled prefix cut                                      */
/* ---------------------------------------------------------------------- */

/* Bytes of the workspace of the two prefix calls: the status word, and for
 * more than 1024 candidates (B*K) the survivals and the candidate order that
 * the call's two kernels pass between them (20 bytes per candidate). */
size_t dspark_prefix_workspace_size(int B, int K, int n_pts);

/*
 * Sequential temperature scaling, survival and the hardware-aware greedy
 * prefix cut (freeaitool 4.1-4.2; yage.ai SPS(B) paragraph; legalagi 五):
 *   c[b,k]        = sigmoid(z[b,k] / temps[k])
 *   survival[b,k] = prod_{j<=k} c[b,j]
 *   candidates (b,k) in order of survival descending, ties by k then b
 *   ascending; starting from N = B verify tokens and E = B expected
 *   emitted tokens, a candidate is committed while E'/t(N') > E/t(N) with
 *   E' = E + survival, N' = N + 1; the first candidate that does not raise
 *   the objective ends the scan.  t(N) = piecewise-linear interpolation of
 *   (cost_tokens, cost_ms), extended linearly past both ends.
 *   verify_len[b] = committed positions of request b (a prefix 1..L_b).
 *   objective[0]  = E / t(N) of the committed set.
 * enable == 0: verify_len[b] = K for every b (c and survival still filled).
 * Inputs: z [B,K], temps [K], cost_tokens [n_pts] (ascending), cost_ms
 * [n_pts]; n_pts >= 2; B*K <= 8192.  Computed in fp64 on the device.
 */
dspark_status dspark_confidence_prefix(
    const float *z, const float *temps, const float *cost_tokens,
    const float *cost_ms, int n_pts, int B, int K, int enable,
    float *c, float *survival, int32_t *verify_len, float *objective,
    void *workspace, size_t ws_bytes, void *stream);

/* Cost-table readings for dspark_confidence_prefix_async. */
#define DSPARK_COST_LINEAR 0    /* piecewise-linear interpolation (as above) */
#define DSPARK_COST_STAIRCASE 1 /* a batch of N tokens costs the entry of the
                                   smallest profiled size >= N; past the last
                                   entry, the last segment's slope */

/*
 * The prefix cut with the asynchronous budget (yage.ai, engineering
 * paragraph: the number of tokens a step verifies is decided from the
 * confidences of two steps back, so the decision never waits for the
 * current step; which tokens fill it is still decided by the current,
 * calibrated confidences) and a choice of cost-table reading (the same
 * paragraph: the measured throughput curve jumps in steps).
 *
 *   staircase   DSPARK_COST_LINEAR or DSPARK_COST_STAIRCASE
 *   budget_in   [1] int32 device, or NULL: verify tokens N (one per request
 *               included) decided earlier; the first N - B candidates of
 *               the current order are committed (N clamped to [B, B + B*K]).
 *               NULL, or a negative value: the greedy cut of
 *               dspark_confidence_prefix.
 *   budget_out  [1] int32 device, or NULL: N of the greedy cut on this
 *               step's confidences (B + B*K when enable = 0), the budget
 *               for two steps later.  May be the same word as budget_in:
 *               the budget is read before the new one is written, so a
 *               two-slot ring (step t uses slot t % 2) replays in a graph.
 * Everything else as for dspark_confidence_prefix, which is this call
 * with DSPARK_COST_LINEAR and no budgets.  The candidate order makes every
 * budget cut a prefix of each request's draft (survival never rises along
 * k; equal survivals go to the earlier position).
 */
dspark_status dspark_confidence_prefix_async(
    const float *z, const float *temps, const float *cost_tokens, const float *cost_ms,
    int n_pts, int staircase, int B, int K, int enable, const int32_t *budget_in,
    float *c, float *survival, int32_t *verify_len, float *objective, int32_t *budget_out,
    void *workspace, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------- */
/* 3. Rejection-sampling verify                                            */
/* ---------------------------------------------------------------------- */

size_t dspark_verify_workspace_size(int V, int r, int B, int K);

/*
 * Lossless verify of one step (legalagi 三; yage.ai rejection-sampling
 * paragraph; textbook speculative sampling):
 *   p_t(row)   = softmax(target_logits[row] * inv_temp[b])
 *   for k = 1..L_b (L_b = verify_len[b]), row = row_start[b] + k - 1:
 *       accept iff u_accept[b,k] < p_t(x_k) / p_tok[b,k]; stop at the first
 *       rejection.  n_accepted[b] = accepted prefix length.
 *   rejected at position j: the correction token is drawn with
 *       u_resample[b] from normalize(max(0, p_t - p_d)) where p_d is the
 *       draft distribution at position j, rebuilt from base_logits, U, W,
 *       the previous token, ref_max[b,j] and ref_sum[b,j] (falls back to
 *       p_t if the residual mass is zero);
 *   all accepted: a bonus token is drawn with u_resample[b] from p_t of
 *       row row_start[b] + L_b.
 *   out_tokens[b, 0..n] = accepted draft tokens then the correction/bonus
 *   token; the rest of the row (up to K) is -1.
 *
 * Inputs
 *   target_logits [n_target_rows, V] fp32: flattened ragged verify rows;
 *       request b uses rows row_start[b] .. row_start[b] + L_b.
 *   row_start [B] int64; verify_len [B] int32 (L_b in [0,K], read on device)
 *   base_logits, U, W, uw_dtype, prev_token, inv_temp: as for the draft
 *   tokens, p_tok, ref_max, ref_sum [B,K]: the draft's outputs
 *   draft_bias [B,K,V] or NULL: the draft's bias rows (see the draft); NULL
 *       makes the verify re-project U[x_{j-1}] . W for the rejected row
 *   u_accept [B,K], u_resample [B] fp32 uniforms
 * Outputs
 *   n_accepted [B] int32; out_tokens [B,K+1] int32;
 *   last_token [B] int32 or NULL: the last emitted token (the next step's
 *       prev_token).
 */
dspark_status dspark_verify(
    const float *target_logits, int64_t n_target_rows, const int64_t *row_start,
    const int32_t *verify_len, const float *base_logits, const void *U,
    const void *W, dspark_dtype uw_dtype, int V, int r, int B, int K,
    const int32_t *prev_token, const float *inv_temp, const int32_t *tokens,
    const float *p_tok, const float *ref_max, const float *ref_sum,
    const float *draft_bias, const float *u_accept, const float *u_resample,
    int32_t *n_accepted,
    int32_t *out_tokens, int32_t *last_token, void *workspace, size_t ws_bytes,
    void *stream);

/* ---------------------------------------------------------------------- */
/* 3b. Verify with the target's LM head projected on chip                  */
/* ---------------------------------------------------------------------- */

size_t dspark_verify_lmhead_workspace_size(int V, int r, int B, int K, int dm,
                                           int64_t n_target_rows);

/*
 * The verify of dspark_verify with the target logits formed from the target
 * model's final hidden states instead of read from stored rows:
 *     target logit (row, v) = hidden[row, :] . lm_head[v, :]
 * (then scaled by inv_temp[b] like a stored row).  freeaitool.com "DeepSeek
 * DSpark complete guide" 6.3 passes the target's last hidden state and
 * projects it through the LM head locally, so O(vocab) rows need not move;
 * yage.ai "DSpark speculative decoding hardware scheduling" (variable-length
 * verify paragraph) lays the verified tokens of all requests out flat.
 * Here the projection runs on the tensor cores and its rows are reduced on
 * chip: no logit row of a verified position is ever written to memory.
 * Only the one correction / bonus row of each request ([B, V] fp32) lands
 * in the workspace, for the residual draw.
 *
 * Inputs
 *   hidden [n_target_rows, dm] bf16: the flattened verified positions'
 *       final hidden states (after the target's last normalisation);
 *       request b uses rows row_start[b] .. row_start[b] + L_b, and these
 *       row sets must be disjoint (a row claimed twice raises
 *       DSPARK_FLAG_BAD_LENGTH);
 *   lm_head [V, dm] bf16: the target's output projection (no bias);
 *   dm: a multiple of 64, at most 16384;
 *   everything else exactly as for dspark_verify (target_logits replaced by
 *   hidden and lm_head).
 * Outputs, ownership, status word: as for dspark_verify.  Rows of hidden
 * that no request verifies are projected too (their results are dropped):
 * pass only the verified positions' states.  The head is read once per
 * 2048 hidden rows.
 */
dspark_status dspark_verify_lmhead(
    const void *hidden, const void *lm_head, int dm, int64_t n_target_rows,
    const int64_t *row_start, const int32_t *verify_len, const float *base_logits,
    const void *U, const void *W, dspark_dtype uw_dtype, int V, int r, int B, int K,
    const int32_t *prev_token, const float *inv_temp, const int32_t *tokens,
    const float *p_tok, const float *ref_max, const float *ref_sum, const float *draft_bias,
    const float *u_accept, const float *u_resample, int32_t *n_accepted, int32_t *out_tokens,
    int32_t *last_token, void *workspace, size_t ws_bytes, void *stream);

/*
 * dspark_verify without a workspace argument (the pages have no counterpart;
 * this is a convenience of this library).
 *
 * Who needs it: callers that cannot call cudaMalloc -- plugins whose host
 * application owns every device allocation and hands out no scratch, and
 * runtimes that run under a fixed device-memory budget decided before the
 * first step.  They still own and pass all inputs and outputs; only the
 * scratch is provided here.
 *
 * Scratch: a fixed 2 MiB array inside the library image, held by every GPU
 * that loads the library until the process exits.  Problems whose
 * dspark_verify_workspace_size exceeds 2 MiB are rejected with
 * DSPARK_ERR_UNSUPPORTED before anything is enqueued (at V = 151936 that
 * is about B <= 50 requests; B <= 16, K <= 16 always fits).
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and caches it.  The
 * function allocates nothing (no cudaMalloc, no cudaFree, no allocating
 * library call).
 *
 * Sharing: every call on a device uses the same array and leaves its
 * contents behind; each call clears the part that must start at zero (the
 * status word).  Calls whose kernels overlap on the GPU (different streams
 * without ordering) race on the array and give wrong results; order them.
 * Device-side data checks clamp bad values and record them in a status
 * word inside the array: dspark_verify_noalloc_status reads it.
 *
 * Arguments and results: exactly those of dspark_verify, minus workspace and
 * ws_bytes.
 */
dspark_status dspark_verify_noalloc(
    const float *target_logits, int64_t n_target_rows, const int64_t *row_start,
    const int32_t *verify_len, const float *base_logits, const void *U,
    const void *W, dspark_dtype uw_dtype, int V, int r, int B, int K,
    const int32_t *prev_token, const float *inv_temp, const int32_t *tokens,
    const float *p_tok, const float *ref_max, const float *ref_sum,
    const float *draft_bias, const float *u_accept, const float *u_resample,
    int32_t *n_accepted, int32_t *out_tokens, int32_t *last_token, void *stream);

/* Status of the last dspark_verify_noalloc call on the current device:
 * synchronises `stream` (the stream that call used) and maps the status
 * word of the built-in scratch like dspark_get_device_status:
 * DSPARK_OK, DSPARK_ERR_TIMEOUT (a device wait ran out) or
 * DSPARK_ERR_DEVICE_DATA (bad token ids, lengths, rows or temperatures were
 * clamped).  The next call on the device overwrites the word. */
dspark_status dspark_verify_noalloc_status(void *stream);

/* ---------------------------------------------------------------------- */
/* status                                                                  */
/* ---------------------------------------------------------------------- */

/* Synchronises `stream`, reads the status word of `workspace` and maps it
 * to DSPARK_OK / DSPARK_ERR_TIMEOUT / DSPARK_ERR_DEVICE_DATA. */
dspark_status dspark_get_device_status(const void *workspace, void *stream);

/* Synchronises `stream`; returns the status word of the last call made
 * with this workspace, low 31 bits (the DSPARK_FLAG_* bits), or -1 on a
 * CUDA error.  A workspace no call has used yet holds no status word: what
 * this returns for it is meaningless. */
int dspark_get_device_flags(const void *workspace, void *stream);

/* Test hook of the timeout path (no counterpart on the pages).  With
 * skew != 0 the first record exchange of the persistent draft for one or
 * two requests ("persistent-cuda-core") and the record exchange of the
 * single-launch verify wait for records that never arrive: their bounded
 * waits run out (after 2 s and at least 4096 polls), the call sets
 * DSPARK_FLAG_TIMEOUT in its status word, finishes its work with
 * meaningless outputs and leaves the device usable.  skew = 0, the default,
 * restores normal operation.  Synchronises the current device and sets it
 * for that device only. */
dspark_status dspark_test_set_exchange_skew(int skew);

/* Static string for a status code. */
const char *dspark_status_string(dspark_status s);

/* Name of the draft projection path these sizes take:
 * "persistent-cuda-core" (bf16, r = 256, B <= 2: all K positions in one
 * launch, GEMV on the CUDA cores), "tcgen05-persistent" (bf16, B <= 16: all
 * K positions in one launch), "tcgen05" (bf16, B > 16: one launch per
 * position) or "cuda-core" (fp32 U/W, or shapes outside those paths). */
const char *dspark_draft_path(int V, int r, int B, int K, dspark_dtype uw_dtype);

/* Name of the path dspark_verify takes for these sizes, with (have_bias
 * != 0) or without the draft's bias rows: "single-launch" (B <= 4, at most
 * 72 verified rows, bias rows given: one cooperative kernel), "staged-bias"
 * (four kernels, the residual row rebuilt from the bias rows),
 * "staged-tcgen05" or "staged-cuda-core" (four kernels, the residual row
 * re-projected from U and W on the tensor or CUDA cores).  Same results
 * either way, up to floating-point summation order. */
const char *dspark_verify_path(int V, int r, int B, int K, dspark_dtype uw_dtype, int have_bias);

/* Name of the path the prefix calls take for B*K candidates with the
 * scheduler on (enable != 0) or off: "multi-cta" (more than 1024 candidates,
 * scheduler on: a survival kernel, then a rank kernel over about B*K / 63
 * CTAs whose last CTA runs the scan) or "single-cta" (one kernel, one CTA).
 * Same results either way. */
const char *dspark_prefix_path(int B, int K, int enable);

/* Library ABI version (major*100 + minor). */
int dspark_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H_ */
