/*
 * dspark_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, double-precision CPU statement of DSpark's per-step
 * speculative-decoding hot path: the Markov-head draft, the
 * confidence-scheduled prefix cut and the lossless rejection-sampling
 * verify.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library
 * shares no code, header, table or helper with it, and neither side
 * includes or calls the other.
 *
 * Sources (page title, section):
 *   [yage]       yage.ai, "DSpark speculative decoding hardware scheduling":
 *                the first-order Markov head paragraph (the formula
 *                p(x_k|x_{k-1}) = softmax(base_logit_k + transition_bias)),
 *                the rejection-sampling paragraph (exact per-token p_d),
 *                the SPS(B) scheduler paragraph (rank by calibrated
 *                survival, stop before throughput drops).
 *   [freeaitool] freeaitool.com, "DeepSeek DSpark complete guide":
 *                section 3.1 (Markov head, rank-256 low-rank transition),
 *                section 4.1 (confidence head c_k, sequential temperature
 *                scaling), section 4.2 (greedy ordering + early stop).
 *   [legalagi]   legalagi.cn, "读懂 DSpark：一个律师外行眼里的 DeepSeek 推理新论文":
 *                section 三 (draft -> verify -> keep the longest accepted
 *                prefix; lossless), section 五 (early stop keeps it lossless).
 * The accept/residual/bonus rule itself is the textbook speculative
 * sampling rule (Leviathan, Kalman & Matias 2023; Chen et al. 2023): the
 * pages only say that verification compares draft and target
 * probabilities and needs the exact p_d.
 *
 * Parity status (what pins each function; the tests live in
 * tests/test_oracle_pins.py, tests/test_oracle_sts_pins.py,
 * tests/test_oracle_async_pins.py, tests/test_oracle_lmhead_pins.py and
 * tests/test_oracle_rnn_pins.py):
 *   oracle_draft_row / oracle_draft : pinned (W=0 reduces to independent
 *       categorical sampling checked against numpy searchsorted; a
 *       constructed deterministic transition chain; exact enumeration of
 *       the Markov chain on V=4, K=3 against a 10^6-sample histogram; a
 *       hand-worked V=4 inverse CDF).
 *   oracle_prefix : pinned (flat / steep cost limits, T_k=1 reduces to the
 *       logistic function, prefix property, linear cost without knee equals
 *       the argmax over prefix lengths of the sorted survival list).
 *   oracle_verify : pinned (p_d = p_t accepts everything, E[accept] =
 *       1 - TV, chi-square losslessness on V=8 at positions 1 and 2, exact
 *       E[n_acc] by enumeration).
 *   oracle_verify_lmhead : pinned (an identity head reproduces the verify
 *       on the hidden rows; small-integer hidden states and head make the
 *       product exact, and the result equals the verify on it bit for bit,
 *       in fp32 and in bf16, and under H*2, E/2).
 *   oracle_draft_rnn / oracle_verify_rnn : pinned (R = 0 reduces the head
 *       to the Markov head on tanh(U); at small amplitude the logits equal
 *       the linear recurrence's to third order; the state carries the token
 *       before the previous one exactly when R != 0; equal target and draft
 *       rows accept everything; chi-square losslessness of the verify).
 *   oracle_prefix_async / oracle_cost_stair_ms : pinned (hand lookups on
 *       a staircase table; a budget commits exactly the top candidates of a
 *       numpy lexsort of the survival order; the greedy N as budget
 *       reproduces the greedy cut; clamping; a stair-edge stop).
 *   oracle_sts_fit : pinned (recovers the temperature that generated
 *       logistic labels on a large sample; agrees with a dense grid search
 *       of the likelihood; z -> a*z gives T -> a*T; separable data ends on
 *       the temperature bounds; unreached positions do not move the fit;
 *       hand-worked ECEs).
 *
 * Numerical conventions (stated once, used everywhere):
 *   - inputs are read exactly (fp32 and bf16 values are exact in double);
 *   - 1/T is supplied by the caller as an fp32 value and used as is;
 *   - inverse CDF: the smallest index i with C_i > u*Z, where C_i is the
 *     running sum of the weights; if rounding leaves no such i, the last
 *     index with non-zero weight;
 *   - margin of a draw = min(u*Z - C_{i-1}, C_i - u*Z) / Z.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* scalar helpers                                                      */
/* ------------------------------------------------------------------ */

static double bf16_value(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* element (row, col) of a [rows, r] matrix stored as fp32 or bf16 */
static double mat_at(const void *m, int is_bf16, int r, long row, int col)
{
    if (is_bf16)
        return bf16_value(((const uint16_t *)m)[row * (long)r + col]);
    return (double)((const float *)m)[row * (long)r + col];
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* draft                                                               */
/* ------------------------------------------------------------------ */

/*
 * One draft distribution row, as logits:
 *   l_v = (base_v + sum_i U[x_prev, i] * W[v, i]) * inv_temp
 * [yage, Markov-head paragraph]: the transition bias is a lookup of the
 * previous token in a V x V low-rank matrix, here U[x_prev] . W^T with
 * rank r ([freeaitool 3.1]).  x_prev < 0 means "no previous token": the
 * bias is left out.
 */
void oracle_draft_row(const float *base_row, const void *U, const void *W,
                      int uw_bf16, int V, int r, int x_prev, double inv_temp,
                      double *logits)
{
    double *u = NULL;
    if (x_prev >= 0) {
        u = (double *)malloc(sizeof(double) * (size_t)r);
        for (int i = 0; i < r; ++i)
            u[i] = mat_at(U, uw_bf16, r, x_prev, i);
    }
    for (int v = 0; v < V; ++v) {
        double bias = 0.0;
        if (u) {
            for (int i = 0; i < r; ++i)
                bias += u[i] * mat_at(W, uw_bf16, r, v, i);
        }
        logits[v] = ((double)base_row[v] + bias) * inv_temp;
    }
    free(u);
}

/* softmax weights w_v = exp(l_v - max l); returns Z = sum w, sets *m */
static double softmax_weights(const double *l, int V, double *w, double *m)
{
    double mx = -INFINITY;
    for (int v = 0; v < V; ++v)
        if (l[v] > mx)
            mx = l[v];
    double z = 0.0;
    for (int v = 0; v < V; ++v) {
        w[v] = exp(l[v] - mx);
        z += w[v];
    }
    *m = mx;
    return z;
}

/* inverse CDF over weights w (total Z): smallest i with C_i > u*Z */
static int inverse_cdf(const double *w, int V, double total, double u,
                       double *margin)
{
    double target = u * total;
    double c = 0.0;
    for (int v = 0; v < V; ++v) {
        double prev = c;
        c += w[v];
        if (c > target) {
            double a = target - prev, b = c - target;
            *margin = (a < b ? a : b) / total;
            return v;
        }
    }
    /* rounding left no crossing: last index with non-zero weight */
    for (int v = V - 1; v >= 0; --v)
        if (w[v] > 0.0) {
            *margin = 0.0;
            return v;
        }
    *margin = 0.0;
    return 0;
}

/*
 * The semi-autoregressive Markov-head draft for a batch of B requests,
 * K sequential positions each ([freeaitool 3.1]: parallel backbone gives
 * base logits for every position, the sequential head corrects them from
 * the token actually sampled at the previous position; [yage, Markov-head
 * paragraph] for the formula).
 *
 *   base       [B, K, V] fp32        base_logit_k per request and position
 *   U, W       [V, r] fp32 or bf16   low-rank transition factors
 *   prev_token [B]                   token before position 1 (<0: no bias)
 *   inv_temp   [B] or NULL           fp32 1/T_b (NULL: 1)
 *   u_draft    [B, K]                uniforms in [0, 1)
 * outputs
 *   tokens [B, K], p_tok [B, K] = p_d(x_k), lse [B, K] = log sum exp(l),
 *   margin [B, K] = CDF margin of each draw.
 */
int oracle_draft(const float *base, const void *U, const void *W, int uw_bf16,
                 int V, int r, int B, int K, const int32_t *prev_token,
                 const float *inv_temp, const float *u_draft, int32_t *tokens,
                 double *p_tok, double *lse, double *margin)
{
    if (V <= 0 || r <= 0 || B < 0 || K < 0)
        return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        double *l = (double *)malloc(sizeof(double) * (size_t)V);
        double *w = (double *)malloc(sizeof(double) * (size_t)V);
        double it = inv_temp ? (double)inv_temp[b] : 1.0;
        int x = prev_token[b];
        for (int k = 0; k < K; ++k) {
            const float *brow = base + ((size_t)b * K + k) * (size_t)V;
            oracle_draft_row(brow, U, W, uw_bf16, V, r, x, it, l);
            double m;
            double z = softmax_weights(l, V, w, &m);
            double mg;
            int xk = inverse_cdf(w, V, z, (double)u_draft[(size_t)b * K + k], &mg);
            size_t o = (size_t)b * K + k;
            tokens[o] = xk;
            p_tok[o] = w[xk] / z;
            lse[o] = m + log(z);
            margin[o] = mg;
            x = xk;
        }
        free(l);
        free(w);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* RNN sequential head                                                 */
/* ------------------------------------------------------------------ */

/*
 * [freeaitool 3.1] names two sequential heads on top of the parallel
 * backbone: the Markov head above, which sees only the previous token, and
 * an optional RNN head that keeps a recurrent state and so captures longer
 * dependencies.  The page gives no formula for it.  Reading taken: the
 * plainest recurrent state in the same rank-r space as the Markov head's
 * lookup (Elman form), whose previous-token input is that lookup:
 *     s_{-1} = h0[b]            (zeros when h0 is NULL)
 *     x_{-1} = prev_token[b]
 *     s_k    = tanh(R s_{k-1} + U[x_{k-1}])   (U[x] left out when x < 0)
 *     l_v    = (base[b, k, v] + s_k . W[v]) * inv_temp
 * and softmax and inverse-CDF sampling exactly as in the Markov head.
 * p_d(x_k | x_{<k}) is still one softmax over the vocabulary, so it is
 * exact, as the rejection-sampling verify needs ([yage, rejection-sampling
 * paragraph]); the state is a deterministic function of the sampled
 * prefix.  With R = 0 and h0 = 0 the head is the Markov head on tanh(U).
 *
 *   R  [r, r] in the dtype of U and W; (R s)_i = sum_j R[i, j] s_j
 *   h0 [B, r] fp32 or NULL
 * outputs as oracle_draft, plus states [B, K, r] (s_k) when not NULL.
 */
static void rnn_step(const void *U, const void *R, int uw_bf16, int r, int x_prev,
                     const double *s_prev, double *s_out)
{
    for (int i = 0; i < r; ++i) {
        double acc = 0.0;
        for (int j = 0; j < r; ++j)
            acc += mat_at(R, uw_bf16, r, i, j) * s_prev[j];
        if (x_prev >= 0)
            acc += mat_at(U, uw_bf16, r, x_prev, i);
        s_out[i] = tanh(acc);
    }
}

/* one draft row of the RNN head from its state: (base_v + s . W[v]) / T */
static void rnn_row(const float *base_row, const void *W, int uw_bf16, int V, int r,
                    const double *s, double inv_temp, double *logits)
{
    for (int v = 0; v < V; ++v) {
        double bias = 0.0;
        for (int i = 0; i < r; ++i)
            bias += s[i] * mat_at(W, uw_bf16, r, v, i);
        logits[v] = ((double)base_row[v] + bias) * inv_temp;
    }
}

/* the state before position j: s_{j} from h0, prev_token and x_0..x_{j-1} */
static void rnn_state_at(const void *U, const void *R, int uw_bf16, int r, const float *h0b,
                         int x_prev0, const int32_t *toks, int j, double *s, double *tmp)
{
    for (int i = 0; i < r; ++i)
        tmp[i] = h0b ? (double)h0b[i] : 0.0;
    int x = x_prev0;
    for (int p = 0; p <= j; ++p) {
        rnn_step(U, R, uw_bf16, r, x, tmp, s);
        memcpy(tmp, s, sizeof(double) * (size_t)r);
        if (p < j)
            x = toks[p];
    }
}

int oracle_draft_rnn(const float *base, const void *U, const void *W, const void *R,
                     int uw_bf16, int V, int r, int B, int K, const int32_t *prev_token,
                     const float *h0, const float *inv_temp, const float *u_draft,
                     int32_t *tokens, double *p_tok, double *lse, double *margin,
                     double *states)
{
    if (V <= 0 || r <= 0 || B < 0 || K < 0 || !R)
        return 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        double *l = (double *)malloc(sizeof(double) * (size_t)V);
        double *w = (double *)malloc(sizeof(double) * (size_t)V);
        double *sp = (double *)malloc(sizeof(double) * (size_t)r);
        double *sn = (double *)malloc(sizeof(double) * (size_t)r);
        double it = inv_temp ? (double)inv_temp[b] : 1.0;
        for (int i = 0; i < r; ++i)
            sp[i] = h0 ? (double)h0[(size_t)b * r + i] : 0.0;
        int x = prev_token[b];
        for (int k = 0; k < K; ++k) {
            rnn_step(U, R, uw_bf16, r, x, sp, sn);
            if (states)
                memcpy(states + ((size_t)b * K + k) * (size_t)r, sn, sizeof(double) * (size_t)r);
            const float *brow = base + ((size_t)b * K + k) * (size_t)V;
            rnn_row(brow, W, uw_bf16, V, r, sn, it, l);
            double m;
            double z = softmax_weights(l, V, w, &m);
            double mg;
            int xk = inverse_cdf(w, V, z, (double)u_draft[(size_t)b * K + k], &mg);
            size_t o = (size_t)b * K + k;
            tokens[o] = xk;
            p_tok[o] = w[xk] / z;
            lse[o] = m + log(z);
            margin[o] = mg;
            x = xk;
            memcpy(sp, sn, sizeof(double) * (size_t)r);
        }
        free(l);
        free(w);
        free(sp);
        free(sn);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* confidence-scheduled prefix cut                                     */
/* ------------------------------------------------------------------ */

/*
 * Cost (ms) of a verify batch of n tokens: piecewise-linear interpolation
 * of the profiled table (tokens ascending), extended linearly from the
 * first and last segments.  [yage, SPS(B) paragraph]: the throughput
 * profile is measured at start-up and consulted by the scheduler.
 */
double oracle_cost_ms(const float *xs, const float *ys, int n, double tokens)
{
    int i = 0;
    while (i < n - 2 && tokens > (double)xs[i + 1])
        ++i;
    double x0 = xs[i], x1 = xs[i + 1], y0 = ys[i], y1 = ys[i + 1];
    return y0 + (y1 - y0) * (tokens - x0) / (x1 - x0);
}

/*
 * Staircase reading of the same table ([yage], engineering paragraph: the
 * real throughput curve SPS(B) jumps in steps, because of tensor-core
 * alignment and cache limits): a batch of n tokens costs the entry of the
 * smallest profiled size that holds it, ys[i] for the first i with
 * xs[i] >= n (ys[0] at or below xs[0]); past the last entry the cost grows
 * along the last segment's slope.
 */
double oracle_cost_stair_ms(const float *xs, const float *ys, int n, double tokens)
{
    if (tokens > (double)xs[n - 1])
        return ys[n - 1] + ((double)ys[n - 1] - ys[n - 2]) * (tokens - xs[n - 1]) /
                               ((double)xs[n - 1] - xs[n - 2]);
    int i = 0;
    while ((double)xs[i] < tokens)
        ++i;
    return ys[i];
}

static double cost_mode(const float *xs, const float *ys, int n, int staircase, double tokens)
{
    return staircase ? oracle_cost_stair_ms(xs, ys, n, tokens)
                     : oracle_cost_ms(xs, ys, n, tokens);
}

typedef struct {
    double s;
    int k;
    int b;
} cand_t;

/* survival descending, then position ascending, then request ascending */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    if (a->k != b->k) return a->k < b->k ? -1 : 1;
    if (a->b != b->b) return a->b < b->b ? -1 : 1;
    return 0;
}

/*
 * [freeaitool 4.1]: c_k in (0,1) is the probability that position k is
 * accepted given every earlier position was; sequential temperature
 * scaling calibrates it position by position, applied here as
 * c_k = sigmoid(z_k / T_k).  [yage, SPS(B) paragraph]: the survival of a
 * draft token together with everything before it is the running product
 * S_k = prod_{j<=k} c_j; all requests' candidates are ranked by it, the
 * most probable added first, stopping before the batch-size cost makes
 * the throughput fall ([freeaitool 4.2] greedy ordering + early stop;
 * [legalagi 五] the early stop keeps the method lossless).
 *
 * Objective: expected emitted tokens per ms, E / t(N), with N the verify
 * tokens (every request verifies at least one position, so N starts at
 * B) and E the expected emitted tokens (every request emits at least one
 * token, so E starts at B).  A candidate is committed while it strictly
 * raises the objective; the first one that does not ends the scan.
 *
 * outputs: c, S [B, K]; L [B] = committed positions per request;
 * objective = E / t(N) of the committed set; margin = relative objective
 * gap at the stopping decision (+inf when every candidate was taken).
 *
 * Asynchronous budget ([yage], engineering paragraph): the number of
 * tokens a step verifies is decided from the confidences of two steps
 * back, while which tokens fill it is decided by the current confidences.
 * With budget >= 0 (verify tokens N, one per request included) the first
 * budget - B candidates of the current order are committed (clamped to
 * [0, B*K]); the order is survival-descending and survival never rises
 * along k, so the set is a prefix of every request's draft.  margin is
 * then the relative survival gap at the cut.  n_greedy always returns N of
 * the greedy scan on the current confidences: the budget for two steps
 * later.  staircase selects the cost reading (see oracle_cost_stair_ms).
 */
int oracle_prefix_async(const float *z, const float *temps, const float *cost_tokens,
                        const float *cost_ms, int n_pts, int staircase, int B, int K,
                        int enable, int budget, double *c, double *S, int32_t *L,
                        double *objective, double *margin, int *n_greedy)
{
    if (B < 0 || K < 0 || n_pts < 2)
        return 1;
    for (int b = 0; b < B; ++b) {
        double run = 1.0;
        for (int k = 0; k < K; ++k) {
            size_t o = (size_t)b * K + k;
            double ck = 1.0 / (1.0 + exp(-(double)z[o] / (double)temps[k]));
            run *= ck;
            c[o] = ck;
            S[o] = run;
        }
    }
    if (!enable) {
        double E = B;
        for (size_t o = 0; o < (size_t)B * K; ++o)
            E += S[o];
        for (int b = 0; b < B; ++b)
            L[b] = K;
        *objective = E / cost_mode(cost_tokens, cost_ms, n_pts, staircase,
                                   (double)B + (double)B * K);
        *margin = INFINITY;
        *n_greedy = B + B * K;
        return 0;
    }
    size_t n = (size_t)B * K;
    cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (n ? n : 1));
    for (int b = 0; b < B; ++b)
        for (int k = 0; k < K; ++k) {
            size_t o = (size_t)b * K + k;
            cand[o].s = S[o];
            cand[o].k = k;
            cand[o].b = b;
        }
    qsort(cand, n, sizeof(cand_t), cand_cmp);
    /* the greedy scan: commit while the objective strictly rises */
    double E = B, N = B;
    double obj = E / cost_mode(cost_tokens, cost_ms, n_pts, staircase, N);
    double gmargin = INFINITY;
    size_t stop = n;
    for (size_t i = 0; i < n; ++i) {
        double E2 = E + cand[i].s, N2 = N + 1.0;
        double obj2 = E2 / cost_mode(cost_tokens, cost_ms, n_pts, staircase, N2);
        if (!(obj2 > obj)) {
            gmargin = fabs(obj2 - obj) / obj;
            stop = i;
            break;
        }
        E = E2;
        N = N2;
        obj = obj2;
    }
    *n_greedy = B + (int)stop;
    size_t m = stop;
    *margin = gmargin;
    if (budget >= 0) {
        long want = (long)budget - B;
        m = want < 0 ? 0 : ((size_t)want > n ? n : (size_t)want);
        *margin = (m == 0 || m == n) ? INFINITY
                                     : (cand[m - 1].s - cand[m].s) / cand[m - 1].s;
    }
    for (int b = 0; b < B; ++b)
        L[b] = 0;
    double Em = B;
    for (size_t i = 0; i < m; ++i) {
        L[cand[i].b] += 1;
        Em += cand[i].s;
    }
    *objective = Em / cost_mode(cost_tokens, cost_ms, n_pts, staircase, (double)B + (double)m);
    free(cand);
    return 0;
}

int oracle_prefix(const float *z, const float *temps, const float *cost_tokens,
                  const float *cost_ms, int n_pts, int B, int K, int enable,
                  double *c, double *S, int32_t *L, double *objective,
                  double *margin)
{
    int n_greedy;
    return oracle_prefix_async(z, temps, cost_tokens, cost_ms, n_pts, 0, B, K, enable, -1, c, S,
                               L, objective, margin, &n_greedy);
}

/* ------------------------------------------------------------------ */
/* verify                                                              */
/* ------------------------------------------------------------------ */

/*
 * Rejection-sampling verify of one step ([legalagi 三]: the target checks
 * the whole draft in one pass and the longest accepted prefix is kept;
 * [yage, rejection-sampling paragraph]: the check compares draft and
 * target probabilities, which is why p_d must be exact).  Textbook rule:
 * position k is accepted iff u_acc < p_t(x_k) / p_d(x_k); at the first
 * rejected position j the replacement token is drawn from
 * normalize(max(0, p_t - p_d)); if all L_b positions are accepted a bonus
 * token is drawn from the target row after them.  The same uniform
 * u_res[b] serves the residual draw or the bonus draw (only one happens).
 * If the residual mass is zero the draw falls back to p_t.
 *
 *   target     rows [n_rows, V] fp32; request b, position p (0-based)
 *              reads row row_start[b] + p, p = 0..L_b (row L_b: bonus)
 *   verify_len [B] L_b in [0, K]
 *   base, U, W, prev_token, inv_temp  as for oracle_draft (used to
 *              rebuild the full draft row at the rejected position)
 *   tokens [B, K], p_d [B, K]  the draft's tokens and their probabilities
 *   u_accept [B, K], u_res [B]
 * outputs
 *   n_acc [B]; out_tokens [B, K+1] (accepted tokens, then the
 *   correction/bonus token, then -1); accept_margin [B] = min |u - ratio|
 *   over the tested positions (+inf if none); res_margin [B] = CDF margin
 *   of the correction/bonus draw.
 */
/*
 * Where the verify's target logits come from: stored rows [n_rows, V], or
 * the target model's final hidden states [n_rows, dm] times its LM head
 * [V, dm] (row v of the head gives vocabulary entry v), accumulated in fp64
 * from the exact stored values.  [freeaitool] 6.3: the target's last hidden
 * state is passed on instead of its vocabulary-sized distribution and the
 * LM-head projection is done locally, O(hidden) instead of O(vocab); here
 * the same projection is applied to the verify's flattened rows ([yage],
 * variable-length verify paragraph), so the logit rows need not exist in
 * memory.  Either way the row is scaled by 1/T after it is formed.
 */
typedef struct {
    const float *logits;   /* [n_rows, V], or NULL */
    const void *hidden;    /* [n_rows, dm] */
    const void *lm_head;   /* [V, dm] */
    int dm, bf16;
} target_src_t;

static void target_row(const target_src_t *t, int64_t row, int V, double it, double *lt)
{
    if (t->logits) {
        const float *trow = t->logits + (size_t)row * (size_t)V;
        for (int v = 0; v < V; ++v)
            lt[v] = (double)trow[v] * it;
        return;
    }
    for (int v = 0; v < V; ++v) {
        double acc = 0.0;
        for (int i = 0; i < t->dm; ++i)
            acc += mat_at(t->hidden, t->bf16, t->dm, (long)row, i) *
                   mat_at(t->lm_head, t->bf16, t->dm, (long)v, i);
        lt[v] = acc * it;
    }
}

/* Where the verify's draft row at the rejected position comes from: the
 * Markov head (R NULL: U[x_{j-1}] . W) or the RNN head (its state s_j,
 * rebuilt from h0, the previous token and the drafted tokens before j). */
typedef struct {
    const void *R;    /* [r, r] or NULL */
    const float *h0;  /* [B, r] or NULL */
} draft_src_t;

static int verify_core(const target_src_t *src, const draft_src_t *dsrc, int64_t n_rows,
                       const int64_t *row_start,
                       const int32_t *verify_len, const float *base, const void *U,
                       const void *W, int uw_bf16, int V, int r, int B, int K,
                       const int32_t *prev_token, const float *inv_temp,
                       const int32_t *tokens, const double *p_d,
                       const float *u_accept, const float *u_res, int32_t *n_acc,
                       int32_t *out_tokens, double *accept_margin,
                       double *res_margin)
{
    for (int b = 0; b < B; ++b) {
        int L = verify_len[b];
        if (L < 0 || L > K || row_start[b] < 0 || row_start[b] + L >= n_rows)
            return 2;
    }
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int b = 0; b < B; ++b) {
        double *lt = (double *)malloc(sizeof(double) * (size_t)V);
        double *pt = (double *)malloc(sizeof(double) * (size_t)V);
        double *ld = (double *)malloc(sizeof(double) * (size_t)V);
        double *pd = (double *)malloc(sizeof(double) * (size_t)V);
        int L = verify_len[b];
        double it = inv_temp ? (double)inv_temp[b] : 1.0;
        int n = 0, rejected = 0;
        double amg = INFINITY;
        for (int p = 0; p < L; ++p) {
            target_row(src, row_start[b] + p, V, it, lt);
            double m;
            double zt = softmax_weights(lt, V, pt, &m);
            int x = tokens[(size_t)b * K + p];
            if (x < 0 || x >= V) {
                bad = 1;
                break;
            }
            double ratio = (pt[x] / zt) / p_d[(size_t)b * K + p];
            double u = (double)u_accept[(size_t)b * K + p];
            double d = fabs(u - ratio);
            if (d < amg)
                amg = d;
            if (u < ratio) {
                ++n;
            } else {
                rejected = 1;
                break;
            }
        }
        int j = n; /* position of the correction (or bonus) token */
        target_row(src, row_start[b] + j, V, it, lt);
        double m;
        double zt = softmax_weights(lt, V, pt, &m);
        for (int v = 0; v < V; ++v)
            pt[v] /= zt;
        int tok;
        double mg;
        double u = (double)u_res[b];
        if (rejected) {
            int xp = (j == 0) ? prev_token[b] : tokens[(size_t)b * K + j - 1];
            const float *brow = base + ((size_t)b * K + j) * (size_t)V;
            if (dsrc && dsrc->R) {
                double *st = (double *)malloc(sizeof(double) * (size_t)r * 2);
                rnn_state_at(U, dsrc->R, uw_bf16, r,
                             dsrc->h0 ? dsrc->h0 + (size_t)b * r : NULL, prev_token[b],
                             tokens + (size_t)b * K, j, st, st + r);
                rnn_row(brow, W, uw_bf16, V, r, st, it, ld);
                free(st);
            } else {
                oracle_draft_row(brow, U, W, uw_bf16, V, r, xp, it, ld);
            }
            double md;
            double zd = softmax_weights(ld, V, pd, &md);
            double q = 0.0;
            for (int v = 0; v < V; ++v) {
                double d = pt[v] - pd[v] / zd;
                pd[v] = d > 0.0 ? d : 0.0; /* reuse pd as the residual */
                q += pd[v];
            }
            if (q > 0.0)
                tok = inverse_cdf(pd, V, q, u, &mg);
            else
                tok = inverse_cdf(pt, V, 1.0, u, &mg);
        } else {
            tok = inverse_cdf(pt, V, 1.0, u, &mg);
        }
        int32_t *out = out_tokens + (size_t)b * (K + 1);
        for (int p = 0; p < K + 1; ++p)
            out[p] = -1;
        for (int p = 0; p < n; ++p)
            out[p] = tokens[(size_t)b * K + p];
        out[n] = tok;
        n_acc[b] = n;
        accept_margin[b] = amg;
        res_margin[b] = mg;
        free(lt);
        free(pt);
        free(ld);
        free(pd);
    }
    return bad ? 3 : 0;
}

int oracle_verify(const float *target, int64_t n_rows, const int64_t *row_start,
                  const int32_t *verify_len, const float *base, const void *U,
                  const void *W, int uw_bf16, int V, int r, int B, int K,
                  const int32_t *prev_token, const float *inv_temp,
                  const int32_t *tokens, const double *p_d,
                  const float *u_accept, const float *u_res, int32_t *n_acc,
                  int32_t *out_tokens, double *accept_margin,
                  double *res_margin)
{
    target_src_t src = {target, NULL, NULL, 0, 0};
    return verify_core(&src, NULL, n_rows, row_start, verify_len, base, U, W, uw_bf16, V, r, B, K,
                       prev_token, inv_temp, tokens, p_d, u_accept, u_res, n_acc, out_tokens,
                       accept_margin, res_margin);
}

/* The verify with the target logits formed from hidden states and the LM
 * head (see target_src_t); hidden [n_rows, dm] and lm_head [V, dm] are both
 * bf16 (hm_bf16 = 1, uint16 bit patterns) or both fp32. */
int oracle_verify_lmhead(const void *hidden, const void *lm_head, int dm, int hm_bf16,
                         int64_t n_rows, const int64_t *row_start,
                         const int32_t *verify_len, const float *base, const void *U,
                         const void *W, int uw_bf16, int V, int r, int B, int K,
                         const int32_t *prev_token, const float *inv_temp,
                         const int32_t *tokens, const double *p_d,
                         const float *u_accept, const float *u_res, int32_t *n_acc,
                         int32_t *out_tokens, double *accept_margin,
                         double *res_margin)
{
    if (dm < 1)
        return 1;
    target_src_t src = {NULL, hidden, lm_head, dm, hm_bf16};
    return verify_core(&src, NULL, n_rows, row_start, verify_len, base, U, W, uw_bf16, V, r, B, K,
                       prev_token, inv_temp, tokens, p_d, u_accept, u_res, n_acc, out_tokens,
                       accept_margin, res_margin);
}


/* The verify of an RNN-head draft: the draft row at the rejected position
 * is the RNN head's (its state rebuilt from h0 and the drafted prefix). */
int oracle_verify_rnn(const float *target, int64_t n_rows, const int64_t *row_start,
                      const int32_t *verify_len, const float *base, const void *U,
                      const void *W, const void *R, int uw_bf16, int V, int r, int B, int K,
                      const int32_t *prev_token, const float *h0, const float *inv_temp,
                      const int32_t *tokens, const double *p_d, const float *u_accept,
                      const float *u_res, int32_t *n_acc, int32_t *out_tokens,
                      double *accept_margin, double *res_margin)
{
    if (!R)
        return 1;
    target_src_t src = {target, NULL, NULL, 0, 0};
    draft_src_t dsrc = {R, h0};
    return verify_core(&src, &dsrc, n_rows, row_start, verify_len, base, U, W, uw_bf16, V, r, B,
                       K, prev_token, inv_temp, tokens, p_d, u_accept, u_res, n_acc, out_tokens,
                       accept_margin, res_margin);
}

/* ------------------------------------------------------------------------
 * Sequential temperature scaling of the confidence head
 * ([freeaitool] section 4.1: c_k estimates the probability that draft token
 * k is accepted given that every earlier one was; the raw scores are
 * over-confident and are calibrated after training by a temperature per
 * position, fitted from left to right, which brings the expected
 * calibration error from 3-8 % to about 1 %.  [yage] scheduler paragraph:
 * the calibration uses an offline set and aligns the estimated
 * probabilities with the observed acceptance rates.)
 *
 * Reading.  The offline set holds N sequences with head scores z[n, k] and
 * the accepted-prefix length n_acc[n] of a full-block verify.  Position j
 * (0-based) of sequence n is observed when n_acc[n] >= j (every earlier
 * token was accepted) and accepted when n_acc[n] > j.  T_j minimises the
 * Bernoulli negative log-likelihood of the observed labels under
 * c = 1 / (1 + exp(-z / T_j)); positions are taken left to right, each on
 * the sequences that reached it.
 *
 * Procedure.  With theta = 1/T the likelihood is convex in theta: its
 * derivative g(theta) = sum (sigma(theta z) - y) z is non-decreasing, with
 * slope h(theta) = sum sigma(theta z) (1 - sigma(theta z)) z^2 >= 0.  theta
 * is kept in [1/T_MAX, 1/T_MIN]: g >= 0 at the lower bound or <= 0 at the
 * upper bound puts the minimiser on that bound.  Otherwise, from theta = 1,
 * each step evaluates g and h and narrows the bracket [lo, hi] (values of
 * theta) by the sign of g.  The search ends when g = 0, when the Newton
 * step -g/h moves theta by at most STS_TOL relative (the step is then
 * taken), or after STS_ITERS steps; otherwise theta becomes theta - g/h, or
 * the bracket's geometric midpoint sqrt(lo * hi) when h is not positive or
 * the step leaves the bracket.  A position with no observed sample,
 * or with only z = 0 (every temperature fits equally), gets T = 1.
 * Samples whose z is not finite are left out.
 *
 * ECE: observed (n, j) pairs pooled, STS_BINS equal-width bins of c on
 * [0, 1] (bin = floor(c * STS_BINS), the top edge in the last bin);
 * ECE = sum over bins of |sum of labels - sum of c| / (number of pairs).
 * ------------------------------------------------------------------------ */
#define STS_T_MIN 0.05
#define STS_T_MAX 20.0
#define STS_ITERS 40
#define STS_TOL 1e-13
#define STS_BINS 15

static double logistic(double x) { return 1.0 / (1.0 + exp(-x)); }

/* derivative (and its slope) of the position-j likelihood at theta; also
 * the number of observed samples and whether any observed z is non-zero */
static double sts_grad(const float *z, const int32_t *n_acc, long N, int K, int j,
                       double theta, double *slope, long *count, int *nonzero)
{
    double g = 0.0, h = 0.0;
    long c = 0;
    int nz = 0;
    for (long n = 0; n < N; ++n) {
        if (n_acc[n] < j)
            continue;
        const double zz = z[n * K + j];
        if (!isfinite(zz))
            continue;
        const double y = n_acc[n] > j ? 1.0 : 0.0;
        const double s = logistic(theta * zz);
        g += (s - y) * zz;
        h += s * (1.0 - s) * zz * zz;
        ++c;
        nz |= zz != 0.0;
    }
    if (slope)
        *slope = h;
    if (count)
        *count = c;
    if (nonzero)
        *nonzero = nz;
    return g;
}

static double sts_ece(const float *z, const int32_t *n_acc, long N, int K,
                      const double *theta)
{
    double sc[STS_BINS] = {0}, sy[STS_BINS] = {0};
    long total = 0;
    for (long n = 0; n < N; ++n) {
        for (int j = 0; j < K && j <= n_acc[n]; ++j) {
            const double zz = z[n * K + j];
            if (!isfinite(zz))
                continue;
            const double c = logistic(theta[j] * zz);
            int m = (int)(c * STS_BINS);
            if (m > STS_BINS - 1)
                m = STS_BINS - 1;
            sc[m] += c;
            sy[m] += n_acc[n] > j ? 1.0 : 0.0;
            ++total;
        }
    }
    if (total == 0)
        return 0.0;
    double e = 0.0;
    for (int m = 0; m < STS_BINS; ++m)
        e += fabs(sy[m] - sc[m]);
    return e / (double)total;
}

/* temps[K] (the fitted T_j), ece[2] (before: every T = 1; after: the fitted
 * temperatures), count[K] (observed samples per position).  n_acc values
 * are clamped to [0, K].  Returns 0, or 1 on bad sizes. */
int oracle_sts_fit(const float *z, const int32_t *n_acc_in, long N, int K, double *temps,
                   double *ece, long *count)
{
    if (N < 0 || K < 1)
        return 1;
    int32_t *n_acc = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    for (long n = 0; n < N; ++n)
        n_acc[n] = n_acc_in[n] < 0 ? 0 : (n_acc_in[n] > K ? K : n_acc_in[n]);
    double *theta = (double *)malloc(sizeof(double) * (size_t)K);
    for (int j = 0; j < K; ++j) {
        long c = 0;
        int nz = 0;
        double lo = 1.0 / STS_T_MAX, hi = 1.0 / STS_T_MIN;
        const double g_lo = sts_grad(z, n_acc, N, K, j, lo, NULL, &c, &nz);
        double th;
        if (c == 0 || !nz) {
            th = 1.0;
        } else if (g_lo >= 0.0) {
            th = lo;
        } else if (sts_grad(z, n_acc, N, K, j, hi, NULL, NULL, NULL) <= 0.0) {
            th = hi;
        } else {
            th = 1.0;
            for (int it = 0; it < STS_ITERS; ++it) {
                double h;
                const double g = sts_grad(z, n_acc, N, K, j, th, &h, NULL, NULL);
                if (g == 0.0)
                    break;
                if (g < 0.0)
                    lo = th;
                else
                    hi = th;
                const double newton = th - g / h;
                if (h > 0.0 && fabs(newton - th) <= STS_TOL * th) {
                    th = newton;
                    break;
                }
                th = (h > 0.0 && newton > lo && newton < hi) ? newton : sqrt(lo * hi);
            }
        }
        theta[j] = th;
        temps[j] = 1.0 / th;
        if (count)
            count[j] = c;
    }
    double *ones = (double *)malloc(sizeof(double) * (size_t)K);
    for (int j = 0; j < K; ++j)
        ones[j] = 1.0;
    ece[0] = sts_ece(z, n_acc, N, K, ones);
    ece[1] = sts_ece(z, n_acc, N, K, theta);
    free(ones);
    free(theta);
    free(n_acc);
    return 0;
}
