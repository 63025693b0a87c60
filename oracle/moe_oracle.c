/*
 * Plain CPU oracle for the forward pass of a token-choice Mixture-of-Experts
 * layer.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's
 * CPU-baseline leg may call it; the product path never does.
 *
 * Everything is computed in double precision, one token at a time, in the
 * order the pages state the method.  Inputs arrive in their storage type
 * (fp32, or bf16 given as raw 16-bit patterns) and are widened exactly to
 * double.  Nothing here is shared with the CUDA library: no header, no helper,
 * no table.
 *
 * Sources (page titles as cited throughout):
 *   [Lab18]  "Lab 18 - Mixture of experts", sections 1-3 and "What to implement"
 *   [Lab01]  "Lab 01 - Router, Load Balancing, Capacity & the MoE Layer",
 *            "Where to start" and "The traps"
 *   [CS336]  "Mixture of Experts - parameters without the FLOPs", section 2
 *   [Lec4]   cs336 lecture 4 field map, "Stability, fine-tuning, and upcycling"
 *
 * Status codes returned: 0 ok, 2 bad shape, 3 capacity factor below 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_SHAPE 2
#define OR_ERR_CAPACITY_FACTOR 3

/* storage type codes of x and of the expert weights */
#define OR_F32 0
#define OR_BF16 1

static double widen(const void *p, int64_t i, int dtype)
{
    if (dtype == OR_F32)
        return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16; /* bf16 = top half of an fp32 */
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Router: logits, scores, top-k, gates.                                     */
/* ------------------------------------------------------------------------ */

/*
 * Per token t (row of x):
 *   z = x W_r (+ logit_bias)                         [Lab18 sec. 1, eq. for z;
 *                                                     CS336 sec. 2 router listing]
 *   softmax: p = exp(z - max z) / sum exp(z - max z)  (stable; [Lab01] step 1)
 *            lse = max z + log sum exp(z - max z)     ([Lab18 sec. 2] z-loss term)
 *   sigmoid: s = 1 / (1 + exp(-z))                   ([Lab18] DeepSeek-V3 note)
 *   selection key: p (softmax) or s + select_bias (sigmoid; the bias is used
 *   for selection only, [Lab18 sec. 2] auxiliary-loss-free balancing)
 *   top-k: the k largest keys, best first; equal keys go to the lower expert
 *   index ([Lab01] traps: break ties by expert index)
 *   gates: renormalized g_j = v_j / sum_sel v when renorm, else raw g_j = v_j,
 *   with v = p or s ([Lab18 sec. 1] gate values); renorm < 0 means "renormalize
 *   exactly when k > 1" (the lab's MoE).
 *
 * Outputs (all optional except topk and gates): z[T*E], scores[T*E] (p or s),
 * topk[T*k], gates[T*k], lse[T].
 */
int oracle_route(int T, int d, int E, int k, int score, int renorm,
                 const void *x, int xdtype, const float *W_r,
                 const float *logit_bias, const float *select_bias,
                 double *z_out, double *scores_out, int32_t *topk,
                 double *gates, double *lse_out)
{
    if (T < 0 || d < 1 || E < 1 || k < 1 || k > E)
        return OR_ERR_SHAPE;
    int do_renorm = renorm < 0 ? (k > 1) : renorm;
    /* tokens are independent: the loop runs on OpenMP threads when available */
#pragma omp parallel
    {
    double *z = malloc(sizeof(double) * E);
    double *v = malloc(sizeof(double) * E);
    double *key = malloc(sizeof(double) * E);
    int *order = malloc(sizeof(int) * E);
#pragma omp for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += widen(x, (int64_t)t * d + c, xdtype) * (double)W_r[(int64_t)c * E + e];
            if (logit_bias)
                acc += (double)logit_bias[e];
            z[e] = acc;
        }
        double m = z[0];
        for (int e = 1; e < E; ++e)
            if (z[e] > m)
                m = z[e];
        double sum = 0.0;
        for (int e = 0; e < E; ++e)
            sum += exp(z[e] - m);
        double lse = m + log(sum);
        for (int e = 0; e < E; ++e) {
            if (score == 0)
                v[e] = exp(z[e] - m) / sum;
            else
                v[e] = 1.0 / (1.0 + exp(-z[e]));
            key[e] = v[e] + ((score == 1 && select_bias) ? (double)select_bias[e] : 0.0);
        }
        /* stable insertion sort of expert indices by key, descending: equal
         * keys keep ascending index order, which is the lower-index tie-break */
        for (int e = 0; e < E; ++e) {
            int i = e;
            while (i > 0 && key[order[i - 1]] < key[e]) {
                order[i] = order[i - 1];
                --i;
            }
            order[i] = e;
        }
        double sel = 0.0;
        for (int j = 0; j < k; ++j)
            sel += v[order[j]];
        for (int j = 0; j < k; ++j) {
            topk[(int64_t)t * k + j] = order[j];
            gates[(int64_t)t * k + j] = do_renorm ? v[order[j]] / sel : v[order[j]];
        }
        if (z_out)
            for (int e = 0; e < E; ++e)
                z_out[(int64_t)t * E + e] = z[e];
        if (scores_out)
            for (int e = 0; e < E; ++e)
                scores_out[(int64_t)t * E + e] = v[e];
        if (lse_out)
            lse_out[t] = lse;
    }
    free(z);
    free(v);
    free(key);
    free(order);
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Capacity.                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * C = ceil(capacity_factor * T k / E)   ([Lab18 sec. 3] capacity formula),
 * held at T when it exceeds T.  A factor below 1 is an error ([Lab01] traps).
 * An infinite factor means no limit; C = T then suffices because a token's k
 * experts are distinct.
 */
int oracle_capacity_value(int T, int E, int k, double cf, int64_t *C)
{
    if (T < 0 || E < 1 || k < 1 || k > E)
        return OR_ERR_SHAPE;
    if (!(cf >= 1.0))
        return OR_ERR_CAPACITY_FACTOR;
    if (isinf(cf)) {
        *C = T;
        return OR_OK;
    }
    /* A token's k experts are distinct, so no expert receives more than T
     * assignments and any C >= T keeps them all: C is held at T, which keeps
     * the integer conversion defined for huge finite factors. */
    const double c = ceil(cf * (double)((int64_t)T * k) / (double)E);
    *C = c >= (double)T ? (int64_t)T : (int64_t)c;
    return OR_OK;
}

/*
 * Walk the T*k assignments in priority order, one per-expert counter each:
 * position = counter++, kept while position < C ([Lab18 sec. 3]).
 *   priority 0: token order, first come first served ([Lab01] step 4)
 *   priority 1: rank-major, every first choice before any second choice, then
 *               token order within a rank ([Lab18 sec. 3], GShard)
 * counts[e] is the number of assignments routed to e before any drop.
 * dropped[t] = 1 when every assignment of token t was dropped.
 * C is given directly here, as the pages' capacity_mask takes it.
 */
int oracle_capacity_walk(int T, int E, int k, int64_t C, int priority,
                         const int32_t *topk, int32_t *counts, int32_t *pos,
                         uint8_t *keep, uint8_t *dropped,
                         int64_t *n_dropped_assignments)
{
    if (T < 0 || E < 1 || k < 1 || k > E || C < 0)
        return OR_ERR_SHAPE;
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    int64_t A = (int64_t)T * k;
    for (int64_t n = 0; n < A; ++n) {
        int64_t t, j;
        if (priority == 0) {
            t = n / k;
            j = n % k;
        } else {
            j = n / (T > 0 ? T : 1);
            t = n % (T > 0 ? T : 1);
        }
        int64_t a = t * k + j;
        int e = topk[a];
        if (e < 0 || e >= E)
            return OR_ERR_SHAPE;
        pos[a] = counts[e]++;
        keep[a] = (uint8_t)(pos[a] < C);
    }
    int64_t nd = 0;
    for (int t = 0; t < T; ++t) {
        int any = 0;
        for (int j = 0; j < k; ++j) {
            any |= keep[(int64_t)t * k + j];
            nd += !keep[(int64_t)t * k + j];
        }
        dropped[t] = (uint8_t)!any;
    }
    if (n_dropped_assignments)
        *n_dropped_assignments = nd;
    return OR_OK;
}

/* the same walk with C from the capacity factor */
int oracle_capacity(int T, int E, int k, double cf, int priority,
                    const int32_t *topk, int64_t *C_out, int32_t *counts,
                    int32_t *pos, uint8_t *keep, uint8_t *dropped,
                    int64_t *n_dropped_assignments)
{
    int64_t C;
    int st = oracle_capacity_value(T, E, k, cf, &C);
    if (st != OR_OK)
        return st;
    if (C_out)
        *C_out = C;
    return oracle_capacity_walk(T, E, k, C, priority, topk, counts, pos, keep,
                                dropped, n_dropped_assignments);
}

/*
 * Batch-prioritized capacity ([Lab18 sec. 3]: V-MoE ranks the assignments by
 * router score).  The T*k assignments are walked from the highest router
 * score down, equal scores in token order and then slot order, with the same
 * per-expert counters as above.  sel_scores[t*k + j] is the router's score of
 * the expert chosen in slot j (softmax probability p, or sigmoid affinity s
 * without the selection bias), given in fp32: the ranking is a decision and
 * is taken in the precision the scores are stored in.
 */
struct scored_assignment {
    float score;
    int64_t a;
};

static int by_score_then_index(const void *l, const void *r)
{
    const struct scored_assignment *x = l, *y = r;
    if (x->score != y->score)
        return x->score > y->score ? -1 : 1;
    return x->a < y->a ? -1 : (x->a > y->a ? 1 : 0);
}

int oracle_capacity_walk_scored(int T, int E, int k, int64_t C, const int32_t *topk,
                                const float *sel_scores, int32_t *counts, int32_t *pos,
                                uint8_t *keep, uint8_t *dropped,
                                int64_t *n_dropped_assignments)
{
    if (T < 0 || E < 1 || k < 1 || k > E || C < 0)
        return OR_ERR_SHAPE;
    int64_t A = (int64_t)T * k;
    struct scored_assignment *order = malloc(sizeof *order * (A > 0 ? A : 1));
    if (!order)
        return OR_ERR_SHAPE;
    for (int64_t a = 0; a < A; ++a) {
        if (topk[a] < 0 || topk[a] >= E || sel_scores[a] != sel_scores[a]) {
            free(order);
            return OR_ERR_SHAPE;
        }
        order[a].score = sel_scores[a];
        order[a].a = a;
    }
    qsort(order, (size_t)A, sizeof *order, by_score_then_index);
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t n = 0; n < A; ++n) {
        int64_t a = order[n].a;
        int e = topk[a];
        pos[a] = counts[e]++;
        keep[a] = (uint8_t)(pos[a] < C);
    }
    free(order);
    int64_t nd = 0;
    for (int t = 0; t < T; ++t) {
        int any = 0;
        for (int j = 0; j < k; ++j) {
            any |= keep[(int64_t)t * k + j];
            nd += !keep[(int64_t)t * k + j];
        }
        dropped[t] = (uint8_t)!any;
    }
    if (n_dropped_assignments)
        *n_dropped_assignments = nd;
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Balancing losses.                                                         */
/* ------------------------------------------------------------------------ */

/*
 * Switch load-balance loss, without the coefficient alpha:
 *   L_aux = E * sum_i f_i P_i,  f_i = counts_i / (T k)  (share of the T k slots,
 *   [Lab01] step 3), P_i = mean over tokens of the full router probability of
 *   expert i ([Lab18 sec. 2]; common bugs: never the renormalized gates).
 *   For sigmoid scores, P_i uses s_i / sum_j s_j per token.
 * Router z-loss: L_z = (1/T) sum_t lse_t^2 ([Lab18 sec. 2], ST-MoE).
 * scores[T*E] are the p (or s) values oracle_route wrote.
 */
int oracle_losses(int T, int E, int k, int score, const double *scores,
                  const int32_t *counts, const double *lse, double *aux,
                  double *zloss)
{
    if (T < 1 || E < 1 || k < 1)
        return OR_ERR_SHAPE;
    double total = 0.0;
    for (int i = 0; i < E; ++i) {
        double P = 0.0;
        for (int t = 0; t < T; ++t) {
            double pi = scores[(int64_t)t * E + i];
            if (score == 1) {
                double row = 0.0;
                for (int j = 0; j < E; ++j)
                    row += scores[(int64_t)t * E + j];
                pi /= row;
            }
            P += pi;
        }
        P /= (double)T;
        double f = (double)counts[i] / ((double)T * (double)k);
        total += f * P;
    }
    *aux = (double)E * total;
    double zs = 0.0;
    for (int t = 0; t < T; ++t)
        zs += lse[t] * lse[t];
    *zloss = zs / (double)T;
    return OR_OK;
}

/*
 * Sequence-wise balance loss: the loss above with one sequence as the
 * balancing unit ([Lec4] "Training a router you cannot differentiate": the
 * balancing unit is where the variants differ; DeepSeek-V3 keeps a small
 * sequence-wise loss beside its bias-based balancing, [Lab18 sec. 2]).
 * Tokens [b L, (b + 1) L) form sequence b; its f_i counts the assignments its
 * tokens sent to expert i (before capacity) over its L k slots and its P_i
 * averages its tokens' probabilities.  mean = average over the T / L
 * sequences; per_seq[b] (optional) = each sequence's value.
 */
int oracle_seq_losses(int T, int E, int k, int score, int L, const double *scores,
                      const int32_t *topk, double *mean, double *per_seq)
{
    if (T < 1 || E < 1 || k < 1 || k > E || L < 1 || T % L != 0)
        return OR_ERR_SHAPE;
    int B = T / L;
    int32_t *counts = malloc(sizeof(int32_t) * E);
    double *lse = calloc((size_t)L, sizeof(double));   /* z-loss part unused here */
    if (!counts || !lse) {
        free(counts);
        free(lse);
        return OR_ERR_SHAPE;
    }
    double total = 0.0;
    int st = OR_OK;
    for (int b = 0; b < B && st == OR_OK; ++b) {
        for (int e = 0; e < E; ++e)
            counts[e] = 0;
        for (int64_t a = (int64_t)b * L * k; a < (int64_t)(b + 1) * L * k; ++a) {
            if (topk[a] < 0 || topk[a] >= E) {
                st = OR_ERR_SHAPE;
                break;
            }
            counts[topk[a]]++;
        }
        if (st != OR_OK)
            break;
        double aux, zl;
        st = oracle_losses(L, E, k, score, scores + (int64_t)b * L * E, counts, lse, &aux, &zl);
        if (per_seq)
            per_seq[b] = aux;
        total += aux;
    }
    free(counts);
    free(lse);
    if (st == OR_OK)
        *mean = total / (double)B;
    return st;
}

/*
 * Auxiliary-loss-free balancing ([Lab18 sec. 2], DeepSeek-V3; [Lec4] "Training
 * a router you cannot differentiate"): after a step each expert's selection
 * bias moves by a fixed step gamma against its load, down for an overloaded
 * expert and up for an underloaded one, unchanged at exactly the balanced
 * load.  Load = counts_i, the assignments routed to expert i before capacity;
 * the balanced load T k / E is compared exactly, as E counts_i against T k.
 * The bias is an fp32 vector and each step is one fp32 addition.
 */
int oracle_bias_update(int T, int E, int k, const int32_t *counts, float gamma,
                       const float *bias_in, float *bias_out)
{
    if (T < 0 || E < 1 || k < 1 || k > E)
        return OR_ERR_SHAPE;
    int64_t balanced = (int64_t)T * k;
    for (int i = 0; i < E; ++i) {
        int64_t load = (int64_t)E * counts[i];
        float b = bias_in[i];
        float nb = b;
        if (load > balanced)
            nb = b - gamma;
        else if (load < balanced)
            nb = b + gamma;
        bias_out[i] = nb;
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* Expert FFNs and the gated combine.                                        */
/* ------------------------------------------------------------------------ */

/* exact GELU, 0.5 u (1 + erf(u / sqrt 2)) */
static double gelu(double u) { return 0.5 * u * (1.0 + erf(u / sqrt(2.0))); }
static double silu(double u) { return u / (1.0 + exp(-u)); }

/*
 * One expert FFN on one token x[d] into o[d].
 *   act 0: two-matrix GELU MLP, o = W2 gelu(W1 x)            ([Lab18 sec. 1])
 *   act 1: three-matrix SwiGLU, o = W2 (silu(W1 x) * (W3 x)) ([Lab18 sec. 1])
 * Layouts: W1, W3 [F][d] (row f holds hidden unit f's input weights),
 * W2 [d][F] (row c holds output c's weights); no biases.
 */
static void expert_ffn(int d, int F, int act, const double *x, const void *W1,
                       const void *W3, const void *W2, int64_t w13_base,
                       int64_t w2_base, int wdtype, double *h, double *o)
{
    for (int f = 0; f < F; ++f) {
        double a = 0.0;
        for (int c = 0; c < d; ++c)
            a += widen(W1, w13_base + (int64_t)f * d + c, wdtype) * x[c];
        if (act == 0) {
            h[f] = gelu(a);
        } else {
            double b = 0.0;
            for (int c = 0; c < d; ++c)
                b += widen(W3, w13_base + (int64_t)f * d + c, wdtype) * x[c];
            h[f] = silu(a) * b;
        }
    }
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int f = 0; f < F; ++f)
            acc += widen(W2, w2_base + (int64_t)c * F + f, wdtype) * h[f];
        o[c] = acc;
    }
}

/*
 * y for the listed tokens ([Lab18 sec. 1] y = sum over the top-k of g_i FFN_i(x);
 * [CS336 sec. 2] router listing):
 *   y_t = sum over slots j with keep[t,j] of gates[t,j] * FFN_{topk[t,j]}(x_t)
 *         + sum over shared experts s of FFN_s(x_t)
 * Slots are added in order j = 0..k-1, then the shared experts.  A dropped slot
 * contributes nothing and the surviving gates are not rescaled ([Lab18 sec. 3]);
 * a token with every slot dropped gets only the shared experts, or zero
 * (the caller's residual carries it, [Lab18] GPU scale-up listing).
 * Shared experts ([Lab18 sec. 1] DeepSeekMoE row; [Phase 02] concept map) use
 * Ws1/Ws3 [S][Fs][d] and Ws2 [S][d][Fs].
 * keep may be NULL (every slot kept).  Tokens are independent, so the loop
 * over them runs on OpenMP threads when the library was built with OpenMP.
 */
int oracle_ffn_tokens(int T, int d, int E, int k, int F, int act,
                      int n_shared, int Fs, const void *x, int xdtype,
                      const int32_t *topk, const double *gates,
                      const uint8_t *keep, const void *W1, const void *W3,
                      const void *W2, const void *Ws1, const void *Ws3,
                      const void *Ws2, int wdtype, const int32_t *tokens,
                      int n_tokens, double *y)
{
    if (d < 1 || E < 1 || k < 1 || k > E || F < 1 || n_shared < 0)
        return OR_ERR_SHAPE;
    if (act == 1 && (!W3 || (n_shared > 0 && !Ws3)))
        return OR_ERR_SHAPE;
    for (int n = 0; n < n_tokens; ++n)
        if (tokens[n] < 0 || tokens[n] >= T)
            return OR_ERR_SHAPE;
    int Fmax = F > Fs ? F : Fs;
#pragma omp parallel
    {
        double *xt = malloc(sizeof(double) * d);
        double *h = malloc(sizeof(double) * (Fmax > 0 ? Fmax : 1));
        double *o = malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
        for (int n = 0; n < n_tokens; ++n) {
            int t = tokens[n];
            double *yt = y + (int64_t)n * d;
            for (int c = 0; c < d; ++c) {
                xt[c] = widen(x, (int64_t)t * d + c, xdtype);
                yt[c] = 0.0;
            }
            for (int j = 0; j < k; ++j) {
                int64_t a = (int64_t)t * k + j;
                if (keep && !keep[a])
                    continue;
                int e = topk[a];
                expert_ffn(d, F, act, xt, W1, W3, W2, (int64_t)e * F * d,
                           (int64_t)e * d * F, wdtype, h, o);
                for (int c = 0; c < d; ++c)
                    yt[c] += gates[a] * o[c];
            }
            for (int s = 0; s < n_shared; ++s) {
                expert_ffn(d, Fs, act, xt, Ws1, Ws3, Ws2, (int64_t)s * Fs * d,
                           (int64_t)s * d * Fs, wdtype, h, o);
                for (int c = 0; c < d; ++c)
                    yt[c] += o[c];
            }
        }
        free(xt);
        free(h);
        free(o);
    }
    return OR_OK;
}

/* number of OpenMP threads the FFN loop uses (1 without OpenMP) */
int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
