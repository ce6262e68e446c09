/*
 * moe_oracle.c -- plain, slow, single-threaded CPU definition of one
 * DeepSeek-V3-style MoE layer forward.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path (combine_expert_ffn_b200/csrc),
 * and nothing in the product path may call it.
 *
 * What it computes, step by step, and where each step comes from:
 *   1. router affinity  s_i = sigmoid(x . e_i (+ o_i))   -- affinities feed
 *      top-k gating ["MoE + Expert-Parallel Overlap (Exp08)", Implemented];
 *      the sigmoid form is DeepSeek-V3's; that page's V4 form
 *      sqrt(softplus(.)) is the variant "affinity kind 1".  o_i is an
 *      optional per-expert logit offset (the skewed-load workload).
 *   2. selection bias  b_i = s_i + bias_i  (auxiliary-loss-free balancing:
 *      "per-expert bias updates", Exp08 Implemented) -- used to choose
 *      experts only, never to weight them.
 *   3. node-limited routing: experts are split into G contiguous groups
 *      (stand-ins for nodes; "four experts per GPU", deepnotes "The real
 *      cluster, and the mesh DeepSeek actually disclosed"); a token's experts
 *      lie in at most M groups ("moe-node-limited-routing", opening
 *      definition).  Group score = sum of the group's top-(K/M) biased
 *      affinities; the M best groups are kept; ties go to the lower index.
 *   4. top-K experts by b inside the kept groups, ordered by descending b
 *      then ascending index; gate w_j = s_j / sum_j s_j over the K chosen
 *      UNBIASED affinities (no routed scaling factor, no epsilon).
 *   5. dispatch: a stable counting sort of the T*K token copies by expert
 *      (tokens ascending inside each expert segment), with per-expert counts,
 *      offsets and the group-to-group send matrix ("send matrices",
 *      shivam2003 "5. Tail latency controls step time").  Source group of
 *      token t is t / (T/G).
 *   6. expert FFN: SwiGLU  y = W_d (SiLU(W_g x) * (W_u x)); the shared
 *      experts are always on with weight 1 ("shared experts (always active) +
 *      fine-grained routed experts", Exp08 Implemented).
 *   7. combine: out_t = sum_shared FFN_s(x_t) + sum_j w_j FFN_{e_j}(x_t).
 * Variants, each behind its own function or flag: the hash router, the
 * per-expert bias update, and the FP8 dispatch payload (the routed copies of
 * x travel as FP8 E4M3 with one fp32 scale per 128 values; "Compression has a
 * numerical price", shivam2003 section 4).
 *
 * All-core runs: oracle_layer_rows_mt hands contiguous shards of the token
 * rows to POSIX threads, each of which calls the unchanged single-threaded
 * oracle_layer_rows_ex on its shard.  Rows never interact, so the output is
 * the same bytes as one call over all rows; only the wall time changes.
 *
 * Arithmetic: dot products accumulate in double from the exact bf16/fp32
 * inputs; sigmoid and SiLU use libm exp() in double.  The selection steps
 * (2-4) and the gate weights are done in fp32 exactly as written above, so
 * that a GPU given the same fp32 affinities must reproduce them bit for bit.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EBADARG 1
#define ORC_EINDEX 2
#define ORC_ENOMEM 3

static double bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* b_i "beats" b_j: larger value, ties to the lower index. */
static int beats(float bi, int i, float bj, int j)
{
    return bi > bj || (bi == bj && i < j);
}

/* ------------------------------------------------------------------ 1 */
/* Router affinity of either kind from a double-precision logit:
 *   kind 0: sigmoid(L)                 (DeepSeek-V3)
 *   kind 1: sqrt(softplus(L)),  softplus(L) = log(1 + e^L)  ("MoE +
 *           Expert-Parallel Overlap (Exp08)", Implemented: top-k gating over
 *           Sqrt(Softplus(.)) affinities, the V4 change)
 * Rounded once to fp32. */
static float affinity_of(double L, int kind)
{
    if (kind == 1) {
        const double sp = L > 0.0 ? L + log1p(exp(-L)) : log1p(exp(L));
        return (float)sqrt(sp);
    }
    return (float)(1.0 / (1.0 + exp(-L)));
}

/* scores[r*E + i] = affinity(sum_k x[rows[r], k] * e[i, k] + off[i]) of the
 * given kind (0 or 1) for the listed token rows (rows == NULL: rows
 * 0..n_rows-1), the sum in double. */
int oracle_router_affinity(int n_rows, const int64_t *rows, int d, int E,
                           const uint16_t *x, const float *e, const float *off,
                           int kind, float *scores)
{
    if (n_rows < 0 || d <= 0 || E <= 0 || !x || !e || !scores || kind < 0 || kind > 1)
        return ORC_EBADARG;
    for (int r = 0; r < n_rows; ++r) {
        int64_t t = rows ? rows[r] : r;
        const uint16_t *xt = x + t * (int64_t)d;
        for (int i = 0; i < E; ++i) {
            const float *ei = e + (int64_t)i * d;
            double acc = 0.0;
            for (int k = 0; k < d; ++k)
                acc += bf16_value(xt[k]) * (double)ei[k];
            if (off)
                acc += (double)off[i];
            scores[(int64_t)r * E + i] = affinity_of(acc, kind);
        }
    }
    return ORC_OK;
}

/* scores[r*E + i] = sigmoid(sum_k x[rows[r], k] * e[i, k] + off[i]) for the
 * listed token rows (rows == NULL: rows 0..n_rows-1).  Rounded once to fp32. */
int oracle_router_scores(int n_rows, const int64_t *rows, int d, int E,
                         const uint16_t *x, const float *e, const float *off,
                         float *scores)
{
    return oracle_router_affinity(n_rows, rows, d, E, x, e, off, 0, scores);
}

/* ------------------------------------------------------------------ 2-4 */
/* Node-limited top-K selection for n_rows tokens whose fp32 affinities are
 * scores[n_rows, E].  Writes topk_idx[n_rows, K] and topk_w[n_rows, K].
 * If group_score != NULL it also receives the fp32 group scores [n_rows, G]. */
int oracle_select(int n_rows, int E, int G, int K, int M,
                  const float *scores, const float *bias,
                  int32_t *topk_idx, float *topk_w, float *group_score)
{
    if (n_rows < 0 || E <= 0 || G <= 0 || K <= 0 || M <= 0 || E % G || K % M)
        return ORC_EBADARG;
    const int gsz = E / G, kpg = K / M;
    if (kpg > gsz || M > G || !scores || !bias || !topk_idx || !topk_w)
        return ORC_EBADARG;

    float *b = malloc(sizeof(float) * E);
    float *gs = malloc(sizeof(float) * G);
    char *taken = malloc(E);
    char *gkeep = malloc(G);
    if (!b || !gs || !taken || !gkeep) {
        free(b); free(gs); free(taken); free(gkeep);
        return ORC_ENOMEM;
    }
    for (int t = 0; t < n_rows; ++t) {
        const float *s = scores + (int64_t)t * E;
        /* step 2: biased affinity, one fp32 add */
        for (int i = 0; i < E; ++i)
            b[i] = s[i] + bias[i];

        /* step 3a: group score = sum of the group's kpg largest b, added in
         * the order they are picked (descending b, ties to lower index) */
        memset(taken, 0, E);
        for (int g = 0; g < G; ++g) {
            float sum = 0.0f;
            for (int r = 0; r < kpg; ++r) {
                int best = -1;
                for (int i = g * gsz; i < (g + 1) * gsz; ++i)
                    if (!taken[i] && (best < 0 || beats(b[i], i, b[best], best)))
                        best = i;
                if (best < 0)
                    break; /* unreachable: kpg <= gsz was checked */
                taken[best] = 1;
                sum = (r == 0) ? b[best] : sum + b[best];
            }
            gs[g] = sum;
        }
        if (group_score)
            memcpy(group_score + (int64_t)t * G, gs, sizeof(float) * G);

        /* step 3b: keep the M best groups (ties to the lower group index) */
        memset(gkeep, 0, G);
        for (int r = 0; r < M; ++r) {
            int best = -1;
            for (int g = 0; g < G; ++g)
                if (!gkeep[g] && (best < 0 || beats(gs[g], g, gs[best], best)))
                    best = g;
            if (best < 0)
                break; /* unreachable: M <= G was checked */
            gkeep[best] = 1;
        }

        /* step 4: top-K experts by b among the kept groups, in pick order */
        memset(taken, 0, E);
        int32_t *idx = topk_idx + (int64_t)t * K;
        for (int j = 0; j < K; ++j) {
            int best = -1;
            for (int i = 0; i < E; ++i)
                if (gkeep[i / gsz] && !taken[i] &&
                    (best < 0 || beats(b[i], i, b[best], best)))
                    best = i;
            if (best < 0)
                break; /* unreachable: K <= M * gsz was checked */
            taken[best] = 1;
            idx[j] = best;
        }

        /* gate weights over the chosen UNBIASED affinities, fp32, slot order */
        float denom = 0.0f;
        for (int j = 0; j < K; ++j)
            denom += s[idx[j]];
        for (int j = 0; j < K; ++j)
            topk_w[(int64_t)t * K + j] = s[idx[j]] / denom;
    }
    free(b); free(gs); free(taken); free(gkeep);
    return ORC_OK;
}

/* ------------------------------------------------------------------ 5 */
/* Stable counting-sort dispatch of the T*K copies by expert.
 *   counts[E], offsets[E+1], send[G*G] (copies src-group -> expert-group),
 *   send_tok[G*G] (tokens src-group -> expert-group, each token counted once
 *   per destination group), perm_token[T*K] (token of each permuted row),
 *   inv_perm[T*K] (row of copy (t, j)).
 * Returns ORC_EINDEX for an expert id out of range or repeated in a token. */
int oracle_dispatch(int T, int E, int G, int K, const int32_t *topk_idx,
                    int32_t *counts, int32_t *offsets, int32_t *send,
                    int32_t *send_tok, int32_t *perm_token, int32_t *inv_perm)
{
    if (T < 0 || E <= 0 || G <= 0 || K <= 0 || E % G || (T > 0 && T % G))
        return ORC_EBADARG;
    const int gsz = E / G, tpg = T > 0 ? T / G : 1;
    for (int64_t c = 0; c < (int64_t)T * K; ++c)
        if (topk_idx[c] < 0 || topk_idx[c] >= E)
            return ORC_EINDEX;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < K; ++j)
            for (int q = 0; q < j; ++q)
                if (topk_idx[(int64_t)t * K + j] == topk_idx[(int64_t)t * K + q])
                    return ORC_EINDEX;

    memset(counts, 0, sizeof(int32_t) * E);
    for (int64_t c = 0; c < (int64_t)T * K; ++c)
        counts[topk_idx[c]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];

    int32_t *cursor = malloc(sizeof(int32_t) * E);
    char *hit = malloc(G);
    if (!cursor || !hit) {
        free(cursor); free(hit);
        return ORC_ENOMEM;
    }
    memcpy(cursor, offsets, sizeof(int32_t) * E);
    memset(send, 0, sizeof(int32_t) * G * G);
    memset(send_tok, 0, sizeof(int32_t) * G * G);
    for (int t = 0; t < T; ++t) {
        int src = t / tpg;
        memset(hit, 0, G);
        for (int j = 0; j < K; ++j) {
            int e = topk_idx[(int64_t)t * K + j];
            int row = cursor[e]++;
            perm_token[row] = t;
            inv_perm[(int64_t)t * K + j] = row;
            send[src * G + e / gsz]++;
            hit[e / gsz] = 1;
        }
        for (int g = 0; g < G; ++g)
            send_tok[src * G + g] += hit[g];
    }
    free(cursor); free(hit);
    return ORC_OK;
}

/* ------------------------------------------------------------------ 6 */
/* One SwiGLU FFN applied to one bf16 row, added into y[d] with weight w:
 *   y += w * Wd (SiLU(Wg x) * (Wu x)),  Wg/Wu [f_ff, d], Wd [d, ld_d] with
 *   the f_ff columns starting at column col0 (ld_d = row stride of Wd).
 * If round_h is set, h is rounded to bf16 (nearest even) before Wd. */
static void swiglu_row_acc(int d, int f_ff, const uint16_t *x,
                           const uint16_t *Wg, const uint16_t *Wu,
                           const uint16_t *Wd, int ld_d, int col0,
                           double w, int round_h, double *h, double *y)
{
    for (int f = 0; f < f_ff; ++f) {
        double u = 0.0, v = 0.0;
        const uint16_t *g = Wg + (int64_t)f * d, *p = Wu + (int64_t)f * d;
        for (int k = 0; k < d; ++k) {
            double xk = bf16_value(x[k]);
            u += xk * bf16_value(g[k]);
            v += xk * bf16_value(p[k]);
        }
        h[f] = u / (1.0 + exp(-u)) * v;
        if (round_h) {
            float hf = (float)h[f];
            uint32_t bits;
            memcpy(&bits, &hf, 4);
            bits += 0x7FFFu + ((bits >> 16) & 1u);
            bits &= 0xFFFF0000u;
            memcpy(&hf, &bits, 4);
            h[f] = hf;
        }
    }
    for (int o = 0; o < d; ++o) {
        double acc = 0.0;
        const uint16_t *dr = Wd + (int64_t)o * ld_d + col0;
        for (int f = 0; f < f_ff; ++f)
            acc += h[f] * bf16_value(dr[f]);
        y[o] += w * acc;
    }
}

/* y[d] = FFN_e(x_row) for one routed expert (Wg/Wu [d_ff,d], Wd [d,d_ff]). */
int oracle_ffn_row(int d, int d_ff, const uint16_t *x_row, const uint16_t *Wg,
                   const uint16_t *Wu, const uint16_t *Wd, int round_h, double *y)
{
    if (d <= 0 || d_ff <= 0 || !x_row || !Wg || !Wu || !Wd || !y)
        return ORC_EBADARG;
    double *h = malloc(sizeof(double) * d_ff);
    if (!h)
        return ORC_ENOMEM;
    memset(y, 0, sizeof(double) * d);
    swiglu_row_acc(d, d_ff, x_row, Wg, Wu, Wd, d_ff, 0, 1.0, round_h, h, y);
    free(h);
    return ORC_OK;
}

/* y[d] = sum over the n_shared shared experts of FFN_s(x_row); shared
 * weights Wsg/Wsu [n_shared, d_ff_s, d], Wsd [n_shared, d, d_ff_s]. */
int oracle_shared_row(int d, int n_shared, int d_ff_s, const uint16_t *x_row,
                      const uint16_t *Wsg, const uint16_t *Wsu,
                      const uint16_t *Wsd, int round_h, double *y)
{
    if (d <= 0 || n_shared < 0 || !x_row || !y)
        return ORC_EBADARG;
    memset(y, 0, sizeof(double) * d);
    if (n_shared == 0)
        return ORC_OK;
    if (d_ff_s <= 0 || !Wsg || !Wsu || !Wsd)
        return ORC_EBADARG;
    double *h = malloc(sizeof(double) * d_ff_s);
    if (!h)
        return ORC_ENOMEM;
    for (int s = 0; s < n_shared; ++s)
        swiglu_row_acc(d, d_ff_s, x_row,
                       Wsg + (int64_t)s * d_ff_s * d, Wsu + (int64_t)s * d_ff_s * d,
                       Wsd + (int64_t)s * d * d_ff_s, d_ff_s, 0, 1.0, round_h, h, y);
    free(h);
    return ORC_OK;
}

/* ------------------------------------------------------------------ 7 */
/* out[t, :] = y_shared[t, :] + sum_j w[t,j] * y_perm[inv_perm[t,j], :]
 * in double from bf16 rows (y_shared may be NULL). */
int oracle_combine(int T, int d, int K, int64_t n_perm_rows,
                   const uint16_t *y_perm, const int32_t *inv_perm,
                   const float *topk_w, const uint16_t *y_shared, double *out)
{
    if (T < 0 || d <= 0 || K <= 0 || !y_perm || !inv_perm || !topk_w || !out)
        return ORC_EBADARG;
    for (int t = 0; t < T; ++t) {
        double *o = out + (int64_t)t * d;
        for (int k = 0; k < d; ++k)
            o[k] = y_shared ? bf16_value(y_shared[(int64_t)t * d + k]) : 0.0;
        for (int j = 0; j < K; ++j) {
            int64_t row = inv_perm[(int64_t)t * K + j];
            if (row < 0 || row >= n_perm_rows)
                return ORC_EINDEX;
            double w = (double)topk_w[(int64_t)t * K + j];
            for (int k = 0; k < d; ++k)
                o[k] += w * bf16_value(y_perm[row * d + k]);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ 1-7 */
/* The whole layer for a list of token rows (routing is per token, so any
 * sample of tokens can be evaluated alone).  Routed expert weights come as
 * per-expert pointer arrays (Wg[e], Wu[e]: [d_ff, d]; Wd[e]: [d, d_ff]); an
 * entry may be NULL if no listed token selects that expert.
 * Outputs: out[n_rows, d] (double), topk_idx/topk_w [n_rows, K],
 * scores [n_rows, E] (may be NULL). */
int oracle_hash_route(int n_rows, const int64_t *token_ids, int E, int G, int K, int M,
                      int32_t *topk_idx, float *topk_w);

/* The layer for the listed rows with a chosen router:
 *   router 0: sigmoid affinities + node-limited top-K (DeepSeek-V3)
 *   router 1: sqrt(softplus) affinities + the same selection (V4)
 *   router 2: hash router keyed by token_ids[rows[r]] (or rows[r] when
 *             token_ids is NULL); e, off, bias unused, scores_out untouched. */
int oracle_fp8_quantize_row(int d, const uint16_t *x, uint8_t *q, float *scale);
int oracle_fp8_dequantize_row(int d, const uint8_t *q, const float *scale, uint16_t *x_hat);

/* payload 0: the routed experts read x; payload 1: they read the FP8 round
 * trip x_hat of the FP8 dispatch payload (shared experts always read x). */
int oracle_layer_rows_ex(int n_rows, const int64_t *rows,
                         int d, int E, int G, int K, int M, int d_ff,
                         int n_shared, int d_ff_s,
                         const uint16_t *x, const float *e, const float *off,
                         const float *bias, int router, const int64_t *token_ids, int payload,
                         const uint16_t *const *Wg, const uint16_t *const *Wu,
                         const uint16_t *const *Wd,
                         const uint16_t *Wsg, const uint16_t *Wsu, const uint16_t *Wsd,
                         int round_h, double *out, int32_t *topk_idx, float *topk_w,
                         float *scores_out)
{
    if (n_rows < 0 || !rows || !x || !Wg || !Wu || !Wd || !out || !topk_idx || !topk_w ||
        router < 0 || router > 2 || (router < 2 && (!e || !bias)) || payload < 0 ||
        payload > 1 || (payload == 1 && d % 128))
        return ORC_EBADARG;
    int rc = ORC_OK;
    float *scores = malloc(sizeof(float) * (size_t)E * (n_rows > 0 ? n_rows : 1));
    double *y = malloc(sizeof(double) * d);
    uint16_t *xq = malloc(sizeof(uint16_t) * d);
    uint8_t *q = malloc((size_t)d);
    float *qs = malloc(sizeof(float) * (size_t)(d / 128 + 1));
    if (!scores || !y || !xq || !q || !qs) {
        rc = ORC_ENOMEM;
        goto done;
    }
    if (router == 2) {
        for (int r = 0; r < n_rows && !rc; ++r) {
            const int64_t id = token_ids ? token_ids[rows[r]] : rows[r];
            rc = oracle_hash_route(1, &id, E, G, K, M, topk_idx + (int64_t)r * K,
                                   topk_w + (int64_t)r * K);
        }
    } else {
        rc = oracle_router_affinity(n_rows, rows, d, E, x, e, off, router, scores);
        if (!rc)
            rc = oracle_select(n_rows, E, G, K, M, scores, bias, topk_idx, topk_w, NULL);
    }
    if (rc)
        goto done;
    for (int r = 0; r < n_rows; ++r) {
        const uint16_t *xr = x + rows[r] * (int64_t)d;
        double *o = out + (int64_t)r * d;
        rc = oracle_shared_row(d, n_shared, d_ff_s, xr, Wsg, Wsu, Wsd, round_h, o);
        if (rc)
            goto done;
        const uint16_t *xe = xr;  /* the routed experts' input row */
        if (payload == 1) {
            oracle_fp8_quantize_row(d, xr, q, qs);
            oracle_fp8_dequantize_row(d, q, qs, xq);
            xe = xq;
        }
        for (int j = 0; j < K; ++j) {
            int ex = topk_idx[(int64_t)r * K + j];
            if (!Wg[ex] || !Wu[ex] || !Wd[ex]) {
                rc = ORC_EBADARG;
                goto done;
            }
            rc = oracle_ffn_row(d, d_ff, xe, Wg[ex], Wu[ex], Wd[ex], round_h, y);
            if (rc)
                goto done;
            double w = (double)topk_w[(int64_t)r * K + j];
            for (int k = 0; k < d; ++k)
                o[k] += w * y[k];
        }
    }
    if (scores_out && router != 2)
        memcpy(scores_out, scores, sizeof(float) * (size_t)E * n_rows);
done:
    free(scores);
    free(y);
    free(xq);
    free(q);
    free(qs);
    return rc;
}

/* ------------------------------------------------------------------ all-core driver */
struct layer_shard {
    int n_rows;
    const int64_t *rows;
    int d, E, G, K, M, d_ff, n_shared, d_ff_s;
    const uint16_t *x;
    const float *e, *off, *bias;
    int router;
    const int64_t *token_ids;
    int payload;
    const uint16_t *const *Wg, *const *Wu, *const *Wd;
    const uint16_t *Wsg, *Wsu, *Wsd;
    int round_h;
    double *out;
    int32_t *topk_idx;
    float *topk_w, *scores_out;
    int rc;
};

static void *layer_shard_run(void *arg)
{
    struct layer_shard *s = arg;
    s->rc = oracle_layer_rows_ex(s->n_rows, s->rows, s->d, s->E, s->G, s->K, s->M, s->d_ff,
                                 s->n_shared, s->d_ff_s, s->x, s->e, s->off, s->bias, s->router,
                                 s->token_ids, s->payload, s->Wg, s->Wu, s->Wd, s->Wsg, s->Wsu,
                                 s->Wsd, s->round_h, s->out, s->topk_idx, s->topk_w,
                                 s->scores_out);
    return NULL;
}

/* oracle_layer_rows_ex over n_threads contiguous shards of `rows`, one POSIX
 * thread each (n_threads <= 1: the calling thread alone).  Same arguments and
 * outputs as oracle_layer_rows_ex; returns the first nonzero shard status. */
int oracle_layer_rows_mt(int n_threads, int n_rows, const int64_t *rows,
                         int d, int E, int G, int K, int M, int d_ff,
                         int n_shared, int d_ff_s,
                         const uint16_t *x, const float *e, const float *off,
                         const float *bias, int router, const int64_t *token_ids, int payload,
                         const uint16_t *const *Wg, const uint16_t *const *Wu,
                         const uint16_t *const *Wd,
                         const uint16_t *Wsg, const uint16_t *Wsu, const uint16_t *Wsd,
                         int round_h, double *out, int32_t *topk_idx, float *topk_w,
                         float *scores_out)
{
    if (n_rows < 0 || !rows || !out || !topk_idx || !topk_w)
        return ORC_EBADARG;
    if (n_threads > n_rows)
        n_threads = n_rows;
    if (n_threads <= 1)
        return oracle_layer_rows_ex(n_rows, rows, d, E, G, K, M, d_ff, n_shared, d_ff_s, x, e,
                                    off, bias, router, token_ids, payload, Wg, Wu, Wd, Wsg, Wsu,
                                    Wsd, round_h, out, topk_idx, topk_w, scores_out);
    struct layer_shard *sh = calloc((size_t)n_threads, sizeof(*sh));
    pthread_t *th = calloc((size_t)n_threads, sizeof(*th));
    int *started = calloc((size_t)n_threads, sizeof(int));
    if (!sh || !th || !started) {
        free(sh);
        free(th);
        free(started);
        return ORC_ENOMEM;
    }
    int rc = ORC_OK;
    for (int i = 0; i < n_threads; ++i) {
        const int r0 = (int)((int64_t)n_rows * i / n_threads);
        const int r1 = (int)((int64_t)n_rows * (i + 1) / n_threads);
        struct layer_shard *s = &sh[i];
        s->n_rows = r1 - r0;
        s->rows = rows + r0;
        s->d = d; s->E = E; s->G = G; s->K = K; s->M = M; s->d_ff = d_ff;
        s->n_shared = n_shared; s->d_ff_s = d_ff_s;
        s->x = x; s->e = e; s->off = off; s->bias = bias;
        s->router = router; s->token_ids = token_ids; s->payload = payload;
        s->Wg = Wg; s->Wu = Wu; s->Wd = Wd;
        s->Wsg = Wsg; s->Wsu = Wsu; s->Wsd = Wsd;
        s->round_h = round_h;
        s->out = out + (int64_t)r0 * d;
        s->topk_idx = topk_idx + (int64_t)r0 * K;
        s->topk_w = topk_w + (int64_t)r0 * K;
        s->scores_out = scores_out ? scores_out + (int64_t)r0 * E : NULL;
        s->rc = ORC_OK;
        if (pthread_create(&th[i], NULL, layer_shard_run, s) == 0)
            started[i] = 1;
        else
            layer_shard_run(s); /* no thread: run the shard here */
    }
    for (int i = 0; i < n_threads; ++i) {
        if (started[i])
            pthread_join(th[i], NULL);
        if (!rc && sh[i].rc)
            rc = sh[i].rc;
    }
    free(sh);
    free(th);
    free(started);
    return rc;
}

int oracle_layer_rows(int n_rows, const int64_t *rows,
                      int d, int E, int G, int K, int M, int d_ff,
                      int n_shared, int d_ff_s,
                      const uint16_t *x, const float *e, const float *off,
                      const float *bias,
                      const uint16_t *const *Wg, const uint16_t *const *Wu,
                      const uint16_t *const *Wd,
                      const uint16_t *Wsg, const uint16_t *Wsu, const uint16_t *Wsd,
                      int round_h, double *out, int32_t *topk_idx, float *topk_w,
                      float *scores_out)
{
    return oracle_layer_rows_ex(n_rows, rows, d, E, G, K, M, d_ff, n_shared, d_ff_s, x, e, off,
                                bias, 0, NULL, 0, Wg, Wu, Wd, Wsg, Wsu, Wsd, round_h, out, topk_idx,
                                topk_w, scores_out);
}

/* ------------------------------------------------------------------ hash router */
/* "a hash router for early-layer emulation" (Exp08, Implemented).  The page
 * gives no formula; the reading used here keeps the node limit: the token's
 * M groups and, inside each, its K/M experts are drawn without replacement by
 * a partial Fisher-Yates shuffle driven by the public "lowbias32" integer hash
 * (C. Wellons) of the token id; every gate is 1/K. */
static uint32_t lowbias32(uint32_t x)
{
    x ^= x >> 16;
    x *= 0x7FEB352Du;
    x ^= x >> 15;
    x *= 0x846CA68Bu;
    x ^= x >> 16;
    return x;
}

uint32_t oracle_lowbias32(uint32_t x) { return lowbias32(x); }

/* m distinct values of [0, n) in draw order: step i swaps position i with
 * position i + (hash(seed ^ i * 0x9E3779B9) mod (n - i)) of the virtual array
 * a[k] = k and takes the value that lands at i. */
static int partial_shuffle(uint32_t n, uint32_t m, uint32_t seed, int32_t *out)
{
    uint32_t pos[64], val[64];
    int used = 0;
    if (m > n || m > 32)
        return ORC_EBADARG;
    for (uint32_t i = 0; i < m; ++i) {
        const uint32_t j = i + lowbias32(seed ^ (i * 0x9E3779B9u)) % (n - i);
        uint32_t vi = i, vj = j;
        int si = -1, sj = -1;
        for (int q = 0; q < used; ++q) {
            if (pos[q] == i) { vi = val[q]; si = q; }
            if (pos[q] == j) { vj = val[q]; sj = q; }
        }
        if (si < 0) { pos[used] = i; si = used++; }
        if (sj < 0 && j != i) { pos[used] = j; sj = used++; }
        val[si] = vj;
        if (j != i)
            val[sj] = vi;
        out[i] = (int32_t)vj;
    }
    return ORC_OK;
}

int oracle_hash_route(int n_rows, const int64_t *token_ids, int E, int G, int K, int M,
                      int32_t *topk_idx, float *topk_w)
{
    if (n_rows < 0 || E <= 0 || G <= 0 || K <= 0 || M <= 0 || E % G || K % M || M > G ||
        K / M > E / G || G > 64 || K > 32 || !topk_idx || !topk_w)
        return ORC_EBADARG;
    const int gsz = E / G, kpg = K / M;
    for (int r = 0; r < n_rows; ++r) {
        const uint64_t tau = token_ids ? (uint64_t)token_ids[r] : (uint64_t)r;
        const uint32_t s0 = lowbias32((uint32_t)tau ^ lowbias32((uint32_t)(tau >> 32) ^ 0x68E31DA4u));
        int32_t groups[64], local[32];
        if (partial_shuffle((uint32_t)G, (uint32_t)M, s0, groups))
            return ORC_EBADARG;
        for (int gi = 0; gi < M; ++gi) {
            const uint32_t g = (uint32_t)groups[gi];
            if (partial_shuffle((uint32_t)gsz, (uint32_t)kpg, lowbias32(s0 ^ ((g + 1u) * 0x85EBCA6Bu)), local))
                return ORC_EBADARG;
            for (int q = 0; q < kpg; ++q) {
                topk_idx[(int64_t)r * K + gi * kpg + q] = (int32_t)(g * gsz) + local[q];
                topk_w[(int64_t)r * K + gi * kpg + q] = 1.0f / (float)K;
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ bias update */
/* Auxiliary-loss-free balancing: "per-expert bias updates" (Exp08,
 * Implemented).  The step rule (DeepSeek-V3's sign rule; the step size is not
 * on the pages, so it is a parameter): an expert above the mean load
 * T*K/E moves down by gamma, one below moves up, one at the mean stays:
 *   bias_i <- bias_i + gamma * sign(T*K/E - counts_i)     (one fp32 add)
 * The comparison is exact: counts_i * E against T * K in integers. */
int oracle_bias_update(int E, int T, int K, const int32_t *counts, float gamma, float *bias)
{
    if (E <= 0 || T < 0 || K <= 0 || !counts || !bias)
        return ORC_EBADARG;
    const int64_t total = (int64_t)T * K;
    for (int i = 0; i < E; ++i) {
        const int64_t c = (int64_t)counts[i] * E;
        const float step = c < total ? gamma : (c > total ? -gamma : 0.0f);
        bias[i] = bias[i] + step;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ FP8 payload */
/* Lower-precision dispatch payload ("sending fewer bytes through
 * lower-precision activations ... quantization and dequantization add kernels
 * and error", shivam2003 "DeepSeek 8.7", section 4).  The pages fix neither
 * the format nor the scaling, so the reading is DeepSeek-V3's published
 * recipe: OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, S.1111.111 = NaN, largest finite 448) with one fp32 scale per
 * token and block of 128 channels:
 *   amax = max |x_i| over the block,  s = amax / 448  (fp32),
 *   q_i  = E4M3(x_i / s)   (fp32 division; nearest, ties to even mantissa;
 *                           |v| >= 448 saturates to 448; amax = 0 gives q = 0)
 * The expert GEMM consumes  x_hat_i = bf16(float(E4M3^-1(q_i)) * s)  (one fp32
 * multiply, then bf16 nearest-even).  Router and shared experts keep x. */
double oracle_e4m3_decode(uint8_t q)
{
    const int sgn = q >> 7, e = (q >> 3) & 15, m = q & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);          /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return sgn ? -v : v;
}

/* Nearest E4M3 code to a finite float by direct search over the 127
 * non-negative finite codes (ties to the even code), saturating at 448. */
uint8_t oracle_e4m3_encode(float f)
{
    const uint8_t sgn = signbit(f) ? 0x80 : 0x00;
    const double a = fabs((double)f);
    if (a >= 448.0)
        return sgn | 0x7E;
    int best = 0;
    double best_err = a;
    for (int c = 1; c <= 0x7E; ++c) {
        const double err = fabs(oracle_e4m3_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return sgn | (uint8_t)best;
}

static float bf16_round_float(float v)
{
    uint32_t bits;
    memcpy(&bits, &v, 4);
    bits += 0x7FFFu + ((bits >> 16) & 1u);
    bits &= 0xFFFF0000u;
    memcpy(&v, &bits, 4);
    return v;
}

/* Quantize one bf16 row of d values (d % 128 == 0): q[d] codes, scale[d/128]. */
int oracle_fp8_quantize_row(int d, const uint16_t *x, uint8_t *q, float *scale)
{
    if (d <= 0 || d % 128 || !x || !q || !scale)
        return ORC_EBADARG;
    for (int b = 0; b < d / 128; ++b) {
        float amax = 0.0f;
        for (int i = 0; i < 128; ++i) {
            const float v = fabsf((float)bf16_value(x[b * 128 + i]));
            if (v > amax)
                amax = v;
        }
        const float sc = amax / 448.0f;
        scale[b] = sc;
        for (int i = 0; i < 128; ++i) {
            const float v = (float)bf16_value(x[b * 128 + i]);
            q[b * 128 + i] = amax == 0.0f ? 0 : oracle_e4m3_encode(v / sc);
        }
    }
    return ORC_OK;
}

/* The bf16 row the expert GEMM sees: x_hat_i = bf16(decode(q_i) * s). */
int oracle_fp8_dequantize_row(int d, const uint8_t *q, const float *scale, uint16_t *x_hat)
{
    if (d <= 0 || d % 128 || !q || !scale || !x_hat)
        return ORC_EBADARG;
    for (int i = 0; i < d; ++i) {
        const float v = bf16_round_float((float)oracle_e4m3_decode(q[i]) * scale[i / 128]);
        uint32_t bits;
        memcpy(&bits, &v, 4);
        x_hat[i] = (uint16_t)(bits >> 16);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ expert parallelism */
/* Row placement of the dispatch all-to-all when the experts are split over
 * `world` ranks in contiguous blocks of El = E / world ("four experts per
 * GPU", deepnotes "The real cluster, and the mesh DeepSeek actually
 * disclosed"; the all-to-all of "moe-node-limited-routing", "Why all to all
 * dominates MoE step time").  Reading of the receive layout at owner o: its
 * experts in order; inside an expert, the copies of rank 0, then rank 1, ...,
 * each rank's in its token order.
 *   counts_all [world, E]: copies of rank r's tokens to expert e
 *   base [world, E] out:   first row of rank r's copies for e at owner(e)
 *   local_offsets [world, El + 1] out: segment starts of owner o's experts
 *                          (last entry: rows o receives)                    */
int oracle_ep_plan(int world, int E, const int32_t *counts_all, int32_t *base,
                   int32_t *local_offsets)
{
    if (world <= 0 || E <= 0 || E % world || !counts_all || !base || !local_offsets)
        return ORC_EBADARG;
    const int El = E / world;
    for (int o = 0; o < world; ++o) {
        int64_t row = 0;
        for (int i = 0; i < El; ++i) {
            const int e = o * El + i;
            local_offsets[o * (El + 1) + i] = (int32_t)row;
            for (int r = 0; r < world; ++r) {
                base[r * E + e] = (int32_t)row;
                row += counts_all[r * E + e];
            }
        }
        local_offsets[o * (El + 1) + El] = (int32_t)row;
    }
    return ORC_OK;
}

/* Token-level placement of the deduplicated dispatch.  With node-limited
 * routing a token's activations need to reach each of its (at most M) nodes
 * once and fan out to its experts there ("moe-node-limited-routing": the
 * limit bounds the nodes a token's activations must reach; the send_tok
 * matrix of the single-GPU dispatch counts exactly these token-node pairs).
 * For one rank's routing topk_idx [T, K], experts in contiguous blocks of
 * El = E / world per owner:
 *   tok_slot [T, world] out: position of token t among this rank's tokens
 *                            that have an expert at owner o, in token
 *                            order; -1 when t has none there
 *   tok_counts [world] out:  this rank's tokens sent to owner o            */
int oracle_ep_token_plan(int T, int K, int E, int world, const int32_t *topk_idx,
                         int32_t *tok_slot, int32_t *tok_counts)
{
    if (T < 0 || K <= 0 || E <= 0 || world <= 0 || E % world || !tok_counts ||
        (T > 0 && (!topk_idx || !tok_slot)))
        return ORC_EBADARG;
    const int El = E / world;
    for (int o = 0; o < world; ++o) tok_counts[o] = 0;
    for (int t = 0; t < T; ++t) {
        for (int o = 0; o < world; ++o) {
            int sends = 0;
            for (int j = 0; j < K; ++j) {
                const int e = topk_idx[(int64_t)t * K + j];
                if (e < 0 || e >= E) return ORC_EBADARG;
                if (e / El == o) sends = 1;
            }
            tok_slot[(int64_t)t * world + o] = sends ? tok_counts[o]++ : -1;
        }
    }
    return ORC_OK;
}

/* Receive rows of the deduplicated dispatch at owner o: the tokens of rank
 * 0, then rank 1, ..., each rank's in its token order.  From tok_counts_all
 * [world, world] (row r = rank r's tok_counts): tok_base [world, world] out,
 * tok_base[r][o] = first row of rank r's tokens at owner o.                */
int oracle_ep_token_base(int world, const int32_t *tok_counts_all, int32_t *tok_base)
{
    if (world <= 0 || !tok_counts_all || !tok_base) return ORC_EBADARG;
    for (int o = 0; o < world; ++o) {
        int64_t row = 0;
        for (int r = 0; r < world; ++r) {
            tok_base[r * world + o] = (int32_t)row;
            row += tok_counts_all[r * world + o];
        }
    }
    return ORC_OK;
}
