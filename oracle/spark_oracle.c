/*
 * spark_oracle.c -- plain, slow, obviously-correct CPU oracle for SparK
 * channel pruning and recover-then-attend decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, shares no code,
 * header, table or helper with it, and fails loudly when its own CUDA
 * library is missing.
 *
 * Sources (web pages on SparK, arXiv 2508.15212):
 *   [W]  "KV Cache 还能再砍一刀：SparK 在通道维度上做了一件被忽略多年的事"
 *        (paper walkthrough, ai-paper-analysis.pages.dev), sections 1, 3.1,
 *        3.2, 3.3 (recovery steps 1-4 and the F table) and Fig. 3.
 *   [A]  "AAAI 2026 AMD论文Spark方法揭秘" (AMD blog): decode runs standard
 *        full attention after the pruned channels are rebuilt.
 *
 * Arithmetic: fp64 everywhere except where the reading below fixes fp32
 * (the channel norm is rounded once to fp32, and the saliency is one fp32
 * multiply, so that the integer outcome -- the mask -- is decided in the
 * same precision on both sides).  Build with -ffp-contract=off and without
 * fast-math.
 *
 * Readings where the pages are silent or disagree (each used everywhere):
 *   R1  window-query channel norm: qn_j = sqrt(sum over the G query heads of
 *       the group and the W window rows of q^2); [W] 3.1 writes ||q^j||_2 for
 *       a channel of the query block, 3.2 replaces the query by the window.
 *   R2  ||k^j_{i,t}||_2 for one key token is |k_t^j|.
 *   R3  top-T ties go to the lower channel index.
 *   R4  the statistic sampled by F is pooled per (batch, kv head) over the
 *       pruned entries only (mu_pruned of [W] 3.3 step 1).
 *   R5  recovered key k~ = w~ / qn_j with no sign ([W] 3.3 step 3); 0 when
 *       qn_j == 0.
 *   R6  softmax scale 1/sqrt(D); decode-time tail tokens are never pruned.
 *   R7  T = round((1 - lambda) * D), half away from zero, in fp64.
 *   R8  an empty context (no prefix, no tail) gives a zero output row.
 *
 * Layouts (row-major, all plain, none shared with the GPU path):
 *   q_obs [BH*G][W][D]     k, v [BH][S][D]      qn [BH][D]  (fp32)
 *   mask  [BH][S][ceil(D/32)] uint32, bit j%32 of word j/32 = channel kept
 *   vals  [BH][S][T] fp32 (kept key values, ascending channel)
 *   stats [BH][4] fp64 = {N_pruned, sum w, sum w^2, mu_pruned}
 *   q, out [BH*G][D]; k_tail, v_tail [BH][tail_cap][D]
 * Query head g of kv head h is row h*G + g (consecutive GQA grouping).
 */
#define _USE_MATH_DEFINES
#include <math.h>
#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* R7: pruning ratio lambda -> number of kept channels T ([W] 4.1, Table 1
 * caption of [A]: lambda is the fraction of key channels pruned). */
int oracle_lambda_to_T(float lambda, int D)
{
    if (!(lambda >= 0.0f && lambda <= 1.0f) || D <= 0)
        return -1;
    return (int)llround((1.0 - (double)lambda) * (double)D);
}

/* R1: observation-window channel norm ([W] 3.1 saliency, 3.2 window). */
void oracle_qnorm(const float *q_obs, long BH, int G, int W, int D, float *qn)
{
    for (long bh = 0; bh < BH; ++bh)
        for (int j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int g = 0; g < G; ++g)
                for (int t = 0; t < W; ++t) {
                    double x = q_obs[((bh * G + g) * (long)W + t) * D + j];
                    acc += x * x;
                }
            qn[bh * D + j] = (float)sqrt(acc);
        }
}

/* Proxy saliency of one entry, [W] 3.1: w = ||q^j||_2 * |k^j| as one fp32
 * multiply (R2). */
static float saliency(float qn_j, float k_tj)
{
    float a = fabsf(k_tj);
    return qn_j * a;
}

typedef struct {
    float w;
    int j;
} chan_score;

/* Greedy order of the relaxed objective ([W] 3.1): larger saliency first,
 * then lower channel index (R3). */
static int by_saliency_desc(const void *pa, const void *pb)
{
    const chan_score *a = (const chan_score *)pa, *b = (const chan_score *)pb;
    if (a->w > b->w) return -1;
    if (a->w < b->w) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

/* Per-token top-T channel selection + packing + pruned-score statistics.
 * [W] 3.1 (relaxed objective max sum w z, sum z = T, solved greedily by
 * sorting), 3.2 (per-token unstructured mask), 3.3 step 1 (cache keeps the
 * pruned key, the mask and the score statistics). */
void oracle_prune(const float *k, const float *qn, long BH, long S, int D,
                  int T, uint32_t *mask, float *vals, double *stats)
{
    const int nw = (D + 31) / 32;
    chan_score *order = (chan_score *)malloc(sizeof(chan_score) * (size_t)D);
    unsigned char *keep = (unsigned char *)malloc((size_t)D);
    float *w = (float *)malloc(sizeof(float) * (size_t)D);
    for (long bh = 0; bh < BH; ++bh) {
        double n = 0.0, sw = 0.0, sw2 = 0.0;
        for (long t = 0; t < S; ++t) {
            const float *krow = k + (bh * S + t) * D;
            for (int j = 0; j < D; ++j) {
                w[j] = saliency(qn[bh * D + j], krow[j]);
                order[j].w = w[j];
                order[j].j = j;
            }
            qsort(order, (size_t)D, sizeof(chan_score), by_saliency_desc);
            memset(keep, 0, (size_t)D);
            for (int r = 0; r < T; ++r)
                keep[order[r].j] = 1;

            uint32_t *mrow = mask + (bh * S + t) * nw;
            for (int q = 0; q < nw; ++q)
                mrow[q] = 0u;
            float *vrow = vals + (bh * S + t) * (long)T;
            int pos = 0;
            for (int j = 0; j < D; ++j) {
                if (keep[j]) {
                    mrow[j / 32] |= 1u << (j % 32);
                    vrow[pos++] = krow[j];
                } else {
                    double x = (double)w[j];
                    n += 1.0;
                    sw += x;
                    sw2 += x * x;
                }
            }
        }
        stats[bh * 4 + 0] = n;
        stats[bh * 4 + 1] = sw;
        stats[bh * 4 + 2] = sw2;
        stats[bh * 4 + 3] = (n > 0.0) ? sw / n : 0.0;
    }
    free(order);
    free(keep);
    free(w);
}

/*
 * SparK-p ([W] 5.2): instead of a fixed ratio, every token keeps the fewest
 * channels whose cumulative saliency reaches a fraction p (0.99 in [W]) of
 * the token's total.  Reading R19 (the pages fix neither the arithmetic of
 * the cumulative sum nor the storage):
 *   - channels are taken in the greedy order of [W] 3.1 (saliency desc,
 *     lower channel first on ties, R3); the cumulative saliency of the first
 *     n channels of that order is P(n), accumulated in fp64 in that order
 *     (fp32 saliencies, so P(n) is the exact sum up to fp64 rounding: a
 *     relative error below 2^-46 for D = 128);
 *   - total = P(D); target = p * total in fp64; the kept set is the shortest
 *     prefix with P(n) >= target ("reaches" is >=, so a token whose
 *     saliencies are all 0, or p = 0, keeps nothing);
 *   - the cache has a capacity of Tcap values per token: a longer prefix is
 *     cut to its first Tcap channels.  vals keeps the kept values in
 *     ascending channel order in the first slots of the token's Tcap slots,
 *     zeros after;
 *   - statistics over the pruned entries as in oracle_prune.
 */
void oracle_prune_topp(const float *k, const float *qn, long BH, long S, int D, float p, int Tcap,
                       uint32_t *mask, float *vals, double *stats)
{
    const int nw = (D + 31) / 32;
    chan_score *order = (chan_score *)malloc(sizeof(chan_score) * (size_t)D);
    unsigned char *in = (unsigned char *)malloc((size_t)D);
    float *w = (float *)malloc(sizeof(float) * (size_t)D);
    for (long bh = 0; bh < BH; ++bh) {
        double n_pruned = 0.0, sw = 0.0, sw2 = 0.0;
        for (long t = 0; t < S; ++t) {
            const float *krow = k + (bh * S + t) * D;
            for (int j = 0; j < D; ++j) {
                w[j] = saliency(qn[bh * D + j], krow[j]);
                order[j].w = w[j];
                order[j].j = j;
            }
            qsort(order, (size_t)D, sizeof(chan_score), by_saliency_desc);
            double total = 0.0;
            for (int r = 0; r < D; ++r)
                total += (double)order[r].w;
            const double target = (double)p * total;
            /* the shortest greedy prefix whose cumulative saliency reaches
             * the target (P(0) = 0) */
            int n = 0;
            double cum = 0.0;
            while (n < D && cum < target) {
                cum += (double)order[n].w;
                n += 1;
            }
            const int n_keep = n < Tcap ? n : Tcap;
            memset(in, 0, (size_t)D);
            for (int r = 0; r < n_keep; ++r)
                in[order[r].j] = 1;

            uint32_t *mrow = mask + (bh * S + t) * nw;
            for (int q = 0; q < nw; ++q)
                mrow[q] = 0u;
            float *vrow = vals + (bh * S + t) * (long)Tcap;
            for (int r = 0; r < Tcap; ++r)
                vrow[r] = 0.0f;
            int slot = 0;
            for (int j = 0; j < D; ++j) {
                if (in[j]) {
                    mrow[j / 32] |= 1u << (j % 32);
                    vrow[slot] = krow[j];
                    slot += 1;
                } else {
                    const double x = (double)w[j];
                    n_pruned += 1.0;
                    sw += x;
                    sw2 += x * x;
                }
            }
        }
        stats[bh * 4 + 0] = n_pruned;
        stats[bh * 4 + 1] = sw;
        stats[bh * 4 + 2] = sw2;
        stats[bh * 4 + 3] = (n_pruned > 0.0) ? sw / n_pruned : 0.0;
    }
    free(order);
    free(in);
    free(w);
}

/*
 * SparK-g ([W] 5.2): channels are split into g groups by importance and each
 * group has its own pruning rate, low-importance groups pruned harder
 * (g = 4 with rates (0.25, 0.5, 0.75, 1.0) in [W]).  Reading R15 (the pages
 * do not say what "importance" is or how large the groups are):
 *   - the importance of channel j of a head is its window-query norm qn_j,
 *     the query factor of the saliency, fixed for the head; channels ordered
 *     by (qn desc, j asc) are cut into g consecutive groups, group k holding
 *     the ranks [k*D/g, (k+1)*D/g) (integer division);
 *   - group k keeps Tg[k] = round((1 - rate_k) * |group k|) channels per
 *     token (half away from zero, as R7): its Tg[k] channels of largest
 *     saliency, ties to the lower channel, i.e. the greedy solution of the
 *     relaxed objective of [W] 3.1 with one budget per group;
 *   - the cache is the plain one with T = sum_k Tg[k] (mask, kept values in
 *     ascending channel order, statistics over the pruned entries).
 * With equal-size groups the mean pruning rate is the mean of the rates
 * (0.625 for [W]'s g = 4 rates); [W] reports 0.44, which equal groups cannot
 * give, so the group sizes of the original are not those of this reading.
 */
typedef struct {
    float q;
    int j;
} chan_norm;

static int by_norm_desc(const void *pa, const void *pb)
{
    const chan_norm *a = (const chan_norm *)pa, *b = (const chan_norm *)pb;
    if (a->q > b->q) return -1;
    if (a->q < b->q) return 1;
    return a->j < b->j ? -1 : (a->j > b->j);  /* equal norms: lower channel first */
}

/* gid [BH][D]: group of every channel (R15). */
void oracle_group_of_channel(const float *qn, long BH, int D, int g, int *gid)
{
    chan_norm *ord = (chan_norm *)malloc(sizeof(chan_norm) * (size_t)D);
    for (long bh = 0; bh < BH; ++bh) {
        for (int j = 0; j < D; ++j) {
            ord[j].q = qn[bh * D + j];
            ord[j].j = j;
        }
        qsort(ord, (size_t)D, sizeof(chan_norm), by_norm_desc);
        for (int k = 0; k < g; ++k)
            for (int r = k * D / g; r < (k + 1) * D / g; ++r)
                gid[bh * D + ord[r].j] = k;
    }
    free(ord);
}

/* Per-group budgets Tg[k] from pruning rates (R15). */
void oracle_group_budget(int D, int g, const float *rates, int *Tg)
{
    for (int k = 0; k < g; ++k) {
        const int size = (k + 1) * D / g - k * D / g;
        Tg[k] = (int)llround((1.0 - (double)rates[k]) * (double)size);
    }
}

/* SparK-g pruning (R15): per token and group, the group's Tg[k] largest
 * saliencies; packing and statistics as in oracle_prune with T = sum Tg. */
void oracle_prune_grouped(const float *k, const float *qn, long BH, long S, int D, int g, const int *Tg,
                          uint32_t *mask, float *vals, double *stats)
{
    const int nw = (D + 31) / 32;
    int T = 0;
    for (int q = 0; q < g; ++q)
        T += Tg[q];
    int *gid = (int *)malloc(sizeof(int) * (size_t)(BH > 0 ? BH : 1) * (size_t)D);
    oracle_group_of_channel(qn, BH, D, g, gid);
    chan_score *order = (chan_score *)malloc(sizeof(chan_score) * (size_t)D);
    unsigned char *keep = (unsigned char *)malloc((size_t)D);
    float *w = (float *)malloc(sizeof(float) * (size_t)D);
    for (long bh = 0; bh < BH; ++bh) {
        double n = 0.0, sw = 0.0, sw2 = 0.0;
        for (long t = 0; t < S; ++t) {
            const float *krow = k + (bh * S + t) * D;
            for (int j = 0; j < D; ++j)
                w[j] = saliency(qn[bh * D + j], krow[j]);
            memset(keep, 0, (size_t)D);
            for (int grp = 0; grp < g; ++grp) {
                int m = 0;
                for (int j = 0; j < D; ++j)
                    if (gid[bh * D + j] == grp) {
                        order[m].w = w[j];
                        order[m].j = j;
                        ++m;
                    }
                qsort(order, (size_t)m, sizeof(chan_score), by_saliency_desc);
                for (int r = 0; r < Tg[grp] && r < m; ++r)
                    keep[order[r].j] = 1;
            }
            uint32_t *mrow = mask + (bh * S + t) * nw;
            for (int q = 0; q < nw; ++q)
                mrow[q] = 0u;
            float *vrow = vals + (bh * S + t) * (long)T;
            int pos = 0;
            for (int j = 0; j < D; ++j) {
                if (keep[j]) {
                    mrow[j / 32] |= 1u << (j % 32);
                    vrow[pos] = krow[j];
                    ++pos;
                } else {
                    const double x = (double)w[j];
                    n += 1.0;
                    sw += x;
                    sw2 += x * x;
                }
            }
        }
        stats[bh * 4 + 0] = n;
        stats[bh * 4 + 1] = sw;
        stats[bh * 4 + 2] = sw2;
        stats[bh * 4 + 3] = n > 0.0 ? (sw / n) : 0.0;
    }
    free(gid);
    free(order);
    free(keep);
    free(w);
}

/*
 * V-channel pruning ([W] 4.4: the value cache is pruned too, with a
 * norm-based heuristic; SparK(0.5+0.5) prunes half of the key and half of
 * the value channels).  Reading R16 (the pages name only "norm-based"): the
 * saliency of value channel j of token t is its magnitude |v_t^j| -- the
 * key rule of [W] 3.1 with the query factor set to 1, since a value channel
 * meets no query -- so pruning is oracle_prune(v, qn = 1, T_v): top-T_v per
 * token, ties to the lower channel, the same mask and packing.  A pruned
 * value entry is recovered as 0 (dropped); the statistics over the pruned
 * entries are computed but unused.  This writes the dense recovered value
 * block Vt [S][D] (fp64) of one (b, h).
 */
void oracle_recover_values(const uint32_t *vmask, const float *vvals, long bh, long S, int D, int Tv, double *Vt)
{
    const int nw = (D + 31) / 32;
    for (long t = 0; t < S; ++t) {
        const uint32_t *mrow = vmask + (bh * S + t) * nw;
        const float *vrow = vvals + (bh * S + t) * (long)Tv;
        int pos = 0;
        for (int j = 0; j < D; ++j)
            Vt[t * D + j] = ((mrow[j / 32] >> (j % 32)) & 1u) ? (double)vrow[pos++] : 0.0;
    }
}

/*
 * ThinK, the structured channel-pruning comparator ([W] 1 and Fig. 2(c): one
 * channel mask shared by all tokens of a head, no recovery; [W] 4.2 compares
 * SparK with it at lambda = 0.5 and 0.8).  Reading R18 (the pages give no
 * ThinK formula): the relaxed objective of [W] 3.1 with one mask for the
 * whole key block of a (b, h) ranks channel j by
 *     score_j = qn_j * ||k^j||_2,   ||k^j||_2 = sqrt(sum_t k_tj^2)  (fp64)
 * over the S prompt tokens; the T channels of largest score (ties -> lower
 * channel) are kept for every token.  The cache is the plain one (every
 * token's mask equal, kept values in ascending channel order); without
 * recovery a pruned entry reads as 0, which the cache states with
 * stats = {N = S*(D-T), 0, 0, mu = 0}.
 */
typedef struct {
    double s;
    int j;
} chan_dscore;

static int by_dscore_desc(const void *pa, const void *pb)
{
    const chan_dscore *a = (const chan_dscore *)pa, *b = (const chan_dscore *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j < b->j) ? -1 : ((a->j > b->j) ? 1 : 0);  /* lower channel first */
}

void oracle_think_prune(const float *k, const float *qn, long BH, long S, int D, int T, uint32_t *mask,
                        float *vals, double *stats)
{
    const int nw = (D + 31) / 32;
    chan_dscore *ord = (chan_dscore *)malloc(sizeof(chan_dscore) * (size_t)D);
    unsigned char *keep = (unsigned char *)malloc((size_t)D);
    for (long bh = 0; bh < BH; ++bh) {
        for (int j = 0; j < D; ++j) {
            double ss = 0.0;
            for (long t = 0; t < S; ++t) {
                const double x = (double)k[(bh * S + t) * D + j];
                ss += x * x;
            }
            ord[j].s = (double)qn[bh * D + j] * sqrt(ss);
            ord[j].j = j;
        }
        qsort(ord, (size_t)D, sizeof(chan_dscore), by_dscore_desc);
        memset(keep, 0, (size_t)D);
        for (int r = 0; r != T; ++r)  /* the T best channels */
            keep[ord[r].j] = 1;
        for (long t = 0; t < S; ++t) {
            uint32_t *mrow = mask + (bh * S + t) * nw;
            float *vrow = vals + (bh * S + t) * (long)T;
            for (int q = 0; q < nw; ++q)
                mrow[q] = 0u;
            int pos = 0;
            for (int j = 0; j < D; ++j)
                if (keep[j]) {
                    mrow[j / 32] |= 1u << (j % 32);
                    vrow[pos] = k[(bh * S + t) * D + j];
                    ++pos;
                }
        }
        stats[bh * 4 + 0] = (double)S * (double)(D - T);
        stats[bh * 4 + 1] = 0.0;
        stats[bh * 4 + 2] = 0.0;
        stats[bh * 4 + 3] = 0.0;
    }
    free(ord);
    free(keep);
}

/* Recovery F = Degenerate, [W] 3.3 steps 2-4 and the F table: the sampled
 * score is mu_pruned, and the key is back-solved from it as
 * k~ = w~ / ||q^j||_2 (R5).  Kept channels are the stored key values.
 * Writes the dense recovered key block Kt [S][D] (fp64) of one (b, h). */
void oracle_recover_keys(const uint32_t *mask, const float *vals,
                         const float *qn, const double *stats, long bh,
                         long S, int D, int T, double *Kt)
{
    const int nw = (D + 31) / 32;
    const double mu = stats[bh * 4 + 3];
    for (long t = 0; t < S; ++t) {
        const uint32_t *mrow = mask + (bh * S + t) * nw;
        const float *vrow = vals + (bh * S + t) * (long)T;
        int pos = 0;
        for (int j = 0; j < D; ++j) {
            int kept = (mrow[j / 32] >> (j % 32)) & 1u;
            if (kept) {
                Kt[t * D + j] = (double)vrow[pos++];
            } else {
                double qj = (double)qn[bh * D + j];
                Kt[t * D + j] = (qj > 0.0) ? mu / qj : 0.0;
            }
        }
    }
}

/* Decode: standard full attention over the recovered keys ([W] Fig. 3,
 * [A]): for each query head, s_t = q . k~_t / sqrt(D) over the pruned
 * prefix then the dense tail, softmax (max-subtracted, two passes), and
 * out = sum_t p_t v_t.  Output rounded once to fp32. */
void oracle_decode(const float *q, const uint32_t *mask, const float *vals,
                   const float *qn, const double *stats, const float *v,
                   const float *k_tail, const float *v_tail, long tail_cap,
                   long n_tail, long BH, int G, long S, int D, int T,
                   float *out)
{
    const long L = S + n_tail;
    double *Kt = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * (size_t)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)D);
    const double scale = 1.0 / sqrt((double)D);
    for (long bh = 0; bh < BH; ++bh) {
        oracle_recover_keys(mask, vals, qn, stats, bh, S, D, T, Kt);
        for (long t = 0; t < n_tail; ++t)
            for (int j = 0; j < D; ++j)
                Kt[(S + t) * D + j] = (double)k_tail[(bh * tail_cap + t) * D + j];
        for (int g = 0; g < G; ++g) {
            const float *qrow = q + (bh * G + g) * (long)D;
            float *orow = out + (bh * G + g) * (long)D;
            if (L == 0) {
                for (int d = 0; d < D; ++d)
                    orow[d] = 0.0f;
                continue;
            }
            double m = -INFINITY;
            for (long t = 0; t < L; ++t) {
                double dot = 0.0;
                for (int j = 0; j < D; ++j)
                    dot += (double)qrow[j] * Kt[t * D + j];
                s[t] = dot * scale;
                if (s[t] > m)
                    m = s[t];
            }
            double l = 0.0;
            for (int d = 0; d < D; ++d)
                acc[d] = 0.0;
            for (long t = 0; t < L; ++t) {
                double p = exp(s[t] - m);
                const float *vrow = (t < S) ? v + (bh * S + t) * D
                                            : v_tail + (bh * tail_cap + (t - S)) * D;
                l += p;
                for (int d = 0; d < D; ++d)
                    acc[d] += p * (double)vrow[d];
            }
            for (int d = 0; d < D; ++d)
                orow[d] = (float)(acc[d] / l);
        }
    }
    free(Kt);
    free(s);
    free(acc);
}

/*
 * SnapKV-style token eviction pre-pass, which [W] stacks SparK on (sections 2
 * and 4.1: SnapKV / PyramidKV bases; 3.2: SparK reuses SnapKV's observation
 * window).  The pages give no detail of SnapKV itself; the reading used here:
 *   R11 the W window queries are the last W prompt positions p = S-W+w; each
 *       of the G*W (query head, window row) pairs attends causally over keys
 *       0..p with scale 1/sqrt(D); the score of a prefix token t < P = S-W is
 *       the sum of its probabilities over the G*W rows;
 *   R12 scores are max-pooled along t with kernel `pool` (odd), stride 1 and
 *       half-width padding that never wins (max over the in-range window);
 *   R13 keep-W prefix tokens with the largest pooled score (ties -> lower t)
 *       plus all W window tokens are kept, in original order.
 */
void oracle_snapkv_scores(const float *q_obs, const float *k, long BH, int G, int W,
                          long S, int D, double *scores /* [BH][S-W] */)
{
    const long P = S - W;
    const double scale = 1.0 / sqrt((double)D);
    double *logit = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
    for (long bh = 0; bh < BH; ++bh) {
        double *sc = scores + bh * (P > 0 ? P : 0);
        for (long t = 0; t < P; ++t)
            sc[t] = 0.0;
        for (int g = 0; g < G; ++g)
            for (int w = 0; w < W; ++w) {
                const float *q = q_obs + ((bh * G + g) * (long)W + w) * D;
                const long p = P + w; /* this query's position */
                double m = -INFINITY;
                for (long t = 0; t <= p; ++t) {
                    const float *kr = k + (bh * S + t) * D;
                    double dot = 0.0;
                    for (int j = 0; j < D; ++j)
                        dot += (double)q[j] * (double)kr[j];
                    logit[t] = dot * scale;
                    if (logit[t] > m)
                        m = logit[t];
                }
                double l = 0.0;
                for (long t = 0; t <= p; ++t)
                    l += exp(logit[t] - m);
                for (long t = 0; t < P; ++t)
                    sc[t] += exp(logit[t] - m) / l;
            }
    }
    free(logit);
}

void oracle_snapkv_pool(const double *scores, long BH, long P, int pool, double *pooled)
{
    const int h = pool / 2;
    for (long bh = 0; bh < BH; ++bh)
        for (long t = 0; t < P; ++t) {
            double m = -INFINITY;
            for (long u = t - h; u <= t + h; ++u)
                if (u >= 0 && u < P && scores[bh * P + u] > m)
                    m = scores[bh * P + u];
            pooled[bh * P + t] = m;
        }
}

typedef struct {
    double s;
    long t;
} tok_score;

static int by_score_desc(const void *pa, const void *pb)
{
    const tok_score *a = (const tok_score *)pa, *b = (const tok_score *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->t > b->t) - (a->t < b->t);
}

static int by_index_asc(const void *pa, const void *pb)
{
    long a = *(const long *)pa, b = *(const long *)pb;
    return (a > b) - (a < b);
}

/* Kept token indices [BH][keep] in original order (R13). */
void oracle_snapkv_select(const double *pooled, long BH, long S, int W, int keep, long *idx)
{
    const long P = S - W;
    const long kp = keep - W; /* prefix tokens kept */
    tok_score *ord = (tok_score *)malloc(sizeof(tok_score) * (size_t)(P > 0 ? P : 1));
    for (long bh = 0; bh < BH; ++bh) {
        long *out = idx + bh * keep;
        for (long t = 0; t < P; ++t) {
            ord[t].s = pooled[bh * P + t];
            ord[t].t = t;
        }
        qsort(ord, (size_t)P, sizeof(tok_score), by_score_desc);
        for (long i = 0; i < kp; ++i)
            out[i] = ord[i].t;
        qsort(out, (size_t)kp, sizeof(long), by_index_asc);
        for (int w = 0; w < W; ++w)
            out[kp + w] = P + w;
    }
    free(ord);
}

/*
 * Sampling recoveries of the F table ([W] 3.3): Gaussian w~ ~ N(mu, sigma^2)
 * and Exponential w~ ~ Exp(1/mu) (mean mu).  Reading R14 (the pages do not
 * say when or how the score is drawn): one draw per pruned (token, channel)
 * entry, fixed for a given seed, from the counter-based generator
 * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC'11) with counter (t, j, bh low word, bh high word) and
 * key (seed low word, seed high word).  Uniforms from the top 24 bits:
 * u1 = (x0 >> 8 + 1) / 2^24 in (0, 1], u2 = (x1 >> 8) / 2^24 in [0, 1).
 * Gaussian: mu + sigma * sqrt(-2 ln u1) * cos(2 pi u2) (Box-Muller), with
 * mu, sigma the mean and population standard deviation of the pruned
 * saliencies of the head; Exponential: -mu ln u1.
 */
static void philox_round(uint32_t c[4], const uint32_t k[2])
{
    const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k[0], n2 = hi0 ^ c[3] ^ k[1];
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
}

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k[0] += 0x9E3779B9u;
            k[1] += 0xBB67AE85u;
        }
        philox_round(c, k);
    }
    for (int i = 0; i < 4; ++i)
        out[i] = c[i];
}

/* mode: 0 Degenerate, 1 Gaussian, 2 Exponential.  Returns the sampled score. */
double oracle_sample_score(int mode, const double *st, unsigned long long seed, long bh, long t, int j)
{
    const double mu = st[3];
    if (mode == 0)
        return mu;
    uint32_t ctr[4] = {(uint32_t)t, (uint32_t)j, (uint32_t)((unsigned long long)bh & 0xffffffffu),
                       (uint32_t)((unsigned long long)bh >> 32)};
    uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t x[4];
    oracle_philox4x32_10(ctr, key, x);
    const double u1 = (double)((x[0] >> 8) + 1u) / 16777216.0;
    const double u2 = (double)(x[1] >> 8) / 16777216.0;
    if (mode == 2)
        return -mu * log(u1);
    double var = (st[0] > 0.0) ? st[2] / st[0] - mu * mu : 0.0;
    if (var < 0.0)
        var = 0.0;
    return mu + sqrt(var) * sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);
}

/* Recovered keys with any F ([W] 3.3 steps 2-4): k~_j = w~ / qn_j. */
void oracle_recover_keys_f(const uint32_t *mask, const float *vals, const float *qn, const double *stats,
                           long bh, long S, int D, int T, int mode, unsigned long long seed, double *Kt)
{
    const int nw = (D + 31) / 32;
    for (long t = 0; t < S; ++t) {
        const uint32_t *mrow = mask + (bh * S + t) * nw;
        const float *vrow = vals + (bh * S + t) * (long)T;
        int pos = 0;
        for (int j = 0; j < D; ++j) {
            int kept = (mrow[j / 32] >> (j % 32)) & 1u;
            if (kept) {
                Kt[t * D + j] = (double)vrow[pos++];
            } else {
                double qj = (double)qn[bh * D + j];
                double w = oracle_sample_score(mode, stats + bh * 4, seed, bh, t, j);
                Kt[t * D + j] = (qj > 0.0) ? w / qj : 0.0;
            }
        }
    }
}

/* Decode with any F: as oracle_decode, keys recovered by oracle_recover_keys_f. */
void oracle_decode_f(const float *q, const uint32_t *mask, const float *vals, const float *qn,
                     const double *stats, const float *v, const float *k_tail, const float *v_tail,
                     long tail_cap, long n_tail, long BH, int G, long S, int D, int T, int mode,
                     unsigned long long seed, float *out)
{
    const long L = S + n_tail;
    double *Kt = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1) * (size_t)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)D);
    const double scale = 1.0 / sqrt((double)D);
    for (long bh = 0; bh < BH; ++bh) {
        oracle_recover_keys_f(mask, vals, qn, stats, bh, S, D, T, mode, seed, Kt);
        for (long t = 0; t < n_tail; ++t)
            for (int j = 0; j < D; ++j)
                Kt[(S + t) * D + j] = (double)k_tail[bh * tail_cap * (long)D + t * D + j];
        for (int g = 0; g < G; ++g) {
            const float *qrow = &q[(bh * G + g) * (long)D];  /* query head g of kv head bh */
            float *orow = out + (bh * G + g) * (long)D;
            if (L == 0) {
                for (int d = 0; d < D; ++d)
                    orow[d] = 0.0f;
                continue;
            }
            double m = -INFINITY;
            for (long t = 0; t < L; ++t) {
                double dot = 0.0;
                for (int j = 0; j < D; ++j)
                    dot += (double)qrow[j] * Kt[t * D + j];
                s[t] = dot * scale;
                if (s[t] > m)
                    m = s[t];
            }
            double l = 0.0;
            for (int d = 0; d < D; ++d)
                acc[d] = 0.0;
            for (long t = 0; t < L; ++t) {
                double p = exp(s[t] - m);
                const float *vrow = (t < S) ? v + (bh * S + t) * D : v_tail + (bh * tail_cap + (t - S)) * D;
                l += p;
                for (int d = 0; d < D; ++d)
                    acc[d] += p * (double)vrow[d];
            }
            for (int d = 0; d < D; ++d)
                orow[d] = (float)(acc[d] / l);
        }
    }
    free(Kt);
    free(s);
    free(acc);
}

/*
 * PyramidKV layer budgets (reading R20).  [W] 4.1 and 4.2 stack SparK on
 * PyramidKV, a token eviction whose budget differs per layer, but give no
 * schedule.  The reading: the budget of layer l of L falls linearly with
 * depth around the mean budget M ("KV-size"), from M (1 + beta) at the first
 * layer to M (1 - beta) at the last, rounded half away from zero, then
 * clamped to [W, S]; a single layer keeps M.
 */
void oracle_pyramid_keep(int L, int M, double beta, int W, int S, int *keep)
{
    for (int l = 0; l < L; ++l) {
        double frac = 0.0;  /* +1 at the first layer, -1 at the last */
        if (L > 1)
            frac = 1.0 - 2.0 * (double)l / (double)(L - 1);
        double x = (double)M + (double)M * beta * frac;
        long r = (long)floor(fabs(x) + 0.5);
        if (x < 0.0)
            r = -r;
        if (r < W)
            r = W;
        if (r > S)
            r = S;
        keep[l] = (int)r;
    }
}
