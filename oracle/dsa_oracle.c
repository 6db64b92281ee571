/*
 * dsa_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of the DeepSeek Sparse Attention (DSA)
 * forward pass.  It exists to check the CUDA library against; nothing in the
 * product links, loads or calls it.  Only the tests, the package's smoke check
 * and the benchmark's CPU-baseline leg use it.  It shares no code with the CUDA
 * path.
 *
 * Source: "Техотчёт DeepSeek-V3.2 (2025): разреженное внимание DSA и
 * масштабирование RL" (ai.flicky.cc), section "DSA: внимание только к важному":
 *   - subsection "Молниеносный индексатор", equation for I_{t,s}:
 *       I[t,s] = sum_{j<H_I} w[t,j] * ReLU(q_I[t,j] . k_I[s]),
 *     computed in FP8 (third bullet under that equation);
 *   - subsection "Отбор и основное внимание", equation for u_t:
 *       u_t = Attn(h_t, { c_s : I[t,s] in Top-k(I[t,:]) }),  k = 2048,
 *     with MLA in MQA mode: one latent KV row c_s serves every query head;
 *   - section "Как учили индексатор" (the indexer's training loss): the target
 *     p[t,:] is the main attention's probabilities summed over all heads and
 *     L1-normalised along the keys; the loss is the KL divergence between p[t,:]
 *     and the softmax of the indexer's scores, over the selected positions only
 *     in the sparse stage (item 2 of that section).
 *
 * Readings where the page is silent (each one is listed with its reason in the
 * repository's design notes):
 *   - the query at position t sees keys s <= t (itself included);
 *   - FP8 values are dequantised with one positive fp32 scale per token;
 *   - top-k ties go to the smaller position; -0.0 equals +0.0;
 *   - a row with t+1 <= k selects every position 0..t;
 *   - V is the leading Dv columns of the latent KV row; K is the whole row;
 *   - the loss is D_KL(p || softmax(I)) (target first), both distributions over
 *     the row's valid selected positions; 0 log 0 = 0; a row with no valid
 *     selected position has loss 0 and target 0.
 *
 * Every sum is a plain loop in fp64, in index order.  OpenMP only splits the
 * independent query rows across host threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- number formats -------------------------------------------------------- */

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is
 * no infinity.  Written from the format definition. */
double oracle_e4m3_value(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- step 1: lightning indexer ---------------------------------------------- */

/*
 * Query rows are given one by one: row r belongs to batch row_b[r] and sits at
 * sequence position row_t[r]; its indexer inputs are q_I[r][H_I][d_I],
 * q_scale[r] and w[r][H_I].  Keys are the whole key side of every batch:
 * k_I[b][Lk][d_I] and k_scale[b][Lk].  For s in [0, Lk):
 *   scores[r][s] = sum_j w[r,j] * max(0, sum_d qd[r,j,d] * kd[b,s,d])  if s <= t,
 *   scores[r][s] = -inf                                               if s >  t,
 * with qd = e4m3(q_I) * q_scale[r] and kd = e4m3(k_I) * k_scale[b,s]
 * (a NULL scale array means 1.0).
 */
int oracle_indexer_scores(int64_t n_rows, const int64_t *row_b, const int64_t *row_t,
                          int H_I, int d_I,
                          const uint8_t *q_I, const float *q_scale, const uint16_t *w,
                          int Lk, const uint8_t *k_I, const float *k_scale,
                          double *scores)
{
    if (n_rows < 0 || H_I <= 0 || d_I <= 0 || Lk <= 0)
        return 1;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < n_rows; ++r) {
        int64_t b = row_b[r], t = row_t[r];
        double sq = q_scale ? (double)q_scale[r] : 1.0;
        double *qd = (double *)malloc(sizeof(double) * (size_t)H_I * d_I);
        double *wt = (double *)malloc(sizeof(double) * (size_t)H_I);
        double *kd = (double *)malloc(sizeof(double) * (size_t)d_I);
        for (int j = 0; j < H_I; ++j) {
            wt[j] = oracle_bf16_value(w[r * H_I + j]);
            for (int d = 0; d < d_I; ++d)
                qd[j * d_I + d] = oracle_e4m3_value(q_I[(r * H_I + j) * d_I + d]) * sq;
        }
        double *row = scores + r * (int64_t)Lk;
        for (int64_t s = 0; s < Lk; ++s) {
            if (s > t) {
                row[s] = -INFINITY;
                continue;
            }
            double sk = k_scale ? (double)k_scale[b * Lk + s] : 1.0;
            for (int d = 0; d < d_I; ++d)
                kd[d] = oracle_e4m3_value(k_I[(b * Lk + s) * d_I + d]) * sk;
            double acc = 0.0;
            for (int j = 0; j < H_I; ++j) {
                double dot = 0.0;
                for (int d = 0; d < d_I; ++d)
                    dot += qd[j * d_I + d] * kd[d];
                acc += wt[j] * (dot > 0.0 ? dot : 0.0);
            }
            row[s] = acc;
        }
        free(qd);
        free(wt);
        free(kd);
    }
    return 0;
}

/* ---- step 2: top-k selection ------------------------------------------------ */

typedef struct {
    double v;
    int64_t s;
} cand_t;

/* larger score first; equal scores: smaller position first */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    if (a->s < b->s) return -1;
    if (a->s > b->s) return 1;
    return 0;
}

static int idx_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * For each row r with query position t = row_t[r]: the m = min(k, t+1, Lk)
 * positions s in [0, min(t, Lk-1)] with the largest scores[r][s], ties to the
 * smaller s.  out[r][0..m) holds them in ascending position order and
 * out[r][m..k) = -1.
 */
int oracle_topk(const double *scores, int64_t n_rows, int Lk, const int64_t *row_t, int k,
                int32_t *out)
{
    if (n_rows < 0 || Lk <= 0 || k <= 0)
        return 1;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 4)
    for (r = 0; r < n_rows; ++r) {
        int64_t t = row_t[r];
        int64_t n = (t + 1 < Lk) ? t + 1 : Lk;
        if (n < 0) n = 0;
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
        for (int64_t s = 0; s < n; ++s) {
            c[s].v = scores[r * (int64_t)Lk + s];
            c[s].s = s;
        }
        qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
        int64_t m = n < k ? n : k;
        int32_t *o = out + r * (int64_t)k;
        for (int64_t x = 0; x < m; ++x)
            o[x] = (int32_t)c[x].s;
        qsort(o, (size_t)m, sizeof(int32_t), idx_cmp);
        for (int64_t x = m; x < k; ++x)
            o[x] = -1;
        free(c);
    }
    return 0;
}

/* ---- step 3: sparse MQA / MLA-absorbed attention ---------------------------- */

/*
 * Row r belongs to batch row_b[r]; its queries are q[r][H][D].  Over the valid
 * entries s of indices[r][0..k) (negative entries are padding), for head h:
 *   z_s = scale * sum_d q[r,h,d] * kv[b,s,d]              (d < D)
 *   p_s = exp(z_s - max z) / sum exp(z - max z)
 *   out[r][h][v] = sum_s p_s * kv[b,s,v]                   (v < Dv)
 *   lse[r][h]    = max z + log(sum exp(z - max z))
 * A row with no valid entry gets out = 0 and lse = -inf.  Returns 2 if an index
 * is >= Lk.
 */
int oracle_sparse_attn(int64_t n_rows, const int64_t *row_b, int H, int D, int Dv, double scale,
                       const uint16_t *q, int Lk, const uint16_t *kv,
                       const int32_t *indices, int k, double *out, double *lse)
{
    if (n_rows < 0 || H <= 0 || D <= 0 || Dv <= 0 || Dv > D || k <= 0 || Lk <= 0)
        return 1;
    int bad = 0;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (r = 0; r < n_rows; ++r) {
        int64_t b = row_b[r];
        const int32_t *idx = indices + r * (int64_t)k;
        double *z = (double *)malloc(sizeof(double) * (size_t)k);
        for (int h = 0; h < H; ++h) {
            const uint16_t *qh = q + (r * H + h) * (int64_t)D;
            double zmax = -INFINITY;
            int nvalid = 0;
            for (int x = 0; x < k; ++x) {
                int32_t s = idx[x];
                if (s < 0) { z[x] = -INFINITY; continue; }
                if (s >= Lk) { bad = 1; z[x] = -INFINITY; continue; }
                const uint16_t *kr = kv + (b * Lk + s) * (int64_t)D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += oracle_bf16_value(qh[d]) * oracle_bf16_value(kr[d]);
                z[x] = scale * dot;
                if (z[x] > zmax) zmax = z[x];
                ++nvalid;
            }
            double *o = out + (r * H + h) * (int64_t)Dv;
            for (int v = 0; v < Dv; ++v)
                o[v] = 0.0;
            if (nvalid == 0) {
                if (lse) lse[r * H + h] = -INFINITY;
                continue;
            }
            double l = 0.0;
            for (int x = 0; x < k; ++x) {
                int32_t s = idx[x];
                if (s < 0 || s >= Lk) continue;
                double p = exp(z[x] - zmax);
                l += p;
                const uint16_t *kr = kv + (b * Lk + s) * (int64_t)D;
                for (int v = 0; v < Dv; ++v)
                    o[v] += p * oracle_bf16_value(kr[v]);
            }
            for (int v = 0; v < Dv; ++v)
                o[v] /= l;
            if (lse) lse[r * H + h] = zmax + log(l);
        }
        free(z);
    }
    return bad ? 2 : 0;
}

/* ---- the indexer's training loss (forward) ---------------------------------- */

/*
 * For each of n_rows query rows (row r of batch row_b[r], query q[r], selection
 * indices[r], the row's indexer scores scores[r][0..Lk)):
 *   per head h, the attention probabilities a_h[x] over the valid selected
 *   positions (the same softmax as oracle_sparse_attn);
 *   P[x] = sum_h a_h[x];  target[r][x] = P[x] / sum_x P[x]    (0 on invalid slots);
 *   lq[x] = log softmax over the valid selected x of scores[r][indices[r][x]];
 *   kl[r] = sum over valid x with target > 0 of target[x] * (log target[x] - lq[x]).
 * Slot x of target corresponds to slot x of indices.  Negative indices are
 * padding; an index >= Lk is an error (returns 2).
 */
int oracle_indexer_kl(int64_t n_rows, const int64_t *row_b, int H, int D, double scale,
                      const uint16_t *q, int Lk, const uint16_t *kv,
                      const int32_t *indices, int k, const double *scores,
                      double *target, double *kl)
{
    if (n_rows < 0 || H <= 0 || D <= 0 || k <= 0 || Lk <= 0)
        return 1;
    int bad = 0;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (r = 0; r < n_rows; ++r) {
        int64_t b = row_b[r];
        const int32_t *idx = indices + r * (int64_t)k;
        const double *I = scores + r * (int64_t)Lk;
        double *tg = target + r * (int64_t)k;
        double *z = (double *)malloc(sizeof(double) * (size_t)k);
        int nvalid = 0;
        for (int x = 0; x < k; ++x) {
            tg[x] = 0.0;
            if (idx[x] >= Lk) bad = 1;
            else if (idx[x] >= 0) ++nvalid;
        }
        kl[r] = 0.0;
        if (nvalid == 0) {
            free(z);
            continue;
        }
        /* Main attention, head by head, accumulated into tg[] (= P before normalising). */
        for (int h = 0; h < H; ++h) {
            const uint16_t *qh = q + (r * H + h) * (int64_t)D;
            double zmax = -INFINITY;
            for (int x = 0; x < k; ++x) {
                int32_t s = idx[x];
                if (s < 0 || s >= Lk) continue;
                const uint16_t *kr = kv + (b * Lk + s) * (int64_t)D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += oracle_bf16_value(qh[d]) * oracle_bf16_value(kr[d]);
                z[x] = scale * dot;
                if (z[x] > zmax) zmax = z[x];
            }
            double l = 0.0;
            for (int x = 0; x < k; ++x) {
                int32_t s = idx[x];
                if (s < 0 || s >= Lk) continue;
                l += exp(z[x] - zmax);
            }
            for (int x = 0; x < k; ++x) {
                int32_t s = idx[x];
                if (s < 0 || s >= Lk) continue;
                tg[x] += exp(z[x] - zmax) / l;
            }
        }
        /* L1 normalisation of the head sum. */
        double total = 0.0;
        for (int x = 0; x < k; ++x)
            total += tg[x];
        for (int x = 0; x < k; ++x)
            tg[x] /= total;
        /* log softmax of the indexer scores over the same positions. */
        double imax = -INFINITY;
        for (int x = 0; x < k; ++x) {
            int32_t s = idx[x];
            if (s < 0 || s >= Lk) continue;
            if (I[s] > imax) imax = I[s];
        }
        double li = 0.0;
        for (int x = 0; x < k; ++x) {
            int32_t s = idx[x];
            if (s < 0 || s >= Lk) continue;
            li += exp(I[s] - imax);
        }
        double log_norm = imax + log(li);
        double acc = 0.0;
        for (int x = 0; x < k; ++x) {
            int32_t s = idx[x];
            if (s < 0 || s >= Lk || tg[x] <= 0.0) continue;
            acc += tg[x] * (log(tg[x]) - (I[s] - log_norm));
        }
        kl[r] = acc;
        free(z);
    }
    return bad ? 2 : 0;
}

/* ---- the whole forward pass -------------------------------------------------- */

/*
 * Indexer -> top-k -> sparse attention for n_rows query rows (same row
 * convention as above).  indices: [n_rows][k]; out: [n_rows][H][Dv];
 * lse: [n_rows][H] (nullable); scores (nullable): [n_rows][Lk] receives the
 * indexer scores.
 */
int oracle_dsa_forward(int64_t n_rows, const int64_t *row_b, const int64_t *row_t,
                       int H_I, int d_I,
                       const uint8_t *q_I, const float *q_scale, const uint16_t *w,
                       int Lk, const uint8_t *k_I, const float *k_scale,
                       int H, int D, int Dv, double scale,
                       const uint16_t *q, const uint16_t *kv, int k,
                       int32_t *indices, double *out, double *lse, double *scores)
{
    double *sc = scores;
    if (sc == NULL) {
        sc = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1) * (size_t)Lk);
        if (!sc) return 3;
    }
    int rc = oracle_indexer_scores(n_rows, row_b, row_t, H_I, d_I, q_I, q_scale, w,
                                   Lk, k_I, k_scale, sc);
    if (rc == 0)
        rc = oracle_topk(sc, n_rows, Lk, row_t, k, indices);
    if (rc == 0)
        rc = oracle_sparse_attn(n_rows, row_b, H, D, Dv, scale, q, Lk, kv, indices, k, out, lse);
    if (sc != scores)
        free(sc);
    return rc;
}
