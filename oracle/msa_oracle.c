/*
 * msa_oracle.c -- plain fp64 CPU oracle for MiniMax Sparse Attention (MSA) over GQA.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package smoke check and the benchmark's CPU
 * baseline leg may load this library. It shares no code, header, table or constant with
 * the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (one function per step, slow and direct on purpose):
 *
 *  Sources. "MiniMax M3 sparse attention agents" (youmind article):
 *    - paragraph "The mechanism that changes this" and figure 1's caption: a light Index
 *      Branch scores the key-value context in blocks and keeps the top-k blocks per query
 *      and GQA group; the main branch attends only to those blocks;
 *    - bullet "Predictable cost at every length": Bk = 128, k = 16, so every query and GQA
 *      group reads 16 blocks = 2,048 key-value tokens.
 *  "MiniMax launches MSA sparse attention method and MiniMax-M3 model" (KuCoin flash),
 *    summary paragraph: MSA is built on grouped query attention; the index branch picks 16
 *    blocks of (default) 128 tokens per GQA group, the main branch runs exact softmax
 *    attention over them, and the top-k is exp-free.
 *
 *  The pages do not give the scoring function; this oracle takes the plainest reading that
 *  the rest supports (mean-pooled index keys, dot-product score scaled by 1/sqrt(d_I)):
 *    1. pooled key of full block j of group g:  kbar[j] = (1/Bk) * sum_{t in block j} k_I[t]
 *    2. score of a fully-past block j < c = floor(t/Bk) for the query at position t:
 *         s_j = q_I[t] . kbar[j] / sqrt(d_I)
 *    3. selection: if c + 1 <= k every block 0..c is taken; otherwise the diagonal block c
 *       plus the k-1 best candidates under the total order (s descending, j ascending).
 *       No exponential is evaluated anywhere in steps 1-3.
 *    4. for each query head h of group g: keys U = {u : floor(u/Bk) in S, u <= t},
 *         z_u = q[t,h] . k[u] / sqrt(d),  o = sum_u softmax(z)_u v[u],  lse = log sum exp z.
 *  Decode is step 2-4 at t = L (the new token's position, after it is appended).
 *
 *  All inputs are bf16 bit patterns, widened exactly to double; all arithmetic is fp64.
 *
 * Layouts (row-major): per-group key/value rows K,V [L][d]; query head rows [Hg][d];
 * index rows [dI]; pooled keys [nb][dI] as double.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

double oracle_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------- step 1: pooling */
/* k_idx: [N][G][dI] bf16 of one sequence. pooled: [G][nb_cap][dI]; only full blocks
 * j < N/Bk are written. tail_sum (nullable): [G][dI], the plain sum of the index keys of
 * the trailing partial block (zero when N is a multiple of Bk). */
void oracle_pool(const uint16_t *k_idx, int64_t N, int64_t G, int64_t dI, int64_t Bk,
                 int64_t nb_cap, double *pooled, double *tail_sum)
{
    int64_t nfull = N / Bk;
    for (int64_t g = 0; g < G; ++g) {
        for (int64_t j = 0; j < nfull && j < nb_cap; ++j) {
            for (int64_t i = 0; i < dI; ++i) {
                double sum = 0.0;
                for (int64_t t = j * Bk; t < (j + 1) * Bk; ++t)
                    sum += oracle_bf16_to_f64(k_idx[(t * G + g) * dI + i]);
                pooled[(g * nb_cap + j) * dI + i] = sum / (double)Bk;
            }
        }
        if (tail_sum) {
            for (int64_t i = 0; i < dI; ++i) {
                double sum = 0.0;
                for (int64_t t = nfull * Bk; t < N; ++t)
                    sum += oracle_bf16_to_f64(k_idx[(t * G + g) * dI + i]);
                tail_sum[g * dI + i] = sum;
            }
        }
    }
}

/* ---------------------------------------------------------------- step 2: scores */
void oracle_block_scores(const uint16_t *q_idx_row, const double *pooled_g, int64_t dI,
                         int64_t n_cand, double *s)
{
    double scale = 1.0 / sqrt((double)dI);
    for (int64_t j = 0; j < n_cand; ++j) {
        double dot = 0.0;
        for (int64_t i = 0; i < dI; ++i)
            dot += oracle_bf16_to_f64(q_idx_row[i]) * pooled_g[j * dI + i];
        s[j] = dot * scale;
    }
}

/* ---------------------------------------------------------------- step 3: selection */
/* "a beats b" in the selection order: higher score, then lower block index. */
static int beats(double sa, int64_t ja, double sb, int64_t jb)
{
    return sa > sb || (sa == sb && ja < jb);
}

static void sort_ids_ascending(int32_t *ids, int64_t n)
{
    for (int64_t i = 1; i < n; ++i)
        for (int64_t j = i; j > 0 && ids[j - 1] > ids[j]; --j) {
            int32_t tmp = ids[j]; ids[j] = ids[j - 1]; ids[j - 1] = tmp;
        }
}

/* Selection for a query whose own block is c, from the scores s[0..c-1] of the fully-past
 * blocks. Writes topk ids in ascending order, padded with -1; returns how many are valid.
 * kth (nullable) receives the (topk-1)-th best candidate score, or NaN when every block is
 * taken. Method: topk-1 rounds of "take the best candidate not yet taken". */
int64_t oracle_select_from_scores(const double *s, int64_t c, int64_t topk, int32_t *sel,
                                  double *kth)
{
    int64_t n = 0;
    if (kth) *kth = NAN;
    if (c + 1 <= topk) {
        for (int64_t j = 0; j <= c; ++j) sel[n++] = (int32_t)j;
    } else {
        char *taken = (char *)calloc((size_t)c, 1);
        for (int64_t r = 0; r < topk - 1; ++r) {
            int64_t best = -1;
            for (int64_t j = 0; j < c; ++j)
                if (!taken[j] && (best < 0 || beats(s[j], j, s[best], best))) best = j;
            taken[best] = 1;
            sel[n++] = (int32_t)best;
            if (kth && r == topk - 2) *kth = s[best];
        }
        free(taken);
        sel[n++] = (int32_t)c;
    }
    sort_ids_ascending(sel, n);
    for (int64_t i = n; i < topk; ++i) sel[i] = -1;
    return n;
}

/* The same selection through a full sort of all candidates (the check the selection must
 * pass: the first topk-1 of a full sort plus the diagonal block). */
typedef struct { double s; int64_t j; } cand_t;

static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (beats(x->s, x->j, y->s, y->j)) return -1;
    if (beats(y->s, y->j, x->s, x->j)) return 1;
    return 0;
}

int64_t oracle_select_fullsort(const double *s, int64_t c, int64_t topk, int32_t *sel)
{
    int64_t n = 0;
    if (c + 1 <= topk) {
        for (int64_t j = 0; j <= c; ++j) sel[n++] = (int32_t)j;
    } else {
        cand_t *all = (cand_t *)malloc((size_t)c * sizeof(cand_t));
        for (int64_t j = 0; j < c; ++j) { all[j].s = s[j]; all[j].j = j; }
        qsort(all, (size_t)c, sizeof(cand_t), cand_cmp);
        for (int64_t r = 0; r < topk - 1; ++r) sel[n++] = (int32_t)all[r].j;
        sel[n++] = (int32_t)c;
        free(all);
    }
    sort_ids_ascending(sel, n);
    for (int64_t i = n; i < topk; ++i) sel[i] = -1;
    return n;
}

/* ---------------------------------------------------------------- exp-free top-k of score rows */
/* The selection step on its own, for rows of n given fp32 scores (KuCoin flash "MiniMax
 * launches MSA sparse attention method and MiniMax-M3 model", "ME AI News" paragraph: the
 * index branch's top-k is exp-free). Order: higher score first, then lower column; every NaN
 * ranks above +inf and NaNs tie with each other; -0 and +0 are equal (as C's == has it). */
static int topk_before(float a, int64_t ja, float b, int64_t jb)
{
    const int na = isnan(a) != 0, nb = isnan(b) != 0;
    if (na != nb) return na;
    if (!na && a != b) return a > b;
    return ja < jb;
}

/* idx[row][r] = the r-th best column of the row: k rounds of "take the best column not yet
 * taken". Requires 1 <= k <= n. */
void oracle_topk_rows(const float *scores, int64_t rows, int64_t n, int64_t k, int32_t *idx)
{
    char *taken = (char *)malloc((size_t)n);
    for (int64_t row = 0; row < rows; ++row) {
        const float *s = scores + row * n;
        memset(taken, 0, (size_t)n);
        for (int64_t r = 0; r < k; ++r) {
            int64_t best = -1;
            for (int64_t j = 0; j < n; ++j)
                if (!taken[j] && (best < 0 || topk_before(s[j], j, s[best], best))) best = j;
            taken[best] = 1;
            idx[row * k + r] = (int32_t)best;
        }
    }
    free(taken);
}

/* ---------------------------------------------------------------- step 4: attention */
static int block_selected(int64_t j, const int32_t *sel, int64_t nsel)
{
    for (int64_t i = 0; i < nsel; ++i)
        if (sel[i] == j) return 1;
    return 0;
}

/* One query head at position t over the keys of the selected blocks (u <= t).
 * sel == NULL means every key 0..t (dense causal attention). Returns the key count. */
int64_t oracle_attend_row(const uint16_t *q_row, const uint16_t *K, const uint16_t *V,
                          int64_t d, int64_t t, const int32_t *sel, int64_t nsel, int64_t Bk,
                          double *o, double *lse)
{
    double scale = 1.0 / sqrt((double)d);
    double *qd = (double *)malloc((size_t)d * sizeof(double));
    double *z = (double *)malloc((size_t)(t + 1) * sizeof(double));
    char *use = (char *)malloc((size_t)(t + 1));
    for (int64_t i = 0; i < d; ++i) qd[i] = oracle_bf16_to_f64(q_row[i]);
    int64_t nk = 0;
    double m = -INFINITY;
    for (int64_t u = 0; u <= t; ++u) {
        use[u] = (sel == NULL) || block_selected(u / Bk, sel, nsel);
        if (!use[u]) continue;
        double dot = 0.0;
        for (int64_t i = 0; i < d; ++i) dot += qd[i] * oracle_bf16_to_f64(K[u * d + i]);
        z[u] = dot * scale;
        if (z[u] > m) m = z[u];
        ++nk;
    }
    double den = 0.0;
    for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
    for (int64_t u = 0; u <= t; ++u) {
        if (!use[u]) continue;
        double p = exp(z[u] - m);
        den += p;
        for (int64_t i = 0; i < d; ++i) o[i] += p * oracle_bf16_to_f64(V[u * d + i]);
    }
    for (int64_t i = 0; i < d; ++i) o[i] /= den;
    if (lse) *lse = m + log(den);
    free(qd); free(z); free(use);
    return nk;
}

/* ---------------------------------------------------------------- step 4, gradient */
/* Gradient of step 4 for one query head at position t, the selection held fixed (it is a
 * discrete choice), given the upstream gradient dO of the output o: writes dQ[d] and adds
 * this row's contributions to dK[u][d] and dV[u][d] for the keys u it attends. With
 * z_u = s q.k_u (s = 1/sqrt(d)), p = softmax(z) and o = sum_u p_u v_u:
 *   dV_u += p_u dO,   dp_u = dO.v_u,   dz_u = p_u (dp_u - dO.o),
 *   dQ = s sum_u dz_u k_u,   dK_u += s dz_u q.                                              */
void oracle_attend_row_grad(const uint16_t *q_row, const uint16_t *K, const uint16_t *V, int64_t d,
                            int64_t t, const int32_t *sel, int64_t nsel, int64_t Bk, const double *dO,
                            double *dQ, double *dK, double *dV)
{
    const double s = 1.0 / sqrt((double)d);
    double *qd = (double *)malloc((size_t)d * sizeof(double));
    double *o = (double *)malloc((size_t)d * sizeof(double));
    double *p = (double *)malloc((size_t)(t + 1) * sizeof(double));
    char *use = (char *)malloc((size_t)(t + 1));
    for (int64_t i = 0; i < d; ++i) qd[i] = oracle_bf16_to_f64(q_row[i]);
    double m = -INFINITY;
    for (int64_t u = 0; u <= t; ++u) {
        use[u] = (sel == NULL) || block_selected(u / Bk, sel, nsel);
        if (!use[u]) continue;
        double dot = 0.0;
        for (int64_t i = 0; i < d; ++i) dot += qd[i] * oracle_bf16_to_f64(K[u * d + i]);
        p[u] = dot * s;
        if (p[u] > m) m = p[u];
    }
    double den = 0.0;
    for (int64_t u = 0; u <= t; ++u)
        if (use[u]) { p[u] = exp(p[u] - m); den += p[u]; }
    for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
    for (int64_t u = 0; u <= t; ++u) {
        if (!use[u]) continue;
        p[u] /= den;
        for (int64_t i = 0; i < d; ++i) o[i] += p[u] * oracle_bf16_to_f64(V[u * d + i]);
    }
    double dOo = 0.0;
    for (int64_t i = 0; i < d; ++i) dOo += dO[i] * o[i];
    for (int64_t i = 0; i < d; ++i) dQ[i] = 0.0;
    for (int64_t u = 0; u <= t; ++u) {
        if (!use[u]) continue;
        double dp = 0.0;
        for (int64_t i = 0; i < d; ++i) dp += dO[i] * oracle_bf16_to_f64(V[u * d + i]);
        const double dz = p[u] * (dp - dOo);
        for (int64_t i = 0; i < d; ++i) {
            dV[u * d + i] += p[u] * dO[i];
            dQ[i] += s * dz * oracle_bf16_to_f64(K[u * d + i]);
            dK[u * d + i] += s * dz * qd[i];
        }
    }
    free(qd); free(o); free(p); free(use);
}

/* ---------------------------------------------------------------- FP8 (e4m3) key-value cache */
/* The compressed cache of the decode variant (KuCoin flash "MiniMax launches MSA sparse
 * attention method and MiniMax-M3 model", "ME AI News" paragraph: the SM100 kernel also
 * takes FP8 inputs). Reading taken: every closed block of Bk keys (or values) of one group
 * is stored as e4m3 codes with one fp32 scale per block; the open block, which is also the
 * newest query's own block, stays in bf16 until it fills.
 *
 * e4m3 ("E4M3FN"): sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, the
 * pattern S.1111.111 is NaN, largest finite value 448, subnormals m * 2^-9. */
double oracle_e4m3_to_f64(uint8_t c)
{
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* The e4m3 code nearest to x (ties to the code with an even mantissa), |x| > 448 saturating
 * to +-448: a search over the 127 non-negative finite codes, ascending. NaN maps to the
 * NaN pattern with the input's sign. */
uint8_t oracle_e4m3_from_f32(float x)
{
    const int s = signbit(x) ? 1 : 0;
    const double a = fabs((double)x);
    int best = 0;
    if (isnan(x)) return (uint8_t)(0x7F | (s << 7));   /* NaN keeps its sign, S.1111.111 */
    double bd = INFINITY;
    for (int c = 0; c <= 126; ++c) {
        const double dist = fabs(oracle_e4m3_to_f64((uint8_t)c) - a);
        if (dist < bd || (dist == bd && (c & 1) == 0)) { bd = dist; best = c; }
    }
    if (a > 448.0) best = 126;
    return (uint8_t)(best | (s << 7));
}

/* One block of n bf16 values: scale = amax / 448 in fp32 (1 for an all-zero block), and
 * codes[i] = e4m3(x_i / scale) with the division in fp32 (the precision that decides the
 * code on both sides). Returns the scale. */
float oracle_fp8_quantize_block(const uint16_t *x, int64_t n, uint8_t *codes)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        const float v = (float)fabs(oracle_bf16_to_f64(x[i]));
        if (v > amax) amax = v;
    }
    const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int64_t i = 0; i < n; ++i) {
        const float q = (float)oracle_bf16_to_f64(x[i]) / scale;
        codes[i] = oracle_e4m3_from_f32(q);
    }
    return scale;
}

/* Step 4 over the FP8 cache: keys and values of the fully-past blocks j < floor(t / Bk) are
 * code * scale (exact in fp64), those of the query's own block come from the bf16 rows;
 * everything else as in oracle_attend_row. Kc, Vc [L][d] codes; ks, vs one scale per block. */
int64_t oracle_attend_row_fp8(const uint16_t *q_row, const uint8_t *Kc, const uint8_t *Vc, const float *ks,
                              const float *vs, const uint16_t *K, const uint16_t *V, int64_t d, int64_t t,
                              const int32_t *sel, int64_t nsel, int64_t Bk, double *o, double *lse)
{
    const double scale = 1.0 / sqrt((double)d);
    const int64_t c = t / Bk;
    double *qd = (double *)malloc((size_t)d * sizeof(double));
    double *z = (double *)malloc((size_t)(t + 1) * sizeof(double));
    char *use = (char *)malloc((size_t)(t + 1));
    for (int64_t i = 0; i < d; ++i) qd[i] = oracle_bf16_to_f64(q_row[i]);
    int64_t nk = 0;
    double m = -INFINITY;
    for (int64_t u = 0; u <= t; ++u) {
        use[u] = (sel == NULL) || block_selected(u / Bk, sel, nsel);
        if (!use[u]) continue;
        const int64_t j = u / Bk;
        double dot = 0.0;
        for (int64_t i = 0; i < d; ++i) {
            const double k = j < c ? oracle_e4m3_to_f64(Kc[u * d + i]) * (double)ks[j]
                                   : oracle_bf16_to_f64(K[u * d + i]);
            dot += qd[i] * k;
        }
        z[u] = dot * scale;
        if (z[u] > m) m = z[u];
        ++nk;
    }
    double den = 0.0;
    for (int64_t i = 0; i < d; ++i) o[i] = 0.0;
    for (int64_t u = 0; u <= t; ++u) {
        if (!use[u]) continue;
        const int64_t j = u / Bk;
        const double p = exp(z[u] - m);
        den += p;
        for (int64_t i = 0; i < d; ++i) {
            const double v = j < c ? oracle_e4m3_to_f64(Vc[u * d + i]) * (double)vs[j]
                                   : oracle_bf16_to_f64(V[u * d + i]);
            o[i] += p * v;
        }
    }
    for (int64_t i = 0; i < d; ++i) o[i] /= den;
    if (lse) *lse = m + log(den);
    free(qd); free(z); free(use);
    return nk;
}

/* ---------------------------------------------------------------- row batches (threads) */
typedef struct {
    int kind;   /* 0 = select, 1 = attend */
    int64_t lo, hi;
    /* select */
    const int64_t *t; const uint16_t *q_idx_rows; const double *pooled_g; int64_t dI;
    int64_t Bk, topk; int32_t *sel; double *kth; int64_t *nsel;
    /* attend */
    const uint16_t *q_rows; int64_t Hg; const uint16_t *K, *V; int64_t d; const int32_t *sel_in;
    int dense; double *o, *lse; int64_t *nkeys;
} job_t;

static void *run_job(void *arg)
{
    job_t *jb = (job_t *)arg;
    for (int64_t r = jb->lo; r < jb->hi; ++r) {
        int64_t t = jb->t[r];
        if (jb->kind == 0) {
            int64_t c = t / jb->Bk;
            double *s = (double *)malloc((size_t)(c > 0 ? c : 1) * sizeof(double));
            oracle_block_scores(jb->q_idx_rows + r * jb->dI, jb->pooled_g, jb->dI, c, s);
            double kth;
            int64_t n = oracle_select_from_scores(s, c, jb->topk, jb->sel + r * jb->topk, &kth);
            if (jb->kth) jb->kth[r] = kth;
            if (jb->nsel) jb->nsel[r] = n;
            free(s);
        } else {
            const int32_t *sr = jb->dense ? NULL : jb->sel_in + r * jb->topk;
            int64_t ns = 0;
            if (sr) while (ns < jb->topk && sr[ns] >= 0) ++ns;
            for (int64_t h = 0; h < jb->Hg; ++h) {
                int64_t nk = oracle_attend_row(jb->q_rows + (r * jb->Hg + h) * jb->d, jb->K, jb->V,
                                               jb->d, t, sr, ns, jb->Bk,
                                               jb->o + (r * jb->Hg + h) * jb->d,
                                               jb->lse ? jb->lse + r * jb->Hg + h : NULL);
                if (jb->nkeys && h == 0) jb->nkeys[r] = nk;
            }
        }
    }
    return NULL;
}

static void run_parallel(job_t proto, int64_t n_rows, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    job_t jobs[256];
    int64_t per = (n_rows + nthreads - 1) / nthreads;
    int used = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = proto;
        jobs[i].lo = i * per;
        jobs[i].hi = (i + 1) * per < n_rows ? (i + 1) * per : n_rows;
        if (jobs[i].lo >= jobs[i].hi) break;
        pthread_create(&th[i], NULL, run_job, &jobs[i]);
        ++used;
    }
    for (int i = 0; i < used; ++i) pthread_join(th[i], NULL);
}

/* Selection for n_rows queries of one (sequence, group): query r sits at position t[r],
 * its index query row is q_idx_rows[r][dI]; pooled_g[nb][dI] holds the group's pooled keys.
 * sel: [n_rows][topk]; kth, nsel nullable [n_rows]. */
void oracle_select_rows(int64_t n_rows, const int64_t *t, const uint16_t *q_idx_rows,
                        const double *pooled_g, int64_t dI, int64_t Bk, int64_t topk,
                        int nthreads, int32_t *sel, double *kth, int64_t *nsel)
{
    job_t j;
    memset(&j, 0, sizeof j);
    j.kind = 0; j.t = t; j.q_idx_rows = q_idx_rows; j.pooled_g = pooled_g; j.dI = dI;
    j.Bk = Bk; j.topk = topk; j.sel = sel; j.kth = kth; j.nsel = nsel;
    run_parallel(j, n_rows, nthreads);
}

/* Attention for n_rows queries of one (sequence, group) on the given selections
 * (sel[n_rows][topk], -1 padded), or dense causal when dense != 0 (sel ignored).
 * q_rows: [n_rows][Hg][d]; K, V: [>= max t + 1][d] of the group; outputs o [n_rows][Hg][d],
 * lse [n_rows][Hg] (nullable), nkeys [n_rows] (nullable). */
void oracle_attend_rows(int64_t n_rows, const int64_t *t, const uint16_t *q_rows, int64_t Hg,
                        const uint16_t *K, const uint16_t *V, int64_t d, const int32_t *sel,
                        int64_t topk, int64_t Bk, int dense, int nthreads, double *o,
                        double *lse, int64_t *nkeys)
{
    job_t j;
    memset(&j, 0, sizeof j);
    j.kind = 1; j.t = t; j.q_rows = q_rows; j.Hg = Hg; j.K = K; j.V = V; j.d = d;
    j.sel_in = sel; j.topk = topk; j.Bk = Bk; j.dense = dense; j.o = o; j.lse = lse;
    j.nkeys = nkeys;
    run_parallel(j, n_rows, nthreads);
}
