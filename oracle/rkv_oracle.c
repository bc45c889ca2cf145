/*
 * rkv_oracle.c -- CPU oracle of the R-KV decode-time KV-cache compression step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only on the seeded bf16 inputs.
 *
 * Plain nested loops in double precision.  Inputs are bf16 bit patterns,
 * widened exactly to double.  One "unit" is one (sequence, layer, KV head).
 *
 * What the step computes, per unit, with N cached tokens, w = window,
 * M = N - w candidates, k = budget - w tokens kept from the candidates
 * (R-KV pages: hysenlabs write-up, "What the redundancy scoring actually
 * does at decode time"; sourcepulse summary, "How It Works"; atlas.scime.ai
 * summary, "Approach", which prints the only formula, Z = lambda I - (1-lambda) R):
 *   1. importance I from the last w queries' scaled softmax attention over the
 *      cached keys, averaged over the w queries and max-pooled over the GQA
 *      query-head group (max pooling: atlas.scime.ai "Measured effects" table,
 *      GQA pooling ablation row), renormalised over the M candidates;
 *   2. redundancy r from the cosine similarity of L2-normalised keys (mean over
 *      the other N-1 cached keys, or their max), R = softmax over candidates;
 *   3. Z = lambda I - (1 - lambda) R;
 *   4. keep the top k candidates by (Z descending, index ascending) plus the
 *      protected window M..N-1, in ascending original order;
 *   5. compact K and V to those rows.
 * Readings of points the pages leave open (which queries, the 1/sqrt(D)
 * scale, the causal mask, the order of window mean and GQA max, the
 * renormalisation of I, the redundancy reduction, the zero-norm clamp, the
 * tie rule, the output order) are listed with the design notes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define RKV_ORACLE_POOL_MAX 0
#define RKV_ORACLE_POOL_MEAN 1
#define RKV_ORACLE_RED_MEAN 0
#define RKV_ORACLE_RED_MAX 1

static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Importance (step 1).  q: [G][w][D], k: [N][D] (row-major bf16 bits).
 * Query j of a head sits at position M + j and attends to keys 0..M+j.
 * I_out: [M], normalised to sum 1 over the candidates.
 * Pages: "importance (derived from attention weights)" (sourcepulse, How It
 * Works); "max pooling to aggregate GQA attention scores" beats mean pooling
 * (atlas.scime.ai, Measured effects table).
 */
void rkv_oracle_importance(const uint16_t *q, const uint16_t *k, int G, int w, int D,
                           int N, int pool, double *I_out)
{
    int M = N - w;
    double scale = 1.0 / sqrt((double)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *a = (double *)malloc(sizeof(double) * (size_t)M);
    double *ihat = (double *)malloc(sizeof(double) * (size_t)M);

    for (int i = 0; i < M; ++i)
        ihat[i] = (pool == RKV_ORACLE_POOL_MAX) ? -INFINITY : 0.0;

    for (int g = 0; g < G; ++g) {
        for (int i = 0; i < M; ++i)
            a[i] = 0.0;
        for (int j = 0; j < w; ++j) {
            const uint16_t *qv = q + ((size_t)g * w + j) * D;
            int visible = M + j + 1; /* keys 0 .. M+j */
            double mx = -INFINITY;
            for (int i = 0; i < visible; ++i) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += widen_bf16(qv[d]) * widen_bf16(k[(size_t)i * D + d]);
                s[i] = dot * scale;
                if (s[i] > mx)
                    mx = s[i];
            }
            double den = 0.0;
            for (int i = 0; i < visible; ++i) {
                s[i] = exp(s[i] - mx);
                den += s[i];
            }
            for (int i = 0; i < M; ++i)
                a[i] += (s[i] / den) / (double)w;
        }
        for (int i = 0; i < M; ++i) {
            if (pool == RKV_ORACLE_POOL_MAX) {
                if (a[i] > ihat[i])
                    ihat[i] = a[i];
            } else {
                ihat[i] += a[i] / (double)G;
            }
        }
    }

    double tot = 0.0;
    for (int i = 0; i < M; ++i)
        tot += ihat[i];
    for (int i = 0; i < M; ++i)
        I_out[i] = ihat[i] / tot;

    free(s);
    free(a);
    free(ihat);
}

/* Inverse key norms 1 / max(||k_i||, 1e-12), for all N keys. */
void rkv_oracle_inv_norm(const uint16_t *k, int N, int D, double *inv)
{
    for (int i = 0; i < N; ++i) {
        double ss = 0.0;
        for (int d = 0; d < D; ++d) {
            double x = widen_bf16(k[(size_t)i * D + d]);
            ss += x * x;
        }
        double nrm = sqrt(ss);
        inv[i] = 1.0 / (nrm > 1e-12 ? nrm : 1e-12);
    }
}

/*
 * Redundancy (step 2), raw per-candidate score r: [M].
 * c_ij = khat_i . khat_j with khat = k / max(||k||, 1e-12).
 * mode MEAN: r_i = (1/(N-1)) sum_{j<N, j!=i} c_ij;  mode MAX: r_i = max_{j<N, j!=i} c_ij.
 * Pages: redundancy is the "key-vector cosine similarity" (atlas.scime.ai,
 * summary and Approach); cosine similarity identifies near-duplicates
 * (sourcepulse, How It Works).
 */
void rkv_oracle_redundancy(const uint16_t *k, int N, int D, int M, int mode, double *r)
{
    double *inv = (double *)malloc(sizeof(double) * (size_t)N);
    double *kh = (double *)malloc(sizeof(double) * (size_t)N * D);
    rkv_oracle_inv_norm(k, N, D, inv);
    for (int i = 0; i < N; ++i)
        for (int d = 0; d < D; ++d)
            kh[(size_t)i * D + d] = widen_bf16(k[(size_t)i * D + d]) * inv[i];

    for (int i = 0; i < M; ++i) {
        double acc = (mode == RKV_ORACLE_RED_MAX) ? -INFINITY : 0.0;
        for (int j = 0; j < N; ++j) {
            if (j == i)
                continue;
            double c = 0.0;
            for (int d = 0; d < D; ++d)
                c += kh[(size_t)i * D + d] * kh[(size_t)j * D + d];
            if (mode == RKV_ORACLE_RED_MAX) {
                if (c > acc)
                    acc = c;
            } else {
                acc += c;
            }
        }
        r[i] = (mode == RKV_ORACLE_RED_MAX) ? acc : acc / (double)(N - 1);
    }
    free(inv);
    free(kh);
}

/* y = softmax(x) over n entries (max-subtracted). */
void rkv_oracle_softmax(const double *x, int n, double *y)
{
    double mx = -INFINITY;
    for (int i = 0; i < n; ++i)
        if (x[i] > mx)
            mx = x[i];
    double den = 0.0;
    for (int i = 0; i < n; ++i) {
        y[i] = exp(x[i] - mx);
        den += y[i];
    }
    for (int i = 0; i < n; ++i)
        y[i] /= den;
}

/* Joint score (step 3): Z = lambda I - (1 - lambda) R  (atlas.scime.ai, Approach). */
void rkv_oracle_joint(const double *I, const double *R, int M, double lambda, double *Z)
{
    for (int i = 0; i < M; ++i)
        Z[i] = lambda * I[i] - (1.0 - lambda) * R[i];
}

typedef struct {
    double z;
    int i;
} scored_t;

static int by_score_then_index(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa;
    const scored_t *b = (const scored_t *)pb;
    if (a->z > b->z)
        return -1;
    if (a->z < b->z)
        return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i) ? 1 : 0;
}

static int ascending_int(const void *pa, const void *pb)
{
    int a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * Selection (step 4): the first k = budget - w candidates in (Z desc, index asc)
 * order, sorted ascending, followed by the window M..N-1.  kept: [budget].
 * Pages: "a joint selection mechanism then retains the top-k tokens within a
 * budget" (sourcepulse, How It Works); "window_size 8 keeps a recent-token
 * window that is exempt from eviction" (hysenlabs, decode-time section).
 */
void rkv_oracle_select(const double *Z, int M, int N, int budget, int32_t *kept)
{
    int w = N - M;
    int kk = budget - w;
    scored_t *c = (scored_t *)malloc(sizeof(scored_t) * (size_t)(M > 0 ? M : 1));
    for (int i = 0; i < M; ++i) {
        c[i].z = Z[i];
        c[i].i = i;
    }
    qsort(c, (size_t)M, sizeof(scored_t), by_score_then_index);
    for (int t = 0; t < kk; ++t)
        kept[t] = c[t].i;
    qsort(kept, (size_t)kk, sizeof(int32_t), ascending_int);
    for (int t = 0; t < w; ++t)
        kept[kk + t] = M + t;
    free(c);
}

/* Compaction (step 5): dst[t] = src[kept[t]] for t < budget, rows of D bf16. */
void rkv_oracle_compact(const uint16_t *src, const int32_t *kept, int budget, int D,
                        uint16_t *dst)
{
    for (int t = 0; t < budget; ++t)
        for (int d = 0; d < D; ++d)
            dst[(size_t)t * D + d] = src[(size_t)kept[t] * D + d];
}

/*
 * The whole step for one unit.  Outputs I, r, R, Z: [M]; kept: [budget].
 */
void rkv_oracle_unit(const uint16_t *q, const uint16_t *k, int G, int w, int D, int N,
                     int budget, double lambda, int red_mode, int pool, double *I,
                     double *r, double *R, double *Z, int32_t *kept)
{
    int M = N - w;
    rkv_oracle_importance(q, k, G, w, D, N, pool, I);
    rkv_oracle_redundancy(k, N, D, M, red_mode, r);
    rkv_oracle_softmax(r, M, R);
    rkv_oracle_joint(I, R, M, lambda, Z);
    rkv_oracle_select(Z, M, N, budget, kept);
}

/*
 * Shared selection across the KV heads of one (sequence, layer): the eviction
 * score of candidate i is the sum over the H heads of their joint scores,
 * Zsum_i = sum_h Z_h[i] (h ascending, double), and every head keeps the same
 * set: the top k of Zsum by (score desc, index asc) plus the window.  This is
 * what a tensor-parallel deployment needs so that all ranks evict the
 * identical tokens: each rank sums its own heads and an all-reduce (sum) over
 * the ranks completes Zsum (hysenlabs write-up, decode-time section: the vLLM
 * port's cross-rank eviction-score all-reduce; every TP rank evicts the
 * identical set).  Z: H rows of stride zstride; Zsum: [M]; kept: [budget].
 */
void rkv_oracle_shared_select(const double *Z, int H, long long zstride, int M, int N,
                              int budget, double *Zsum, int32_t *kept)
{
    for (int i = 0; i < M; ++i) {
        double s = 0.0;
        for (int h = 0; h < H; ++h)
            s += Z[(size_t)h * zstride + i];
        Zsum[i] = s;
    }
    rkv_oracle_select(Zsum, M, N, budget, kept);
}

/*
 * Many units at once (OpenMP over units when built with -fopenmp).
 * q: [U][G*w*D]; k: [U][kstride] with the first N[u] rows valid;
 * outputs with row strides ostride (I, r, R, Z) and kstride_out (kept).
 */
void rkv_oracle_units(int U, const uint16_t *q, const uint16_t *k, long long kstride,
                      const int32_t *N, const int32_t *budget, const double *lambda, int G,
                      int w, int D, int red_mode, int pool, double *I, double *r, double *R,
                      double *Z, long long ostride, int32_t *kept, long long kept_stride,
                      int n_threads)
{
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
#endif
    for (int u = 0; u < U; ++u) {
        rkv_oracle_unit(q + (size_t)u * G * w * D, k + (size_t)u * kstride, G, w, D, N[u],
                        budget[u], lambda[u], red_mode, pool, I + (size_t)u * ostride,
                        r + (size_t)u * ostride, R + (size_t)u * ostride,
                        Z + (size_t)u * ostride, kept + (size_t)u * kept_stride);
    }
    (void)n_threads;
}
