/*
 * lloyd_oracle.c -- plain, slow, fp64 CPU reference for one exact Lloyd's k-means
 * iteration.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg may load this library.  It shares no code, header or constant with the
 * CUDA path in exact_lloyd_means_b200/, and it never receives a value computed there.
 *
 * What it computes, and where that is defined:
 *   - One Lloyd iteration = assign every point to its nearest centroid, then recompute
 *     every centroid as the mean of its points.  Flash-KMeans article (lumevalley.com,
 *     "UC Berkeley + UT Austin Flash-KMeans"), section "为什么"快"这件事被拖了这么久":
 *     an iteration assigns N points to K clusters and recomputes the centroids.  The
 *     opening paragraph states the method is exact standard Lloyd's, no approximation,
 *     so the plain definition below is the oracle.
 *   - The distance is squared Euclidean (same article, section "它不是银弹，但切中了一个
 *     真痛点": L2 and cosine only; LEANN FlashLib guide, section "距离度量只有 squared L2
 *     如何支持 mips / cosine").
 *   - Cosine mode = L2-normalise rows, a zero-norm row is divided by 1 (LEANN FlashLib
 *     guide, same section).
 *   - The sorted inverse index (a permutation grouping points by cluster id) and the CSR
 *     cluster offsets: Flash-KMeans article, section "Sort-Inverse Update：原子操作的
 *     另一种解法" (sort assignments by cluster id into an inverse index), and LEANN
 *     FlashLib guide, section "工作原理" (cell-contiguous rows, row ids, CSR offsets).
 *
 * Every loop below is the textbook definition, in fp64, with no blocking, no expansion of
 * the distance and no reordering beyond "in index order".  OpenMP splits only the
 * independent per-point (or per-centroid) loops; every sum that crosses points runs
 * sequentially in index order, so results do not depend on the thread count.
 *
 * Readings where the pages are silent (each is listed in the design notes as well):
 *   - argmin ties go to the lowest centroid index (first occurrence);
 *   - a cluster with no points keeps its previous centroid bit for bit;
 *   - the objective J is sum_i ||x_i - c_{l_i}||^2 against the centroids the labels
 *     were assigned with.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the parallel loops below (n >= 1); results do not depend on it. */
void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* x_i <- x_i / ||x_i||, with ||x_i|| replaced by 1 when it is 0 (LEANN FlashLib guide,
 * "距离度量只有 squared L2如何支持 mips / cosine": zero-norm vectors are protected as 1). */
void orc_normalize_rows(double *X, int64_t n, int d) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double *x = X + i * (int64_t)d;
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += x[j] * x[j];
        double nrm = sqrt(s);
        if (nrm == 0.0) nrm = 1.0;
        for (int j = 0; j < d; ++j) x[j] = x[j] / nrm;
    }
}

/* Squared Euclidean distance in difference form: sum_j (x_j - c_j)^2. */
static double sqdist(const double *x, const double *c, int d) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) {
        double t = x[j] - c[j];
        s += t * t;
    }
    return s;
}

/* Assignment step.  For every point i: D_ik = ||x_i - c_k||^2 for all k; the label is the
 * smallest k attaining the minimum.  dmin[i] = min_k D_ik, d2nd[i] = the second smallest
 * value over all k (equal to dmin[i] when the minimum is attained twice; +inf when K=1).
 * dmin and d2nd may be NULL. */
void orc_assign(const double *X, int64_t n, int d, const double *C, int K,
                int32_t *labels, double *dmin, double *d2nd) {
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        const double *x = X + i * (int64_t)d;
        double best = INFINITY, second = INFINITY;
        int32_t bk = 0;
        for (int k = 0; k < K; ++k) {
            double s = sqdist(x, C + (int64_t)k * d, d);
            if (s < best) {
                second = best;
                best = s;
                bk = k;
            } else if (s < second) {
                second = s;
            }
        }
        labels[i] = bk;
        if (dmin) dmin[i] = best;
        if (d2nd) d2nd[i] = second;
    }
}

/* Objective J = sum_i ||x_i - c_{labels[i]}||^2, summed in index order. */
double orc_objective(const double *X, int64_t n, int d, const double *C,
                     const int32_t *labels) {
    double *per = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        per[i] = sqdist(X + i * (int64_t)d, C + (int64_t)labels[i] * d, d);
    double J = 0.0;
    for (int64_t i = 0; i < n; ++i) J += per[i];
    free(per);
    return J;
}

/* Sorted inverse index by cluster id.  counts[k] = #{i : labels[i] == k};
 * offsets = exclusive prefix sum of counts (K+1 entries, offsets[K] = n);
 * perm = the point indices ordered by (label, index): a stable counting sort.
 * Returns 0, or -1 if a label lies outside [0, K). */
int orc_csr(const int32_t *labels, int64_t n, int K, int32_t *counts,
            int32_t *offsets, int32_t *perm) {
    for (int k = 0; k < K; ++k) counts[k] = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (labels[i] < 0 || labels[i] >= K) return -1;
        counts[labels[i]] += 1;
    }
    offsets[0] = 0;
    for (int k = 0; k < K; ++k) offsets[k + 1] = offsets[k] + counts[k];
    int32_t *cursor = (int32_t *)malloc((size_t)K * sizeof(int32_t));
    for (int k = 0; k < K; ++k) cursor[k] = offsets[k];
    for (int64_t i = 0; i < n; ++i) perm[cursor[labels[i]]++] = (int32_t)i;
    free(cursor);
    return 0;
}

/* Update step.  For each cluster k with at least one point:
 *   c_k <- (sum of its points, added in index order) / (number of its points);
 * a cluster with no points keeps C_old[k] unchanged. */
void orc_update(const double *X, int64_t n, int d, const int32_t *labels,
                const double *C_old, int K, double *C_new) {
    double *sums = (double *)calloc((size_t)K * d, sizeof(double));
    int64_t *cnt = (int64_t *)calloc((size_t)K, sizeof(int64_t));
    for (int64_t i = 0; i < n; ++i) {
        const double *x = X + i * (int64_t)d;
        double *s = sums + (int64_t)labels[i] * d;
        for (int j = 0; j < d; ++j) s[j] += x[j];
        cnt[labels[i]] += 1;
    }
    #pragma omp parallel for schedule(static)
    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < d; ++j) {
            int64_t o = (int64_t)k * d + j;
            C_new[o] = cnt[k] > 0 ? sums[o] / (double)cnt[k] : C_old[o];
        }
    }
    free(sums);
    free(cnt);
}
