/*
 * ivf_search_oracle.c -- plain, slow, fp64 CPU reference for IVF-Flat search over the
 * cells of a clustering.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg may load this library.  It shares no code, header or constant with the
 * CUDA path in exact_lloyd_means_b200/, and it never receives a value computed there.
 *
 * What it computes, and where that is defined (LEANN FlashLib guide, lumevalley mirror of
 * the LEANN docs, "LEANN FlashLib 后端实战指南"):
 *   - An IVF-Flat index is fitted on a corpus and answers the k nearest neighbours of a
 *     batch of queries (section "什么是 FlashLib 后端").
 *   - Its cells are the clusters of the coarse k-means: the centroids, and for every cell
 *     the points assigned to it (section "工作原理").
 *   - A query probes nprobe cells (sections "nlist 与 nprobe 的推导规则" and "参数速查");
 *     the plain reading, which the guide's remark that the probed candidate set is the
 *     one of the standard IVF-Flat implementations supports, is: the nprobe cells whose
 *     centroids are nearest to the query.
 *   - The only distance is squared L2 (section "距离度量只有 squared L2如何支持 mips /
 *     cosine"); cosine search runs on L2-normalised vectors, which the caller prepares.
 *
 * For each query q, in fp64 and with the distance in difference form sum_j (a_j - b_j)^2:
 *   1. the distance from q to every centroid;
 *   2. the nprobe cells with the smallest distance, ties to the lower cell index, listed in
 *      ascending (distance, cell) order;
 *   3. the candidates: every point whose cell label is one of those cells;
 *   4. the k candidates with the smallest distance, ties to the lower point index, listed
 *      in ascending (distance, index) order; when fewer than k candidates exist the
 *      remaining slots hold index -1 and distance +inf.
 * Readings where the guide is silent: the tie rules in 2 and 4 and the padding in 4.
 *
 * OpenMP splits the independent per-query loop only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/* (da, ia) comes strictly before (db, ib) in ascending (distance, index) order. */
static int before(double da, int32_t ia, double db, int32_t ib) {
    return da < db || (da == db && ia < ib);
}

/* Keep in (dl, il) the `cap` smallest entries seen so far, sorted ascending. */
static void keep_smallest(double *dl, int32_t *il, int *len, int cap, double dv, int32_t iv) {
    int n = *len;
    if (n == cap) {
        if (!before(dv, iv, dl[cap - 1], il[cap - 1])) return;
        n = cap - 1; /* the current last entry drops out */
    }
    int p = n;
    while (p > 0 && before(dv, iv, dl[p - 1], il[p - 1])) {
        dl[p] = dl[p - 1];
        il[p] = il[p - 1];
        --p;
    }
    dl[p] = dv;
    il[p] = iv;
    *len = n + 1;
}

static double sq_dist(const double *a, const double *b, int d) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) {
        const double t = a[j] - b[j];
        s += t * t;
    }
    return s;
}

/* Returns 0, or 1 when an argument is out of range (a label outside [0, nlist), nprobe
 * outside [1, nlist], k < 1). */
int orc_ivf_search(const double *Q, int64_t nq, int d, const double *C, int nlist,
                   const double *X, int64_t n, const int32_t *labels, int nprobe, int k,
                   int32_t *probes, int32_t *ids, double *dist) {
    if (nlist < 1 || nprobe < 1 || nprobe > nlist || k < 1 || d < 1) return 1;
    for (int64_t i = 0; i < n; ++i)
        if (labels[i] < 0 || labels[i] >= nlist) return 1;

    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t q = 0; q < nq; ++q) {
        const double *qv = Q + q * (int64_t)d;
        double *pd = (double *)malloc(sizeof(double) * (size_t)nprobe);
        int32_t *pi = (int32_t *)malloc(sizeof(int32_t) * (size_t)nprobe);
        char *probed = (char *)calloc((size_t)nlist, 1);
        double *kd = (double *)malloc(sizeof(double) * (size_t)k);
        int32_t *ki = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        int plen = 0, klen = 0;

        for (int c = 0; c < nlist; ++c)
            keep_smallest(pd, pi, &plen, nprobe, sq_dist(qv, C + (int64_t)c * d, d), c);
        for (int t = 0; t < plen; ++t) probed[pi[t]] = 1;

        for (int64_t i = 0; i < n; ++i)
            if (probed[labels[i]])
                keep_smallest(kd, ki, &klen, k, sq_dist(qv, X + i * (int64_t)d, d),
                              (int32_t)i);

        for (int t = 0; t < nprobe; ++t) probes[q * nprobe + t] = pi[t];
        for (int t = 0; t < k; ++t) {
            ids[q * k + t] = t < klen ? ki[t] : -1;
            dist[q * k + t] = t < klen ? kd[t] : INFINITY;
        }
        free(pd);
        free(pi);
        free(probed);
        free(kd);
        free(ki);
    }
    return 0;
}
