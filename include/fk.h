/*
 * fk.h -- C ABI of the exact Lloyd's k-means library (libfk.so), sm_100a (B200).
 *
 * One Lloyd iteration = (1) assign every point to its nearest centroid under squared
 * L2, without materialising the N x K distance matrix, and (2) recompute every centroid
 * as the mean of its points through a sorted inverse index, with no atomics.  Sources:
 *   - Flash-KMeans article (lumevalley.com, "UC Berkeley + UT Austin Flash-KMeans"),
 *     opening paragraph: exact standard Lloyd's, no approximation;
 *     section "为什么"快"这件事被拖了这么久": an iteration assigns N points to K
 *     clusters, then recomputes the centroids;
 *     section "FlashAssign：把距离矩阵按块切成流水线": distances are computed tile by
 *     tile and reduced to an argmin on chip, so only O(Nd + Kd) data moves;
 *     section "Sort-Inverse Update：原子操作的另一种解法": sort the assignments by
 *     cluster id into an inverse index, then reduce each cluster by reading its points
 *     contiguously, with no atomics;
 *     section "它不是银弹，但切中了一个真痛点": L2 and cosine only.
 *   - LEANN FlashLib guide (mhpn.cn, "LEANN FlashLib 后端实战指南"),
 *     section "距离度量只有 squared L2如何支持 mips / cosine": cosine = L2-normalise the
 *     vectors, a zero-norm vector is divided by 1;
 *     section "nlist 与 nprobe 的推导规则": the cluster count is clamped to n (here
 *     K > N is an argument error; a caller may clamp);
 *     section "工作原理": the build output is CSR cluster offsets plus cell-ordered row
 *     ids.
 *
 * Conventions for every call:
 *   - All matrices are row-major and contiguous: X is N x d, centroids are K x d.
 *   - Pointers are DEVICE pointers unless a parameter says "host".  Input buffers are
 *     read-only unless stated; the caller owns every buffer, including the workspace.
 *   - The library never allocates device memory: scratch comes from the caller's
 *     workspace `ws` of `ws_bytes` bytes (query the size with fk_workspace_size; the
 *     pointer must be 256-byte aligned).  One workspace must not be used by two calls
 *     that can run at the same time.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) unless stated.  Argument checks are synchronous and return an error before
 *     anything is launched.  A failed launch returns FK_ERR_CUDA.
 *   - Device-side checks (a label outside [0, K), a bounded wait that expired inside a
 *     kernel) set an error word in the first 256 bytes of the workspace; fk_lloyd clears
 *     it on entry and reports it on return, fk_get_device_error reads and clears it for
 *     the asynchronous calls.  Zero a new workspace once (or call fk_get_device_error on
 *     it) before the first fk_assign / fk_update.  No kernel traps.
 *   - Results are deterministic: the same inputs on the same device give the same bits,
 *     run after run (no atomics on any floating-point value, fixed reduction orders).
 *   - Limits: 1 <= K <= N < 2^31, d >= 1; FK_F32 needs d % 4 == 0 and X 16-byte
 *     aligned; FK_BF16 needs d % 8 == 0 and X 16-byte aligned; FK_COSINE needs FK_F32.
 *     Violations return FK_ERR_INVALID_ARG (shape/pointer) or FK_ERR_UNSUPPORTED
 *     (dtype/alignment/device other than sm_100).
 */
#ifndef FK_H
#define FK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FK_API __attribute__((visibility("default")))
#else
#define FK_API
#endif

typedef struct CUstream_st *fk_stream_t; /* same type as cudaStream_t */

typedef enum fk_status {
    FK_OK = 0,
    FK_ERR_INVALID_ARG = 1, /* bad shape, null required pointer, K > N, ...          */
    FK_ERR_UNSUPPORTED = 2, /* dtype/metric/alignment/device not supported            */
    FK_ERR_WORKSPACE = 3,   /* ws null, misaligned or smaller than fk_workspace_size  */
    FK_ERR_CUDA = 4,        /* a CUDA runtime/driver call or a launch failed          */
    FK_ERR_TIMEOUT = 5,     /* a bounded wait inside a kernel expired                 */
    FK_ERR_DEVICE = 6       /* a device-side argument check failed (label range)      */
} fk_status;

typedef enum fk_dtype {
    FK_F32 = 0,   /* fp32 points; products emulated to fp32 accuracy with three bf16
                     tensor-core products (hi*hi + lo*hi + hi*lo)                     */
    FK_BF16 = 1,  /* bf16 points; bf16 tensor-core products (exact), fp32 accumulation */
    FK_BF16X2 = 2 /* fp32 points given already split by fk_split_points (bf16 hi/lo
                     planes, then ||x||^2 per row); fk_assign only                     */
} fk_dtype;

typedef enum fk_metric {
    FK_L2 = 0,     /* squared Euclidean distance                                     */
    FK_COSINE = 1  /* L2-normalise points and initial centroids, then squared L2     */
} fk_metric;

/* Per-phase device time of an fk_lloyd call, summed over its iterations (CUDA events
 * recorded on the caller's stream around each phase). */
typedef struct fk_timing {
    double ms_setup;   /* once per call: normalisation (cosine), the fp32 split of X and
                          the screening probe                                          */
    double ms_prep;    /* per iteration: centroid norms and operand preparation        */
    double ms_assign;  /* per iteration: the whole assignment (every kernel of it)     */
    double ms_sort;    /* per iteration: radix sort of labels -> perm + CSR offsets   */
    double ms_update;  /* per iteration: segmented reduction, combine, finalize, J     */
    int iterations;
    int launches;      /* kernels this call launched (library kernels only)            */
    double ms_assign_mma; /* per iteration: the main tensor-core kernel of the assignment
                             alone (the single-product screening pass on the screened
                             route, else the assign kernel)                           */
    int screened;      /* iterations that took the screened route                      */
    int empty_clusters; /* last iteration: clusters that received no point (kept their
                           previous centroid)                                           */
    int max_cluster;    /* last iteration: points in the largest cluster                */
    int fallback_rows;  /* last iteration, screened route: rows sent to the three-product
                           pass (0 when the iteration was not screened)                 */
    int kernel_only;    /* IN: 1 times only the main tensor-core kernel of each
                           assignment (two events per iteration), 2 only that of the last
                           iteration (two events per call): ms_assign_mma, mma_timed,
                           iterations, launches and screened are filled, every other field
                           is 0.  The lightest timing, for loops of short calls, where the
                           events between the phases would cost a noticeable share.  0
                           times every phase.  The call keeps this field as given.       */
    int mma_timed;      /* launches of the main kernel whose device time ms_assign_mma
                           sums (niter, or 1 with kernel_only = 2)                      */
} fk_timing;

/* Human-readable name of a status code (static string, never NULL). */
FK_API const char *fk_status_string(fk_status s);

/* Library ABI version (incremented on any signature or struct change). */
FK_API int fk_version(void);

/* Number of kernels this library has launched from the calling host thread since it was
 * loaded (every entry point counts its own launches).  Host-only; for accounting. */
FK_API int64_t fk_launch_count(void);

/* Bytes of workspace that fk_assign, fk_update and fk_lloyd need for this problem
 * (any of them; the largest need).  Host-only, synchronous.  `bytes` is a host pointer. */
FK_API fk_status fk_workspace_size(int64_t N, int d, int K, fk_dtype dtype, fk_metric metric,
                            size_t *bytes);

/* Row L2 normalisation (cosine mode, step 0): X_out[i] = X_in[i] / ||X_in[i]||, where a
 * zero norm is replaced by 1 (LEANN FlashLib guide, "距离度量只有 squared L2如何支持
 * mips / cosine").  The norm is accumulated in fp64 and each output is rounded once to
 * fp32.  fp32 only; X_out may equal X_in (in place).  N x d row-major. */
FK_API fk_status fk_normalize_rows(const float *X_in, float *X_out, int64_t N, int d,
                            fk_stream_t stream);

/* Split fp32 points once for repeated assignment (the first step of fk_assign for
 * FK_F32).  `planes` (device, 16-byte aligned, 4*N*d_p + 4*N bytes, d_p = roundup(d, 64))
 * receives [2][N][d_p] bf16, hi = RN_bf16(x) then lo = RN_bf16(x - hi), zero padded,
 * followed by [N] fp32 ||x||^2 (fp64 accumulation, one rounding).  It can then be passed
 * to fk_assign as X with dtype FK_BF16X2, skipping the per-call split.  fp32 only
 * (d % 4 == 0, X 16-byte aligned). */
FK_API fk_status fk_split_points(const float *X, int64_t N, int d, void *planes,
                                 fk_stream_t stream);

/* Centroid norms: cn[k] = sum_j c_kj^2 over the values the tensor cores consume (the
 * fp32 centroids for FK_F32, their bf16 rounding for FK_BF16), accumulated in fp64 and
 * rounded once to fp32.  C is K x d fp32; cn has K floats. */
FK_API fk_status fk_centroid_norms(const float *C, int K, int d, fk_dtype dtype, float *cn,
                            fk_stream_t stream);

/* Assignment step (Flash-KMeans article, "FlashAssign：把距离矩阵按块切成流水线").
 *   labels[i] = argmin_k ||x_i - c_k||^2, lowest k on exact ties, for i < N.
 *   mind[i]   = min_k ||x_i - c_k||^2 (optional, pass NULL to skip), within
 *               1e-4 (||x_i||^2 + max_k ||c_k||^2): the re-ranking's fp64
 *               difference form on the screened route below, else the tensor-core
 *               expansion ||x||^2 + (||c||^2 - 2 x.c).
 * X: N x d, dtype `dtype`.  C: K x d fp32 (for FK_BF16 the kernel uses C rounded to
 * bf16).  labels: N int32.  The N x K distance matrix is never stored: a tcgen05 kernel
 * keeps one 128 x 256 fp32 tile in tensor memory and a running min/argmin per row.
 * For FK_F32 each call first splits X into bf16 hi/lo planes inside `ws` (one extra
 * pass over X; fk_lloyd does this once per call instead of once per iteration); callers
 * that assign the same points repeatedly split once with fk_split_points and pass the
 * planes with FK_BF16X2.
 * Screened route (fp32 points, N >= 18,944 rows, d >= 256 or K * d >= 2^22, C 16-byte
 * aligned): one bf16 product
 * per term finds, for every row, the centroids within a proven bound of the nearest; their
 * distances (fp64, difference form) pick the label, and rows with more such
 * centroids than the kernel keeps are assigned by the three-product form.  Labels are the
 * same as the three-product form's outside the parity tie window.
 * Deep fp32 points (d rounded up to 64 above 768): the three-product form's error is not
 * shown to stay within half the tie window there, so every such call takes the screened
 * route whatever N, and rows whose candidates overflow are assigned by an exact fp64 scan
 * over all K centroids instead; C must then be 16-byte aligned (else
 * FK_ERR_UNSUPPORTED).  With FK_BF16X2 input the re-ranking (and that scan) measures the
 * distances from hi + lo, which is within 2^-16 |x| of x; fk_assign_split keeps them
 * exact. */
FK_API fk_status fk_assign(const void *X, fk_dtype dtype, int64_t N, int d, const float *C,
                    int K, int32_t *labels, float *mind, void *ws, size_t ws_bytes,
                    fk_stream_t stream);

/* fk_assign for fp32 points passed twice: as the rows X (N x d fp32, 16-byte aligned),
 * which the exact fp64 re-ranking of the screened route reads, and as `planes`, the output
 * of fk_split_points on that same X, which the tensor cores read.  A caller that assigns
 * the same points repeatedly (the data-parallel Lloyd) splits them once and still gets
 * exact re-ranking.  Labels and mind equal fk_assign(X, FK_F32) bit for bit; X and
 * `planes` must stay unchanged between the split and this call.  Workspace:
 * fk_workspace_size(N, d, K, FK_BF16X2, FK_L2).  Same errors as fk_assign. */
FK_API fk_status fk_assign_split(const float *X, const void *planes, int64_t N, int d,
                                 const float *C, int K, int32_t *labels, float *mind,
                                 void *ws, size_t ws_bytes, fk_stream_t stream);

/* Update step (Flash-KMeans article, "Sort-Inverse Update：原子操作的另一种解法").
 *   counts[k]  = #{i : labels[i] == k}                         (K int32, required)
 *   offsets    = exclusive prefix sum of counts, offsets[K] = N (K+1 int32, required)
 *   perm       = point indices ordered by (label, index)        (N int32, optional)
 *   C_new[k]   = mean of the points with label k, or C_old[k] bit for bit when the
 *                cluster is empty                              (K x d fp32, required;
 *                must not overlap C_old)
 *   *objective = sum_i ||x_i - c_old[labels[i]]||^2 in fp64 (device double, optional),
 *                where c_old is C_old for FK_F32 and C_old rounded to bf16 for FK_BF16
 *                (the centroids the labels were assigned with).
 * The labels are sorted with an atomic-free, stable LSD radix sort; each cluster's sum is
 * accumulated in fp64 in a fixed order (rows in index order within fixed chunks, chunk
 * partials combined in chunk order), so the result does not depend on timing.
 * A label outside [0, K) sets FK_ERR_DEVICE in the workspace error word. */
FK_API fk_status fk_update(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                    const int32_t *labels, const float *C_old, float *C_new,
                    int32_t *counts, int32_t *offsets, int32_t *perm, double *objective,
                    void *ws, size_t ws_bytes, fk_stream_t stream);

/* `niter` Lloyd iterations from the initial centroids in C (K x d fp32, overwritten with
 * the final centroids).  Cosine mode normalises X (into the workspace; X itself is not
 * modified) and the initial C first.  On return (this call synchronises `stream` at the
 * end, and once more after the screening probe where fp32 points may take the screened
 * route):
 *   labels           N int32, the labels of the last assignment (device);
 *   counts, offsets  of the last assignment (device; optional, may be NULL);
 *   objective_host   niter doubles (HOST pointer, optional): entry t is the objective
 *                    of iteration t's labels against the centroids they were assigned
 *                    with;
 *   timing           HOST pointer (optional): device milliseconds of every phase, or of
 *                    the assignment kernel alone (see fk_timing.kernel_only).
 * niter = 0 only normalises C (cosine) and returns.
 * A short call (at most 1e12 useful flops, 2 N K d niter: launches are a large share of
 * it) that repeats the previous call on the same host thread (same pointers, sizes,
 * metric, iteration count below 4096, timing mode, device and probe decision) records
 * its iteration loop and end-of-call copies into a CUDA graph, and later identical calls
 * replay it (up to four graphs per thread).  The graph reads X and C when it runs, so new
 * values need no new capture; results are the same bits either way.  FK_LOOP_GRAPH=0 in
 * the environment runs every call eagerly.  For this the library keeps per-thread
 * streams, events, pinned host staging and graphs, each tied to the CUDA context it was
 * made in and dropped when that context changes. */
FK_API fk_status fk_lloyd(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                   fk_metric metric, int niter, float *C, int32_t *labels,
                   int32_t *counts, int32_t *offsets, double *objective_host,
                   fk_timing *timing, void *ws, size_t ws_bytes, fk_stream_t stream);

/* Data-parallel Lloyd over shards of X (one call per shard, typically one per GPU; X
 * rows split, centroids replicated).  Same steps as fk_update, but instead of centroids
 * the shard's per-cluster sums are returned for a combine across shards:
 *   sums      K x d fp64 (device): sum of the shard's points with label k (zeros when none)
 *   counts    K int32: points of the shard per cluster; offsets: the shard's CSR (K+1)
 *   objective fp64 (device, optional): sum over the shard of ||x_i - c_used[l_i]||^2
 * The sums are accumulated in fp64 in the fixed order of fk_update. */
FK_API fk_status fk_update_partial(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                                   const int32_t *labels, const float *C_old, double *sums,
                                   int32_t *counts, int32_t *offsets, double *objective,
                                   void *ws, size_t ws_bytes, fk_stream_t stream);

/* Combine W shards gathered side by side (device arrays): sums [W][K][d] fp64, counts_w
 * [W][K] int64, objectives_w [W] fp64 (may be NULL with objective NULL).  In shard order,
 * in fp64: C_new[k] = (sum_w sums[w][k]) / (sum_w counts_w[w][k]) rounded once to fp32, or
 * C_old[k] bit for bit when every count is 0; counts[k] (int64, optional) = sum_w counts;
 * *objective (optional) = sum_w objectives_w[w].  The order is fixed, so every rank that
 * runs it on the same gathered data gets the same bits. */
FK_API fk_status fk_finalize_shards(const double *sums, const int64_t *counts_w,
                                    const double *objectives_w, int W, int K, int d,
                                    const float *C_old, float *C_new, int64_t *counts,
                                    double *objective, fk_stream_t stream);

/* Lloyd's iterations over points held in HOST memory (the out-of-core mode of the
 * Flash-KMeans article: the data set can exceed the GPU's memory).  Each iteration streams
 * X from the host in chunks of chunk_rows rows: while one chunk is assigned and reduced on
 * `stream`, the next is copied in on a second stream (double buffering).  Every chunk's
 * fp64 per-cluster sums, counts and objective share are added to the iteration's totals in
 * chunk order, then the centroids are formed once (an empty cluster keeps its centroid).
 * The result is deterministic; it equals fk_lloyd's up to the order of the fp64 sums.
 *   X_host        : N x d points (fp32 or bf16), host memory; page-locked (pinned) memory
 *                   lets the copies overlap the compute
 *   C             : K x d fp32, device: initial centroids in, final centroids out
 *   labels_host   : optional N int32, host: labels of the last iteration
 *   objective_host: optional niter doubles, host: objective of every iteration
 *   chunk_rows    : rows per chunk (>= K; clamped to N); the workspace holds two chunks
 * Same metric semantics as fk_lloyd (cosine: each chunk and the initial C normalised).
 * niter <= 4096.  Synchronous: returns after the last copy has landed. */
FK_API fk_status fk_lloyd_streamed(const void *X_host, fk_dtype dtype, int64_t N, int d,
                                   int K, fk_metric metric, int niter, float *C,
                                   int32_t *labels_host, double *objective_host,
                                   int64_t chunk_rows, void *ws, size_t ws_bytes,
                                   fk_stream_t stream);

/* Workspace bytes of fk_lloyd_streamed for this chunk size (the per-chunk workspace of
 * fk_assign / fk_update, two chunk buffers, and K x d fp64 sums twice). */
FK_API fk_status fk_streamed_workspace_size(int64_t chunk_rows, int d, int K, fk_dtype dtype,
                                            fk_metric metric, size_t *bytes);

/* Inverted lists of a clustering (LEANN FlashLib guide, "工作原理": an IVF index keeps,
 * per cell, the ids of its points in CSR form and the points of a cell contiguous).
 *   offsets[k] .. offsets[k+1] - 1 : the positions of cell k (offsets: K+1 int32)
 *   row_ids[p] : the point at position p, stable order by (label, index) (N int32)
 *   X_lists[p] : X[row_ids[p]], same dtype and row length as X (N x d; optional, NULL to
 *                skip the gather)
 * X (fp32 or bf16, N x d, 16-byte aligned rows as for fk_update) and labels (values in
 * [0, K)) are device pointers; so are the outputs, which must not overlap X.  Workspace
 * as for fk_update.  Asynchronous; a label outside [0, K) is reported by
 * fk_get_device_error. */
FK_API fk_status fk_ivf_lists(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                              const int32_t *labels, int32_t *offsets, int32_t *row_ids,
                              void *X_lists, void *ws, size_t ws_bytes, fk_stream_t stream);

/* Squared norms in fp64 for IVF-Flat search: norms[i] = sum_j V[i][j]^2 of the fp32 rows
 * (each square exact in fp64, summed in fp64).  V: n x d fp32, device, 16-byte aligned,
 * d % 4 == 0.  norms: n doubles, device.  Asynchronous on `stream`.  For fk_ivf_search
 * this is computed once per index over X_lists, in list order. */
FK_API fk_status fk_ivf_norms(const float *V, int64_t n, int d, double *norms,
                              fk_stream_t stream);

/* Cell radii for IVF-Flat search: radius[c] >= max over the points x of cell c of
 * ||x - C[c]|| (fp64 distances, rounded up to fp32 with a relative margin), 0 for an empty
 * cell.  C nlist x d fp32, X_lists N x d fp32 in cell order, offsets nlist + 1 int32
 * (fk_ivf_lists), radius nlist floats; all device; d % 4 == 0, C and X_lists 16-byte
 * aligned.  Computed once per index; fk_ivf_search uses it to skip, in its screened fine
 * pass, the points that cannot be among a query's k nearest. */
FK_API fk_status fk_ivf_radii(const float *C, int nlist, const float *X_lists,
                              const int32_t *offsets, int d, float *radius, fk_stream_t stream);

/* Workspace bytes of fk_ivf_search for these sizes. */
FK_API fk_status fk_ivf_search_workspace_size(int64_t nq, int d, int nlist, int64_t N,
                                              int nprobe, int k, size_t *bytes);

/* IVF-Flat search (LEANN FlashLib guide: "什么是 FlashLib 后端" -- k nearest neighbours of
 * a batch of queries; "工作原理" -- cells are the coarse k-means clusters, cell-contiguous
 * with row ids and CSR offsets; "nlist 与 nprobe 的推导规则" -- nprobe cells probed per
 * query; "距离度量只有 squared L2" -- squared L2, with cosine / inner product served by
 * L2-normalising both sides first, which the caller does with fk_normalize_rows).
 *
 * For each query q (row of Q):
 *   probes[q][0..nprobe)  the nprobe cells whose centroids are nearest to q, ascending by
 *                         (distance, cell);
 *   ids[q][0..k)          the k points of those cells nearest to q, ascending by
 *                         (distance, original index), as original indices (row_ids);
 *   distances[q][0..k)    their squared L2 distances (fp32 rounding of an fp64 value,
 *                         clamped at 0); slots beyond the number of candidates hold id -1
 *                         and distance +inf.
 * Distances are evaluated in fp64 as ||q||^2 + ||x||^2 - 2 q.x; the selections agree with
 * an exact fp64 evaluation except between candidates whose fp64 distances differ by the
 * rounding of that expression (about 1e-16 of the squared norms).
 * Coarse pass: by default (flags 0, nlist <= 8192) the query-centroid products run on the
 * tensor cores with one bf16 product per term; every centroid within a proven error window
 * of the nprobe-th screened value is then re-ranked in fp64 (difference form), so the
 * probes are those of the fp64 evaluation.  FK_SEARCH_FP64_COARSE computes every coarse
 * distance in fp64 instead (same probes, more work).
 * Fine pass: with X_planes given (fk_split_points of X_lists), k <= 16 and nprobe <= 256,
 * each (query, point) product is screened on the tensor cores (three bf16 products, fp32
 * accumulation); per query, the points within a proven window of the k-th screened
 * distance are re-ranked in fp64 (difference form), and a query whose per-cell candidate
 * lists may have dropped one is recomputed exactly over its probed cells.  Otherwise, or
 * with FK_SEARCH_FP64_FINE, every fine distance is fp64.
 *
 * Inputs (device pointers, read only): Q nq x d fp32; C nlist x d fp32 centroids; X_lists
 * N x d fp32, the points in cell order (fk_ivf_lists); X_norms N doubles, fk_ivf_norms of
 * X_lists; X_planes NULL or the 4 N d_p + 4 N bytes that fk_split_points writes for
 * X_lists (16-byte aligned); cell_radius NULL or fk_ivf_radii of (C, X_lists) (with the
 * screened fine pass, each query then skips the points farther than a bound on its k-th
 * nearest that the nearest probed cells give); offsets nlist + 1 int32 (offsets[0] = 0, offsets[nlist] = N,
 * non-decreasing);
 * row_ids N int32 (fk_ivf_lists).  Outputs (device): distances nq x k fp32, ids nq x k
 * int32, probes nq x nprobe int32 or NULL (then kept in the workspace).
 * Requirements: d % 4 == 0; Q, C, X_lists 16-byte aligned; 1 <= nprobe <= min(nlist,
 * 1024); 1 <= k <= 32; nq * nprobe < 2^31; N < 2^31; finite inputs.  Violations return
 * FK_ERR_INVALID_ARG (sizes, null pointers) or FK_ERR_UNSUPPORTED (alignment, d % 4).
 * Asynchronous on `stream`; the workspace (fk_ivf_search_workspace_size, 256-byte aligned)
 * must stay untouched until the call's work on the stream is done.  `timing` (host, may be
 * NULL): when given, CUDA events on `stream` time each phase and the call synchronises the
 * stream before it returns, to fill it in. */
typedef struct fk_search_timing {
    double ms_coarse; /* query and centroid norms, coarse distances, probe selection */
    double ms_sort;   /* (query, probe) pairs sorted by cell, work items */
    double ms_fine;   /* the fine distance kernel (per-pair candidate lists) */
    double ms_merge;  /* the per-query selection (and exact re-ranking) of the k nearest */
    int screened_coarse; /* 1 when the coarse pass ran on the tensor cores (see flags) */
    int screened_fine;   /* 1 when the fine pass ran on the tensor cores (see flags)   */
    int fallback_queries; /* screened fine pass: queries recomputed exactly over their
                             probed cells (their candidate lists may have dropped a point) */
} fk_search_timing;

/* fk_ivf_search flags. */
#define FK_SEARCH_FP64_COARSE 1 /* every coarse distance in fp64 (no tensor-core screening) */
#define FK_SEARCH_FP64_FINE 2   /* every fine distance in fp64 (no tensor-core screening)   */

FK_API fk_status fk_ivf_search(const float *Q, int64_t nq, int d, const float *C, int nlist,
                               const float *X_lists, const double *X_norms,
                               const void *X_planes, const float *cell_radius,
                               const int32_t *offsets,
                               const int32_t *row_ids, int64_t N, int nprobe, int k,
                               int flags, float *distances, int32_t *ids,
                               int32_t *probes, void *ws, size_t ws_bytes,
                               fk_search_timing *timing, fk_stream_t stream);

/* Scratch held by fk_assign_noalloc: one static device array of this many bytes. */
#define FK_NOALLOC_SCRATCH_BYTES (8u << 20)

/* fk_assign without a workspace, for callers that cannot allocate device memory: code
 * that runs under another framework's memory manager (which owns all device memory and
 * does not allow cudaMalloc behind its back), or on a latency-critical path where
 * cudaMalloc / cudaFree would implicitly synchronise the device.  The paper has no
 * counterpart; it is an interface variant of the assignment step above, with the same
 * labels (bit for bit) as fk_assign on the same inputs, since both run the same kernel.
 *   - Scratch (error words, centroid operand planes and norms, and for FK_F32 -- or
 *     FK_BF16 with d % 64 != 0 -- the bf16 planes of X) lives in one file-scope device
 *     array of FK_NOALLOC_SCRATCH_BYTES (8 MiB) inside libfk; every GPU that loads the
 *     library holds it until the process exits.  The call allocates and frees nothing.
 *   - A problem whose scratch does not fit returns FK_ERR_WORKSPACE before any launch
 *     (roughly: FK_F32 needs 4*N*roundup(d,64) + 4*roundup(K,256)*roundup(d,64) bytes,
 *     FK_BF16 with d % 64 == 0 needs 2*roundup(K,256)*d bytes, plus a few KB).
 *   - fp32 problems that fk_assign would send to its screened route (every
 *     roundup(d,64) > 768, and large-N shapes that never fit the array anyway) return
 *     FK_ERR_UNSUPPORTED: that route needs buffers the array does not hold.
 *   - Each call looks up the array's address on the current device
 *     (cudaGetSymbolAddress) and checks the result; nothing about the device is cached.
 *   - Every call shares the one array and it keeps the previous call's contents (the
 *     call clears its error words itself).  Calls whose kernels overlap on the GPU (two
 *     host threads, two streams) race on it: serialise them.
 *   - No mind output.  The call is synchronous: it reads the error words back with a
 *     device-to-host copy and waits for `stream`, so it cannot be called while `stream`
 *     is being captured into a CUDA graph.  It returns FK_ERR_TIMEOUT if a bounded wait
 *     inside the kernel expired and FK_ERR_DEVICE if the kernel met a bad value. */
FK_API fk_status fk_assign_noalloc(const void *X, fk_dtype dtype, int64_t N, int d,
                                   const float *C, int K, int32_t *labels,
                                   fk_stream_t stream);

/* Diagnostics for the failure path, without any fault: launches a one-warp kernel that
 * waits (bounded by limit_ns, at most 10 s) on an mbarrier nothing ever arrives on; the
 * wait expires and the kernel records FK_ERR_TIMEOUT in the workspace error word, which
 * fk_get_device_error then returns.  Asynchronous on `stream`. */
FK_API fk_status fk_selftest_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns,
                              fk_stream_t stream);

/* Synchronise `stream`, then read and clear the workspace's device error word.
 * *code (host int) receives FK_OK, FK_ERR_TIMEOUT or FK_ERR_DEVICE; the return value
 * is FK_OK unless reading failed. */
FK_API fk_status fk_get_device_error(void *ws, size_t ws_bytes, int *code, fk_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FK_H */
