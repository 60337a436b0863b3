// fk_common.cuh -- constants, workspace layout and small helpers shared by the kernels
// and the C-ABI host code of libfk.
#pragma once

#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "../../include/fk.h"

namespace fk {

// ----------------------------------------------------------------- assign tiling
constexpr int kBM = 128;  // rows of X per tile (one TMEM lane per row)
constexpr int kBN = 256;  // centroids per tile (fp32 accumulator columns)
constexpr int kBK = 64;   // bf16 elements per 128-byte swizzle row
constexpr int kAug = 16;  // bf16 columns of the norm-folding K step (32-byte rows)

// ----------------------------------------------------------------- sort tiling
constexpr int kSortThreads = 256;
constexpr int kSortItems = 8;       // keys per thread of a large-input tile
constexpr int kSortItemsSmall = 4;  // keys per thread when the input is small
constexpr int kSortTile = kSortThreads * kSortItems;  // keys per block (the largest tile)
// Inputs up to this size use the small tile: twice the blocks, each with half the serial
// work, which is what bounds a sort whose tiles all fit on the GPU at once.
constexpr int64_t kSortSmallN = int64_t(1) << 22;
// digit width bound: 256 bins (a tile's per-digit bookkeeping grows with the bins, so two
// narrow passes beat one wide one from about 1024 bins)
constexpr int kSortMaxBits = 8;
// Words of the 256-byte error block at the start of a workspace that a call clears: [0] a
// bounded wait expired, [1] a label out of range ([4..5]: the last iteration's statistics).
constexpr int kErrWords = 2;

// ----------------------------------------------------------------- update tiling
constexpr int kUpdWarps = 8;          // warps per block of the update kernels
constexpr int kUpdGroup = 16;         // units of one combine level per unit of the next
constexpr int kUpdMinRows = 64;       // smallest chunk of sorted positions per warp
constexpr int kUpdMaxRows = 256;      // largest chunk
constexpr int64_t kUpdTargetWarps = 148 * 64;  // enough warps to cover the GPU twice
// Level-1 units up to which every combine level runs in one launch (wide_combine_kernel),
// for at most kUpdWideMaxK clusters: its blocks walk their clusters one after another, so
// beyond a few clusters per block the level-by-level launches (a warp per cluster in the
// tail) are faster
constexpr int64_t kUpdWideUnits = 2048;
constexpr int kUpdWideMaxK = 4096;

// ----------------------------------------------------------------- screening (fp32)
// The single-product pass writes, per row, up to kCandPerRow candidate columns (unused
// slots -1; a row whose list ran out of room has kCandOverflow in its first slot and goes
// to the three-product pass).
constexpr int kCandPerRow = 16;
constexpr int kScreenSlots = kCandPerRow;  // candidate columns the screening pass keeps
constexpr int32_t kCandOverflow = -2;
// Screened values at or above this are never candidates: padding centroids (whose first
// norm piece is the largest finite bf16, about 3.39e38) lie above it, and real data whose
// ||c||^2 + 2|x.c| reaches it is outside the supported range.
constexpr float kScreenMax = 1e38f;
// Screening pays where the tensor-core work per row is large next to its fixed per-row
// costs (candidate list, re-ranking): from d = 256 on, and below that from K * d = 2^22
// (measured on B200: d = 128 wins from K = 32768, loses at K <= 8192; d = 192, K = 4096
// breaks even).
constexpr int kScreenMinD = 256;
constexpr int64_t kScreenMinKD = int64_t(1) << 22;
// fk_lloyd screens a call only if, on a sample of kScreenProbeRows rows with the initial
// centroids, at most 1/kScreenMaxFallback of them would need the three-product pass
// (mixtures whose heavy components hold many nearly equidistant centroids do not qualify).
constexpr int kScreenMaxFallback = 4;
constexpr int64_t kScreenProbeRows = 2 * 128 * 148;
// The three-product form (hi.hi + lo.hi + hi.lo in one fp32 accumulator) misses the exact
// x.c by the dropped lo.lo and residual terms plus its fp32 accumulation.  Emulated under
// every modelled accumulation order (one rounding per MMA step or per product, to nearest
// or toward zero), that error stays within half the parity rule's tie window up to a
// padded depth of 768; beyond it, rounding toward zero after every product reaches 1.55
// half windows at 1024.  So from d_p > 768 on no label of fp32 points is decided by the
// three-product form: every call takes the screened route (any N, whatever the probe
// says), and rows whose candidates overflow get an exact fp64 scan over all centroids.
constexpr int kThreeProductMaxDp = 768;

// Width of the screening window for one row: twice a bound E on |v~ - v|, where
// v = ||c||^2 - 2 x.c is exact and v~ is what the single-product pass accumulates from
// bf16 x~ = RN(x) and c~ = RN(c) (each within a relative 2^-8 of its value; u = 2^-8):
//   operand rounding   |sum x~c~ - sum xc| <= (2u + u^2) sum |x_j||c_j| <= (2u + u^2)|x||c|,
//                      doubled by the factor -2;
//   accumulation       each of the dp/16 + 1 MMA steps adds 16 exact products to the fp32
//                      accumulator; assume up to 17 units of 2^-23 of the largest partial
//                      value, which is at most ||c||^2 + 2|x||c| (with margin);
//   norm               ||c||^2 rounded once to fp32 (2^-24 relative).
// If k* is the true argmin, v~(k*) <= v(k*) + E <= v(k) + E <= v~(k) + 2E for every k, so
// k* lies within 2E of the screened minimum.  Likewise, if T~ is the m-th smallest
// screened value, the m columns with the smallest screened values have v <= T~ + E, so
// the m-th smallest exact value is at most T~ + E and every column among the m exact
// smallest has v~ <= T~ + 2E.  ||c|| is bounded by cmax = max_k ||c_k||.
// The result carries a 1% margin for the rounding of this expression itself.
__host__ __device__ __forceinline__ float screen_window(float xnorm2, float cmax2, int dp) {
    const float xn = sqrtf(xnorm2), cm = sqrtf(cmax2);
    const float u = 0.00390625f;
    const float prod = 2.f * (2.f * u + u * u) * xn * cm;
    const float accum = static_cast<float>(dp / 16 + 1) * 17.f * 1.1920929e-7f *
                        (cmax2 + 2.f * xn * cm) * 1.01f;
    const float norm = 5.9604645e-8f * cmax2;
    return 2.f * (prod + accum + norm) * 1.01f;
}

// Window coefficients of the IVF-Flat search's screened fine pass for rows padded to dp:
// |s~ - s| <= ce_dot ||q|| ||x|| + ce_round (||q||^2 + ||x||^2), where s = ||q - x||^2 and s~
// = ||q||^2 + ||x||^2 - 2 q.x~ rounded to fp32, with q.x~ the three bf16 products
// hi.hi + hi.lo + lo.hi of the RN-bf16 splits v = hi + lo (+ a residual below 2^-16 |v|)
// accumulated in fp32.  With u = 2^-8 (bf16 rounding), the three products miss at most
// 3.1 u^2 sum |q_j||x_j| <= 3.1 u^2 |q||x|; the 3 dp / 16 mma steps add at most 17 units of
// 2^-23 of a partial sum bounded by 1.02 |q||x| each; the factor 2 of -2 q.x; the fp32
// rounding of s~ at most 2^-23 (||q||^2 + ||x||^2); a 1% margin on both.
inline void fine_window_coeffs(int dp, float *ce_dot, float *ce_round) {
    const double u = 1.0 / 256.0;
    const double e_dot = 3.1 * u * u + 3.0 * (dp / 16) * 17.0 * std::ldexp(1.0, -23) * 1.02;
    *ce_dot = static_cast<float>(2.0 * e_dot * 1.01);
    *ce_round = static_cast<float>(std::ldexp(1.0, -23) * 1.01);
}

// Objective slots kept on the device by fk_lloyd before a copy to the host.
constexpr int kObjRing = 4096;

// Bound on every in-kernel wait of a library call (2 s).
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

// Device error word bits (workspace offset 0).
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrLabel = 2u;

// Programmatic dependent launch.  A kernel launched with launch_pdl may be scheduled while
// the kernel before it in the stream is finishing; it calls pdl_wait() first, which
// returns once that kernel has completed and its writes are visible, so the order of the
// stream is kept and only the launch latency overlaps.  pdl_trigger() lets the next such
// kernel be scheduled once every block of this one has started.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline int key_bits(int K) {
    if (K <= 1) return 0;
    unsigned v = static_cast<unsigned>(K - 1);
    int b = 0;
    while (v) {
        ++b;
        v >>= 1;
    }
    return b;
}

struct SortPlan {
    int nbits = 0;
    int passes = 0;
    int bits = 0;  // digit width per pass (last pass may use fewer significant bits)
    int items = kSortItems;  // keys per thread; a block's tile is kSortThreads * items keys
    int64_t nblocks = 0;
};

inline SortPlan sort_plan(int64_t N, int K) {
    SortPlan p;
    p.nbits = key_bits(K);
    p.passes = p.nbits == 0 ? 0 : static_cast<int>(ceil_div(p.nbits, kSortMaxBits));
    p.bits = p.passes == 0 ? 0 : static_cast<int>(ceil_div(p.nbits, p.passes));
    p.items = N <= kSortSmallN ? kSortItemsSmall : kSortItems;
    p.nblocks = ceil_div(N, static_cast<int64_t>(kSortThreads) * p.items);
    return p;
}

// Level-1 work split of the update: a warp owns `rows` consecutive sorted positions and one
// 128-column block of the rows (grid.y = column blocks), so a 3 KB row (d = 768) is read
// by six warps as six contiguous 512-byte pieces.  `rows` is a power of two chosen so the
// grid has enough warps to hide memory latency even for small N.
struct UpdPlan {
    int ncolblk = 1;   // 128-column blocks
    int dcov = 128;    // padded row length of a piece (ncolblk * 128)
    int rows = kUpdMaxRows;
    int64_t nwarps = 0;  // warps per column block
};

inline UpdPlan upd_plan(int64_t N, int d) {
    UpdPlan p;
    p.ncolblk = static_cast<int>(ceil_div(d, 128));
    p.dcov = p.ncolblk * 128;
    int64_t r = N * p.ncolblk / kUpdTargetWarps;
    int rows = kUpdMinRows;
    while (rows < kUpdMaxRows && rows * 2 <= r) rows *= 2;
    p.rows = rows;
    p.nwarps = ceil_div(N, rows);
    return p;
}

// The one-launch combine (at most kUpdWideUnits level-1 units): the shared-memory entries
// (128 doubles each) of its two level buffers.  A cluster's units are consecutive, so its
// level-2 partials span at most (units - 1) / kUpdGroup + 1 groups; its level-3 partials at
// most that / kUpdGroup + 1, and the buffers alternate from there on.
inline int upd_wide_l2cap(int64_t units) { return static_cast<int>((units - 1) / kUpdGroup + 1); }
inline int upd_wide_l3cap(int64_t units) { return upd_wide_l2cap(units) / kUpdGroup + 2; }
inline size_t upd_wide_smem(int64_t units) {
    return size_t(upd_wide_l2cap(units) + upd_wide_l3cap(units)) * 128 * sizeof(double);
}

// Byte offsets of every scratch buffer inside the caller's workspace (256-byte aligned).
struct WsLayout {
    size_t err = 0, obj = 0, xn = 0, xs = 0, xnorm = 0, cs = 0, cn = 0, cused = 0,
           calt = 0, keys0 = 0, keys1 = 0, vals0 = 0, vals1 = 0, hist = 0, dtot = 0,
           caug = 0, pieces = 0, pkeys = 0, piecesb = 0, pkeysb = 0, jpart = 0, jdev = 0, cnt = 0,
           off = 0, cand = 0, nfb = 0, fbrows = 0, fblab = 0, xsfb = 0, cmax2 = 0,
           total = 0;
    int64_t dp = 0, Kp = 0;
    int xplanes = 0;  // bf16 planes of X prepared in the workspace (0, 1 or 2)
    int cplanes = 0;  // bf16 planes of the centroids (1 or 2)
    SortPlan sp;
    UpdPlan up;
};

inline WsLayout ws_layout(int64_t N, int d, int K, fk_dtype dtype, fk_metric metric) {
    WsLayout L;
    L.dp = round_up(d, kBK);
    L.Kp = round_up(K, kBN);
    L.cplanes = dtype == FK_BF16 ? 1 : 2;
    L.xplanes = dtype == FK_F32 ? 2 : ((dtype == FK_BF16 && (d % kBK) != 0) ? 1 : 0);
    L.sp = sort_plan(N, K);
    L.up = upd_plan(N, d);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += static_cast<size_t>(round_up(static_cast<int64_t>(bytes > 0 ? bytes : 1), 256));
        return at;
    };
    L.err = take(256);
    L.obj = take(sizeof(double) * kObjRing);
    L.xn = take(metric == FK_COSINE ? sizeof(float) * N * d : 0);
    L.xs = take(sizeof(uint16_t) * L.xplanes * N * L.dp);
    L.xnorm = take(sizeof(float) * N);
    L.cs = take(sizeof(uint16_t) * L.cplanes * L.Kp * L.dp);
    L.cn = take(sizeof(float) * L.Kp);
    L.caug = take(sizeof(uint16_t) * L.Kp * kAug);
    L.cused = take(sizeof(float) * K * d);
    L.calt = take(sizeof(float) * K * d);
    L.keys0 = take(sizeof(int32_t) * N);
    L.keys1 = take(sizeof(int32_t) * N);
    L.vals0 = take(sizeof(int32_t) * N);
    L.vals1 = take(sizeof(int32_t) * N);
    const int64_t bins = int64_t(1) << (L.sp.bits > 0 ? L.sp.bits : 1);
    L.hist = take(sizeof(uint32_t) * bins * L.sp.nblocks);
    L.dtot = take(sizeof(uint32_t) * bins);
    L.pieces = take(sizeof(double) * L.up.nwarps * 2 * L.up.dcov);
    L.pkeys = take(sizeof(int32_t) * L.up.nwarps * 2);
    const int64_t units2 = ceil_div(L.up.nwarps, kUpdGroup) + 1;
    L.piecesb = take(sizeof(double) * units2 * 2 * L.up.dcov);
    L.pkeysb = take(sizeof(int32_t) * units2 * 2);
    L.jpart = take(sizeof(double) * L.up.nwarps * L.up.ncolblk);
    L.jdev = take(sizeof(double) * 2);
    L.cnt = take(sizeof(int32_t) * K);
    L.off = take(sizeof(int32_t) * (K + 1));
    // screened assignment of fp32 points (single bf16 product, exact re-ranking, and the
    // three-product pass for rows whose candidates did not fit)
    const bool screen = dtype == FK_F32 || dtype == FK_BF16X2;
    L.cand = take(screen ? sizeof(int32_t) * kCandPerRow * N : 0);
    L.nfb = take(screen ? 256 : 0);
    L.fbrows = take(screen ? sizeof(int32_t) * N : 0);
    L.fblab = take(screen ? sizeof(int32_t) * N : 0);
    L.xsfb = take(screen ? sizeof(uint16_t) * 2 * N * L.dp : 0);
    L.cmax2 = take(screen ? 256 : 0);
    L.total = o;
    return L;
}

template <typename T>
inline T *ws_ptr(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

// ----------------------------------------------------------------- launch helpers
// (declared here, defined in the .cu files)
struct AssignArgs {
    const void *a_planes;  // bf16 X planes: [xplanes][N][lda]
    int a_nplanes;         // 2 = hi/lo (fp32 emulation), 1 = bf16
    int64_t lda;           // row stride of an X plane, elements
    const void *b_planes;  // bf16 centroid planes [cplanes][Kp][dp], scaled by -2
    const float *cn;       // [Kp], +inf beyond K
    const void *caug;      // [Kp][16] bf16: ||c||^2 as hi + mid + lo, then zeros
    int64_t N;
    int d, dp, K, Kp;
    int32_t *labels;
    float *best;           // optional [N]: min_k (cn_k - 2 x.c_k)
    const float *xnorm;    // optional [N]: ||x||^2, with mind
    float *mind;           // optional [N]
    uint32_t *err;         // workspace error words
    uint64_t wait_ns;      // bound on every mbarrier wait inside the kernel
    const uint32_t *n_dev; // optional: row count read on the device (N bounds the maps)
    int32_t *cand;         // screening pass: [N][kCandPerRow] candidates instead of labels
    const float *cmax2;    // screening pass: device max_k ||c_k||^2
    float *dump;           // single-product pass that writes every screened value instead:
                           // dump[row * ldd + col] = ||c||^2 - 2 x~.c~ for col < Kp
    int64_t ldd;
};

cudaError_t launch_split_x(const float *X, int64_t N, int d, int64_t dp, uint16_t *hi,
                           uint16_t *lo, float *xnorm, cudaStream_t st);
cudaError_t launch_pad_bf16(const uint16_t *X, int64_t N, int d, int64_t dp, uint16_t *out,
                            cudaStream_t st);
cudaError_t launch_normalize(const float *X, float *Y, int64_t N, int d, cudaStream_t st);
cudaError_t launch_xnorm_bf16(const uint16_t *X, int64_t N, int d, float *xnorm,
                              cudaStream_t st);
cudaError_t launch_prep_centroids(const float *C, int K, int d, int64_t Kp, int64_t dp,
                                  fk_dtype dtype, uint16_t *planes, float *cn, float *cused,
                                  uint16_t *caug, cudaStream_t st);
cudaError_t launch_centroid_norms(const float *C, int K, int d, fk_dtype dtype, float *cn,
                                  cudaStream_t st);
cudaError_t launch_assign(const AssignArgs &a, cudaStream_t st);
bool assign_can_screen(int64_t N, int dp, int Kp);
// The single-product pass with every screened value written out (AssignArgs::dump) can run
// for this shape (any number of rows).
bool assign_can_dump(int dp, int Kp);

// Screened fp32 assignment (screen.cu): the single-product pass over plane 0 of `a`'s X
// planes, exact re-ranking of the candidates, and the three-product pass over the rows
// whose candidates did not fit.  `a` describes the two-plane (hi, lo) problem; X32 is the
// fp32 points (or null: re-rank from hi + lo).
struct ScreenBufs {
    int32_t *cand;     // [N][kCandPerRow]
    uint32_t *nfb;     // [1] rows sent to the three-product pass
    int32_t *fbrows;   // [N]
    int32_t *fblab;    // [N]
    uint16_t *xsfb;    // [2][N][dp]
    float *cmax2;      // [1]
};
// The screening pass and re-ranking over the first n_probe rows, counting in sb.nfb the
// rows that would need the three-product pass (their labels are not final).
cudaError_t launch_screen_probe(const AssignArgs &a, int64_t n_probe, const float *X32,
                                const float *C, const ScreenBufs &sb, cudaStream_t st);
cudaError_t launch_assign_screened(const AssignArgs &a, const float *X32, const float *C,
                                   const ScreenBufs &sb, cudaStream_t st,
                                   cudaEvent_t ev_mma0 = nullptr,
                                   cudaEvent_t ev_mma1 = nullptr);
cudaError_t launch_sort_csr(const int32_t *labels, int64_t N, int K, const SortPlan &sp,
                            int32_t *keys0, int32_t *keys1, int32_t *vals0, int32_t *vals1,
                            int32_t *perm_out, uint32_t *hist, uint32_t *dtot,
                            int32_t *offsets, const int32_t **sorted_keys,
                            const int32_t **perm, uint32_t *err, cudaStream_t st);
// The assign operands of the centroids (prep_centroids_kernel's outputs): planes
// [cplanes][Kp][dp] bf16, norms cn[Kp], cused[K][d] (bf16 points only) and the norm pieces
// caug[Kp][kAug].
struct CentroidOperands {
    uint16_t *planes;
    float *cn;
    float *cused;
    uint16_t *caug;
    int64_t Kp, dp;
    int two_planes;
};
// next (may be null): where a small problem's update (one column block, the one-launch
// combine) may also prepare the new centroids' operands as it finishes them; *prepped
// tells whether it did, so the next iteration can skip prep_centroids.
cudaError_t launch_update(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                          const UpdPlan &up, const int32_t *skeys, const int32_t *perm,
                          const int32_t *offsets, const float *C_old, const float *C_used,
                          float *C_new, int32_t *counts, double *pieces_a, int32_t *pkeys_a,
                          double *pieces_b, int32_t *pkeys_b, double *jpart,
                          double *objective, uint32_t *err, double *sums_out,
                          cudaStream_t st, const CentroidOperands *next = nullptr,
                          bool *prepped = nullptr);
cudaError_t launch_gather_rows(const void *X, int64_t N, int64_t row_bytes,
                               const int32_t *row_ids, void *out, cudaStream_t st);
cudaError_t launch_accumulate_chunk(double *tot, const double *part, int64_t KD,
                                    int64_t *cnt_tot, const int32_t *cnt, int K,
                                    double *obj_tot, const double *obj, cudaStream_t st);
cudaError_t launch_finalize_shards(const double *sums, const int64_t *cnts, const double *objs,
                                   int W, int K, int d, const float *C_old, float *C_new,
                                   int64_t *counts, double *objective, cudaStream_t st);

// IVF-Flat search (ivf_search.cu).
cudaError_t launch_sqnorm_f64(const float *V, int64_t n, int d, double *out, cudaStream_t st);
cudaError_t launch_ivf_coarse(const float *Q, const double *qn, int64_t q0, int nqb, int d,
                              const float *C, const double *cn, int nlist, double *D,
                              cudaStream_t st);
cudaError_t launch_ivf_select(const double *D, const uint32_t *I, int64_t ld, int64_t rows, int L,
                              int m, int32_t *out_id, float *out_dist, int64_t ldo,
                              cudaStream_t st);
cudaError_t launch_ivf_items(const int32_t *pair_off, int nlist, int2 *items, int *nitems,
                             int *ctr, cudaStream_t st);
// The screened coarse pass: the assignment kernel's single-product pass writes every
// screened value (AssignArgs::dump), then the candidates within the window above the
// nprobe-th are re-ranked in fp64 (ivf_search.cu).
bool ivf_coarse_can_screen(int nlist, int dp, int Kp);
cudaError_t launch_ivf_cmax(const float *cn, int K, float *out, cudaStream_t st);
cudaError_t launch_ivf_coarse_rerank(const float *Vs, int64_t ldv, int64_t rows, int L, int m,
                                     const float *Q, int64_t q0, const float *C, int d, int dp,
                                     const float *xnorm, const float *cmax2, int32_t *probes,
                                     cudaStream_t st);
cudaError_t launch_ivf_fine(const float *Q, const double *qn, int d, const float *X_lists,
                            const double *xn, const int32_t *offsets, const int32_t *row_ids,
                            const int32_t *pair_sorted, const int32_t *pair_off,
                            const int2 *items, const int *nitems, int *item_ctr, int64_t max_items,
                            int nprobe, int k, double *Ld, uint32_t *Li, cudaStream_t st);

// The screened fine pass (ivf_search.cu): bf16 three-product screening per (query, point),
// per-pair lists of the 32 smallest screened distances, a per-query merge that re-ranks the
// window in fp64, and an exact fallback for the queries whose lists may have dropped a
// point of their top-k.
cudaError_t launch_ivf_fine_scr(const uint16_t *Qp, int64_t nq, const uint16_t *Xp, int64_t N,
                                int dp, const double *qn, const double *xn,
                                const int32_t *offsets, const int32_t *pair_sorted,
                                const int32_t *pair_off, const int2 *items, const int *nitems,
                                int *item_ctr, int64_t max_items, int nprobe, float *Sv,
                                uint32_t *Sp, float *Slost, const float *cut, cudaStream_t st);
cudaError_t launch_ivf_query_rerank(const float *Sv, const uint32_t *Sp, const float *Slost,
                                    int64_t nq, int nprobe, int k, const float *Q,
                                    const float *X, int d, int dp, const double *qn,
                                    const float *xmax2, const int32_t *row_ids,
                                    float *out_dist, int32_t *out_id, int32_t *fallback,
                                    const float *cut, cudaStream_t st);
cudaError_t launch_ivf_fallback(const int32_t *fallback, const int32_t *probes, int64_t nq,
                                int nprobe, int k, const float *Q, const float *X, int d,
                                const int32_t *offsets, const int32_t *row_ids, float *out_dist,
                                int32_t *out_id, cudaStream_t st);
cudaError_t launch_max_norm(const double *xn, int64_t n, float *out, cudaStream_t st);
cudaError_t launch_count_flags(const int32_t *f, int64_t n, int *out, cudaStream_t st);
// Cell radii of an index, and per query a cut on the fine pass's screened distances.
cudaError_t launch_cell_radius(const float *C, int nlist, const float *X, const int32_t *offsets,
                               int d, float *radius, cudaStream_t st);
cudaError_t launch_query_cut(const float *Q, const float *C, const int32_t *probes,
                             const int32_t *offsets, const float *radius, const double *qn,
                             const float *xmax2, int dp, int64_t nq, int nprobe, int k, int d,
                             float *cut, cudaStream_t st);

// Limits of fk_ivf_search: k is held one rank per lane, nprobe by the selection's sort.
constexpr int kSearchMaxK = 32;
constexpr int kSearchMaxProbe = 1024;
// The screened fine pass: k up to half a pair list (the rest is slack against dropping a
// point of the top-k), and a query's nprobe lists staged in shared memory at once.
constexpr int kSearchScrMaxK = 16;
constexpr int kSearchScrMaxProbe = 256;
constexpr int kSearchScrList = 32;
constexpr int kSearchPairsPerItem = 32;
// Rows of the coarse distance matrix held at once: a query batch of at most this many bytes.
constexpr int64_t kSearchCoarseBytes = int64_t(512) << 20;

struct SearchLayout {
    size_t err = 0, qn = 0, cn = 0, D = 0, probes = 0, keys0 = 0, keys1 = 0, vals0 = 0,
           vals1 = 0, hist = 0, dtot = 0, psorted = 0, poff = 0, items = 0, nitems = 0,
           Ld = 0, Li = 0, qplanes = 0, qxn = 0, cplanes = 0, ccn = 0, cused = 0, caug = 0,
           cmax2 = 0, Sv = 0, Sp = 0, Slost = 0, fb = 0, ubound = 0, xmax2 = 0, total = 0;
    int64_t P = 0, qbatch = 0, max_items = 0, dp = 0, Kp = 0;
    SortPlan sp;
};

inline SearchLayout search_layout(int64_t nq, int d, int nlist, int nprobe, int k) {
    SearchLayout L;
    L.P = nq * nprobe;
    L.dp = round_up(d, kBK);
    L.Kp = round_up(nlist, kBN);
    int64_t qb = kSearchCoarseBytes / (static_cast<int64_t>(nlist) * 8);
    qb = qb / 32 * 32;
    if (qb < 32) qb = 32;
    L.qbatch = qb < nq ? qb : nq;
    L.sp = sort_plan(L.P, nlist);
    L.max_items = nlist + ceil_div(L.P, kSearchPairsPerItem);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += static_cast<size_t>(round_up(static_cast<int64_t>(bytes > 0 ? bytes : 1), 256));
        return at;
    };
    L.err = take(256);
    L.qn = take(sizeof(double) * nq);
    L.cn = take(sizeof(double) * nlist);
    // fp64 coarse distances, or the screened values (fp32, rows of Kp) of a batch
    const int64_t dbytes = sizeof(double) * L.qbatch * nlist;
    const int64_t sbytes = sizeof(float) * L.qbatch * L.Kp;
    L.D = take(static_cast<size_t>(dbytes > sbytes ? dbytes : sbytes));
    L.probes = take(sizeof(int32_t) * L.P);
    L.keys0 = take(sizeof(int32_t) * L.P);
    L.keys1 = take(sizeof(int32_t) * L.P);
    L.vals0 = take(sizeof(int32_t) * L.P);
    L.vals1 = take(sizeof(int32_t) * L.P);
    const int64_t bins = int64_t(1) << (L.sp.bits > 0 ? L.sp.bits : 1);
    L.hist = take(sizeof(uint32_t) * bins * L.sp.nblocks);
    L.dtot = take(sizeof(uint32_t) * bins);
    L.psorted = take(sizeof(int32_t) * L.P);
    L.poff = take(sizeof(int32_t) * (nlist + 1));
    L.items = take(sizeof(int32_t) * 2 * L.max_items);
    L.nitems = take(sizeof(int32_t) * 2);
    L.Ld = take(sizeof(double) * L.P * k);
    L.Li = take(sizeof(uint32_t) * L.P * k);
    // screened passes: bf16 planes of the queries and of the centroids
    L.qplanes = take(sizeof(uint16_t) * 2 * nq * L.dp);
    L.qxn = take(sizeof(float) * nq);
    L.cplanes = take(sizeof(uint16_t) * 2 * L.Kp * L.dp);
    L.ccn = take(sizeof(float) * L.Kp);
    L.cused = take(sizeof(float) * nlist * d);
    L.caug = take(sizeof(uint16_t) * L.Kp * kAug);
    L.cmax2 = take(256);
    // screened fine pass: per-pair lists, per-query fallback flags, the largest point norm
    const bool scr_fine = k <= kSearchScrMaxK && nprobe <= kSearchScrMaxProbe;
    L.Sv = take(scr_fine ? sizeof(float) * L.P * kSearchScrList : 0);
    L.Sp = take(scr_fine ? sizeof(uint32_t) * L.P * kSearchScrList : 0);
    L.Slost = take(scr_fine ? sizeof(float) * L.P : 0);
    L.fb = take(scr_fine ? sizeof(int32_t) * nq : 0);
    L.ubound = take(scr_fine ? sizeof(float) * nq : 0);
    L.xmax2 = take(256);
    L.total = o;
    return L;
}

// Empty clusters and the largest cluster of counts[K], written to out[0], out[1].
cudaError_t launch_cluster_stats(const int32_t *counts, int K, uint32_t *out, cudaStream_t st);

int device_sm_count();

// Argument and device checks shared by every entry point (fk_api.cu).
bool aligned(const void *p, size_t a);
// FK_OK on an sm_100 device, FK_ERR_UNSUPPORTED on any other, FK_ERR_CUDA if it cannot tell.
fk_status check_device();
// Shape, dtype and metric rules of the assign / update / Lloyd calls (FK_BF16X2 only
// where planes_ok).
fk_status validate_shape(int64_t N, int d, int K, fk_dtype dtype, fk_metric metric,
                         bool planes_ok = false);
// Host-side fault injection for tests of the error paths (environment variable FK_FAULT,
// read when the library is first used): "workspace" fails every workspace check, "launch"
// fails the computing calls as a failed launch would, before any device work.
enum Fault { kFaultNone = 0, kFaultWorkspace = 1, kFaultLaunch = 2 };
Fault injected_fault();
// Status of the two device error words (word 0: a bounded wait expired; word 1: a label
// outside [0, K) was met).
inline fk_status decode_err(const uint32_t (&e)[2]) {
    return e[0] ? FK_ERR_TIMEOUT : (e[1] ? FK_ERR_DEVICE : FK_OK);
}
// Whether fk_assign takes the screened route for two-plane (fp32) points of this shape
// when its buffers are at hand: always beyond kThreeProductMaxDp, otherwise where
// screening pays and the CTA-pair kernel has rows enough.
bool screened_route(int64_t N, int dp, int Kp, int K);

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current device.  The
// attribute belongs to the device, so each call site records the devices it has set it
// on, one bit per ordinal in `done` (ordinals from 64 up set it on every call).
template <typename Kernel>
cudaError_t smem_opt_in(Kernel kernel, int bytes, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? uint64_t(1) << dev : 0;
    if (bit != 0 && (done.load(std::memory_order_relaxed) & bit) != 0) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// A timing event at the current point of stream st.  Outside a capture, a plain record.
// Under stream capture the record goes on a side branch: this thread's side stream forks
// from st there and records the event as external (an event-record node of the graph; a
// plain record during a capture records nothing when the graph runs).  The kernels on st
// then keep their programmatic edges to one another, which an event node between them
// would break.  join_side_stream(st) joins the branch back before the capture ends.
cudaError_t record_event(cudaEvent_t e, cudaStream_t st);
cudaError_t join_side_stream(cudaStream_t st);

// Milliseconds between two recorded events; false (with the runtime's last-error state
// cleared, so a later launch check does not see it) when they cannot be timed.
inline bool elapsed_ms(cudaEvent_t a, cudaEvent_t b, float *ms) {
    if (cudaEventElapsedTime(ms, a, b) == cudaSuccess) return true;
    cudaGetLastError();
    return false;
}

// Kernels launched by this host thread since the last reset (fk_lloyd reports it).
extern thread_local long g_launches;
inline void note_launch(int n = 1) { g_launches += n; }

}  // namespace fk
