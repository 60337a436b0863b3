// screen.cu -- screened assignment of fp32 points.
//
// The Flash-KMeans article (section "FlashAssign：把距离矩阵按块切成流水线") computes the
// distances tile by tile and keeps only the running argmin.  For fp32 points the tensor
// cores need three bf16 products per term to reach fp32 accuracy.  This file makes most
// rows need only one:
//
//  1. Screening pass (assign_pair_kernel<1, *, true>): one bf16 product per term over the
//     hi plane of X.  For every row it keeps the columns whose screened value lies within
//     a proven error window of the screened minimum, so the exact argmin is always among
//     them (the bound is derived beside screen_window in assign_sm100.cu).
//  2. Exact re-ranking (rerank_kernel): each candidate's squared distance in the difference
//     form sum_j (x_j - c_j)^2, fp64, fixed reduction order; the smallest wins, the lowest
//     centroid index on equal values.
//  3. Rows whose candidates did not fit in their slots are gathered (fb_gather_kernel) and
//     assigned by the three-product pass, which reads their count on the device, and the
//     labels are scattered back (fb_scatter_kernel).  Beyond a padded depth of 768, where
//     the three-product form's error is not shown to stay inside half the tie window,
//     those rows get an exact fp64 scan over all centroids instead (exact_scan_kernel).
//
// Everything stays on the stream: no host synchronisation, no data-dependent launches.
#include <cuda_bf16.h>

#include "fk_common.cuh"

namespace fk {
namespace {

// max_k ||c_k||^2 over the real centroids, and a zeroed count of rows for the
// three-product pass.  One block.
__global__ void window_kernel(const float *__restrict__ cn, int K, float *__restrict__ cmax2,
                              uint32_t *__restrict__ nfb) {
    __shared__ float red[32];
    float m = 0.f;
    for (int k = threadIdx.x; k < K; k += blockDim.x) m = fmaxf(m, cn[k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (threadIdx.x == 0) {
            *cmax2 = m;
            *nfb = 0u;
        }
    }
}

__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Four consecutive coordinates of row i: fp32 X when given, else hi + lo of its planes.
__device__ __forceinline__ float4 load_x4(const float *__restrict__ X32,
                                          const uint16_t *__restrict__ xhi,
                                          const uint16_t *__restrict__ xlo, int64_t lda,
                                          int d, int64_t i, int j) {
    if (X32 != nullptr) return *reinterpret_cast<const float4 *>(X32 + i * d + j);
    const uint2 h = *reinterpret_cast<const uint2 *>(xhi + i * lda + j);
    const uint2 l = *reinterpret_cast<const uint2 *>(xlo + i * lda + j);
    return make_float4(bf16_lo_f(h.x) + bf16_lo_f(l.x), bf16_hi_f(h.x) + bf16_hi_f(l.x),
                       bf16_lo_f(h.y) + bf16_lo_f(l.y), bf16_hi_f(h.y) + bf16_hi_f(l.y));
}

// Lane `sub`'s share of the squared distance ||x_i - c_k||^2 in the difference form, in
// fp64 (the difference of two fp32 values is formed exactly in fp64, so only the squares
// and sums round): columns 4 * (sub + t * L) .. + 3.  group_sum then adds the L lanes'
// shares by a butterfly (every lane of the group ends with the same bits), so the result
// is accurate to about 1e-15 relative and does not depend on which group or pass made it.
__device__ __forceinline__ double lane_dist2(const float *__restrict__ X32,
                                             const uint16_t *__restrict__ xhi,
                                             const uint16_t *__restrict__ xlo, int64_t lda,
                                             const float *__restrict__ C, int d, int64_t i,
                                             int k, int sub, int L) {
    double acc = 0.0;
    const float *c = C + static_cast<int64_t>(k) * d;
    for (int j = sub * 4; j < d; j += 4 * L) {
        const float4 x = load_x4(X32, xhi, xlo, lda, d, i, j);
        const float4 y = *reinterpret_cast<const float4 *>(c + j);
        const double e0 = static_cast<double>(x.x) - y.x, e1 = static_cast<double>(x.y) - y.y;
        const double e2 = static_cast<double>(x.z) - y.z, e3 = static_cast<double>(x.w) - y.w;
        acc = fma(e0, e0, acc);
        acc = fma(e1, e1, acc);
        acc = fma(e2, e2, acc);
        acc = fma(e3, e3, acc);
    }
    return acc;
}

// Sum over each aligned group of L lanes (all 32 lanes take part).
__device__ __forceinline__ double group_sum(double v, int L) {
    for (int o = L >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Lanes per candidate: enough for four float4 per lane, at least 4 and at most 32.
__host__ __device__ inline int rerank_lanes(int d) {
    int L = 4;
    while (L < 32 && L * 16 < d) L <<= 1;
    return L;
}

// (dist, k) pairs: smaller distance first, then the lower centroid index.
__device__ __forceinline__ bool better(double da, int ka, double db, int kb) {
    return kb < 0 || (ka >= 0 && (da < db || (da == db && ka < kb)));
}

// One warp per row: exact distances of the row's candidates, 32 / L of them at a time;
// rows that overflowed (or, for inputs outside the supported range, have no candidate) are
// queued for the three-product pass.  The queue's order depends on scheduling; the labels
// do not.  A row with a single candidate needs no distance unless `mind` is wanted.
__global__ void rerank_kernel(const float *__restrict__ X32, const uint16_t *__restrict__ xhi,
                              const uint16_t *__restrict__ xlo, int64_t lda,
                              const float *__restrict__ C, int64_t N, int d, int K,
                              const int32_t *__restrict__ cand, int32_t *__restrict__ labels,
                              float *__restrict__ mind, uint32_t *__restrict__ nfb,
                              int32_t *__restrict__ fbrows) {
    const int lane = threadIdx.x & 31;
    const int L = rerank_lanes(d);
    const int G = 32 / L;  // candidates per pass
    const int q = lane / L, sub = lane % L;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // Most rows need only their candidate slots, so a warp keeps the slots of its next
    // kPrefetch rows in flight while it handles the current one.
    constexpr int kPrefetch = 4;
    auto slots = [&](int64_t r) {
        return (r < N && lane < kCandPerRow) ? cand[r * kCandPerRow + lane] : -1;
    };
    int ring[kPrefetch];
#pragma unroll
    for (int t = 0; t < kPrefetch; ++t) ring[t] = slots(warp + t * nwarps);
    for (int64_t i = warp; i < N; i += nwarps) {
        const int c = ring[0];
#pragma unroll
        for (int t = 0; t + 1 < kPrefetch; ++t) ring[t] = ring[t + 1];
        ring[kPrefetch - 1] = slots(i + kPrefetch * nwarps);
        const bool ovf = __any_sync(0xffffffffu, c == kCandOverflow);
        const uint32_t valid = __ballot_sync(0xffffffffu, c >= 0 && c < K);
        if (ovf || valid == 0u) {
            if (lane == 0) fbrows[atomicAdd(nfb, 1u)] = static_cast<int32_t>(i);
            continue;
        }
        const int n = __popc(valid);
        if (mind == nullptr && n == 1) {
            const int k = __shfl_sync(0xffffffffu, c, __ffs(valid) - 1);
            if (lane == 0) labels[i] = k;
            continue;
        }
        double best = 0.0;
        int bestk = -1;
        for (int p = 0; p < n; p += G) {
            const int slot = p + q;  // this group's candidate: the slot-th valid lane
            const int src = slot < n ? static_cast<int>(__fns(valid, 0, slot + 1)) : 0;
            const int k = __shfl_sync(0xffffffffu, c, src);
            const double part =
                slot < n ? lane_dist2(X32, xhi, xlo, lda, C, d, i, k, sub, L) : 0.0;
            const double dk = group_sum(part, L);
            const int kk = slot < n ? k : -1;
            if (better(dk, kk, best, bestk)) {
                best = dk;
                bestk = kk;
            }
        }
        // combine the groups' winners (same order-free rule everywhere)
        for (int o = L; o < 32; o <<= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int ok = __shfl_xor_sync(0xffffffffu, bestk, o);
            if (better(ob, ok, best, bestk)) {
                best = ob;
                bestk = ok;
            }
        }
        if (lane == 0) {
            labels[i] = bestk;
            if (mind) mind[i] = static_cast<float>(best);
        }
    }
}

// Copy the hi and lo planes of the queued rows into a compact [2][N][dp] buffer.
__global__ void fb_gather_kernel(const uint32_t *__restrict__ nfb,
                                 const int32_t *__restrict__ fbrows,
                                 const uint16_t *__restrict__ xs, int64_t lda, int64_t N,
                                 int dp, uint16_t *__restrict__ xsfb) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t n = *nfb;
    const int vec = dp / 8;  // 16-byte vectors per plane row
    for (int64_t j = warp; j < n; j += nwarps) {
        const int64_t row = fbrows[j];
        for (int p = 0; p < 2; ++p) {
            const uint4 *src = reinterpret_cast<const uint4 *>(xs + p * N * lda + row * lda);
            uint4 *dst = reinterpret_cast<uint4 *>(xsfb + (p * N + j) * dp);
            for (int v = lane; v < vec; v += 32) dst[v] = src[v];
        }
    }
}

// Labels of the queued rows back to their places, with their exact distances for `mind`.
__global__ void fb_scatter_kernel(const uint32_t *__restrict__ nfb,
                                  const int32_t *__restrict__ fbrows,
                                  const int32_t *__restrict__ fblab, int32_t *__restrict__ labels,
                                  float *__restrict__ mind, const float *__restrict__ X32,
                                  const uint16_t *__restrict__ xhi,
                                  const uint16_t *__restrict__ xlo, int64_t lda,
                                  const float *__restrict__ C, int d) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t n = *nfb;
    for (int64_t j = warp; j < n; j += nwarps) {
        const int64_t row = fbrows[j];
        const int k = fblab[j];
        double dk = 0.0;
        if (mind) dk = group_sum(lane_dist2(X32, xhi, xlo, lda, C, d, row, k, lane, 32), 32);
        if (lane == 0) {
            labels[row] = k;
            if (mind) mind[row] = static_cast<float>(dk);
        }
    }
}

// Rows queued by the re-ranking whose labels the three-product pass may not decide (padded
// depth beyond kThreeProductMaxDp): the exact argmin over all K centroids, each distance in
// the fp64 difference form of lane_dist2 (the re-ranking's own form at these depths), the
// lowest index on equal values.  One block per queued row at a time (the count is read on
// the device); warp w takes centroids w, w + 8, ...
constexpr int kScanWarps = 8;
__global__ void __launch_bounds__(kScanWarps * 32)
    exact_scan_kernel(const uint32_t *__restrict__ nfb, const int32_t *__restrict__ fbrows,
                      const float *__restrict__ X32, const uint16_t *__restrict__ xhi,
                      const uint16_t *__restrict__ xlo, int64_t lda,
                      const float *__restrict__ C, int d, int K, int32_t *__restrict__ labels,
                      float *__restrict__ mind) {
    __shared__ double s_best[kScanWarps];
    __shared__ int s_k[kScanWarps];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t n = *nfb;
    for (int64_t j = blockIdx.x; j < n; j += gridDim.x) {
        const int64_t row = fbrows[j];
        double best = 0.0;
        int bestk = -1;
        for (int k = warp; k < K; k += kScanWarps) {
            const double dk = group_sum(lane_dist2(X32, xhi, xlo, lda, C, d, row, k, lane, 32), 32);
            if (better(dk, k, best, bestk)) {
                best = dk;
                bestk = k;
            }
        }
        if (lane == 0) {
            s_best[warp] = best;
            s_k[warp] = bestk;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 0; w < kScanWarps; ++w)
                if (better(s_best[w], s_k[w], best, bestk)) {
                    best = s_best[w];
                    bestk = s_k[w];
                }
            labels[row] = bestk;
            if (mind) mind[row] = static_cast<float>(best);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_assign_screened(const AssignArgs &a, const float *X32, const float *C,
                                   const ScreenBufs &sb, cudaStream_t st, cudaEvent_t ev_mma0,
                                   cudaEvent_t ev_mma1) {
    const uint16_t *xhi = static_cast<const uint16_t *>(a.a_planes);
    const uint16_t *xlo = xhi + a.N * a.lda;
    window_kernel<<<1, 1024, 0, st>>>(a.cn, a.K, sb.cmax2, sb.nfb);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    AssignArgs s1 = a;  // single product over the hi plane
    s1.a_nplanes = 1;
    s1.cand = sb.cand;
    s1.cmax2 = sb.cmax2;
    s1.mind = nullptr;
    s1.best = nullptr;
    s1.n_dev = nullptr;
    if (ev_mma0 && (e = record_event(ev_mma0, st)) != cudaSuccess) return e;
    if ((e = launch_assign(s1, st)) != cudaSuccess) return e;
    if (ev_mma1 && (e = record_event(ev_mma1, st)) != cudaSuccess) return e;

    const int64_t rr_blocks = ceil_div(a.N, 8);
    const int rgrid = static_cast<int>(rr_blocks < 148 * 16 ? rr_blocks : 148 * 16);
    rerank_kernel<<<rgrid, 256, 0, st>>>(X32, xhi, xlo, a.lda, C, a.N, a.d, a.K, sb.cand,
                                         a.labels, a.mind, sb.nfb, sb.fbrows);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    if (a.dp > kThreeProductMaxDp) {  // overflow rows: exact scan instead of three products
        exact_scan_kernel<<<device_sm_count() * 8, kScanWarps * 32, 0, st>>>(
            sb.nfb, sb.fbrows, X32, xhi, xlo, a.lda, C, a.d, a.K, a.labels, a.mind);
        note_launch();
        return cudaGetLastError();
    }

    fb_gather_kernel<<<148 * 4, 256, 0, st>>>(sb.nfb, sb.fbrows, xhi, a.lda, a.N, a.dp,
                                              sb.xsfb);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    AssignArgs f = a;  // three products over the queued rows (count read on the device)
    f.a_planes = sb.xsfb;
    f.a_nplanes = 2;
    f.lda = a.dp;
    f.n_dev = sb.nfb;
    f.labels = sb.fblab;
    f.mind = nullptr;
    f.best = nullptr;
    f.xnorm = nullptr;
    f.cand = nullptr;
    if ((e = launch_assign(f, st)) != cudaSuccess) return e;

    fb_scatter_kernel<<<148 * 4, 256, 0, st>>>(sb.nfb, sb.fbrows, sb.fblab, a.labels, a.mind,
                                               X32, xhi, xlo, a.lda, C, a.d);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk

namespace fk {

cudaError_t launch_screen_probe(const AssignArgs &a, int64_t n_probe, const float *X32,
                                const float *C, const ScreenBufs &sb, cudaStream_t st) {
    // the screening pass and the re-ranking over the first n_probe rows only; the rows
    // that would need the three-product pass are counted in sb.nfb, not assigned
    window_kernel<<<1, 1024, 0, st>>>(a.cn, a.K, sb.cmax2, sb.nfb);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    AssignArgs s1 = a;
    s1.N = n_probe;
    s1.a_nplanes = 1;
    s1.cand = sb.cand;
    s1.cmax2 = sb.cmax2;
    s1.mind = nullptr;
    s1.best = nullptr;
    s1.n_dev = nullptr;
    if ((e = launch_assign(s1, st)) != cudaSuccess) return e;
    const uint16_t *xhi = static_cast<const uint16_t *>(a.a_planes);
    const int64_t rr_blocks = ceil_div(n_probe, 8);
    const int rgrid = static_cast<int>(rr_blocks < 148 * 16 ? rr_blocks : 148 * 16);
    rerank_kernel<<<rgrid, 256, 0, st>>>(X32, xhi, xhi + a.N * a.lda, a.lda, C, n_probe, a.d,
                                         a.K, sb.cand, a.labels, nullptr, sb.nfb, sb.fbrows);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk
