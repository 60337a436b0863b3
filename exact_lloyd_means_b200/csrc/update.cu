// update.cu -- atomic-free centroid update over the sorted inverse index.
//
// Flash-KMeans article, section "Sort-Inverse Update：原子操作的另一种解法": after the
// assignments are sorted by cluster id, each cluster is reduced by reading its points
// contiguously through the inverse index, with no atomics, so hot clusters cause no
// contention.  The new centroid is the mean of the cluster's points (section
// "为什么"快"这件事被拖了这么久"); an empty cluster keeps its previous centroid.
//
// B200 design:
//   level 1  : the sorted order [0, N) is cut into fixed chunks of 512 positions, one per
//              warp, independent of where clusters start.  A warp gathers its rows through
//              perm (each row is d contiguous values, read as 16-byte vectors across the
//              lanes, several rows in flight), adds them in position order in fp64 and,
//              whenever the cluster id changes, either finishes the cluster (all of it
//              lies in this chunk: mean = sum / count, rounded once to fp32) or emits a
//              "piece" (the chunk's first or last cluster, which continues outside).  The
//              same pass accumulates the objective sum ||x - c_used[label]||^2 in fp64.
//   level L>1: groups of 64 consecutive units of the previous level are reduced the same
//              way over their pieces, in piece order.  A cluster is finished at the first
//              level whose unit (512 * 64^(L-1) positions) contains all of it, so a
//              cluster with millions of points is split over thousands of warps at
//              level 1 and finished after a few levels with short, parallel sums.
//   finalize : counts from the CSR offsets; empty clusters copy C_old bit for bit.
//   objective: the per-warp partials are summed in a fixed tree by one block.
// Every sum has a fixed order that depends only on N, d and the offsets, so the result is
// the same on every run.
#include <cuda_bf16.h>

#include "fk_common.cuh"

namespace fk {
namespace {

constexpr int kGroup = 64;  // units of level L-1 per unit of level L

template <bool BF16>
__device__ __forceinline__ void load4(const void *X, int64_t off, float (&v)[4]) {
    if constexpr (BF16) {
        const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(X) + off);
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xffff0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
        const float4 f = *reinterpret_cast<const float4 *>(static_cast<const float *>(X) + off);
        v[0] = f.x;
        v[1] = f.y;
        v[2] = f.z;
        v[3] = f.w;
    }
}

// Write the mean of a finished cluster: C_new[k][col..col+3] = acc / cnt.
__device__ __forceinline__ void store_mean(float *C_new, int64_t k, int d, int col,
                                           const double (&acc)[4], double cnt) {
    float4 o;
    o.x = static_cast<float>(acc[0] / cnt);
    o.y = static_cast<float>(acc[1] / cnt);
    o.z = static_cast<float>(acc[2] / cnt);
    o.w = static_cast<float>(acc[3] / cnt);
    *reinterpret_cast<float4 *>(C_new + k * d + col) = o;
}

// Level 1.  grid.x covers warps (8 per block), grid.y the column passes.
template <int SL, bool BF16>
__global__ void __launch_bounds__(kUpdWarps * 32)
    seg_rows_kernel(const void *__restrict__ X, int64_t N, int d, int64_t nwarps, int dcov,
                    const int32_t *__restrict__ skeys, const int32_t *__restrict__ perm,
                    const int32_t *__restrict__ offsets, const float *__restrict__ C_used,
                    float *__restrict__ C_new, double *__restrict__ pieces,
                    int32_t *__restrict__ pkeys, double *__restrict__ jpart) {
    constexpr int B = SL >= 4 ? 2 : (SL >= 2 ? 4 : 8);  // rows in flight per lane
    const int lane = threadIdx.x & 31;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * kUpdWarps + (threadIdx.x >> 5);
    if (w >= nwarps) return;
    const int cb = blockIdx.y;
    const int col0 = cb * 128 * SL;
    const int64_t p0 = w * kRowsPerWarp;
    const int64_t p1 = p0 + kRowsPerWarp < N ? p0 + kRowsPerWarp : N;

    double acc[SL][4];
    float cu[SL][4];
    double jacc = 0.0;
    int cur = -1, first = -1, slot1 = -1;

    auto flush = [&](int k) {
        const int64_t lo = offsets[k], hi = offsets[k + 1];
        if (lo >= p0 && hi <= p1) {
            const double cnt = static_cast<double>(hi - lo);
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                const int col = col0 + s * 128 + lane * 4;
                if (col < d) store_mean(C_new, k, d, col, acc[s], cnt);
            }
        } else {
            const int slot = (k == first) ? 0 : 1;
            if (slot == 1) slot1 = k;
            double *dst = pieces + (w * 2 + slot) * static_cast<int64_t>(dcov) + col0;
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                double2 *q = reinterpret_cast<double2 *>(dst + s * 128 + lane * 4);
                q[0] = make_double2(acc[s][0], acc[s][1]);
                q[1] = make_double2(acc[s][2], acc[s][3]);
            }
        }
    };

    for (int64_t p = p0; p < p1; p += B) {
        const int nb = p1 - p < B ? static_cast<int>(p1 - p) : B;
        int myk = 0, myi = 0;
        if (lane < nb) {
            myk = skeys[p + lane];
            myi = perm[p + lane];
        }
        float xr[B][SL][4];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int i = __shfl_sync(0xffffffffu, myi, j);
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                const int col = col0 + s * 128 + lane * 4;
                if (j < nb && col < d) {
                    load4<BF16>(X, static_cast<int64_t>(i) * d + col, xr[j][s]);
                } else {
                    xr[j][s][0] = xr[j][s][1] = xr[j][s][2] = xr[j][s][3] = 0.f;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int k = __shfl_sync(0xffffffffu, myk, j);
            if (j < nb) {
                if (k != cur) {
                    if (cur >= 0) flush(cur);
                    if (cur < 0) first = k;
                    cur = k;
#pragma unroll
                    for (int s = 0; s < SL; ++s) {
                        const int col = col0 + s * 128 + lane * 4;
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[s][e] = 0.0;
                        if (col < d) {
                            const float4 c =
                                *reinterpret_cast<const float4 *>(C_used + int64_t(k) * d + col);
                            cu[s][0] = c.x;
                            cu[s][1] = c.y;
                            cu[s][2] = c.z;
                            cu[s][3] = c.w;
                        } else {
                            cu[s][0] = cu[s][1] = cu[s][2] = cu[s][3] = 0.f;
                        }
                    }
                }
#pragma unroll
                for (int s = 0; s < SL; ++s) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const double xv = xr[j][s][e];
                        acc[s][e] += xv;
                        const double df = xv - static_cast<double>(cu[s][e]);
                        jacc += df * df;
                    }
                }
            }
        }
    }
    if (cur >= 0) flush(cur);
    if (cb == 0 && lane == 0) {
        // slot 0 holds the first cluster if it was not finished here; slot 1 the last
        const int64_t lo = offsets[first], hi = offsets[first + 1];
        const bool first_done = lo >= p0 && hi <= p1;
        pkeys[w * 2 + 0] = first_done ? -1 : first;
        pkeys[w * 2 + 1] = slot1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) jacc += __shfl_xor_sync(0xffffffffu, jacc, o);
    if (lane == 0) jpart[static_cast<int64_t>(cb) * nwarps + w] = jacc;
}

// Level L >= 2: one warp per group of kGroup units of the previous level (2 piece slots
// each).  `span` = positions covered by one unit of THIS level.
template <int SL>
__global__ void __launch_bounds__(kUpdWarps * 32)
    seg_pieces_kernel(const double *__restrict__ pin, const int32_t *__restrict__ kin,
                      int64_t nslots_in, double *__restrict__ pout,
                      int32_t *__restrict__ kout, int64_t nunits, int64_t span, int d,
                      int dcov, const int32_t *__restrict__ offsets, float *__restrict__ C_new) {
    const int lane = threadIdx.x & 31;
    const int64_t u = static_cast<int64_t>(blockIdx.x) * kUpdWarps + (threadIdx.x >> 5);
    if (u >= nunits) return;
    const int cb = blockIdx.y;
    const int col0 = cb * 128 * SL;
    const int64_t s0 = u * 2 * kGroup;
    const int64_t s1 = s0 + 2 * kGroup < nslots_in ? s0 + 2 * kGroup : nslots_in;

    double acc[SL][4];
    int cur = -1, first = -1, slot1 = -1;
    bool first_done = false;

    auto flush = [&](int k) {
        const int64_t lo = offsets[k], hi = offsets[k + 1];
        const bool done = (lo / span) == ((hi - 1) / span);
        if (k == first) first_done = done;
        if (done) {
            const double cnt = static_cast<double>(hi - lo);
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                const int col = col0 + s * 128 + lane * 4;
                if (col < d) store_mean(C_new, k, d, col, acc[s], cnt);
            }
        } else {
            const int slot = (k == first) ? 0 : 1;
            if (slot == 1) slot1 = k;
            double *dst = pout + (u * 2 + slot) * static_cast<int64_t>(dcov) + col0;
#pragma unroll
            for (int s = 0; s < SL; ++s) {
                double2 *q = reinterpret_cast<double2 *>(dst + s * 128 + lane * 4);
                q[0] = make_double2(acc[s][0], acc[s][1]);
                q[1] = make_double2(acc[s][2], acc[s][3]);
            }
        }
    };

    for (int64_t sl = s0; sl < s1; ++sl) {
        const int k = kin[sl];
        if (k < 0) continue;
        const double *src = pin + sl * static_cast<int64_t>(dcov) + col0;
        double v[SL][4];
#pragma unroll
        for (int s = 0; s < SL; ++s) {
            const double2 *q = reinterpret_cast<const double2 *>(src + s * 128 + lane * 4);
            const double2 a = q[0], b = q[1];
            v[s][0] = a.x;
            v[s][1] = a.y;
            v[s][2] = b.x;
            v[s][3] = b.y;
        }
        if (k != cur) {
            if (cur >= 0) flush(cur);
            if (cur < 0) first = k;
            cur = k;
#pragma unroll
            for (int s = 0; s < SL; ++s)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[s][e] = 0.0;
        }
#pragma unroll
        for (int s = 0; s < SL; ++s)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[s][e] += v[s][e];
    }
    if (cur >= 0) flush(cur);
    if (cb == 0 && lane == 0) {
        kout[u * 2 + 0] = (first >= 0 && !first_done) ? first : -1;
        kout[u * 2 + 1] = slot1;
    }
}

// counts[k] = offsets[k+1] - offsets[k]; an empty cluster keeps C_old bit for bit.
__global__ void finalize_kernel(const int32_t *__restrict__ offsets, int K, int d,
                                const float *__restrict__ C_old, float *__restrict__ C_new,
                                int32_t *__restrict__ counts) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t k = warp; k < K; k += nw) {
        const int32_t c = offsets[k + 1] - offsets[k];
        if (lane == 0 && counts) counts[k] = c;
        if (c == 0)
            for (int j = lane; j < d; j += 32) C_new[k * d + j] = C_old[k * d + j];
    }
}

// One block sums n partials: thread t adds t, t+1024, ... in order, then a fixed tree.
__global__ void __launch_bounds__(1024)
    objective_kernel(const double *__restrict__ part, int64_t n, double *__restrict__ out) {
    __shared__ double sh[1024];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += 1024) s += part[i];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int o = 512; o > 0; o >>= 1) {
        if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = sh[0];
}

template <int SL>
cudaError_t run_levels(const void *X, bool bf16, int64_t N, int d, const UpdPlan &up,
                       const int32_t *skeys, const int32_t *perm, const int32_t *offsets,
                       const float *C_used, float *C_new, double *pa, int32_t *ka,
                       double *pb, int32_t *kb, double *jpart, cudaStream_t st) {
    const dim3 block(kUpdWarps * 32);
    dim3 grid(static_cast<unsigned>(ceil_div(up.nwarps, kUpdWarps)), up.ncolblk);
    if (bf16)
        seg_rows_kernel<SL, true><<<grid, block, 0, st>>>(X, N, d, up.nwarps, up.dcov, skeys,
                                                          perm, offsets, C_used, C_new, pa, ka,
                                                          jpart);
    else
        seg_rows_kernel<SL, false><<<grid, block, 0, st>>>(X, N, d, up.nwarps, up.dcov, skeys,
                                                           perm, offsets, C_used, C_new, pa,
                                                           ka, jpart);
    note_launch();
    int64_t units = up.nwarps;
    int64_t span = kRowsPerWarp;
    double *pin = pa, *pout = pb;
    int32_t *kin = ka, *kout = kb;
    while (units > 1) {
        const int64_t nunits = ceil_div(units, kGroup);
        span *= kGroup;
        dim3 g2(static_cast<unsigned>(ceil_div(nunits, kUpdWarps)), up.ncolblk);
        seg_pieces_kernel<SL><<<g2, block, 0, st>>>(pin, kin, units * 2, pout, kout, nunits,
                                                    span, d, up.dcov, offsets, C_new);
        note_launch();
        units = nunits;
        double *tp = pin;
        pin = pout;
        pout = tp;
        int32_t *tk = kin;
        kin = kout;
        kout = tk;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_update(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                          const UpdPlan &up, const int32_t *skeys, const int32_t *perm,
                          const int32_t *offsets, const float *C_old, const float *C_used,
                          float *C_new, int32_t *counts, double *pieces_a, int32_t *pkeys_a,
                          double *pieces_b, int32_t *pkeys_b, double *jpart,
                          double *objective, cudaStream_t st) {
    const bool bf16 = dtype == FK_BF16;
    cudaError_t e;
    switch (up.slices) {
#define FK_SL(n)                                                                            \
    case n:                                                                                 \
        e = run_levels<n>(X, bf16, N, d, up, skeys, perm, offsets, C_used, C_new, pieces_a, \
                          pkeys_a, pieces_b, pkeys_b, jpart, st);                           \
        break;
        FK_SL(1)
        FK_SL(2)
        FK_SL(3)
        FK_SL(4)
        FK_SL(5)
        FK_SL(6)
        FK_SL(7)
        FK_SL(8)
#undef FK_SL
        default:
            return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    int64_t fgrid = ceil_div(K, 8);
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (fgrid > cap) fgrid = cap;
    finalize_kernel<<<static_cast<unsigned>(fgrid), 256, 0, st>>>(offsets, K, d, C_old, C_new,
                                                                   counts);
    note_launch();
    if (objective) {
        objective_kernel<<<1, 1024, 0, st>>>(jpart, up.nwarps * up.ncolblk, objective);
        note_launch();
    }
    return cudaGetLastError();
}

}  // namespace fk
