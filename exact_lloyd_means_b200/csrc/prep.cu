// prep.cu -- operand preparation for the assign kernel, and cosine-mode normalisation.
//
//  * split_x:   fp32 X -> two bf16 planes hi = RN_bf16(x), lo = RN_bf16(x - hi), padded
//               with zeros to dp columns.  x - hi is exact in fp32, so hi + lo carries 16
//               significant bits of x and the three tensor-core products hi*hi' + lo*hi' +
//               hi*lo' reproduce x.c to about 3 * 2^-16 relative (fp32 emulation).
//  * prep_centroids: the same split of each centroid, scaled by -2 (exact in bf16), so the
//               MMA accumulates -2 x.c directly; cn[k] = ||c_k||^2 (fp64 accumulation of
//               the values the MMA consumes, rounded once to fp32); caug[k] = the three
//               bf16 pieces hi + mid + lo that sum exactly to that fp32 value (for norms
//               of at least 2^-110), then zeros.  One extra K = 16 MMA step against
//               constant (1, 1, 1, 0, ...) columns of X folds them into the accumulator,
//               to within one fp32 ulp: the MMA adds the three products in an order the
//               ISA does not fix, and hi + lo first can round.  Padding centroids get
//               cn = +inf, a largest-finite bf16 first piece and zero planes, so they
//               never win.
//  * normalize: cosine mode (LEANN FlashLib guide, "距离度量只有 squared L2如何支持 mips /
//               cosine"): x / ||x|| with a zero norm replaced by 1; the norm and the
//               quotient are computed in fp64 and rounded once to fp32.
#include <cuda_bf16.h>

#include "fk_common.cuh"
#include "prep_row.cuh"

namespace fk {
namespace {

// One warp per row; lanes walk the row four columns at a time.
__global__ void split_x_kernel(const float *__restrict__ X, int64_t N, int d, int64_t dp,
                               uint16_t *__restrict__ hi, uint16_t *__restrict__ lo,
                               float *__restrict__ xnorm) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t i = warp; i < N; i += nwarps) {
        const float *x = X + i * d;
        uint16_t *h = hi + i * dp;
        uint16_t *l = lo + i * dp;
        double s = 0.0;
        for (int64_t j = lane * 4; j < dp; j += 128) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < d) v = *reinterpret_cast<const float4 *>(x + j);
            const float e[4] = {v.x, v.y, v.z, v.w};
            uint16_t hb[4], lb[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                hb[t] = bf16_bits(e[t]);
                lb[t] = bf16_bits(e[t] - bf16_val(hb[t]));
                s += static_cast<double>(e[t]) * e[t];
            }
            uint2 hv, lv;
            hv.x = hb[0] | (static_cast<uint32_t>(hb[1]) << 16);
            hv.y = hb[2] | (static_cast<uint32_t>(hb[3]) << 16);
            lv.x = lb[0] | (static_cast<uint32_t>(lb[1]) << 16);
            lv.y = lb[2] | (static_cast<uint32_t>(lb[3]) << 16);
            *reinterpret_cast<uint2 *>(h + j) = hv;
            *reinterpret_cast<uint2 *>(l + j) = lv;
        }
        if (xnorm) {
            s = warp_sum_d(s);
            if (lane == 0) xnorm[i] = static_cast<float>(s);
        }
    }
}

// bf16 X with d % 64 != 0 copied into a zero-padded [N][dp] plane (TMA boxes are 64 wide).
__global__ void pad_bf16_kernel(const uint16_t *__restrict__ X, int64_t N, int d, int64_t dp,
                                uint16_t *__restrict__ out) {
    const int64_t total = N * dp;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = t / dp;
        const int64_t j = t - i * dp;
        out[t] = j < d ? X[i * d + j] : static_cast<uint16_t>(0);
    }
}

__global__ void xnorm_bf16_kernel(const uint16_t *__restrict__ X, int64_t N, int d,
                                  float *__restrict__ xnorm) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t i = warp; i < N; i += nwarps) {
        double s = 0.0;
        for (int j = lane; j < d; j += 32) {
            const double v = bf16_val(X[i * d + j]);
            s += v * v;
        }
        s = warp_sum_d(s);
        if (lane == 0) xnorm[i] = static_cast<float>(s);
    }
}

__global__ void normalize_kernel(const float *__restrict__ X, float *__restrict__ Y, int64_t N,
                                 int d) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t i = warp; i < N; i += nwarps) {
        const float *x = X + i * d;
        double s = 0.0;
        for (int j = lane * 4; j < d; j += 128) {
            const float4 v = *reinterpret_cast<const float4 *>(x + j);
            s += static_cast<double>(v.x) * v.x + static_cast<double>(v.y) * v.y +
                 static_cast<double>(v.z) * v.z + static_cast<double>(v.w) * v.w;
        }
        s = warp_sum_d(s);
        double nrm = sqrt(s);
        if (nrm == 0.0) nrm = 1.0;
        float *y = Y + i * d;
        for (int j = lane * 4; j < d; j += 128) {
            const float4 v = *reinterpret_cast<const float4 *>(x + j);
            float4 o;
            o.x = static_cast<float>(static_cast<double>(v.x) / nrm);
            o.y = static_cast<float>(static_cast<double>(v.y) / nrm);
            o.z = static_cast<float>(static_cast<double>(v.z) / nrm);
            o.w = static_cast<float>(static_cast<double>(v.w) / nrm);
            *reinterpret_cast<float4 *>(y + j) = o;
        }
    }
}

// One warp per (padded) centroid row (prep_row.cuh).
__global__ void prep_centroids_kernel(const float *__restrict__ C, int K, int d,
                                      CentroidOperands o) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t k = warp; k < o.Kp; k += nwarps) prep_centroid_row(C, K, d, o, k, lane);
}

__global__ void centroid_norms_kernel(const float *__restrict__ C, int K, int d, int round_bf16,
                                      float *__restrict__ cn) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t k = warp; k < K; k += nwarps) {
        double s = 0.0;
        for (int j = lane; j < d; j += 32) {
            float c = C[k * d + j];
            if (round_bf16) c = bf16_val(bf16_bits(c));
            s += static_cast<double>(c) * c;
        }
        s = warp_sum_d(s);
        if (lane == 0) cn[k] = static_cast<float>(s);
    }
}

int grid_for_warps(int64_t warps, int threads) {
    const int64_t per_block = threads / 32;
    int64_t g = (warps + per_block - 1) / per_block;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (g > cap) g = cap;
    return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_split_x(const float *X, int64_t N, int d, int64_t dp, uint16_t *hi,
                           uint16_t *lo, float *xnorm, cudaStream_t st) {
    split_x_kernel<<<grid_for_warps(N, 256), 256, 0, st>>>(X, N, d, dp, hi, lo, xnorm);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_pad_bf16(const uint16_t *X, int64_t N, int d, int64_t dp, uint16_t *out,
                            cudaStream_t st) {
    pad_bf16_kernel<<<device_sm_count() * 8, 256, 0, st>>>(X, N, d, dp, out);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_normalize(const float *X, float *Y, int64_t N, int d, cudaStream_t st) {
    normalize_kernel<<<grid_for_warps(N, 256), 256, 0, st>>>(X, Y, N, d);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_xnorm_bf16(const uint16_t *X, int64_t N, int d, float *xnorm,
                              cudaStream_t st) {
    xnorm_bf16_kernel<<<grid_for_warps(N, 256), 256, 0, st>>>(X, N, d, xnorm);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_prep_centroids(const float *C, int K, int d, int64_t Kp, int64_t dp,
                                  fk_dtype dtype, uint16_t *planes, float *cn, float *cused,
                                  uint16_t *caug, cudaStream_t st) {
    const CentroidOperands o{planes, cn, cused, caug, Kp, dp, dtype == FK_BF16 ? 0 : 1};
    prep_centroids_kernel<<<grid_for_warps(Kp, 256), 256, 0, st>>>(C, K, d, o);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_centroid_norms(const float *C, int K, int d, fk_dtype dtype, float *cn,
                                  cudaStream_t st) {
    centroid_norms_kernel<<<grid_for_warps(K, 256), 256, 0, st>>>(
        C, K, d, dtype == FK_BF16 ? 1 : 0, cn);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk
