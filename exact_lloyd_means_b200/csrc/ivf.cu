// ivf.cu -- inverted lists of a finished clustering (the coarse quantizer's output).
//
// LEANN FlashLib guide, section "工作原理": after k-means, an IVF index stores, per cell,
// the ids of its points in CSR form (offsets per cell, then row ids), and the points of a
// cell next to each other.  The ids come from the same stable sort of the labels that the
// update uses; this file adds the gather of the points into cell order.
#include "fk_common.cuh"

namespace fk {
namespace {

// X_lists[i] = X[row_ids[i]]: rows of 16-byte vectors, each copied by a group of G lanes
// (G = 32, or 16 for rows of at most 16 vectors, so that short rows keep the whole warp
// busy).  Reads and writes are contiguous within a row; rows are read in cell order.
__global__ void gather_rows_kernel(const uint4 *__restrict__ X, int64_t N, int vec_per_row,
                                   const int32_t *__restrict__ row_ids,
                                   uint4 *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int G = vec_per_row <= 16 ? 16 : 32;
    const int rows_per_warp = 32 / G;
    const int sub = lane % G;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t i0 = warp * rows_per_warp; i0 < N; i0 += nwarps * rows_per_warp) {
        const int64_t i = i0 + lane / G;
        if (i >= N) continue;
        const int64_t src = row_ids[i];
        const uint4 *s = X + src * vec_per_row;
        uint4 *t = out + i * vec_per_row;
        for (int v = sub; v < vec_per_row; v += G) t[v] = s[v];
    }
}

}  // namespace

cudaError_t launch_gather_rows(const void *X, int64_t N, int64_t row_bytes,
                               const int32_t *row_ids, void *out, cudaStream_t st) {
    if (N <= 0) return cudaSuccess;
    const int vec = static_cast<int>(row_bytes / 16);
    const int64_t blocks = ceil_div(N, 8);
    const int grid = static_cast<int>(blocks < 148 * 16 ? blocks : 148 * 16);
    gather_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint4 *>(X), N, vec, row_ids,
                                             static_cast<uint4 *>(out));
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk
