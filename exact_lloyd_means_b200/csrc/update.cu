// update.cu -- atomic-free centroid update over the sorted inverse index.
//
// Flash-KMeans article, section "Sort-Inverse Update：原子操作的另一种解法": after the
// assignments are sorted by cluster id, each cluster is reduced by reading its points
// contiguously through the inverse index, with no atomics, so hot clusters cause no
// contention.  The new centroid is the mean of the cluster's points (section
// "为什么"快"这件事被拖了这么久"); an empty cluster keeps its previous centroid.
//
// B200 design:
//   level 1  : the sorted order [0, N) is cut into fixed chunks of R positions (a power of
//              two, 64..256, chosen from N), one per warp and 128-column block, independent
//              of where clusters start.  A warp gathers its rows through perm (512
//              contiguous bytes of a row per warp, read as 16-byte vectors across the lanes,
//              eight rows in flight), adds them in position order in fp64 and,
//              whenever the cluster id changes, either finishes the cluster (all of it
//              lies in this chunk, which the keys just outside the chunk tell: mean =
//              sum / count, rounded once to fp32) or emits a "piece" (the chunk's first or
//              last cluster, which continues outside).  The same pass accumulates the
//              objective sum ||x - c_used[label]||^2 in fp64.
//   level L>1: groups of 16 consecutive units of the previous level are reduced the same
//              way over their pieces, in piece order.  A cluster is finished at the first
//              level whose unit (R * 16^(L-1) positions) contains all of it, so a
//              cluster with millions of points is split over thousands of warps at
//              level 1 and finished after a few levels with short, parallel sums.
//   finalize : counts from the CSR offsets; empty clusters copy C_old bit for bit.
//   objective: the per-warp partials are summed in a fixed tree by one block.
// Every sum has a fixed order that depends only on N, d and the offsets, so the result is
// the same on every run.
#include <cuda_bf16.h>

#include "fk_common.cuh"
#include "prep_row.cuh"
#include "ptx_sm100.cuh"

namespace fk {
namespace {

constexpr int kGroup = kUpdGroup;  // units of level L-1 per unit of level L
static_assert((kGroup & (kGroup - 1)) == 0, "combine spans must stay powers of two");

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

// A finished cluster: its mean into C_new (fp32), or, when sums_out is given (a shard of a
// data-parallel run), its fp64 sum into sums_out for a later combine across shards.
__device__ __forceinline__ void store_done(float *C_new, double *sums_out, int64_t k, int d,
                                          int col, const double (&acc)[4], double cnt) {
    if (sums_out) {
        double2 *q = reinterpret_cast<double2 *>(sums_out + k * d + col);
        q[0] = make_double2(acc[0], acc[1]);
        q[1] = make_double2(acc[2], acc[3]);
    } else {
        store_mean(C_new, k, d, col, acc, cnt);
    }
}

__device__ __forceinline__ void store_piece(double *dst, const double (&acc)[4]) {
    double2 *q = reinterpret_cast<double2 *>(dst);
    q[0] = make_double2(acc[0], acc[1]);
    q[1] = make_double2(acc[2], acc[3]);
}

// Level 1 for fp32 points (bf16 points use seg_rows_cp_kernel below).  A warp owns
// sorted positions [w*R, w*R + R) and the 128 columns of block blockIdx.y (lane l holds
// columns 4l .. 4l+3).  The warp first stages the R cluster ids and row ids of its chunk in
// shared memory (one coalesced read).  Rows are then gathered with 1-D bulk copies (one
// 512-byte 128-column slice of one row per lane) into a ring of kRowRing batches of B = 8
// rows in shared memory, each batch completing on its own mbarrier, so four batches are in
// flight per warp without holding any registers.  When a batch lies in one cluster its rows are
// first added pairwise in fp32 (a fixed tree) and the batch sum is added to the fp64
// accumulator once; otherwise rows are added one by one in fp64.  The objective term
// (x - c_used)^2 of a row is formed in fp32 and accumulated in fp64.
constexpr int kRowWarps = 4;       // warps per block of the level-1 kernel
constexpr int kRowBatchRows = 8;   // rows per batch (one mbarrier each)

template <bool BF16>
struct RowVec;
template <>
struct RowVec<false> {
    static constexpr int kBatch = kRowBatchRows;
    static constexpr int kSlice = 512;  // bytes of a 128-column slice
    static constexpr int kRing = 4;     // batches in flight per warp: 16 KB
    __device__ static void load(const uint8_t *p, float (&f)[4]) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        f[0] = v.x;
        f[1] = v.y;
        f[2] = v.z;
        f[3] = v.w;
    }
};
template <bool BF16>
constexpr int kRowBatchBytes = kRowBatchRows * RowVec<BF16>::kSlice;
template <bool BF16>
constexpr int kRowRing = RowVec<BF16>::kRing;
// the dynamic shared memory of a block: every warp's ring of batches
template <bool BF16>
constexpr size_t kRowSmem = size_t(kRowWarps) * kRowRing<BF16> * kRowBatchBytes<BF16>;

template <bool BF16>
__global__ void __launch_bounds__(kRowWarps * 32, 3)
    seg_rows_kernel(const void *__restrict__ X, int64_t N, int d, int R, int64_t nwarps,
                    int dcov, const int32_t *__restrict__ skeys,
                    const int32_t *__restrict__ perm,
                    const float *__restrict__ C_used, float *__restrict__ C_new,
                    double *__restrict__ sums_out, double *__restrict__ pieces,
                    int32_t *__restrict__ pkeys, double *__restrict__ jpart,
                    uint32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    using RV = RowVec<BF16>;
    constexpr int B = RV::kBatch;
    constexpr int SL = RV::kSlice;
    constexpr int kRing = kRowRing<BF16>;
    constexpr int kBatchBytes = kRowBatchBytes<BF16>;
    constexpr int E = BF16 ? 2 : 4;
    constexpr uint64_t kWaitNs = 2000000000ull;
    extern __shared__ __align__(128) uint8_t s_rows_all[];  // [warp][ring][B][SL]
    __shared__ int32_t s_key[kRowWarps][kUpdMaxRows];
    __shared__ int32_t s_row[kRowWarps][kUpdMaxRows];
    __shared__ __align__(8) uint64_t s_bar[kRowWarps][kRing];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * kRowWarps + wib;
    if (w >= nwarps) return;
    const int cb = blockIdx.y;
    const int col = cb * 128 + lane * 4;
    const bool colv = col < d;
    const int col0 = cb * 128;
    const uint32_t slice = static_cast<uint32_t>((d - col0 < 128 ? d - col0 : 128) * E);
    const int64_t p0 = w * R;
    const int n = static_cast<int>((p0 + R < N ? p0 + R : N) - p0);
    const int64_t p1 = p0 + n;
    int32_t *sk = s_key[wib];
    int32_t *si = s_row[wib];
    uint64_t *bar = s_bar[wib];
    uint8_t *rows = s_rows_all + static_cast<size_t>(wib) * kRing * kBatchBytes;
    if (lane < kRing) ptx::mbar_init(&bar[lane], 1);
    ptx::fence_mbar_init();
    for (int j = lane; j < n; j += 32) {
        sk[j] = skeys[p0 + j];
        si[j] = perm[p0 + j];
    }
    const int k_before = p0 > 0 ? skeys[p0 - 1] : -1;
    const int k_after = p1 < N ? skeys[p1] : -1;
    __syncwarp();

    const uint8_t *Xb = static_cast<const uint8_t *>(X);
    // Gather the rows of the batch starting at sorted position b into ring slot `slot`.
    auto issue = [&](int b, int slot) {
        if (b >= n) return;
        const int nb = n - b < B ? n - b : B;
        if (lane == 0) ptx::mbar_arrive_expect_tx(&bar[slot], nb * slice);
        __syncwarp();
        if (lane < nb)
            ptx::bulk_load(rows + slot * kBatchBytes + lane * SL,
                           Xb + (static_cast<int64_t>(si[b + lane]) * d + col0) * E, slice,
                           &bar[slot]);
    };

    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    float cu[4] = {0.f, 0.f, 0.f, 0.f};
    double jacc = 0.0;
    int cur = -1, first = -1, slot1 = -1, ncur = 0;
    bool ok = true;

    // A cluster is finished inside this warp unless it continues from the position before
    // p0 or into the one at p1 (positions are sorted, so only the first and the last
    // cluster can); its count is then the rows added here.
    auto finished = [&](int k) { return k != k_before && k != k_after; };
    auto flush = [&](int k) {
        if (finished(k)) {
            if (colv) store_done(C_new, sums_out, k, d, col, acc, static_cast<double>(ncur));
        } else {
            const int slot = (k == first) ? 0 : 1;
            if (slot == 1) slot1 = k;
            store_piece(pieces + (w * 2 + slot) * static_cast<int64_t>(dcov) + col, acc);
        }
    };
    auto start = [&](int k) {
        if (cur >= 0) flush(cur);
        if (cur < 0) first = k;
        cur = k;
        ncur = 0;
        acc[0] = acc[1] = acc[2] = acc[3] = 0.0;
        if (colv) {
            const float4 c = *reinterpret_cast<const float4 *>(C_used + int64_t(k) * d + col);
            cu[0] = c.x;
            cu[1] = c.y;
            cu[2] = c.z;
            cu[3] = c.w;
        }
    };

    for (int i = 0; i < kRing; ++i) issue(i * B, i);
    int it = 0;
    for (int b = 0; b < n; b += B, ++it) {
        const int slot = it % kRing;
        uint32_t got = 1;
        if (lane == 0) got = ptx::mbar_wait(&bar[slot], (it / kRing) & 1u, nullptr, kWaitNs);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
            if (lane == 0) err[0] = kErrTimeout;
            ok = false;
            break;
        }
        const uint8_t *base = rows + slot * kBatchBytes + lane * (4 * E);
        const int nb = n - b < B ? n - b : B;
        const int kf = sk[b], kl = sk[b + nb - 1];
        if (kf == kl) {
            // one cluster for the whole batch (positions are sorted by cluster id)
            if (kf != cur) start(kf);
            float xs[B][4];
            float jr[B];
#pragma unroll
            for (int j = 0; j < B; ++j) {
                if (j < nb && colv) {
                    RV::load(base + j * SL, xs[j]);
                } else {
                    xs[j][0] = xs[j][1] = xs[j][2] = xs[j][3] = 0.f;
                }
                float t = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float df = j < nb ? xs[j][e] - cu[e] : 0.f;
                    t = fmaf(df, df, t);
                }
                jr[j] = t;
            }
#pragma unroll
            for (int h = B / 2; h > 0; h >>= 1) {
#pragma unroll
                for (int j = 0; j < h; ++j) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) xs[j][e] += xs[j + h][e];
                    jr[j] += jr[j + h];
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] += static_cast<double>(xs[0][e]);
            jacc += static_cast<double>(jr[0]);
            ncur += nb;
        } else {
            for (int j = 0; j < nb; ++j) {
                const int k = sk[b + j];
                if (k != cur) start(k);
                ++ncur;
                float x[4] = {0.f, 0.f, 0.f, 0.f};
                if (colv) RV::load(base + j * SL, x);
                float t = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[e] += static_cast<double>(x[e]);
                    const float df = x[e] - cu[e];
                    t = fmaf(df, df, t);
                }
                jacc += static_cast<double>(t);
            }
        }
        ptx::fence_proxy_async_smem();  // this lane's reads of the slot precede the refill
        __syncwarp();                   // every lane has read the slot before it is refilled
        issue(b + kRing * B, slot);
    }
    if (!ok) {
        // let the (at most kRing) copies still outstanding land before the warp leaves
        for (int i2 = it; i2 < it + kRing && i2 * B < n; ++i2) {
            if (lane == 0)
                ptx::mbar_wait(&bar[i2 % kRing], (i2 / kRing) & 1u, nullptr, kWaitNs);
        }
        return;
    }
    if (cur >= 0) flush(cur);
    if (cb == 0 && lane == 0) {
        // slot 0 holds the first cluster if it was not finished here; slot 1 the last
        pkeys[w * 2 + 0] = finished(first) ? -1 : first;
        pkeys[w * 2 + 1] = slot1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) jacc += __shfl_xor_sync(0xffffffffu, jacc, o);
    if (lane == 0) jpart[static_cast<int64_t>(cb) * nwarps + w] = jacc;
}

// A lane's 8 bytes (four bf16 columns) of a row, unpacked to fp32.
template <bool BF16>
struct RegRowVec;
template <>
struct RegRowVec<true> {
    using T = uint2;
    static constexpr int kBatch = 8;
    __device__ static void unpack(const uint2 &u, float (&f)[4]) {
        f[0] = __uint_as_float(u.x << 16);
        f[1] = __uint_as_float(u.x & 0xffff0000u);
        f[2] = __uint_as_float(u.y << 16);
        f[3] = __uint_as_float(u.y & 0xffff0000u);
    }
    __device__ static uint2 zero() { return make_uint2(0u, 0u); }
};

// Level 1 for bf16 rows.  A 128-column slice of a bf16 row is only 256 bytes: one bulk copy
// per row is limited by the copy engine's request rate, and rows loaded into registers
// (two batches in flight per warp) leave too few bytes in flight.  Here every lane copies
// 16-byte pieces of the rows with cp.async into a ring of kCpStages stages of kCpRows rows
// per warp, so kCpStages - 1 stages are in flight without holding registers (measured at
// 100M rows, K = 32768: sort + update 8.14 -> 7.23 ms against the register form, the same
// bits).  Each stage is added batch by batch with the arithmetic of seg_rows_kernel.
constexpr int kCpWarps = 4;    // warps per block
constexpr int kCpRows = 16;    // rows per stage (two batches of eight)
constexpr int kCpStages = 3;   // stages per warp (4 and 6 measured slower: fewer blocks fit)
constexpr int kCpRowBytes = 256;  // a 128-column bf16 slice
constexpr size_t kCpSmem = size_t(kCpWarps) * kCpStages * kCpRows * kCpRowBytes;  // 48 KB

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_u32(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kCpWarps * 32, 4)
    seg_rows_cp_kernel(const void *__restrict__ X, int64_t N, int d, int R, int64_t nwarps,
                       int dcov, const int32_t *__restrict__ skeys,
                       const int32_t *__restrict__ perm, const float *__restrict__ C_used,
                       float *__restrict__ C_new, double *__restrict__ sums_out,
                       double *__restrict__ pieces, int32_t *__restrict__ pkeys,
                       double *__restrict__ jpart) {
    pdl_wait();
    pdl_trigger();
    using RV = RegRowVec<true>;
    using V = typename RV::T;
    constexpr int B = RV::kBatch;
    static_assert(kCpRows % B == 0, "a stage is whole batches");
    extern __shared__ __align__(128) uint8_t s_ring_all[];  // [warp][stage][row][256 B]
    __shared__ int32_t s_key[kCpWarps][kUpdMaxRows];
    __shared__ int32_t s_row[kCpWarps][kUpdMaxRows];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int64_t w = static_cast<int64_t>(blockIdx.x) * kCpWarps + wib;
    if (w >= nwarps) return;
    const int cb = blockIdx.y;
    const int col = cb * 128 + lane * 4;
    const bool colv = col < d;
    const int col0 = cb * 128;
    const int pieces16 = ((d - col0 < 128 ? d - col0 : 128) * 2) / 16;  // 16-byte pieces
    const int64_t p0 = w * R;
    const int n = static_cast<int>((p0 + R < N ? p0 + R : N) - p0);
    const int64_t p1 = p0 + n;
    int32_t *sk = s_key[wib];
    int32_t *si = s_row[wib];
    uint8_t *ring = s_ring_all + static_cast<size_t>(wib) * kCpStages * kCpRows * kCpRowBytes;
    for (int j = lane; j < n; j += 32) {
        sk[j] = skeys[p0 + j];
        si[j] = perm[p0 + j];
    }
    const int k_before = p0 > 0 ? skeys[p0 - 1] : -1;
    const int k_after = p1 < N ? skeys[p1] : -1;
    __syncwarp();

    const uint8_t *Xb = static_cast<const uint8_t *>(X);
    // copy the rows of stage g (sorted positions g * kCpRows ..) into its ring slot: lane
    // l takes pieces l, l + 32, ... of the stage's kCpRows x 16 pieces
    auto issue = [&](int g) {
        const int r0 = g * kCpRows;
        if (r0 < n) {
            uint8_t *dst = ring + (g % kCpStages) * (kCpRows * kCpRowBytes);
#pragma unroll
            for (int t = 0; t < (kCpRows * 16) / 32; ++t) {
                const int c = lane + 32 * t;
                const int r = c >> 4, pc = c & 15;
                if (r0 + r < n && pc < pieces16)
                    cp_async16(dst + r * kCpRowBytes + pc * 16,
                               Xb + (static_cast<int64_t>(si[r0 + r]) * d + col0) * 2 + pc * 16);
            }
        }
        cp_async_commit();  // an empty group past the end keeps the count uniform
    };

    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    float cu[4] = {0.f, 0.f, 0.f, 0.f};
    double jacc = 0.0;
    int cur = -1, first = -1, slot1 = -1, ncur = 0;
    auto finished = [&](int k) { return k != k_before && k != k_after; };
    auto flush = [&](int k) {
        if (finished(k)) {
            if (colv) store_done(C_new, sums_out, k, d, col, acc, static_cast<double>(ncur));
        } else {
            const int slot = (k == first) ? 0 : 1;
            if (slot == 1) slot1 = k;
            store_piece(pieces + (w * 2 + slot) * static_cast<int64_t>(dcov) + col, acc);
        }
    };
    auto start = [&](int k) {
        if (cur >= 0) flush(cur);
        if (cur < 0) first = k;
        cur = k;
        ncur = 0;
        acc[0] = acc[1] = acc[2] = acc[3] = 0.0;
        if (colv) {
            const float4 c = *reinterpret_cast<const float4 *>(C_used + int64_t(k) * d + col);
            cu[0] = c.x;
            cu[1] = c.y;
            cu[2] = c.z;
            cu[3] = c.w;
        }
    };
    // one batch of B rows starting at sorted position b, read from the ring: the same sums
    // in the same order as the register form
    auto process = [&](int b, const uint8_t *rows) {
        const int nb = n - b < B ? n - b : B;
        V buf[B];
#pragma unroll
        for (int j = 0; j < B; ++j)
            buf[j] = (j < nb && colv)
                         ? *reinterpret_cast<const V *>(rows + j * kCpRowBytes + lane * 8)
                         : RV::zero();
        const int kf = sk[b], kl = sk[b + nb - 1];
        if (kf == kl) {
            if (kf != cur) start(kf);
            float xs[B][4];
            float jr[B];
#pragma unroll
            for (int j = 0; j < B; ++j) {
                RV::unpack(buf[j], xs[j]);
                float t = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float df = j < nb ? xs[j][e] - cu[e] : 0.f;
                    t = fmaf(df, df, t);
                }
                jr[j] = t;
            }
#pragma unroll
            for (int h = B / 2; h > 0; h >>= 1) {
#pragma unroll
                for (int j = 0; j < h; ++j) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) xs[j][e] += xs[j + h][e];
                    jr[j] += jr[j + h];
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] += static_cast<double>(xs[0][e]);
            jacc += static_cast<double>(jr[0]);
            ncur += nb;
        } else {
#pragma unroll
            for (int j = 0; j < B; ++j) {
                if (j < nb) {
                    const int k = sk[b + j];
                    if (k != cur) start(k);
                    ++ncur;
                    float x[4];
                    RV::unpack(buf[j], x);
                    float t = 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[e] += static_cast<double>(x[e]);
                        const float df = x[e] - cu[e];
                        t = fmaf(df, df, t);
                    }
                    jacc += static_cast<double>(t);
                }
            }
        }
    };

    const int nstages = (n + kCpRows - 1) / kCpRows;
#pragma unroll
    for (int g = 0; g < kCpStages - 1; ++g) issue(g);
    for (int g = 0; g < nstages; ++g) {
        issue(g + kCpStages - 1);     // into the slot processed one step ago
        cp_async_wait<kCpStages - 1>();  // this lane's copies of stage g have landed
        __syncwarp();                    // and every other lane's
        const uint8_t *st = ring + (g % kCpStages) * (kCpRows * kCpRowBytes);
#pragma unroll
        for (int h = 0; h < kCpRows / B; ++h) {
            const int b = g * kCpRows + h * B;
            if (b < n) process(b, st + h * B * kCpRowBytes);
        }
        __syncwarp();  // the slot is read by every lane before it is refilled
    }
    cp_async_wait<0>();
    if (cur >= 0) flush(cur);
    if (cb == 0 && lane == 0) {
        pkeys[w * 2 + 0] = finished(first) ? -1 : first;
        pkeys[w * 2 + 1] = slot1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) jacc += __shfl_xor_sync(0xffffffffu, jacc, o);
    if (lane == 0) jpart[static_cast<int64_t>(cb) * nwarps + w] = jacc;
}

// Level L >= 2: one warp per group of kGroup units of the previous level (2 piece slots
// each), one 128-column block per grid.y.  `span` = sorted positions covered by one unit
// of THIS level.  The group's slot keys are staged in shared memory first and the pieces
// are read 8 slots at a time, so the loop is not a chain of dependent loads.  The CSR
// bounds of every slot's cluster are staged with the keys, so finishing a cluster waits on
// no global load.
// One warp: unit u of a combine level, column block cb; sk = the warp's shared key slots,
// sb = their clusters' [lo, hi) sorted positions.
__device__ __forceinline__ void pieces_unit(const double *__restrict__ pin,
                                            const int32_t *__restrict__ kin, int64_t nslots_in,
                                            double *__restrict__ pout,
                                            int32_t *__restrict__ kout, int64_t u, int cb,
                                            int64_t span, int d, int dcov,
                                            const int32_t *__restrict__ offsets,
                                            float *__restrict__ C_new,
                                            double *__restrict__ sums_out, int32_t *sk,
                                            int2 *sb) {
    constexpr int S = 2 * kGroup;
    constexpr int B = 8;
    // span is a power of two (a power-of-two row count times powers of kGroup), so the
    // "same unit" test below is a shift rather than a 64-bit division
    const int span_log2 = __ffsll(static_cast<long long>(span)) - 1;
    const int lane = threadIdx.x & 31;
    const int col = cb * 128 + lane * 4;
    const int64_t s0 = u * S;
    const int ns = static_cast<int>((s0 + S < nslots_in ? s0 + S : nslots_in) - s0);
    for (int j = lane; j < ns; j += 32) {
        const int k = kin[s0 + j];
        sk[j] = k;
        if (k >= 0) sb[j] = make_int2(offsets[k], offsets[k + 1]);
    }
    __syncwarp();

    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    int cur = -1, curq = -1, first = -1, slot1 = -1;
    bool first_done = false;

    auto flush = [&](int k) {
        const int64_t lo = sb[curq].x, hi = sb[curq].y;
        const bool done = (lo >> span_log2) == ((hi - 1) >> span_log2);
        if (k == first) first_done = done;
        if (done) {
            if (col < d) store_done(C_new, sums_out, k, d, col, acc, static_cast<double>(hi - lo));
        } else {
            const int slot = (k == first) ? 0 : 1;
            if (slot == 1) slot1 = k;
            store_piece(pout + (u * 2 + slot) * static_cast<int64_t>(dcov) + col, acc);
        }
    };

    for (int b = 0; b < ns; b += B) {
        double2 va[B], vb[B];
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int q = b + j;
            if (q < ns && sk[q] >= 0) {
                const double2 *src =
                    reinterpret_cast<const double2 *>(pin + (s0 + q) * int64_t(dcov) + col);
                va[j] = src[0];
                vb[j] = src[1];
            } else {
                va[j] = vb[j] = make_double2(0.0, 0.0);
            }
        }
#pragma unroll
        for (int j = 0; j < B; ++j) {
            const int q = b + j;
            if (q >= ns) break;
            const int k = sk[q];
            if (k < 0) continue;
            if (k != cur) {
                if (cur >= 0) flush(cur);
                if (cur < 0) first = k;
                cur = k;
                curq = q;
                acc[0] = acc[1] = acc[2] = acc[3] = 0.0;
            }
            acc[0] += va[j].x;
            acc[1] += va[j].y;
            acc[2] += vb[j].x;
            acc[3] += vb[j].y;
        }
    }
    if (cur >= 0) flush(cur);
    if (cb == 0 && lane == 0) {
        kout[u * 2 + 0] = (first >= 0 && !first_done) ? first : -1;
        kout[u * 2 + 1] = slot1;
    }
}

__global__ void __launch_bounds__(kUpdWarps * 32)
    seg_pieces_kernel(const double *__restrict__ pin, const int32_t *__restrict__ kin,
                      int64_t nslots_in, double *__restrict__ pout,
                      int32_t *__restrict__ kout, int64_t nunits, int64_t span, int d,
                      int dcov, const int32_t *__restrict__ offsets, float *__restrict__ C_new,
                      double *__restrict__ sums_out) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t s_key[kUpdWarps][2 * kGroup];
    __shared__ int2 s_bnd[kUpdWarps][2 * kGroup];
    const int wib = threadIdx.x >> 5;
    const int64_t u = static_cast<int64_t>(blockIdx.x) * kUpdWarps + wib;
    if (u >= nunits) return;
    pieces_unit(pin, kin, nslots_in, pout, kout, u, blockIdx.y, span, d, dcov, offsets, C_new,
                sums_out, s_key[wib], s_bnd[wib]);
}

// Combine W shards of a data-parallel iteration, in shard order: c_k = (sum_w S_wk) /
// (sum_w n_wk) in fp64, rounded once to fp32, or C_old[k] bit for bit when no shard holds
// a point of cluster k; counts[k] = sum_w n_wk; *objective = sum_w J_w (shard order).
__global__ void finalize_shards_kernel(const double *__restrict__ sums,
                                       const int64_t *__restrict__ cnts,
                                       const double *__restrict__ objs, int W, int K, int d,
                                       const float *__restrict__ C_old, float *__restrict__ C_new,
                                       int64_t *__restrict__ counts,
                                       double *__restrict__ objective) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    if (warp == 0 && lane == 0 && objective) {
        double j = 0.0;
        for (int w = 0; w < W; ++w) j += objs[w];
        *objective = j;
    }
    const int64_t KD = static_cast<int64_t>(K) * d;
    for (int64_t k = warp; k < K; k += nw) {
        int64_t c = 0;
        for (int w = 0; w < W; ++w) c += cnts[w * static_cast<int64_t>(K) + k];
        if (lane == 0 && counts) counts[k] = c;
        for (int j = lane; j < d; j += 32) {
            if (c == 0) {
                C_new[k * d + j] = C_old[k * d + j];
            } else {
                double acc = 0.0;
                for (int w = 0; w < W; ++w) acc += sums[w * KD + k * d + j];
                C_new[k * d + j] = static_cast<float>(acc / static_cast<double>(c));
            }
        }
    }
}

// The objective partials summed in a fixed order by one block of 256 threads: thread t
// adds entries t, t + 256, ... in index order (eight loads are issued before the eight
// additions, so the loop is not a chain of dependent loads), then a fixed tree over the
// threads.  sh: 256 doubles of shared memory.
__device__ __forceinline__ void sum_objective(const double *__restrict__ part, int64_t n,
                                              double *__restrict__ objective, double *sh) {
    double s = 0.0;
    int64_t i = threadIdx.x;
    for (; i + 7 * 256 < n; i += 8 * 256) {
        double v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = part[i + j * 256];
#pragma unroll
        for (int j = 0; j < 8; ++j) s += v[j];
    }
    for (; i < n; i += 256) s += part[i];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *objective = sh[0];
}

// The update's tail steps in one launch.  Block 0 sums the n objective partials (thread t
// adds t, t + 256, ... in order, then a fixed tree).  Blocks 1 .. nfin run the last combine
// level (one unit; warp 0 of block 1 + cb handles column block cb).  The other blocks
// finalize: counts[k] = offsets[k+1] - offsets[k], an empty cluster keeps C_old bit for
// bit (or, for a shard's partial sums, gets a zero sum).  The combine writes only clusters
// that hold points and the finalize only empty ones, so the blocks touch disjoint rows.
__global__ void __launch_bounds__(256)
    finalize_objective_kernel(const int32_t *__restrict__ offsets, int K, int d,
                              const float *__restrict__ C_old, float *__restrict__ C_new,
                              int32_t *__restrict__ counts, double *__restrict__ sums_out,
                              const double *__restrict__ part, int64_t n,
                              double *__restrict__ objective, int nfin,
                              const double *__restrict__ pin, const int32_t *__restrict__ kin,
                              int64_t nslots, double *__restrict__ pout,
                              int32_t *__restrict__ kout, int64_t span, int dcov) {
    pdl_wait();
    pdl_trigger();
    if (blockIdx.x == 0) {
        if (objective == nullptr) return;
        __shared__ double sh[256];
        sum_objective(part, n, objective, sh);
        return;
    }
    if (static_cast<int>(blockIdx.x) <= nfin) {
        __shared__ int32_t s_key[2 * kGroup];
        __shared__ int2 s_bnd[2 * kGroup];
        if (threadIdx.x < 32)
            pieces_unit(pin, kin, nslots, pout, kout, 0, static_cast<int>(blockIdx.x) - 1, span,
                        d, dcov, offsets, C_new, sums_out, s_key, s_bnd);
        return;
    }
    const int lane = threadIdx.x & 31;
    const int64_t warp =
        (static_cast<int64_t>(blockIdx.x - 1 - nfin) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x - 1 - nfin) * blockDim.x) >> 5;
    for (int64_t k = warp; k < K; k += nw) {
        const int32_t c = offsets[k + 1] - offsets[k];
        if (lane == 0 && counts) counts[k] = c;
        if (c == 0) {
            if (sums_out)
                for (int j = lane; j < d; j += 32) sums_out[k * d + j] = 0.0;
            else
                for (int j = lane; j < d; j += 32) C_new[k * d + j] = C_old[k * d + j];
        }
    }
}

// Every combine level of a small problem (at most kUpdWideUnits level-1 units) in one
// launch.  A block evaluates, for one cluster at a time and one column block, the cluster's
// share of every combine level: the sums it forms are those of seg_pieces_kernel and of the
// tail's last level (the same pieces added in the same order, kGroup units of one level to
// a unit of the next), so the centroids are bit for bit those of the level-by-level
// launches; only the chain of dependent launches is gone.  A cluster's units are
// consecutive, so its level-2 partials number at most l2cap = (units - 1) / kGroup + 1 and
// fit in shared memory; higher levels use a second buffer of l2cap / kGroup + 2 entries.
// The last block sums the objective.  counts[k] comes from the offsets, and an empty
// cluster keeps C_old bit for bit (a zero sum for a shard).
constexpr int kWideWarps = 8;
static_assert(kWideWarps * 32 == 256, "sum_objective runs on 256 threads");


__global__ void __launch_bounds__(kWideWarps * 32)
    wide_combine_kernel(const double *__restrict__ pieces, int rows_log2, int l2cap, int K,
                        int d, int dcov, const int32_t *__restrict__ offsets,
                        const float *__restrict__ C_old, float *__restrict__ C_new,
                        double *__restrict__ sums_out, int32_t *__restrict__ counts,
                        const double *__restrict__ jpart, int64_t njpart,
                        double *__restrict__ objective, CentroidOperands next) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ __align__(16) double s_part[];  // [l2cap][128], then [l3cap][128]
    __shared__ double s_obj[256];
    const int cb = blockIdx.y;
    if (blockIdx.x == gridDim.x - 1) {
        if (cb == 0 && objective) sum_objective(jpart, njpart, objective, s_obj);
        return;
    }
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int col = cb * 128 + lane * 4;
    const bool colv = col < d;
    const int cend = d < cb * 128 + 128 ? d : cb * 128 + 128;
    const int64_t R = int64_t(1) << rows_log2;
    const int stride = static_cast<int>(gridDim.x) - 1;
    for (int k = blockIdx.x; k < K; k += stride) {
        const int64_t lo = offsets[k], hi = offsets[k + 1];
        if (cb == 0 && tid == 0 && counts) counts[k] = static_cast<int32_t>(hi - lo);
        int64_t a0 = lo >> rows_log2, a1 = (hi - 1) >> rows_log2;  // units of the level below
        if (hi == lo) {
            for (int j = cb * 128 + tid; j < cend; j += kWideWarps * 32) {
                if (sums_out)
                    sums_out[int64_t(k) * d + j] = 0.0;
                else
                    C_new[int64_t(k) * d + j] = C_old[int64_t(k) * d + j];
            }
            a1 = a0;  // no combine
        }
        const double *src = nullptr;  // the level below in shared memory (level 1: pieces)
        double *dst = s_part;
        while (a0 != a1) {  // a0 == a1: finished by the level-1 kernel (or empty)
            const int64_t g0 = a0 / kGroup, g1 = a1 / kGroup;
            const bool done = g0 == g1;  // the cluster lies in one unit of this level
            for (int64_t g = g0 + warp; g <= g1; g += kWideWarps) {
                const int64_t ia = a0 > g * kGroup ? a0 : g * kGroup;
                const int64_t ib = a1 < g * kGroup + kGroup - 1 ? a1 : g * kGroup + kGroup - 1;
                double acc[4] = {0.0, 0.0, 0.0, 0.0};
                for (int64_t b = ia; b <= ib; b += 8) {
                    double2 va[8], vb[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int64_t i = b + j;
                        va[j] = vb[j] = make_double2(0.0, 0.0);
                        if (i <= ib && colv) {
                            const double *q;
                            if (src == nullptr)  // a level-1 unit: slot 0 when the cluster
                                                 // holds the unit's first position
                                q = pieces + (i * 2 + (lo <= i * R ? 0 : 1)) * int64_t(dcov) + col;
                            else
                                q = src + (i - a0) * 128 + lane * 4;
                            va[j] = reinterpret_cast<const double2 *>(q)[0];
                            vb[j] = reinterpret_cast<const double2 *>(q)[1];
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (b + j > ib) break;
                        acc[0] += va[j].x;
                        acc[1] += va[j].y;
                        acc[2] += vb[j].x;
                        acc[3] += vb[j].y;
                    }
                }
                if (done) {
                    if (colv)
                        store_done(C_new, sums_out, k, d, col, acc, static_cast<double>(hi - lo));
                } else {
                    double2 *o = reinterpret_cast<double2 *>(dst + (g - g0) * 128 + lane * 4);
                    o[0] = make_double2(acc[0], acc[1]);
                    o[1] = make_double2(acc[2], acc[3]);
                }
            }
            __syncthreads();  // this level's partials are written before the next reads them
            if (done) break;
            a0 = g0;
            a1 = g1;
            src = dst;
            dst = dst == s_part ? s_part + l2cap * 128 : s_part;
        }
        if (next.planes != nullptr) {
            // row k of C_new is final (written by the level-1 kernel, or by this block
            // before the barrier): its operands for the next iteration's assignment
            __syncthreads();
            if (warp == 0) prep_centroid_row(C_new, K, d, next, k, lane);
        }
    }
}

// The last combine level (a single unit), left for the update's tail launch.
struct FinalLevel {
    bool pending = false;
    const double *pin = nullptr;
    const int32_t *kin = nullptr;
    int64_t nslots = 0;
    double *pout = nullptr;
    int32_t *kout = nullptr;
    int64_t span = 0;
};

cudaError_t run_levels(const void *X, bool bf16, int64_t N, int d, const UpdPlan &up,
                       const int32_t *skeys, const int32_t *perm, const int32_t *offsets,
                       const float *C_used, float *C_new, double *sums_out, double *pa,
                       int32_t *ka,
                       double *pb, int32_t *kb, double *jpart, uint32_t *err,
                       cudaStream_t st, FinalLevel *final_level, bool level1_only) {
    static std::atomic<uint64_t> smem_set{0};
    {
        const cudaError_t e =
            smem_opt_in(seg_rows_kernel<false>, static_cast<int>(kRowSmem<false>), smem_set);
        if (e != cudaSuccess) return e;
    }
    const dim3 rblock(kRowWarps * 32);
    dim3 rgrid(static_cast<unsigned>(ceil_div(up.nwarps, kRowWarps)), up.ncolblk);
    static std::atomic<uint64_t> smem_set_cp{0};
    {
        const cudaError_t e =
            smem_opt_in(seg_rows_cp_kernel, static_cast<int>(kCpSmem), smem_set_cp);
        if (e != cudaSuccess) return e;
    }
    if (bf16)
        launch_pdl(seg_rows_cp_kernel,
                   dim3(static_cast<unsigned>(ceil_div(up.nwarps, kCpWarps)), up.ncolblk),
                   dim3(kCpWarps * 32), kCpSmem, st, X, N, d, up.rows, up.nwarps, up.dcov, skeys,
                   perm, C_used, C_new, sums_out, pa, ka, jpart);
    else
        launch_pdl(seg_rows_kernel<false>, rgrid, rblock, kRowSmem<false>, st, X, N, d, up.rows,
                   up.nwarps, up.dcov, skeys, perm, C_used, C_new, sums_out, pa, ka, jpart,
                   err);
    note_launch();
    const dim3 block(kUpdWarps * 32);
    int64_t units = up.nwarps;
    int64_t span = up.rows;
    double *pin = pa, *pout = pb;
    int32_t *kin = ka, *kout = kb;
    while (units > 1 && !level1_only) {
        const int64_t nunits = ceil_div(units, kGroup);
        span *= kGroup;
        if (nunits == 1) {  // the last level runs inside the tail launch
            final_level->pending = true;
            final_level->pin = pin;
            final_level->kin = kin;
            final_level->nslots = units * 2;
            final_level->pout = pout;
            final_level->kout = kout;
            final_level->span = span;
            break;
        }
        dim3 g2(static_cast<unsigned>(ceil_div(nunits, kUpdWarps)), up.ncolblk);
        launch_pdl(seg_pieces_kernel, g2, block, 0, st, pin, kin, units * 2, pout, kout, nunits,
                   span, d, up.dcov, offsets, C_new, sums_out);
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
                          double *objective, uint32_t *err, double *sums_out,
                          cudaStream_t st, const CentroidOperands *next, bool *prepped) {
    const bool bf16 = dtype == FK_BF16;
    if (prepped) *prepped = false;
    FinalLevel fl;
    const bool wide = up.nwarps <= kUpdWideUnits && K <= kUpdWideMaxK;
    cudaError_t e = run_levels(X, bf16, N, d, up, skeys, perm, offsets, C_used, C_new,
                               sums_out, pieces_a, pkeys_a, pieces_b, pkeys_b, jpart, err, st,
                               &fl, wide);
    if (e != cudaSuccess) return e;
    if (wide) {
        // a small problem: every combine level, the finalize and the objective in one launch
        static std::atomic<uint64_t> smem_set{0};
        if ((e = smem_opt_in(wide_combine_kernel, static_cast<int>(upd_wide_smem(kUpdWideUnits)),
                             smem_set)) != cudaSuccess)
            return e;
        int rows_log2 = 0;
        while ((1 << rows_log2) < up.rows) ++rows_log2;  // rows is a power of two
        const size_t smem = upd_wide_smem(up.nwarps);
        // one column block: a block owns whole rows and can prepare the next operands
        const bool fuse = next != nullptr && sums_out == nullptr && up.ncolblk == 1;
        // blocks that fit on an SM at once (228 KB of shared memory, 1 KB reserved and
        // 2 KB static per block), so the cluster loop runs in one wave
        const int64_t fit = static_cast<int64_t>((228u << 10) / (smem + (3u << 10)));
        int64_t blocks = K;
        const int64_t cap = static_cast<int64_t>(device_sm_count()) * (fit < 1 ? 1 : fit);
        if (blocks > cap) blocks = cap;
        launch_pdl(wide_combine_kernel, dim3(static_cast<unsigned>(blocks + 1), up.ncolblk),
                   dim3(kWideWarps * 32), smem, st, pieces_a, rows_log2,
                   upd_wide_l2cap(up.nwarps), K, d,
                   up.dcov, offsets, C_old, C_new, sums_out, counts, jpart,
                   up.nwarps * up.ncolblk, objective, fuse ? *next : CentroidOperands{});
        note_launch();
        if ((e = cudaGetLastError()) == cudaSuccess && prepped) *prepped = fuse;
        return e;
    }
    // the update's tail in one launch: the objective (block 0), the last combine level (one
    // block per 128-column block) and the empty clusters (the remaining blocks)
    int64_t fgrid = ceil_div(K, 8);
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (fgrid > cap) fgrid = cap;
    const int nfin = fl.pending ? up.ncolblk : 0;
    launch_pdl(finalize_objective_kernel, dim3(static_cast<unsigned>(1 + nfin + fgrid)),
               dim3(256), 0, st, offsets, K, d, C_old, C_new, counts, sums_out, jpart,
               up.nwarps * up.ncolblk, objective, nfin, fl.pin, fl.kin, fl.nslots, fl.pout,
               fl.kout, fl.span, up.dcov);
    note_launch();
    return cudaGetLastError();
}

namespace {

// Running totals of a streamed iteration: tot += one chunk's sums, counts and objective
// (the chunks are added in their order, so the totals do not depend on scheduling).
__global__ void accumulate_chunk_kernel(double *__restrict__ tot, const double *__restrict__ part,
                                        int64_t KD, int64_t *__restrict__ cnt_tot,
                                        const int32_t *__restrict__ cnt, int K,
                                        double *__restrict__ obj_tot,
                                        const double *__restrict__ obj) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int64_t i = t0; i < KD; i += stride) tot[i] += part[i];
    for (int64_t k = t0; k < K; k += stride) cnt_tot[k] += cnt[k];
    if (t0 == 0) *obj_tot += *obj;
}

}  // namespace

cudaError_t launch_accumulate_chunk(double *tot, const double *part, int64_t KD,
                                    int64_t *cnt_tot, const int32_t *cnt, int K,
                                    double *obj_tot, const double *obj, cudaStream_t st) {
    int64_t g = ceil_div(KD, 256);
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
    if (g > cap) g = cap;
    accumulate_chunk_kernel<<<static_cast<unsigned>(g < 1 ? 1 : g), 256, 0, st>>>(
        tot, part, KD, cnt_tot, cnt, K, obj_tot, obj);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_finalize_shards(const double *sums, const int64_t *cnts, const double *objs,
                                   int W, int K, int d, const float *C_old, float *C_new,
                                   int64_t *counts, double *objective, cudaStream_t st) {
    int64_t g = ceil_div(K, 8);
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (g > cap) g = cap;
    finalize_shards_kernel<<<static_cast<unsigned>(g < 1 ? 1 : g), 256, 0, st>>>(
        sums, cnts, objs, W, K, d, C_old, C_new, counts, objective);
    note_launch();
    return cudaGetLastError();
}

namespace {
// Empty clusters and the largest cluster of a count array (one block).
__global__ void cluster_stats_kernel(const int32_t *__restrict__ counts, int K,
                                     uint32_t *__restrict__ out) {
    __shared__ uint32_t e_red[32], m_red[32];
    uint32_t empty = 0, mx = 0;
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const uint32_t c = static_cast<uint32_t>(counts[k]);
        empty += c == 0u;
        mx = c > mx ? c : mx;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        empty += __shfl_xor_sync(0xffffffffu, empty, o);
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if ((threadIdx.x & 31) == 0) {
        e_red[threadIdx.x >> 5] = empty;
        m_red[threadIdx.x >> 5] = mx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) {
            empty += e_red[w];
            mx = max(mx, m_red[w]);
        }
        out[0] = empty;
        out[1] = mx;
    }
}
}  // namespace

cudaError_t launch_cluster_stats(const int32_t *counts, int K, uint32_t *out, cudaStream_t st) {
    cluster_stats_kernel<<<1, 1024, 0, st>>>(counts, K, out);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk
