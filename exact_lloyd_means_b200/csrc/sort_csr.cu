// sort_csr.cu -- labels -> sorted inverse index (perm) + CSR cluster offsets.
//
// Flash-KMeans article, section "Sort-Inverse Update：原子操作的另一种解法": the
// assignments are sorted by cluster id into an inverse index so that each cluster's
// points can be read contiguously; LEANN FlashLib guide, section "工作原理": the coarse
// quantizer's output is CSR offsets plus cell-ordered row ids.
//
// A stable least-significant-digit radix sort with digits of up to 8 bits (one pass for
// K <= 256, two for K <= 65536, three beyond), whose ranks need no atomics:
//   upsweep   : each block of 2048 keys (1024 when the input has at most 4M keys, so that
//               small sorts run on twice the blocks) counts its digits into per-warp
//               histograms in shared memory (shared-memory atomic adds: the counts do not
//               depend on their order);
//   scan      : one block per digit scans the per-block counts (digit-major order) and
//               stores the digit total;
//   downsweep : each lane loads its keys once and ranks each among the equal digits of its
//               warp (peers from one ballot per digit bit, rank = earlier peers + the
//               warp's running count); the warps' counts give each warp's base per digit
//               (digits in order, then warps in order), every key goes to shared memory at
//               base + rank, and each digit's run of the tile is written to its global
//               place (digits, then blocks in order) with consecutive threads on
//               consecutive addresses.  Ranks follow the index order, so the sort is
//               stable and the output is unique.
// offsets[k] = first sorted position whose key is >= k, written once per k: by the first
// downsweep tile for a one-pass sort (the digit bases are the offsets), else by a kernel of
// its own after the last pass.
#include "fk_common.cuh"

namespace fk {
namespace {

constexpr int kWarps = kSortThreads / 32;

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Check labels (first pass) and count digits of one tile of kSortThreads * ITEMS keys
// into per-warp histograms wh[kWarps][bins].  Each thread reads ITEMS consecutive keys
// with 16-byte loads and adds them with shared-memory atomics: counts do not depend on the
// order of the additions, so the result is the same on every run.
template <int ITEMS>
__device__ __forceinline__ void count_tile(const int32_t *__restrict__ keys, int64_t n,
                                           int64_t tile0, int shift, uint32_t mask, int K,
                                           uint32_t *__restrict__ err, int check,
                                           uint32_t *wh, int bins) {
    const int warp = threadIdx.x >> 5;
    uint32_t *h = wh + warp * bins;
    const int64_t start = tile0 + static_cast<int64_t>(threadIdx.x) * ITEMS;
    // labels need only 4-byte alignment: 16-byte loads only from a 16-byte aligned array
    // (start is a multiple of 4 keys, so then every load below is aligned)
    const bool vec = (reinterpret_cast<uintptr_t>(keys) & 15u) == 0u;
#pragma unroll
    for (int j = 0; j < ITEMS; j += 4) {
        const int64_t idx = start + j;
        int k4[4];
        if (vec && idx + 3 < n) {
            const int4 v = *reinterpret_cast<const int4 *>(keys + idx);
            k4[0] = v.x;
            k4[1] = v.y;
            k4[2] = v.z;
            k4[3] = v.w;
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) k4[t] = idx + t < n ? keys[idx + t] : -1;
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            if (idx + t >= n) continue;
            int key = k4[t];
            if (key < 0 || key >= K) {
                if (check) err[1] = 1u;
                key = key < 0 ? 0 : K - 1;
            }
            atomicAdd(&h[(static_cast<uint32_t>(key) >> shift) & mask], 1u);
        }
    }
}

template <int ITEMS>
__global__ void __launch_bounds__(kSortThreads)
    upsweep_kernel(const int32_t *__restrict__ keys, int64_t n, int shift, int bits, int K,
                   uint32_t *__restrict__ hist, int64_t nblocks, uint32_t *__restrict__ err,
                   int check) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t wh[];
    const int bins = 1 << bits;
    for (int i = threadIdx.x; i < kWarps * bins; i += blockDim.x) wh[i] = 0;
    __syncthreads();
    count_tile<ITEMS>(keys, n, static_cast<int64_t>(blockIdx.x) * (kSortThreads * ITEMS), shift,
                      bins - 1, K, err,
               check, wh, bins);
    __syncthreads();
    for (int b = threadIdx.x; b < bins; b += blockDim.x) {
        uint32_t t = 0;
        for (int w = 0; w < kWarps; ++w) t += wh[w * bins + b];
        hist[static_cast<int64_t>(b) * nblocks + blockIdx.x] = t;
    }
}

// Exclusive scan of 1024 per-thread values held in registers; returns the exclusive
// prefix of this thread and writes the block total to *total.
__device__ __forceinline__ uint32_t block_exclusive_scan_1024(uint32_t v, uint32_t *sh,
                                                              uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < (blockDim.x >> 5) ? sh[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        sh[32 + lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const uint32_t warp_base = warp == 0 ? 0 : sh[32 + warp - 1];
    *total = sh[32 + (blockDim.x >> 5) - 1];
    return warp_base + x - v;
}

// One block (1024 threads) per digit: exclusive scan of hist[b][0..nblocks).
__global__ void __launch_bounds__(1024)
    scan_rows_kernel(uint32_t *__restrict__ hist, int64_t nblocks, uint32_t *__restrict__ dtot) {
    pdl_wait();
    pdl_trigger();
    __shared__ uint32_t sh[64];
    uint32_t *row = hist + static_cast<int64_t>(blockIdx.x) * nblocks;
    const int64_t per = (nblocks + blockDim.x - 1) / blockDim.x;
    const int64_t lo = threadIdx.x * per;
    const int64_t hi = lo + per < nblocks ? lo + per : nblocks;
    uint32_t s = 0;
    for (int64_t i = lo; i < hi; ++i) s += row[i];
    uint32_t total;
    uint32_t run = block_exclusive_scan_1024(s, sh, &total);
    for (int64_t i = lo; i < hi; ++i) {
        const uint32_t t = row[i];
        row[i] = run;
        run += t;
    }
    if (threadIdx.x == 0) dtot[blockIdx.x] = total;
}

// Exclusive scan of cnt[0..bins) into out[0..bins) by one block: every thread sums a
// contiguous run of entries, the run totals are scanned with warp shuffles (each warp,
// then the eight warp totals), then the runs are filled in.
__device__ __forceinline__ void block_scan_bins(const uint32_t *cnt, uint32_t *out, int bins,
                                                uint32_t *part) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (bins + kSortThreads - 1) / kSortThreads;
    const int lo = threadIdx.x * per;
    const int hi = lo + per < bins ? lo + per : bins;
    uint32_t s = 0;
    for (int b = lo; b < hi; ++b) s += cnt[b];
    uint32_t x = s;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) part[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t t = lane < kWarps ? part[lane] : 0u;
#pragma unroll
        for (int o = 1; o < kWarps; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kWarps) part[kWarps + lane] = t;  // inclusive warp totals
    }
    __syncthreads();
    uint32_t run = (warp == 0 ? 0u : part[kWarps + warp - 1]) + x - s;
    for (int b = lo; b < hi; ++b) {
        const uint32_t v = cnt[b];
        out[b] = run;
        run += v;
    }
    __syncthreads();
}

// Scatter one tile of kSortThreads * ITEMS keys.  Every lane holds ITEMS keys (positions
// base + 32*step + lane of its warp's stretch) and ranks each among the keys of equal digit
// in its warp, in position order: the peers come from one ballot per digit bit, the rank
// is the count of earlier peers plus the warp's running count of that digit.  The warps'
// digit counts then give each warp's base per digit (digits in order, then warps in
// order), the keys are placed in shared memory at base + rank, and each digit's run is
// written to its global place with consecutive threads on consecutive addresses.  Ranks
// follow the index order, so the sort is stable and its output unique.
template <int ITEMS>
__global__ void __launch_bounds__(kSortThreads)
    downsweep_kernel(const int32_t *__restrict__ kin, const int32_t *__restrict__ vin,
                     int32_t *__restrict__ kout, int32_t *__restrict__ vout, int64_t n64,
                     int shift, int bits, int K, const uint32_t *__restrict__ hist,
                     const uint32_t *__restrict__ dtot, int64_t nblocks,
                     int32_t *__restrict__ offsets) {
    pdl_wait();
    pdl_trigger();
    constexpr int kTile = kSortThreads * ITEMS;
    extern __shared__ uint32_t sm[];
    const int bins = 1 << bits;
    const uint32_t mask = bins - 1;
    uint32_t *wh = sm;                      // [kWarps][bins] digit counts, then warp bases
    uint32_t *lstart = wh + kWarps * bins;  // [bins] this tile's digit starts (local)
    uint32_t *gofs = lstart + bins;         // [bins] global start minus local start
    uint32_t *bcnt = gofs + bins;           // [bins] scratch
    int32_t *skey = reinterpret_cast<int32_t *>(bcnt + bins);  // [kTile]
    int32_t *sval = skey + kTile;                               // [kTile]
    __shared__ uint32_t part[kSortThreads];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the callers bound n below 2^31, so positions (and a last tile running past n) fit
    // in 32 unsigned bits
    const uint32_t n = static_cast<uint32_t>(n64);
    const uint32_t tile0 = blockIdx.x * static_cast<uint32_t>(kTile);
    const uint32_t base = tile0 + static_cast<uint32_t>(warp * (32 * ITEMS));

    // this lane's keys and values, loaded up front (-1 marks a position past n)
    int key[ITEMS], val[ITEMS];
#pragma unroll
    for (int step = 0; step < ITEMS; ++step) {
        const uint32_t idx = base + static_cast<uint32_t>(step * 32 + lane);
        key[step] = -1;
        val[step] = 0;
        if (idx < n) {
            const int k = kin[idx];
            key[step] = k < 0 ? 0 : (k >= K ? K - 1 : k);
            val[step] = vin ? vin[idx] : static_cast<int32_t>(idx);
        }
    }

    for (int i = threadIdx.x; i < kWarps * bins; i += blockDim.x) wh[i] = 0;
    // global digit bases: exclusive scan of the digit totals (its barriers also order the
    // zeroing above before the counting below)
    block_scan_bins(dtot, gofs, bins, part);
    for (int b = threadIdx.x; b < bins; b += blockDim.x) {
        // a one-pass sort's digit is the whole key: the CSR offsets are the digit bases,
        // written by the first tile
        if (offsets && blockIdx.x == 0 && b < K) offsets[b] = static_cast<int32_t>(gofs[b]);
        gofs[b] += hist[static_cast<int64_t>(b) * nblocks + blockIdx.x];
    }
    if (offsets && blockIdx.x == 0 && threadIdx.x == 0) offsets[K] = static_cast<int32_t>(n);

    uint32_t *h = wh + warp * bins;
    const uint32_t lt = lanemask_lt();
    uint32_t rank[ITEMS];
#pragma unroll
    for (int step = 0; step < ITEMS; ++step) {
        const bool valid = key[step] >= 0;
        const uint32_t digit = (static_cast<uint32_t>(key[step]) >> shift) & mask;
        uint32_t peers = __ballot_sync(0xffffffffu, valid);
        for (int b = 0; b < bits; ++b) {
            const bool on = (digit >> b) & 1u;
            const uint32_t bal = __ballot_sync(0xffffffffu, on);
            peers &= on ? bal : ~bal;
        }
        uint32_t r = 0;
        if (valid) r = h[digit] + __popc(peers & lt);
        __syncwarp();
        if (valid && lane == __ffs(peers) - 1) h[digit] += __popc(peers);
        __syncwarp();
        rank[step] = r;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < bins; b += blockDim.x) {
        uint32_t t = 0;
        for (int w = 0; w < kWarps; ++w) t += wh[w * bins + b];
        bcnt[b] = t;
    }
    __syncthreads();
    block_scan_bins(bcnt, lstart, bins, part);
    for (int b = threadIdx.x; b < bins; b += blockDim.x) {
        uint32_t run = lstart[b];
        for (int w = 0; w < kWarps; ++w) {
            const uint32_t t = wh[w * bins + b];
            wh[w * bins + b] = run;
            run += t;
        }
        gofs[b] -= lstart[b];  // modulo 2^32: gofs + local position is the global one
    }
    __syncthreads();
#pragma unroll
    for (int step = 0; step < ITEMS; ++step) {
        if (key[step] >= 0) {
            const uint32_t digit = (static_cast<uint32_t>(key[step]) >> shift) & mask;
            const uint32_t pos = h[digit] + rank[step];
            skey[pos] = key[step];
            sval[pos] = val[step];
        }
    }
    __syncthreads();

    // a plan sized for a larger input (a streamed chunk's capacity) launches blocks whose
    // tile starts at or past n: they hold no keys and write nothing
    const int64_t left = static_cast<int64_t>(n) - static_cast<int64_t>(tile0);
    const int cnt = left <= 0 ? 0 : static_cast<int>(left < kTile ? left : kTile);
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
        const int32_t k = skey[i];
        const uint32_t digit = (static_cast<uint32_t>(k) >> shift) & mask;
        const uint32_t g = gofs[digit] + static_cast<uint32_t>(i);
        kout[g] = k;
        vout[g] = sval[i];
    }
}

// K == 1: nothing to sort; check the labels and emit the identity permutation.
__global__ void single_cluster_kernel(const int32_t *__restrict__ labels, int64_t n,
                                      int32_t *__restrict__ kout, int32_t *__restrict__ vout,
                                      uint32_t *__restrict__ err) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (labels[i] != 0) err[1] = 1u;
        kout[i] = 0;
        vout[i] = static_cast<int32_t>(i);
    }
}

// offsets[k] = first position p with skeys[p] >= k (offsets[K] = n): position i writes
// every k in (skeys[i-1], skeys[i]], so each entry is written exactly once.
__global__ void csr_offsets_kernel(const int32_t *__restrict__ skeys, int64_t n, int K,
                                   int32_t *__restrict__ offsets) {
    pdl_wait();
    pdl_trigger();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i <= n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int prev = i == 0 ? -1 : skeys[i - 1];
        const int cur = i == n ? K : skeys[i];
        for (int k = prev + 1; k <= cur; ++k) offsets[k] = static_cast<int32_t>(i);
    }
}

int grid_cap(int64_t items, int threads) {
    int64_t g = (items + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 32;
    if (g > cap) g = cap;
    return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_sort_csr(const int32_t *labels, int64_t N, int K, const SortPlan &sp,
                            int32_t *keys0, int32_t *keys1, int32_t *vals0, int32_t *vals1,
                            int32_t *perm_out, uint32_t *hist, uint32_t *dtot,
                            int32_t *offsets, const int32_t **sorted_keys,
                            const int32_t **perm, uint32_t *err, cudaStream_t st) {
    if (sp.passes == 0) {
        int32_t *vo = perm_out ? perm_out : vals0;
        launch_pdl(single_cluster_kernel, dim3(grid_cap(N, 256)), dim3(256), 0, st, labels, N,
                   keys0, vo, err);
        note_launch();
        *sorted_keys = keys0;
        *perm = vo;
    } else {
        const int bins = 1 << sp.bits;
        const int tile = kSortThreads * sp.items;
        const size_t up_smem = sizeof(uint32_t) * kWarps * bins;
        const size_t dn_smem =
            sizeof(uint32_t) * ((kWarps + 3) * bins) + sizeof(int32_t) * 2 * tile;
        // the largest tile and digit need 27 KB, under the default 48 KB limit: no opt-in
        static_assert(sizeof(uint32_t) * (kWarps + 3) * (1 << kSortMaxBits) +
                              sizeof(int32_t) * 2 * kSortTile <= 48 * 1024,
                      "sort shared memory above the default limit");
        const bool small = sp.items == kSortItemsSmall;
        // a one-pass sort's downsweep writes the CSR offsets (no offsets launch)
        const bool one_pass = sp.passes == 1;
        const int32_t *kin = labels;
        const int32_t *vin = nullptr;
        int32_t *kb[2] = {keys0, keys1};
        int32_t *vb[2] = {vals0, vals1};
        for (int p = 0; p < sp.passes; ++p) {
            const int shift = p * sp.bits;
            const dim3 grid(static_cast<unsigned>(sp.nblocks));
            launch_pdl(small ? upsweep_kernel<kSortItemsSmall> : upsweep_kernel<kSortItems>, grid,
                       dim3(kSortThreads), up_smem, st, kin, N, shift, sp.bits, K, hist,
                       sp.nblocks, err, p == 0 ? 1 : 0);
            note_launch();
            launch_pdl(scan_rows_kernel, dim3(bins), dim3(1024), 0, st, hist, sp.nblocks, dtot);
            note_launch();
            int32_t *vo = (p == sp.passes - 1 && perm_out) ? perm_out : vb[p & 1];
            launch_pdl(small ? downsweep_kernel<kSortItemsSmall> : downsweep_kernel<kSortItems>,
                       grid, dim3(kSortThreads), dn_smem, st, kin, vin, kb[p & 1], vo, N, shift,
                       sp.bits, K, hist, dtot, sp.nblocks, one_pass ? offsets : nullptr);
            note_launch();
            kin = kb[p & 1];
            vin = vo;
        }
        *sorted_keys = kin;
        *perm = vin;
        if (one_pass) return cudaGetLastError();  // offsets written by the downsweep
    }
    launch_pdl(csr_offsets_kernel, dim3(grid_cap(N + 1, 256)), dim3(256), 0, st, *sorted_keys, N,
               K, offsets);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk
