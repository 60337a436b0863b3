// assign_sm100.cu -- fused nearest-centroid assignment on B200 tensor cores.
//
// Flash-KMeans article, section "FlashAssign：把距离矩阵按块切成流水线": distances of a
// block of points to all centroids are produced on the fly and reduced to an argmin on
// chip, so the N x K distance matrix never reaches memory and only O(Nd + Kd) bytes move.
//
// B200 design (a new kernel; the article's H200 kernel is prior art only):
//   * persistent grid, one CTA per SM; a CTA owns 128-row blocks of X in turn and sweeps
//     all centroid tiles of 256 for each;
//   * warp 0, one thread: TMA producer.  Per 64-column chunk of d it loads the X chunk(s)
//     (128 x 64 bf16 per plane) and the centroid chunk(s) (256 x 64 bf16 per plane) into
//     a ring of shared-memory stages, 128-byte swizzled; completion by mbarrier tx-count;
//   * warp 1, one thread: tcgen05.mma issuer, kind::f16 (bf16 x bf16 -> fp32), M=128,
//     N=256, K=16 per instruction, accumulating a 128 x 256 fp32 tile in tensor memory;
//     two accumulators (512 TMEM columns) so the epilogue of tile t overlaps the MMAs of
//     tile t+1; tcgen05.commit releases smem stages and hands tiles to the epilogue;
//   * warps 2..17 (four warpgroups, one per 64-column quarter of the tile; within a group
//     one thread per row / TMEM lane): epilogue.  tcgen05.ld of 64 columns, v = acc +
//     ||c||^2 (the B operand holds -2c; the norms arrive in shared memory by bulk copy),
//     a three-input-min reduction and a running (min, argmin) per row in registers; ties
//     keep the lowest centroid index.  The four quarters are merged per 128-row block
//     through mbarrier-guarded shared memory.  Only the label (and optionally the minimum)
//     is written to HBM.
//   * fp32 points (NP = 2): x.c is formed from three bf16 products hi*hi' + lo*hi' +
//     hi*lo' into one fp32 accumulator (the X and centroid planes come split from prep).
//     bf16 points (NP = 1): one product, exact in fp32.
//   * every mbarrier wait is bounded; on expiry the CTA raises the abort flag, records
//     the timeout in the workspace error word and winds down (TMEM is always freed).
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "fk_common.cuh"
#include "ptx_sm100.cuh"

namespace fk {
namespace {


// Tile configuration.  NP = bf16 planes per operand (2: fp32 emulation hi/lo, 1: bf16).
// RES = the 128-row X block stays resident in shared memory for the whole sweep over the
// centroid tiles (d <= 128 only), so only centroid chunks stream through the ring; the X
// block is double-buffered when it is small enough (NP = 1) so the next block's load
// overlaps the current block's MMAs.
template <int NP, bool RES>
struct AsgCfg {
    static constexpr int kABytes = kBM * kBK * 2;  // 16 KB: one X plane chunk
    static constexpr int kBBytes = kBN * kBK * 2;  // 32 KB: one centroid plane chunk
    static constexpr int kAChunks = RES ? 2 : 0;   // resident k-chunks (d <= 128)
    static constexpr int kABufs = RES ? (NP == 1 ? 2 : 1) : 1;  // (1 unused when !RES)
    static constexpr int kABufBytes = kAChunks * NP * kABytes;
    static constexpr int kARegion = RES ? kABufs * kABufBytes : 0;
    static constexpr int kStageBytes = RES ? NP * kBBytes : NP * (kABytes + kBBytes);
    static constexpr int kStages = RES ? (NP == 1 ? 4 : 2) : (NP == 2 ? 2 : 4);
    static constexpr int kDataBytes = kARegion + kStages * kStageBytes;  // 192 KB
    static constexpr int kBarBytes = 512;
    static constexpr int kEpiGroups = 4;               // warpgroups splitting the columns
    static constexpr int kEpiCols = kBN / kEpiGroups;  // 64 columns per group per tile
    // per-row (min, argmin) of groups 1..3, two slots
    static constexpr int kRedBytes = (kEpiGroups - 1) * 2 * kBM * 8;
    static constexpr int kAugA = kBM * kAug * 2;       // 4 KB: constant (1, 1, 1, 0, ...) rows
    static constexpr int kAugB = kBN * kAug * 2;       // 8 KB: tile's ||c||^2 pieces
    static constexpr int kAugRegion = kAugA + 2 * kAugB;
    static constexpr int kSmemBytes = kDataBytes + kAugRegion + kBarBytes + kRedBytes + 1024;
    static constexpr int kEpiWarps = 4 * kEpiGroups;
    static constexpr int kThreads = 64 + kEpiWarps * 32;
    static constexpr int kTmemCols = 2 * kBN;  // two 256-column fp32 accumulators
    static_assert(kSmemBytes <= 232448, "shared memory");
};

__device__ __forceinline__ void raise_timeout(volatile uint32_t *abort_flag, uint32_t *err) {
    *abort_flag = 1u;
    err[0] = kErrTimeout;
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast to the warp so every
// lane takes the same path (the tcgen05.ld that follows is a warp-aligned instruction).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity,
                                          volatile uint32_t *abort_flag, uint64_t wait_ns) {
    uint32_t ok = 0;
    if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, abort_flag, wait_ns);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// The constant A block of the norm-folding K step: 128 rows of (1, 1, 1, 0, ..., 0) bf16
// (16 columns, 32 bytes per row) in the 32-byte-swizzled K-major layout (the two 16-byte
// halves of row r are swapped when bit 2 of r is set).  One thread per row; the caller
// fences the generic-proxy writes before the tensor core reads them.
__device__ __forceinline__ void init_aug_a(uint8_t *aaug, int r) {
    const uint4 ones = make_uint4(0x3f803f80u, 0x00003f80u, 0u, 0u);  // 1, 1, 1, 0, ...
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    uint4 *row = reinterpret_cast<uint4 *>(aaug + r * 32);
    const int sw = (r >> 2) & 1;
    row[0 ^ sw] = ones;
    row[1 ^ sw] = zero;
}

// Calls f(std::integral_constant<int, i>{}) for i = 0 .. n - 1, unrolled at compile time.
template <int I, int N, typename F>
__device__ __forceinline__ void static_for_impl(F &&f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for_impl<I + 1, N>(f);
    }
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F &&f) {
    static_for_impl<0, N>(f);
}

// Minimum of 64 values with three-input mins: 21 + 7 + 3 + 1 instructions.

__device__ __forceinline__ float min64(const float (&v)[64]) {
    float t[22];
#pragma unroll
    for (int i = 0; i < 21; ++i) t[i] = ptx::fmin3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    t[21] = v[63];
    float u[8];
#pragma unroll
    for (int i = 0; i < 7; ++i) u[i] = ptx::fmin3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
    u[7] = t[21];
    const float a = ptx::fmin3(u[0], u[1], u[2]);
    const float b = ptx::fmin3(u[3], u[4], u[5]);
    return ptx::fmin3(a, b, fminf(u[6], u[7]));
}

// Minimum of 64 values as the minimum of eight groups of eight (their minima in g8): 36
// three-input mins, a few more than min64, so that the first index of the minimum can be
// found group by group.
__device__ __forceinline__ float min64_groups(const float (&v)[64], float (&g8)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
        g8[i] = ptx::fmin3(ptx::fmin3(v[8 * i], v[8 * i + 1], v[8 * i + 2]),
                           ptx::fmin3(v[8 * i + 3], v[8 * i + 4], v[8 * i + 5]),
                           fminf(v[8 * i + 6], v[8 * i + 7]));
    return ptx::fmin3(ptx::fmin3(g8[0], g8[1], g8[2]), ptx::fmin3(g8[3], g8[4], g8[5]),
                      fminf(g8[6], g8[7]));
}

// First column of v equal to m (the minimum), for the lanes with `want`.  Every lane of
// the warp must call it, together (it votes across the full warp).  The group holding it
// is the first whose minimum is m; a group's eight columns are scanned only if some lane
// of the warp needs that group, so a warp in which one row improved pays for one group
// rather than all 64 columns.
__device__ __forceinline__ int first_index_of(const float (&v)[64], const float (&g8)[8],
                                              float m, bool want) {
    int gi = 7;
#pragma unroll
    for (int i = 6; i >= 0; --i) gi = g8[i] == m ? i : gi;
    int idx = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (__any_sync(0xffffffffu, want && gi == i)) {
            int j = 7;
#pragma unroll
            for (int q = 6; q >= 0; --q) j = v[8 * i + q] == m ? q : j;
            idx = gi == i ? 8 * i + j : idx;
        }
    }
    return idx;
}

// Screening: add the columns base + bit of `mask` (screened values >= m, the minimum of
// their chunk) to a row's candidate list.  A free slot holds +inf.  When the list is full,
// the entry with the largest bound gives way (or the new column, if its bound is not
// smaller) and the smallest bound ever dropped is kept in `lost`: the row overflows if it
// is still inside the final window.
template <int KS>
__device__ __forceinline__ void scr_insert(uint32_t mask, int base, float m, float (&lb)[KS],
                                           int (&cc)[KS], float &lost) {
    const float inf = __int_as_float(0x7f800000);
    for (; mask != 0u; mask &= mask - 1u) {
        const int col = base + __ffs(mask) - 1;
        bool placed = false;
#pragma unroll
        for (int t = 0; t < KS; ++t) {
            if (!placed && lb[t] == inf) {
                lb[t] = m;
                cc[t] = col;
                placed = true;
            }
        }
        if (placed) continue;
        float mx = lb[0];
#pragma unroll
        for (int t = 1; t < KS; ++t) mx = fmaxf(mx, lb[t]);
        if (!(m < mx)) {  // full of bounds <= m: every remaining column of the chunk
            lost = fminf(lost, m);  // (same bound m) would be dropped, so drop them at once
            return;
        }
        bool done = false;
#pragma unroll
        for (int t = 0; t < KS; ++t) {
            if (!done && lb[t] == mx) {
                lb[t] = m;
                cc[t] = col;
                done = true;
            }
        }
        lost = fminf(lost, mx);
    }
}

template <int NP, bool RES>
__global__ void __launch_bounds__(AsgCfg<NP, RES>::kThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap tmA0,
                  const __grid_constant__ CUtensorMap tmA1,
                  const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmB1,
                  const __grid_constant__ CUtensorMap tmC,
                  int64_t N, int nkc, int ntiles, int64_t nmb, int32_t *__restrict__ labels,
                  float *__restrict__ best_out, const float *__restrict__ xnorm,
                  float *__restrict__ mind, uint32_t *__restrict__ err, uint64_t wait_ns,
                  const uint32_t *__restrict__ n_dev) {
    using Cfg = AsgCfg<NP, RES>;
    constexpr int S = Cfg::kStages;
    if (n_dev != nullptr) {  // row count written on the device by an earlier kernel
        N = *n_dev;
        nmb = (N + kBM - 1) / kBM;
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem + Cfg::kARegion;
    uint8_t *aaug = smem + Cfg::kDataBytes;  // constant A block of the norm step
    uint8_t *baug = aaug + Cfg::kAugA;       // [2][256 rows][32 B], one slot per accumulator
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kDataBytes + Cfg::kAugRegion);
    uint64_t *empty = full + S;
    uint64_t *tfull = empty + S;
    uint64_t *tempty = tfull + 2;
    uint64_t *afull = tempty + 2;
    uint64_t *aempty = afull + 2;
    uint64_t *redfull = aempty + 2;
    uint64_t *redempty = redfull + 2;
    uint64_t *augfull = redempty + 2;
    uint64_t *drain = augfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    // [group-1][slot][row]
    float *red_v = reinterpret_cast<float *>(smem + Cfg::kDataBytes + Cfg::kAugRegion +
                                             Cfg::kBarBytes);
    int *red_k = reinterpret_cast<int *>(red_v + (Cfg::kEpiGroups - 1) * 2 * kBM);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&tfull[a], 1);
            ptx::mbar_init(&tempty[a], Cfg::kEpiWarps * 32);
            ptx::mbar_init(&afull[a], 1);
            ptx::mbar_init(&aempty[a], 1);
            ptx::mbar_init(&redfull[a], (Cfg::kEpiGroups - 1) * kBM);
            ptx::mbar_init(&redempty[a], kBM);
            ptx::mbar_init(&augfull[a], 1);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0u;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmA0);
        ptx::prefetch_tmap(&tmB0);
        ptx::prefetch_tmap(&tmC);
        if (NP == 2) {
            ptx::prefetch_tmap(&tmA1);
            ptx::prefetch_tmap(&tmB1);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, Cfg::kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp >= 2 && warp < 6) {
        init_aug_a(aaug, (warp & 3) * 32 + lane);
        ptx::fence_proxy_async_smem();  // visible to the tensor core (async proxy)
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, mbi = 0, titer = 0;
            uint32_t issued_mask = 0, issued_par = 0;    // ring stages: loaded, last parity
            uint32_t g_mask = 0, g_par = 0;              // norm slots
            uint32_t a_mask = 0, a_par = 0;              // resident X buffers
            bool ok = true;
            for (int64_t mb = blockIdx.x; mb < nmb && ok; mb += gridDim.x, ++mbi) {
                const int row0 = static_cast<int>(mb * kBM);
                if (RES) {
                    const uint32_t ab = mbi % Cfg::kABufs;
                    const uint32_t apar = (mbi / Cfg::kABufs) & 1u;
                    if (!ptx::mbar_wait(&aempty[ab], apar ^ 1u, abort_flag, wait_ns)) {
                        raise_timeout(abort_flag, err);
                        ok = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&afull[ab], nkc * NP * Cfg::kABytes);
                    uint8_t *ar = smem + ab * Cfg::kABufBytes;
                    for (int kc = 0; kc < nkc; ++kc) {
                        ptx::tma_load_2d(ar + (kc * NP) * Cfg::kABytes, &tmA0, &afull[ab],
                                         kc * kBK, row0);
                        if (NP == 2)
                            ptx::tma_load_2d(ar + (kc * NP + 1) * Cfg::kABytes, &tmA1,
                                             &afull[ab], kc * kBK, row0);
                    }
                    a_mask |= 1u << ab;
                    a_par = (a_par & ~(1u << ab)) | (apar << ab);
                }
                for (int nt = 0; nt < ntiles && ok; ++nt, ++titer) {
                    {
                        // the norm slot of this accumulator is free once the MMAs of the tile
                        // two back (same slot) are complete, i.e. its accumulator is full
                        const uint32_t acc = titer & 1u;
                        const uint32_t aphase = (titer >> 1) & 1u;
                        if (!ptx::mbar_wait(&tfull[acc], aphase ^ 1u, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        ptx::mbar_arrive_expect_tx(&augfull[acc], Cfg::kAugB);
                        ptx::tma_load_2d(baug + acc * Cfg::kAugB, &tmC, &augfull[acc], 0,
                                         nt * kBN);
                        g_mask |= 1u << acc;
                        g_par = (g_par & ~(1u << acc)) | (aphase << acc);
                    }
                    for (int kc = 0; kc < nkc; ++kc) {
                        if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        ptx::mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
                        uint8_t *st = ring + stage * Cfg::kStageBytes;
                        uint8_t *sb = st;
                        if (!RES) {
                            ptx::tma_load_2d(st, &tmA0, &full[stage], kc * kBK, row0);
                            if (NP == 2)
                                ptx::tma_load_2d(st + Cfg::kABytes, &tmA1, &full[stage],
                                                 kc * kBK, row0);
                            sb = st + NP * Cfg::kABytes;
                        }
                        ptx::tma_load_2d(sb, &tmB0, &full[stage], kc * kBK, nt * kBN);
                        if (NP == 2)
                            ptx::tma_load_2d(sb + Cfg::kBBytes, &tmB1, &full[stage], kc * kBK,
                                             nt * kBN);
                        issued_mask |= 1u << stage;
                        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                        if (++stage == S) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (!ok) {
                // Let every load already issued land before the CTA can exit.
                for (int s = 0; s < S; ++s)
                    if (issued_mask & (1u << s))
                        ptx::mbar_wait(&full[s], (issued_par >> s) & 1u, nullptr, wait_ns);
                for (int s = 0; s < 2; ++s) {
                    if (a_mask & (1u << s))
                        ptx::mbar_wait(&afull[s], (a_par >> s) & 1u, nullptr, wait_ns);
                    if (g_mask & (1u << s))
                        ptx::mbar_wait(&augfull[s], (g_par >> s) & 1u, nullptr, wait_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(kBM, kBN);
            uint32_t stage = 0, phase = 0, titer = 0, mbi = 0;
            const uint32_t aaug_s = ptx::smem_u32(aaug);
            const uint32_t baug_s = ptx::smem_u32(baug);
            bool ok = true;
            for (int64_t mb = blockIdx.x; mb < nmb && ok; mb += gridDim.x, ++mbi) {
                uint32_t abase = 0, ab = 0;
                if (RES) {
                    ab = mbi % Cfg::kABufs;
                    const uint32_t apar = (mbi / Cfg::kABufs) & 1u;
                    if (!ptx::mbar_wait(&afull[ab], apar, abort_flag, wait_ns)) {
                        raise_timeout(abort_flag, err);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    abase = ptx::smem_u32(smem + ab * Cfg::kABufBytes);
                }
                for (int nt = 0; nt < ntiles && ok; ++nt, ++titer) {
                    const uint32_t acc = titer & 1u;
                    const uint32_t aphase = (titer >> 1) & 1u;
                    if (!ptx::mbar_wait(&tempty[acc], aphase ^ 1u, abort_flag, wait_ns)) {
                        raise_timeout(abort_flag, err);
                        ok = false;
                        break;
                    }
                    if (!ptx::mbar_wait(&augfull[acc], aphase, abort_flag, wait_ns)) {
                        raise_timeout(abort_flag, err);
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t dt = tmem + acc * kBN;
                    // D = ||c||^2 (hi + mid + lo against the constant ones): the norm step
                    ptx::mma_bf16_ss(dt, ptx::sdesc_k_sw32(aaug_s),
                                     ptx::sdesc_k_sw32(baug_s + acc * Cfg::kAugB), idesc, 0u);
                    for (int kc = 0; kc < nkc; ++kc) {
                        if (!ptx::mbar_wait(&full[stage], phase, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t st = ptx::smem_u32(ring + stage * Cfg::kStageBytes);
                        const uint32_t a0 = RES ? abase + (kc * NP) * Cfg::kABytes : st;
                        const uint32_t a1 = a0 + Cfg::kABytes;
                        const uint32_t b0 = RES ? st : st + NP * Cfg::kABytes;
                        const uint32_t b1 = b0 + Cfg::kBBytes;
                        // descriptors built once; +2 advances the start address by 32 bytes
                        // (16 bf16 along K) inside the 128-byte swizzle row
                        const uint64_t da0 = ptx::sdesc_k_sw128(a0), da1 = ptx::sdesc_k_sw128(a1);
                        const uint64_t db0 = ptx::sdesc_k_sw128(b0), db1 = ptx::sdesc_k_sw128(b1);
#pragma unroll
                        for (int ks = 0; ks < kBK / 16; ++ks) {
                            const uint64_t o = 2u * ks;
                            ptx::mma_bf16_ss(dt, da0 + o, db0 + o, idesc, 1u);
                            if (NP == 2) {
                                ptx::mma_bf16_ss(dt, da1 + o, db0 + o, idesc, 1u);
                                ptx::mma_bf16_ss(dt, da0 + o, db1 + o, idesc, 1u);
                            }
                        }
                        ptx::mma_commit(&empty[stage]);
                        if (++stage == S) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    ptx::mma_commit(&tfull[acc]);  // also frees this tile's norm slot
                }
                if (RES && ok) ptx::mma_commit(&aempty[ab]);  // X buffer free after these MMAs
            }
            if (!ok) {
                // Make sure no MMA issued by this thread is still writing tensor memory and
                // every norm copy it started has landed.
                ptx::mma_commit(drain);
                ptx::mbar_wait(drain, 0u, nullptr, wait_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warpgroup g (warps 2+4g .. 5+4g) scans columns [64 g, 64 g + 64) of every tile;
        // warp w may read TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, i.e. those rows.
        constexpr int EC = Cfg::kEpiCols;
        const int g = (warp - 2) >> 2;
        const int q = warp & 3;
        const int r = q * 32 + lane;
        uint32_t titer = 0, mbi = 0;
        bool ok = true;
        for (int64_t mb = blockIdx.x; mb < nmb && ok; mb += gridDim.x, ++mbi) {
            float best = __int_as_float(0x7f800000);
            int bestk = 0;
            for (int nt = 0; nt < ntiles; ++nt, ++titer) {
                const uint32_t acc = titer & 1u;
                const uint32_t aphase = (titer >> 1) & 1u;
                if (!warp_wait(&tfull[acc], aphase, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tb =
                    tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * kBN + g * EC;
                const int colbase = nt * kBN + g * EC;
                __syncwarp();
                float v[EC];  // ||c||^2 - 2 x.c, the norm already folded in by the MMA
                ptx::tmem_ld64_sync(tb, v);
                ptx::tc_fence_before();
                ptx::mbar_arrive(&tempty[acc]);  // accumulator consumed
                const float m = min64(v);
                if (m < best) {
                    int idx = 0;
#pragma unroll
                    for (int j = EC - 1; j >= 0; --j)
                        if (v[j] == m) idx = j;
                    best = m;
                    bestk = colbase + idx;
                }
            }
            if (!ok) break;
            // combine the column groups of each row: (min, lowest index)
            const uint32_t slot = mbi & 1u;
            const uint32_t spar = (mbi >> 1) & 1u;
            if (g > 0) {
                if (!warp_wait(&redempty[slot], spar ^ 1u, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
                red_v[((g - 1) * 2 + slot) * kBM + r] = best;
                red_k[((g - 1) * 2 + slot) * kBM + r] = bestk;
                ptx::mbar_arrive(&redfull[slot]);
            } else {
                if (!warp_wait(&redfull[slot], spar, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
#pragma unroll
                for (int gg = 0; gg < Cfg::kEpiGroups - 1; ++gg) {
                    const float b1 = red_v[(gg * 2 + slot) * kBM + r];
                    const int k1 = red_k[(gg * 2 + slot) * kBM + r];
                    if (b1 < best || (b1 == best && k1 < bestk)) {
                        best = b1;
                        bestk = k1;
                    }
                }
                ptx::mbar_arrive(&redempty[slot]);
                const int64_t row = mb * kBM + r;
                if (row < N) {
                    labels[row] = bestk;
                    if (best_out) best_out[row] = best;
                    if (mind) mind[row] = xnorm[row] + best;
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// ============================================================================ CTA pairs
// The same computation on a cluster of two CTAs (two SMs) with cta_group::2 MMAs: the
// pair owns a 256-row block of X, each CTA staging its own 128 rows and its own half (128
// centroids) of every 256-centroid tile; the even CTA issues M = 256, N = 256 MMAs that
// read A and B from both CTAs' shared memory and leave each CTA's 128 x 256 accumulator
// in its own tensor memory.  Shared-memory operand traffic per flop is half that of the
// single-CTA kernel.  Stage and accumulator hand-offs are mbarriers: loads of both CTAs
// complete on the even CTA's barriers, MMA completion is signalled to both CTAs
// (tcgen05.commit multicast), and both CTAs' epilogues release the accumulator to the
// even CTA by remote arrive.  No load is multicast.
template <int NP, bool RES, int EG = 4>
struct PairCfg {
    static constexpr int kABytes = kBM * kBK * 2;         // 16 KB: 128 X rows, one chunk
    static constexpr int kBBytes = (kBN / 2) * kBK * 2;   // 16 KB: 128 centroids, one chunk
    static constexpr int kAChunks = RES ? 2 : 0;
    static constexpr int kABufs = RES ? (NP == 1 ? 2 : 1) : 1;
    static constexpr int kABufBytes = kAChunks * NP * kABytes;
    static constexpr int kARegion = RES ? kABufs * kABufBytes : 0;
    // resident X: one stage holds all (<= 2) k-chunks of a tile's centroids, so a tile costs
    // one full-wait and one empty-commit; streamed X: one k-chunk of X and centroids
    static constexpr int kStageChunks = RES ? kAChunks : 1;
    static constexpr int kAugA = kBM * kAug * 2;         // 4 KB: constant (1, 1, 1, 0, ...)
    static constexpr int kAugB = (kBN / 2) * kAug * 2;   // 4 KB: this CTA's 128 norms
    // resident X: a stage is one tile, its centroid chunks followed by its norm pieces (so
    // one barrier covers both); streamed X: a stage is one chunk of X and of the centroids,
    // and the norm pieces have a ring of kAugSlots slots of their own, each freed by a
    // commit right after its norm MMA
    static constexpr int kNormOff = kStageChunks * NP * kBBytes;  // resident X only
    static constexpr int kStageBytes =
        RES ? kNormOff + kAugB : NP * (kABytes + kBBytes);
    static constexpr int kStages = RES ? (NP == 1 ? 4 : 2) : (NP == 2 ? 3 : 6);
    static constexpr int kDataBytes = kARegion + kStages * kStageBytes;
    static constexpr int kBarBytes = 512;
    // epilogue warpgroups splitting a tile's columns: 4 for the argmin; 1 for the screening
    // pass, whose per-row candidate list must see all 256 columns of every tile
    static constexpr int kEpiGroups = EG;
    static constexpr int kEpiCols = kBN / kEpiGroups;
    static constexpr int kRedBytes = (kEpiGroups - 1) * 2 * kBM * 8;
    static constexpr int kAugSlots = RES ? 0 : 4;
    static constexpr int kAugRegion = kAugA + kAugSlots * kAugB;
    static constexpr int kSmemBytes = kDataBytes + kAugRegion + kBarBytes + kRedBytes + 1024;
    static constexpr int kEpiWarps = 4 * kEpiGroups;
    static constexpr int kThreads = 64 + kEpiWarps * 32;
    static constexpr int kTmemCols = 2 * kBN;
    static_assert(kStages <= 8, "stage masks");
    static_assert(kStageBytes % 1024 == 0, "stage bases stay 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert(8 * (2 * kStages + 12 + 2 * kAugSlots + 1) + 8 <= kBarBytes, "barriers");
};

template <int NP, bool RES, bool SCR>
__global__ void __launch_bounds__(PairCfg<NP, RES, SCR ? 1 : 4>::kThreads, 1)
    assign_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                       const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmC,
                       int64_t N, int nkc, int ntiles, int64_t nmb,
                       int32_t *__restrict__ labels, float *__restrict__ best_out,
                       const float *__restrict__ xnorm, float *__restrict__ mind,
                       uint32_t *__restrict__ err, uint64_t wait_ns,
                       const uint32_t *__restrict__ n_dev, int32_t *__restrict__ cand,
                       const float *__restrict__ cmax2, float *__restrict__ dump,
                       int64_t ldd) {
    static_assert(!SCR || NP == 1, "screening runs the single-product form");
    using Cfg = PairCfg<NP, RES, SCR ? 1 : 4>;
    constexpr int S = Cfg::kStages;
    constexpr int EC = Cfg::kEpiCols;
    if (n_dev != nullptr) {  // row count written on the device by an earlier kernel
        N = *n_dev;
        nmb = (N + 2 * kBM - 1) / (2 * kBM);
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *ring = smem + Cfg::kARegion;
    uint8_t *aaug = smem + Cfg::kDataBytes;  // constant A block of the norm step
    uint8_t *baug = aaug + Cfg::kAugA;       // [kAugSlots][128 rows][32 B]
    uint64_t *full =
        reinterpret_cast<uint64_t *>(smem + Cfg::kDataBytes + Cfg::kAugRegion);  // even CTA
    uint64_t *empty = full + S;
    uint64_t *tfull = empty + S;
    uint64_t *tempty = tfull + 2;  // even CTA
    uint64_t *afull = tempty + 2;  // even CTA
    uint64_t *aempty = afull + 2;
    uint64_t *redfull = aempty + 2;
    uint64_t *redempty = redfull + 2;
    uint64_t *augfull = redempty + 2;  // even CTA, [kAugSlots]
    uint64_t *augempty = augfull + Cfg::kAugSlots;  // both CTAs, [kAugSlots]
    uint64_t *drain = augempty + Cfg::kAugSlots;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    float *red_v = reinterpret_cast<float *>(smem + Cfg::kDataBytes + Cfg::kAugRegion +
                                             Cfg::kBarBytes);
    int *red_k = reinterpret_cast<int *>(red_v + (Cfg::kEpiGroups - 1) * 2 * kBM);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const int64_t pair = blockIdx.x >> 1;
    const int64_t npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&tfull[a], 1);
            ptx::mbar_init(&tempty[a], 2 * Cfg::kEpiWarps);
            ptx::mbar_init(&afull[a], 1);
            ptx::mbar_init(&aempty[a], 1);
            if (Cfg::kEpiGroups > 1) {
                ptx::mbar_init(&redfull[a], (Cfg::kEpiGroups - 1) * kBM);
                ptx::mbar_init(&redempty[a], kBM);
            }
        }
        for (int a = 0; a < Cfg::kAugSlots; ++a) {
            ptx::mbar_init(&augfull[a], 1);
            ptx::mbar_init(&augempty[a], 1);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0u;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tmA0);
        ptx::prefetch_tmap(&tmB0);
        ptx::prefetch_tmap(&tmC);
        if (NP == 2) {
            ptx::prefetch_tmap(&tmA1);
            ptx::prefetch_tmap(&tmB1);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    if (warp >= 2 && warp < 6) {
        init_aug_a(aaug, (warp & 3) * 32 + lane);
        ptx::fence_proxy_async_smem();  // visible to the tensor core (async proxy)
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // barriers of both CTAs initialised, tensor memory allocated
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // shared::cluster addresses of the even CTA's barriers
    const uint32_t full_c = ptx::mapa_shared(ptx::smem_u32(full), 0);
    const uint32_t afull_c = ptx::mapa_shared(ptx::smem_u32(afull), 0);
    const uint32_t tempty_c = ptx::mapa_shared(ptx::smem_u32(tempty), 0);
    const uint32_t augfull_c = ptx::mapa_shared(ptx::smem_u32(augfull), 0);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer (both)
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, mbi = 0, titer = 0;
            bool ok = true;
            for (int64_t mb = pair; mb < nmb && ok; mb += npairs, ++mbi) {
                const int row0 = static_cast<int>(mb * 2 * kBM + rank * kBM);
                if (RES) {
                    const uint32_t ab = mbi % Cfg::kABufs;
                    const uint32_t apar = (mbi / Cfg::kABufs) & 1u;
                    if (!ptx::mbar_wait(&aempty[ab], apar ^ 1u, abort_flag, wait_ns)) {
                        raise_timeout(abort_flag, err);
                        ok = false;
                        break;
                    }
                    if (rank == 0)
                        ptx::mbar_arrive_expect_tx(&afull[ab], 2 * nkc * NP * Cfg::kABytes);
                    uint8_t *ar = smem + ab * Cfg::kABufBytes;
                    for (int kc = 0; kc < nkc; ++kc) {
                        ptx::tma_load_2d_pair(ar + (kc * NP) * Cfg::kABytes, &tmA0,
                                              afull_c + ab * 8, kc * kBK, row0);
                        if (NP == 2)
                            ptx::tma_load_2d_pair(ar + (kc * NP + 1) * Cfg::kABytes, &tmA1,
                                                  afull_c + ab * 8, kc * kBK, row0);
                    }
                }
                for (int nt = 0; nt < ntiles && ok; ++nt, ++titer) {
                    const int crow = nt * kBN + static_cast<int>(rank) * (kBN / 2);
                    if constexpr (!RES) {
                        // the norm slot is free once the norm MMA of its previous tile ran
                        const uint32_t as = titer % Cfg::kAugSlots;
                        const uint32_t asp = (titer / Cfg::kAugSlots) & 1u;
                        if (!ptx::mbar_wait(&augempty[as], asp ^ 1u, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        if (rank == 0) ptx::mbar_arrive_expect_tx(&augfull[as], 2 * Cfg::kAugB);
                        ptx::tma_load_2d_pair(baug + as * Cfg::kAugB, &tmC, augfull_c + as * 8,
                                              0, crow);
                    }
                    for (int kc = 0; kc < nkc; kc += Cfg::kStageChunks) {
                        if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        const int nch = nkc - kc < Cfg::kStageChunks ? nkc - kc
                                                                     : Cfg::kStageChunks;
                        if (rank == 0)
                            ptx::mbar_arrive_expect_tx(
                                &full[stage], RES ? 2 * (nch * NP * Cfg::kBBytes + Cfg::kAugB)
                                                  : 2 * nch * NP * (Cfg::kABytes + Cfg::kBBytes));
                        uint8_t *st = ring + stage * Cfg::kStageBytes;
                        const uint32_t fb = full_c + stage * 8;
                        if (RES)  // the tile's norm pieces, behind its centroid chunks
                            ptx::tma_load_2d_pair(st + Cfg::kNormOff, &tmC, fb, 0, crow);
                        for (int c = 0; c < nch; ++c) {
                            uint8_t *sb = st + c * NP * Cfg::kBBytes;
                            if (!RES) {
                                ptx::tma_load_2d_pair(st, &tmA0, fb, (kc + c) * kBK, row0);
                                if (NP == 2)
                                    ptx::tma_load_2d_pair(st + Cfg::kABytes, &tmA1, fb,
                                                          (kc + c) * kBK, row0);
                                sb = st + NP * Cfg::kABytes;
                            }
                            ptx::tma_load_2d_pair(sb, &tmB0, fb, (kc + c) * kBK, crow);
                            if (NP == 2)
                                ptx::tma_load_2d_pair(sb + Cfg::kBBytes, &tmB1, fb,
                                                      (kc + c) * kBK, crow);
                        }
                        if (++stage == S) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t titer = 0;
            bool ok = true;
            if (rank == 0) {
                // -------------------------------------------------- MMA issuer (even CTA)
                constexpr uint32_t idesc = ptx::idesc_bf16_f32(2 * kBM, kBN);
                uint32_t stage = 0, phase = 0, mbi = 0;
                const uint32_t aaug_s = ptx::smem_u32(aaug);
                const uint32_t baug_s = ptx::smem_u32(baug);
                if constexpr (RES) {
                    // Resident X: a tile is one stage (its centroid chunks and its norm
                    // pieces, behind one barrier).  Issuing an MMA blocks while the tensor
                    // pipe's short queue (about one MMA) is full, so whatever the issuing
                    // thread does between tiles leaves the pipe idle: the boundary is kept
                    // short (two commits, non-blocking tests of the next stage and
                    // accumulator that nearly always pass at once, bounded waits behind
                    // them) and the MMA sequence is unrolled with its descriptors folded.
                    // Waiting for the next tile earlier, inside the current tile's MMAs, was
                    // measured slower: the accumulator is released only while the current
                    // tile runs.
                    constexpr int P = NP == 2 ? 3 : 1;           // MMAs per K step
                    constexpr int kMaxM = Cfg::kAChunks * (kBK / 16) * P;
                    const int nm = nkc * (kBK / 16) * P;         // data MMAs per tile
                    auto wait_bar = [&](uint64_t *bar, uint32_t par) -> bool {
                        if (ptx::mbar_test(bar, par) ||
                            ptx::mbar_wait(bar, par, abort_flag, wait_ns))
                            return true;
                        raise_timeout(abort_flag, err);
                        return false;
                    };
                    // tile ti's stage (the producer's order) and accumulator
                    auto wait_tile = [&](uint32_t ti, uint32_t stg, uint32_t ph) -> bool {
                        return wait_bar(&full[stg], ph) &&
                               wait_bar(&tempty[ti & 1u], ((ti >> 1) & 1u) ^ 1u);
                    };
                    auto wait_block = [&](uint32_t bi) -> bool {
                        return wait_bar(&afull[bi % Cfg::kABufs], (bi / Cfg::kABufs) & 1u);
                    };
                    int64_t mb = pair;
                    int nt = 0;
                    if (mb < nmb) ok = wait_block(0) && wait_tile(0, 0, 0);
                    while (ok && mb < nmb) {
                        ptx::tc_fence_after();
                        const uint32_t ab = mbi % Cfg::kABufs;
                        const uint32_t acc = titer & 1u;
                        const uint32_t dt = tmem + acc * kBN;
                        const uint32_t st = ptx::smem_u32(ring + stage * Cfg::kStageBytes);
                        const uint64_t dA = ptx::sdesc_k_sw128(
                            ptx::smem_u32(smem + ab * Cfg::kABufBytes));
                        const uint64_t dB = ptx::sdesc_k_sw128(st);
                        // D = ||c||^2 (hi + mid + lo against the constant ones)
                        ptx::mma_bf16_ss_pair(dt, ptx::sdesc_k_sw32(aaug_s),
                                              ptx::sdesc_k_sw32(st + Cfg::kNormOff), idesc, 0u);
                        // data MMA i: chunk c, K step ks, product (hi.hi, lo.hi, hi.lo); a
                        // descriptor's address field advances by bytes / 16
                        static_for<kMaxM>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            constexpr int c = i / ((kBK / 16) * P);
                            constexpr int ks = (i / P) % (kBK / 16);
                            constexpr int pa = i % P == 1 ? 1 : 0;
                            constexpr int pb = i % P == 2 ? 1 : 0;
                            constexpr uint64_t oa = ((c * NP + pa) * Cfg::kABytes) / 16 + 2 * ks;
                            constexpr uint64_t ob = ((c * NP + pb) * Cfg::kBBytes) / 16 + 2 * ks;
                            if (i < nm) ptx::mma_bf16_ss_pair(dt, dA + oa, dB + ob, idesc, 1u);
                        });
                        ptx::mma_commit_pair(&empty[stage], 0x3);
                        ptx::mma_commit_pair(&tfull[acc], 0x3);
                        // the next tile in this pair's order
                        if (++nt == ntiles) {
                            ptx::mma_commit_pair(&aempty[ab], 0x3);  // this X block is done
                            nt = 0;
                            mb += npairs;
                            ++mbi;
                        }
                        ++titer;
                        if (++stage == S) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        if (mb < nmb)
                            ok = (nt != 0 || wait_block(mbi)) && wait_tile(titer, stage, phase);
                    }
                } else {
                for (int64_t mb = pair; mb < nmb && ok; mb += npairs, ++mbi) {
                    for (int nt = 0; nt < ntiles && ok; ++nt, ++titer) {
                        const uint32_t acc = titer & 1u;
                        const uint32_t aphase = (titer >> 1) & 1u;
                        if (!ptx::mbar_wait(&tempty[acc], aphase ^ 1u, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        const uint32_t as = titer % Cfg::kAugSlots;
                        const uint32_t asp = (titer / Cfg::kAugSlots) & 1u;
                        if (!ptx::mbar_wait(&augfull[as], asp, abort_flag, wait_ns)) {
                            raise_timeout(abort_flag, err);
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t dt = tmem + acc * kBN;
                        // D = ||c||^2 (hi + mid + lo against the constant ones)
                        ptx::mma_bf16_ss_pair(dt, ptx::sdesc_k_sw32(aaug_s),
                                              ptx::sdesc_k_sw32(baug_s + as * Cfg::kAugB),
                                              idesc, 0u);
                        ptx::mma_commit_pair(&augempty[as], 0x3);  // the slot may be refilled
                        for (int kc = 0; kc < nkc; ++kc) {  // streamed X: a stage per chunk
                            if (!ptx::mbar_wait(&full[stage], phase, abort_flag, wait_ns)) {
                                raise_timeout(abort_flag, err);
                                ok = false;
                                break;
                            }
                            ptx::tc_fence_after();
                            const uint32_t st = ptx::smem_u32(ring + stage * Cfg::kStageBytes);
                            const uint32_t a0 = st;
                            const uint32_t a1 = a0 + Cfg::kABytes;
                            const uint32_t b0 = st + NP * Cfg::kABytes;
                            const uint32_t b1 = b0 + Cfg::kBBytes;
                            const uint64_t da0 = ptx::sdesc_k_sw128(a0);
                            const uint64_t da1 = ptx::sdesc_k_sw128(a1);
                            const uint64_t db0 = ptx::sdesc_k_sw128(b0);
                            const uint64_t db1 = ptx::sdesc_k_sw128(b1);
#pragma unroll
                            for (int ks = 0; ks < kBK / 16; ++ks) {
                                const uint64_t o = 2u * ks;  // +32 bytes along K
                                ptx::mma_bf16_ss_pair(dt, da0 + o, db0 + o, idesc, 1u);
                                if (NP == 2) {
                                    ptx::mma_bf16_ss_pair(dt, da1 + o, db0 + o, idesc, 1u);
                                    ptx::mma_bf16_ss_pair(dt, da0 + o, db1 + o, idesc, 1u);
                                }
                            }
                            ptx::mma_commit_pair(&empty[stage], 0x3);
                            if (++stage == S) {
                                stage = 0;
                                phase ^= 1u;
                            }
                        }
                        if (!ok) break;
                        ptx::mma_commit_pair(&tfull[acc], 0x3);
                    }
                }
                }
                if (!ok) {
                    ptx::mma_commit_pair(drain, 0x1);
                    ptx::mbar_wait(drain, 0u, nullptr, wait_ns);
                }
            }
        }
    } else if constexpr (SCR) {
        // ------------------------------------------------------ screening epilogue (both)
        // One warpgroup owns all 256 columns of every tile: warp q holds the rows of tensor
        // memory lanes 32q .. 32q + 31 and reads each tile as four 64-column chunks.  Per
        // row it keeps the running screened minimum and a list of up to kScreenSlots
        // candidate columns, each with a lower bound on its screened value (the minimum of
        // the chunk it came from).
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const float cm2 = *cmax2;
        const float inf = __int_as_float(0x7f800000);
        uint32_t titer = 0;
        bool ok = true;
        // ||x||^2 of this thread's row in the next row block, loaded a block ahead
        float xn_next = 0.f;
        {
            const int64_t row0 = pair * 2 * kBM + static_cast<int64_t>(rank) * kBM + r;
            if (pair < nmb && row0 < N) xn_next = xnorm[row0];
        }
        for (int64_t mb = pair; mb < nmb && ok; mb += npairs) {
            const int64_t row = mb * 2 * kBM + static_cast<int64_t>(rank) * kBM + r;
            const float W = screen_window(xn_next, cm2, nkc * kBK);
            {
                const int64_t rn = row + npairs * 2 * kBM;
                xn_next = (mb + npairs < nmb && rn < N) ? xnorm[rn] : 0.f;
            }
            float best = inf, lost = inf;
            float lb[kScreenSlots];
            int cc[kScreenSlots];
#pragma unroll
            for (int t = 0; t < kScreenSlots; ++t) {
                lb[t] = inf;
                cc[t] = -1;
            }
            for (int nt = 0; nt < ntiles; ++nt, ++titer) {
                const uint32_t acc = titer & 1u;
                const uint32_t aphase = (titer >> 1) & 1u;
                if (!warp_wait(&tfull[acc], aphase, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * kBN;
#pragma unroll 1
                for (int c4 = 0; c4 < kBN / 64; ++c4) {
                    __syncwarp();
                    float v[64];  // ||c||^2 - 2 x~.c~ for 64 columns
                    ptx::tmem_ld64_sync(tb + c4 * 64, v);
                    if (c4 == kBN / 64 - 1) {  // the whole tile is in registers: release it
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive_cluster(tempty_c + acc * 8);
                    }
                    if (dump != nullptr) {  // every screened value goes out: no candidates
                        if (row < N) {
                            float4 *dst = reinterpret_cast<float4 *>(
                                dump + row * ldd + static_cast<int64_t>(nt) * kBN + c4 * 64);
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2],
                                                     v[4 * j + 3]);
                        }
                        continue;
                    }
                    const float m = min64(v);
                    // a chunk with columns inside the window; a chunk no better than a column
                    // already dropped cannot matter (if the final window reaches that column
                    // the row overflows anyway; if not, neither does this chunk)
                    if (m <= best + W && m < lost) {
                        if (m < best) {
                            best = m;
                            const float T0 = fminf(best + W, kScreenMax);
#pragma unroll
                            for (int t = 0; t < kScreenSlots; ++t)
                                if (lb[t] > T0) lb[t] = inf;  // left the window for good
                        }
                        const float T = fminf(best + W, kScreenMax);
                        uint32_t lo = 0u, hi = 0u;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            lo |= (v[j] <= T ? 1u : 0u) << j;
                            hi |= (v[32 + j] <= T ? 1u : 0u) << j;
                        }
                        const int base = nt * kBN + c4 * 64;
                        scr_insert(lo, base, m, lb, cc, lost);
                        scr_insert(hi, base + 32, m, lb, cc, lost);
                    }
                }
            }
            if (!ok) break;
            if (dump != nullptr) continue;
            // candidates: every kept column whose chunk minimum is inside the final window;
            // the row overflows if a column dropped for lack of room could still be inside
            const float T = fminf(best + W, kScreenMax);
            const bool over = lost <= T;
            if (row < N) {
                int4 *dst = reinterpret_cast<int4 *>(cand + row * kCandPerRow);
#pragma unroll
                for (int t4 = 0; t4 < kScreenSlots / 4; ++t4) {
                    int4 o;
                    o.x = lb[4 * t4 + 0] <= T ? cc[4 * t4 + 0] : -1;
                    o.y = lb[4 * t4 + 1] <= T ? cc[4 * t4 + 1] : -1;
                    o.z = lb[4 * t4 + 2] <= T ? cc[4 * t4 + 2] : -1;
                    o.w = lb[4 * t4 + 3] <= T ? cc[4 * t4 + 3] : -1;
                    if (t4 == 0 && over) o.x = kCandOverflow;
                    dst[t4] = o;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both)
        const int g = (warp - 2) >> 2;
        const int q = warp & 3;
        const int r = q * 32 + lane;
        uint32_t titer = 0, mbi = 0;
        bool ok = true;
        for (int64_t mb = pair; mb < nmb && ok; mb += npairs, ++mbi) {
            const int64_t row = mb * 2 * kBM + static_cast<int64_t>(rank) * kBM + r;
            float best = __int_as_float(0x7f800000);
            int bestk = 0;
            for (int nt = 0; nt < ntiles; ++nt, ++titer) {
                const uint32_t acc = titer & 1u;
                const uint32_t aphase = (titer >> 1) & 1u;
                if (!warp_wait(&tfull[acc], aphase, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t tb =
                    tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * kBN + g * EC;
                const int colbase = nt * kBN + g * EC;
                __syncwarp();
                float v[EC];  // ||c||^2 - 2 x.c, the norm already folded in by the MMA
                ptx::tmem_ld64_sync(tb, v);
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster(tempty_c + acc * 8);  // consumed
                float g8[8];  // minima of the eight groups of eight columns
                const float m = min64_groups(v, g8);
                const bool imp = m < best;
                if (__any_sync(0xffffffffu, imp)) {
                    // every lane of the warp takes part in the search (it votes across the
                    // warp); only the lanes whose row improved keep its result
                    const int idx = first_index_of(v, g8, m, imp);
                    if (imp) {
                        best = m;
                        bestk = colbase + idx;
                    }
                }
            }
            if (!ok) break;
            const uint32_t slot = mbi & 1u;
            const uint32_t spar = (mbi >> 1) & 1u;
            if (g > 0) {
                if (!warp_wait(&redempty[slot], spar ^ 1u, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
                red_v[((g - 1) * 2 + slot) * kBM + r] = best;
                red_k[((g - 1) * 2 + slot) * kBM + r] = bestk;
                ptx::mbar_arrive(&redfull[slot]);
            } else {
                if (!warp_wait(&redfull[slot], spar, abort_flag, wait_ns)) {
                    if (lane == 0) raise_timeout(abort_flag, err);
                    ok = false;
                    break;
                }
#pragma unroll
                for (int gg = 0; gg < Cfg::kEpiGroups - 1; ++gg) {
                    const float b1 = red_v[(gg * 2 + slot) * kBM + r];
                    const int k1 = red_k[(gg * 2 + slot) * kBM + r];
                    if (b1 < best || (b1 == best && k1 < bestk)) {
                        best = b1;
                        bestk = k1;
                    }
                }
                ptx::mbar_arrive(&redempty[slot]);
                if (row < N) {
                    labels[row] = bestk;
                    if (best_out) best_out[row] = best;
                    if (mind) mind[row] = xnorm[row] + best;
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    __syncwarp();
    ptx::cluster_sync();  // neither CTA leaves while the pair may still touch its memory
    if (*abort_flag) {
        // after a timeout, give copies already in flight a moment to land (bounded)
        const uint64_t t0 = ptx::globaltimer_ns();
        while (ptx::globaltimer_ns() - t0 < 200000ull) {
        }
    }
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, Cfg::kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] plane with the given row stride,
// box_cols x box_rows boxes (64 columns = 128 bytes with 128-byte swizzle, or 16 columns =
// 32 bytes with 32-byte swizzle); out-of-range rows/columns read as zero.
bool make_tmap(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
               int64_t row_stride_elems, int box_rows, int box_cols = kBK) {
    auto fn = tmap_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_stride_elems * 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_cols == kAug ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int NP, bool RES>
cudaError_t launch_assign_cfg(const AssignArgs &a, const CUtensorMap (&tA)[2],
                              const CUtensorMap (&tB)[2], const CUtensorMap &tC,
                              cudaStream_t st) {
    using Cfg = AsgCfg<NP, RES>;
    static std::atomic<uint64_t> smem_set{0};
    {
        const cudaError_t e = smem_opt_in(assign_kernel<NP, RES>, Cfg::kSmemBytes, smem_set);
        if (e != cudaSuccess) return e;
    }
    const int64_t nmb = ceil_div(a.N, kBM);
    const int64_t sms = device_sm_count();
    const int grid = static_cast<int>(nmb < sms ? nmb : sms);
    assign_kernel<NP, RES><<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(
        tA[0], tA[1], tB[0], tB[1], tC, a.N, static_cast<int>(a.dp / kBK),
        static_cast<int>(a.Kp / kBN), nmb, a.labels, a.best, a.xnorm, a.mind, a.err,
        a.wait_ns, a.n_dev);
    note_launch();
    return cudaGetLastError();
}

template <int NP, bool RES, bool SCR>
cudaError_t launch_assign_pair_cfg(const AssignArgs &a, const CUtensorMap (&tA)[2],
                                   const CUtensorMap (&tB)[2], const CUtensorMap &tC,
                                   int max_pairs, cudaStream_t st) {
    using Cfg = PairCfg<NP, RES, SCR ? 1 : 4>;
    const int64_t nmb = ceil_div(a.N, 2 * kBM);
    const int pairs = static_cast<int>(nmb < max_pairs ? nmb : max_pairs);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, assign_pair_kernel<NP, RES, SCR>, tA[0], tA[1], tB[0], tB[1], tC, a.N,
        static_cast<int>(a.dp / kBK), static_cast<int>(a.Kp / kBN), nmb, a.labels, a.best,
        a.xnorm, a.mind, a.err, a.wait_ns, a.n_dev, a.cand, a.cmax2, a.dump, a.ldd);
    note_launch();
    return e;
}

// Largest number of CTA pairs of this configuration that can be resident at once (the
// persistent grid must not exceed it, or part of it would wait for a second wave).
template <int NP, bool RES, bool SCR>
int max_resident_pairs() {
    using Cfg = PairCfg<NP, RES, SCR ? 1 : 4>;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cached[dev]) return cached[dev];
    if (cudaFuncSetAttribute(assign_pair_kernel<NP, RES, SCR>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmemBytes) != cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(Cfg::kThreads);
    cfg.dynamicSmemBytes = Cfg::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, assign_pair_kernel<NP, RES, SCR>, &cfg) !=
        cudaSuccess)
        n = 0;
    cached[dev] = n;
    return n;
}

// X block resident in shared memory when it fits (d <= 128) and, for the fp32 emulation
// (one X buffer, so a short gap at each new block), when the sweep over the centroid tiles
// is long enough to hide that gap.
inline bool resident_x(int NP, int dp, int Kp) {
    const int nkc = dp / kBK;
    const int ntiles = Kp / kBN;
    return nkc <= 2 && (NP == 1 || ntiles >= 16);
}

// CTA pairs (M = 256 per MMA) once there are enough 256-row blocks to fill the GPU.
inline bool pair_rows(int64_t N) { return N >= int64_t(2 * kBM) * device_sm_count() / 2; }

template <int NP, bool SCR>
cudaError_t launch_assign_pair(const AssignArgs &a, cudaStream_t st, bool res, bool *done) {
    *done = false;
    const int mp = res ? max_resident_pairs<NP, true, SCR>()
                       : max_resident_pairs<NP, false, SCR>();
    if (mp <= 0) return cudaSuccess;  // pairs cannot be scheduled: use the single-CTA form
    CUtensorMap tA[2], tB[2];
    const uint16_t *ap = static_cast<const uint16_t *>(a.a_planes);
    const uint16_t *bp = static_cast<const uint16_t *>(a.b_planes);
    for (int p = 0; p < NP; ++p) {
        if (!make_tmap(&tA[p], ap + p * a.N * a.lda, a.N, a.dp, a.lda, kBM))
            return cudaErrorInvalidValue;
        if (!make_tmap(&tB[p], bp + p * static_cast<int64_t>(a.Kp) * a.dp, a.Kp, a.dp, a.dp,
                       kBN / 2))
            return cudaErrorInvalidValue;
    }
    if (NP == 1) {
        tA[1] = tA[0];
        tB[1] = tB[0];
    }
    CUtensorMap tC;
    if (!make_tmap(&tC, a.caug, a.Kp, kAug, kAug, kBN / 2, kAug)) return cudaErrorInvalidValue;
    *done = true;
    return res ? launch_assign_pair_cfg<NP, true, SCR>(a, tA, tB, tC, mp, st)
               : launch_assign_pair_cfg<NP, false, SCR>(a, tA, tB, tC, mp, st);
}

template <int NP>
cudaError_t launch_assign_np(const AssignArgs &a, cudaStream_t st) {
    const bool res = resident_x(NP, a.dp, a.Kp);
    if (pair_rows(a.N)) {
        bool done = false;
        const cudaError_t e = launch_assign_pair<NP, false>(a, st, res, &done);
        if (done || e != cudaSuccess) return e;
    }
    CUtensorMap tA[2], tB[2];
    const uint16_t *ap = static_cast<const uint16_t *>(a.a_planes);
    const uint16_t *bp = static_cast<const uint16_t *>(a.b_planes);
    for (int p = 0; p < NP; ++p) {
        if (!make_tmap(&tA[p], ap + p * a.N * a.lda, a.N, a.dp, a.lda, kBM))
            return cudaErrorInvalidValue;
        if (!make_tmap(&tB[p], bp + p * static_cast<int64_t>(a.Kp) * a.dp, a.Kp, a.dp, a.dp,
                       kBN))
            return cudaErrorInvalidValue;
    }
    if (NP == 1) {
        tA[1] = tA[0];
        tB[1] = tB[0];
    }
    CUtensorMap tC;
    if (!make_tmap(&tC, a.caug, a.Kp, kAug, kAug, kBN, kAug)) return cudaErrorInvalidValue;
    if (res) return launch_assign_cfg<NP, true>(a, tA, tB, tC, st);
    return launch_assign_cfg<NP, false>(a, tA, tB, tC, st);
}

}  // namespace

cudaError_t launch_assign(const AssignArgs &a, cudaStream_t st) {
    if (a.N <= 0) return cudaSuccess;
    if (a.cand != nullptr || a.dump != nullptr) {  // only in the CTA-pair form, any N
        if (a.a_nplanes != 1 || !assign_can_dump(a.dp, a.Kp)) return cudaErrorNotSupported;
        bool done = false;
        const cudaError_t e =
            launch_assign_pair<1, true>(a, st, resident_x(1, a.dp, a.Kp), &done);
        return e != cudaSuccess ? e : (done ? cudaSuccess : cudaErrorNotSupported);
    }
    return a.a_nplanes == 2 ? launch_assign_np<2>(a, st) : launch_assign_np<1>(a, st);
}

bool assign_can_screen(int64_t N, int dp, int Kp) {
    if (!pair_rows(N)) return false;
    return assign_can_dump(dp, Kp);
}

bool assign_can_dump(int dp, int Kp) {
    return resident_x(1, dp, Kp) ? max_resident_pairs<1, true, true>() > 0
                                 : max_resident_pairs<1, false, true>() > 0;
}

}  // namespace fk
