// ivf_search.cu -- IVF-Flat search over the inverted lists of a finished clustering.
//
// LEANN FlashLib guide: an IVF-Flat index fitted on a corpus answers the k nearest
// neighbours of a batch of queries (section "什么是 FlashLib 后端"); its cells are the coarse
// k-means clusters, stored cell-contiguous with row ids and CSR offsets (section "工作原理");
// a query probes nprobe cells (sections "nlist 与 nprobe 的推导规则", "参数速查"); the only
// distance is squared L2 (section "距离度量只有 squared L2").
//
// One search call, per batch of queries:
//   1. fp64 norms of the queries and centroids (the points' norms come with the index);
//   2. coarse: the fp64 distance of every query to every centroid (tile kernel, COARSE
//      mode, written to a query-batch x nlist matrix), then per query the nprobe smallest
//      by (distance, cell) (radix select);
//   3. the (query, probe) pairs sorted by cell with the same stable LSD sort as the update,
//      cut into work items of up to 32 pairs of one cell;
//   4. fine: for every item, the fp64 distances of its queries to every point of its cell
//      (tile kernel, FINE mode), keeping per pair the k smallest by (distance, point id)
//      in registers;
//   5. per query, the k smallest of its nprobe pair lists (radix select).
//
// Every distance is ||q||^2 + ||v||^2 - 2 q.v in fp64: products of two fp32 values are exact
// in fp64, the dot product accumulates with fp64 FMAs in dimension order, and the norms are
// fp64 sums of squares.  The result differs from the difference form sum_j (q_j - v_j)^2 by
// rounding at the 1e-16 relative level of the norms, so the selections agree with an fp64
// evaluation except between candidates that close.  Selections use the strict total order
// (distance, id): the k smallest entries form a unique set, whatever order they were seen in.
#include <cmath>

#include "fk_common.cuh"

namespace fk {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------- fp64 tile geometry
// A tile is 32 queries x 128 vectors, 4 warps.  The dot products run on the fp64 tensor
// instruction mma.m8n8k4 (8 queries x 8 vectors x 4 dimensions per instruction): warp w
// covers queries 16 (w >> 1) .. +15 (two 8-row blocks) and vectors 64 (w & 1) .. +63 (eight
// 8-column blocks), so per 4 dimensions it loads 2 + 8 operand fragments for 16 products.
// Blocks of 8 queries or vectors beyond the item's count are skipped.
// Dimensions are staged in chunks of 32 fp32 values per row, copied global -> shared with
// cp.async into two alternating stages (the next chunk lands while this one is used), in
// rows of 36 floats: a fragment read (8 rows x 4 consecutive dimensions) then hits 32
// distinct banks.  Each fragment value is widened to fp64 (exactly) as it is read.  After
// the last chunk the accumulators go through shared memory (rows of 136 doubles, over the
// stages) so that each warp reads whole rows of 128 products.
constexpr int kTQ = 32;
constexpr int kTV = 128;
constexpr int kTD = 32;
constexpr int kS = kTD + 4;
constexpr int kDS = kTV + 8;
constexpr int kTThreads = 128;
constexpr int kStages = 2;

struct StageBuf {
    float q[kTQ * kS];  // [query][dim]
    float v[kTV * kS];  // [vector][dim]
};

struct TileSmem {
    union {
        StageBuf st[kStages];
        double dot[kTQ * kDS];  // [query][vector]: the tile's dot products
    };
};

__device__ __forceinline__ bool before(double da, uint32_t ia, double db, uint32_t ib) {
    return da < db || (da == db && ia < ib);
}

// Exact squared distance of two fp32 rows in fp64 (difference form), a warp cooperating:
// lane l sums the columns 4l .. 4l + 3 (mod 128) in order, then a fixed butterfly; every
// lane returns the same value.
__device__ __forceinline__ double exact_sq_dist(const float *q, const float *x, int d, int lane) {
    double acc = 0.0;
    for (int j = lane * 4; j < d; j += 128) {
        const float4 u = __ldg(reinterpret_cast<const float4 *>(q + j));
        const float4 v = __ldg(reinterpret_cast<const float4 *>(x + j));
        const double e0 = static_cast<double>(u.x) - v.x, e1 = static_cast<double>(u.y) - v.y;
        const double e2 = static_cast<double>(u.z) - v.z, e3 = static_cast<double>(u.w) - v.w;
        acc = fma(e0, e0, acc);
        acc = fma(e1, e1, acc);
        acc = fma(e2, e2, acc);
        acc = fma(e3, e3, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    return acc;
}

// 16-byte global -> shared copy; src_bytes = 0 fills zeros without reading.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Copy chunk j0 .. j0 + 31 of the tile's vectors (rows 0 .. nv - 1 of V) and queries into
// a stage: element f = tid + 128 r is row f / 8, 16-byte column f % 8, so a row's 128-byte
// piece is read by 8 consecutive lanes.  Rows past the data and columns past d are zeros.
__device__ __forceinline__ void stage_issue(StageBuf &sb, const float *V, int nv,
                                            const float *qrow0, const float *qrow1, int d,
                                            int j0, int tid) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int f = tid + kTThreads * r;
        const int row = f >> 3;
        const int j = j0 + (f & 7) * 4;
        const bool ok = row < nv && j < d;
        cp_async16(sb.v + row * kS + (f & 7) * 4, ok ? V + static_cast<int64_t>(row) * d + j : V,
                   ok ? 16 : 0);
    }
    const int j = j0 + (tid & 7) * 4;
    const int qr0 = tid >> 3, qr1 = (tid + kTThreads) >> 3;
    const bool ok0 = qrow0 && j < d, ok1 = qrow1 && j < d;
    cp_async16(sb.q + qr0 * kS + (tid & 7) * 4, ok0 ? qrow0 + j : V, ok0 ? 16 : 0);
    cp_async16(sb.q + qr1 * kS + (tid & 7) * 4, ok1 ? qrow1 + j : V, ok1 ? 16 : 0);
}

// D (8 x 8) += A (8 x 4) B (4 x 8) in fp64.  Fragments: this lane holds A[g][t] and B[t][g]
// and accumulates D[g][2t], D[g][2t + 1], with g = lane / 4 and t = lane % 4.
__device__ __forceinline__ void dmma(double &d0, double &d1, double a, double b) {
    asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
        : "+d"(d0), "+d"(d1)
        : "d"(a), "d"(b));
}

// acc[a][n] += the chunk's dot products of query block (2 wq + a) with vector block
// (8 wp + n), for the mact query blocks and nact vector blocks this warp has.
__device__ __forceinline__ void tile_mma(const StageBuf &sb, int wq, int wp, int lane, int mact,
                                         int nact, double (&acc)[2][8][2]) {
    const int g = lane >> 2, t = lane & 3;
    const float *qa = sb.q + (wq * 16 + g) * kS + t;
    const float *vb = sb.v + (wp * 64 + g) * kS + t;
#pragma unroll
    for (int ks = 0; ks < kTD / 4; ++ks) {
        const double a0 = qa[ks * 4];
        const double a1 = qa[8 * kS + ks * 4];
        double b[8];
#pragma unroll
        for (int n = 0; n < 8; ++n) b[n] = vb[n * 8 * kS + ks * 4];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            if (n < nact) {
                dmma(acc[0][n][0], acc[0][n][1], a0, b[n]);
                if (mact > 1) dmma(acc[1][n][0], acc[1][n][1], a1, b[n]);
            }
        }
    }
}

struct TileArgs {
    const float *Q;       // [nq][d] queries
    const double *qn;     // [nq] ||q||^2
    const float *V;       // COARSE: centroids [nlist][d]; FINE: cell-contiguous points [N][d]
    const double *vn;     // ||v||^2 of the rows of V
    int d;
    // COARSE
    int64_t q0;           // first query of the batch
    int nqb;              // queries in the batch
    int nv;               // centroids
    int vchunk;           // centroids per work item (a multiple of kTV)
    int nvchunks;
    double *D;            // [nqb][nv]
    // FINE
    const int32_t *offsets;      // [nlist + 1] cell starts in V
    const int32_t *row_ids;      // [N] original index of every row of V
    const int32_t *pair_sorted;  // pairs (q * nprobe + t) in cell order
    const int32_t *pair_off;     // [nlist + 1] first sorted position of every cell
    const int2 *items;           // (cell, first sorted position)
    const int *nitems;
    int *item_ctr;               // zero at launch
    int nprobe, k;
    double *Ld;                  // [nq * nprobe][k]
    uint32_t *Li;
};

// COARSE: blockIdx.x = query block * nvchunks + centroid chunk; writes distances.
// FINE: persistent blocks take work items from a counter; writes per-pair top-k lists.
// Padding ids of a pair list are 0x80000000 | (t * k + rank), unique within a query, above
// every point id and recognised as "no point" by the final selection.
template <bool FINE>
__global__ void __launch_bounds__(kTThreads, 4) ivf_tile_kernel(TileArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    TileSmem &sm = *reinterpret_cast<TileSmem *>(smem_raw);
    __shared__ int s_item;
    __shared__ int s_pair[kTQ];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = a.d;

    for (int round = 0;; ++round) {
        int item;
        if (FINE) {
            if (tid == 0) s_item = atomicAdd(a.item_ctr, 1);
            __syncthreads();
            item = s_item;
            if (item >= *a.nitems) return;
        } else {
            if (round > 0) return;
            item = blockIdx.x;
        }
        int nq_i;
        int64_t vbeg, vend, q_first = 0;
        if (FINE) {
            const int2 it = a.items[item];
            nq_i = min(kTQ, a.pair_off[it.x + 1] - it.y);
            vbeg = a.offsets[it.x];
            vend = a.offsets[it.x + 1];
            if (tid < kTQ) s_pair[tid] = tid < nq_i ? a.pair_sorted[it.y + tid] : 0;
        } else {
            const int qb = item / a.nvchunks, vc = item % a.nvchunks;
            q_first = static_cast<int64_t>(qb) * kTQ;
            nq_i = static_cast<int>(min(static_cast<int64_t>(kTQ), a.nqb - q_first));
            vbeg = static_cast<int64_t>(vc) * a.vchunk;
            vend = min(vbeg + a.vchunk, static_cast<int64_t>(a.nv));
        }
        __syncthreads();

        auto query_of = [&](int qi) -> int64_t {
            return FINE ? static_cast<int64_t>(s_pair[qi] / a.nprobe) : a.q0 + q_first + qi;
        };
        const int sq0 = tid >> 3, sq1 = (tid + kTThreads) >> 3;  // query rows this thread stages
        const float *qrow0 = sq0 < nq_i ? a.Q + query_of(sq0) * d : nullptr;
        const float *qrow1 = sq1 < nq_i ? a.Q + query_of(sq1) * d : nullptr;

        // per-pair top-k lists: lane r holds rank r of each of the warp's 8 queries
        double ld[8];
        uint32_t li[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
            ld[q8] = INFINITY;
            li[q8] = 0xffffffffu;
            if (FINE) {
                const int qi = warp * 8 + q8;
                if (qi < nq_i && lane < a.k)
                    li[q8] = 0x80000000u |
                             static_cast<uint32_t>((s_pair[qi] % a.nprobe) * a.k + lane);
            }
        }

        for (int64_t v0 = vbeg; v0 < vend; v0 += kTV) {
            const int nv_t = static_cast<int>(min(static_cast<int64_t>(kTV), vend - v0));
            const float *Vt = a.V + v0 * d;
            // this warp's blocks of 8 queries (of 2) and of 8 vectors (of 8) that hold data
            const int wq = warp >> 1, wp = warp & 1;
            const int mact = max(0, min(2, (nq_i + 7) / 8 - 2 * wq));
            const int nact = max(0, min(8, (nv_t + 7) / 8 - 8 * wp));
            double acc[2][8][2];
#pragma unroll
            for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
                for (int n = 0; n < 8; ++n) acc[a2][n][0] = acc[a2][n][1] = 0.0;
            const int nch = (d + kTD - 1) / kTD;
            __syncthreads();  // the previous tile's readers of the dot rows are done
            stage_issue(sm.st[0], Vt, nv_t, qrow0, qrow1, d, 0, tid);
            cp_async_commit();
            for (int c = 0; c < nch; ++c) {
                cp_async_wait<0>();  // chunk c, the only copy in flight, has landed
                // ... for every thread, and every warp is done with chunk c - 1, whose
                // stage the next copy overwrites
                __syncthreads();
                if (c + 1 < nch) {
                    stage_issue(sm.st[(c + 1) & 1], Vt, nv_t, qrow0, qrow1, d, (c + 1) * kTD, tid);
                    cp_async_commit();
                }
                if (mact > 0) tile_mma(sm.st[c & 1], wq, wp, lane, mact, nact, acc);
            }
            __syncthreads();  // every warp is done with the last stage
            {  // the dot-product rows overwrite the stages (every reader passed the last barrier)
                const int g = lane >> 2, t = lane & 3;
#pragma unroll
                for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
                    for (int n = 0; n < 8; ++n)
                        if (a2 < mact && n < nact)
                            *reinterpret_cast<double2 *>(
                                sm.dot + (wq * 16 + a2 * 8 + g) * kDS + wp * 64 + n * 8 + 2 * t) =
                                make_double2(acc[a2][n][0], acc[a2][n][1]);
            }
            __syncthreads();

            double vn_i[4];
            uint32_t id_i[4];
            bool ok_i[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int vl = lane + 32 * i;
                ok_i[i] = vl < nv_t;
                vn_i[i] = ok_i[i] ? a.vn[v0 + vl] : 0.0;
                id_i[i] = FINE ? (ok_i[i] ? static_cast<uint32_t>(a.row_ids[v0 + vl]) : 0u)
                               : static_cast<uint32_t>(v0 + vl);
            }
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {
                const int qi = warp * 8 + q8;
                if (qi >= nq_i) continue;  // warp-uniform
                const double qn = a.qn[query_of(qi)];
                if (!FINE) {
                    double *Drow = a.D + (q_first + qi) * static_cast<int64_t>(a.nv);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (ok_i[i])
                            Drow[v0 + lane + 32 * i] =
                                fma(-2.0, sm.dot[qi * kDS + lane + 32 * i], qn + vn_i[i]);
                } else {
                    double td = __shfl_sync(kFull, ld[q8], a.k - 1);
                    uint32_t ti = __shfl_sync(kFull, li[q8], a.k - 1);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const double cd = fma(-2.0, sm.dot[qi * kDS + lane + 32 * i], qn + vn_i[i]);
                        const uint32_t ci = id_i[i];
                        bool pend = ok_i[i] && before(cd, ci, td, ti);
                        unsigned m = __ballot_sync(kFull, pend);
                        while (m) {
                            const int src = __ffs(m) - 1;
                            const double xd = __shfl_sync(kFull, cd, src);
                            const uint32_t xi = __shfl_sync(kFull, ci, src);
                            const int pos = __popc(__ballot_sync(
                                kFull, lane < a.k && before(ld[q8], li[q8], xd, xi)));
                            const double ud = __shfl_up_sync(kFull, ld[q8], 1);
                            const uint32_t ui = __shfl_up_sync(kFull, li[q8], 1);
                            if (lane == pos) {
                                ld[q8] = xd;
                                li[q8] = xi;
                            } else if (lane > pos && lane < a.k) {
                                ld[q8] = ud;
                                li[q8] = ui;
                            }
                            td = __shfl_sync(kFull, ld[q8], a.k - 1);
                            ti = __shfl_sync(kFull, li[q8], a.k - 1);
                            if (lane == src) pend = false;
                            pend = pend && before(cd, ci, td, ti);
                            m = __ballot_sync(kFull, pend);
                        }
                    }
                }
            }
        }

        if (FINE) {
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {
                const int qi = warp * 8 + q8;
                if (qi < nq_i && lane < a.k) {
                    const int64_t at = static_cast<int64_t>(s_pair[qi]) * a.k + lane;
                    a.Ld[at] = ld[q8];
                    a.Li[at] = li[q8];
                }
            }
        }
    }
}

// ---------------------------------------------------------------- row selection
// Per row (one block each): the m smallest entries by (distance, id), output in ascending
// order.
// Rows of up to kSelCache entries are staged in shared memory and go through a histogram:
// the fp32 rounding of each distance is mapped linearly onto kSelBins bins between the
// row's smallest and largest finite values (a non-decreasing map of the distance), the bin
// holding the m-th entry is found with a prefix sum, and every entry in it or below is a
// candidate: no entry above it can be among the m smallest.  The candidates (at least m,
// usually a few more) are sorted by (distance, id) and the first m kept.
// A row whose candidates would not fit (many equal distances), and every row too long to
// stage, takes the radix path instead: the m-th smallest 96-bit key (order-preserving
// distance bits, then id) is found digit by digit, 8 bits at a time, with a 256-bin
// histogram of the entries that still match the decided digits, stopping as soon as every
// entry of the chosen bin is inside the first m; exactly m entries are gathered.
constexpr int kSelThreads = 256;
constexpr int kSelCache = 8192;    // rows up to this length are staged in shared memory
constexpr int kSelBins = 2048;     // histogram bins of the staged path
constexpr int kSelMaxCand = 2048;  // candidates the staged path sorts

__device__ __forceinline__ uint64_t order_key(double x) {
    const uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ double key_value(uint64_t k) {
    const uint64_t u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
    return __longlong_as_double(static_cast<long long>(u));
}

struct SelArgs {
    const double *D;    // [rows][ld] distances
    const uint32_t *I;  // [rows][ld] ids, or null: the id of entry j is j
    int64_t ld;
    int L, m;
    int32_t *out_id;    // [rows][ldo]; ids with bit 31 set are written as -1
    float *out_dist;    // optional [rows][ldo]; +inf for those
    int64_t ldo;
};

template <bool CACHE>
__global__ void __launch_bounds__(kSelThreads) select_rows_kernel(SelArgs a) {
    extern __shared__ __align__(16) unsigned char sel_raw[];
    uint64_t *ck = reinterpret_cast<uint64_t *>(sel_raw);
    uint32_t *ci = reinterpret_cast<uint32_t *>(sel_raw + sizeof(uint64_t) * (CACHE ? a.L : 0));
    __shared__ uint32_t hist[kSelBins];  // the radix path uses the first 256
    __shared__ uint64_t sel_k[kSelMaxCand];
    __shared__ uint32_t sel_i[kSelMaxCand];
    __shared__ float s_min[kSelThreads / 32], s_max[kSelThreads / 32];
    __shared__ uint32_t s_wsum[kSelThreads / 32];
    __shared__ uint64_t s_phi;
    __shared__ uint32_t s_plo;
    __shared__ int s_r, s_done, s_cnt, s_bstar, s_ncand;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.x;
    const double *drow = a.D + row * a.ld;
    const uint32_t *irow = a.I ? a.I + row * a.ld : nullptr;
    const int L = a.L, m = a.m;
    const int Lpad = (L + kSelThreads - 1) / kSelThreads * kSelThreads;

    if (tid == 0) {
        s_phi = 0;
        s_plo = 0;
        s_r = m - 1;
        s_done = 0;
        s_cnt = 0;
        s_ncand = kSelMaxCand + 1;
    }
    int n_sel = -1;  // candidates gathered into sel_k / sel_i
    if (CACHE) {
        float lmin = INFINITY, lmax = -INFINITY;
        // eight loads in flight per thread before any is used
        constexpr int kU = 8;
        for (int j0 = tid; j0 < L; j0 += kSelThreads * kU) {
            double x[kU];
            uint32_t id[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int j = j0 + u * kSelThreads;
                x[u] = j < L ? drow[j] : 0.0;
                id[u] = (j < L && irow) ? irow[j] : static_cast<uint32_t>(j);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int j = j0 + u * kSelThreads;
                if (j < L) {
                    ck[j] = order_key(x[u]);
                    ci[j] = id[u];
                    const float fx = static_cast<float>(x[u]);
                    if (fx < INFINITY) {
                        lmin = fminf(lmin, fx);
                        lmax = fmaxf(lmax, fx);
                    }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lmin = fminf(lmin, __shfl_xor_sync(kFull, lmin, o));
            lmax = fmaxf(lmax, __shfl_xor_sync(kFull, lmax, o));
        }
        if (lane == 0) {
            s_min[warp] = lmin;
            s_max[warp] = lmax;
        }
        for (int t = tid; t < kSelBins; t += kSelThreads) hist[t] = 0;
        __syncthreads();
        float fmn = s_min[0], fmx = s_max[0];
#pragma unroll
        for (int w = 1; w < kSelThreads / 32; ++w) {
            fmn = fminf(fmn, s_min[w]);
            fmx = fmaxf(fmx, s_max[w]);
        }
        const float scale = fmx > fmn ? static_cast<float>(kSelBins - 1) / (fmx - fmn) : 0.f;
        auto bin_of = [&](uint64_t k) -> int {
            const float fx = static_cast<float>(key_value(k));
            if (!(fx < fmx)) return kSelBins - 1;  // the largest finite value and +inf
            const int bq = static_cast<int>((fx - fmn) * scale);
            return bq < 0 ? 0 : (bq > kSelBins - 1 ? kSelBins - 1 : bq);
        };
        for (int j = tid; j < L; j += kSelThreads) atomicAdd(&hist[bin_of(ck[j])], 1u);
        __syncthreads();
        // prefix over the bins: thread t owns bins 8t .. 8t + 7
        constexpr int kPer = kSelBins / kSelThreads;
        uint32_t h[kPer], sum = 0;
#pragma unroll
        for (int t = 0; t < kPer; ++t) {
            h[t] = hist[tid * kPer + t];
            sum += h[t];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        uint32_t base = 0;
        for (int w = 0; w < warp; ++w) base += s_wsum[w];
        uint32_t c = base + incl - sum;  // entries in bins below 8 tid
        const uint32_t need = static_cast<uint32_t>(m);
        if (c < need && need <= c + sum) {
#pragma unroll
            for (int t = 0; t < kPer; ++t) {
                if (c < need && need <= c + h[t]) {
                    s_bstar = tid * kPer + t;
                    s_ncand = static_cast<int>(c + h[t]);
                }
                c += h[t];
            }
        }
        __syncthreads();
        if (s_ncand <= kSelMaxCand) {
            const int bstar = s_bstar;
            for (int j = tid; j < L; j += kSelThreads) {
                const uint64_t kh = ck[j];
                if (bin_of(kh) <= bstar) {
                    const int at = atomicAdd(&s_cnt, 1);
                    sel_k[at] = kh;
                    sel_i[at] = ci[j];
                }
            }
            n_sel = s_ncand;
        }
        __syncthreads();
    }
    auto load = [&](int j, uint64_t &kh, uint32_t &kl) {
        if (CACHE) {
            kh = ck[j];
            kl = ci[j];
        } else {
            kh = order_key(drow[j]);
            kl = irow ? irow[j] : static_cast<uint32_t>(j);
        }
    };
    if (n_sel < 0) {
        auto hi_mask = [](int b) -> uint64_t {
            return b >= 8 ? ~0ull : (b == 0 ? 0ull : ~0ull << (64 - 8 * b));
        };
        auto lo_mask = [](int b) -> uint32_t { return b <= 8 ? 0u : ~0u << (32 - 8 * (b - 8)); };
        int b = 0;
        while (b < 12) {
            hist[tid] = 0;
            __syncthreads();
            const uint64_t phi = s_phi, mhi = hi_mask(b);
            const uint32_t plo = s_plo, mlo = lo_mask(b);
            for (int j = tid; j < Lpad; j += kSelThreads) {
                uint64_t kh = 0;
                uint32_t kl = 0;
                const bool valid = j < L;
                if (valid) load(j, kh, kl);
                const bool match = valid && (kh & mhi) == phi && (kl & mlo) == plo;
                int dig = b < 8 ? static_cast<int>((kh >> (56 - 8 * b)) & 255u)
                                : static_cast<int>((kl >> (24 - 8 * (b - 8))) & 255u);
                dig = match ? dig : 256;
                const unsigned peers = __match_any_sync(kFull, dig);
                if (match && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], __popc(peers));
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t h[8], sum = 0;
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    h[t] = hist[lane * 8 + t];
                    sum += h[t];
                }
                uint32_t incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(kFull, incl, o);
                    if (lane >= o) incl += y;
                }
                const uint32_t excl = incl - sum;
                const uint32_t r = static_cast<uint32_t>(s_r);
                if (excl <= r && r < incl) {
                    uint32_t c = excl;
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        if (r >= c && r < c + h[t]) {
                            const uint32_t bin = lane * 8 + t;
                            if (b < 8)
                                s_phi = phi | (static_cast<uint64_t>(bin) << (56 - 8 * b));
                            else
                                s_plo = plo | (bin << (24 - 8 * (b - 8)));
                            s_r = static_cast<int>(r - c);
                            s_done = (r - c + 1 == h[t]) ? 1 : 0;
                        }
                        c += h[t];
                    }
                }
            }
            __syncthreads();
            ++b;
            if (s_done) break;
        }
        // every entry whose first b digits are at most the decided prefix: exactly m
        const uint64_t phi = s_phi, mhi = hi_mask(b);
        const uint32_t plo = s_plo, mlo = lo_mask(b);
        for (int j = tid; j < L; j += kSelThreads) {
            uint64_t kh;
            uint32_t kl;
            load(j, kh, kl);
            const uint64_t th = kh & mhi;
            const uint32_t tl = kl & mlo;
            if (th < phi || (th == phi && tl <= plo)) {
                const int at = atomicAdd(&s_cnt, 1);
                if (at < kSelMaxCand) {
                    sel_k[at] = kh;
                    sel_i[at] = kl;
                }
            }
        }
        n_sel = m;
    }
    int M = 1;
    while (M < n_sel) M <<= 1;
    __syncthreads();
    for (int t = n_sel + tid; t < M; t += kSelThreads) {
        sel_k[t] = ~0ull;
        sel_i[t] = ~0u;
    }
    __syncthreads();
    for (int size = 2; size <= M; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < (M >> 1); t += kSelThreads) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const uint64_t ka = sel_k[lo], kb = sel_k[hi];
                const uint32_t ia = sel_i[lo], ib = sel_i[hi];
                const bool gt = ka > kb || (ka == kb && ia > ib);
                if (gt == up) {
                    sel_k[lo] = kb;
                    sel_k[hi] = ka;
                    sel_i[lo] = ib;
                    sel_i[hi] = ia;
                }
            }
            __syncthreads();
        }
    }
    for (int t = tid; t < m; t += kSelThreads) {
        const uint32_t id = sel_i[t];
        const bool pad = (id & 0x80000000u) != 0;
        a.out_id[row * a.ldo + t] = pad ? -1 : static_cast<int32_t>(id);
        if (a.out_dist)
            a.out_dist[row * a.ldo + t] =
                pad ? INFINITY : static_cast<float>(fmax(key_value(sel_k[t]), 0.0));
    }
}

// ---------------------------------------------------------------- screened coarse pass
// The coarse distances as a dense product on the tensor cores: the single-product pass of
// the assignment kernel (one bf16 product per term, norms folded in exactly) writes the
// screened value v~ = ||c||^2 - 2 q~.c~ of every (query, centroid), each within E of the
// exact ||c||^2 - 2 q.c (screen_window).  Per query, if T~ is the nprobe-th smallest
// screened value, every centroid among the nprobe nearest has v~ <= T~ + 2E; those
// candidates are re-ranked exactly (fp64, difference form) and the nprobe smallest by
// (distance, cell) kept.  The same probes as the fp64 coarse pass, for a fraction of the
// work; only the candidates (typically a few more than nprobe) see fp64 arithmetic.
constexpr int kCoarseThreads = 256;
constexpr int kCoarseMaxL = 8192;  // centroids a block stages

struct CoarseArgs {
    const float *V;        // [rows][ldv] screened values of the batch
    int64_t ldv;
    int L, m;              // centroids, probes
    const float *Q;        // fp32 queries; row q0 + r is the block's
    int64_t q0;
    const float *C;        // fp32 centroids [L][d]
    int d, dp;             // dimension, and the padded width the screening pass ran over
    const float *xnorm;    // [nq] ||q||^2 (fp32) the window is derived from
    const float *cmax2;    // max_k ||c_k||^2
    int32_t *probes;       // [nq][m]
};

__device__ __forceinline__ uint32_t fkey(float x) {
    const uint32_t u = __float_as_uint(x);
    return (u >> 31) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_value(uint32_t k) {
    return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k);
}

__global__ void __launch_bounds__(kCoarseThreads) coarse_rerank_kernel(CoarseArgs a) {
    extern __shared__ __align__(16) unsigned char co_raw[];
    int P = 1;
    while (P < a.L) P <<= 1;
    double *cd = reinterpret_cast<double *>(co_raw);               // [P] candidate distances
    uint32_t *cid = reinterpret_cast<uint32_t *>(cd + P);          // [P] candidate cells
    uint32_t *key = cid + P;                                       // [L] screened-value keys
    __shared__ uint32_t hist[kSelBins];
    __shared__ float s_min[kCoarseThreads / 32], s_max[kCoarseThreads / 32];
    __shared__ uint32_t s_wsum[kCoarseThreads / 32];
    __shared__ int s_bstar, s_n;
    __shared__ uint32_t s_tmax;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r = blockIdx.x;
    const int64_t q = a.q0 + r;
    const float *vrow = a.V + r * a.ldv;
    const int L = a.L, m = a.m;
    if (tid == 0) {
        s_n = 0;
        s_tmax = 0u;
    }
    for (int t = tid; t < kSelBins; t += kCoarseThreads) hist[t] = 0;

    // 1. the row's screened values, as order keys, and their range
    float lmin = INFINITY, lmax = -INFINITY;
    constexpr int kU = 8;
    for (int j0 = tid; j0 < L; j0 += kCoarseThreads * kU) {
        float x[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int j = j0 + u * kCoarseThreads;
            x[u] = j < L ? vrow[j] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int j = j0 + u * kCoarseThreads;
            if (j < L) {
                key[j] = fkey(x[u]);
                lmin = fminf(lmin, x[u]);
                lmax = fmaxf(lmax, x[u]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lmin = fminf(lmin, __shfl_xor_sync(kFull, lmin, o));
        lmax = fmaxf(lmax, __shfl_xor_sync(kFull, lmax, o));
    }
    if (lane == 0) {
        s_min[warp] = lmin;
        s_max[warp] = lmax;
    }
    __syncthreads();
    float fmn = s_min[0], fmx = s_max[0];
#pragma unroll
    for (int w = 1; w < kCoarseThreads / 32; ++w) {
        fmn = fminf(fmn, s_min[w]);
        fmx = fmaxf(fmx, s_max[w]);
    }
    const float scale = fmx > fmn ? static_cast<float>(kSelBins - 1) / (fmx - fmn) : 0.f;
    auto bin_of = [&](uint32_t k) -> int {
        const float x = fkey_value(k);
        if (!(x < fmx)) return kSelBins - 1;
        const int b = static_cast<int>((x - fmn) * scale);
        return b < 0 ? 0 : (b > kSelBins - 1 ? kSelBins - 1 : b);
    };
    // 2. histogram; the bin holding the m-th smallest value
    for (int j = tid; j < L; j += kCoarseThreads) atomicAdd(&hist[bin_of(key[j])], 1u);
    __syncthreads();
    constexpr int kPer = kSelBins / kCoarseThreads;
    uint32_t h[kPer], sum = 0;
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
        h[t] = hist[tid * kPer + t];
        sum += h[t];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    {
        uint32_t c = incl - sum;
        for (int w = 0; w < warp; ++w) c += s_wsum[w];
        const uint32_t need = static_cast<uint32_t>(m);
        if (c < need && need <= c + sum) {
#pragma unroll
            for (int t = 0; t < kPer; ++t) {
                if (c < need && need <= c + h[t]) s_bstar = tid * kPer + t;
                c += h[t];
            }
        }
    }
    __syncthreads();
    // 3. T~ <= the largest value in that bin; candidates within the window above it
    const int bstar = s_bstar;
    for (int j = tid; j < L; j += kCoarseThreads)
        if (bin_of(key[j]) == bstar) atomicMax(&s_tmax, key[j]);
    __syncthreads();
    const float W = screen_window(a.xnorm[q], *a.cmax2, a.dp);
    const uint32_t kthr = fkey(fkey_value(s_tmax) + W);
    for (int j = tid; j < L; j += kCoarseThreads)
        if (key[j] <= kthr) cid[atomicAdd(&s_n, 1)] = static_cast<uint32_t>(j);
    __syncthreads();
    const int n = s_n;
    // 4. exact fp64 distance of each candidate, a warp each: fixed lane split, fixed tree
    // (coalesced 512-byte reads of the L2-resident centroid rows; measured faster than a
    // lane per candidate)
    const float *qv = a.Q + q * a.d;
    for (int t = warp; t < n; t += kCoarseThreads / 32) {
        const double e = exact_sq_dist(qv, a.C + static_cast<int64_t>(cid[t]) * a.d, a.d, lane);
        if (lane == 0) cd[t] = e;
    }
    // 5. sort the candidates by (distance, cell) and keep the first m
    int M = 1;
    while (M < n) M <<= 1;
    for (int t = n + tid; t < M; t += kCoarseThreads) {
        cd[t] = INFINITY;
        cid[t] = ~0u;
    }
    __syncthreads();
    for (int size = 2; size <= M; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < (M >> 1); t += kCoarseThreads) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const double da = cd[lo], db = cd[hi];
                const uint32_t ia = cid[lo], ib = cid[hi];
                const bool gt = da > db || (da == db && ia > ib);
                if (gt == up) {
                    cd[lo] = db;
                    cd[hi] = da;
                    cid[lo] = ib;
                    cid[hi] = ia;
                }
            }
            __syncthreads();
        }
    }
    for (int t = tid; t < m; t += kCoarseThreads)
        a.probes[q * m + t] = static_cast<int32_t>(cid[t]);
}

// max_k ||c_k||^2 over the real centroids (one block).
__global__ void cmax_kernel(const float *__restrict__ cn, int K, float *__restrict__ out) {
    __shared__ float red[32];
    float mx = 0.f;
    for (int k = threadIdx.x; k < K; k += blockDim.x) mx = fmaxf(mx, cn[k]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x < 32) {
        mx = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
        if (threadIdx.x == 0) *out = mx;
    }
}

// ---------------------------------------------------------------- screened fine pass
// The fine products on the tensor cores.  Each (query, point) dot product is taken as three
// bf16 products of the RN-bf16 split x = hi + lo (+ a residual below 2^-16 |x|) of both
// sides, hi.hi + hi.lo + lo.hi, accumulated in fp32 by mma.m16n8k16; the screened distance
// s~ = ||q||^2 + ||x||^2 - 2 q.x~ (rounded to fp32) is within E(q) of the exact one
// (fine_window_coeffs).  Per pair a lane-held list keeps the kScrList smallest s~ with the points'
// positions, and the smallest s~ it dropped ("lost").  query_rerank_kernel merges a query's
// lists: every point of the exact top-k has s~ within 2E of the k-th smallest s~, so
// re-ranking those entries in fp64 gives the exact result -- unless a pair dropped an
// entry inside that window, which sends the query to fallback_kernel.
// Tile: 128 points x 32 queries; warp w owns points 32w .. 32w + 31 (two 16-row blocks)
// and all four 8-query blocks.  bf16 chunks of 32 dimensions of both planes arrive by
// cp.async in two stages, rows of 40 elements (80 bytes: the 8 rows an ldmatrix reads
// fall on distinct banks).  Measured on B200: a 4-stage pipeline (2 blocks per SM) and an
// XOR-swizzled unpadded layout were both slower than this (4 blocks per SM).
constexpr int kScrList = kSearchScrList;  // entries per pair list, one per lane
constexpr int kBS = kTD + 8;   // bf16 row stride of a stage: 80 bytes, so the 8 rows an
                               // ldmatrix reads fall on distinct banks
constexpr int kDSF = kTV + 4;  // fp32 row stride of the dot-product rows
constexpr int kFineStages = 2; // chunks in flight: one behind the one in use

struct StageB {
    uint16_t vh[kTV * kBS], vl[kTV * kBS];  // points: hi, lo
    uint16_t qh[kTQ * kBS], ql[kTQ * kBS];  // queries: hi, lo
};

struct FineSmem {
    union {
        StageB st[kFineStages];
        float dot[kTQ * kDSF];  // [query][point]
    };
};

// Element offset of 16-byte piece `piece` of stage row `row`.
__device__ __forceinline__ int swz(int row, int piece) { return row * kBS + (piece << 3); }

struct FineArgs {
    const uint16_t *Qp;        // [2][nq][dp] bf16 planes of the queries
    int64_t nq;
    const uint16_t *Xp;        // [2][N][dp] bf16 planes of the cell-ordered points
    int64_t N;
    int dp;
    const double *qn, *xn;     // fp64 squared norms
    const int32_t *offsets, *pair_sorted, *pair_off;
    const int2 *items;
    const int *nitems;
    int *item_ctr;
    int nprobe;
    float *Sv;                 // [P][kScrList] screened values, ascending
    uint32_t *Sp;              // [P][kScrList] point positions (0xffffffff: no point)
    float *Slost;              // [P]
    const float *cut;          // optional [nq]: screened values above it are dropped uncounted
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a)
                 : "memory");
}

// C (16 x 8, fp32) += A (16 x 16, bf16, row) B (16 x 8, bf16, col).  This lane holds
// A[g][2t..], A[g+8][2t..], A[g][2t+8..], A[g+8][2t+8..], B[2t..][g], B[2t+8..][g] and
// C[g][2t], C[g][2t+1], C[g+8][2t], C[g+8][2t+1], with g = lane / 4, t = lane % 4.
__device__ __forceinline__ void hmma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                     uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Chunk j0 .. j0 + 31 of both planes of the tile's points (rows 0 .. nv - 1 from v0) and
// of the item's queries: thread t copies 16-byte piece t % 4 of point rows t / 4 + 32 r
// and of query row t / 4.  Rows past the data are zeros.
__device__ __forceinline__ void stage_issue_b(StageB &sb, const uint16_t *Xh, const uint16_t *Xl,
                                              int64_t v0, int nv, int dp, const uint16_t *qh,
                                              const uint16_t *ql, int j0, int tid) {
    const int c16 = tid & 3;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int row = (tid >> 2) + 32 * r;
        const bool ok = row < nv;
        const int64_t off = ok ? (v0 + row) * dp + j0 + c16 * 8 : 0;
        cp_async16(sb.vh + swz(row, c16), Xh + off, ok ? 16 : 0);
        cp_async16(sb.vl + swz(row, c16), Xl + off, ok ? 16 : 0);
    }
    const int qr = tid >> 2;
    cp_async16(sb.qh + swz(qr, c16), qh ? qh + j0 + c16 * 8 : Xh, qh ? 16 : 0);
    cp_async16(sb.ql + swz(qr, c16), ql ? ql + j0 + c16 * 8 : Xh, ql ? 16 : 0);
}

// acc[m][n] += the chunk's three-product dot products of point block (2 warp + m) with
// query block n, for the mact point blocks and nact query blocks that hold data.
__device__ __forceinline__ void fine_mma(const StageB &sb, int warp, int lane, int mact,
                                         int nact, float (&acc)[2][4][4]) {
    const int i = lane >> 3, r = lane & 7;
#pragma unroll
    for (int ks = 0; ks < kTD / 16; ++ks) {
        uint32_t bh[2][4], bl[2][4];
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            if (2 * np < nact) {
                const int q = np * 16 + (i >> 1) * 8 + r;
                const int piece = ks * 2 + (i & 1);
                ldsm_x4(bh[np], sb.qh + swz(q, piece));
                ldsm_x4(bl[np], sb.ql + swz(q, piece));
            }
        }
        uint32_t ah[2][4], al[2][4];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            if (m < mact) {
                const int p = warp * 32 + m * 16 + (i & 1) * 8 + r;
                const int piece = ks * 2 + (i >> 1);
                ldsm_x4(ah[m], sb.vh + swz(p, piece));
                ldsm_x4(al[m], sb.vl + swz(p, piece));
            }
        }
        // one product at a time over all eight accumulators, so that consecutive
        // instructions do not wait on one another
#pragma unroll
        for (int prod = 0; prod < 3; ++prod) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    if (m < mact && n < nact) {
                        const int o = (n & 1) * 2;
                        const uint32_t(&aa)[4] = prod == 2 ? al[m] : ah[m];
                        const uint32_t *bb = prod == 1 ? bl[n >> 1] : bh[n >> 1];
                        hmma(acc[m][n], aa, bb[o], bb[o + 1]);
                    }
                }
            }
        }
    }
}

__device__ __forceinline__ bool before_f(float a, uint32_t pa, float b, uint32_t pb) {
    return a < b || (a == b && pa < pb);
}

__global__ void __launch_bounds__(kTThreads, 4) ivf_fine_scr_kernel(FineArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    FineSmem &sm = *reinterpret_cast<FineSmem *>(smem_raw);
    __shared__ int s_item;
    __shared__ int s_pair[kTQ];
    __shared__ double s_qn[kTQ];
    __shared__ float s_cut[kTQ];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int dp = a.dp;
    const uint16_t *Xh = a.Xp, *Xl = a.Xp + a.N * dp;
    const uint16_t *Qh = a.Qp, *Ql = a.Qp + a.nq * dp;

    for (;;) {
        if (tid == 0) s_item = atomicAdd(a.item_ctr, 1);
        __syncthreads();
        const int item = s_item;
        if (item >= *a.nitems) return;
        const int2 it = a.items[item];
        const int nq_i = min(kTQ, a.pair_off[it.x + 1] - it.y);
        const int64_t vbeg = a.offsets[it.x], vend = a.offsets[it.x + 1];
        if (tid < kTQ) {
            const int pr = tid < nq_i ? a.pair_sorted[it.y + tid] : 0;
            s_pair[tid] = pr;
            const int64_t qg = pr / a.nprobe;
            s_qn[tid] = tid < nq_i ? a.qn[qg] : 0.0;
            s_cut[tid] = (tid < nq_i && a.cut) ? a.cut[qg] : INFINITY;
        }
        __syncthreads();

        const int sq = tid >> 2;  // the query row this thread stages
        const int64_t qrow = sq < nq_i ? static_cast<int64_t>(s_pair[sq] / a.nprobe) * dp : -1;
        const uint16_t *qh = qrow >= 0 ? Qh + qrow : nullptr;
        const uint16_t *ql = qrow >= 0 ? Ql + qrow : nullptr;
        const int nact = (nq_i + 7) >> 3;

        // per-pair lists: lane r holds rank r of each of the warp's 8 queries
        float lv[8], lost[8];
        uint32_t lp[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
            lv[q8] = INFINITY;
            lp[q8] = 0xffffffffu;
            lost[q8] = INFINITY;
        }

        for (int64_t v0 = vbeg; v0 < vend; v0 += kTV) {
            const int nv_t = static_cast<int>(min(static_cast<int64_t>(kTV), vend - v0));
            const int mact = max(0, min(2, (nv_t + 15) / 16 - 2 * warp));
            float acc[2][4][4];
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int n = 0; n < 4; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;
            const int nch = dp / kTD;
            __syncthreads();  // the previous tile's readers of the dot rows are done
#pragma unroll
            for (int c = 0; c < kFineStages - 1; ++c) {  // every commit makes one group
                if (c < nch)
                    stage_issue_b(sm.st[c], Xh, Xl, v0, nv_t, dp, qh, ql, c * kTD, tid);
                cp_async_commit();
            }
            for (int c = 0; c < nch; ++c) {
                cp_async_wait<kFineStages - 2>();  // chunk c has landed for this thread
                // ... for every thread, and every warp is done with chunk c - 1, whose stage
                // the copy below refills
                __syncthreads();
                const int cn = c + kFineStages - 1;
                if (cn < nch)
                    stage_issue_b(sm.st[cn % kFineStages], Xh, Xl, v0, nv_t, dp, qh, ql, cn * kTD,
                                  tid);
                cp_async_commit();
                if (mact > 0) fine_mma(sm.st[c % kFineStages], warp, lane, mact, nact, acc);
            }
            cp_async_wait<0>();
            __syncthreads();  // every warp is done with the last stage
            {
                const int g = lane >> 2, t = lane & 3;
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int n = 0; n < 4; ++n)
                        if (m < mact && n < nact) {
                            const int p = warp * 32 + m * 16 + g, q = n * 8 + 2 * t;
                            sm.dot[q * kDSF + p] = acc[m][n][0];
                            sm.dot[(q + 1) * kDSF + p] = acc[m][n][1];
                            sm.dot[q * kDSF + p + 8] = acc[m][n][2];
                            sm.dot[(q + 1) * kDSF + p + 8] = acc[m][n][3];
                        }
            }
            __syncthreads();

            double xn_i[4];
            bool ok_i[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int vl = lane + 32 * i;
                ok_i[i] = vl < nv_t;
                xn_i[i] = ok_i[i] ? a.xn[v0 + vl] : 0.0;
            }
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {
                const int qi = warp * 8 + q8;
                if (qi >= nq_i) continue;  // warp-uniform
                const double qn = s_qn[qi];
                const float cut = s_cut[qi];
                float tv = __shfl_sync(kFull, lv[q8], kScrList - 1);
                uint32_t tp = __shfl_sync(kFull, lp[q8], kScrList - 1);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float cv = ok_i[i] ? static_cast<float>(fma(
                                                   -2.0, static_cast<double>(sm.dot[qi * kDSF + lane + 32 * i]),
                                                   qn + xn_i[i]))
                                             : INFINITY;
                    const uint32_t cp = static_cast<uint32_t>(v0 + lane + 32 * i);
                    const bool in = ok_i[i] && cv <= cut;  // else outside every window
                    bool pend = in && before_f(cv, cp, tv, tp);
                    if (in && !pend) lost[q8] = fminf(lost[q8], cv);
                    unsigned m = __ballot_sync(kFull, pend);
                    while (m) {
                        const int src = __ffs(m) - 1;
                        const float xv = __shfl_sync(kFull, cv, src);
                        const uint32_t xp = __shfl_sync(kFull, cp, src);
                        const int pos = __popc(__ballot_sync(kFull, before_f(lv[q8], lp[q8], xv, xp)));
                        // the last entry leaves a full list: it joins the dropped values
                        if (lane == kScrList - 1 && lp[q8] != 0xffffffffu)
                            lost[q8] = fminf(lost[q8], lv[q8]);
                        const float uv = __shfl_up_sync(kFull, lv[q8], 1);
                        const uint32_t up = __shfl_up_sync(kFull, lp[q8], 1);
                        if (lane == pos) {
                            lv[q8] = xv;
                            lp[q8] = xp;
                        } else if (lane > pos) {
                            lv[q8] = uv;
                            lp[q8] = up;
                        }
                        tv = __shfl_sync(kFull, lv[q8], kScrList - 1);
                        tp = __shfl_sync(kFull, lp[q8], kScrList - 1);
                        if (lane == src) pend = false;
                        if (pend && !before_f(cv, cp, tv, tp)) {
                            pend = false;
                            lost[q8] = fminf(lost[q8], cv);
                        }
                        m = __ballot_sync(kFull, pend);
                    }
                }
            }
        }

#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
            const int qi = warp * 8 + q8;
            if (qi >= nq_i) continue;
            float lo = lost[q8];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lo = fminf(lo, __shfl_xor_sync(kFull, lo, o));
            const int64_t pr = s_pair[qi];
            a.Sv[pr * kScrList + lane] = lv[q8];
            a.Sp[pr * kScrList + lane] = lp[q8];
            if (lane == 0) a.Slost[pr] = lo;
        }
    }
}

// Per query (one block): the nprobe pair lists merged.  T~ bounds the k-th smallest screened
// value from above (the largest value of the histogram bin holding it); every point of the
// exact top-k has s~ <= T~ + W, W = 2 E(q).  If a pair dropped a value at or below that,
// its list may lack such a point: the query is flagged for fallback_kernel.  Otherwise the
// entries up to T~ + W are re-ranked exactly (fp64, difference form; a warp per entry) and
// the k smallest by (distance, original id) written.
constexpr int kQThreads = 256;

struct QueryArgs {
    const float *Sv;
    const uint32_t *Sp;
    const float *Slost;
    int nprobe, k;
    const float *Q, *X;        // fp32 queries [nq][d] and cell-ordered points [N][d]
    int d;
    const double *qn;          // fp64 ||q||^2
    const float *xmax2;        // max ||x||^2 over the points
    float ce_dot;              // |s~ - s| <= ce_dot ||q|| ||x|| + ce_round (||q||^2 + ||x||^2)
    float ce_round;
    const int32_t *row_ids;
    float *out_dist;
    int32_t *out_id;
    int32_t *fallback;         // [nq]: 1 for queries left to fallback_kernel
    const float *cut;          // optional [nq]: the fine pass's cut (query_cut_kernel)
};


__global__ void __launch_bounds__(kQThreads) query_rerank_kernel(QueryArgs a) {
    extern __shared__ __align__(16) unsigned char qr_raw[];
    const int L = a.nprobe * kScrList;
    int P2 = 1;
    while (P2 < L) P2 <<= 1;
    double *cd = reinterpret_cast<double *>(qr_raw);           // [P2] candidate distances
    uint32_t *cid = reinterpret_cast<uint32_t *>(cd + P2);     // [P2] candidate ids
    uint32_t *cpos = cid + P2;                                 // [P2] candidate positions
    uint32_t *key = cpos + P2;                                 // [L] screened-value keys
    __shared__ uint32_t hist[kSelBins];
    __shared__ float s_min[kQThreads / 32], s_max[kQThreads / 32];
    __shared__ uint32_t s_wsum[kQThreads / 32];
    __shared__ int s_bstar, s_n, s_over, s_cbelow, s_nb;
    __shared__ uint32_t s_tmax, s_tk;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t q = blockIdx.x;
    const float *sv = a.Sv + q * L;
    const uint32_t *sp = a.Sp + q * L;
    const int k = a.k;
    if (tid == 0) {
        s_n = 0;
        s_nb = 0;
        s_tmax = 0u;
        s_over = 0;
    }
    for (int t = tid; t < kSelBins; t += kQThreads) hist[t] = 0;
    float lmin = INFINITY, lmax = -INFINITY;
    for (int j = tid; j < L; j += kQThreads) {
        const float v = sv[j];
        key[j] = fkey(v);
        if (v < INFINITY) {
            lmin = fminf(lmin, v);
            lmax = fmaxf(lmax, v);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lmin = fminf(lmin, __shfl_xor_sync(kFull, lmin, o));
        lmax = fmaxf(lmax, __shfl_xor_sync(kFull, lmax, o));
    }
    if (lane == 0) {
        s_min[warp] = lmin;
        s_max[warp] = lmax;
    }
    __syncthreads();
    float fmn = s_min[0], fmx = s_max[0];
#pragma unroll
    for (int w = 1; w < kQThreads / 32; ++w) {
        fmn = fminf(fmn, s_min[w]);
        fmx = fmaxf(fmx, s_max[w]);
    }
    const float scale = fmx > fmn ? static_cast<float>(kSelBins - 1) / (fmx - fmn) : 0.f;
    auto bin_of = [&](uint32_t kk) -> int {
        const float x = fkey_value(kk);
        if (!(x < fmx)) return kSelBins - 1;
        const int b = static_cast<int>((x - fmn) * scale);
        return b < 0 ? 0 : (b > kSelBins - 1 ? kSelBins - 1 : b);
    };
    for (int j = tid; j < L; j += kQThreads) atomicAdd(&hist[bin_of(key[j])], 1u);
    __syncthreads();
    constexpr int kPer = kSelBins / kQThreads;
    uint32_t h[kPer], sum = 0;
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
        h[t] = hist[tid * kPer + t];
        sum += h[t];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    {
        uint32_t c = incl - sum;
        for (int w = 0; w < warp; ++w) c += s_wsum[w];
        const uint32_t need = static_cast<uint32_t>(k);
        if (c < need && need <= c + sum) {
#pragma unroll
            for (int t = 0; t < kPer; ++t) {
                if (c < need && need <= c + h[t]) {
                    s_bstar = tid * kPer + t;
                    s_cbelow = static_cast<int>(c);
                }
                c += h[t];
            }
        }
    }
    __syncthreads();
    // T~: the k-th smallest screened value, ranked exactly among the entries of its bin
    // (or, for a bin of more than kQRank entries, the bin's largest value: an upper bound)
    constexpr int kQRank = 1024;
    const int bstar = s_bstar;
    for (int j = tid; j < L; j += kQThreads)
        if (bin_of(key[j]) == bstar) {
            const int at = atomicAdd(&s_nb, 1);
            if (at < kQRank && at < P2) {  // the candidate buffers are free until later
                cid[at] = key[j];
                cpos[at] = static_cast<uint32_t>(j);
            }
            atomicMax(&s_tmax, key[j]);
        }
    __syncthreads();
    const int nb = s_nb;
    if (nb > kQRank || nb > P2) {
        if (tid == 0) s_tk = s_tmax;
    } else {
        const int want = k - 1 - s_cbelow;  // 0-based rank inside the bin
        for (int u = tid; u < nb; u += kQThreads) {
            const uint32_t ku = cid[u], ju = cpos[u];
            int rank = 0;
            for (int v = 0; v < nb; ++v)
                rank += (cid[v] < ku || (cid[v] == ku && cpos[v] < ju)) ? 1 : 0;
            if (rank == want) s_tk = ku;
        }
    }
    __syncthreads();
    const double qn = a.qn[q];
    const float xm2 = *a.xmax2;
    const float E = a.ce_dot * sqrtf(static_cast<float>(qn) * xm2) +
                    a.ce_round * (static_cast<float>(qn) + xm2);
    const float thr = fkey_value(s_tk) + 2.f * E;  // +inf when fewer than k points exist
    const uint32_t kthr = fkey(thr);
    for (int t = tid; t < a.nprobe; t += kQThreads)
        if (a.Slost[q * a.nprobe + t] < INFINITY && a.Slost[q * a.nprobe + t] <= thr) s_over = 1;
    if (tid == 0 && a.cut && !(thr <= a.cut[q])) s_over = 1;  // the cut dropped values uncounted
    __syncthreads();  // the ranking's use of the candidate buffers is over
    for (int j = tid; j < L; j += kQThreads)
        if (key[j] <= kthr && sp[j] != 0xffffffffu) cpos[atomicAdd(&s_n, 1)] = sp[j];
    __syncthreads();
    if (s_over) {
        if (tid == 0) a.fallback[q] = 1;
        return;
    }
    if (tid == 0) a.fallback[q] = 0;
    const int n = s_n;
    const float *qv = a.Q + q * a.d;
    for (int t = warp; t < n; t += kQThreads / 32) {
        const uint32_t pos = cpos[t];
        const double e = exact_sq_dist(qv, a.X + static_cast<int64_t>(pos) * a.d, a.d, lane);
        if (lane == 0) {
            cd[t] = e;
            cid[t] = static_cast<uint32_t>(a.row_ids[pos]);
        }
    }
    int M = 1;
    while (M < n) M <<= 1;
    for (int t = n + tid; t < M; t += kQThreads) {
        cd[t] = INFINITY;
        cid[t] = ~0u;
    }
    __syncthreads();
    for (int size = 2; size <= M; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < (M >> 1); t += kQThreads) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const double da = cd[lo], db = cd[hi];
                const uint32_t ia = cid[lo], ib = cid[hi];
                const bool gt = da > db || (da == db && ia > ib);
                if (gt == up) {
                    cd[lo] = db;
                    cd[hi] = da;
                    cid[lo] = ib;
                    cid[hi] = ia;
                }
            }
            __syncthreads();
        }
    }
    for (int t = tid; t < k; t += kQThreads) {
        const bool real = t < n;
        a.out_id[q * k + t] = real ? static_cast<int32_t>(cid[t]) : -1;
        a.out_dist[q * k + t] = real ? static_cast<float>(cd[t]) : INFINITY;
    }
}

// Queries whose pair lists may have dropped a point of their top-k: the exact k nearest
// over every point of the probed cells.  Each lane takes a whole point (fp64, difference
// form, in dimension order), so a warp streams 32 rows at once; each warp keeps a
// lane-held list, and the eight lists are merged.  Rarely taken (many points whose
// screened distances fall within 2E of one another in one cell).
struct FallbackArgs {
    const int32_t *fallback;
    const int32_t *probes;
    int nprobe, k;
    const float *Q, *X;
    int d;
    const int32_t *offsets, *row_ids;
    float *out_dist;
    int32_t *out_id;
};

__global__ void __launch_bounds__(kQThreads) fallback_kernel(FallbackArgs a) {
    __shared__ double s_d[kQThreads];
    __shared__ uint32_t s_i[kQThreads];
    const int64_t q = blockIdx.x;
    if (a.fallback[q] == 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k, d = a.d;
    const float *qv = a.Q + q * d;
    double ld = INFINITY;
    uint32_t li = 0xffffffffu;
    double td = INFINITY;
    uint32_t ti = 0xffffffffu;
    for (int t = 0; t < a.nprobe; ++t) {
        const int cell = a.probes[q * a.nprobe + t];
        const int e = a.offsets[cell + 1];
        for (int p0 = a.offsets[cell] + warp * 32; p0 < e; p0 += kQThreads) {
            const int pos = p0 + lane;
            const bool ok = pos < e;
            double cd = INFINITY;
            uint32_t ci = 0xffffffffu;
            if (ok) {
                const float *xv = a.X + static_cast<int64_t>(pos) * d;
                double acc = 0.0;
                for (int j = 0; j < d; j += 4) {
                    const float4 u = __ldg(reinterpret_cast<const float4 *>(qv + j));
                    const float4 v = __ldg(reinterpret_cast<const float4 *>(xv + j));
                    const double e0 = static_cast<double>(u.x) - v.x;
                    const double e1 = static_cast<double>(u.y) - v.y;
                    const double e2 = static_cast<double>(u.z) - v.z;
                    const double e3 = static_cast<double>(u.w) - v.w;
                    acc = fma(e0, e0, acc);
                    acc = fma(e1, e1, acc);
                    acc = fma(e2, e2, acc);
                    acc = fma(e3, e3, acc);
                }
                cd = acc;
                ci = static_cast<uint32_t>(a.row_ids[pos]);
            }
            bool pend = ok && before(cd, ci, td, ti);
            unsigned m = __ballot_sync(kFull, pend);
            while (m) {
                const int src = __ffs(m) - 1;
                const double xd = __shfl_sync(kFull, cd, src);
                const uint32_t xi = __shfl_sync(kFull, ci, src);
                const int at = __popc(__ballot_sync(kFull, lane < k && before(ld, li, xd, xi)));
                const double ud = __shfl_up_sync(kFull, ld, 1);
                const uint32_t ui = __shfl_up_sync(kFull, li, 1);
                if (lane == at) {
                    ld = xd;
                    li = xi;
                } else if (lane > at && lane < k) {
                    ld = ud;
                    li = ui;
                }
                td = __shfl_sync(kFull, ld, k - 1);
                ti = __shfl_sync(kFull, li, k - 1);
                if (lane == src) pend = false;
                pend = pend && before(cd, ci, td, ti);
                m = __ballot_sync(kFull, pend);
            }
        }
    }
    s_d[tid] = lane < k ? ld : INFINITY;
    s_i[tid] = lane < k ? li : 0xffffffffu;
    __syncthreads();
    for (int size = 2; size <= kQThreads; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < kQThreads / 2; t += kQThreads) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = (lo & size) == 0;
                const double da = s_d[lo], db = s_d[hi];
                const uint32_t ia = s_i[lo], ib = s_i[hi];
                const bool gt = da > db || (da == db && ia > ib);
                if (gt == up) {
                    s_d[lo] = db;
                    s_d[hi] = da;
                    s_i[lo] = ib;
                    s_i[hi] = ia;
                }
            }
            __syncthreads();
        }
    }
    for (int t = tid; t < k; t += kQThreads) {
        const bool real = s_i[t] != 0xffffffffu;
        a.out_id[q * k + t] = real ? static_cast<int32_t>(s_i[t]) : -1;
        a.out_dist[q * k + t] = real ? static_cast<float>(s_d[t]) : INFINITY;
    }
}

// Cell radii: radius[c] >= max over the points x of cell c of ||x - c||, one block per
// cell, a warp per point (fp64 difference form), rounded up to fp32 with a relative
// margin far above the fp64 rounding; 0 for an empty cell.
__global__ void __launch_bounds__(256) cell_radius_kernel(const float *__restrict__ C,
                                                          const float *__restrict__ X,
                                                          const int32_t *__restrict__ offsets,
                                                          int d, float *__restrict__ radius) {
    __shared__ double red[8];
    const int c = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float *cv = C + static_cast<int64_t>(c) * d;
    double mx = 0.0;
    for (int p = offsets[c] + warp; p < offsets[c + 1]; p += 8)
        mx = fmax(mx, exact_sq_dist(cv, X + static_cast<int64_t>(p) * d, d, lane));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) mx = fmax(mx, red[w]);
        radius[c] = __double2float_ru(sqrt(mx) * (1.0 + 1e-9));
    }
}

// Per query, a cut on the screened distances of the fine pass.  Every probed cell with at
// least k points holds k points within (sqrt(D_c) + r_c)^2 of the query (D_c its fp64
// squared distance to the centroid), so the smallest such value U bounds the query's k-th
// smallest exact distance, and the k-th smallest screened value T~ <= U + E.  An entry
// above cut = U + 3.1 E is therefore above T~ + 2E, outside the re-ranking window: the
// fine pass drops it without counting it, and the merge sends the query to the exact
// fallback should its own window ever reach past the cut.  +inf when no probed cell has k
// points.  A warp per query.
__global__ void __launch_bounds__(256) query_cut_kernel(
    const float *__restrict__ Q, const float *__restrict__ C, const int32_t *__restrict__ probes,
    const int32_t *__restrict__ offsets, const float *__restrict__ radius,
    const double *__restrict__ qn, const float *__restrict__ xmax2, float ce_dot,
    float ce_round, int64_t nq, int nprobe, int k, int d, float *__restrict__ cut) {
    const int lane = threadIdx.x & 31;
    const int64_t q = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (q >= nq) return;
    double u = INFINITY;
    for (int t = 0; t < nprobe; ++t) {
        const int c = probes[q * nprobe + t];
        if (offsets[c + 1] - offsets[c] < k) continue;
        const double D = exact_sq_dist(Q + q * d, C + static_cast<int64_t>(c) * d, d, lane);
        const double r = sqrt(D) * (1.0 + 1e-9) + static_cast<double>(radius[c]);
        u = fmin(u, r * r * (1.0 + 1e-9));
    }
    if (lane == 0) {
        const float xm2 = *xmax2, qf = static_cast<float>(qn[q]);
        const float E = ce_dot * sqrtf(qf * xm2) + ce_round * (qf + xm2);
        cut[q] = __fadd_ru(__double2float_ru(u), 3.1f * E);
    }
}

// Number of flagged queries (one block), for the caller's diagnostics.
__global__ void count_flags_kernel(const int32_t *__restrict__ f, int64_t n, int *__restrict__ out) {
    __shared__ int red[32];
    int c = 0;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) c += f[i] != 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x < 32) {
        c = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
        if (threadIdx.x == 0) *out = c;
    }
}

// max_i ||x_i||^2 of fp64 norms, rounded up to fp32: block maxima combined by an integer
// max on the bits (non-negative floats order as their bit patterns; *out starts at 0).
__global__ void max_norm_kernel(const double *__restrict__ xn, int64_t n,
                                uint32_t *__restrict__ out) {
    __shared__ double red[32];
    double mx = 0.0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        mx = fmax(mx, xn[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFull, mx, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x < 32) {
        mx = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFull, mx, o));
        if (threadIdx.x == 0) atomicMax(out, __float_as_uint(__double2float_ru(mx)));
    }
}

// ---------------------------------------------------------------- small kernels
// ||v||^2 in fp64, a warp per row: lane partial sums over float4 columns, then a fixed
// butterfly.
__global__ void sqnorm_f64_kernel(const float *__restrict__ V, int64_t n, int d,
                                  double *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t r = w0; r < n; r += nw) {
        const float *x = V + r * d;
        double s = 0.0;
        for (int j = lane * 4; j < d; j += 128) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(x + j));
            s = fma(static_cast<double>(v.x), static_cast<double>(v.x), s);
            s = fma(static_cast<double>(v.y), static_cast<double>(v.y), s);
            s = fma(static_cast<double>(v.z), static_cast<double>(v.z), s);
            s = fma(static_cast<double>(v.w), static_cast<double>(v.w), s);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
        if (lane == 0) out[r] = s;
    }
}

// Work items of the fine pass: a cell probed by n pairs gives ceil(n / 32) items, in cell
// order.  One block; cells in rounds of 1024 with a running base.
__global__ void __launch_bounds__(1024) build_items_kernel(const int32_t *__restrict__ pair_off,
                                                           int nlist, int2 *__restrict__ items,
                                                           int *nitems, int *ctr) {
    __shared__ int wsum[32];
    __shared__ int s_base;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_base = 0;
    __syncthreads();
    for (int c0 = 0; c0 < nlist; c0 += 1024) {
        const int c = c0 + tid;
        const int start = c < nlist ? pair_off[c] : 0;
        const int cnt = c < nlist ? (pair_off[c + 1] - start + kTQ - 1) / kTQ : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, w, o);
                if (lane >= o) w += y;
            }
            wsum[lane] = w;  // inclusive
        }
        __syncthreads();
        const int base = s_base + (warp ? wsum[warp - 1] : 0) + incl - cnt;
        for (int t = 0; t < cnt; ++t) items[base + t] = make_int2(c, start + t * kTQ);
        __syncthreads();
        if (tid == 0) s_base += wsum[31];
        __syncthreads();
    }
    if (tid == 0) {
        *nitems = s_base;
        *ctr = 0;
    }
}

}  // namespace

// ---------------------------------------------------------------- host side
size_t ivf_tile_smem() { return sizeof(TileSmem); }

cudaError_t launch_sqnorm_f64(const float *V, int64_t n, int d, double *out, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = ceil_div(n, 8);
    const int grid = static_cast<int>(blocks < 148 * 16 ? blocks : 148 * 16);
    sqnorm_f64_kernel<<<grid, 256, 0, st>>>(V, n, d, out);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_coarse(const float *Q, const double *qn, int64_t q0, int nqb, int d,
                              const float *C, const double *cn, int nlist, double *D,
                              cudaStream_t st) {
    TileArgs a{};
    a.Q = Q;
    a.qn = qn;
    a.V = C;
    a.vn = cn;
    a.d = d;
    a.q0 = q0;
    a.nqb = nqb;
    a.nv = nlist;
    a.D = D;
    const int64_t qblocks = ceil_div(nqb, kTQ);
    // enough items for about four waves of three blocks per SM
    const int64_t want = static_cast<int64_t>(device_sm_count()) * 3 * 4;
    int64_t chunks = ceil_div(want, qblocks);
    const int64_t maxchunks = ceil_div(nlist, kTV);
    if (chunks > maxchunks) chunks = maxchunks;
    if (chunks < 1) chunks = 1;
    a.vchunk = static_cast<int>(round_up(ceil_div(nlist, chunks), kTV));
    a.nvchunks = static_cast<int>(ceil_div(nlist, a.vchunk));
    const int64_t grid = qblocks * a.nvchunks;
    ivf_tile_kernel<false><<<static_cast<unsigned>(grid), kTThreads, sizeof(TileSmem), st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_select(const double *D, const uint32_t *I, int64_t ld, int64_t rows, int L,
                              int m, int32_t *out_id, float *out_dist, int64_t ldo,
                              cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    SelArgs a{D, I, ld, L, m, out_id, out_dist, ldo};
    if (L <= kSelCache) {
        const size_t smem = static_cast<size_t>(L) * (sizeof(uint64_t) + sizeof(uint32_t));
        static std::atomic<uint64_t> smem_set{0};
        const cudaError_t e = smem_opt_in(
            select_rows_kernel<true>,
            static_cast<int>(kSelCache * (sizeof(uint64_t) + sizeof(uint32_t))), smem_set);
        if (e != cudaSuccess) return e;
        select_rows_kernel<true><<<static_cast<unsigned>(rows), kSelThreads, smem, st>>>(a);
    } else {
        select_rows_kernel<false><<<static_cast<unsigned>(rows), kSelThreads, 0, st>>>(a);
    }
    note_launch();
    return cudaGetLastError();
}

bool ivf_coarse_can_screen(int nlist, int dp, int Kp) {
    return nlist <= kCoarseMaxL && assign_can_dump(dp, Kp);
}

cudaError_t launch_ivf_cmax(const float *cn, int K, float *out, cudaStream_t st) {
    cmax_kernel<<<1, 1024, 0, st>>>(cn, K, out);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_coarse_rerank(const float *Vs, int64_t ldv, int64_t rows, int L, int m,
                                     const float *Q, int64_t q0, const float *C, int d, int dp,
                                     const float *xnorm, const float *cmax2, int32_t *probes,
                                     cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    CoarseArgs a{Vs, ldv, L, m, Q, q0, C, d, dp, xnorm, cmax2, probes};
    int P = 1;
    while (P < L) P <<= 1;
    const size_t smem = static_cast<size_t>(P) * (sizeof(double) + sizeof(uint32_t)) +
                        static_cast<size_t>(L) * sizeof(uint32_t);
    static std::atomic<uint64_t> smem_set{0};
    const cudaError_t e = smem_opt_in(
        coarse_rerank_kernel,
        static_cast<int>(kCoarseMaxL * (sizeof(double) + 2 * sizeof(uint32_t))), smem_set);
    if (e != cudaSuccess) return e;
    coarse_rerank_kernel<<<static_cast<unsigned>(rows), kCoarseThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_fine_scr(const uint16_t *Qp, int64_t nq, const uint16_t *Xp, int64_t N,
                                int dp, const double *qn, const double *xn,
                                const int32_t *offsets, const int32_t *pair_sorted,
                                const int32_t *pair_off, const int2 *items, const int *nitems,
                                int *item_ctr, int64_t max_items, int nprobe, float *Sv,
                                uint32_t *Sp, float *Slost, const float *cut, cudaStream_t st) {
    FineArgs a{Qp, nq, Xp, N, dp, qn, xn, offsets, pair_sorted, pair_off, items, nitems,
               item_ctr, nprobe, Sv, Sp, Slost, cut};
    static std::atomic<uint64_t> smem_set{0};
    const cudaError_t e =
        smem_opt_in(ivf_fine_scr_kernel, static_cast<int>(sizeof(FineSmem)), smem_set);
    if (e != cudaSuccess) return e;
    static int occ = 0;  // blocks per SM: the same on every B200
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, ivf_fine_scr_kernel, kTThreads,
                                                          sizeof(FineSmem)) != cudaSuccess ||
            occ < 1)
            occ = 1;
    }
    int64_t grid = static_cast<int64_t>(device_sm_count()) * occ;
    if (grid > max_items) grid = max_items;
    if (grid < 1) grid = 1;
    ivf_fine_scr_kernel<<<static_cast<unsigned>(grid), kTThreads, sizeof(FineSmem), st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_query_rerank(const float *Sv, const uint32_t *Sp, const float *Slost,
                                    int64_t nq, int nprobe, int k, const float *Q,
                                    const float *X, int d, int dp, const double *qn,
                                    const float *xmax2, const int32_t *row_ids,
                                    float *out_dist, int32_t *out_id, int32_t *fallback,
                                    const float *cut, cudaStream_t st) {
    if (nq <= 0) return cudaSuccess;
    QueryArgs a{};
    a.cut = cut;
    a.Sv = Sv;
    a.Sp = Sp;
    a.Slost = Slost;
    a.nprobe = nprobe;
    a.k = k;
    a.Q = Q;
    a.X = X;
    a.d = d;
    a.qn = qn;
    a.xmax2 = xmax2;
    fine_window_coeffs(dp, &a.ce_dot, &a.ce_round);
    a.row_ids = row_ids;
    a.out_dist = out_dist;
    a.out_id = out_id;
    a.fallback = fallback;
    const int L = nprobe * kScrList;
    int P2 = 1;
    while (P2 < L) P2 <<= 1;
    const size_t smem = static_cast<size_t>(P2) * (sizeof(double) + 2 * sizeof(uint32_t)) +
                        static_cast<size_t>(L) * sizeof(uint32_t);
    static std::atomic<uint64_t> smem_set{0};
    const cudaError_t e = smem_opt_in(query_rerank_kernel,
                                      static_cast<int>(kSearchScrMaxProbe * kScrList *
                                                       (sizeof(double) + 3 * sizeof(uint32_t))),
                                      smem_set);
    if (e != cudaSuccess) return e;
    query_rerank_kernel<<<static_cast<unsigned>(nq), kQThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_fallback(const int32_t *fallback, const int32_t *probes, int64_t nq,
                                int nprobe, int k, const float *Q, const float *X, int d,
                                const int32_t *offsets, const int32_t *row_ids, float *out_dist,
                                int32_t *out_id, cudaStream_t st) {
    if (nq <= 0) return cudaSuccess;
    FallbackArgs a{fallback, probes, nprobe, k, Q, X, d, offsets, row_ids, out_dist, out_id};
    fallback_kernel<<<static_cast<unsigned>(nq), kQThreads, 0, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_cell_radius(const float *C, int nlist, const float *X, const int32_t *offsets,
                               int d, float *radius, cudaStream_t st) {
    cell_radius_kernel<<<nlist, 256, 0, st>>>(C, X, offsets, d, radius);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_query_cut(const float *Q, const float *C, const int32_t *probes,
                             const int32_t *offsets, const float *radius, const double *qn,
                             const float *xmax2, int dp, int64_t nq, int nprobe, int k, int d,
                             float *cut, cudaStream_t st) {
    if (nq <= 0) return cudaSuccess;
    float ce_dot, ce_round;
    fine_window_coeffs(dp, &ce_dot, &ce_round);
    const int64_t blocks = ceil_div(nq, 8);
    query_cut_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        Q, C, probes, offsets, radius, qn, xmax2, ce_dot, ce_round, nq, nprobe, k, d, cut);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_count_flags(const int32_t *f, int64_t n, int *out, cudaStream_t st) {
    count_flags_kernel<<<1, 1024, 0, st>>>(f, n, out);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_max_norm(const double *xn, int64_t n, float *out, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float), st);
    if (e != cudaSuccess) return e;
    const int64_t blocks = ceil_div(n, 1024);
    const int grid = static_cast<int>(blocks < 148 * 4 ? (blocks < 1 ? 1 : blocks) : 148 * 4);
    max_norm_kernel<<<grid, 1024, 0, st>>>(xn, n, reinterpret_cast<uint32_t *>(out));
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_items(const int32_t *pair_off, int nlist, int2 *items, int *nitems,
                             int *ctr, cudaStream_t st) {
    build_items_kernel<<<1, 1024, 0, st>>>(pair_off, nlist, items, nitems, ctr);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_ivf_fine(const float *Q, const double *qn, int d, const float *X_lists,
                            const double *xn, const int32_t *offsets, const int32_t *row_ids,
                            const int32_t *pair_sorted, const int32_t *pair_off,
                            const int2 *items, const int *nitems, int *item_ctr, int64_t max_items,
                            int nprobe, int k, double *Ld, uint32_t *Li, cudaStream_t st) {
    TileArgs a{};
    a.Q = Q;
    a.qn = qn;
    a.V = X_lists;
    a.vn = xn;
    a.d = d;
    a.offsets = offsets;
    a.row_ids = row_ids;
    a.pair_sorted = pair_sorted;
    a.pair_off = pair_off;
    a.items = items;
    a.nitems = nitems;
    a.item_ctr = item_ctr;
    a.nprobe = nprobe;
    a.k = k;
    a.Ld = Ld;
    a.Li = Li;
    static int occ = 0;
    if (occ == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, ivf_tile_kernel<true>, kTThreads,
                                                          sizeof(TileSmem)) != cudaSuccess ||
            occ < 1)
            occ = 1;
    }
    int64_t grid = static_cast<int64_t>(device_sm_count()) * occ;
    if (grid > max_items) grid = max_items;
    if (grid < 1) grid = 1;
    ivf_tile_kernel<true><<<static_cast<unsigned>(grid), kTThreads, sizeof(TileSmem), st>>>(a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fk
