// fk_api.cu -- the extern "C" boundary of libfk: argument validation, workspace carving,
// stream plumbing and the Lloyd loop.  Every arithmetic step runs in the kernels of
// prep.cu, assign_sm100.cu, sort_csr.cu and update.cu; this file only launches them.
#include <cstdlib>
#include <cstring>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "fk_common.cuh"
#include "ptx_sm100.cuh"

namespace fk {

thread_local long g_launches = 0;

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
    int n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

// Host-side fault injection, chosen by the environment variable FK_FAULT when the library
// is first used (see fk_common.cuh).  Nothing is injected on the device.
Fault injected_fault() {
    static const Fault f = [] {
        const char *e = std::getenv("FK_FAULT");
        if (!e) return kFaultNone;
        if (std::strcmp(e, "workspace") == 0) return kFaultWorkspace;
        if (std::strcmp(e, "launch") == 0) return kFaultLaunch;
        return kFaultNone;
    }();
    return f;
}

fk_status check_device() {
    static int verdict[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FK_ERR_CUDA;
    if (dev >= 0 && dev < 64 && verdict[dev]) return verdict[dev] == 1 ? FK_OK : FK_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return FK_ERR_CUDA;
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) verdict[dev] = ok ? 1 : 2;
    return ok ? FK_OK : FK_ERR_UNSUPPORTED;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

namespace {
// The unique id of the calling thread's current CUDA context (0 if there is none or the
// driver cannot tell).  The per-thread caches below (streams, events, pinned staging,
// instantiated graphs) belong to the context they were made in: each is tagged with this
// id and is dropped, not used, once the id changes (a device reset, a new primary
// context).  Dropped handles are not destroyed: their context is gone with them.
uint64_t context_id() {
    using GetCurrent = int (*)(void **);
    using GetId = int (*)(void *, unsigned long long *);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static const bool found = [] {
        void *p = nullptr, *q = nullptr;
        cudaDriverEntryPointQueryResult r1, r2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) !=
                cudaSuccess ||
            r1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) != cudaSuccess ||
            r2 != cudaDriverEntryPointSuccess)
            return false;
        get_current = reinterpret_cast<GetCurrent>(p);
        get_id = reinterpret_cast<GetId>(q);
        return true;
    }();
    void *ctx = nullptr;
    unsigned long long id = 0;
    if (!found || get_current(&ctx) != 0 || ctx == nullptr || get_id(ctx, &id) != 0) return 0;
    return id;
}

struct SideStream {
    uint64_t ctx = 0;
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr;  // ordering only (no timing)
    bool used = false;           // forked since the last join
};

SideStream *side_stream() {
    thread_local SideStream side[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    const uint64_t ctx = context_id();
    if (ctx == 0) return nullptr;
    SideStream &ss = side[dev];
    if (ss.ctx != ctx) ss = SideStream{};
    if (!ss.s) {
        if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess) {
            ss = SideStream{};
            return nullptr;
        }
        ss.ctx = ctx;
    }
    return &ss;
}
}  // namespace

cudaError_t record_event(cudaEvent_t e, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t r = cudaStreamIsCapturing(st, &cs);
    if (r != cudaSuccess) return r;
    if (cs != cudaStreamCaptureStatusActive) return cudaEventRecord(e, st);
    SideStream *ss = side_stream();
    if (!ss) return cudaErrorUnknown;
    if ((r = cudaEventRecord(ss->fork, st)) != cudaSuccess ||
        (r = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess)
        return r;
    ss->used = true;
    return cudaEventRecordWithFlags(e, ss->s, cudaEventRecordExternal);
}

cudaError_t join_side_stream(cudaStream_t st) {
    SideStream *ss = side_stream();
    if (!ss) return cudaErrorUnknown;
    if (!ss->used) return cudaSuccess;
    ss->used = false;
    cudaError_t r = cudaEventRecord(ss->fork, ss->s);
    return r != cudaSuccess ? r : cudaStreamWaitEvent(st, ss->fork, 0);
}

fk_status validate_shape(int64_t N, int d, int K, fk_dtype dtype, fk_metric metric,
                         bool planes_ok) {
    if (N < 1 || N > 2147483647LL - 1) return FK_ERR_INVALID_ARG;
    if (d < 1 || K < 1 || K > N) return FK_ERR_INVALID_ARG;
    if (dtype == FK_BF16X2 && !planes_ok) return FK_ERR_UNSUPPORTED;
    if (dtype != FK_F32 && dtype != FK_BF16 && dtype != FK_BF16X2) return FK_ERR_UNSUPPORTED;
    if (dtype == FK_BF16X2 && metric != FK_L2) return FK_ERR_UNSUPPORTED;
    if (metric != FK_L2 && metric != FK_COSINE) return FK_ERR_UNSUPPORTED;
    if (dtype == FK_F32 && d % 4 != 0) return FK_ERR_UNSUPPORTED;
    if (dtype == FK_BF16 && d % 8 != 0) return FK_ERR_UNSUPPORTED;
    if (metric == FK_COSINE && dtype != FK_F32) return FK_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(K) * d > 2147483647LL) return FK_ERR_UNSUPPORTED;
    return FK_OK;
}

bool screened_route(int64_t N, int dp, int Kp, int K) {
    if (dp > kThreeProductMaxDp) return assign_can_dump(dp, Kp);
    const bool pays = dp >= kScreenMinD || static_cast<int64_t>(K) * dp >= kScreenMinKD;
    return pays && assign_can_screen(N, dp, Kp);
}

namespace {

// NVTX range for the phases of a call (visible to profilers that record NVTX; without
// one attached the calls cost a branch).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

fk_status check_ws(void *ws, size_t ws_bytes, const WsLayout &L) {
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < L.total) return FK_ERR_WORKSPACE;
    if (injected_fault() == kFaultWorkspace) return FK_ERR_WORKSPACE;
    return FK_OK;
}

bool overlap(const void *a, size_t an, const void *b, size_t bn) {
    const char *pa = static_cast<const char *>(a), *pb = static_cast<const char *>(b);
    return pa < pb + bn && pb < pa + an;
}

#define FK_TRY_CUDA(expr)                              \
    do {                                               \
        if ((expr) != cudaSuccess) return FK_ERR_CUDA; \
    } while (0)

// The operand X planes the assign kernel reads, prepared from the (possibly normalised)
// points.  Returns the planes pointer, plane count and row stride.  `xnorm` receives
// ||x||^2 per row when given; for pre-split points the norms already follow the planes and
// *xnorm_ready points at them.
fk_status prepare_x(const void *Xp, fk_dtype dtype, int64_t N, int d, const WsLayout &L,
                    void *ws, float *xnorm, cudaStream_t st, const void **planes,
                    int *nplanes, int64_t *lda, const float **xnorm_ready = nullptr) {
    uint16_t *xs = ws_ptr<uint16_t>(ws, L.xs);
    if (xnorm_ready) *xnorm_ready = xnorm;
    if (dtype == FK_BF16X2) {  // already split by fk_split_points
        *planes = Xp;
        *nplanes = 2;
        *lda = L.dp;
        if (xnorm_ready)
            *xnorm_ready = reinterpret_cast<const float *>(static_cast<const uint16_t *>(Xp) +
                                                           2 * N * L.dp);
        return FK_OK;
    }
    if (dtype == FK_F32) {
        FK_TRY_CUDA(launch_split_x(static_cast<const float *>(Xp), N, d, L.dp, xs, xs + N * L.dp,
                                   xnorm, st));
        *planes = xs;
        *nplanes = 2;
        *lda = L.dp;
    } else {
        if (xnorm)
            FK_TRY_CUDA(launch_xnorm_bf16(static_cast<const uint16_t *>(Xp), N, d, xnorm, st));
        if (L.xplanes == 1) {
            FK_TRY_CUDA(launch_pad_bf16(static_cast<const uint16_t *>(Xp), N, d, L.dp, xs, st));
            *planes = xs;
            *lda = L.dp;
        } else {
            *planes = Xp;
            *lda = d;
        }
        *nplanes = 1;
    }
    return FK_OK;
}

// Assignment from prepared planes.  Two-plane (fp32) problems large enough for the CTA-pair
// kernel take the screened route (single product, exact re-ranking, three products for the
// rows that need them); it needs ||x||^2 in `xnorm`, the centroids C (fp32, the values the
// planes were made from) and, when available, the fp32 points X32 for the re-ranking.
fk_status run_assign(const void *planes, int nplanes, int64_t lda, int64_t N, int d, int K,
                     const WsLayout &L, void *ws, int32_t *labels, const float *xnorm,
                     float *mind, cudaStream_t st, const float *X32 = nullptr,
                     const float *C = nullptr, bool allow_screen = true,
                     bool *screened = nullptr, cudaEvent_t ev_mma0 = nullptr,
                     cudaEvent_t ev_mma1 = nullptr, int64_t probe_rows = 0) {
    // probe_rows > 0: only the screening pass and re-ranking over the first probe_rows rows
    // (if the screened route applies), counting the rows that would need the fallback
    if (screened) *screened = false;
    AssignArgs a{};
    a.a_planes = planes;
    a.a_nplanes = nplanes;
    a.lda = lda;
    a.b_planes = ws_ptr<uint16_t>(ws, L.cs);
    a.cn = ws_ptr<float>(ws, L.cn);
    a.caug = ws_ptr<uint16_t>(ws, L.caug);
    a.N = N;
    a.d = d;
    a.dp = static_cast<int>(L.dp);
    a.K = K;
    a.Kp = static_cast<int>(L.Kp);
    a.labels = labels;
    a.best = nullptr;
    a.xnorm = xnorm;
    a.mind = mind;
    a.err = ws_ptr<uint32_t>(ws, L.err);
    a.wait_ns = kDefaultWaitNs;
    // beyond kThreeProductMaxDp the three-product form decides no label: screen every call
    const bool exact_only = nplanes == 2 && L.dp > kThreeProductMaxDp;
    const bool can_screen = nplanes == 2 && C != nullptr && xnorm != nullptr &&
                            lda == L.dp && d % 4 == 0 && aligned(C, 16) &&
                            (X32 == nullptr || aligned(X32, 16));
    if (exact_only && !can_screen) return FK_ERR_UNSUPPORTED;
    if (exact_only && probe_rows > 0) return FK_OK;  // nothing to decide: no probe
    if ((allow_screen || exact_only) && can_screen &&
        screened_route(N, a.dp, a.Kp, K)) {
        ScreenBufs sb;
        sb.cand = ws_ptr<int32_t>(ws, L.cand);
        sb.nfb = ws_ptr<uint32_t>(ws, L.nfb);
        sb.fbrows = ws_ptr<int32_t>(ws, L.fbrows);
        sb.fblab = ws_ptr<int32_t>(ws, L.fblab);
        sb.xsfb = ws_ptr<uint16_t>(ws, L.xsfb);
        sb.cmax2 = ws_ptr<float>(ws, L.cmax2);
        if (probe_rows > 0)
            FK_TRY_CUDA(launch_screen_probe(a, N < probe_rows ? N : probe_rows, X32, C, sb, st));
        else
            FK_TRY_CUDA(launch_assign_screened(a, X32, C, sb, st, ev_mma0, ev_mma1));
        if (screened) *screened = true;
        return FK_OK;
    }
    if (exact_only) return FK_ERR_UNSUPPORTED;  // the pair kernel cannot run on this device
    if (probe_rows > 0) return FK_OK;
    if (ev_mma0) FK_TRY_CUDA(record_event(ev_mma0, st));
    FK_TRY_CUDA(launch_assign(a, st));
    if (ev_mma1) FK_TRY_CUDA(record_event(ev_mma1, st));
    return FK_OK;
}

fk_status run_update(const void *Xp, fk_dtype dtype, int64_t N, int d, int K,
                     const WsLayout &L, void *ws, const int32_t *labels, const float *C_old,
                     const float *C_used, float *C_new, int32_t *counts, int32_t *offsets,
                     int32_t *perm_out, double *objective, double *sums_out,
                     cudaStream_t st) {
    const int32_t *skeys = nullptr, *perm = nullptr;
    FK_TRY_CUDA(launch_sort_csr(labels, N, K, L.sp, ws_ptr<int32_t>(ws, L.keys0),
                                ws_ptr<int32_t>(ws, L.keys1), ws_ptr<int32_t>(ws, L.vals0),
                                ws_ptr<int32_t>(ws, L.vals1), perm_out,
                                ws_ptr<uint32_t>(ws, L.hist), ws_ptr<uint32_t>(ws, L.dtot),
                                offsets, &skeys, &perm, ws_ptr<uint32_t>(ws, L.err), st));
    FK_TRY_CUDA(launch_update(Xp, dtype, N, d, K, L.up, skeys, perm, offsets, C_old, C_used,
                              C_new, counts, ws_ptr<double>(ws, L.pieces),
                              ws_ptr<int32_t>(ws, L.pkeys), ws_ptr<double>(ws, L.piecesb),
                              ws_ptr<int32_t>(ws, L.pkeysb), ws_ptr<double>(ws, L.jpart),
                              objective, ws_ptr<uint32_t>(ws, L.err), sums_out, st));
    return FK_OK;
}

// Read (and optionally clear) the two device error words after a stream sync.
fk_status read_err(void *ws, const WsLayout &L, cudaStream_t st, bool clear, int *code) {
    uint32_t e[2] = {0, 0};
    uint32_t *dev = ws_ptr<uint32_t>(ws, L.err);
    FK_TRY_CUDA(cudaMemcpyAsync(e, dev, sizeof(e), cudaMemcpyDeviceToHost, st));
    if (clear) FK_TRY_CUDA(cudaMemsetAsync(dev, 0, kErrWords * sizeof(uint32_t), st));
    FK_TRY_CUDA(cudaStreamSynchronize(st));
    *code = e[0] ? FK_ERR_TIMEOUT : (e[1] ? FK_ERR_DEVICE : FK_OK);
    return FK_OK;
}

// Workspace of fk_lloyd_streamed: the per-chunk workspace (an fk_assign / fk_update
// workspace for chunk_rows points, L2), then two chunk buffers of points and labels, one
// chunk's partial sums, counts, offsets and objective, the iteration's running totals, the
// objectives of every iteration and the alternate centroids.
struct StreamLayout {
    WsLayout L;  // per-chunk workspace, at offset 0
    size_t xbuf[2] = {0, 0}, lab[2] = {0, 0}, sums = 0, cnt = 0, off = 0, objc = 0,
           sums_tot = 0, cnt_tot = 0, obj_tot = 0, calt = 0, total = 0;
};

StreamLayout stream_layout(int64_t chunk, int d, int K, fk_dtype dtype) {
    StreamLayout S;
    S.L = ws_layout(chunk, d, K, dtype, FK_L2);
    size_t o = S.L.total;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += static_cast<size_t>(round_up(static_cast<int64_t>(bytes > 0 ? bytes : 1), 256));
        return at;
    };
    const size_t e = dtype == FK_F32 ? 4 : 2;
    const size_t KD = static_cast<size_t>(K) * d;
    for (int b = 0; b < 2; ++b) S.xbuf[b] = take(e * chunk * d);
    for (int b = 0; b < 2; ++b) S.lab[b] = take(sizeof(int32_t) * chunk);
    S.sums = take(sizeof(double) * KD);
    S.cnt = take(sizeof(int32_t) * K);
    S.off = take(sizeof(int32_t) * (K + 1));
    S.objc = take(sizeof(double));
    S.sums_tot = take(sizeof(double) * KD);
    S.cnt_tot = take(sizeof(int64_t) * K);
    S.obj_tot = take(sizeof(double) * kObjRing);
    S.calt = take(sizeof(float) * KD);
    S.total = o;
    return S;
}

// A kernel whose mbarrier is never arrived on: its bounded wait must expire and record
// a timeout in the workspace error word (exercises the failure path without a fault).
__global__ void wait_selftest_kernel(uint32_t *err, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!ptx::mbar_wait(&bar, 0u, nullptr, limit_ns)) err[0] = kErrTimeout;
    }
}

fk_status validate_search(int64_t nq, int d, int nlist, int64_t N, int nprobe, int k) {
    if (nq < 1 || d < 1 || nlist < 1 || N < 1 || N > 2147483647LL - 1) return FK_ERR_INVALID_ARG;
    if (nprobe < 1 || nprobe > nlist || nprobe > kSearchMaxProbe) return FK_ERR_INVALID_ARG;
    if (k < 1 || k > kSearchMaxK) return FK_ERR_INVALID_ARG;
    if (nq > (2147483647LL - 1) / nprobe) return FK_ERR_INVALID_ARG;
    if (d % 4 != 0) return FK_ERR_UNSUPPORTED;
    return FK_OK;
}

fk_status run_ivf_search(const float *Q, int64_t nq, int d, const float *C, int nlist,
                         const float *X_lists, const double *X_norms, const void *X_planes,
                         const float *cell_radius, const int32_t *offsets, const int32_t *row_ids, int64_t N, int nprobe,
                         int k, bool screen, bool screen_fine, float *distances, int32_t *ids,
                         int32_t *probes, void *ws, const SearchLayout &L, cudaStream_t st,
                         const cudaEvent_t *ev) {
    // ev (optional): five events recorded between the phases
    auto mark = [&](int i) { return !ev || cudaEventRecord(ev[i], st) == cudaSuccess; };
    if (!mark(0)) return FK_ERR_CUDA;
    double *qn = ws_ptr<double>(ws, L.qn), *cn = ws_ptr<double>(ws, L.cn);
    FK_TRY_CUDA(launch_sqnorm_f64(Q, nq, d, qn, st));
    FK_TRY_CUDA(launch_sqnorm_f64(C, nlist, d, cn, st));
    // coarse: distances to every centroid, then the nprobe nearest per query
    int32_t *pr = probes ? probes : ws_ptr<int32_t>(ws, L.probes);
    double *D = ws_ptr<double>(ws, L.D);
    uint16_t *qh = ws_ptr<uint16_t>(ws, L.qplanes);
    float *qxn = ws_ptr<float>(ws, L.qxn);
    if (screen || screen_fine)  // bf16 hi / lo planes of every query, and ||q||^2
        FK_TRY_CUDA(launch_split_x(Q, nq, d, L.dp, qh, qh + nq * L.dp, qxn, st));
    if (screen) {
        // tensor-core screening of every (query, centroid), fp64 re-ranking of the window
        AssignArgs a{};
        uint16_t *cpl = ws_ptr<uint16_t>(ws, L.cplanes);
        float *ccn = ws_ptr<float>(ws, L.ccn);
        float *cmax2 = ws_ptr<float>(ws, L.cmax2), *Vs = ws_ptr<float>(ws, L.D);
        FK_TRY_CUDA(launch_prep_centroids(C, nlist, d, L.Kp, L.dp, FK_F32, cpl, ccn,
                                          ws_ptr<float>(ws, L.cused),
                                          ws_ptr<uint16_t>(ws, L.caug), st));
        FK_TRY_CUDA(launch_ivf_cmax(ccn, nlist, cmax2, st));
        a.a_nplanes = 1;
        a.lda = L.dp;
        a.b_planes = cpl;
        a.cn = ccn;
        a.caug = ws_ptr<uint16_t>(ws, L.caug);
        a.d = d;
        a.dp = static_cast<int>(L.dp);
        a.K = nlist;
        a.Kp = static_cast<int>(L.Kp);
        a.err = ws_ptr<uint32_t>(ws, L.err);
        a.wait_ns = kDefaultWaitNs;
        a.cmax2 = cmax2;
        a.dump = Vs;
        a.ldd = L.Kp;
        for (int64_t q0 = 0; q0 < nq; q0 += L.qbatch) {
            const int64_t nqb = nq - q0 < L.qbatch ? nq - q0 : L.qbatch;
            a.a_planes = qh + q0 * L.dp;  // rows q0 .. of the hi plane
            a.xnorm = qxn + q0;
            a.N = nqb;
            FK_TRY_CUDA(launch_assign(a, st));
            FK_TRY_CUDA(launch_ivf_coarse_rerank(Vs, L.Kp, nqb, nlist, nprobe, Q, q0, C, d,
                                                 static_cast<int>(L.dp), qxn + q0, cmax2, pr,
                                                 st));
        }
    } else {
        for (int64_t q0 = 0; q0 < nq; q0 += L.qbatch) {
            const int nqb = static_cast<int>(nq - q0 < L.qbatch ? nq - q0 : L.qbatch);
            FK_TRY_CUDA(launch_ivf_coarse(Q, qn, q0, nqb, d, C, cn, nlist, D, st));
            FK_TRY_CUDA(launch_ivf_select(D, nullptr, nlist, nqb, nlist, nprobe,
                                          pr + q0 * nprobe, nullptr, nprobe, st));
        }
    }
    if (!mark(1)) return FK_ERR_CUDA;
    // the (query, probe) pairs in cell order, cut into work items
    const int32_t *skeys = nullptr, *psorted = nullptr;
    int32_t *poff = ws_ptr<int32_t>(ws, L.poff);
    FK_TRY_CUDA(launch_sort_csr(pr, L.P, nlist, L.sp, ws_ptr<int32_t>(ws, L.keys0),
                                ws_ptr<int32_t>(ws, L.keys1), ws_ptr<int32_t>(ws, L.vals0),
                                ws_ptr<int32_t>(ws, L.vals1), ws_ptr<int32_t>(ws, L.psorted),
                                ws_ptr<uint32_t>(ws, L.hist), ws_ptr<uint32_t>(ws, L.dtot), poff,
                                &skeys, &psorted, ws_ptr<uint32_t>(ws, L.err), st));
    int2 *items = ws_ptr<int2>(ws, L.items);
    int *nitems = ws_ptr<int>(ws, L.nitems);
    FK_TRY_CUDA(launch_ivf_items(poff, nlist, items, nitems, nitems + 1, st));
    if (!mark(2)) return FK_ERR_CUDA;
    if (screen_fine) {
        // per pair the 32 smallest screened distances; per query the window re-ranked in
        // fp64; the queries whose lists may have dropped a candidate, exactly
        float *Sv = ws_ptr<float>(ws, L.Sv), *Slost = ws_ptr<float>(ws, L.Slost);
        uint32_t *Sp = ws_ptr<uint32_t>(ws, L.Sp);
        int32_t *fb = ws_ptr<int32_t>(ws, L.fb);
        float *xmax2 = ws_ptr<float>(ws, L.xmax2);
        const uint16_t *Xp = static_cast<const uint16_t *>(X_planes);
        float *cut = cell_radius ? ws_ptr<float>(ws, L.ubound) : nullptr;
        FK_TRY_CUDA(launch_max_norm(X_norms, N, xmax2, st));
        if (cut)
            FK_TRY_CUDA(launch_query_cut(Q, C, pr, offsets, cell_radius, qn, xmax2,
                                         static_cast<int>(L.dp), nq, nprobe, k, d, cut, st));
        FK_TRY_CUDA(launch_ivf_fine_scr(qh, nq, Xp, N, static_cast<int>(L.dp), qn, X_norms,
                                        offsets, psorted, poff, items, nitems, nitems + 1,
                                        L.max_items, nprobe, Sv, Sp, Slost, cut, st));
        if (!mark(3)) return FK_ERR_CUDA;
        FK_TRY_CUDA(launch_ivf_query_rerank(Sv, Sp, Slost, nq, nprobe, k, Q, X_lists, d,
                                            static_cast<int>(L.dp), qn, xmax2, row_ids,
                                            distances, ids, fb, cut, st));
        FK_TRY_CUDA(launch_ivf_fallback(fb, pr, nq, nprobe, k, Q, X_lists, d, offsets, row_ids,
                                        distances, ids, st));
    } else {
        // fine: per pair, the k nearest points of its cell; then per query the k nearest
        double *Ld = ws_ptr<double>(ws, L.Ld);
        uint32_t *Li = ws_ptr<uint32_t>(ws, L.Li);
        FK_TRY_CUDA(launch_ivf_fine(Q, qn, d, X_lists, X_norms, offsets, row_ids, psorted, poff,
                                    items, nitems, nitems + 1, L.max_items, nprobe, k, Ld, Li,
                                    st));
        if (!mark(3)) return FK_ERR_CUDA;
        const int64_t Lrow = static_cast<int64_t>(nprobe) * k;
        FK_TRY_CUDA(launch_ivf_select(Ld, Li, Lrow, nq, static_cast<int>(Lrow), k, ids,
                                      distances, k, st));
    }
    if (!mark(4)) return FK_ERR_CUDA;
    return FK_OK;
}

// Timing events, created once per thread and device and reused by every call: each call
// ends with a synchronisation, so no event is still pending when the next call records it.
bool pooled_events(size_t n, std::vector<cudaEvent_t> **out) {
    thread_local std::vector<cudaEvent_t> pools[64];
    thread_local uint64_t pool_ctx[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const uint64_t ctx = context_id();
    if (ctx == 0) return false;
    std::vector<cudaEvent_t> &p = pools[dev];
    if (pool_ctx[dev] != ctx) {  // events of another context: drop them
        p.clear();
        pool_ctx[dev] = ctx;
    }
    while (p.size() < n) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return false;
        p.push_back(e);
    }
    *out = &p;
    return true;
}

// fk_lloyd's iteration loop as a CUDA graph.  The loop's launches are fixed by the call's
// arguments and by the screening probe's decision, so a short call (kLoopGraphMaxFlops)
// that repeats the previous call on the same thread (same pointers, sizes, metric,
// iteration count, timing flag, device and probe decision) captures its loop once and
// replays it as one graph launch, and later identical calls replay it again.  The graph reads device memory when it runs, so new
// point or centroid values need no new capture.  FK_LOOP_GRAPH=0 in the environment turns
// the cache off.
struct LoopKey {
    const void *X;
    float *C;
    int32_t *labels, *counts, *offsets;
    void *ws;
    size_t ws_bytes;
    int64_t N;
    int d, K, niter, device;
    uint64_t ctx;  // the CUDA context the graph belongs to
    fk_dtype dtype;
    fk_metric metric;
    int timing;  // 0 none, 1 kernel only, 2 every phase
    bool allow_screen;
    bool operator==(const LoopKey &o) const {
        return X == o.X && C == o.C && labels == o.labels && counts == o.counts &&
               offsets == o.offsets && ws == o.ws && ws_bytes == o.ws_bytes && N == o.N &&
               d == o.d && K == o.K && niter == o.niter && device == o.device && ctx == o.ctx &&
               dtype == o.dtype && metric == o.metric && timing == o.timing &&
               allow_screen == o.allow_screen;
    }
};

struct LoopGraph {
    LoopKey key{};
    cudaGraphExec_t exec = nullptr;
    std::vector<cudaEvent_t> ev;  // timing: 4 per iteration, then 2 per iteration
    int nscreened = 0;
    bool last_screened = false;
    long launches = 0;  // kernels in the graph
    uint64_t used = 0;  // exec == nullptr: the capture failed; the call runs eagerly
};

constexpr size_t kLoopGraphs = 4;

// Calls up to this many useful flops (2 N K d niter, about a millisecond of tensor work)
// replay their loop from a graph.  There the launches are a large share of the call; above
// it they are not, and a capture's host time (tens of milliseconds for a long loop with
// timing events) would take hundreds of calls to repay.
constexpr double kLoopGraphMaxFlops = 1e12;

struct LoopGraphCache {
    bool have_last = false;
    LoopKey last{};
    std::vector<LoopGraph> graphs;
    uint64_t clock = 0;
    cudaStream_t capture[64] = {};  // one capture stream per device
    uint64_t capture_ctx[64] = {};   // its context
};

LoopGraphCache &loop_graphs() {
    thread_local LoopGraphCache c;
    return c;
}

bool loop_graphs_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("FK_LOOP_GRAPH");
        return !(e && std::strcmp(e, "0") == 0);
    }();
    return on;
}

// Pinned host staging for the end of an fk_lloyd call, one per thread and device: the
// objectives of the iterations since the last ring copy and words 0..6 of the error block
// (error flags, then the last iteration's statistics), read back by one copy each and one
// synchronisation.  Pinned, so that the copies can sit in a captured graph.
struct CallStage {
    double obj[kObjRing];
    uint32_t words[8];
};

CallStage *call_stage() {
    thread_local CallStage *stages[64] = {};
    thread_local uint64_t stage_ctx[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    const uint64_t ctx = context_id();
    if (ctx == 0) return nullptr;
    if (stage_ctx[dev] != ctx) {  // pinned memory of another context is gone with it
        stages[dev] = nullptr;
        stage_ctx[dev] = ctx;
    }
    if (!stages[dev]) {
        void *p = nullptr;
        if (cudaHostAlloc(&p, sizeof(CallStage), cudaHostAllocDefault) != cudaSuccess)
            return nullptr;
        stages[dev] = static_cast<CallStage *>(p);
    }
    return stages[dev];
}

void release(LoopGraph &g) {
    if (g.exec) cudaGraphExecDestroy(g.exec);
    for (cudaEvent_t e : g.ev) cudaEventDestroy(e);
    g.exec = nullptr;
    g.ev.clear();
}
}  // namespace
}  // namespace fk

using namespace fk;

extern "C" {

const char *fk_status_string(fk_status s) {
    switch (s) {
        case FK_OK: return "FK_OK";
        case FK_ERR_INVALID_ARG: return "FK_ERR_INVALID_ARG";
        case FK_ERR_UNSUPPORTED: return "FK_ERR_UNSUPPORTED";
        case FK_ERR_WORKSPACE: return "FK_ERR_WORKSPACE";
        case FK_ERR_CUDA: return "FK_ERR_CUDA";
        case FK_ERR_TIMEOUT: return "FK_ERR_TIMEOUT";
        case FK_ERR_DEVICE: return "FK_ERR_DEVICE";
    }
    return "FK_UNKNOWN_STATUS";
}

int fk_version(void) { return 4; }

int64_t fk_launch_count(void) { return g_launches; }

fk_status fk_workspace_size(int64_t N, int d, int K, fk_dtype dtype, fk_metric metric,
                            size_t *bytes) {
    if (!bytes) return FK_ERR_INVALID_ARG;
    fk_status s = validate_shape(N, d, K, dtype, metric, true);
    if (s != FK_OK) return s;
    const size_t a = ws_layout(N, d, K, dtype, metric).total;
    const size_t b = ws_layout(N, d, K, dtype, FK_L2).total;
    *bytes = a > b ? a : b;
    return FK_OK;
}

fk_status fk_normalize_rows(const float *X_in, float *X_out, int64_t N, int d,
                            fk_stream_t stream) {
    if (N < 0 || d < 1 || !X_in || !X_out) return FK_ERR_INVALID_ARG;
    if (d % 4 != 0 || !aligned(X_in, 16) || !aligned(X_out, 16)) return FK_ERR_UNSUPPORTED;
    if (N == 0) return FK_OK;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    FK_TRY_CUDA(launch_normalize(X_in, X_out, N, d, stream));
    return FK_OK;
}

fk_status fk_split_points(const float *X, int64_t N, int d, void *planes, fk_stream_t stream) {
    if (N < 1 || d < 1 || !X || !planes) return FK_ERR_INVALID_ARG;
    if (d % 4 != 0 || !aligned(X, 16) || !aligned(planes, 16)) return FK_ERR_UNSUPPORTED;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    const int64_t dp = round_up(d, kBK);
    uint16_t *p = static_cast<uint16_t *>(planes);
    float *norms = reinterpret_cast<float *>(p + 2 * N * dp);
    FK_TRY_CUDA(launch_split_x(X, N, d, dp, p, p + N * dp, norms, stream));
    return FK_OK;
}

fk_status fk_centroid_norms(const float *C, int K, int d, fk_dtype dtype, float *cn,
                            fk_stream_t stream) {
    if (K < 1 || d < 1 || !C || !cn) return FK_ERR_INVALID_ARG;
    if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    FK_TRY_CUDA(launch_centroid_norms(C, K, d, dtype, cn, stream));
    return FK_OK;
}

fk_status fk_assign(const void *X, fk_dtype dtype, int64_t N, int d, const float *C, int K,
                    int32_t *labels, float *mind, void *ws, size_t ws_bytes,
                    fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, FK_L2, true);
    if (s != FK_OK) return s;
    if (!X || !C || !labels) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(C, 4) || !aligned(labels, 4) || (mind && !aligned(mind, 4)))
        return FK_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(N, d, K, dtype, FK_L2);
    if ((s = check_ws(ws, ws_bytes, L)) != FK_OK) return s;
    if ((s = check_device()) != FK_OK) return s;
    if (injected_fault() == kFaultLaunch) return FK_ERR_CUDA;
    cudaStream_t st = stream;
    FK_TRY_CUDA(launch_prep_centroids(C, K, d, L.Kp, L.dp, dtype, ws_ptr<uint16_t>(ws, L.cs),
                                      ws_ptr<float>(ws, L.cn), ws_ptr<float>(ws, L.cused),
                                      ws_ptr<uint16_t>(ws, L.caug), st));
    // ||x||^2 per row: for the distances of `mind`, and for the screening window of fp32
    // points (the split computes it in the same pass)
    float *xnorm = (mind || dtype == FK_F32) ? ws_ptr<float>(ws, L.xnorm) : nullptr;
    const void *planes = nullptr;
    const float *xn = nullptr;
    int nplanes = 0;
    int64_t lda = 0;
    if ((s = prepare_x(X, dtype, N, d, L, ws, xnorm, st, &planes, &nplanes, &lda, &xn)) !=
        FK_OK)
        return s;
    return run_assign(planes, nplanes, lda, N, d, K, L, ws, labels, xn, mind, st,
                      dtype == FK_F32 ? static_cast<const float *>(X) : nullptr, C);
}

fk_status fk_assign_split(const float *X, const void *planes, int64_t N, int d,
                          const float *C, int K, int32_t *labels, float *mind, void *ws,
                          size_t ws_bytes, fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, FK_F32, FK_L2);
    if (s != FK_OK) return s;
    if (!X || !planes || !C || !labels) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(planes, 16) || !aligned(C, 4) || !aligned(labels, 4) ||
        (mind && !aligned(mind, 4)))
        return FK_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(N, d, K, FK_BF16X2, FK_L2);
    if ((s = check_ws(ws, ws_bytes, L)) != FK_OK) return s;
    if ((s = check_device()) != FK_OK) return s;
    if (injected_fault() == kFaultLaunch) return FK_ERR_CUDA;
    cudaStream_t st = stream;
    FK_TRY_CUDA(launch_prep_centroids(C, K, d, L.Kp, L.dp, FK_F32, ws_ptr<uint16_t>(ws, L.cs),
                                      ws_ptr<float>(ws, L.cn), ws_ptr<float>(ws, L.cused),
                                      ws_ptr<uint16_t>(ws, L.caug), st));
    const void *pl = nullptr;
    const float *xn = nullptr;
    int nplanes = 0;
    int64_t lda = 0;
    if ((s = prepare_x(planes, FK_BF16X2, N, d, L, ws, nullptr, st, &pl, &nplanes, &lda,
                       &xn)) != FK_OK)
        return s;
    // the planes feed the tensor cores, the fp32 rows the exact re-ranking
    return run_assign(pl, nplanes, lda, N, d, K, L, ws, labels, xn, mind, st, X, C);
}

fk_status fk_update(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                    const int32_t *labels, const float *C_old, float *C_new, int32_t *counts,
                    int32_t *offsets, int32_t *perm, double *objective, void *ws,
                    size_t ws_bytes, fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, FK_L2);
    if (s != FK_OK) return s;
    if (!X || !labels || !C_old || !C_new || !counts || !offsets) return FK_ERR_INVALID_ARG;
    const size_t cbytes = sizeof(float) * static_cast<size_t>(K) * d;
    if (overlap(C_old, cbytes, C_new, cbytes)) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(C_old, 16) || !aligned(C_new, 16) || !aligned(labels, 4) ||
        !aligned(counts, 4) || !aligned(offsets, 4) || (perm && !aligned(perm, 4)) ||
        (objective && !aligned(objective, 8)))
        return FK_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(N, d, K, dtype, FK_L2);
    if ((s = check_ws(ws, ws_bytes, L)) != FK_OK) return s;
    if ((s = check_device()) != FK_OK) return s;
    if (injected_fault() == kFaultLaunch) return FK_ERR_CUDA;
    cudaStream_t st = stream;
    const float *C_used = C_old;
    if (dtype == FK_BF16) {
        FK_TRY_CUDA(launch_prep_centroids(C_old, K, d, L.Kp, L.dp, dtype,
                                          ws_ptr<uint16_t>(ws, L.cs), ws_ptr<float>(ws, L.cn),
                                          ws_ptr<float>(ws, L.cused), nullptr, st));
        C_used = ws_ptr<float>(ws, L.cused);
    }
    return run_update(X, dtype, N, d, K, L, ws, labels, C_old, C_used, C_new, counts, offsets,
                      perm, objective, nullptr, st);
}

fk_status fk_lloyd(const void *X, fk_dtype dtype, int64_t N, int d, int K, fk_metric metric,
                   int niter, float *C, int32_t *labels, int32_t *counts, int32_t *offsets,
                   double *objective_host, fk_timing *timing, void *ws, size_t ws_bytes,
                   fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, metric);
    if (s != FK_OK) return s;
    if (!X || !C || !labels || niter < 0) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(C, 16) || !aligned(labels, 4) ||
        (counts && !aligned(counts, 4)) || (offsets && !aligned(offsets, 4)))
        return FK_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(N, d, K, dtype, metric);
    if ((s = check_ws(ws, ws_bytes, L)) != FK_OK) return s;
    if ((s = check_device()) != FK_OK) return s;
    if (injected_fault() == kFaultLaunch) return FK_ERR_CUDA;
    cudaStream_t st = stream;

    // Timing events: [0] call start, [1] end of the setup, then (pool or graph) 4 per
    // iteration (after prep, assign, sort, update) and 2 per iteration around the
    // assignment's tensor-core kernel; with kernel_only, only the last two.
    const bool kernel_only = timing && timing->kernel_only != 0;
    const bool mma_last_only = kernel_only && timing->kernel_only == 2;
    const bool phases = timing && !kernel_only;
    std::vector<cudaEvent_t> *pool = nullptr;
    if (timing && !pooled_events(2 + 6 * static_cast<size_t>(niter), &pool))
        return FK_ERR_CUDA;

    NvtxRange call_range("fk_lloyd");
    if (cudaMemsetAsync(ws_ptr<uint32_t>(ws, L.err), 0, kErrWords * sizeof(uint32_t), st) != cudaSuccess)
        return FK_ERR_CUDA;
    const long launches0 = g_launches;
    if (phases && cudaEventRecord((*pool)[0], st) != cudaSuccess) return FK_ERR_CUDA;
    const void *Xp = X;
    if (metric == FK_COSINE) {
        float *xn = ws_ptr<float>(ws, L.xn);
        if (launch_normalize(static_cast<const float *>(X), xn, N, d, st) != cudaSuccess ||
            launch_normalize(C, C, K, d, st) != cudaSuccess)
            return FK_ERR_CUDA;
        Xp = xn;
    }
    const void *planes = nullptr;
    int nplanes = 0;
    int64_t lda = 0;
    // fp32 points: ||x||^2 per row for the screening window, computed by the split
    float *xnorm = dtype == FK_F32 ? ws_ptr<float>(ws, L.xnorm) : nullptr;
    if (niter > 0 &&
        (s = prepare_x(Xp, dtype, N, d, L, ws, xnorm, st, &planes, &nplanes, &lda)) != FK_OK)
        return s;

    float *C_alt = ws_ptr<float>(ws, L.calt);
    int32_t *cnt = counts ? counts : ws_ptr<int32_t>(ws, L.cnt);
    int32_t *off = offsets ? offsets : ws_ptr<int32_t>(ws, L.off);
    double *obj = ws_ptr<double>(ws, L.obj);
    float *cused = ws_ptr<float>(ws, L.cused);
    bool allow_screen = true;
    // the probe runs where fk_assign would take the screened route for these fp32 points by
    // choice (beyond kThreeProductMaxDp it has no choice: nothing to probe)
    const bool probe = niter > 0 && dtype == FK_F32 && lda == L.dp &&
                       L.dp <= kThreeProductMaxDp &&
                       screened_route(N, static_cast<int>(L.dp), static_cast<int>(L.Kp), K);
    if (probe) {
        // Where the screened route applies, try it first on a sample of the rows with the
        // initial centroids and read how many would need the three-product pass (a single
        // host synchronisation per call); screen the call only if few would.
        bool probed = false;
        if (launch_prep_centroids(C, K, d, L.Kp, L.dp, dtype, ws_ptr<uint16_t>(ws, L.cs),
                                  ws_ptr<float>(ws, L.cn), cused, ws_ptr<uint16_t>(ws, L.caug),
                                  st) != cudaSuccess)
            return FK_ERR_CUDA;
        if ((s = run_assign(planes, nplanes, lda, N, d, K, L, ws, labels, xnorm, nullptr, st,
                            static_cast<const float *>(Xp), C, true, &probed, nullptr,
                            nullptr, kScreenProbeRows)) != FK_OK)
            return s;
        if (probed) {
            uint32_t nfb = 0;
            if (cudaMemcpyAsync(&nfb, ws_ptr<uint32_t>(ws, L.nfb), sizeof(nfb),
                                cudaMemcpyDeviceToHost, st) != cudaSuccess ||
                cudaStreamSynchronize(st) != cudaSuccess)
                return FK_ERR_CUDA;
            const int64_t n = N < kScreenProbeRows ? N : kScreenProbeRows;
            allow_screen = static_cast<int64_t>(nfb) * kScreenMaxFallback <= n;
        }
    }
    if (phases && cudaEventRecord((*pool)[1], st) != cudaSuccess) return FK_ERR_CUDA;

    // The iteration loop, issued on stream s.  lev holds 4 events per iteration and mev 2,
    // both null without timing.  With sync_objective the objective ring is copied to the
    // host whenever it fills (never inside a graph, which is only used below the ring size).
    int copied = 0;
    auto issue_loop = [&](cudaStream_t s_, const cudaEvent_t *lev, const cudaEvent_t *mev,
                          bool sync_objective, int *nscreened_out,
                          bool *last_screened_out) -> fk_status {
        float *Ccur = C, *Cnext = C_alt;
        auto rec = [&](int i) { return !lev || record_event(lev[i], s_) == cudaSuccess; };
        int nscr = 0;
        bool last = false;
        // the centroid operands; a small problem's update prepares the next iteration's
        const CentroidOperands ops{ws_ptr<uint16_t>(ws, L.cs), ws_ptr<float>(ws, L.cn),
                                   dtype == FK_F32 ? nullptr : cused,
                                   ws_ptr<uint16_t>(ws, L.caug), L.Kp, L.dp,
                                   dtype == FK_F32 ? 1 : 0};
        bool prepped = false;
        for (int t = 0; t < niter; ++t) {
            NvtxRange iter_range("fk_lloyd iteration");
            if ((!prepped &&
                 launch_prep_centroids(Ccur, K, d, L.Kp, L.dp, dtype, ws_ptr<uint16_t>(ws, L.cs),
                                       ws_ptr<float>(ws, L.cn), cused,
                                       ws_ptr<uint16_t>(ws, L.caug), s_) != cudaSuccess) ||
                !rec(4 * t))
                return FK_ERR_CUDA;
            bool screened = false;
            const bool timed = mev && (!mma_last_only || t == niter - 1);
            fk_status r = run_assign(planes, nplanes, lda, N, d, K, L, ws, labels, xnorm, nullptr,
                                     s_, dtype == FK_F32 ? static_cast<const float *>(Xp) : nullptr,
                                     Ccur, allow_screen, &screened, timed ? mev[2 * t] : nullptr,
                                     timed ? mev[2 * t + 1] : nullptr);
            if (r != FK_OK) return r;
            nscr += screened ? 1 : 0;
            last = screened;
            if (!rec(4 * t + 1)) return FK_ERR_CUDA;
            NvtxRange upd_range("sort + update");
            const int32_t *skeys = nullptr, *perm = nullptr;
            if (launch_sort_csr(labels, N, K, L.sp, ws_ptr<int32_t>(ws, L.keys0),
                                ws_ptr<int32_t>(ws, L.keys1), ws_ptr<int32_t>(ws, L.vals0),
                                ws_ptr<int32_t>(ws, L.vals1), nullptr,
                                ws_ptr<uint32_t>(ws, L.hist), ws_ptr<uint32_t>(ws, L.dtot), off,
                                &skeys, &perm, ws_ptr<uint32_t>(ws, L.err), s_) != cudaSuccess ||
                !rec(4 * t + 2))
                return FK_ERR_CUDA;
            if (launch_update(Xp, dtype, N, d, K, L.up, skeys, perm, off, Ccur,
                              dtype == FK_F32 ? Ccur : cused, Cnext, cnt,
                              ws_ptr<double>(ws, L.pieces), ws_ptr<int32_t>(ws, L.pkeys),
                              ws_ptr<double>(ws, L.piecesb), ws_ptr<int32_t>(ws, L.pkeysb),
                              ws_ptr<double>(ws, L.jpart), obj + (t % kObjRing),
                              ws_ptr<uint32_t>(ws, L.err), nullptr, s_, &ops,
                              &prepped) != cudaSuccess ||
                !rec(4 * t + 3))
                return FK_ERR_CUDA;
            float *tmp = Ccur;
            Ccur = Cnext;
            Cnext = tmp;
            if (sync_objective && (t + 1) % kObjRing == 0) {
                // the ring is full: hand it to the caller before it wraps
                if (objective_host &&
                    (cudaMemcpyAsync(objective_host + copied, obj, sizeof(double) * kObjRing,
                                     cudaMemcpyDeviceToHost, s_) != cudaSuccess ||
                     cudaStreamSynchronize(s_) != cudaSuccess))
                    return FK_ERR_CUDA;
                copied += kObjRing;
            }
        }
        *nscreened_out = nscr;
        *last_screened_out = last;
        return FK_OK;
    };

    // The end of the call on stream s: the final centroids back into C, the last
    // iteration's statistics (timing of every phase), then the error words, the
    // statistics and the objectives not yet copied into the pinned stage, and the error
    // flags cleared for the next call.
    CallStage *stage = call_stage();
    if (!stage) return FK_ERR_CUDA;
    auto issue_tail = [&](cudaStream_t s_, bool last_scr) -> fk_status {
        float *Cfinal = niter % 2 ? C_alt : C;
        uint32_t *errw = ws_ptr<uint32_t>(ws, L.err);
        if (Cfinal != C &&
            cudaMemcpyAsync(C, Cfinal, sizeof(float) * static_cast<size_t>(K) * d,
                            cudaMemcpyDeviceToDevice, s_) != cudaSuccess)
            return FK_ERR_CUDA;
        if (phases && niter > 0) {
            // words 4, 5 of the error block: the empty-cluster count and the largest cluster
            if (launch_cluster_stats(cnt, K, errw + 4, s_) != cudaSuccess) return FK_ERR_CUDA;
            if (last_scr && cudaMemcpyAsync(&stage->words[6], ws_ptr<uint32_t>(ws, L.nfb),
                                            sizeof(uint32_t), cudaMemcpyDeviceToHost,
                                            s_) != cudaSuccess)
                return FK_ERR_CUDA;
        }
        if (cudaMemcpyAsync(stage->words, errw, 6 * sizeof(uint32_t), cudaMemcpyDeviceToHost,
                            s_) != cudaSuccess ||
            (niter > copied &&
             cudaMemcpyAsync(stage->obj, obj, sizeof(double) * (niter - copied),
                             cudaMemcpyDeviceToHost, s_) != cudaSuccess) ||
            cudaMemsetAsync(errw, 0, 2 * sizeof(uint32_t), s_) != cudaSuccess)
            return FK_ERR_CUDA;
        return FK_OK;
    };

    int nscreened = 0;
    bool last_screened = false;
    const cudaEvent_t *lev = phases ? pool->data() + 2 : nullptr;
    const cudaEvent_t *mev = timing ? pool->data() + 2 + 4 * static_cast<size_t>(niter) : nullptr;
    bool replayed = false;
    int dev = 0;
    const uint64_t ctx = context_id();
    const bool short_call = 2.0 * static_cast<double>(N) * K * d * niter <= kLoopGraphMaxFlops;
    if (niter > 0 && niter < kObjRing && short_call && loop_graphs_enabled() && ctx != 0 &&
        cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
        LoopGraphCache &cache = loop_graphs();
        // graphs and capture streams of another context are dropped unreleased
        for (size_t i = cache.graphs.size(); i-- > 0;)
            if (cache.graphs[i].key.ctx != ctx)
                cache.graphs.erase(cache.graphs.begin() + static_cast<long>(i));
        if (cache.capture_ctx[dev] != ctx) {
            cache.capture[dev] = nullptr;
            cache.capture_ctx[dev] = ctx;
        }
        const LoopKey key{X,    C,     labels, counts, offsets, ws,     ws_bytes, N,
                          d,    K,     niter,  dev,    ctx,     dtype,  metric,
                          timing ? (kernel_only ? (mma_last_only ? 3 : 1) : 2) : 0,
                          allow_screen};
        LoopGraph *g = nullptr;
        for (LoopGraph &c : cache.graphs)
            if (c.key == key) g = &c;
        if (!g && cache.have_last && cache.last == key) {
            // second identical call in a row: capture the loop on this thread's capture
            // stream (nothing runs during a capture) and keep the instantiated graph
            LoopGraph ng;
            ng.key = key;
            bool ok = true;
            if (timing) {
                ng.ev.reserve(6 * static_cast<size_t>(niter));
                for (int i = 0; ok && i < 6 * niter; ++i) {
                    cudaEvent_t e;
                    ok = cudaEventCreate(&e) == cudaSuccess;
                    if (ok) ng.ev.push_back(e);
                }
            }
            if (ok && !cache.capture[dev])
                ok = cudaStreamCreateWithFlags(&cache.capture[dev], cudaStreamNonBlocking) ==
                     cudaSuccess;
            cudaStream_t cs = cache.capture[dev];
            if (ok && timing) {  // the side stream is created outside the capture
                SideStream *ss = side_stream();
                ok = ss != nullptr;
                if (ok) ss->used = false;  // nothing left over from a failed capture
            }
            if (ok && cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) == cudaSuccess) {
                const long l0 = g_launches;
                fk_status r =
                    issue_loop(cs, phases ? ng.ev.data() : nullptr,
                               timing ? ng.ev.data() + 4 * niter : nullptr, false,
                               &ng.nscreened, &ng.last_screened);
                if (r == FK_OK) r = issue_tail(cs, ng.last_screened);
                if (join_side_stream(cs) != cudaSuccess) r = FK_ERR_CUDA;
                cudaGraph_t graph = nullptr;
                const cudaError_t ee = cudaStreamEndCapture(cs, &graph);
                ng.launches = g_launches - l0;
                g_launches = l0;
                ok = r == FK_OK && ee == cudaSuccess && graph != nullptr &&
                     cudaGraphInstantiate(&ng.exec, graph, 0) == cudaSuccess;
                if (graph) cudaGraphDestroy(graph);
            } else {
                ok = false;
            }
            if (!ok) {
                // a failed capture leaves this call (and, remembered, later ones with the
                // same key) to the eager path
                release(ng);
                cudaGetLastError();
            }
            if (cache.graphs.size() >= kLoopGraphs) {
                size_t lru = 0;
                for (size_t i = 1; i < cache.graphs.size(); ++i)
                    if (cache.graphs[i].used < cache.graphs[lru].used) lru = i;
                release(cache.graphs[lru]);
                cache.graphs.erase(cache.graphs.begin() + static_cast<long>(lru));
            }
            cache.graphs.push_back(std::move(ng));
            g = &cache.graphs.back();
        }
        cache.last = key;
        cache.have_last = true;
        if (g) g->used = ++cache.clock;
        if (g && g->exec) {
            if (cudaGraphLaunch(g->exec, st) != cudaSuccess) return FK_ERR_CUDA;
            note_launch(static_cast<int>(g->launches));
            nscreened = g->nscreened;
            last_screened = g->last_screened;
            if (timing) {
                lev = phases ? g->ev.data() : nullptr;
                mev = g->ev.data() + 4 * niter;
            }
            replayed = true;
        }
    }
    if (!replayed &&
        ((s = issue_loop(st, lev, mev, true, &nscreened, &last_screened)) != FK_OK ||
         (s = issue_tail(st, last_screened)) != FK_OK))
        return s;
    if (cudaStreamSynchronize(st) != cudaSuccess) return FK_ERR_CUDA;
    if (objective_host && niter > copied)
        std::memcpy(objective_host + copied, stage->obj, sizeof(double) * (niter - copied));
    const uint32_t flags[2] = {stage->words[0], stage->words[1]};
    const int code = decode_err(flags);
    uint32_t stats[3] = {0, 0, 0};
    if (phases && niter > 0) {
        stats[0] = stage->words[4];
        stats[1] = stage->words[5];
        stats[2] = last_screened ? stage->words[6] : 0u;
    }
    if (timing) {
        float ms = 0.f;
        std::memset(timing, 0, sizeof(*timing));
        timing->kernel_only = kernel_only ? (mma_last_only ? 2 : 1) : 0;
        timing->empty_clusters = static_cast<int>(stats[0]);
        timing->max_cluster = static_cast<int>(stats[1]);
        timing->fallback_rows = static_cast<int>(stats[2]);
        const cudaEvent_t e0 = (*pool)[0], e1 = (*pool)[1];
        if (phases && elapsed_ms(e0, e1, &ms)) timing->ms_setup = ms;
        double *slot[4] = {&timing->ms_prep, &timing->ms_assign, &timing->ms_sort,
                           &timing->ms_update};
        for (int t = 0; t < niter; ++t) {
            for (int p = 0; phases && p < 4; ++p) {
                const int a = 4 * t + p;  // phase p of iteration t ends at lev[a]
                const cudaEvent_t from = a == 0 ? e1 : lev[a - 1];
                if (elapsed_ms(from, lev[a], &ms)) *slot[p] += ms;
            }
            if ((!mma_last_only || t == niter - 1) && elapsed_ms(mev[2 * t], mev[2 * t + 1], &ms)) {
                timing->ms_assign_mma += ms;
                ++timing->mma_timed;
            }
        }
        timing->iterations = niter;
        timing->launches = static_cast<int>(g_launches - launches0);
        timing->screened = nscreened;
    }
    return static_cast<fk_status>(code);
}

fk_status fk_ivf_lists(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                       const int32_t *labels, int32_t *offsets, int32_t *row_ids,
                       void *X_lists, void *ws, size_t ws_bytes, fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, FK_L2);
    if (s != FK_OK) return s;
    if (!X || !labels || !offsets || !row_ids) return FK_ERR_INVALID_ARG;
    const size_t xbytes = static_cast<size_t>(N) * d * (dtype == FK_F32 ? 4 : 2);
    if (X_lists && overlap(X, xbytes, X_lists, xbytes)) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(labels, 4) || !aligned(offsets, 4) ||
        !aligned(row_ids, 4) || (X_lists && !aligned(X_lists, 16)))
        return FK_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(N, d, K, dtype, FK_L2);
    if ((s = check_ws(ws, ws_bytes, L)) != FK_OK) return s;
    if ((s = check_device()) != FK_OK) return s;
    cudaStream_t st = stream;
    const int32_t *skeys = nullptr, *perm = nullptr;
    FK_TRY_CUDA(launch_sort_csr(labels, N, K, L.sp, ws_ptr<int32_t>(ws, L.keys0),
                                ws_ptr<int32_t>(ws, L.keys1), ws_ptr<int32_t>(ws, L.vals0),
                                ws_ptr<int32_t>(ws, L.vals1), row_ids,
                                ws_ptr<uint32_t>(ws, L.hist), ws_ptr<uint32_t>(ws, L.dtot),
                                offsets, &skeys, &perm, ws_ptr<uint32_t>(ws, L.err), st));
    if (X_lists)
        FK_TRY_CUDA(launch_gather_rows(X, N, static_cast<int64_t>(d) * (dtype == FK_F32 ? 4 : 2),
                                       row_ids, X_lists, st));
    return FK_OK;
}

fk_status fk_update_partial(const void *X, fk_dtype dtype, int64_t N, int d, int K,
                            const int32_t *labels, const float *C_old, double *sums,
                            int32_t *counts, int32_t *offsets, double *objective, void *ws,
                            size_t ws_bytes, fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, FK_L2);
    if (s != FK_OK) return s;
    if (!X || !labels || !C_old || !sums || !counts || !offsets) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(C_old, 16) || !aligned(sums, 16) || !aligned(labels, 4) ||
        !aligned(counts, 4) || !aligned(offsets, 4) || (objective && !aligned(objective, 8)))
        return FK_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(N, d, K, dtype, FK_L2);
    if ((s = check_ws(ws, ws_bytes, L)) != FK_OK) return s;
    if ((s = check_device()) != FK_OK) return s;
    cudaStream_t st = stream;
    const float *C_used = C_old;
    if (dtype == FK_BF16) {
        FK_TRY_CUDA(launch_prep_centroids(C_old, K, d, L.Kp, L.dp, dtype,
                                          ws_ptr<uint16_t>(ws, L.cs), ws_ptr<float>(ws, L.cn),
                                          ws_ptr<float>(ws, L.cused), nullptr, st));
        C_used = ws_ptr<float>(ws, L.cused);
    }
    return run_update(X, dtype, N, d, K, L, ws, labels, C_old, C_used, nullptr, counts,
                      offsets, nullptr, objective, sums, st);
}

fk_status fk_streamed_workspace_size(int64_t chunk_rows, int d, int K, fk_dtype dtype,
                                     fk_metric metric, size_t *bytes) {
    if (!bytes) return FK_ERR_INVALID_ARG;
    fk_status s = validate_shape(chunk_rows, d, K, dtype, metric);
    if (s != FK_OK) return s;
    *bytes = stream_layout(chunk_rows, d, K, dtype).total;
    return FK_OK;
}

fk_status fk_lloyd_streamed(const void *X_host, fk_dtype dtype, int64_t N, int d, int K,
                            fk_metric metric, int niter, float *C, int32_t *labels_host,
                            double *objective_host, int64_t chunk_rows, void *ws,
                            size_t ws_bytes, fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, metric);
    if (s != FK_OK) return s;
    if (!X_host || !C || niter < 0 || niter > kObjRing || chunk_rows < 1)
        return FK_ERR_INVALID_ARG;
    if (chunk_rows > N) chunk_rows = N;
    if (chunk_rows < K) return FK_ERR_INVALID_ARG;
    if (!aligned(C, 16)) return FK_ERR_UNSUPPORTED;
    const StreamLayout S = stream_layout(chunk_rows, d, K, dtype);
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < S.total) return FK_ERR_WORKSPACE;
    if ((s = check_device()) != FK_OK) return s;
    const WsLayout &L = S.L;
    cudaStream_t st = stream;

    // the copy stream, its events, and their release on every exit
    cudaStream_t cs = nullptr;
    cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
    auto cleanup = [&]() {
        for (auto e : ev)
            if (e) cudaEventDestroy(e);
        if (cs) cudaStreamDestroy(cs);
    };
    auto fail = [&](fk_status f) {
        if (cs) cudaStreamSynchronize(cs);
        cleanup();
        return f;
    };
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return FK_ERR_CUDA;
    for (auto &e : ev)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess)
            return fail(FK_ERR_CUDA);
    cudaEvent_t *copied = ev, *done = ev + 2, entry = ev[4];
    // nothing on the copy stream may start before the caller's earlier work on `stream`
    if (cudaEventRecord(entry, st) != cudaSuccess || cudaStreamWaitEvent(cs, entry, 0) != cudaSuccess)
        return fail(FK_ERR_CUDA);

    const size_t row_bytes = static_cast<size_t>(d) * (dtype == FK_F32 ? 4 : 2);
    const size_t KD = static_cast<size_t>(K) * d;
    const int64_t nchunks = ceil_div(N, chunk_rows);
    const char *Xh = static_cast<const char *>(X_host);
    double *sums = ws_ptr<double>(ws, S.sums), *sums_tot = ws_ptr<double>(ws, S.sums_tot);
    int32_t *cnt = ws_ptr<int32_t>(ws, S.cnt), *off = ws_ptr<int32_t>(ws, S.off);
    int64_t *cnt_tot = ws_ptr<int64_t>(ws, S.cnt_tot);
    double *objc = ws_ptr<double>(ws, S.objc), *obj_tot = ws_ptr<double>(ws, S.obj_tot);
    float *xnorm = dtype == FK_F32 ? ws_ptr<float>(ws, L.xnorm) : nullptr;
    float *cused = ws_ptr<float>(ws, L.cused);
    auto rows_of = [&](int64_t c) { return N - c * chunk_rows < chunk_rows ? N - c * chunk_rows : chunk_rows; };

    if (cudaMemsetAsync(ws_ptr<uint32_t>(ws, L.err), 0, kErrWords * sizeof(uint32_t), st) != cudaSuccess)
        return fail(FK_ERR_CUDA);
    if (metric == FK_COSINE && launch_normalize(C, C, K, d, st) != cudaSuccess)
        return fail(FK_ERR_CUDA);
    float *Ccur = C, *Cnext = ws_ptr<float>(ws, S.calt);
    int64_t pend[2] = {-1, -1};  // chunk whose labels wait in lab[slot] for the host copy
    bool allow_screen = true, probed = false;
    int64_t g = 0;
    for (int t = 0; t < niter; ++t) {
        if (cudaMemsetAsync(sums_tot, 0, sizeof(double) * KD, st) != cudaSuccess ||
            cudaMemsetAsync(cnt_tot, 0, sizeof(int64_t) * K, st) != cudaSuccess ||
            cudaMemsetAsync(obj_tot + t, 0, sizeof(double), st) != cudaSuccess)
            return fail(FK_ERR_CUDA);
        if (launch_prep_centroids(Ccur, K, d, L.Kp, L.dp, dtype, ws_ptr<uint16_t>(ws, L.cs),
                                  ws_ptr<float>(ws, L.cn), cused, ws_ptr<uint16_t>(ws, L.caug),
                                  st) != cudaSuccess)
            return fail(FK_ERR_CUDA);
        for (int64_t c = 0; c < nchunks; ++c, ++g) {
            const int slot = static_cast<int>(g & 1);
            const int64_t rows = rows_of(c);
            void *xb = ws_ptr<void>(ws, S.xbuf[slot]);
            int32_t *lab = ws_ptr<int32_t>(ws, S.lab[slot]);
            // copy stream: once the chunk two back is done with this slot, hand its labels
            // to the host (last iteration) and bring in this chunk's points
            if (g >= 2 && cudaStreamWaitEvent(cs, done[slot], 0) != cudaSuccess)
                return fail(FK_ERR_CUDA);
            if (pend[slot] >= 0) {
                if (cudaMemcpyAsync(labels_host + pend[slot] * chunk_rows, lab,
                                    sizeof(int32_t) * rows_of(pend[slot]),
                                    cudaMemcpyDeviceToHost, cs) != cudaSuccess)
                    return fail(FK_ERR_CUDA);
                pend[slot] = -1;
            }
            if (cudaMemcpyAsync(xb, Xh + c * chunk_rows * row_bytes, rows * row_bytes,
                                cudaMemcpyHostToDevice, cs) != cudaSuccess ||
                cudaEventRecord(copied[slot], cs) != cudaSuccess ||
                cudaStreamWaitEvent(st, copied[slot], 0) != cudaSuccess)
                return fail(FK_ERR_CUDA);
            // compute stream: normalise (cosine), assign, partial update, add to the totals
            if (metric == FK_COSINE &&
                launch_normalize(static_cast<float *>(xb), static_cast<float *>(xb), rows, d,
                                 st) != cudaSuccess)
                return fail(FK_ERR_CUDA);
            const void *planes = nullptr;
            const float *xn = nullptr;
            int nplanes = 0;
            int64_t lda = 0;
            if ((s = prepare_x(xb, dtype, rows, d, L, ws, xnorm, st, &planes, &nplanes, &lda,
                               &xn)) != FK_OK)
                return fail(s);
            const float *X32 = dtype == FK_F32 ? static_cast<const float *>(xb) : nullptr;
            if (!probed && dtype == FK_F32) {
                // the screening probe of fk_lloyd, on the first chunk
                probed = true;
                bool p = false;
                if ((s = run_assign(planes, nplanes, lda, rows, d, K, L, ws, lab, xn, nullptr,
                                    st, X32, Ccur, true, &p, nullptr, nullptr,
                                    kScreenProbeRows)) != FK_OK)
                    return fail(s);
                if (p) {
                    uint32_t nfb = 0;
                    if (cudaMemcpyAsync(&nfb, ws_ptr<uint32_t>(ws, L.nfb), sizeof(nfb),
                                        cudaMemcpyDeviceToHost, st) != cudaSuccess ||
                        cudaStreamSynchronize(st) != cudaSuccess)
                        return fail(FK_ERR_CUDA);
                    const int64_t n = rows < kScreenProbeRows ? rows : kScreenProbeRows;
                    allow_screen = static_cast<int64_t>(nfb) * kScreenMaxFallback <= n;
                }
            }
            if ((s = run_assign(planes, nplanes, lda, rows, d, K, L, ws, lab, xn, nullptr, st,
                                X32, Ccur, allow_screen)) != FK_OK)
                return fail(s);
            if ((s = run_update(xb, dtype, rows, d, K, L, ws, lab, Ccur,
                                dtype == FK_BF16 ? cused : Ccur, nullptr, cnt, off, nullptr,
                                objc, sums, st)) != FK_OK)
                return fail(s);
            if (launch_accumulate_chunk(sums_tot, sums, static_cast<int64_t>(KD), cnt_tot, cnt,
                                        K, obj_tot + t, objc, st) != cudaSuccess ||
                cudaEventRecord(done[slot], st) != cudaSuccess)
                return fail(FK_ERR_CUDA);
            if (labels_host && t == niter - 1) pend[slot] = c;
        }
        // new centroids from the iteration's totals (an empty cluster keeps its centroid)
        if (launch_finalize_shards(sums_tot, cnt_tot, nullptr, 1, K, d, Ccur, Cnext, nullptr,
                                   nullptr, st) != cudaSuccess)
            return fail(FK_ERR_CUDA);
        float *tmp = Ccur;
        Ccur = Cnext;
        Cnext = tmp;
    }
    for (int k = 0; k < 2; ++k) {  // the last labels still waiting for their host copy
        const int slot = static_cast<int>((g + k) & 1);
        if (pend[slot] < 0) continue;
        if (cudaStreamWaitEvent(cs, done[slot], 0) != cudaSuccess ||
            cudaMemcpyAsync(labels_host + pend[slot] * chunk_rows,
                            ws_ptr<int32_t>(ws, S.lab[slot]),
                            sizeof(int32_t) * rows_of(pend[slot]), cudaMemcpyDeviceToHost,
                            cs) != cudaSuccess)
            return fail(FK_ERR_CUDA);
    }
    if (Ccur != C && cudaMemcpyAsync(C, Ccur, sizeof(float) * KD, cudaMemcpyDeviceToDevice,
                                     st) != cudaSuccess)
        return fail(FK_ERR_CUDA);
    if (objective_host && niter > 0 &&
        cudaMemcpyAsync(objective_host, obj_tot, sizeof(double) * niter,
                        cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return fail(FK_ERR_CUDA);
    if (cudaStreamSynchronize(cs) != cudaSuccess) return fail(FK_ERR_CUDA);
    int code = FK_OK;
    if (read_err(ws, L, st, true, &code) != FK_OK) return fail(FK_ERR_CUDA);
    cleanup();
    return static_cast<fk_status>(code);
}

fk_status fk_finalize_shards(const double *sums, const int64_t *counts_w,
                             const double *objectives_w, int W, int K, int d,
                             const float *C_old, float *C_new, int64_t *counts,
                             double *objective, fk_stream_t stream) {
    if (W < 1 || K < 1 || d < 1 || !sums || !counts_w || !C_old || !C_new)
        return FK_ERR_INVALID_ARG;
    if ((objective && !objectives_w) || static_cast<int64_t>(K) * d > 2147483647LL)
        return FK_ERR_INVALID_ARG;
    const size_t cbytes = sizeof(float) * static_cast<size_t>(K) * d;
    if (overlap(C_old, cbytes, C_new, cbytes)) return FK_ERR_INVALID_ARG;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    FK_TRY_CUDA(launch_finalize_shards(sums, counts_w, objectives_w, W, K, d, C_old, C_new,
                                       counts, objective, stream));
    return FK_OK;
}

fk_status fk_ivf_norms(const float *V, int64_t n, int d, double *norms, fk_stream_t stream) {
    if (!V || !norms || n < 1 || d < 1) return FK_ERR_INVALID_ARG;
    if (d % 4 != 0 || !aligned(V, 16) || !aligned(norms, 8)) return FK_ERR_UNSUPPORTED;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    FK_TRY_CUDA(launch_sqnorm_f64(V, n, d, norms, stream));
    return FK_OK;
}


fk_status fk_ivf_radii(const float *C, int nlist, const float *X_lists, const int32_t *offsets,
                       int d, float *radius, fk_stream_t stream) {
    if (!C || !X_lists || !offsets || !radius || nlist < 1 || d < 1) return FK_ERR_INVALID_ARG;
    if (d % 4 != 0 || !aligned(C, 16) || !aligned(X_lists, 16) || !aligned(offsets, 4) ||
        !aligned(radius, 4))
        return FK_ERR_UNSUPPORTED;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    FK_TRY_CUDA(launch_cell_radius(C, nlist, X_lists, offsets, d, radius, stream));
    return FK_OK;
}

fk_status fk_ivf_search_workspace_size(int64_t nq, int d, int nlist, int64_t N, int nprobe,
                                       int k, size_t *bytes) {
    if (!bytes) return FK_ERR_INVALID_ARG;
    fk_status s = validate_search(nq, d, nlist, N, nprobe, k);
    if (s != FK_OK) return s;
    *bytes = search_layout(nq, d, nlist, nprobe, k).total;
    return FK_OK;
}

fk_status fk_ivf_search(const float *Q, int64_t nq, int d, const float *C, int nlist,
                        const float *X_lists, const double *X_norms, const void *X_planes,
                        const float *cell_radius, const int32_t *offsets, const int32_t *row_ids, int64_t N, int nprobe,
                        int k, int flags,
                        float *distances, int32_t *ids, int32_t *probes, void *ws,
                        size_t ws_bytes, fk_search_timing *timing, fk_stream_t stream) {
    fk_status s = validate_search(nq, d, nlist, N, nprobe, k);
    if (s != FK_OK) return s;
    if (!Q || !C || !X_lists || !X_norms || !offsets || !row_ids || !distances || !ids)
        return FK_ERR_INVALID_ARG;
    if (!aligned(Q, 16) || !aligned(C, 16) || !aligned(X_lists, 16) || !aligned(X_norms, 8) ||
        !aligned(offsets, 4) || !aligned(row_ids, 4) || !aligned(distances, 4) ||
        !aligned(ids, 4) || (probes && !aligned(probes, 4)) ||
        (X_planes && !aligned(X_planes, 16)) || (cell_radius && !aligned(cell_radius, 4)))
        return FK_ERR_UNSUPPORTED;
    const SearchLayout L = search_layout(nq, d, nlist, nprobe, k);
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < L.total) return FK_ERR_WORKSPACE;
    if (injected_fault() == kFaultWorkspace) return FK_ERR_WORKSPACE;
    if ((s = check_device()) != FK_OK) return s;
    if (injected_fault() == kFaultLaunch) return FK_ERR_CUDA;
    cudaStream_t st = stream;
    cudaEvent_t ev[5] = {};
    auto destroy = [&]() {
        for (cudaEvent_t &e : ev)
            if (e) cudaEventDestroy(e);
    };
    if (timing) {
        for (cudaEvent_t &e : ev)
            if (cudaEventCreate(&e) != cudaSuccess) {
                destroy();
                return FK_ERR_CUDA;
            }
    }
    const bool screen = (flags & FK_SEARCH_FP64_COARSE) == 0 &&
                        ivf_coarse_can_screen(nlist, static_cast<int>(L.dp),
                                              static_cast<int>(L.Kp));
    const bool screen_fine = X_planes != nullptr && (flags & FK_SEARCH_FP64_FINE) == 0 &&
                             k <= kSearchScrMaxK && nprobe <= kSearchScrMaxProbe;
    NvtxRange call_range("fk_ivf_search");
    const fk_status r = run_ivf_search(Q, nq, d, C, nlist, X_lists, X_norms, X_planes,
                                       cell_radius, offsets, row_ids, N, nprobe, k, screen,
                                       screen_fine, distances, ids, probes, ws, L, st,
                                       timing ? ev : nullptr);
    if (r == FK_OK && timing) {
        int nfb = 0;
        if (screen_fine) {  // the flagged-query count sits in the word after the max norm
            int *cnt = ws_ptr<int>(ws, L.xmax2) + 1;
            if (launch_count_flags(ws_ptr<int32_t>(ws, L.fb), nq, cnt, st) != cudaSuccess ||
                cudaMemcpyAsync(&nfb, cnt, sizeof(int), cudaMemcpyDeviceToHost, st) !=
                    cudaSuccess) {
                destroy();
                return FK_ERR_CUDA;
            }
        }
        if (cudaStreamSynchronize(st) != cudaSuccess) {
            destroy();
            return FK_ERR_CUDA;
        }
        timing->fallback_queries = nfb;
        float ms[4] = {0, 0, 0, 0};
        for (int i = 0; i < 4; ++i)
            if (!elapsed_ms(ev[i], ev[i + 1], &ms[i])) ms[i] = 0.f;
        timing->ms_coarse = ms[0];
        timing->ms_sort = ms[1];
        timing->ms_fine = ms[2];
        timing->ms_merge = ms[3];
        timing->screened_coarse = screen ? 1 : 0;
        timing->screened_fine = screen_fine ? 1 : 0;
    }
    destroy();
    return r;
}


fk_status fk_get_device_error(void *ws, size_t ws_bytes, int *code, fk_stream_t stream) {
    if (!ws || !code || ws_bytes < 256 || !aligned(ws, 256)) return FK_ERR_INVALID_ARG;
    WsLayout L;
    L.err = 0;
    return read_err(ws, L, stream, true, code);
}

fk_status fk_selftest_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns,
                              fk_stream_t stream) {
    if (!ws || ws_bytes < 256 || !aligned(ws, 256)) return FK_ERR_INVALID_ARG;
    fk_status s = check_device();
    if (s != FK_OK) return s;
    if (limit_ns > 10000000000ull) return FK_ERR_INVALID_ARG;
    wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint32_t *>(ws), limit_ns);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? FK_OK : FK_ERR_CUDA;
}

}  // extern "C"
