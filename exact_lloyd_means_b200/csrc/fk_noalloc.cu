// fk_noalloc.cu -- fk_assign_noalloc: the assignment step without any caller workspace.
//
// Some callers cannot allocate device memory at all: code running under another
// framework's memory manager (which owns every byte of device memory and forbids
// cudaMalloc behind its back), and latency-critical paths where cudaMalloc/cudaFree would
// implicitly synchronise the device.  For them this entry point takes its scratch (the
// error words, the centroid operand planes, norms and norm pieces, and the bf16 planes of
// X when the points need splitting or padding) from one file-scope device array of fixed
// size, instead of from a caller-provided workspace.  The array is part of the library image:
// every GPU that loads libfk holds it until the process exits.
#include "fk_common.cuh"

namespace fk {
namespace {

constexpr size_t kStaticScratchBytes = FK_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

size_t take(size_t &o, size_t bytes) {
    const size_t at = o;
    o += (bytes + 255) / 256 * 256;
    return at;
}

}  // namespace
}  // namespace fk

using namespace fk;

extern "C" FK_API fk_status fk_assign_noalloc(const void *X, fk_dtype dtype, int64_t N, int d,
                                              const float *C, int K, int32_t *labels,
                                              fk_stream_t stream) {
    fk_status s = validate_shape(N, d, K, dtype, FK_L2);
    if (s != FK_OK) return s;
    if (!X || !C || !labels) return FK_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(C, 4) || !aligned(labels, 4)) return FK_ERR_UNSUPPORTED;

    // scratch layout inside the static array
    const int64_t dp = round_up(d, kBK), Kp = round_up(K, kBN);
    const int cplanes = dtype == FK_F32 ? 2 : 1;
    const int xplanes = dtype == FK_F32 ? 2 : ((d % kBK) != 0 ? 1 : 0);
    size_t o = 0;
    const size_t o_err = take(o, 256);
    const size_t o_cs = take(o, sizeof(uint16_t) * cplanes * Kp * dp);
    const size_t o_cn = take(o, sizeof(float) * Kp);
    const size_t o_ca = take(o, sizeof(uint16_t) * Kp * kAug);
    const size_t o_xs = take(o, sizeof(uint16_t) * xplanes * N * dp);
    if (o > kStaticScratchBytes) return FK_ERR_WORKSPACE;  // beyond the static maximum
    if ((s = check_device()) != FK_OK) return s;
    // fk_assign sends some fp32 problems to the screened route, whose candidate and
    // re-ranking buffers this array does not hold; those are refused here, so the labels
    // always come from the same kernel as fk_assign's.  (Every depth beyond 768 is such a
    // problem; below it, no problem that fits the array has enough rows to be screened.)
    if (dtype == FK_F32 && screened_route(N, static_cast<int>(dp), static_cast<int>(Kp), K))
        return FK_ERR_UNSUPPORTED;
    if (injected_fault() == kFaultLaunch) return FK_ERR_CUDA;

    // In host code g_noalloc_scratch names a host-side stand-in, not device memory: the
    // array's address on the current device is looked up on every call (cheap next to the
    // launches and the synchronisation below), so nothing cached can outlive a context.
    void *base = nullptr;
    if (cudaGetSymbolAddress(&base, g_noalloc_scratch) != cudaSuccess || base == nullptr)
        return FK_ERR_CUDA;
    char *sc = static_cast<char *>(base);
    cudaStream_t st = stream;
    uint32_t *err = reinterpret_cast<uint32_t *>(sc + o_err);
    uint16_t *cs = reinterpret_cast<uint16_t *>(sc + o_cs);
    float *cn = reinterpret_cast<float *>(sc + o_cn);
    uint16_t *caug = reinterpret_cast<uint16_t *>(sc + o_ca);
    uint16_t *xs = reinterpret_cast<uint16_t *>(sc + o_xs);

    // the array keeps the previous call's contents: the error words must start at zero
    if (cudaMemsetAsync(err, 0, 2 * sizeof(uint32_t), st) != cudaSuccess) return FK_ERR_CUDA;
    if (launch_prep_centroids(C, K, d, Kp, dp, dtype, cs, cn, nullptr, caug, st) != cudaSuccess)
        return FK_ERR_CUDA;
    AssignArgs a{};
    if (dtype == FK_F32) {
        if (launch_split_x(static_cast<const float *>(X), N, d, dp, xs, xs + N * dp, nullptr,
                           st) != cudaSuccess)
            return FK_ERR_CUDA;
        a.a_planes = xs;
        a.a_nplanes = 2;
        a.lda = dp;
    } else if (xplanes == 1) {
        if (launch_pad_bf16(static_cast<const uint16_t *>(X), N, d, dp, xs, st) != cudaSuccess)
            return FK_ERR_CUDA;
        a.a_planes = xs;
        a.a_nplanes = 1;
        a.lda = dp;
    } else {
        a.a_planes = X;
        a.a_nplanes = 1;
        a.lda = d;
    }
    a.b_planes = cs;
    a.cn = cn;
    a.caug = caug;
    a.N = N;
    a.d = d;
    a.dp = static_cast<int>(dp);
    a.K = K;
    a.Kp = static_cast<int>(Kp);
    a.labels = labels;
    a.best = nullptr;
    a.xnorm = nullptr;
    a.mind = nullptr;
    a.err = err;
    a.wait_ns = kDefaultWaitNs;
    if (launch_assign(a, st) != cudaSuccess) return FK_ERR_CUDA;

    // synchronous: read the device error words back (pageable host memory, no allocation)
    uint32_t e[2] = {0, 0};
    if (cudaMemcpyAsync(e, err, sizeof(e), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return FK_ERR_CUDA;
    return decode_err(e);
}
