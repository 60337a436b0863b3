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
#include <mutex>

#include "fk_common.cuh"

namespace fk {
namespace {

constexpr size_t kStaticScratchBytes = FK_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device with
// cudaGetSymbolAddress (that device current) and cached.
fk_status scratch_address(void **out) {
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return FK_ERR_CUDA;
        addr[dev] = p;
    }
    *out = addr[dev];
    return FK_OK;
}

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
    if (N < 1 || N > 2147483646LL || d < 1 || K < 1 || K > N) return FK_ERR_INVALID_ARG;
    if (!X || !C || !labels) return FK_ERR_INVALID_ARG;
    if (dtype != FK_F32 && dtype != FK_BF16) return FK_ERR_UNSUPPORTED;
    if ((dtype == FK_F32 && d % 4 != 0) || (dtype == FK_BF16 && d % 8 != 0))
        return FK_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(X) % 16 != 0 || reinterpret_cast<uintptr_t>(C) % 4 != 0 ||
        reinterpret_cast<uintptr_t>(labels) % 4 != 0)
        return FK_ERR_UNSUPPORTED;

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

    int major = 0, minor = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return FK_ERR_CUDA;
    if (major != 10 || minor != 0) return FK_ERR_UNSUPPORTED;

    void *base = nullptr;
    fk_status s = scratch_address(&base);
    if (s != FK_OK) return s;
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
    a.wait_ns = 2000000000ull;
    if (launch_assign(a, st) != cudaSuccess) return FK_ERR_CUDA;

    // synchronous: read the device error words back (no allocation involved)
    uint32_t e[2] = {0, 0};
    if (cudaMemcpyAsync(e, err, sizeof(e), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return FK_ERR_CUDA;
    return e[0] ? FK_ERR_TIMEOUT : FK_OK;
}
