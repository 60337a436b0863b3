// prep_row.cuh -- the assign operands of one centroid row: its bf16 planes scaled by -2,
// its squared norm and the norm's exact three-piece bf16 split (see prep.cu).  Shared by
// the per-iteration preparation kernel and the small-problem update, which prepares the
// next iteration's rows as it finishes them; both run this one routine, so the operands
// are the same bits either way.
#pragma once

#include <cuda_bf16.h>

#include "fk_common.cuh"

namespace fk {

__device__ __forceinline__ uint16_t bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float bf16_val(uint16_t b) {
    return __bfloat162float(__ushort_as_bfloat16(b));
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp (all 32 lanes): row k < o.Kp of the operands from the fp32 centroids C (K rows
// of d; rows k >= K are padding).  Planes: [cplanes][Kp][dp] bf16 holding -2*hi (and -2*lo
// for the fp32 emulation); cused (bf16 mode only): the bf16-rounded centroid widened to
// fp32, i.e. exactly what the MMA sees.
__device__ __forceinline__ void prep_centroid_row(const float *__restrict__ C, int K, int d,
                                                  const CentroidOperands &o, int64_t k,
                                                  int lane) {
    uint16_t *p0 = o.planes + k * o.dp;
    uint16_t *p1 = o.planes + (o.Kp + k) * o.dp;
    double s = 0.0;
    for (int64_t j = lane; j < o.dp; j += 32) {
        const float c = (k < K && j < d) ? C[k * d + j] : 0.f;
        const uint16_t h = bf16_bits(c);
        const float hv = bf16_val(h);
        // -2 * bf16 value is exact in bf16 (a power-of-two scale)
        p0[j] = bf16_bits(-2.f * hv);
        if (o.two_planes) {
            const uint16_t l = bf16_bits(c - hv);
            p1[j] = bf16_bits(-2.f * bf16_val(l));
            s += static_cast<double>(c) * c;
        } else {
            s += static_cast<double>(hv) * hv;
            if (k < K && j < d && o.cused) o.cused[k * d + j] = hv;
        }
    }
    s = warp_sum_d(s);
    const float c2 = static_cast<float>(s);
    if (lane == 0) o.cn[k] = k < K ? c2 : __int_as_float(0x7f800000);
    if (o.caug != nullptr && lane < kAug) {
        // exact split: hi captures the top 8 bits, mid the next 8, lo the rest (a
        // multiple of the fp32 ulp with at most 8 significant bits)
        const uint16_t h = bf16_bits(c2);
        const float r1 = c2 - bf16_val(h);
        const uint16_t m = bf16_bits(r1);
        const uint16_t l = bf16_bits(r1 - bf16_val(m));
        uint16_t v = 0;
        if (k < K) v = lane == 0 ? h : (lane == 1 ? m : (lane == 2 ? l : 0));
        else v = lane == 0 ? static_cast<uint16_t>(0x7f7f) : 0;  // largest finite bf16
        o.caug[k * kAug + lane] = v;
    }
}

}  // namespace fk
