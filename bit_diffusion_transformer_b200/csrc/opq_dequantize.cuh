// opq_dequantize.cuh — packed planes -> bf16 W'.
//
// "OPQ INT4 Z-Image" model card, "inference decoding": w = sign * (q/15)^(1/alpha)
// * max. The 16 magnitudes (q/15)^(1/alpha) arrive as fp64 (formed on the host),
// the product with the row scale is formed in fp64 and rounded once to bf16.
// One thread per code word (8 weights): 4 + 1 bytes in, 16 bytes out.
#pragma once
#include "opq_device.cuh"

namespace opqk {

struct DequantParams {
    double lut[16];   // (q/15)^(1/alpha), q = 0..15
};

// fp64 -> bf16, round to nearest even. The fp64 value is first truncated to
// fp32 with a sticky bit in the last place when inexact (round to odd: fp32
// keeps 16 more bits than bf16, so the final rounding sees the true sign of
// the discarded part), then rounded to bf16 on the bit pattern.
__device__ __forceinline__ uint32_t f64_to_bf16_rne(double p) {
    const float f = __double2float_rz(p);
    uint32_t fb = __float_as_uint(f);
    if ((double)f != p) fb |= 1u;
    if ((fb & 0x7F800000u) == 0x7F800000u && (fb & 0x007FFFFFu) != 0u) return (fb >> 16) | 0x40u;  // NaN
    return (fb + 0x7FFFu + ((fb >> 16) & 1u)) >> 16;
}

__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t *__restrict__ codes,
                                                         const uint32_t *__restrict__ signs,
                                                         const float *__restrict__ scales, uint32_t rows,
                                                         uint32_t nvec, const __grid_constant__ DequantParams dp,
                                                         uint16_t *__restrict__ out) {
    __shared__ double lut[16];
    if (threadIdx.x < 16) lut[threadIdx.x] = dp.lut[threadIdx.x];
    __syncthreads();
    const uint64_t total = (uint64_t)rows * nvec;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t n = i / nvec;
        const uint32_t j = (uint32_t)(i - n * nvec);
        const uint32_t c = __ldg(codes + i);
        const uint32_t sb = (__ldg(signs + n * (nvec / 4) + j / 4) >> (8 * (j & 3))) & 0xFFu;
        const double sc = (double)__ldg(scales + n);
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            uint32_t h[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int idx = 2 * p + e;
                double v = lut[(c >> (4 * idx)) & 0xFu] * sc;
                if ((sb >> idx) & 1u) v = -v;
                h[e] = f64_to_bf16_rne(v);
            }
            o[p] = h[0] | (h[1] << 16);
        }
        reinterpret_cast<uint4 *>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace opqk
