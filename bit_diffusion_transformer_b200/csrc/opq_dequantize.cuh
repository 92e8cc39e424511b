// opq_dequantize.cuh — packed planes -> bf16 W'.
//
// "OPQ INT4 Z-Image" model card, "inference decoding": w = sign * (q/15)^(1/alpha)
// * max. The 16 magnitudes (q/15)^(1/alpha) arrive as fp64 (formed on the host);
// per row, the 16 products with the row scale are formed in fp64 and rounded once
// to bf16 (one per lane), and every weight of the row is then a byte-plane table
// lookup (opq_bits.h decode8) with its sign bit ORed in — the same bits as forming
// the product per weight, since RNE is symmetric under negation.
// One warp per row; a lane takes 32 weights at a time (16 B of codes + one sign word
// in, 64 B out), consecutive lanes on consecutive chunks.
#pragma once
#include "opq_bits.h"
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
                                                         uint32_t chunks, const __grid_constant__ DequantParams dp,
                                                         uint16_t *__restrict__ out) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warps = gridDim.x * (blockDim.x >> 5);
    // lane q (and q + 16) holds LUT[q] for the products
    const double lut_q = dp.lut[lane & 15u];
    for (uint32_t n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < rows; n += warps) {
        const uint4 *crow = reinterpret_cast<const uint4 *>(codes + (size_t)n * chunks * 4u);
        const uint32_t *srow = signs + (size_t)n * chunks;
        uint4 *orow = reinterpret_cast<uint4 *>(out + (size_t)n * chunks * 32u);
        // the first pass's loads go out before the row's table is formed, so that the fp64
        // products and shuffles overlap their latency
        uint4 c[4];
        uint32_t sw[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint32_t i = lane + 32u * u;
            c[u] = i < chunks ? __ldg(crow + i) : make_uint4(0u, 0u, 0u, 0u);
            sw[u] = i < chunks ? __ldg(srow + i) : 0u;
        }
        const uint32_t e = f64_to_bf16_rne(lut_q * (double)__ldg(scales + n));
        opqbits::DecodeTable T;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t l = 0, h = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const uint32_t v = __shfl_sync(0xFFFFFFFFu, e, 4 * j + t);
                l |= (v & 0xFFu) << (8 * t);
                h |= ((v >> 8) & 0xFFu) << (8 * t);
            }
            T.L[j] = l;
            T.H[j] = h;
        }
        // up to four chunks per lane per pass, the next pass's loads issued before decoding
        for (uint32_t i0 = lane; i0 < chunks; i0 += 128u) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t i = i0 + 32u * u;
                if (i >= chunks) break;
                uint32_t o[16];
                opqbits::decode8(c[u].x, sw[u] & 0xFFu, T, &o[0]);
                opqbits::decode8(c[u].y, (sw[u] >> 8) & 0xFFu, T, &o[4]);
                opqbits::decode8(c[u].z, (sw[u] >> 16) & 0xFFu, T, &o[8]);
                opqbits::decode8(c[u].w, sw[u] >> 24, T, &o[12]);
                uint4 *dst = orow + (size_t)i * 4u;
                dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                dst[2] = make_uint4(o[8], o[9], o[10], o[11]);
                dst[3] = make_uint4(o[12], o[13], o[14], o[15]);
            }
            const uint32_t i1 = i0 + 128u;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t i = i1 + 32u * u;
                c[u] = i < chunks ? __ldg(crow + i) : make_uint4(0u, 0u, 0u, 0u);
                sw[u] = i < chunks ? __ldg(srow + i) : 0u;
            }
        }
    }
}

}  // namespace opqk
