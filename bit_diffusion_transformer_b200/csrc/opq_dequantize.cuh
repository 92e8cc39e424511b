// opq_dequantize.cuh — packed planes -> bf16 W'.
//
// "OPQ INT4 Z-Image" model card, "inference decoding": w = sign * (q/15)^(1/alpha)
// * max. The 16 magnitudes (q/15)^(1/alpha) arrive as fp64 (formed on the host);
// per row, the 16 products with the row scale are formed in fp64 and rounded once
// to bf16 (one per lane), and every weight of the row is then a byte-plane table
// lookup (opq_bits.h decode8) with its sign bit ORed in — the same bits as forming
// the product per weight, since RNE is symmetric under negation.
// One warp per row, four rows per block; a lane takes one code word (8 weights) at a
// time, consecutive lanes on consecutive words; a launch runs one matrix or a list.
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

// Lane l of a row's warp takes the code words l, l + 32, ... (8 weights each): per word a
// 4-byte code load, its sign byte, and a 16-byte bf16 store, so that each warp-wide store
// covers 512 contiguous bytes. The first batch of loads goes out before the row's table
// is formed, so the fp64 products and shuffles overlap their latency.
// One launch runs a list of matrices (one for opq_dequantize, up to DQ_MAX_JOBS for
// opq_dequantize_batched): their rows form one sequence that the warps take in strides, so
// the matrices' ends overlap instead of each launch ramping up and draining on its own.
constexpr int DQ_BATCH = 16;   // code words per lane in flight
constexpr int DQ_MAX_JOBS = 128;

struct DqJob {
    const uint32_t *codes;   // [N, K/8]
    const uint32_t *signs;   // [N, K/32]
    const float *scales;     // [N]
    uint16_t *out;           // bf16 [N, K]
    int64_t row_begin;       // first row of this matrix in the launch's row sequence
    uint32_t N, chunks;      // rows, K / 32
};

struct DqParams {
    DequantParams dp;
    int64_t rows;            // all rows of the launch
    int32_t njobs;
    int32_t pad;
    DqJob job[DQ_MAX_JOBS];
};

__global__ void __launch_bounds__(128) dequantize_kernel(const __grid_constant__ DqParams p) {
    const uint32_t lane = threadIdx.x & 31u;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    // lane q (and q + 16) holds LUT[q] for the products
    const double lut_q = p.dp.lut[lane & 15u];
    int jb = 0;
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < p.rows; u += warps) {
        while (jb + 1 < p.njobs && u >= p.job[jb + 1].row_begin) ++jb;   // rows only grow per warp
        const DqJob &J = p.job[jb];
        const int64_t n = u - J.row_begin;
        const uint32_t chunks = J.chunks;
        const uint32_t nwords = chunks * 4u;   // code words per row
        const uint32_t *crow = J.codes + (size_t)n * nwords;
        const uint8_t *sbytes = reinterpret_cast<const uint8_t *>(J.signs + (size_t)n * chunks);
        uint4 *orow = reinterpret_cast<uint4 *>(J.out + (size_t)n * chunks * 32u);
        uint32_t c[DQ_BATCH], sb[DQ_BATCH];
#pragma unroll
        for (int k = 0; k < DQ_BATCH; ++k) {
            const uint32_t j = lane + 32u * k;
            c[k] = j < nwords ? __ldg(crow + j) : 0u;
            sb[k] = j < nwords ? (uint32_t)__ldg(sbytes + j) : 0u;
        }
        const uint32_t e = f64_to_bf16_rne(lut_q * (double)__ldg(J.scales + n));
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
        for (uint32_t j0 = lane;; j0 += 32u * DQ_BATCH) {
#pragma unroll
            for (int k = 0; k < DQ_BATCH; ++k) {
                const uint32_t j = j0 + 32u * k;
                if (j < nwords) {
                    uint32_t o[4];
                    opqbits::decode8(c[k], sb[k], T, o);
                    orow[j] = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            const uint32_t j1 = j0 + 32u * DQ_BATCH;
            if (j1 - lane >= nwords) break;   // warp-uniform: no word of the next batch exists
#pragma unroll
            for (int k = 0; k < DQ_BATCH; ++k) {
                const uint32_t j = j1 + 32u * k;
                c[k] = j < nwords ? __ldg(crow + j) : 0u;
                sb[k] = j < nwords ? (uint32_t)__ldg(sbytes + j) : 0u;
            }
        }
    }
}

}  // namespace opqk
