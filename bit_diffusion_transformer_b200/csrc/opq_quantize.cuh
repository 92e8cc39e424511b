// opq_quantize.cuh — fused row absmax + power quantization + packing.
//
// "OPQ INT4 Z-Image" model card, "OPQ principle": u = |w|/max, v = u^alpha,
// q = round(15 v); "storage format": 8 magnitudes and 32 signs per uint32.
//
// One row is handled by a group of G warps (G = 1 for K <= 4096, 8 above).
// Every lane loads its 16-byte vectors of the row once (coalesced, kept in
// registers), the group reduces max |w| in the bf16 bit domain, lanes 0..14
// form the 15 exact per-row thresholds in fp64, and each vector of 8 weights is
// coded by a branch-free binary search on two bf16 halves at a time with packed
// bf16 compares (opqbits::quant_pair_f) — no pow on the device.
#pragma once
#include "opq_bits.h"
#include "opq_device.cuh"

namespace opqk {

struct QuantParams {
    double t[16];      // t[k] = ((k - 1/2) / 15)^(1/alpha) for k = 1..15; t[0] unused
    int alpha_is_one;  // thresholds formed as max * (2k - 1) / 30 (exact quotient)
};

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Smallest bf16 magnitude (as bits) that codes to >= k in row with max |w| = mxf.
// Exact with respect to the fp64 threshold th = max * t_k: a bf16 |w| satisfies
// |w| >= th  iff  |w| >= RU_bf16(th). Level k is reached on an exact tie only
// when k is even (round half to even), so odd k needs |w| > th.
__device__ __forceinline__ uint32_t level_threshold(float mxf, int k, const QuantParams &qp) {
    const double th = qp.alpha_is_one ? ((double)mxf * (double)(2 * k - 1)) / 30.0 : (double)mxf * qp.t[k];
    const float f = __double2float_ru(th);
    const uint32_t fb = __float_as_uint(f);
    uint32_t tb = (fb >> 16) + ((fb & 0xFFFFu) != 0u ? 1u : 0u);
    const bool exact = ((fb & 0xFFFFu) == 0u) && ((double)f == th);
    if ((k & 1) && exact) tb += 1u;
    return tb < 0x7F80u ? tb : 0x7F80u;   // +inf: unreachable (only for a non-finite max)
}

template <int G, int VPL>
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t *__restrict__ w, int64_t N, int64_t K,
                                                       int64_t ldw, const __grid_constant__ QuantParams qp,
                                                       uint32_t *__restrict__ codes, uint32_t *__restrict__ signs,
                                                       float *__restrict__ scales) {
    constexpr int ROWS = 8 / G;  // rows per CTA iteration
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = warp / G;
    const int gl = (warp % G) * 32 + lane;  // lane index inside the row group
    const int64_t nvec = K / 8;
    __shared__ uint32_t red[8];

    for (int64_t row0 = (int64_t)blockIdx.x * ROWS; row0 < N; row0 += (int64_t)gridDim.x * ROWS) {
        const int64_t n = row0 + slot;
        const bool valid = n < N;
        const uint16_t *rp = w + (valid ? n : 0) * ldw;
        uint4 v[VPL];
        uint32_t mx2 = 0;
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int64_t vi = (int64_t)j * 32 * G + gl;
            if (valid && vi < nvec) {
                v[j] = ld_stream_v4(rp + vi * 8);
            } else {
                v[j] = make_uint4(0, 0, 0, 0);
            }
            mx2 = __vmaxu2(mx2, v[j].x & 0x7FFF7FFFu);
            mx2 = __vmaxu2(mx2, v[j].y & 0x7FFF7FFFu);
            mx2 = __vmaxu2(mx2, v[j].z & 0x7FFF7FFFu);
            mx2 = __vmaxu2(mx2, v[j].w & 0x7FFF7FFFu);
        }
        uint32_t mx = max(mx2 & 0xFFFFu, mx2 >> 16);
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (G > 1) {
            if (lane == 0) red[warp] = mx;
            __syncthreads();
#pragma unroll
            for (int g = 0; g < G; ++g) mx = max(mx, red[slot * G + g]);
            __syncthreads();
        }
        const float mxf = __uint_as_float(mx << 16);
        // +inf marks a level no finite weight reaches (all levels of an all-zero row)
        uint32_t myT = 0x7F80u;
        if (lane < 15 && mx != 0u) myT = level_threshold(mxf, lane + 1, qp);
        uint32_t P[16];
        P[0] = 0;
#pragma unroll
        for (int k = 1; k < 16; ++k) P[k] = __shfl_sync(0xFFFFFFFFu, myT, k - 1) * 0x00010001u;

        if (valid && gl == 0) scales[n] = mxf;
        uint32_t *crow = codes + (valid ? n : 0) * nvec;
        uint32_t *srow = signs + (valid ? n : 0) * (nvec / 4);
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int64_t vi = (int64_t)j * 32 * G + gl;
            const uint4 x = v[j];
            const uint32_t code = opqbits::pack_codes(opqbits::quant_pair_f(x.x, P), opqbits::quant_pair_f(x.y, P),
                                                      opqbits::quant_pair_f(x.z, P), opqbits::quant_pair_f(x.w, P));
            // sign bit = w < 0 (so -0.0 stores 0): a packed compare with zero gives 0xFFFF per
            // negative half, whose top bit sign_byte collects
            const uint32_t sb = opqbits::sign_byte(opqbits::bf16x2_neg_mask(x.x), opqbits::bf16x2_neg_mask(x.y),
                                                   opqbits::bf16x2_neg_mask(x.z), opqbits::bf16x2_neg_mask(x.w));
            // four consecutive vectors (lanes gl..gl+3) form one sign word
            uint32_t sw = sb << (8 * (gl & 3));
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 1);
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 2);
            if (valid && vi < nvec) {
                crow[vi] = code;
                if ((gl & 3) == 0) srow[vi / 4] = sw;
            }
        }
    }
}

}  // namespace opqk
