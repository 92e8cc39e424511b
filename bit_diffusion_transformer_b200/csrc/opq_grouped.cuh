// opq_grouped.cuh — the group-wise format: one float16 max per GS consecutive
// weights of a row.
//
// "OPQ INT4 Z-Image" model card, "Technical details / storage format": every 128
// weights share one float16 group max (the card's configuration also lists group
// sizes 32, 64 and 256); "OPQ principle" and "inference decoding" as for the
// per-row format, with the group's max in place of the row's. The stored float16
// max (round to nearest even, saturating at 65504) is the one both quantization
// and decoding use.
#pragma once
#include <cuda_fp16.h>

#include "opq_bits.h"
#include "opq_device.cuh"
#include "opq_dequantize.cuh"
#include "opq_quantize.cuh"

namespace opqk {

// float16 bits of a non-negative float: round to nearest even, saturating at 65504
__device__ __forceinline__ uint16_t fp16_bits_sat(float v) {
    const __half h = __float2half_rn(fminf(v, 65504.0f));
    return __half_as_ushort(h);
}

// One warp per row; a round is 256 consecutive weights: lane l holds 16-byte vector
// 32 r + l. A group is VPG = GS / 8 consecutive lanes of a round. Per round: the
// group's max (bf16 bits of |w|) over its lanes, stored as float16; the group's 15
// thresholds, computed by its lanes (lane i of the group takes levels i + 1,
// i + 1 + VPG, ...) and gathered by shuffles; then each lane codes its 8 weights
// with the same branch-free search as the per-row kernel.
template <int GS>
__global__ void __launch_bounds__(256) quantize_grouped_kernel(const uint16_t *__restrict__ w, int64_t N, int64_t K,
                                                               int64_t ldw, const __grid_constant__ QuantParams qp,
                                                               uint32_t *__restrict__ codes,
                                                               uint32_t *__restrict__ signs,
                                                               uint16_t *__restrict__ gmax) {
    constexpr int VPG = GS / 8;                   // lanes per group
    constexpr int TPL = (15 + VPG - 1) / VPG;     // thresholds a lane computes
    static_assert(GS == 32 || GS == 64 || GS == 128 || GS == 256, "group size");
    const int lane = threadIdx.x & 31;
    const int seg = lane & ~(VPG - 1);            // the group's first lane
    const int gl = lane - seg;                    // lane within the group
    const int64_t nvec = K / 8, rounds = (nvec + 31) / 32, ngroups = K / GS;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += warps) {
        const uint16_t *rp = w + n * ldw;
        uint32_t *crow = codes + n * nvec;
        uint32_t *srow = signs + n * (nvec / 4);
        uint4 nxt = make_uint4(0, 0, 0, 0);
        if (lane < nvec) nxt = ld_stream_v4(rp + (int64_t)lane * 8);
        for (int64_t r = 0; r < rounds; ++r) {
            const int64_t vi = r * 32 + lane;
            const bool valid = vi < nvec;             // whole groups only: K % GS == 0
            const uint4 x = nxt;
            if (r + 1 < rounds && vi + 32 < nvec) nxt = ld_stream_v4(rp + (vi + 32) * 8);   // next round in flight
            uint32_t mx2 = __vmaxu2(__vmaxu2(x.x & 0x7FFF7FFFu, x.y & 0x7FFF7FFFu),
                                    __vmaxu2(x.z & 0x7FFF7FFFu, x.w & 0x7FFF7FFFu));
            uint32_t mx = max(mx2 & 0xFFFFu, mx2 >> 16);
#pragma unroll
            for (int o = 1; o < VPG; o <<= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            const uint16_t gb = fp16_bits_sat(__uint_as_float(mx << 16));
            if (valid && gl == 0) gmax[n * ngroups + vi / VPG] = gb;
            const float gm = __half2float(__ushort_as_half(gb));
            uint32_t myT[TPL];
#pragma unroll
            for (int t = 0; t < TPL; ++t) {
                const int k = gl + 1 + t * VPG;
                myT[t] = (k <= 15 && gm != 0.0f) ? level_threshold(gm, k, qp) : 0x7F80u;
            }
            uint32_t P[16];
            P[0] = 0;
#pragma unroll
            for (int k = 1; k < 16; ++k)
                P[k] = __shfl_sync(0xFFFFFFFFu, myT[(k - 1) / VPG], seg + (k - 1) % VPG) * 0x00010001u;
            const uint32_t code = opqbits::pack_codes(opqbits::quant_pair_f(x.x, P), opqbits::quant_pair_f(x.y, P),
                                                      opqbits::quant_pair_f(x.z, P), opqbits::quant_pair_f(x.w, P));
            const uint32_t sb = opqbits::sign_byte(opqbits::bf16x2_neg_mask(x.x), opqbits::bf16x2_neg_mask(x.y),
                                                   opqbits::bf16x2_neg_mask(x.z), opqbits::bf16x2_neg_mask(x.w));
            uint32_t sw = sb << (8 * (lane & 3));
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 1);
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 2);
            if (valid) {
                crow[vi] = code;
                if ((lane & 3) == 0) srow[vi / 4] = sw;
            }
        }
    }
}

// One warp per row; lane l takes 32-weight chunks l, l + 32, ... Every chunk lies in
// one group (GS >= 32); per chunk the lane forms the group's 16 decoded magnitudes
// bf16(LUT[q] * max) from fp64 products, rounded once, and decodes its 32 weights by
// byte-plane lookups (opq_bits.h decode8), the sign bit ORed in.
template <int GS>
__global__ void __launch_bounds__(256) dequantize_grouped_kernel(const uint32_t *__restrict__ codes,
                                                                 const uint32_t *__restrict__ signs,
                                                                 const uint16_t *__restrict__ gmax, uint32_t rows,
                                                                 uint32_t chunks,
                                                                 const __grid_constant__ DequantParams dp,
                                                                 uint16_t *__restrict__ out) {
    constexpr uint32_t CPG = GS / 32;   // chunks per group
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warps = gridDim.x * (blockDim.x >> 5);
    const uint32_t ngroups = chunks / CPG;
    for (uint32_t n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < rows; n += warps) {
        const uint4 *crow = reinterpret_cast<const uint4 *>(codes + (size_t)n * chunks * 4u);
        const uint32_t *srow = signs + (size_t)n * chunks;
        uint4 *orow = reinterpret_cast<uint4 *>(out + (size_t)n * chunks * 32u);
        for (uint32_t i = lane; i < chunks; i += 32u) {
            const uint4 c = __ldg(crow + i);
            const uint32_t sw = __ldg(srow + i);
            const double gm = (double)__half2float(__ushort_as_half(__ldg(gmax + (size_t)n * ngroups + i / CPG)));
            opqbits::DecodeTable T;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t l = 0, h = 0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const uint32_t e = f64_to_bf16_rne(dp.lut[4 * j + t] * gm);
                    l |= (e & 0xFFu) << (8 * t);
                    h |= ((e >> 8) & 0xFFu) << (8 * t);
                }
                T.L[j] = l;
                T.H[j] = h;
            }
            uint32_t o[16];
            opqbits::decode8(c.x, sw & 0xFFu, T, &o[0]);
            opqbits::decode8(c.y, (sw >> 8) & 0xFFu, T, &o[4]);
            opqbits::decode8(c.z, (sw >> 16) & 0xFFu, T, &o[8]);
            opqbits::decode8(c.w, sw >> 24, T, &o[12]);
            uint4 *dst = orow + (size_t)i * 4u;
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
            dst[2] = make_uint4(o[8], o[9], o[10], o[11]);
            dst[3] = make_uint4(o[12], o[13], o[14], o[15]);
        }
    }
}

}  // namespace opqk

namespace opqk {

// Quantization error of one alpha, for the alpha search: per row n, the squared error of the
// decoded weights (sign equal, so (w - w')^2 = (|w| - LUT[q] max)^2 with LUT[q] max in fp32)
// and the weights' squared sum, both accumulated in fp64 in a fixed order. GS = 0: the per-row
// format (the row max first, then the row again); GS > 0: the group-wise format, rounds of 256
// weights as in quantize_grouped_kernel. Codes come from the same exact threshold search.
struct ErrorParams {
    QuantParams qp;
    float lutf[16];   // (q/15)^(1/alpha)
};

template <int GS>
__global__ void __launch_bounds__(256) quant_error_kernel(const uint16_t *__restrict__ w, int64_t N, int64_t K,
                                                          int64_t ldw, const __grid_constant__ ErrorParams ep,
                                                          double *__restrict__ err, double *__restrict__ sig) {
    constexpr int VPG = GS > 0 ? GS / 8 : 32;     // lanes sharing one max in a round (the warp for GS = 0)
    constexpr int TPL = (15 + VPG - 1) / VPG;
    __shared__ float lut_s[16];
    if (threadIdx.x < 16) lut_s[threadIdx.x] = ep.lutf[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int seg = lane & ~(VPG - 1);
    const int gl = lane - seg;
    const int64_t nvec = K / 8, rounds = (nvec + 31) / 32;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); n < N; n += warps) {
        const uint16_t *rp = w + n * ldw;
        uint32_t rowmx = 0;
        if (GS == 0) {
            for (int64_t vi = lane; vi < nvec; vi += 32) {
                const uint4 x = ld_stream_v4(rp + vi * 8);
                const uint32_t m2 = __vmaxu2(__vmaxu2(x.x & 0x7FFF7FFFu, x.y & 0x7FFF7FFFu),
                                             __vmaxu2(x.z & 0x7FFF7FFFu, x.w & 0x7FFF7FFFu));
                rowmx = max(rowmx, max(m2 & 0xFFFFu, m2 >> 16));
            }
            rowmx = __reduce_max_sync(0xFFFFFFFFu, rowmx);
        }
        double e_acc = 0.0, s_acc = 0.0;
        uint32_t P[16];
        P[0] = 0;
        float mxf = __uint_as_float(rowmx << 16);
        if (GS == 0) {
            uint32_t myT = 0x7F80u;
            if (lane < 15 && rowmx != 0u) myT = level_threshold(mxf, lane + 1, ep.qp);
#pragma unroll
            for (int k = 1; k < 16; ++k) P[k] = __shfl_sync(0xFFFFFFFFu, myT, k - 1) * 0x00010001u;
        }
        for (int64_t r = 0; r < rounds; ++r) {
            const int64_t vi = r * 32 + lane;
            const bool valid = vi < nvec;
            const uint4 x = valid ? ld_stream_v4(rp + vi * 8) : make_uint4(0, 0, 0, 0);
            if (GS > 0) {
                const uint32_t m2 = __vmaxu2(__vmaxu2(x.x & 0x7FFF7FFFu, x.y & 0x7FFF7FFFu),
                                             __vmaxu2(x.z & 0x7FFF7FFFu, x.w & 0x7FFF7FFFu));
                uint32_t mx = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
                for (int o = 1; o < VPG; o <<= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                const uint16_t gb = fp16_bits_sat(__uint_as_float(mx << 16));
                mxf = __half2float(__ushort_as_half(gb));
                uint32_t myT[TPL];
#pragma unroll
                for (int t = 0; t < TPL; ++t) {
                    const int k = gl + 1 + t * VPG;
                    myT[t] = (k <= 15 && mxf != 0.0f) ? level_threshold(mxf, k, ep.qp) : 0x7F80u;
                }
#pragma unroll
                for (int k = 1; k < 16; ++k)
                    P[k] = __shfl_sync(0xFFFFFFFFu, myT[(k - 1) / VPG], seg + (k - 1) % VPG) * 0x00010001u;
            }
            const uint32_t words[4] = {x.x, x.y, x.z, x.w};
            float e_r = 0.0f, s_r = 0.0f;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint32_t q2 = opqbits::quant_pair_f(words[p], P);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float a = __uint_as_float(((words[p] >> (16 * h)) & 0x7FFFu) << 16);
                    const float d = a - lut_s[(q2 >> (16 * h)) & 0xFu] * mxf;
                    e_r = fmaf(d, d, e_r);
                    s_r = fmaf(a, a, s_r);
                }
            }
            if (valid) {
                e_acc += (double)e_r;
                s_acc += (double)s_r;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            e_acc += __shfl_xor_sync(0xFFFFFFFFu, e_acc, o);
            s_acc += __shfl_xor_sync(0xFFFFFFFFu, s_acc, o);
        }
        if (lane == 0) {
            err[n] = e_acc;
            sig[n] = s_acc;
        }
    }
}

}  // namespace opqk

namespace opqk {

// ------------------------------------------------------------------------------------------
// Other bit widths (3, 5, 6; 4 is the card's format): 2^BITS - 1 levels per row, the codes of
// a row as one little-endian bit stream (element k at bits k * BITS of the row's words). Their
// quantize is the row-streaming kernel (opq_quantize_stream.cuh) at BITS.
// ------------------------------------------------------------------------------------------
struct BitsDequantParams {
    double lut[64];    // (q/L)^(1/alpha), q = 0..L
};

// One warp per row: the row's L + 1 decoded magnitudes bf16(LUT[q] * scale) (fp64 products,
// rounded once) in shared memory, then lane l takes 32-weight chunks l, l + 32, ...: BITS
// consecutive code words and one sign word in, 64 bytes of bf16 out.
template <int BITS>
__global__ void __launch_bounds__(256) dequantize_bits_kernel(const uint32_t *__restrict__ codes,
                                                              const uint32_t *__restrict__ signs,
                                                              const float *__restrict__ scales, uint32_t rows,
                                                              uint32_t chunks,
                                                              const __grid_constant__ BitsDequantParams dp,
                                                              uint16_t *__restrict__ out) {
    constexpr int L = (1 << BITS) - 1;
    __shared__ uint16_t tab[8][64];
    const uint32_t lane = threadIdx.x & 31u, wi = threadIdx.x >> 5;
    const uint32_t warps = gridDim.x * (blockDim.x >> 5);
    for (uint32_t n = blockIdx.x * (blockDim.x >> 5) + wi; n < rows; n += warps) {
        const double sc = (double)__ldg(scales + n);
        for (int q = lane; q <= L; q += 32) tab[wi][q] = (uint16_t)f64_to_bf16_rne(dp.lut[q] * sc);
        __syncwarp();
        const uint32_t *crow = codes + (size_t)n * chunks * BITS;
        const uint32_t *srow = signs + (size_t)n * chunks;
        uint4 *orow = reinterpret_cast<uint4 *>(out + (size_t)n * chunks * 32u);
        for (uint32_t i = lane; i < chunks; i += 32u) {
            uint32_t cwd[BITS];
#pragma unroll
            for (int j = 0; j < BITS; ++j) cwd[j] = __ldg(crow + (size_t)i * BITS + j);
            const uint32_t sw = __ldg(srow + i);
            uint32_t o[16];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int bit = e * BITS;
                uint32_t q = cwd[bit >> 5] >> (bit & 31);
                if ((bit & 31) + BITS > 32) q |= cwd[(bit >> 5) + 1] << (32 - (bit & 31));
                q &= (uint32_t)L;
                const uint32_t v = (uint32_t)tab[wi][q] | (((sw >> e) & 1u) << 15);
                if (e & 1) o[e >> 1] |= v << 16; else o[e >> 1] = v;
            }
            uint4 *dst = orow + (size_t)i * 4u;
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
            dst[2] = make_uint4(o[8], o[9], o[10], o[11]);
            dst[3] = make_uint4(o[12], o[13], o[14], o[15]);
        }
        __syncwarp();
    }
}

}  // namespace opqk
