// opq_quantize.cuh — the per-row arithmetic shared by the quantize kernels: the exact
// thresholds of the 15 levels (and of the 2^bits - 1 levels of the other bit widths).
//
// "OPQ INT4 Z-Image" model card, "OPQ principle": u = |w|/max, v = u^alpha, q = round(15 v).
// No pow is evaluated on the device: the host forms t_k = ((k - 1/2)/15)^(1/alpha) in fp64,
// and a row's level k starts at the bf16 magnitude T_k = RU_bf16(max * t_k) (strictly above an
// exact tie for odd k: round half to even), so q(|w|) = #{k : T_k <= |w|} exactly.
// The kernels: opq_quantize_stream.cuh (per-row scale), opq_grouped.cuh (group-wise scale,
// error measurement for the alpha search).
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

// The same for a row coded on L levels (other bit widths): t_k = ((k - 1/2) / L)^(1/alpha), or
// with alpha = 1 the exact quotient max (2k - 1) / (2L).
__device__ __forceinline__ uint32_t level_threshold_levels(float mxf, int k, int L, double tk, int alpha_is_one) {
    const double th = alpha_is_one ? ((double)mxf * (double)(2 * k - 1)) / (double)(2 * L) : (double)mxf * tk;
    const float f = __double2float_ru(th);
    const uint32_t fb = __float_as_uint(f);
    uint32_t tb = (fb >> 16) + ((fb & 0xFFFFu) != 0u ? 1u : 0u);
    const bool exact = ((fb & 0xFFFFu) == 0u) && ((double)f == th);
    if ((k & 1) && exact) tb += 1u;
    return tb < 0x7F80u ? tb : 0x7F80u;
}

}  // namespace opqk
