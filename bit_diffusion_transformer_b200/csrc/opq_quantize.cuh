// opq_quantize.cuh — fused row absmax + power quantization + packing.
//
// "OPQ INT4 Z-Image" model card, "OPQ principle": u = |w|/max, v = u^alpha,
// q = round(15 v); "storage format": 8 magnitudes and 32 signs per uint32.
//
// quantize_kernel (K > 4096): one row is handled by a group of G = 8 warps.
// Every lane loads its 16-byte vectors of the row once (coalesced, kept in
// registers), the group reduces max |w| in the bf16 bit domain, and lanes 0..14
// form the 15 exact per-row thresholds T_k in fp64 — no pow on the device.
//
// Coding by table. For a non-negative bf16 value the bit pattern is monotone in
// the value, so q(|w|) = #{k : T_k <= |w|} is a non-increasing step function of
// d = bits(max) - bits(|w|), and q = 0 from d_z = bits(max) - T_1 + 1 on. The group
// writes the row's table q(d), d = 0..d_z, one byte per entry, into shared memory
// (each thread walks a contiguous run of entries down the thresholds), and every
// weight is then one packed subtract, one clamp and one byte lookup. Rows whose
// table would not fit (d_z >= TAB_ENTRIES: alpha below about 0.16) or whose max is
// NaN take the branch-free binary search on bf16 pairs (opqbits::quant_pair_f).
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

constexpr uint32_t TAB_ENTRIES = 4096;   // bytes of a row's code table

// Table lookups (opqbits::table_pair) index a block's tables with the row's table offset
// base <= 7 * TAB_ENTRIES = 28672 folded in; with max <= 0x7F80 no half passes 16 bits.

template <int G, int VPL>
__global__ void __launch_bounds__(256, 2) quantize_kernel(const uint16_t *__restrict__ w, int64_t N, int64_t K,
                                                       int64_t ldw, const __grid_constant__ QuantParams qp,
                                                       uint32_t *__restrict__ codes, uint32_t *__restrict__ signs,
                                                       float *__restrict__ scales) {
    constexpr int ROWS = 8 / G;  // rows per CTA iteration
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = warp / G;
    const int gl = (warp % G) * 32 + lane;  // lane index inside the row group
    const int64_t nvec = K / 8;
    __shared__ uint32_t red[8];
    __shared__ __align__(16) uint32_t tab[ROWS][TAB_ENTRIES / 4];
    __shared__ uint16_t thr[ROWS][16];

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
        const uint32_t T1 = __shfl_sync(0xFFFFFFFFu, myT, 0);
        const uint32_t dz = T1 <= mx ? mx - T1 + 1u : 0u;
        // group-uniform: mx is the group's max
        const bool by_table = mx <= 0x7F80u && dz < TAB_ENTRIES;

        if (valid && gl == 0) scales[n] = mxf;
        uint32_t *crow = codes + (valid ? n : 0) * nvec;
        uint32_t *srow = signs + (valid ? n : 0) * (nvec / 4);
        uint32_t cw[VPL];
        if (by_table) {
            if (gl < 15) thr[slot][gl + 1] = (uint16_t)myT;
            if (G == 1) __syncwarp(); else __syncthreads();
            // entries 0..dz as words of 4; a thread takes a contiguous run, starting from
            // q(e0) = #{k : T_k <= max - e0} and lowering q as max - e drops below T_q
            const uint32_t words = (dz + 4u) >> 2, per = (words + 32u * G - 1u) / (32u * G);
            const uint32_t w0 = (uint32_t)gl * per, w1 = min(w0 + per, words);
            opqbits::code_table_run(&thr[slot][0], mx, w0, w1, &tab[slot][0]);
            if (G == 1) __syncwarp(); else __syncthreads();
            const uint8_t *tb = reinterpret_cast<const uint8_t *>(&tab[0][0]);
            const uint32_t base = (uint32_t)slot * TAB_ENTRIES;
            const uint32_t mmb = (mx + base) * 0x00010001u, dzb = (dz + base) * 0x00010001u;
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const uint4 x = v[j];
                // q_p holds element 2p in bits 0..3 and element 2p+1 in bits 16..19
                cw[j] = opqbits::pack_codes(opqbits::table_pair(tb, x.x, mmb, dzb), opqbits::table_pair(tb, x.y, mmb, dzb),
                                            opqbits::table_pair(tb, x.z, mmb, dzb), opqbits::table_pair(tb, x.w, mmb, dzb));
            }
            // the table and thresholds are rewritten for the next row only after every
            // thread of the group has finished its lookups
            if (G == 1) __syncwarp(); else __syncthreads();
        } else {
            uint32_t P[16];
            P[0] = 0;
#pragma unroll
            for (int k = 1; k < 16; ++k) P[k] = __shfl_sync(0xFFFFFFFFu, myT, k - 1) * 0x00010001u;
#pragma unroll
            for (int j = 0; j < VPL; ++j) {
                const uint4 x = v[j];
                cw[j] = opqbits::pack_codes(opqbits::quant_pair_f(x.x, P), opqbits::quant_pair_f(x.y, P),
                                            opqbits::quant_pair_f(x.z, P), opqbits::quant_pair_f(x.w, P));
            }
        }
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int64_t vi = (int64_t)j * 32 * G + gl;
            const uint4 x = v[j];
            // sign bit = w < 0 (so -0.0 stores 0): a packed compare with zero gives 0xFFFF per
            // negative half, whose top bit sign_byte collects
            const uint32_t sb = opqbits::sign_byte(opqbits::bf16x2_neg_mask(x.x), opqbits::bf16x2_neg_mask(x.y),
                                                   opqbits::bf16x2_neg_mask(x.z), opqbits::bf16x2_neg_mask(x.w));
            // four consecutive vectors (lanes gl..gl+3) form one sign word
            uint32_t sw = sb << (8 * (gl & 3));
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 1);
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 2);
            if (valid && vi < nvec) {
                crow[vi] = cw[j];
                if ((gl & 3) == 0) srow[vi / 4] = sw;
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// K <= 4096: one warp per row, two rows per 64-thread block, and the row read twice — a first
// pass for max |w| (8 vectors per lane in flight), a second for the codes (the row is then in
// L2). Holding no row in registers keeps a thread near 60 registers, so every row of a
// projection-sized matrix is in flight at once (about 26 rows per SM) instead of 16 rows per
// SM in two uneven waves. Coding as in quantize_kernel: the row's table where it fits, the
// packed binary search otherwise.
// ------------------------------------------------------------------------------------------
constexpr int QR_ROWS = 2;

struct TableCoder {
    const uint8_t *tb;
    uint32_t mmb, dzb;
    __device__ __forceinline__ uint32_t operator()(const uint4 &x) const {
        return opqbits::pack_codes(opqbits::table_pair(tb, x.x, mmb, dzb), opqbits::table_pair(tb, x.y, mmb, dzb),
                                   opqbits::table_pair(tb, x.z, mmb, dzb), opqbits::table_pair(tb, x.w, mmb, dzb));
    }
};

struct SearchCoder {
    uint32_t P[16];
    __device__ __forceinline__ uint32_t operator()(const uint4 &x) const {
        return opqbits::pack_codes(opqbits::quant_pair_f(x.x, P), opqbits::quant_pair_f(x.y, P),
                                   opqbits::quant_pair_f(x.z, P), opqbits::quant_pair_f(x.w, P));
    }
};

// the coding pass of one row by one warp: vectors lane, lane + 32, ... in batches of B per lane
template <int B, class Coder>
__device__ __forceinline__ void code_row(const Coder &cd, const uint16_t *rp, int64_t nvec, int lane,
                                         uint32_t *crow, uint32_t *srow) {
    for (int64_t v0 = 0; v0 < nvec; v0 += 32 * B) {
        uint4 x[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int64_t vi = v0 + 32 * u + lane;
            x[u] = vi < nvec ? ld_stream_v4(rp + vi * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int64_t vi = v0 + 32 * u + lane;
            const uint32_t code = cd(x[u]);
            const uint32_t sb = opqbits::sign_byte(opqbits::bf16x2_neg_mask(x[u].x), opqbits::bf16x2_neg_mask(x[u].y),
                                                   opqbits::bf16x2_neg_mask(x[u].z), opqbits::bf16x2_neg_mask(x[u].w));
            // four consecutive vectors (lanes 4m .. 4m+3 of one batch slot) form one sign word
            uint32_t sw = sb << (8 * (lane & 3));
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 1);
            sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 2);
            if (vi < nvec) {
                crow[vi] = code;
                if ((lane & 3) == 0) srow[vi / 4] = sw;
            }
        }
    }
}

__global__ void __launch_bounds__(64) quantize_rows_kernel(const uint16_t *__restrict__ w, int64_t N, int64_t K,
                                                           int64_t ldw, const __grid_constant__ QuantParams qp,
                                                           uint32_t *__restrict__ codes,
                                                           uint32_t *__restrict__ signs,
                                                           float *__restrict__ scales) {
    constexpr int B = 8;
    const int lane = threadIdx.x & 31, slot = threadIdx.x >> 5;
    const int64_t nvec = K / 8;
    __shared__ __align__(16) uint32_t tab[QR_ROWS][TAB_ENTRIES / 4];
    __shared__ uint16_t thr[QR_ROWS][16];

    // warps never wait on one another (only __syncwarp below), so a warp without a row leaves
    for (int64_t n = (int64_t)blockIdx.x * QR_ROWS + slot; n < N; n += (int64_t)gridDim.x * QR_ROWS) {
        const uint16_t *rp = w + n * ldw;
        uint32_t mx2 = 0;
        for (int64_t v0 = 0; v0 < nvec; v0 += 32 * B) {
            uint4 x[B];
#pragma unroll
            for (int u = 0; u < B; ++u) {
                const int64_t vi = v0 + 32 * u + lane;
                x[u] = vi < nvec ? ld_stream_v4(rp + vi * 8) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < B; ++u) {
                mx2 = __vmaxu2(mx2, x[u].x & 0x7FFF7FFFu);
                mx2 = __vmaxu2(mx2, x[u].y & 0x7FFF7FFFu);
                mx2 = __vmaxu2(mx2, x[u].z & 0x7FFF7FFFu);
                mx2 = __vmaxu2(mx2, x[u].w & 0x7FFF7FFFu);
            }
        }
        uint32_t mx = max(mx2 & 0xFFFFu, mx2 >> 16);
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        const float mxf = __uint_as_float(mx << 16);
        uint32_t myT = 0x7F80u;
        if (lane < 15 && mx != 0u) myT = level_threshold(mxf, lane + 1, qp);
        const uint32_t T1 = __shfl_sync(0xFFFFFFFFu, myT, 0);
        const uint32_t dz = T1 <= mx ? mx - T1 + 1u : 0u;
        if (lane == 0) scales[n] = mxf;
        uint32_t *crow = codes + n * nvec;
        uint32_t *srow = signs + n * (nvec / 4);
        if (mx <= 0x7F80u && dz < TAB_ENTRIES) {
            if (lane < 15) thr[slot][lane + 1] = (uint16_t)myT;
            __syncwarp();
            const uint32_t words = (dz + 4u) >> 2, per = (words + 31u) >> 5;
            const uint32_t w0 = (uint32_t)lane * per, w1 = min(w0 + per, words);
            opqbits::code_table_run(&thr[slot][0], mx, w0, w1, &tab[slot][0]);
            __syncwarp();
            const uint32_t base = (uint32_t)slot * TAB_ENTRIES;
            const TableCoder cd{reinterpret_cast<const uint8_t *>(&tab[0][0]), (mx + base) * 0x00010001u,
                                (dz + base) * 0x00010001u};
            code_row<B>(cd, rp, nvec, lane, crow, srow);
            // the row's table and thresholds are rewritten for the next row only after every
            // lane has finished its lookups
            __syncwarp();
        } else {
            SearchCoder cd;
            cd.P[0] = 0;
#pragma unroll
            for (int k = 1; k < 16; ++k) cd.P[k] = __shfl_sync(0xFFFFFFFFu, myT, k - 1) * 0x00010001u;
            code_row<4>(cd, rp, nvec, lane, crow, srow);
        }
    }
}

}  // namespace opqk
