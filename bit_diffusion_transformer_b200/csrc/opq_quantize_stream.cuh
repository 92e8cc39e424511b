// opq_quantize_stream.cuh — the row-streaming quantize: one persistent CTA per SM runs a
// list of weight matrices (one matrix, or every linear layer of a model) through a
// shared-memory ring fed by bulk copies.
//
// "OPQ INT4 Z-Image" model card, "OPQ principle": per output row, u = |w| / max,
// v = u^alpha, q = round(15 v); "storage format": 8 magnitudes and 32 signs per uint32.
// The card's whole-model pass ("Quantize and save") quantizes every linear layer of
// the transformer in one go; here that pass is one launch per row-width class.
//
// A row is coded by a group of G warps (G = 1 for K <= 4096, 4 for K <= 16384, 8 up to
// 32768), so that every lane holds at most 16 vectors of 8 weights in registers:
//   warp 16      producer: one bulk copy (cp.async.bulk, completion counted in bytes on the
//                slot's `full` barrier) per row into ring slot i % S, once the slot's
//                previous row has been copied out (`empty`, one arrival per warp of the group)
//   warps 0..15  16 / G consumer groups; group c takes the CTA's rows c, c + 16/G, ...:
//                  copy its part of the row from the slot into registers and hand the slot
//                  back at once; signs (w < 0) and max |w| in one pass over the registers;
//                  the 15 exact thresholds T_k (fp64, lanes 0..14 of every warp); the row's
//                  code table q(d), d = bits(max) - bits(|w|), entries q * 17, built by the
//                  group from the level boundaries with warp ballots; one table read per
//                  weight, a pair's code byte is one merge.
// Every weight is read from HBM once. The ring holds the copies of many rows in flight, the
// registers hold the rows being coded, so the stream does not pause between rows.
// The card's configuration also lists 3, 5 and 6 bits per magnitude: the same kernel at BITS
// codes 2^BITS - 1 levels (thresholds in lanes 0..L-1, and 32..62 a second time for 6 bits),
// table entries q itself, and writes each row's codes as one bit stream: the four lanes that
// hold 32 consecutive weights assemble their BITS words with funnel shifts.
#pragma once
#include "opq_quantize.cuh"

namespace opqk {

using namespace opqdev;

__device__ __forceinline__ uint4 qs_lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

constexpr int QS_MAX_JOBS = 128;          // matrices per launch (they travel as a kernel parameter)
constexpr int QS_CONS_WARPS = 16;
constexpr int QS_THREADS = QS_CONS_WARPS * 32 + 32;   // + the producer warp
constexpr int QS_VMAX = 16;               // 16-byte vectors per lane and row
constexpr int QS_MAX_SLOTS = 64;
constexpr int QS_SMEM_LIMIT = 232448;     // shared memory per CTA (sm_100)
constexpr int QS_OFF_BAR = 0;             // dynamic shared memory: barriers, then the ring
constexpr int QS_OFF_RING = 2 * QS_MAX_SLOTS * 8;

// rows of up to 32 G vectors x QS_VMAX per lane
__host__ __device__ constexpr int qs_group_warps(int64_t K) { return K <= 4096 ? 1 : (K <= 16384 ? 4 : 8); }

// code-table entries per group: 16 groups of one warp share 32 KiB (a group's table offset plus
// max |w| must stay below 2^16 in the packed lookups); larger groups get 4096 entries. With the
// shared mantissa tables (STAB) the per-group tables only serve rows whose max is zero or tiny.
template <int G, bool STAB = false>
struct QsCfg {
    static constexpr int NG = QS_CONS_WARPS / G;           // groups
    static constexpr int TAB = STAB ? 4 : (G == 1 ? 2048 : 4096);   // table entries (bytes) per group
    static constexpr int STATIC_BYTES = NG * TAB + NG * G * 4;
    static constexpr int RING_MAX = QS_SMEM_LIMIT - QS_OFF_RING - STATIC_BYTES - 1024;
    static_assert((NG - 1) * TAB + 0x7F80 < 0x10000, "table offset + max must fit a 16-bit half");
};

struct QsJob {
    const uint16_t *w;     // bf16 [N, ldw]
    uint32_t *codes;       // [N, K bits / 32]: the row's codes (for 4 bits, 8 nibbles per word)
    uint32_t *signs;       // [N, K/32]
    float *scales;         // [N]
    int64_t ldw;
    int64_t row_begin;     // first row of this matrix in the launch's row sequence
    int32_t N, K;
};

struct QsParams {
    QuantParams qp;        // the 15 levels of the 4-bit format (and alpha_is_one for every width)
    double tl[64];         // other widths: t_k = ((k - 1/2) / L)^(1/alpha), k = 1..L
    int64_t rows;          // all rows of the launch
    int32_t njobs;
    int32_t nslots;        // ring slots S
    int32_t slot_bytes;    // a multiple of 128, at least 2 K of every matrix
    int32_t stab_bytes;    // STAB: bytes of the shared mantissa tables before the ring (else 0)
    int32_t stab_stride;   // STAB: bytes per mantissa table (a multiple of 16)
    int32_t pad;
    QsJob job[QS_MAX_JOBS];
};

// The code table q(e) = #{k : B_k > e}, e = 0 .. dz, as dz / 4 + 1 words from the level boundaries
// B_k = bits(max) - T_k + 1 held by lanes (Bk: levels lane + 1, Bk2: 6 bits, lane + 33): per
// stretch of GT words (one per thread tg of the group) one ballot counts the levels that hold over
// the whole stretch and the few boundaries inside it correct each word (no per-entry walk).
// Word w goes to dst[w] times mult (4 bits: 0x11, q in both nibbles; else 1).
template <int GT, int L>
__device__ __forceinline__ void qs_build_table(uint32_t *dst, int Bk, int Bk2, uint32_t dz, int tg, uint32_t mult) {
    const uint32_t words = (dz + 4u) >> 2;
    for (uint32_t i0 = 0; i0 < words; i0 += GT) {
        const int lo_e = (int)(4u * i0), hi_e = lo_e + 4 * GT - 1;
        const uint32_t w = i0 + (uint32_t)tg;
        uint32_t cnt = __popc(__ballot_sync(0xFFFFFFFFu, Bk > hi_e));
        if (L > 32) cnt += __popc(__ballot_sync(0xFFFFFFFFu, Bk2 > hi_e));
        uint32_t word = cnt * 0x01010101u;
        auto inside = [&](int Bl) {
            uint32_t in_m = __ballot_sync(0xFFFFFFFFu, Bl > lo_e && Bl <= hi_e);
            while (in_m) {
                const int k = __ffs(in_m) - 1;
                in_m &= in_m - 1u;
                const int B = __shfl_sync(0xFFFFFFFFu, Bl, k);
                const int c = min(max(B - (int)(4u * w), 0), 4);
                word += __funnelshift_rc(0x01010101u, 0u, 8 * (4 - c));
            }
        };
        inside(Bk);
        if (L > 32) inside(Bk2);
        if (w < words) dst[w] = word * mult;
    }
}

__device__ __forceinline__ void group_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// named-barrier AND over the group's predicates (every thread gets the verdict)
__device__ __forceinline__ bool group_sync_and(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// the job of global row u, moving the caller's cursor forward (rows only grow per thread)
__device__ __forceinline__ int qs_job_of(const QsParams &p, int64_t u, int j) {
    while (j + 1 < p.njobs && u >= p.job[j + 1].row_begin) ++j;
    return j;
}

// The 8 codes q[] of vector v (BITS bits each) into the row's bit stream crow: every lane calls
// this (it shuffles within the lane's quad of consecutive vectors); `valid` lanes store.
template <int BITS>
__device__ __forceinline__ void qs_store_codes(uint32_t *crow, int v, const uint32_t (&q)[8], int lane, bool valid) {
    uint32_t lo, hi;
    opqbits::pack_chunk<BITS>(q, lo, hi);
    const uint32_t nlo = __shfl_down_sync(0xFFFFFFFFu, lo, 1), nhi = __shfl_down_sync(0xFFFFFFFFu, hi, 1);
    uint32_t *quad = crow + (size_t)(v >> 2) * BITS;
#pragma unroll
    for (uint32_t t = 0; t < 2; ++t) {
        uint32_t w, word;
        if (opqbits::quad_word<BITS>(lo, hi, nlo, nhi, (uint32_t)lane & 3u, t, w, word) && valid) quad[w] = word;
    }
}

// BITS = 4: the card's nibble format; 3, 5, 6: 2^BITS - 1 levels, each row's codes one
// little-endian bit stream (element k at bits k BITS .. k BITS + BITS - 1 of the row's words).
// STAB (G = 1, BITS = 4): the thresholds of a row scale exactly with its max's power of two (the
// fp64 product, the rounding up to fp32 and to bf16 and the tie test are all exact under such a
// scaling while the thresholds stay normal), so B_k and the code table depend only on the 7
// mantissa bits of the max. Each CTA builds the 128 tables once (from a max of each mantissa with
// exponent 0) into shared memory in front of the ring, and a row whose smallest threshold is a
// normal bf16 reads its mantissa's table instead of building its own.
template <int G, int BITS = 4, bool STAB = false>
__global__ void __launch_bounds__(QS_THREADS, 1) quantize_stream_kernel(const __grid_constant__ QsParams p) {
    using C = QsCfg<G, STAB>;
    static_assert(!STAB || (G == 1 && BITS == 4), "shared mantissa tables: one-warp rows at 4 bits");
    constexpr int L = (1 << BITS) - 1;
    constexpr int NG = C::NG, GT = 32 * G;
    extern __shared__ __align__(128) uint8_t qs_smem[];
    __shared__ __align__(16) uint32_t qs_tab[NG * C::TAB / 4];
    __shared__ uint32_t qs_red[NG][G];

    uint64_t *full = reinterpret_cast<uint64_t *>(qs_smem + QS_OFF_BAR);
    uint64_t *empty = full + QS_MAX_SLOTS;
    const int ring_off = QS_OFF_RING + (STAB ? p.stab_bytes : 0);
    const uint32_t ring = smem_u32(qs_smem + ring_off);
    uint16_t *stab_dz = reinterpret_cast<uint16_t *>(qs_smem + QS_OFF_RING);           // STAB: dz per mantissa
    uint32_t *stab_w = reinterpret_cast<uint32_t *>(qs_smem + QS_OFF_RING + 256);     // STAB: the tables
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.nslots;
    const int64_t grid = gridDim.x, cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);     // the producer's expect_tx arrival (+ the copy's bytes)
            mbar_init(&empty[s], G);    // one arrival per warp of the consuming group
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == QS_CONS_WARPS) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            int j = 0, s = 0;
            uint32_t ph = 0;            // parity of slot s's current use
            int64_t issued = 0;
            for (int64_t u = cta; u < p.rows; u += grid) {
                j = qs_job_of(p, u, j);
                const QsJob &J = p.job[j];
                // the slot's previous row (issued S rows ago) has been copied out
                if (issued >= S && !mbar_wait(&empty[s], ph ^ 1u)) break;
                const uint32_t rb = (uint32_t)J.K * 2u;
                mbar_arrive_expect_tx(&full[s], rb);
                bulk_load(qs_smem + ring_off + (size_t)s * p.slot_bytes, J.w + (u - J.row_begin) * J.ldw, rb,
                          &full[s]);
                ++issued;
                if (++s == S) { s = 0; ph ^= 1u; }
            }
            // the copies of the last S rows issued have landed before the CTA can exit (on a normal
            // run the consumers waited for them; after a time-out they may still be in flight)
            for (int64_t k = 0; k < issued && k < S; ++k) {
                if (--s < 0) { s = S - 1; ph ^= 1u; }
                (void)mbar_wait(&full[s], ph);
            }
        }
    } else {
        // ------------------------------------------------------------------ consumers
        const int g = warp / G, wg = warp % G;
        const int tg = wg * 32 + lane;             // thread index in the group
        const int bar_id = 1 + g;
        const uint8_t *tb = reinterpret_cast<const uint8_t *>(qs_tab);
        const uint32_t base = (uint32_t)g * C::TAB;
        if constexpr (STAB) {
            // the 128 mantissa tables: warp w builds those of mantissas w, w + 16, ...; a table that
            // would not fit its stride is marked unusable (its rows build their own)
            for (int m = warp; m < 128; m += QS_CONS_WARPS) {
                const uint32_t mxr = (127u << 7) | (uint32_t)m;
                const uint32_t myT = lane < 15 ? level_threshold(__uint_as_float(mxr << 16), lane + 1, p.qp) : 0x7F80u;
                const uint32_t dz = mxr - __shfl_sync(0xFFFFFFFFu, myT, 0) + 1u;
                const bool fits = 4u * ((dz + 4u) >> 2) <= (uint32_t)p.stab_stride;
                if (lane == 0) stab_dz[m] = fits ? (uint16_t)dz : (uint16_t)0xFFFFu;
                if (fits) {
                    const int Bk = (lane < 15 && myT <= mxr) ? (int)mxr - (int)myT + 1 : 0;
                    qs_build_table<32, 15>(stab_w + (uint32_t)m * (uint32_t)p.stab_stride / 4u, Bk, 0, dz, lane, 0x11u);
                }
            }
            asm volatile("bar.sync 1, %0;" ::"r"(QS_CONS_WARPS * 32) : "memory");   // the consumers only
        }
        int j = 0, s = g;
        uint32_t ph = 0;
        while (s >= S) { s -= S; ph ^= 1u; }
        for (int64_t u = cta + (int64_t)g * grid; u < p.rows; u += (int64_t)NG * grid) {
            j = qs_job_of(p, u, j);
            const QsJob &J = p.job[j];
            const int64_t n = u - J.row_begin;
            const int nvec = J.K / 8;
            // ---- the row's vectors tg, tg + GT, ... from the slot into registers; slot handed back
            const bool got = mbar_wait(&full[s], ph);
            uint4 a[QS_VMAX];
            const uint32_t rp = ring + (uint32_t)s * (uint32_t)p.slot_bytes;
#pragma unroll
            for (int k = 0; k < QS_VMAX; ++k) {
                const int v = k * GT + tg;
                a[k] = (got && v < nvec) ? qs_lds_v4(rp + 16u * (uint32_t)v) : make_uint4(0, 0, 0, 0);
            }
            // a warp whose copy did not land within the wait limit keeps the slot (the producer's
            // bounded wait for it then ends the stream) and the group stops below
            if (__all_sync(0xFFFFFFFFu, got) && lane == 0) mbar_arrive(&empty[s]);
            s += NG;
            while (s >= S) { s -= S; ph ^= 1u; }
            // ---- signs (w < 0: -0.0 and NaN store 0) and max |w| from the registers
            uint32_t *srow = J.signs + n * (int64_t)(nvec / 4);
            uint32_t mx2 = 0;
#pragma unroll
            for (int k = 0; k < QS_VMAX; ++k) {
                const int v = k * GT + tg;
                if (k * GT < nvec) {   // the batch is in the row for some lane: shuffles need them all
                    const uint4 x = a[k];
                    const uint32_t sb = opqbits::sign_byte(opqbits::bf16x2_neg_mask(x.x), opqbits::bf16x2_neg_mask(x.y),
                                                           opqbits::bf16x2_neg_mask(x.z), opqbits::bf16x2_neg_mask(x.w));
                    // lanes 4m .. 4m + 3 hold four consecutive vectors: one sign word (nvec % 4 == 0)
                    uint32_t sw = sb << (8 * (lane & 3));
                    sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 1);
                    sw |= __shfl_xor_sync(0xFFFFFFFFu, sw, 2);
                    if (v < nvec && (lane & 3) == 0) srow[v >> 2] = sw;
                    a[k] = make_uint4(x.x & 0x7FFF7FFFu, x.y & 0x7FFF7FFFu, x.z & 0x7FFF7FFFu, x.w & 0x7FFF7FFFu);
                    // packed bf16 max: the magnitudes' largest bit pattern per half (NaN propagates)
                    mx2 = opqbits::bf16x2_max(mx2, opqbits::bf16x2_max(opqbits::bf16x2_max(a[k].x, a[k].y),
                                                                       opqbits::bf16x2_max(a[k].z, a[k].w)));
                }
            }
            // halves of the packed max (a NaN half is 0x7FFF, above +inf: such rows take the search)
            uint32_t mx = max(mx2 & 0x7FFFu, (mx2 >> 16) & 0x7FFFu);
            mx = __reduce_max_sync(0xFFFFFFFFu, mx);
            if (G > 1) {
                if (lane == 0) qs_red[g][wg] = mx;
                // every thread of the group got its copy (or none goes on)
                if (!group_sync_and(bar_id, GT, got)) break;
#pragma unroll
                for (int i = 0; i < G; ++i) mx = max(mx, qs_red[g][i]);
            } else if (!__all_sync(0xFFFFFFFFu, got)) {
                break;
            }
            const float mxf = __uint_as_float(mx << 16);
            uint32_t *crow = J.codes + n * ((int64_t)nvec * BITS / 4);
            if constexpr (STAB) {
                // the row's mantissa table, if its smallest threshold mx - dz + 1 is a normal bf16
                const uint32_t dzm = (mx != 0u && mx <= 0x7F7Fu) ? (uint32_t)stab_dz[mx & 0x7Fu] : 0xFFFFu;
                if (dzm != 0xFFFFu && mx + 1u >= dzm + 0x80u) {
                    if (tg == 0) J.scales[n] = mxf;
                    const uint8_t *tbm = reinterpret_cast<const uint8_t *>(stab_w) + (mx & 0x7Fu) * (uint32_t)p.stab_stride;
                    const uint32_t mm = mx * 0x00010001u, lo2 = (mx - dzm) * 0x00010001u;
#pragma unroll
                    for (int k = 0; k < QS_VMAX; ++k) {
                        const int v = k * GT + tg;
                        if (v < nvec) {
                            const uint4 x = a[k];
                            crow[v] = opqbits::codes_word(opqbits::table_byte_clamped(tbm, x.x, lo2, mm),
                                                          opqbits::table_byte_clamped(tbm, x.y, lo2, mm),
                                                          opqbits::table_byte_clamped(tbm, x.z, lo2, mm),
                                                          opqbits::table_byte_clamped(tbm, x.w, lo2, mm));
                        }
                    }
                    __syncwarp();
                    continue;
                }
            }
            // the thresholds of levels lane + 1 and (6 bits) lane + 33; +inf: a level no finite
            // weight reaches (every level of a zero row)
            uint32_t myT = 0x7F80u, myT2 = 0x7F80u;
            if (mx != 0u) {
                if (BITS == 4) {
                    if (lane < 15) myT = level_threshold(mxf, lane + 1, p.qp);
                } else {
                    if (lane < L) myT = level_threshold_levels(mxf, lane + 1, L, p.tl[lane + 1], p.qp.alpha_is_one);
                    if (L > 32 && lane + 32 < L)
                        myT2 = level_threshold_levels(mxf, lane + 33, L, p.tl[lane + 33], p.qp.alpha_is_one);
                }
            }
            const uint32_t T1 = __shfl_sync(0xFFFFFFFFu, myT, 0);
            const uint32_t dz = T1 <= mx ? mx - T1 + 1u : 0u;
            if (tg == 0) J.scales[n] = mxf;
            // group-uniform: mx is the group's max
            if (mx <= 0x7F80u && dz < (uint32_t)C::TAB) {
                const int Bk = (lane < L && myT <= mx) ? (int)mx - (int)myT + 1 : 0;
                const int Bk2 = (L > 32 && lane + 32 < L && myT2 <= mx) ? (int)mx - (int)myT2 + 1 : 0;
                // 4 bits: q in both nibbles (a pair's code byte is one merge); else q itself
                qs_build_table<GT, L>(qs_tab + base / 4, Bk, Bk2, dz, tg, BITS == 4 ? 0x11u : 1u);
                if (G > 1) group_sync(bar_id, GT); else __syncwarp();
                const uint32_t mmb = (mx + base) * 0x00010001u, lo2 = (mx - dz) * 0x00010001u;
#pragma unroll
                for (int k = 0; k < QS_VMAX; ++k) {
                    const int v = k * GT + tg;
                    if constexpr (BITS == 4) {
                        if (v < nvec) {
                            const uint4 x = a[k];
                            crow[v] = opqbits::codes_word(opqbits::table_byte_clamped(tb, x.x, lo2, mmb),
                                                          opqbits::table_byte_clamped(tb, x.y, lo2, mmb),
                                                          opqbits::table_byte_clamped(tb, x.z, lo2, mmb),
                                                          opqbits::table_byte_clamped(tb, x.w, lo2, mmb));
                        }
                    } else if (k * GT < nvec) {   // the batch is in the row for some lane: shuffles need them all
                        const uint4 x = a[k];
                        uint32_t q[8];
                        opqbits::table_pair_bytes(tb, x.x, lo2, mmb, q[0], q[1]);
                        opqbits::table_pair_bytes(tb, x.y, lo2, mmb, q[2], q[3]);
                        opqbits::table_pair_bytes(tb, x.z, lo2, mmb, q[4], q[5]);
                        opqbits::table_pair_bytes(tb, x.w, lo2, mmb, q[6], q[7]);
                        qs_store_codes<BITS>(crow, v, q, lane, v < nvec);
                    }
                }
            } else if (BITS != 4) {
                // rows whose table would not fit (small alpha) or whose max is not finite: a binary
                // search per weight over the L thresholds, held in the group's table area
                uint16_t *thr = reinterpret_cast<uint16_t *>(qs_tab) + base / 2;   // thr[k], k = 1..L
                if (wg == 0) {
                    if (lane < L) thr[lane + 1] = (uint16_t)myT;
                    if (L > 32 && lane + 32 < L) thr[lane + 33] = (uint16_t)myT2;
                }
                if (G > 1) group_sync(bar_id, GT); else __syncwarp();
#pragma unroll
                for (int k = 0; k < QS_VMAX; ++k) {   // unrolled: the row stays in registers
                    const int v = k * GT + tg;
                    if (k * GT < nvec) {
                        const uint32_t m[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
                        uint32_t q[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint32_t mag = (m[e >> 1] >> (16 * (e & 1))) & 0x7FFFu;
                            uint32_t qq = 0;
#pragma unroll
                            for (int step = (L + 1) / 2; step > 0; step >>= 1)
                                if (mag >= thr[qq + step]) qq += step;
                            q[e] = qq;
                        }
                        qs_store_codes<BITS>(crow, v, q, lane, v < nvec);
                    }
                }
            } else {
                // rows whose table would not fit (small alpha) or whose max is not finite: the
                // branch-free search over the 15 thresholds
                uint32_t P[16];
                P[0] = 0;
#pragma unroll
                for (int k = 1; k < 16; ++k) P[k] = __shfl_sync(0xFFFFFFFFu, myT, k - 1) * 0x00010001u;
#pragma unroll
                for (int k = 0; k < QS_VMAX; ++k) {
                    const int v = k * GT + tg;
                    if (v < nvec) {
                        const uint4 x = a[k];
                        crow[v] = opqbits::pack_codes(opqbits::quant_pair_f(x.x, P), opqbits::quant_pair_f(x.y, P),
                                                      opqbits::quant_pair_f(x.z, P), opqbits::quant_pair_f(x.w, P));
                    }
                }
            }
            // every lookup of this row is done before the table (and the group's reduction
            // words) are rewritten for the next row
            if (G > 1) group_sync(bar_id, GT); else __syncwarp();
        }
    }
    __syncwarp();
    __syncthreads();
}

}  // namespace opqk
