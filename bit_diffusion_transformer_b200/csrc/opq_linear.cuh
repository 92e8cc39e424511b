// opq_linear.cuh — y = x W'^T with W' decoded on the fly from the OPQ planes.
//
// "OPQ INT4 Z-Image" model card: the OPQLinear forward decodes
// w = sign * (q/15)^(1/alpha) * max ("inference decoding") and multiplies.
// Here the row scale max is deferred to the epilogue, so the tensor cores see
// sign * bf16((q/15)^(1/alpha)) and the fp32 sum is multiplied by scale[n] once.
//
// Two kernels, both tcgen05 (5th-generation tensor cores, accumulators in TMEM):
//
//  tile kernel (large M): D[128 x 256] = x_tile[128 x K] * W'_tile[256 x K]^T.
//    x tiles arrive by TMA (128-byte swizzle); W' tiles are decoded by 8 warps
//    (one weight row per thread) from codes/signs that each thread streams into
//    its own shared-memory ring with cp.async, and are stored in the same
//    swizzled K-major layout the MMA reads. One thread issues the MMAs, four
//    warps drain the double-buffered accumulator (2 x 256 TMEM columns) while
//    the next tile accumulates. Persistent: one CTA per SM walks the tiles.
//
//  weight-streaming kernel (small M): the roles swap so that the weights fill
//    the MMA's 128-row side: D^T[128 x BX] = W'_tile[128 x K] * x[BX x K]^T,
//    BX = M rounded up to 16. Each CTA decodes one 128-row weight tile over a
//    slice of K (split-K); fp32 partial sums go to the workspace and a second
//    kernel adds them in a fixed order, scales and rounds (or, unsplit, the
//    epilogue writes y directly).
#pragma once
#include <cuda_bf16.h>

#include "opq_bits.h"
#include "opq_device.cuh"

namespace opqk {

using namespace opqdev;

// ------------------------------------------------------------ cp.async helpers --
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_4(void *smem_dst, const void *gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]),
                 "r"(v[3])
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

struct LinearArgs {
    const uint32_t *codes;
    const uint32_t *signs;
    const float *scales;
    uint16_t *y;
    float *ws;   // split-K partials [splits, M, N] (weight-streaming kernel only)
    int M, N, K;
    int splits;  // weight-streaming kernel
    int bx;      // weight-streaming kernel: MMA N (x rows per CTA, multiple of 16)
    opqbits::DecodeTable tab;
};

// Decode one 8-weight chunk and store it as 16 swizzled bytes.
__device__ __forceinline__ void decode_store(uint32_t code, uint32_t sb, const opqbits::DecodeTable &tab,
                                             uint32_t dst) {
    uint32_t o[4];
    opqbits::decode8(code, sb, tab, o);
    st_shared_v4(dst, o);
}

// ============================================================================
// Tile kernel (path 0)
// ============================================================================
namespace tile {
constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 3;
constexpr int RD = 4;                       // per-thread cp.async ring depth
constexpr int A_BYTES = BM * BK * 2;        // 16 KiB
constexpr int B_BYTES = BN * BK * 2;        // 32 KiB
constexpr int RAW_CODE_BYTES = RD * BN * 32;
constexpr int RAW_SIGN_BYTES = RD * BN * 8;
constexpr int NUM_DECODE_WARPS = BN / 32;   // one weight row per thread
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_DEC0 = 2;
constexpr int WARP_EPI0 = WARP_DEC0 + NUM_DECODE_WARPS;  // 10..13
constexpr int THREADS = (WARP_EPI0 + 4) * 32;             // 448
constexpr int ACC_COLS = BN;                // fp32 columns per accumulator
constexpr int TMEM_COLS = 2 * ACC_COLS;     // double-buffered
// shared memory map (offsets from the 1 KiB-aligned base)
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_RAWC = OFF_B + STAGES * B_BYTES;
constexpr int OFF_RAWS = OFF_RAWC + RAW_CODE_BYTES;
constexpr int OFF_BAR = OFF_RAWS + RAW_SIGN_BYTES;
constexpr int NUM_BARS = 3 * STAGES + 4 + 1;              // a_full, b_full, empty, acc_full x2, acc_empty x2, drain
constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;          // + alignment slack
static_assert(SMEM_BYTES <= 232448, "tile kernel shared memory");
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
}  // namespace tile

__global__ void __launch_bounds__(tile::THREADS, 1)
    linear_tile_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ LinearArgs args) {
    using namespace tile;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_base + pad;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *a_full = bars;
    uint64_t *b_full = bars + STAGES;
    uint64_t *empty = bars + 2 * STAGES;
    uint64_t *acc_full = bars + 3 * STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_TMEM);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = args.M, N = args.N, K = args.K;
    const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int nkb = (K + BK - 1) / BK;
    const int my_tiles = (blockIdx.x < num_tiles) ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&b_full[s], NUM_DECODE_WARPS);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], 4);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == WARP_TMA && lane == 0) tma_prefetch_desc(&tmap_x);
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == WARP_TMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int armed = 0;  // loads issued whose completion has not been observed
            for (int t = 0; t < my_tiles && ok; ++t) {
                const int tile_id = blockIdx.x + t * gridDim.x;
                const int m_blk = tile_id % num_m;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
                    mbar_arrive_expect_tx(&a_full[stage], A_BYTES);
                    tma_load_2d(smem + OFF_A + stage * A_BYTES, &tmap_x, kb * BK, m_blk * BM, &a_full[stage]);
                    armed = armed < STAGES ? armed + 1 : STAGES;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // let the copies already in flight land before the CTA can exit
                for (int i = 0; i < armed; ++i) {
                    if (--stage < 0) { stage = STAGES - 1; phase ^= 1; }
                    (void)mbar_wait(&a_full[stage], phase);
                }
            }
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = 0; t < my_tiles && ok; ++t) {
                const int as = t & 1;
                const uint32_t aph = (t >> 1) & 1;
                if (!mbar_wait(&acc_empty[as], aph ^ 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + as * ACC_COLS;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&a_full[stage], phase) || !mbar_wait(&b_full[stage], phase)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t adesc = smem_desc_sw128(sbase + OFF_A + stage * A_BYTES);
                    const uint64_t bdesc = smem_desc_sw128(sbase + OFF_B + stage * B_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, IDESC, (kb | k) != 0 ? 1u : 0u);
                    umma_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (ok) umma_commit(&acc_full[as]);
            }
            // every MMA issued by this thread has completed once `drain` flips
            umma_commit(drain);
            (void)mbar_wait(drain, 0);
        }
    } else if (warp < WARP_EPI0) {
        // ------------------------------------------------------------ decoders
        const int d = threadIdx.x - WARP_DEC0 * 32;   // weight row inside the tile
        uint8_t *rawc = smem + OFF_RAWC;
        uint8_t *raws = smem + OFF_RAWS;
        const int total = my_tiles * nkb;
        const int cw = K / 8, swd = K / 32;
        auto issue = [&](int it) {
            if (it < total) {
                const int t = it / nkb, kb = it - t * nkb;
                const int tile_id = blockIdx.x + t * gridDim.x;
                const int n = (tile_id / num_m) * BN + d;
                const bool rv = n < N;
                const uint32_t *crow = args.codes + (size_t)(rv ? n : 0) * cw;
                const uint32_t *srow = args.signs + (size_t)(rv ? n : 0) * swd;
                const int slot = it % RD;
                const bool full = (kb + 1) * BK <= K;   // else only the first 32 columns exist
                uint8_t *dc = rawc + (slot * BN + d) * 32;
                uint8_t *ds = raws + (slot * BN + d) * 8;
                cp_async_16(dc, crow + kb * 8, rv ? 16u : 0u);
                cp_async_16(dc + 16, crow + kb * 8 + (full ? 4 : 0), (rv && full) ? 16u : 0u);
                cp_async_4(ds, srow + kb * 2, rv ? 4u : 0u);
                cp_async_4(ds + 4, srow + kb * 2 + (full ? 1 : 0), (rv && full) ? 4u : 0u);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < RD - 1; ++i) issue(i);
        int stage = 0;
        uint32_t phase = 0;
        for (int it = 0; it < total; ++it) {
            issue(it + RD - 1);
            cp_async_wait<RD - 1>();
            const int slot = it % RD;
            const uint4 c0 = *reinterpret_cast<const uint4 *>(rawc + (slot * BN + d) * 32);
            const uint4 c1 = *reinterpret_cast<const uint4 *>(rawc + (slot * BN + d) * 32 + 16);
            const uint2 sg = *reinterpret_cast<const uint2 *>(raws + (slot * BN + d) * 8);
            if (!mbar_wait(&empty[stage], phase ^ 1)) break;
            const uint32_t dst = sbase + OFF_B + stage * B_BYTES;
            decode_store(c0.x, sg.x & 0xFFu, args.tab, dst + sw128_offset(d, 0));
            decode_store(c0.y, (sg.x >> 8) & 0xFFu, args.tab, dst + sw128_offset(d, 1));
            decode_store(c0.z, (sg.x >> 16) & 0xFFu, args.tab, dst + sw128_offset(d, 2));
            decode_store(c0.w, sg.x >> 24, args.tab, dst + sw128_offset(d, 3));
            decode_store(c1.x, sg.y & 0xFFu, args.tab, dst + sw128_offset(d, 4));
            decode_store(c1.y, (sg.y >> 8) & 0xFFu, args.tab, dst + sw128_offset(d, 5));
            decode_store(c1.z, (sg.y >> 16) & 0xFFu, args.tab, dst + sw128_offset(d, 6));
            decode_store(c1.w, sg.y >> 24, args.tab, dst + sw128_offset(d, 7));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_full[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        cp_async_wait_all();
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const bool vec_ok = (N % 8) == 0;
        for (int t = 0; t < my_tiles; ++t) {
            const int tile_id = blockIdx.x + t * gridDim.x;
            const int m_blk = tile_id % num_m, n_blk = tile_id / num_m;
            const int as = t & 1;
            const uint32_t aph = (t >> 1) & 1;
            if (!mbar_wait(&acc_full[as], aph)) break;
            tc_fence_after();
            const int m = m_blk * BM + q * 32 + lane;
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + as * ACC_COLS;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + cc * 32, r);
                const int n0 = n_blk * BN + cc * 32;
                // lane i holds scale[n0 + i]; shuffles broadcast it to the row owners
                const float scl = (n0 + lane < N) ? __ldg(args.scales + n0 + lane) : 0.0f;
                tmem_ld_wait();
                uint32_t p[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    p[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * __shfl_sync(0xFFFFFFFFu, scl, 2 * i),
                                       __uint_as_float(r[2 * i + 1]) * __shfl_sync(0xFFFFFFFFu, scl, 2 * i + 1));
                if (m < M && n0 < N) {
                    uint16_t *yrow = args.y + (size_t)m * N;
                    if (vec_ok && n0 + 32 <= N) {
                        uint4 *dst = reinterpret_cast<uint4 *>(yrow + n0);
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (n0 + i < N) yrow[n0 + i] = (uint16_t)((p[i / 2] >> (16 * (i & 1))) & 0xFFFFu);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[as]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ============================================================================
// Weight-streaming split-K kernel (path 1)
// ============================================================================
namespace stream {
constexpr int BW = 128, BK = 64;            // weight rows per CTA (MMA M), K per stage
constexpr int STAGES = 4;
constexpr int RD = 4;
constexpr int A_BYTES = BW * BK * 2;        // 16 KiB decoded weights per stage
constexpr int DEC_THREADS = 256;            // two threads per weight row (32 columns each)
constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_DEC0 = 2;
constexpr int THREADS = (WARP_DEC0 + DEC_THREADS / 32) * 32;  // 320
constexpr int RAW_CODE_BYTES = RD * DEC_THREADS * 16;
constexpr int RAW_SIGN_BYTES = RD * DEC_THREADS * 4;
__host__ __device__ constexpr int b_bytes(int bx) { return bx * BK * 2; }
__host__ __device__ constexpr int off_b() { return STAGES * A_BYTES; }
__host__ __device__ constexpr int off_rawc(int bx) { return off_b() + STAGES * b_bytes(bx); }
__host__ __device__ constexpr int off_raws(int bx) { return off_rawc(bx) + RAW_CODE_BYTES; }
__host__ __device__ constexpr int off_bar(int bx) { return off_raws(bx) + RAW_SIGN_BYTES; }
constexpr int NUM_BARS = 3 * STAGES + 1 + 1;  // a_full(x), b_full(decoded), empty, acc_full, drain
__host__ __device__ constexpr int off_tmem(int bx) { return off_bar(bx) + NUM_BARS * 8; }
__host__ __device__ constexpr int smem_bytes(int bx) { return off_tmem(bx) + 16 + 1024; }
__host__ __device__ constexpr uint32_t tmem_cols(int bx) {
    return bx <= 32 ? 32u : bx <= 64 ? 64u : bx <= 128 ? 128u : 256u;
}
}  // namespace stream

__global__ void __launch_bounds__(stream::THREADS)
    linear_stream_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ LinearArgs args) {
    using namespace stream;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_base + pad;
    const int bx = args.bx;
    const int BX_BYTES = b_bytes(bx);

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + off_bar(bx));
    uint64_t *x_full = bars;
    uint64_t *w_full = bars + STAGES;
    uint64_t *empty = bars + 2 * STAGES;
    uint64_t *acc_full = bars + 3 * STAGES;
    uint64_t *drain = acc_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + off_tmem(bx));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int M = args.M, N = args.N, K = args.K;
    const int nkb_total = (K + BK - 1) / BK;
    const int split = blockIdx.y;
    const int kb_per = (nkb_total + args.splits - 1) / args.splits;
    const int kb_begin = split * kb_per;
    const int kb_end = min(nkb_total, kb_begin + kb_per);
    const int nkb = max(0, kb_end - kb_begin);
    const int n_base = blockIdx.x * BW;
    const uint32_t ncols = tmem_cols(bx);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&x_full[s], 1);
            mbar_init(&w_full[s], DEC_THREADS / 32);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == WARP_TMA && lane == 0) tma_prefetch_desc(&tmap_x);
    if (warp == WARP_MMA) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == WARP_TMA) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int armed = 0;
            bool ok = true;
            for (int i = 0; i < nkb; ++i) {
                if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
                mbar_arrive_expect_tx(&x_full[stage], BX_BYTES);
                tma_load_2d(smem + off_b() + stage * BX_BYTES, &tmap_x, (kb_begin + i) * BK, 0, &x_full[stage]);
                armed = armed < STAGES ? armed + 1 : STAGES;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) {
                for (int i = 0; i < armed; ++i) {
                    if (--stage < 0) { stage = STAGES - 1; phase ^= 1; }
                    (void)mbar_wait(&x_full[stage], phase);
                }
            }
        }
    } else if (warp == WARP_MMA) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            const uint32_t idesc = idesc_bf16_f32(BW, bx);
            for (int i = 0; i < nkb; ++i) {
                if (!mbar_wait(&w_full[stage], phase) || !mbar_wait(&x_full[stage], phase)) { ok = false; break; }
                tc_fence_after();
                const uint64_t adesc = smem_desc_sw128(sbase + stage * A_BYTES);
                const uint64_t bdesc = smem_desc_sw128(sbase + off_b() + stage * BX_BYTES);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    umma_bf16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (i | k) != 0 ? 1u : 0u);
                umma_commit(&empty[stage]);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (ok) umma_commit(acc_full);
            umma_commit(drain);
            (void)mbar_wait(drain, 0);
        }
    } else {
        // ---------------------------------------------------- decoders, then epilogue
        const int d = threadIdx.x - WARP_DEC0 * 32;
        const int r = d >> 1, h = d & 1;          // weight row, column half (32 of 64)
        const int n = n_base + r;
        const bool rv = n < N;
        const int cw = K / 8, swd = K / 32;
        const uint32_t *crow = args.codes + (size_t)(rv ? n : 0) * cw;
        const uint32_t *srow = args.signs + (size_t)(rv ? n : 0) * swd;
        uint8_t *rawc = smem + off_rawc(bx);
        uint8_t *raws = smem + off_raws(bx);
        auto issue = [&](int i) {
            if (i < nkb) {
                const int kb = kb_begin + i;
                const bool present = rv && (kb * BK + h * 32) < K;
                const int slot = i % RD;
                cp_async_16(rawc + (slot * DEC_THREADS + d) * 16, crow + (present ? kb * 8 + h * 4 : 0),
                            present ? 16u : 0u);
                cp_async_4(raws + (slot * DEC_THREADS + d) * 4, srow + (present ? kb * 2 + h : 0),
                           present ? 4u : 0u);
            }
            cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < RD - 1; ++i) issue(i);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int i = 0; i < nkb; ++i) {
            issue(i + RD - 1);
            cp_async_wait<RD - 1>();
            const int slot = i % RD;
            const uint4 c = *reinterpret_cast<const uint4 *>(rawc + (slot * DEC_THREADS + d) * 16);
            const uint32_t sg = *reinterpret_cast<const uint32_t *>(raws + (slot * DEC_THREADS + d) * 4);
            if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
            const uint32_t dst = sbase + stage * A_BYTES;
            decode_store(c.x, sg & 0xFFu, args.tab, dst + sw128_offset(r, 4 * h + 0));
            decode_store(c.y, (sg >> 8) & 0xFFu, args.tab, dst + sw128_offset(r, 4 * h + 1));
            decode_store(c.z, (sg >> 16) & 0xFFu, args.tab, dst + sw128_offset(r, 4 * h + 2));
            decode_store(c.w, sg >> 24, args.tab, dst + sw128_offset(r, 4 * h + 3));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&w_full[stage]);
            if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        cp_async_wait_all();

        // epilogue: warps 2..5 hold TMEM lane quarters 2, 3, 0, 1
        if (ok && warp < WARP_DEC0 + 4 && nkb > 0) {
            const int q = warp & 3;
            const int row = q * 32 + lane;
            const int nn = n_base + row;
            if (mbar_wait(acc_full, 0)) {
                tc_fence_after();
                const float scale = (nn < N) ? __ldg(args.scales + nn) : 0.0f;
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
                for (int c0 = 0; c0 < bx; c0 += 8) {
                    uint32_t v[8];
                    tmem_ld_32x32b_x8(taddr + c0, v);
                    tmem_ld_wait();
                    if (nn < N) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int m = c0 + j;
                            if (m < M) {
                                const float acc = __uint_as_float(v[j]);
                                if (args.splits == 1) {
                                    const __nv_bfloat16 o = __float2bfloat16_rn(acc * scale);
                                    args.y[(size_t)m * N + nn] = *reinterpret_cast<const uint16_t *>(&o);
                                } else {
                                    args.ws[((size_t)split * M + m) * N + nn] = acc;
                                }
                            }
                        }
                    }
                }
            }
        } else if (nkb == 0 && warp < WARP_DEC0 + 4 && args.splits > 1) {
            // an empty K slice still owns its partial-sum rows: write zeros
            const int q = warp & 3;
            const int nn = n_base + q * 32 + lane;
            if (nn < N)
                for (int m = 0; m < M; ++m) args.ws[((size_t)split * M + m) * N + nn] = 0.0f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, ncols);
    }
}

// y[m, n] = bf16(scale[n] * sum_{s = 0..splits-1} ws[s, m, n]), summed in order s = 0, 1, ...
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *__restrict__ ws,
                                                            const float *__restrict__ scales, int M, int N,
                                                            int splits, uint16_t *__restrict__ y) {
    const size_t total = (size_t)M * N;
    const size_t plane = total;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        float acc = ws[i];
        for (int s = 1; s < splits; ++s) acc += ws[(size_t)s * plane + i];
        const int n = (int)(i % (size_t)N);
        const __nv_bfloat16 o = __float2bfloat16_rn(acc * __ldg(scales + n));
        y[i] = *reinterpret_cast<const uint16_t *>(&o);
    }
}

}  // namespace opqk
