// opq_linear_wide.cuh — y = x W'^T for wide activation tiles (more than 128 rows of x).
//
// "OPQ INT4 Z-Image" model card: the OPQLinear forward decodes
// w = sign * (q/15)^(1/alpha) * max ("inference decoding") and multiplies. As in
// opq_linear.cuh, the tensor cores see sign * bf16((q/15)^(1/alpha)) and each fp32 sum is
// multiplied by scale[n] once in the epilogue.
//
// Tiles of 128 weight rows x 256 activation rows, one persistent CTA per SM, tensor-bound:
//   warp 0       raw producer: codes (TMA, 64-byte swizzle) and signs of 128 rows x 128 K
//                per stage, one 128-K block per copy
//   warp 1       TMEM allocation and the MMA issue; A from TMEM, B = x from shared memory
//   warp 2       x producer: 256 rows x 64 K per copy, two per block (128-byte swizzle)
//   warps 4..11  two decoder groups (4 warps = the 128 TMEM lanes) through the pair table,
//                A written to TMEM with tcgen05.st
//   warps 12..15 epilogue: the tile's sums into registers as bf16 pairs, the accumulator
//                released, then y stored while the next tile's MMAs run (the producers'
//                warpgroup hands registers to the epilogue's with setmaxnreg)
// Whole tiles are strided over the CTAs; tiles past the last whole wave (at most half as
// many as CTAs) run as two 128-row halves on two CTAs. The narrow-tile kernel
// (opq_linear.cuh) fetches several blocks per copy and splits K over CTAs instead; at this
// width its wait structure measured ~6% slower, so the two regimes keep separate kernels.
#pragma once
#include <cuda_fp16.h>

#include "opq_linear.cuh"

namespace opqk_wide {

using namespace opqk;

struct LinearArgs {
    const uint32_t *signs;  // sign plane [N, K/32]
    const float *scales;
    uint16_t *y;
    float *ws;              // tail_split 3: fp32 partial sums [tail tile][lane quarter][BX m][32 n]
    uint32_t *counters;     // tail_split 3: per (tail tile, TMEM lane quarter) an arrival count and a
                            // published flag, 8 words per tail tile; zero between calls
    int signs_tma;          // 1: sign plane rows are 16-byte aligned (K % 128 == 0), load it by TMA
    int M, N, K;
    int m_tiles, n_tiles;
    int kblocks;            // 128-K blocks per tile
    int mode;               // 0: whole tiles strided over CTAs (the only schedule this kernel runs)
    int tail_split;         // mode 0, tiles past the last whole wave: 2 = each runs as two half-width
                            // (BX/2 activation rows) runs on two CTAs; 3 = each runs as two
                            // half-K runs on two CTAs whose partial sums meet in `ws`; 1 = whole
    uint16_t lut[16];       // bf16 (q/15)^(1/alpha)
    uint16_t lutb[64];      // other bit widths: bf16 (q/L)^(1/alpha), q = 0..L, L = 2^BITS - 1
    // group-wise format (GS > 0)
    const uint16_t *gmax;   // float16 [N, K / GS]
    int ngk;                // groups per row (K / GS)
    float lutf[16];         // (q/15)^(1/alpha) in fp32
    // fused epilogue
    const uint16_t *bias;   // bf16 [N] added to every output row, or null
    int act;                // EPI_NONE, EPI_SILU, EPI_GELU_TANH
};


// The sequence of runs of one CTA; every role walks the same sequence. A run is one
// weight tile, a range of its 128-K blocks and a range of its activation rows. Whole tiles
// are handed out strided over the CTAs; the tiles past the last whole wave are split over
// two CTAs each (tail_split 2: activation rows, 3: K) or run whole (1).
struct RunIter {
    int tiles, kblocks, grid, cta;
    int t_next;
    int full_end;       // tiles in whole waves
    int split;          // tail_split
    bool tail_done;
    int run_idx;
    __device__ __forceinline__ void init(const LinearArgs &a, int tiles_, int grid_, int cta_) {
        tiles = tiles_;
        kblocks = a.kblocks;
        grid = grid_;
        cta = cta_;
        run_idx = 0;
        t_next = cta_;
        split = a.tail_split;
        full_end = split >= 2 ? (tiles_ / grid_) * grid_ : tiles_;
        tail_done = false;
    }
    // next run: tile, block range [r0, r1), run index j, activation rows [xoff, xoff + xrows)
    // of the tile's bx; false at the end
    __device__ __forceinline__ bool next(int &tile, int &r0, int &r1, int &j, int &xoff, int &xrows, int bx) {
        xoff = 0;
        xrows = bx;
        r0 = 0;
        r1 = kblocks;
        if (t_next < full_end) {
            tile = t_next;
            t_next += grid;
        } else if (split >= 2) {
            // tail tile t is run by CTAs 2 (t - full_end) and 2 (t - full_end) + 1, one half
            // of its activation rows (split 2) or of its 128-K blocks (split 3) each
            if (tail_done || cta >= 2 * (tiles - full_end)) return false;
            tile = full_end + (cta >> 1);
            tail_done = true;
            if (split == 2) {
                xrows = bx / 2;
                xoff = (cta & 1) * xrows;
            } else {
                // the even CTA takes the smaller share of K, so that it has usually published
                // its partial sums by the time the odd CTA, which then adds them, is done
                const int k0 = kblocks * 7 / 16;
                if (cta & 1) r0 = k0; else r1 = k0;
            }
        } else {
            return false;
        }
        j = run_idx++;
        return true;
    }
    __device__ __forceinline__ bool next(int &tile, int &r0, int &r1, int &j) {
        int xo, xr;
        return next(tile, r0, r1, j, xo, xr, 2);
    }
};

// BITS: bits per magnitude code. 4 is the nibble format, decoded two weights per lookup of the
// pair table; 3, 5 and 6 are per-row bit streams (element k at bits k*BITS .. k*BITS + BITS - 1
// of the row's words), decoded one code at a time.
template <int BX, int BITS = 4>
struct Cfg {
    static constexpr int BW = 128;                     // weight rows per tile (MMA M)
    static constexpr int KR = 128;                     // K per raw (codes/signs) stage
    static constexpr int KA = 64;                      // K per A stage (TMEM) and per x stage (smem)
    // the 5- and 6-bit stages are larger: two of them keep the shared memory within bounds
    static constexpr int RAW_STAGES = BITS >= 5 ? 2 : (BX >= 256 ? 3 : (BX >= 128 ? 4 : 6));
    static constexpr int A_STAGES = 8;                 // 32 TMEM columns each (64 K of bf16 pairs)
    static constexpr int A_BLOCKS = A_STAGES / 2;      // 128-K blocks of A held in TMEM
    static constexpr int A_COLS = A_STAGES * 32;
    // x stages hold a whole 128-K block (two 64-K swizzle atoms' worth of columns)
    static constexpr int X_STAGES = BX >= 256 ? 2 : (BX >= 128 ? 3 : (BX >= 64 ? 4 : (BX >= 32 ? 8 : 10)));
    // One tcgen05.commit per 128-K block frees both its A slot and its x stage: a commit
    // stalls the tensor pipe for a few hundred cycles, so there is one per 8 MMAs, not per 4.
    // Slot b % NDONE of `blk_done` completes when the MMAs of the CTA's block b are done.
    static constexpr int NDONE = X_STAGES > A_BLOCKS ? X_STAGES : A_BLOCKS;
    // independent accumulation chains per tile: consecutive MMAs into one accumulator
    // serialize on its latency, which dominates when N (= BX) is small; K-step k of a
    // stage goes to chain k % NCHAIN and the epilogue adds the chains in a fixed order
    static constexpr int NCHAIN = BX <= 32 ? 4 : (BX <= 64 ? 2 : 1);
    static constexpr int ACC_COLS = NCHAIN * BX;       // one accumulator buffer (all chains)
    static constexpr int NACC = (A_COLS + 2 * ACC_COLS <= 512) ? 2 : 1;   // accumulator buffers
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int RAW_CODE_BYTES = BW * KR * BITS / 8;   // [128 rows][4 BITS words] (4 bits: 64-byte swizzle)
    static constexpr int CODE_WORDS = KR * BITS / 32;           // code words per row and block
    static constexpr int RAW_SIGN_BYTES = BW * KR / 8;    // 2 KiB: [128 rows][4 words]
    static constexpr int RAW_BYTES = RAW_CODE_BYTES + RAW_SIGN_BYTES;
    static constexpr int X_HALF_BYTES = BX * KA * 2;   // one 64-K half: BX rows x 128 bytes, 128-byte swizzle
    static constexpr int X_BYTES = 2 * X_HALF_BYTES;
    static constexpr int OFF_TABLE = 0;
    static constexpr int OFF_RAW = OFF_TABLE + (int)opqbits::kPairTableBytes;
    static constexpr int OFF_X = OFF_RAW + RAW_STAGES * RAW_BYTES;
    static constexpr int OFF_BAR = OFF_X + X_STAGES * X_BYTES;
    static constexpr int NUM_BARS = 2 * RAW_STAGES + A_BLOCKS + NDONE + 2 * NACC + 1 + 4;
    static constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
    // no alignment slack: the third raw stage needs it, and the kernel checks on entry that the
    // dynamic window starts on the 1 KiB boundary the swizzled stages need
    static constexpr int SMEM_BYTES = OFF_TMEM + 16;
    // decoder groups of 4 warps: group g decodes the CTA's 128-K blocks g, g + G, ...;
    // thread r of a group owns weight row r (TMEM lane r) and decodes its whole 128-K block row
    static constexpr int GROUPS = BX >= 256 ? 2 : 3;
    // a group waits on raw stage blk % RAW_STAGES knowing only that its own previous block
    // (blk - GROUPS) was loaded, so the stage's previous phase (block blk - RAW_STAGES) must
    // be at least that old for the parity test to be exact
    static_assert(RAW_STAGES >= GROUPS, "raw ring shorter than the decoder rotation");
    // a decoder waits for block b - A_BLOCKS on blk_done knowing only that its own previous wait
    // (block b - GROUPS - A_BLOCKS) succeeded; the parity test is exact only if that implies block
    // b - A_BLOCKS - NDONE has completed, i.e. NDONE >= GROUPS (completions come in block order)
    static_assert(NDONE >= GROUPS, "done ring shorter than the decoder rotation");
    // Warpgroup-aligned roles (the register split below goes by warpgroup): warps 0..3 the
    // producers and the MMA issuer (warp 3 idle), then the decoder groups, then the epilogue.
    static constexpr int WARP_LOAD = 0, WARP_MMA = 1, WARP_XLOAD = 2, WARP_DEC0 = 4, NUM_DEC_WARPS = 4 * GROUPS;
    static constexpr int WARP_EPI0 = WARP_DEC0 + NUM_DEC_WARPS;
    // One MMA-issuing thread per accumulation chain: a thread issues one tcgen05.mma every
    // few dozen cycles, far slower than the tensor pipe runs a narrow (N <= 64) MMA, so the
    // chains are issued from separate warps (warp 1, then warps WARP_ISS1...).
    static constexpr int NISS = NCHAIN;
    static constexpr int WARP_ISS1 = WARP_EPI0 + 4;
    static constexpr int THREADS = (WARP_ISS1 + NISS - 1) * 32;
    // Register split (BX = 256: four warpgroups). The epilogue holds the whole tile's sums as
    // bf16 pairs (BX / 2 registers) so that it can release the single accumulator before it
    // stores y; the producers' warpgroup gives up what the epilogue takes. The host checks that
    // the kernel was built for exactly REG_LAUNCH registers per thread before launching it.
    static constexpr bool REG_SPLIT = THREADS == 512 && GROUPS == 2 && NISS == 1;
    static constexpr int REG_LAUNCH = 128;
    static constexpr int REG_PROD = 80, REG_DEC = 120, REG_EPI = 4 * REG_LAUNCH - REG_PROD - 2 * REG_DEC;
    static_assert(!REG_SPLIT || (REG_PROD + 2 * REG_DEC + REG_EPI == 4 * REG_LAUNCH && REG_EPI <= 256 &&
                                 REG_PROD % 8 == 0 && REG_DEC % 8 == 0 && REG_EPI % 8 == 0 &&
                                 THREADS * REG_LAUNCH == 65536),
                  "register split must add up to the launch's registers");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(BX % 16 == 0 && BX >= 16 && BX <= 256, "MMA N");
    static_assert(A_COLS + NACC * ACC_COLS <= 512, "TMEM columns");
    static_assert(RAW_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "stage alignment");
    static_assert(A_STAGES % 2 == 0, "a block is two A half-stages");
    // `ready` slot b % A_BLOCKS takes block b's x copy and its A tile: the x producer re-arms it
    // for block b only after blk_done of block b - X_STAGES, which must come after the MMAs
    // that waited on the slot's previous phase (block b - A_BLOCKS)
    static_assert(A_BLOCKS >= X_STAGES, "ready ring shorter than the x ring");
};

// GS = 0: one fp32 scale per weight row, applied to the accumulated sums in the epilogue.
// GS = 32 .. 256: one float16 max per GS weights of a row (the group-wise format); the
// decoders form each group's 16 magnitudes bf16(LUT[q] * max) in registers and decode by
// byte-plane lookups, and the epilogue applies no scale.
// One 64-K half of a weight row in a BITS-bit stream (its 2 BITS code words in cw, its two sign
// words in sw) -> the 64 weights sign * bf16 LUT[q] as 32 bf16 pairs, pair P (weights 2P, 2P + 1)
// in o[P / 16][P % 16]. The table entry of code q holds LUT[q] in both halves (one copy per lane
// at byte 256 q + 4 lane); the sign spreads are the pair table's (opq_bits.h).
template <int BITS, class Load>
__device__ __forceinline__ void decode_half_bits(const uint32_t (&cw)[2 * BITS], const uint32_t (&sw)[2], uint32_t lw,
                                                 uint32_t lw2, Load load, uint32_t (&o)[2][16]) {
    constexpr uint32_t MASK = (1u << BITS) - 1u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {          // sign byte j: weights 8j .. 8j + 7
        const uint32_t x = load(opqbits::prmt(sw[j >> 2], lw2, 0x5504u | ((uint32_t)(j & 3) << 4)));
#pragma unroll
        for (int e = 0; e < 4; ++e) {      // pair 4j + e
            uint32_t m[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int bit = (8 * j + 2 * e + t) * BITS, wi = bit >> 5, sh = bit & 31;
                const uint32_t q = (sh + BITS <= 32) ? ((cw[wi] >> sh) & MASK)
                                                     : (__funnelshift_r(cw[wi], cw[(wi + 1) % (2 * BITS)], sh) & MASK);
                m[t] = load((q << 8) | lw);
            }
            o[j >> 2][(j & 3) * 4 + e] = __byte_perm(m[0], m[1], 0x7610u) ^ ((x << e) & 0x80008000u);
        }
    }
}

template <int BX, int GS = 0, int BITS = 4>
__global__ void __launch_bounds__(Cfg<BX, BITS>::THREADS, 1)
    wide_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_xh,
                  const __grid_constant__ CUtensorMap tmap_codes, const __grid_constant__ CUtensorMap tmap_signs,
                  const __grid_constant__ LinearArgs args) {
    using C = Cfg<BX, BITS>;
    static_assert(BITS == 4 || GS == 0, "the other bit widths take per-row scales");
    static_assert(C::NISS == 1, "one MMA issuer (warp 1)");
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    if ((sbase & 1023u) != 0u) {   // the same for every CTA: nothing has been started yet
        if (threadIdx.x == 0) atomicOr(&g_error, kErrSmemAlign);
        return;
    }

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *raw_full = bars;
    uint64_t *raw_empty = raw_full + C::RAW_STAGES;
    // ready[b % A_BLOCKS]: block b's x copy has landed (the x producer's expect_tx arrival and
    // the copy's bytes) and its A tile is in TMEM (one arrival per decoder warp) -- the MMA
    // issuer waits once per block
    uint64_t *ready = raw_empty + C::RAW_STAGES;
    uint64_t *blk_done = ready + C::A_BLOCKS;
    uint64_t *acc_full = blk_done + C::NDONE;
    uint64_t *acc_empty = acc_full + C::NACC;
    uint64_t *drain = acc_empty + C::NACC;
    uint64_t *fixb = drain + 1;   // per TMEM lane quarter: the partner's partial sums have landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_TMEM);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = args.m_tiles * args.n_tiles;
    const bool signs_by_tma = args.signs_tma != 0;

    RunIter it;
    it.init(args, tiles, gridDim.x, blockIdx.x);
    int tile, r0, r1, j;

    // one 128-K block of codes and signs (signs by TMA) into raw stage rs
    auto issue_raw = [&](int rs, int r, int n_blk) {
        mbar_arrive_expect_tx(&raw_full[rs], C::RAW_BYTES);
        tma_load_2d(smem + C::OFF_RAW + rs * C::RAW_BYTES, &tmap_codes, r * C::CODE_WORDS, n_blk * C::BW, &raw_full[rs]);
        tma_load_2d(smem + C::OFF_RAW + rs * C::RAW_BYTES + C::RAW_CODE_BYTES, &tmap_signs, r * (C::KR / 32),
                    n_blk * C::BW, &raw_full[rs]);
    };
    // the CTA's block b (block r of its tile): x (BX rows, or BX/2 for a half-width run) into
    // x stage b % X_STAGES, completing on ready[b % A_BLOCKS]
    auto issue_x = [&](int b, int r, int tile_, int xoff, int xrows) {
        const bool half = xrows != BX;
        const void *xmap = half ? (const void *)&tmap_xh : (const void *)&tmap_x;
        const int xrow = (tile_ % args.m_tiles) * BX + xoff;
        uint64_t *bar = &ready[b % C::A_BLOCKS];
        mbar_arrive_expect_tx(bar, half ? C::X_BYTES / 2 : C::X_BYTES);
        uint8_t *dst = smem + C::OFF_X + (b % C::X_STAGES) * C::X_BYTES;
        tma_load_2d(dst, xmap, r * C::KR, xrow, bar);
        tma_load_2d(dst + C::X_HALF_BYTES, xmap, r * C::KR + C::KA, xrow, bar);
    };

    // The first copies go out before anything else: a cold copy takes microseconds to land,
    // and building the pair table and allocating TMEM hide most of that. Thread 0 (the raw
    // producer's lane) initialises every barrier but `ready` and fills the raw ring; the x
    // producer's lane initialises `ready` and fills the x ring. Nobody else touches a barrier
    // before the CTA-wide barrier below.
    int pre_raw = 0, pre_x = 0;   // blocks already issued by the two producers
    if (threadIdx.x == 0) pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::RAW_STAGES; ++s) {
            // the codes' (and signs') expect_tx arrival, plus 32 cp.async arrivals when signs are copied by threads
            mbar_init(&raw_full[s], signs_by_tma ? 1 : 1 + 32);
            mbar_init(&raw_empty[s], 4);          // the 4 warps of the group that decodes the block
        }
        for (int s = 0; s < C::NDONE; ++s) mbar_init(&blk_done[s], C::NISS);   // one commit per issuer
        for (int s = 0; s < C::NACC; ++s) {
            mbar_init(&acc_full[s], C::NISS);
            mbar_init(&acc_empty[s], 4);
        }
        mbar_init(drain, C::NISS);
        for (int s = 0; s < 4; ++s) mbar_init(&fixb[s], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmap_codes);
        if (signs_by_tma) {
            tma_prefetch_desc(&tmap_signs);
            pdl_wait();
            RunIter pit = it;
            while (pre_raw < C::RAW_STAGES && pit.next(tile, r0, r1, j)) {
                const int n_blk = tile / args.m_tiles;
                for (int r = r0; r < r1 && pre_raw < C::RAW_STAGES; ++r, ++pre_raw) issue_raw(pre_raw, r, n_blk);
            }
        }
    }
    if (warp == C::WARP_XLOAD && lane == 0) {
        // the x producer's expect_tx arrival and the 4 warps of the decoding group
        for (int s = 0; s < C::A_BLOCKS; ++s) mbar_init(&ready[s], 1 + 4);
        fence_mbar_init();
        tma_prefetch_desc(&tmap_x);
        if (args.tail_split == 2) tma_prefetch_desc(&tmap_xh);
        pdl_wait();
        RunIter pit = it;
        int xoff, xrows;
        while (pre_x < C::X_STAGES && pit.next(tile, r0, r1, j, xoff, xrows, BX)) {
            for (int r = r0; r < r1 && pre_x < C::X_STAGES; ++r, ++pre_x) issue_x(pre_x, r, tile, xoff, xrows);
        }
    }
    // ---- pair table: 32 copies of value(b) then 32 copies of spread(b) per entry b
    // (4 bits: entry b holds the pair of magnitudes of code byte b; other widths: entry q < 2^BITS
    // holds the magnitude of code q in both halves)
    if (BITS == 4)
        opqbits::build_pair_table<4>(sbase + C::OFF_TABLE, warp, C::THREADS / 32, lane, (uint32_t)args.lut[lane & 15]);
    else
        opqbits::build_pair_table<BITS>(sbase + C::OFF_TABLE, warp, C::THREADS / 32, lane, (uint32_t)args.lutb[lane],
                                        (uint32_t)args.lutb[32 + lane]);
    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < C::WARP_DEC0) {
        // the producers' warpgroup (warp 3 idle) gives registers to the epilogue's
        if constexpr (C::REG_SPLIT) setmaxnreg_dec<C::REG_PROD>();
        if (warp == C::WARP_LOAD) {
            // ----------------------------------------------------------- raw producer
            pdl_wait();
            const int swd = args.K / 32;        // sign words per row
            int rs = 0;
            uint32_t rph = 0;
            int raw_issued = 0;
            bool ok = true;
            pre_raw = __shfl_sync(0xFFFFFFFFu, pre_raw, 0);
            while (ok && it.next(tile, r0, r1, j)) {
                const int n_blk = tile / args.m_tiles;
                for (int r = r0; r < r1 && ok; ++r) {
                    if (raw_issued < pre_raw) {   // issued before the CTA-wide barrier
                        ++raw_issued;
                        if (++rs == C::RAW_STAGES) { rs = 0; rph ^= 1; }
                        continue;
                    }
                    // lane 0 waits for the stage; the verdict and the ordering reach the other lanes
                    int okw = 1;
                    if (lane == 0) okw = mbar_wait(&raw_empty[rs], rph ^ 1) ? 1 : 0;
                    okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
                    __syncwarp();
                    if (!okw) { ok = false; break; }
                    const uint32_t dst = sbase + C::OFF_RAW + rs * C::RAW_BYTES;
                    if (lane == 0) {
                        if (signs_by_tma) {
                            issue_raw(rs, r, n_blk);
                        } else {
                            mbar_arrive_expect_tx(&raw_full[rs], C::RAW_CODE_BYTES);
                            tma_load_2d(smem + C::OFF_RAW + rs * C::RAW_BYTES, &tmap_codes, r * C::CODE_WORDS,
                                        n_blk * C::BW, &raw_full[rs]);
                        }
                    }
                    if (!signs_by_tma) {
                        // sign words: 128 rows x 4 words; copy i of lane l is word 32 i + l of the stage
                        // (consecutive lanes, consecutive banks); out-of-range words read as 0
    #pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int e = i * 32 + lane;
                            const int row = e >> 2, w = e & 3;
                            const int n = n_blk * C::BW + row, kw = r * 4 + w;
                            const bool in = n < args.N && kw < swd;
                            const uint32_t *src = args.signs + (in ? (size_t)n * swd + kw : 0);
                            cp_async_4(dst + C::RAW_CODE_BYTES + row * 16 + w * 4, src, in ? 4u : 0u);
                        }
                        cp_async_mbar_arrive(&raw_full[rs]);
                    }
                    ++raw_issued;
                    if (++rs == C::RAW_STAGES) { rs = 0; rph ^= 1; }
                }
            }
            if (!ok) {
                // let every copy already issued land before the CTA can exit
                asm volatile("cp.async.wait_all;" ::: "memory");
                if (lane == 0) {
                    for (int i = 0; i < raw_issued && i < C::RAW_STAGES; ++i) {
                        if (--rs < 0) { rs = C::RAW_STAGES - 1; rph ^= 1; }
                        (void)mbar_wait(&raw_full[rs], rph);
                    }
                }
            }
        } else if (warp == C::WARP_XLOAD) {
            // ----------------------------------------------------------- x producer
            if (lane == 0) {
                int b = 0;                 // the CTA's block index
                bool ok = true;
                int xoff, xrows;
                while (ok && it.next(tile, r0, r1, j, xoff, xrows, BX)) {
                    for (int r = r0; r < r1; ++r, ++b) {
                        if (b < pre_x) continue;   // issued before the CTA-wide barrier
                        // stage b % X_STAGES last held block b - X_STAGES
                        const int prev = b - C::X_STAGES;
                        if (prev >= 0 && !mbar_wait(&blk_done[prev % C::NDONE], (uint32_t)(prev / C::NDONE) & 1u)) {
                            ok = false;
                            break;
                        }
                        // a half-width run loads its BX/2 activation rows with the half-height box
                        issue_x(b, r, tile, xoff, xrows);
                    }
                }
                if (!ok) {
                    // let the copies already issued land before the CTA can exit (a slot whose decoder
                    // arrivals never come ends this wait by its time limit)
                    for (int i = 1; i <= C::X_STAGES && b - i >= 0; ++i)
                        (void)mbar_wait(&ready[(b - i) % C::A_BLOCKS], (uint32_t)((b - i) / C::A_BLOCKS) & 1u);
                }
            }
        } else if (warp == C::WARP_MMA) {
            // ----------------------------------------------------------- MMA issuers
            // Issuer i accumulates K-steps k = i, i + NISS, ... of every 64-K half into chain i.
            if (lane == 0) {
                const int iss = warp == C::WARP_MMA ? 0 : warp - C::WARP_ISS1 + 1;
                int ab = 0;
                uint32_t abph = 0;
                int as0 = 0, xs = 0, ds = 0;       // A half-stage of the block's first half, x stage, blk_done slot
                uint32_t rph = 0;                  // parity of ready[as0 / 2]
                bool ok = true;
                constexpr uint32_t idesc_full = idesc_bf16_f32(128, BX);
                constexpr uint32_t idesc_half = idesc_bf16_f32(128, BX / 2);
                int xoff, xrows;
                while (ok && it.next(tile, r0, r1, j, xoff, xrows, BX)) {
                    const uint32_t idesc = xrows == BX ? idesc_full : idesc_half;
                    if (!mbar_wait(&acc_empty[ab], abph ^ 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + C::A_COLS + ab * C::ACC_COLS + iss * BX;
                    uint32_t acc = 0;              // 0 for the chain's first MMA of the run
                    for (int r = r0; r < r1; ++r) {
                        const uint32_t xaddr = sbase + C::OFF_X + xs * C::X_BYTES;
                        if (!mbar_wait(&ready[as0 >> 1], rph)) { ok = false; break; }
                        tc_fence_after();
    #pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t a_tmem = tmem_base + (as0 + h) * 32;
                            const uint64_t bdesc = smem_desc_sw128(xaddr + h * C::X_HALF_BYTES);
    #pragma unroll
                            for (int k = 0; k < C::KA / 16; ++k) {
                                if (k % C::NISS != iss % C::NISS) continue;
                                umma_bf16_ts(d_tmem, a_tmem + 8 * k, bdesc + 2 * k, idesc, acc);
                                acc = 1;
                            }
                        }
                        umma_commit(&blk_done[ds]);
                        as0 += 2;
                        if (as0 == C::A_STAGES) { as0 = 0; rph ^= 1; }
                        if (++xs == C::X_STAGES) xs = 0;
                        if (++ds == C::NDONE) ds = 0;
                    }
                    if (ok) umma_commit(&acc_full[ab]);
                    if (++ab == C::NACC) { ab = 0; abph ^= 1; }
                }
                // every MMA issued by this thread has completed once `drain` flips
                umma_commit(drain);
                (void)mbar_wait(drain, 0);
            }
        }
    } else if (warp < C::WARP_EPI0) {
        if constexpr (C::REG_SPLIT && C::REG_DEC != C::REG_LAUNCH) setmaxnreg_dec<C::REG_DEC>();
        // ----------------------------------------------------------- decoders
        pdl_wait();   // the group-wise scales are read from global memory
        const int g = (warp - C::WARP_DEC0) >> 2;        // decoder group
        const int q = warp & 3;                          // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;                   // weight row in the tile = TMEM lane
        const uint32_t lw = 4u * lane, lw2 = 128u + 4u * lane;
        const uint32_t *tabp = reinterpret_cast<const uint32_t *>(smem + C::OFF_TABLE);
        auto load = [&](uint32_t off) { return tabp[off >> 2]; };
        // 64-byte swizzle of the codes stage: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
        const uint32_t sw64 = (uint32_t)((row >> 1) & 3);
        const uint32_t tm_row = tmem_base + ((uint32_t)(q * 32) << 16);
        // one 128-K block of this group: raw words in, A tile (both 64-K halves) out to TMEM;
        // block r of a tile whose weight rows start at n_base (r, n_base used by the group-wise format)
        auto run_block = [&](int blk, int r, int n_base) -> bool {
            const int n_row = n_base + row;
            auto gmax_at = [&](int gi) -> float {
                return n_row < args.N ? __half2float(__ushort_as_half(__ldg(args.gmax + (size_t)n_row * args.ngk + gi)))
                                      : 0.0f;
            };
            (void)gmax_at;
            (void)r;
            const int rs = blk % C::RAW_STAGES;
            const uint32_t rph = (uint32_t)(blk / C::RAW_STAGES) & 1u;
            if (!warp_wait(&raw_full[rs], rph)) return false;
            const uint8_t *rawc = smem + C::OFF_RAW + rs * C::RAW_BYTES + row * (C::CODE_WORDS * 4);
            const uint8_t *raws = smem + C::OFF_RAW + rs * C::RAW_BYTES + C::RAW_CODE_BYTES + row * (C::KR / 8);
#pragma unroll
            for (int h = 0; h < C::KR / C::KA; ++h) {     // two 64-K A stages per block
                const int sidx = blk * 2 + h;
                const int as = sidx % C::A_STAGES;
                // this half's 2 BITS code words (4 bits: two 16-byte chunks, 64-byte swizzle) and 2 sign words
                uint32_t cw[2 * BITS];
                if constexpr (BITS == 4) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(rawc + ((((uint32_t)(2 * h + c)) ^ sw64) << 4));
                        cw[4 * c] = v.x; cw[4 * c + 1] = v.y; cw[4 * c + 2] = v.z; cw[4 * c + 3] = v.w;
                    }
                } else {
                    // unswizzled rows of 16 BITS bytes; the half starts at word 2 BITS h (8-byte aligned)
#pragma unroll
                    for (int c = 0; c < BITS; ++c) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(rawc + 8 * (BITS * h + c));
                        cw[2 * c] = v.x; cw[2 * c + 1] = v.y;
                    }
                }
                const uint2 sv = *reinterpret_cast<const uint2 *>(raws + 8 * h);
                const uint32_t sw[2] = {sv.x, sv.y};
                if (h == 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&raw_empty[rs]);   // the block's raw words are in registers now
                }
                uint32_t o[2][16];
                if constexpr (BITS != 4) {
                    decode_half_bits<BITS>(cw, sw, lw, lw2, load, o);
                } else if constexpr (GS == 0) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        uint32_t t4[4];
                        opqbits::decode8_table(cw[i], sw[i >> 2], (uint32_t)(i & 3), lw, lw2, load, t4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) o[i >> 2][(i & 3) * 4 + e] = t4[e];
                    }
                } else {
                    // the half's group (two groups of 32 weights when GS = 32)
                    const int gi = (r * C::KR + h * C::KA) / GS;
                    opqbits::DecodeTable Ta, Tb;
                    make_group_table(Ta, args.lutf, gmax_at(gi));
                    if constexpr (GS == 32) make_group_table(Tb, args.lutf, gmax_at(gi + 1));
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        uint32_t t4[4];
                        opqbits::decode8(cw[i], (sw[i >> 2] >> (8 * (i & 3))) & 0xFFu,
                                         (GS == 32 && i >= 4) ? Tb : Ta, t4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) o[i >> 2][(i & 3) * 4 + e] = t4[e];
                    }
                }
                // the block's A slot last held block blk - A_BLOCKS
                const int prev = blk - C::A_BLOCKS;
                if (h == 0 && prev >= 0 &&
                    !warp_wait(&blk_done[prev % C::NDONE], (uint32_t)(prev / C::NDONE) & 1u))
                    return false;
                tc_fence_after();
                tmem_st_32x32b_x16(tm_row + as * 32, o[0]);
                tmem_st_32x32b_x16(tm_row + as * 32 + 16, o[1]);
                if (h == 1) {   // both halves stored: the block's A tile is complete
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ready[blk % C::A_BLOCKS]);
                }
            }
            return true;
        };
        bool ok = true;
        if constexpr (GS == 0) {
            int nblocks = 0;
            while (it.next(tile, r0, r1, j)) nblocks += r1 - r0;
            for (int blk = g; blk < nblocks && ok; blk += C::GROUPS) ok = run_block(blk, 0, 0);
        } else {
            int blk = 0;
            while (ok && it.next(tile, r0, r1, j)) {
                const int n_base = (tile / args.m_tiles) * C::BW;
                for (int r = r0; r < r1 && ok; ++r, ++blk)
                    if (blk % C::GROUPS == g) ok = run_block(blk, r, n_base);
            }
        }
    } else {
        if constexpr (C::REG_SPLIT) setmaxnreg_inc<C::REG_EPI>();
        // ----------------------------------------------------------- epilogue
        pdl_wait();
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const bool vec_y = (args.N % 8) == 0;
        int ab = 0;
        uint32_t abph = 0;
        int xoff, xrows;
        // y[m0 .. m0 + 15][n] for this lane's weight row n from the 8 bf16 pairs pk[i] =
        // (row m0 + 2i, row m0 + 2i + 1)
        auto store_pairs = [&](const uint32_t (&pk)[8], int m0, int n, int n0) {
            if (vec_y && n0 + 32 <= args.N) {
                // lanes n and n ^ 1 swap halves so that the even lane holds row m0 + 2i and the odd
                // lane row m0 + 2i + 1, each for weight rows n & ~1 and (n & ~1) + 1: one 4-byte
                // store per lane per row pair
                const uint32_t odd = (uint32_t)lane & 1u;
                const uint32_t sel = odd ? 0x3276u : 0x5410u;
                uint32_t *yw = reinterpret_cast<uint32_t *>(args.y + (size_t)(m0 + (int)odd) * args.N + n0 +
                                                            (lane & ~1));
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, pk[i], 1);
                    const uint32_t word = __byte_perm(pk[i], other, sel);
                    if (m0 + 2 * i + (int)odd < args.M) yw[(size_t)i * (size_t)args.N] = word;
                }
            } else if (n < args.N) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + i;
                    if (m < args.M) args.y[(size_t)m * args.N + n] = (uint16_t)(pk[i >> 1] >> (16 * (i & 1)));
                }
            }
        };
        // y[m0 .. m0 + 15][n] = bf16(fv(v[i])) (rounded to nearest even)
        auto store16 = [&](const uint32_t (&v)[16], int m0, int n, int n0, auto &&fv) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2_rn(fv(__uint_as_float(v[2 * i])), fv(__uint_as_float(v[2 * i + 1])));
            store_pairs(pk, m0, n, n0);
        };
        while (it.next(tile, r0, r1, j, xoff, xrows, BX)) {
            const int n_blk = tile / args.m_tiles, m_blk = tile % args.m_tiles;
            const int n = n_blk * C::BW + row;
            const int n0 = n_blk * C::BW + q * 32;           // first row of this warp's quarter
            const bool full = (r0 == 0 && r1 == args.kblocks);
            const float scale = GS > 0 ? 1.0f : (n < args.N ? __ldg(args.scales + n) : 0.0f);
            const float bias = bias_at(args.bias, n, args.N);
            // the plain product, or the fused epilogue (bias, activation): chosen per tile, one
            // specialised store loop per kind, so no loop carries another kind's code. The kind is
            // read from the parameters once: inside the loop, every y store could alias them.
            const int act = args.act;
            const bool plain = args.bias == nullptr && act == EPI_NONE;
            auto fv_plain = [scale](float a) { return a * scale; };
            auto fv_bias = [scale, bias](float a) { return epi_value(a, scale, bias, EPI_NONE); };
            auto fv_silu = [scale, bias](float a) { return epi_value(a, scale, bias, EPI_SILU); };
            auto fv_gelu = [scale, bias](float a) { return epi_value(a, scale, bias, EPI_GELU_TANH); };
            auto store = [&](const uint32_t (&v)[16], int m0) {
                if (plain) store16(v, m0, n, n0, fv_plain);
                else if (act == EPI_SILU) store16(v, m0, n, n0, fv_silu);
                else if (act == EPI_GELU_TANH) store16(v, m0, n, n0, fv_gelu);
                else store16(v, m0, n, n0, fv_bias);
            };
            if (!warp_wait(&acc_full[ab], abph)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + C::A_COLS + ab * C::ACC_COLS;
            bool released = false;
            if (full && act != EPI_SILU && act != EPI_GELU_TANH) {
                // The whole tile's outputs into registers as bf16 pairs (column pair (2i, 2i + 1)
                // in pk[i]), then the accumulator goes back to the MMA issuer at once and y is
                // stored from registers while the next tile's MMAs run. (An activation's math
                // would hold too many registers here: those tiles take the streaming loop below.)
                uint32_t pk[BX / 2];
                auto gather = [&](auto &&fv) {
#pragma unroll
                    for (int c0 = 0; c0 < BX; c0 += 16) {
                        if (c0 < xrows) {
                            uint32_t v[16];
                            tmem_ld_32x32b_x16(taddr + c0, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                pk[c0 / 2 + i] = pack_bf16x2_rn(fv(__uint_as_float(v[2 * i])), fv(__uint_as_float(v[2 * i + 1])));
                        }
                    }
                };
                if (plain) gather(fv_plain);
                else gather(fv_bias);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ab]);
                released = true;
#pragma unroll
                for (int c0 = 0; c0 < BX; c0 += 16) {
                    if (c0 < xrows) {
                        uint32_t p8[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) p8[i] = pk[c0 / 2 + i];
                        store_pairs(p8, m_blk * BX + xoff + c0, n, n0);
                    }
                }
            } else if (full) {
                // with an activation: 16 columns at a time, loaded, computed and stored
#pragma unroll 1
                for (int c0 = 0; c0 < xrows; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(taddr + c0, v);
                    tmem_ld_wait();
                    store(v, m_blk * BX + xoff + c0);
                }
            } else {
                // Half-K tail run (the CTA's last): the tile's other half of K ran on the partner
                // CTA. Per lane quarter, the first of the two to get here publishes its fp32
                // partial sums to the workspace and raises a flag; the second waits for the flag
                // (the first is running and waits on nothing), copies the partner's sums in and
                // writes y from the total. p0 + p1 is the same in either order, so y does not
                // depend on which CTA arrives first.
                const int tt = tile - it.full_end;
                uint32_t *arrivals = args.counters + (size_t)tt * 8 + 2 * q;
                uint32_t *published = arrivals + 1;
                float *part = args.ws + ((size_t)tt * 4 + q) * (size_t)(BX * 32);   // [BX m][32 n] fp32
                uint32_t old = 0;
                if (lane == 0) old = atomicAdd(arrivals, 1u);
                old = __shfl_sync(0xFFFFFFFFu, old, 0);
                if (old == 0) {
#pragma unroll 1
                    for (int c0 = 0; c0 < BX; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(taddr + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) part[(size_t)(c0 + i) * 32 + lane] = __uint_as_float(v[i]);
                    }
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) flag_store_release(published, 1u);
                } else {
                    int okw = 1;
                    if (lane == 0) okw = flag_wait(published, 1u) ? 1 : 0;
                    okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
                    // this is the CTA's last run and its MMAs are complete, so the x ring is idle:
                    // quarter q's partner sums land in its 32 KiB there
                    const uint32_t pbuf = sbase + C::OFF_X + (uint32_t)q * (uint32_t)(BX * 32 * 4);
                    if (okw && lane == 0) {
                        fence_proxy_async_all();
                        mbar_arrive_expect_tx(&fixb[q], BX * 32 * 4);
                        bulk_load(smem + C::OFF_X + q * (BX * 32 * 4), part, BX * 32 * 4, &fixb[q]);
                    }
                    if (okw && warp_wait(&fixb[q], 0)) {
#pragma unroll 1
                        for (int c0 = 0; c0 < BX; c0 += 16) {
                            uint32_t v[16];
                            tmem_ld_32x32b_x16(taddr + c0, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float o;
                                asm volatile("ld.shared.f32 %0, [%1];"
                                             : "=f"(o) : "r"(pbuf + (uint32_t)((c0 + i) * 32 + lane) * 4u));
                                v[i] = __float_as_uint(__uint_as_float(v[i]) + o);
                            }
                            store(v, m_blk * BX + c0);
                        }
                    }
                    // ready for the next call (after a timeout the workspace must be zeroed again)
                    if (lane == 0) {
                        arrivals[0] = 0u;
                        published[0] = 0u;
                    }
                }
            }
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ab]);
            }
            if (++ab == C::NACC) { ab = 0; abph ^= 1; }
        }
    }

    // roles run on single lanes: reconverge every warp before the CTA barrier, so that the
    // barrier (and the warp-wide TMEM release after it) waits for every lane's last operation
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace opqk_wide
