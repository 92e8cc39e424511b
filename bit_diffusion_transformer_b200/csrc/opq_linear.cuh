// opq_linear.cuh — y = x W'^T with W' decoded on the fly from the OPQ planes,
// for narrow activation tiles (M <= 128: the weight-streaming regime).
//
// "OPQ INT4 Z-Image" model card: the OPQLinear forward decodes
// w = sign * (q/15)^(1/alpha) * max ("inference decoding") and multiplies.
// Here the row scale max is deferred to the epilogue: the tensor cores see
// sign * bf16((q/15)^(1/alpha)) and each fp32 sum is multiplied by scale[n] once.
//
// One kernel, templated on BX (activation rows per tile, 16..128):
//
//   D^T[128 x BX] = W'_tile[128 x K] * x_tile[BX x K]^T     (tcgen05, kind::f16)
//
// Weights sit on the MMA's 128-row side so that each decoded weight meets BX
// activation rows. Per CTA (one per SM, persistent):
//   warp 0       raw producer: codes (64-byte swizzle) and signs of 128 weight rows,
//                one load group (GRP consecutive 128-K blocks) per pair of TMA copies
//   warp 1       TMEM allocation and MMA issue; A comes from TMEM. For BX <= 64 warps 19, 20
//                issue too: one issuer per decoder group, each with its own accumulator
//   warp 2       x producer: the load group's x (BX rows, 128-byte swizzle), one copy
//   warps 3..14  three decoder groups of 4 warps (= the 128 TMEM lanes): each thread owns
//                one weight row and decodes 128 weights per block through the shared-memory
//                pair table (opq_bits.h), written to TMEM with tcgen05.st as the A operand
//   warps 15..18 epilogue: accumulator TMEM -> registers -> * scale[n] -> bf16 y,
//                or fp32 partial sums for tiles split across CTAs
// TMEM columns: [0, A_COLS) the A ring; then NACC accumulator buffers of NCH_ALL chains x BX.
//
// Work is a list of runs (tile, range of load groups). Mode 1 (stream-K) cuts the
// flattened (tile, load group) sequence into one contiguous range per CTA; a tile covered
// by several CTAs leaves fp32 partial sums in the workspace, and the epilogue warp that
// arrives last on the tile's counter (one per 32-row quarter) adds all partials in CTA
// order (deterministic), scales, rounds, stores y and resets the counter to zero.
// Mode 0 (whole tiles strided over CTAs) serves shapes with more tiles than counters.
// Wide tiles (M > 128) use opq_linear_wide.cuh.
#pragma once
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "opq_bits.h"
#include "opq_device.cuh"

namespace opqk {

using namespace opqdev;

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
// A load from read-only shared data (the pair table): not volatile, so the compiler may batch
// independent lookups; its address depends on data loaded after the table was published.
__device__ __forceinline__ uint32_t lds_ro_u32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
// a + b as a multiply-add by an opaque 1, so that it issues on the FMA pipe and
// leaves the integer ALU pipe to the decode's PRMT / LOP3
__device__ __forceinline__ uint32_t add_fma(uint32_t a, uint32_t b, uint32_t one) {
    uint32_t r;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(one), "r"(b));
    return r;
}

__device__ __forceinline__ void cp_async_4(uint32_t smem_dst, const void *gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_dst), "l"(gsrc), "r"(src_bytes)
                 : "memory");
}
// The mbarrier counts one arrival when all of this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
                 : "memory");
}

// tcgen05.st: 32 lanes x 16 consecutive 32-bit columns (thread i -> lane base + i)
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// tcgen05.ld: 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Every lane waits (and so acquires); the verdict is made warp-uniform, so a
// time-out seen by one lane can never leave the others behind at a warp barrier.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xFFFFFFFFu, ok) != 0;
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate), one CTA.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct LinearArgs {
    const uint32_t *signs;  // sign plane [N, K/32]
    const float *scales;
    uint16_t *y;
    float *ws;              // mode 1: fp32 partials [grid][runs_max][BX][128]
    uint32_t *counters;     // mode 1: arrivals per (tile, TMEM lane quarter); zero between calls
    int signs_tma;          // 1: sign plane rows are 16-byte aligned (K % 128 == 0), load it by TMA
    int M, N, K;
    int m_tiles, n_tiles;
    int kblocks;            // 128-K blocks per tile
    int ngroups;            // load groups per tile: consecutive blocks fetched by one copy per plane
                            // (balanced sizes ceil / floor of kblocks / ngroups, never above GRP)
    int mode;               // 0 whole tiles strided over CTAs, 1 contiguous unit ranges (stream-K)
    int runs_max;           // mode 1: most runs one CTA can have
    int tail_split;         // mode 0: 2 = tiles past the last full wave run as two half-width
                            // (BX/2 activation rows) runs on different CTAs; 1 = whole tiles
    uint16_t lut[16];       // bf16 (q/15)^(1/alpha)
    uint16_t lutb[64];      // other bit widths (wide kernel): bf16 (q/L)^(1/alpha), q = 0..L, L = 2^bits - 1
    // group-wise format (GS > 0)
    const uint16_t *gmax;   // float16 [N, K / GS]
    int ngk;                // groups per row (K / GS)
    float lutf[16];         // (q/15)^(1/alpha) in fp32
    // fused epilogue
    const uint16_t *bias;   // bf16 [N] added to every output row, or null
    int act;                // EPI_NONE, EPI_SILU, EPI_GELU_TANH
};

enum { EPI_NONE = 0, EPI_SILU = 1, EPI_GELU_TANH = 2 };

// tanh by the hardware approximation (tanh.approx.f32, absolute error about 5e-4), one MUFU op
__device__ __forceinline__ float tanh_hw(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One output before its bf16 rounding: the fp32 sum times the row scale, plus the bias, through
// the activation. SiLU v / (1 + e^-v) = v (1/2 + tanh(v/2) / 2); GELU's tanh form
// 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))). Both take one hardware tanh, so the epilogue
// that the next tile's MMAs wait for stays short; the approximation's error (at most about
// 2.5e-4 |v| in the output) is far inside the linear's tolerance. With no bias and no
// activation this is the plain product acc * scale.
__device__ __forceinline__ float epi_value(float acc, float scale, float bias, int act) {
    float v = fmaf(acc, scale, bias);
    if (act == EPI_SILU) {
        v = v * fmaf(0.5f, tanh_hw(0.5f * v), 0.5f);
    } else if (act == EPI_GELU_TANH) {
        const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
        v = 0.5f * v * (1.0f + tanh_hw(u));
    }
    return v;
}

__device__ __forceinline__ float bias_at(const uint16_t *bias, int n, int N) {
    return (bias != nullptr && n < N) ? __uint_as_float((uint32_t)__ldg(bias + n) << 16) : 0.0f;
}

// a group's 16 decoded magnitudes bf16(lutf[q] * gm) as byte planes (opq_bits.h DecodeTable)
__device__ __forceinline__ void make_group_table(opqbits::DecodeTable &T, const float (&lutf)[16], float gm) {
    uint32_t wd[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) wd[j] = pack_bf16x2_rn(lutf[2 * j] * gm, lutf[2 * j + 1] * gm);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        T.L[i] = __byte_perm(wd[2 * i], wd[2 * i + 1], 0x6420u);   // low bytes of entries 4i .. 4i + 3
        T.H[i] = __byte_perm(wd[2 * i], wd[2 * i + 1], 0x7531u);   // their high bytes
    }
}

// Units (tile, load group) of CTA c out of C in stream-K mode: [begin(c), begin(c + 1)).
// 32-bit arithmetic (a 64-bit division is a long software routine on the critical path of every
// role's start and of the fix-up): the host plans stream-K only when U * C < 2^31.
__host__ __device__ __forceinline__ uint32_t unit_begin(uint32_t c, uint32_t C, uint32_t U) { return (c * U) / C; }
// The CTA whose range holds unit u.
__host__ __device__ __forceinline__ uint32_t unit_owner(uint32_t u, uint32_t C, uint32_t U) {
    return ((u + 1) * C - 1) / U;
}

// Load groups of a tile: ng groups of consecutive 128-K blocks, sizes as even as possible
// (the first kb % ng groups one block longer), group g starting at block start(g).
struct LGroups {
    int q, rem;
    __device__ __forceinline__ void init(int kb, int ng) {
        q = kb / ng;
        rem = kb - q * ng;
    }
    __device__ __forceinline__ int start(int g) const { return g * q + (g < rem ? g : rem); }
};

// One run of a CTA: a weight tile, a range of its load groups [g0, g1) (blocks [r0, r1)),
// its index j among the CTA's runs, and the activation rows [xoff, xoff + xrows) of the tile.
struct Run {
    int tile, g0, g1, r0, r1, j, xoff, xrows;
};

// The sequence of runs of one CTA; every role walks the same sequence.
struct RunIter {
    int mode, tiles, ng, grid, cta;
    LGroups lg;
    int t_cur, g_cur;   // mode 1: the next unit (tile, load group)
    int left;           // mode 1: units left
    int t_next;         // mode 0
    int full_end;       // mode 0: tiles in whole waves (handed out strided)
    int split;          // mode 0: 1 or 2 runs per tile after the whole waves
    bool tail_done;
    int run_idx;
    __device__ __forceinline__ void init(const LinearArgs &a, int tiles_, int grid_, int cta_) {
        mode = a.mode;
        tiles = tiles_;
        ng = a.ngroups;
        lg.init(a.kblocks, a.ngroups);
        grid = grid_;
        cta = cta_;
        run_idx = 0;
        t_next = cta_;
        split = a.tail_split;
        full_end = split == 2 ? (tiles_ / grid_) * grid_ : tiles_;
        tail_done = false;
        const uint32_t U = (uint32_t)tiles * (uint32_t)ng;
        const uint32_t u = unit_begin((uint32_t)cta_, (uint32_t)grid_, U);
        left = (int)(unit_begin((uint32_t)cta_ + 1u, (uint32_t)grid_, U) - u);
        t_cur = (int)(u / (uint32_t)ng);
        g_cur = (int)(u - (uint32_t)t_cur * (uint32_t)ng);
    }
    // the next run for a tile of bx activation rows; false at the end
    __device__ __forceinline__ bool next(Run &R, int bx) {
        R.xoff = 0;
        R.xrows = bx;
        if (mode == 0) {
            if (t_next < full_end) {
                R.tile = t_next;
                t_next += grid;
            } else if (split == 2) {
                // tail tile t is run by CTAs 2 (t - full_end) and 2 (t - full_end) + 1, one half each
                if (tail_done || cta >= 2 * (tiles - full_end)) return false;
                R.tile = full_end + (cta >> 1);
                R.xrows = bx / 2;
                R.xoff = (cta & 1) * R.xrows;
                tail_done = true;
            } else {
                return false;
            }
            R.g0 = 0;
            R.g1 = ng;
        } else {
            if (left <= 0) return false;
            R.tile = t_cur;
            R.g0 = g_cur;
            R.g1 = g_cur + left < ng ? g_cur + left : ng;
            left -= R.g1 - R.g0;
            ++t_cur;
            g_cur = 0;
        }
        R.r0 = lg.start(R.g0);
        R.r1 = lg.start(R.g1);
        R.j = run_idx++;
        return true;
    }
};

template <int BX>
struct Cfg {
    static constexpr int BW = 128;                     // weight rows per tile (MMA M)
    static constexpr int KR = 128;                     // K per raw (codes/signs) stage
    static constexpr int KA = 64;                      // K per A stage (TMEM) and per x stage (smem)
    // Blocks per load group (one TMA copy per plane and per group: under load the SM's copy
    // engine serves a copy every few hundred ns almost whatever its size, so narrow tiles,
    // whose per-block data is small, fetch several blocks per copy). GRP > 1 needs K % 128 == 0.
    static constexpr int GRP = BX <= 16 ? 4 : (BX <= 64 ? 2 : 1);
    // raw stages hold one load group each; a decoder group waiting on a stage knows only that
    // the block three before its own was loaded, so at least three stages keep parity waits exact
    static constexpr int RAW_STAGES = GRP > 1 ? 3 : (BX >= 256 ? 2 : (BX >= 128 ? 4 : 6));
    // decoder groups of 4 warps: group g decodes the CTA's 128-K blocks g, g + G, ...;
    // thread r of a group owns weight row r (TMEM lane r) and decodes its whole 128-K block row
    static constexpr int GROUPS = BX >= 256 ? 2 : 3;
    // MMA issuers. A narrow block's 8 MMAs take one issuing thread longer than a decoder group
    // takes to decode the block, so narrow tiles (BX <= 64) give every decoder group an issuer
    // of its own (issuer i issues the blocks group i decodes, into its own accumulator) and
    // the tensor pipe takes MMAs from three threads at once; wider tiles keep one issuer.
    static constexpr int NISS = BX <= 64 ? GROUPS : 1;
    // A ring in TMEM, in 128-K blocks (two 64-K half-stages of 32 columns each). With one
    // issuer per group, block b uses slot b % A_BLOCKS and A_BLOCKS is a multiple of GROUPS,
    // so every slot is used by one decoder group and one issuer only: two slots per group for
    // BX <= 32, one for BX = 64 (whose three accumulators take 192 columns).
    static constexpr int A_BLOCKS = NISS > 1 ? (BX <= 32 ? 2 : 1) * GROUPS : 4;
    static constexpr int A_STAGES = 2 * A_BLOCKS;      // 32 TMEM columns each (64 K of bf16 pairs)
    static constexpr int A_COLS = A_STAGES * 32;
    // x stages hold one load group (two 64-K swizzle atoms' worth of columns per block)
    static constexpr int X_STAGES = GRP == 4 ? 2 : (GRP == 2 ? (BX >= 64 ? 2 : 4) : (BX >= 256 ? 2 : 3));
    // One tcgen05.commit per 128-K block frees both its A slot and its x stage: a commit
    // stalls the tensor pipe for a few hundred cycles, so there is one per 8 MMAs, not per 4.
    // `blk_done` is one ring of NDONE slots per issuer; issuer i's t-th block (CTA block
    // b = t NISS + i) completes slot i NDONE + t % NDONE. An issuer's blocks complete in its
    // issue order, so the parity of each wait is exact when:
    //  - one issuer: the x producer waits for the last block of the group X_STAGES groups back,
    //    with up to (X_STAGES - 1) GRP blocks in between (NDONE >= 1 + (X_STAGES - 1) GRP); a
    //    decoder waits for block b - A_BLOCKS knowing only that its own previous wait (block
    //    b - GROUPS - A_BLOCKS) succeeded, which implies block b - A_BLOCKS - NDONE completed
    //    if NDONE >= GROUPS;
    //  - an issuer per group: a decoder's previous wait was on the same issuer's ring, one of
    //    its blocks earlier, and block b - A_BLOCKS + NISS NDONE cannot complete before block
    //    b is decoded if NDONE > A_BLOCKS / NISS; the x producer waits for the last NISS blocks
    //    up to the group X_STAGES back (each issuer's latest), advancing at most
    //    ceil(GRP / NISS) <= NDONE of an issuer's blocks per group, and the newest block that
    //    could alias a slot, last - (NISS - 1) + NISS NDONE, lies in a group not yet loaded if
    //    NISS (NDONE - 1) >= (X_STAGES - 1) GRP.
    static constexpr int NDONE_X = 1 + (X_STAGES - 1) * GRP;
    static constexpr int NDONE = NISS > 1 ? A_BLOCKS / NISS + 1 : (NDONE_X > A_BLOCKS ? NDONE_X : A_BLOCKS);
    static constexpr int NDONE_ALL = NISS * NDONE;
    // independent accumulation chains per tile: consecutive MMAs into one accumulator
    // serialize on its latency, which dominates when N (= BX) is small; with one issuer, K-step
    // k of a stage goes to chain k % NCHAIN; with an issuer per group, each issuer's blocks form
    // one chain. The epilogue adds the chains in a fixed order.
    static constexpr int NCHAIN = NISS > 1 ? 1 : (BX <= 32 ? 4 : (BX <= 64 ? 2 : 1));
    static constexpr int NCH_ALL = NISS * NCHAIN;         // chains per accumulator buffer
    static constexpr int ACC_COLS = NCH_ALL * BX;         // one accumulator buffer (all chains)
    static constexpr int NACC = (A_COLS + 2 * ACC_COLS <= 512) ? 2 : 1;   // accumulator buffers
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int BLK_CODE_BYTES = BW * KR / 2;    // 8 KiB per block: [128 rows][16 words], 64-byte swizzle
    static constexpr int BLK_SIGN_BYTES = BW * KR / 8;    // 2 KiB per block: [128 rows][4 words]
    static constexpr int RAW_CODE_BYTES = GRP * BLK_CODE_BYTES;   // a stage: GRP blocks of codes, then of signs
    static constexpr int RAW_BYTES = GRP * (BLK_CODE_BYTES + BLK_SIGN_BYTES);
    static constexpr int X_HALF_BYTES = BX * KA * 2;   // one 64-K half: BX rows x 128 bytes, 128-byte swizzle
    static constexpr int X_BYTES = GRP * 2 * X_HALF_BYTES;   // a stage: the group's halves in K order
    static constexpr int STAGE_EPI_BYTES = 4 * 2 * 16 * 32 * 2;   // 4 warps x 2 buffers x [16 m][32 n] bf16
    static constexpr int OFF_TABLE = 0;
    static constexpr int OFF_RAW = OFF_TABLE + (int)opqbits::kPairTableBytes;
    static constexpr int OFF_X = OFF_RAW + RAW_STAGES * RAW_BYTES;
    static constexpr int OFF_EPI = OFF_X + X_STAGES * X_BYTES;
    static constexpr int OFF_BAR = OFF_EPI + STAGE_EPI_BYTES;
    static constexpr int NUM_BARS = 2 * RAW_STAGES + X_STAGES + A_BLOCKS + NDONE_ALL + 2 * NACC + 1;
    static constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;
    // a group waits on raw stage blk % RAW_STAGES knowing only that its own previous block
    // (blk - GROUPS) was loaded, so the stage's previous phase (block blk - RAW_STAGES) must
    // be at least that old for the parity test to be exact
    static_assert(RAW_STAGES >= GROUPS, "raw ring shorter than the decoder rotation");
    static_assert(NISS > 1 || NDONE >= GROUPS, "done ring shorter than the decoder rotation");
    static_assert(NISS > 1 || NDONE >= NDONE_X, "done ring shorter than the x ring's reach");
    static_assert(NISS == 1 || (NISS == GROUPS && A_BLOCKS % NISS == 0 && NDONE > A_BLOCKS / NISS &&
                                NISS * (NDONE - 1) >= (X_STAGES - 1) * GRP && (GRP + NISS - 1) / NISS <= NDONE),
                  "issuer rings too short for exact parity waits");
    static constexpr int WARP_LOAD = 0, WARP_MMA = 1, WARP_XLOAD = 2, WARP_DEC0 = 3, NUM_DEC_WARPS = 4 * GROUPS;
    static constexpr int WARP_EPI0 = WARP_DEC0 + NUM_DEC_WARPS;
    // issuer 0 is warp WARP_MMA (which also owns the TMEM allocation), issuer i > 0 warp WARP_ISS1 + i - 1
    static constexpr int WARP_ISS1 = WARP_EPI0 + 4;
    static constexpr int THREADS = (WARP_ISS1 + NISS - 1) * 32;
    // the blk_done slot and parity of the CTA's block b
    __device__ __forceinline__ static int done_slot(int b) { return (b % NISS) * NDONE + (b / NISS) % NDONE; }
    __device__ __forceinline__ static uint32_t done_parity(int b) { return (uint32_t)((b / NISS) / NDONE) & 1u; }
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert(BX % 16 == 0 && BX >= 16 && BX <= 256, "MMA N");
    static_assert(A_COLS + NACC * ACC_COLS <= 512, "TMEM columns");
    static_assert(RAW_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "stage alignment");
    static_assert(A_STAGES % 2 == 0, "a block is two A half-stages");
};

// GS = 0: one fp32 scale per weight row, applied in the epilogue; GS = 32 .. 256: one float16
// max per GS weights of a row (the group-wise format), applied in the decode, no epilogue scale
template <int BX, int GS = 0>
__global__ void __launch_bounds__(Cfg<BX>::THREADS, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_xh,
                  const __grid_constant__ CUtensorMap tmap_codes, const __grid_constant__ CUtensorMap tmap_signs,
                  const __grid_constant__ LinearArgs args) {
    using C = Cfg<BX>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t pad = ((raw_base + 1023u) & ~1023u) - raw_base;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_base + pad;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *raw_full = bars;
    uint64_t *raw_empty = raw_full + C::RAW_STAGES;
    uint64_t *x_full = raw_empty + C::RAW_STAGES;
    uint64_t *a_full = x_full + C::X_STAGES;    // per A slot (128-K block): its A tile is in TMEM
    uint64_t *blk_done = a_full + C::A_BLOCKS;
    uint64_t *acc_full = blk_done + C::NDONE_ALL;
    uint64_t *acc_empty = acc_full + C::NACC;
    uint64_t *drain = acc_empty + C::NACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_TMEM);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = args.m_tiles * args.n_tiles;
    const bool signs_by_tma = args.signs_tma != 0;

    if (threadIdx.x == 0) pdl_launch_dependents();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::RAW_STAGES; ++s) {
            // the copies' expect_tx arrival, plus 32 cp.async arrivals when signs are copied by threads
            mbar_init(&raw_full[s], (C::GRP > 1 || signs_by_tma) ? 1 : 1 + 32);
            // the 4 warps of the decoding group, once per block of the stage's load group
            mbar_init(&raw_empty[s], 4 * C::GRP);
        }
        for (int s = 0; s < C::X_STAGES; ++s) mbar_init(&x_full[s], 1);
        for (int s = 0; s < C::A_BLOCKS; ++s) mbar_init(&a_full[s], 4);   // the 4 warps of the decoding group
        for (int s = 0; s < C::NDONE_ALL; ++s) mbar_init(&blk_done[s], 1);   // one commit (the block's issuer)
        for (int s = 0; s < C::NACC; ++s) {
            mbar_init(&acc_full[s], C::NISS);
            mbar_init(&acc_empty[s], 4);
        }
        mbar_init(drain, C::NISS);
        fence_mbar_init();
    }
    if (warp == C::WARP_LOAD && lane == 0) {
        tma_prefetch_desc(&tmap_codes);
        if (signs_by_tma) tma_prefetch_desc(&tmap_signs);
    }
    if (warp == C::WARP_XLOAD && lane == 0) {
        tma_prefetch_desc(&tmap_x);
        if (args.tail_split == 2) tma_prefetch_desc(&tmap_xh);
    }
    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    RunIter it;
    it.init(args, tiles, gridDim.x, blockIdx.x);
    Run R;
    const LGroups lg = it.lg;

    if (warp == C::WARP_LOAD) {
        // ----------------------------------------------------------- raw producer
        // one stage per load group: GRP blocks of codes and of signs. The first run is planned
        // before the wait for the previous kernel (planning reads no global memory).
        bool more = it.next(R, BX);
        pdl_wait();
        const int swd = args.K / 32;        // sign words per row
        int rs = 0;
        uint32_t rph = 0;
        int raw_issued = 0;
        bool ok = true;
        for (; ok && more; more = it.next(R, BX)) {
            const int n_blk = R.tile / args.m_tiles;
            for (int g = R.g0; g < R.g1 && ok; ++g) {
                const int r = lg.start(g), nb = lg.start(g + 1) - r;
                // lane 0 waits for the stage; the verdict and the ordering reach the other lanes
                int okw = 1;
                if (lane == 0) okw = mbar_wait(&raw_empty[rs], rph ^ 1) ? 1 : 0;
                okw = __shfl_sync(0xFFFFFFFFu, okw, 0);
                __syncwarp();
                if (!okw) { ok = false; break; }
                const uint32_t dst = sbase + C::OFF_RAW + rs * C::RAW_BYTES;
                if (lane == 0) {
                    uint8_t *sd = smem + C::OFF_RAW + rs * C::RAW_BYTES;
                    if (C::GRP > 1) {
                        // 3-D boxes {words, 128 rows, GRP blocks}: the group's blocks one after the
                        // other (blocks past the tile's end read as zero, blocks of the next group
                        // are fetched and not used)
                        mbar_arrive_expect_tx(&raw_full[rs], C::RAW_BYTES);
                        tma_load_3d(sd, &tmap_codes, 0, n_blk * C::BW, r, &raw_full[rs]);
                        tma_load_3d(sd + C::RAW_CODE_BYTES, &tmap_signs, 0, n_blk * C::BW, r, &raw_full[rs]);
                        // the decoders arrive once per block and warp: supply the arrivals of the
                        // group's missing blocks so that the stage's phase can complete
                        if (nb < C::GRP) mbar_arrive_count(&raw_empty[rs], 4u * (uint32_t)(C::GRP - nb));
                    } else {
                        mbar_arrive_expect_tx(&raw_full[rs], signs_by_tma ? C::RAW_BYTES : C::RAW_CODE_BYTES);
                        tma_load_2d(sd, &tmap_codes, r * (C::KR / 8), n_blk * C::BW, &raw_full[rs]);
                        if (signs_by_tma)
                            tma_load_2d(sd + C::RAW_CODE_BYTES, &tmap_signs, r * (C::KR / 32), n_blk * C::BW,
                                        &raw_full[rs]);
                    }
                }
                if (C::GRP == 1 && !signs_by_tma) {
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
        bool more = it.next(R, BX);
        pdl_wait();
        if (lane == 0) {
            int b = 0;                 // the CTA's block index
            int v = 0;                 // the CTA's load-group index
            int last_blk[C::X_STAGES]; // last block of the group each x stage holds
            bool ok = true;
            for (; ok && more; more = it.next(R, BX)) {
                const int m_blk = R.tile % args.m_tiles;
                // a half-width run loads its BX/2 activation rows with the half-height box
                const bool half = R.xrows != BX;
                const void *xmap = half ? (const void *)&tmap_xh : (const void *)&tmap_x;
                const uint32_t xbytes = half ? C::X_BYTES / 2 : C::X_BYTES;
                const int xrow = m_blk * BX + R.xoff;
                for (int g = R.g0; g < R.g1; ++g, ++v) {
                    const int r = lg.start(g), nb = lg.start(g + 1) - r;
                    const int xs = v % C::X_STAGES;
                    // the stage last held group v - X_STAGES: wait until its blocks' MMAs are done
                    // (each issuer's latest block up to the group's last: an issuer's blocks
                    // complete in order)
                    if (v >= C::X_STAGES) {
                        const int last = last_blk[xs];
                        for (int i = 0; i < C::NISS && last - i >= 0 && ok; ++i)
                            ok = mbar_wait(&blk_done[C::done_slot(last - i)], C::done_parity(last - i));
                        if (!ok) break;
                    }
                    mbar_arrive_expect_tx(&x_full[xs], xbytes);
                    uint8_t *dst = smem + C::OFF_X + xs * C::X_BYTES;
                    if (C::GRP > 1) {
                        // box {64, BX, 2 GRP}: the group's 64-K halves one after the other
                        tma_load_3d(dst, xmap, 0, xrow, 2 * r, &x_full[xs]);
                    } else {
                        tma_load_2d(dst, xmap, r * C::KR, xrow, &x_full[xs]);
                        tma_load_2d(dst + C::X_HALF_BYTES, xmap, r * C::KR + C::KA, xrow, &x_full[xs]);
                    }
                    b += nb;
                    last_blk[xs] = b - 1;
                }
            }
            if (!ok) {
                // let the copies already issued land before the CTA can exit
                for (int i = 1; i <= C::X_STAGES && v - i >= 0; ++i)
                    (void)mbar_wait(&x_full[(v - i) % C::X_STAGES], (uint32_t)((v - i) / C::X_STAGES) & 1u);
            }
        }
    } else if (warp == C::WARP_MMA || warp >= C::WARP_ISS1) {
        // ----------------------------------------------------------- MMA issuers
        // One issuer: every block, the run's i-th MMA (K-step k of a 64-K half) accumulating into
        // chain i % NCHAIN (= k % NCHAIN, NCHAIN divides the 4 K-steps of a half). An issuer per
        // decoder group: issuer `iss` takes the CTA's blocks b with b % NISS == iss (the blocks
        // its group decodes, in their A slots b % A_BLOCKS), all into its own chain. A chain's
        // first MMA of the run starts it afresh. Every issuer waits for every x stage in order,
        // so that each of its parity waits is exact.
        const int iss = warp == C::WARP_MMA ? 0 : warp - C::WARP_ISS1 + 1;
        if (lane == 0) {
            int ab = 0;
            uint32_t abph = 0;
            int xs = 0;
            uint32_t xph = 0;
            int b = 0;                         // the CTA's block index
            bool ok = true;
            constexpr uint32_t idesc_full = idesc_bf16_f32(128, BX);
            constexpr uint32_t idesc_half = idesc_bf16_f32(128, BX / 2);
            while (ok && it.next(R, BX)) {
                const uint32_t idesc = R.xrows == BX ? idesc_full : idesc_half;
                if (!mbar_wait(&acc_empty[ab], abph ^ 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_base = tmem_base + C::A_COLS + ab * C::ACC_COLS + (uint32_t)(iss * C::NCHAIN * BX);
                uint32_t started = 0;          // MMAs of this run issued so far by this thread
                for (int g = R.g0; g < R.g1 && ok; ++g) {
                    const int nb = lg.start(g + 1) - lg.start(g);
                    if (!mbar_wait(&x_full[xs], xph)) { ok = false; break; }
                    const uint32_t xbase = sbase + C::OFF_X + xs * C::X_BYTES;
                    for (int jj = 0; jj < nb; ++jj, ++b) {
                        if (C::NISS > 1 && b % C::NISS != iss) continue;
                        const int slot = b % C::A_BLOCKS;
                        // one wait per block: a wait right before an MMA costs the issuing thread
                        // about as much as the MMAs of a narrow block
                        if (!mbar_wait(&a_full[slot], (uint32_t)(b / C::A_BLOCKS) & 1u)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t a_tmem = tmem_base + (uint32_t)((2 * slot + h) * 32);
                            const uint64_t bdesc = smem_desc_sw128(xbase + (2 * jj + h) * C::X_HALF_BYTES);
                            // a fixed count of MMAs and no branch between them (a branch around
                            // tcgen05.mma costs the issuing thread far more than the MMA itself)
#pragma unroll
                            for (int k = 0; k < C::KA / 16; ++k) {
                                umma_bf16_ts(d_base + (uint32_t)((k % C::NCHAIN) * BX), a_tmem + 8 * k, bdesc + 2 * k,
                                             idesc, started >= (uint32_t)C::NCHAIN ? 1u : 0u);
                                ++started;
                            }
                        }
                        umma_commit(&blk_done[C::done_slot(b)]);
                    }
                    if (++xs == C::X_STAGES) { xs = 0; xph ^= 1; }
                }
                if (ok) umma_commit(&acc_full[ab]);
                if (++ab == C::NACC) { ab = 0; abph ^= 1; }
            }
            // every MMA issued by this thread has completed once `drain` flips
            umma_commit(drain);
            (void)mbar_wait(drain, 0);
        }
    } else if (warp < C::WARP_EPI0) {
        // ----------------------------------------------------------- decoders
        // The pair table (only the decoders read it) is built here, while the producers' first
        // copies are in flight: 32 copies of value(b) then 32 copies of spread(b) per entry b.
        opqbits::build_pair_table(sbase + C::OFF_TABLE, warp - C::WARP_DEC0, C::NUM_DEC_WARPS, lane,
                                  (uint32_t)args.lut[lane & 15]);
        // all decoder warps (named barrier 1) see the whole table before decoding
        asm volatile("bar.sync 1, %0;" ::"r"(C::NUM_DEC_WARPS * 32) : "memory");
        pdl_wait();   // the group-wise scales are read from global memory
        const int g_dec = (warp - C::WARP_DEC0) >> 2;    // decoder group
        const int q = warp & 3;                          // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;                   // weight row in the tile = TMEM lane
        const uint32_t lw = 4u * lane, lw2 = 128u + 4u * lane;
        // table lookups by byte offset from the table's shared-memory address (one add per lookup)
        const uint32_t tab = sbase + C::OFF_TABLE;
        auto load = [&](uint32_t off) { return lds_ro_u32(tab + off); };
        // 64-byte swizzle of the codes stage: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
        const uint32_t sw64 = (uint32_t)((row >> 1) & 3);
        const uint32_t tm_row = tmem_base + ((uint32_t)(q * 32) << 16);
        bool ok = true;
        int blk = 0;                 // the CTA's block index
        int u = 0;                   // the CTA's load-group index (= raw stage use)
        // group g_dec decodes the CTA's blocks g_dec, g_dec + GROUPS, ...
        while (ok && it.next(R, BX)) {
            for (int g = R.g0; g < R.g1 && ok; ++g, ++u) {
                const int nb = lg.start(g + 1) - lg.start(g);
                const int rs = u % C::RAW_STAGES;
                const uint32_t rph = (uint32_t)(u / C::RAW_STAGES) & 1u;
                for (int jj = 0; jj < nb; ++jj, ++blk) {
                    if (blk % C::GROUPS != g_dec) continue;
                    if (!warp_wait(&raw_full[rs], rph)) { ok = false; break; }
                    const uint8_t *rawc = smem + C::OFF_RAW + rs * C::RAW_BYTES + jj * C::BLK_CODE_BYTES + row * (C::KR / 2);
                    uint32_t cw[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 vv = *reinterpret_cast<const uint4 *>(rawc + ((((uint32_t)c) ^ sw64) << 4));
                        cw[4 * c] = vv.x; cw[4 * c + 1] = vv.y; cw[4 * c + 2] = vv.z; cw[4 * c + 3] = vv.w;
                    }
                    const uint4 sv = *reinterpret_cast<const uint4 *>(smem + C::OFF_RAW + rs * C::RAW_BYTES +
                                                                     C::RAW_CODE_BYTES + jj * C::BLK_SIGN_BYTES +
                                                                     row * (C::KR / 8));
                    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&raw_empty[rs]);   // the raw words are in registers now
#pragma unroll
                    for (int h = 0; h < C::KR / C::KA; ++h) {     // two 64-K A stages per block
                        const int sidx = blk * 2 + h;
                        const int as = sidx % C::A_STAGES;
                        uint32_t o[2][16];
                        if constexpr (GS == 0) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int w = 8 * h + i;
                                uint32_t t4[4];
                                opqbits::decode8_table(cw[w], sw[w >> 2], (uint32_t)(w & 3), lw, lw2, load, t4);
#pragma unroll
                                for (int e = 0; e < 4; ++e) o[i >> 2][(i & 3) * 4 + e] = t4[e];
                            }
                        } else {
                            // the half's group (two groups of 32 weights when GS = 32), of weight row n
                            const int n = (R.tile / args.m_tiles) * C::BW + row;
                            const int gi = ((lg.start(g) + jj) * C::KR + h * C::KA) / GS;
                            auto gmax_at = [&](int gx) -> float {
                                return n < args.N
                                           ? __half2float(__ushort_as_half(__ldg(args.gmax + (size_t)n * args.ngk + gx)))
                                           : 0.0f;
                            };
                            opqbits::DecodeTable Ta, Tb;
                            make_group_table(Ta, args.lutf, gmax_at(gi));
                            if constexpr (GS == 32) make_group_table(Tb, args.lutf, gmax_at(gi + 1));
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int w = 8 * h + i;
                                uint32_t t4[4];
                                opqbits::decode8(cw[w], (sw[w >> 2] >> (8 * (w & 3))) & 0xFFu,
                                                 (GS == 32 && i >= 4) ? Tb : Ta, t4);
#pragma unroll
                                for (int e = 0; e < 4; ++e) o[i >> 2][(i & 3) * 4 + e] = t4[e];
                            }
                        }
                        // the block's A slot last held block blk - A_BLOCKS
                        const int prev = blk - C::A_BLOCKS;
                        if (h == 0 && prev >= 0 && !warp_wait(&blk_done[C::done_slot(prev)], C::done_parity(prev))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        tmem_st_32x32b_x16(tm_row + as * 32, o[0]);
                        tmem_st_32x32b_x16(tm_row + as * 32 + 16, o[1]);
                        if (h == 1) {   // both halves stored: the block's A tile is complete
                            tmem_st_wait();
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&a_full[blk % C::A_BLOCKS]);
                        }
                    }
                    if (!ok) break;
                }
                if (!ok) break;
            }
        }
    } else {
        // ----------------------------------------------------------- epilogue
        pdl_wait();
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t U = (uint32_t)tiles * (uint32_t)args.ngroups;
        const bool vec_y = (args.N % 8) == 0;
        // per-warp staging for y: 2 buffers of [16 m][32 n] bf16
        const uint32_t stage0 = sbase + C::OFF_EPI + (uint32_t)(warp - C::WARP_EPI0) * 2048u;
        int ab = 0;
        uint32_t abph = 0;
        int sb = 0;
        int bstart = 0;              // the CTA's block index at the run's start
        while (it.next(R, BX)) {
            const int tile = R.tile, r0 = R.r0, r1 = R.r1, j = R.j, xoff = R.xoff, xrows = R.xrows;
            // the accumulator chains that hold this run's sums: all of them with one issuer; with
            // an issuer per decoder group, issuer i's only if the run has one of its blocks
            uint32_t cmask = (1u << C::NCH_ALL) - 1u;
            if (C::NISS > 1) {
                cmask = 0u;
                for (int i = 0; i < C::NISS; ++i)
                    if ((i - bstart % C::NISS + C::NISS) % C::NISS < r1 - r0) cmask |= 1u << i;
            }
            bstart += r1 - r0;
            const int ch0 = __ffs((int)cmask) - 1;
            const int n_blk = tile / args.m_tiles, m_blk = tile % args.m_tiles;
            const int n = n_blk * C::BW + row;
            const int n0 = n_blk * C::BW + q * 32;           // first row of this warp's quarter
            const bool full = (r0 == 0 && r1 == args.kblocks);
            const float scale = GS > 0 ? 1.0f : (n < args.N ? __ldg(args.scales + n) : 0.0f);
            const float bias = bias_at(args.bias, n, args.N);
            // the plain product, or the fused epilogue (bias, activation): chosen per tile, one
            // specialised store loop per kind, so no loop carries another kind's code. The kind is
            // read from the parameters once: inside the loops, every y store could alias them.
            const int act = args.act;
            const bool plain = args.bias == nullptr && act == EPI_NONE;
            auto fv_plain = [scale](float a) { return a * scale; };
            auto fv_bias = [scale, bias](float a) { return epi_value(a, scale, bias, EPI_NONE); };
            auto fv_silu = [scale, bias](float a) { return epi_value(a, scale, bias, EPI_SILU); };
            auto fv_gelu = [scale, bias](float a) { return epi_value(a, scale, bias, EPI_GELU_TANH); };
            if (!warp_wait(&acc_full[ab], abph)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + C::A_COLS + ab * C::ACC_COLS;
            float *wsp = full ? nullptr
                              : args.ws + ((size_t)blockIdx.x * args.runs_max + j) * (size_t)(BX * C::BW);
            const int pcols = min(BX, args.M - m_blk * BX);   // partial sums: columns a run stores
#pragma unroll 1
            for (int c0 = 0; c0 < xrows; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(taddr + ch0 * BX + c0, v);
                if (C::NCH_ALL > 1) {
                    // the chains in a fixed order (warp-uniform skips)
#pragma unroll
                    for (int ch = 1; ch < C::NCH_ALL; ++ch) {
                        if (ch <= ch0 || ((cmask >> ch) & 1u) == 0u) continue;
                        uint32_t u[16];
                        tmem_ld_32x32b_x16(taddr + ch * BX + c0, u);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(u[i]));
                    }
                }
                tmem_ld_wait();
                if (full) {
                    auto store_full = [&](auto &&fv) {
                        const int m0 = m_blk * BX + xoff + c0;
                        if (vec_y && n0 + 32 <= args.N) {
                            // stage [16 m][32 n] bf16, then each lane stores 32 contiguous bytes of one m row
                            const uint32_t sbuf = stage0 + (uint32_t)sb * 1024u;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const __nv_bfloat16 o = __float2bfloat16_rn(fv(__uint_as_float(v[i])));
                                asm volatile("st.shared.u16 [%0], %1;" ::"r"(sbuf + (uint32_t)i * 64u + (uint32_t)lane * 2u),
                                             "h"(*reinterpret_cast<const unsigned short *>(&o)) : "memory");
                            }
                            __syncwarp();
                            const int mi = lane >> 1, hf = lane & 1;
                            if (m0 + mi < args.M) {
                                const uint4 w0 = lds_v4(sbuf + (uint32_t)mi * 64u + (uint32_t)hf * 32u);
                                const uint4 w1 = lds_v4(sbuf + (uint32_t)mi * 64u + (uint32_t)hf * 32u + 16u);
                                uint4 *dst = reinterpret_cast<uint4 *>(args.y + (size_t)(m0 + mi) * args.N + n0 + hf * 16);
                                dst[0] = w0;
                                dst[1] = w1;
                            }
                            sb ^= 1;
                        } else if (n < args.N) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int m = m0 + i;
                                if (m < args.M) {
                                    const __nv_bfloat16 o = __float2bfloat16_rn(fv(__uint_as_float(v[i])));
                                    args.y[(size_t)m * args.N + n] = *reinterpret_cast<const uint16_t *>(&o);
                                }
                            }
                        }
                    };
                    if (plain) store_full(fv_plain);
                    else if (act == EPI_SILU) store_full(fv_silu);
                    else if (act == EPI_GELU_TANH) store_full(fv_gelu);
                    else store_full(fv_bias);
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i)   // the activation rows the fix-up reads (< M)
                        if (c0 + i < pcols) wsp[(size_t)(c0 + i) * C::BW + row] = __uint_as_float(v[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            if (++ab == C::NACC) { ab = 0; abph ^= 1; }
            if (!full) {
                // The last of the tile's CTAs to get here (per lane quarter) adds every
                // CTA's partial rows in CTA order, so the sum does not depend on timing.
                const uint32_t c_lo = unit_owner((uint32_t)tile * (uint32_t)args.ngroups, gridDim.x, U);
                const uint32_t c_hi = unit_owner((uint32_t)(tile + 1) * (uint32_t)args.ngroups - 1u, gridDim.x, U);
                const uint32_t parts = (uint32_t)(c_hi - c_lo + 1);
                // Publication without full fences: the warp's partial stores are ordered before lane
                // 0's release-acquire add by a 32-thread named barrier (ids 2..5, one per warp), and
                // the last arriver's acquire is ordered before every lane's loads by the same barrier.
                asm volatile("bar.sync %0, 32;" ::"r"(2 + q) : "memory");
                uint32_t old = 0;
                if (lane == 0)
                    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                                 : "=r"(old)
                                 : "l"(args.counters + (size_t)tile * 4 + q)
                                 : "memory");
                old = __shfl_sync(0xFFFFFFFFu, old, 0);
                if (old == parts - 1) {
                    asm volatile("bar.sync %0, 32;" ::"r"(2 + q) : "memory");
                    // lane i (< parts) resolves part i's base; bases are broadcast by shuffles
                    const float *mybase = nullptr;
                    if ((uint32_t)lane < parts) {
                        const uint32_t c = c_lo + (uint32_t)lane;
                        const uint32_t jj = (uint32_t)tile - unit_begin(c, gridDim.x, U) / (uint32_t)args.ngroups;
                        mybase = args.ws + ((size_t)c * args.runs_max + (size_t)jj) * (size_t)(BX * C::BW);
                    }
                    // Every lane runs the loops (shuffles need all lanes); only rows < N store.
                    // 8 columns per pass, the next part's 8 loads issued before the current
                    // part's adds; each sum still runs over parts 0, 1, ... from 0.0f.
                    auto part_base = [&](uint32_t p) -> const float * {
                        if (p < 32)
                            return reinterpret_cast<const float *>(
                                __shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(mybase), (int)p));
                        const uint32_t c = c_lo + p;
                        const uint32_t jj = (uint32_t)tile - unit_begin(c, gridDim.x, U) / (uint32_t)args.ngroups;
                        return args.ws + ((size_t)c * args.runs_max + (size_t)jj) * (size_t)(BX * C::BW);
                    };
                    const int mcols = min(BX, args.M - m_blk * BX);
                    for (int c0 = 0; c0 < mcols; c0 += 8) {
                        float acc[8], cur[8], nxt[8];
                        const float *b0 = part_base(0) + (size_t)c0 * C::BW + row;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            acc[i] = 0.0f;
                            cur[i] = (c0 + i < mcols) ? __ldcg(b0 + (size_t)i * C::BW) : 0.0f;
                        }
                        for (uint32_t p = 0; p < parts; ++p) {
                            if (p + 1 < parts) {
                                const float *bn = part_base(p + 1) + (size_t)c0 * C::BW + row;
#pragma unroll
                                for (int i = 0; i < 8; ++i) nxt[i] = (c0 + i < mcols) ? __ldcg(bn + (size_t)i * C::BW) : 0.0f;
                            }
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                acc[i] += cur[i];
                                cur[i] = nxt[i];
                            }
                        }
                        auto store8 = [&](auto &&fv) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                if (c0 + i < mcols) {
                                    const __nv_bfloat16 o = __float2bfloat16_rn(fv(acc[i]));
                                    args.y[(size_t)(m_blk * BX + c0 + i) * args.N + n] = *reinterpret_cast<const uint16_t *>(&o);
                                }
                            }
                        };
                        if (n < args.N) {
                            if (plain) store8(fv_plain);
                            else if (act == EPI_SILU) store8(fv_silu);
                            else if (act == EPI_GELU_TANH) store8(fv_gelu);
                            else store8(fv_bias);
                        }
                    }
                    if (lane == 0) atomicExch(args.counters + (size_t)tile * 4 + q, 0u);   // ready for the next call
                }
            }
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

}  // namespace opqk
