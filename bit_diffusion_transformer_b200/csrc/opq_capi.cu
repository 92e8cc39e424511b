// opq_capi.cu — the C ABI of libopq.so (declared in include/opq.h): argument
// validation, the alpha-dependent tables, TMA descriptors, kernel selection and
// launches. The whole library is this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "opq.h"
#include "opq_dequantize.cuh"
#include "opq_grouped.cuh"
#include "opq_linear.cuh"
#include "opq_linear_wide.cuh"
#include "opq_quantize.cuh"
#include "opq_quantize_stream.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

constexpr int kPlanSMs = 148;   // B200 SM count; the split-K plan is fixed by shape alone

opq_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = (int)e;
    return OPQ_ERR_CUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tensor pointers: all non-null and 16-byte aligned first, then each must be
// device-accessible memory (device or managed), so that the cheapest argument
// error is reported regardless of pointer order.
opq_status check_ptrs(std::initializer_list<const void *> ptrs) {
    for (const void *p : ptrs)
        if (p == nullptr) return OPQ_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p)) return OPQ_ERR_MISALIGNED;
    for (const void *p : ptrs) {
        cudaPointerAttributes attr;
        cudaError_t e = cudaPointerGetAttributes(&attr, p);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return OPQ_ERR_NOT_DEVICE_MEMORY;
        }
        if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return OPQ_ERR_NOT_DEVICE_MEMORY;
    }
    return OPQ_OK;
}

bool alpha_ok(float alpha) { return std::isfinite(alpha) && alpha > 0.0f; }

// fp64 -> bf16 bits, round to nearest even, for the small decode table (host).
// The value is first truncated to fp32 with a sticky last bit when inexact
// (round to odd), then rounded to bf16 on the bit pattern.
uint16_t host_bf16(double v) {
    float t = (float)v;
    if (std::fabs((double)t) > std::fabs(v)) t = std::nextafter(t, 0.0f);   // truncate toward zero
    uint32_t b;
    std::memcpy(&b, &t, 4);
    if ((double)t != v) b |= 1u;
    return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

struct DeviceInfo {
    int sms = 0;
    bool stream_quant_attr[3][4] = {};   // dynamic shared memory raised for quantize_stream_kernel<G, BITS>
    bool stream_quant_stab_attr = false; // and for its shared-mantissa-table variant
    // dynamic shared memory raised, per [group size index: 0 per-row, 1..4 GS 32..256][kernel: BX 16, 32,
    // 64, 128, wide]
    bool linear_attr[5][5] = {};
    bool bits_attr[3] = {};           // the wide kernel at 3, 5 and 6 bits
};
std::mutex g_mu;
DeviceInfo g_dev[64];

opq_status device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return OPQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (d.sms == 0) {
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    *out = &d;
    return OPQ_OK;
}

// --------------------------------------------------------------- TMA maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

// bf16 [rows, K] row-major, box {64 columns, box_rows}, 128-byte swizzle, zero fill out of bounds.
opq_status make_x_map(CUtensorMap *map, const void *x, int64_t rows, int64_t K, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return OPQ_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        t_last_cuda_error = (int)r;
        return OPQ_ERR_CUDA;
    }
    return OPQ_OK;
}

// bf16 (q/15)^(1/alpha) for q = 0..15 (the decoded magnitudes before the row scale)
void lut_bf16(float alpha, uint16_t (&lut)[16]) {
    const double inv = 1.0 / (double)alpha;
    for (int q = 0; q < 16; ++q) lut[q] = host_bf16(std::pow((double)q / 15.0, inv));
}

// uint32 plane [rows, words] row-major, box {box_words, box_rows}, zero fill. With the
// 64-byte swizzle (box rows of 64 bytes) 16-byte chunk c of row r lands at c ^ ((r >> 1) & 3).
// uint32 plane [rows, words_per_row] viewed as 3-D {w (words within a 128-K block), rows, blocks}:
// box {w, box_rows, box_blocks} lands as box_blocks consecutive [box_rows][w] images. Needs
// words_per_row == w * blocks (K % 128 == 0) and 16-byte rows.
opq_status make_u32_block_map(CUtensorMap *map, const void *p, int64_t rows, uint32_t w, int64_t blocks,
                              uint32_t box_rows, uint32_t box_blocks, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return OPQ_ERR_CUDA;
    cuuint64_t dims[3] = {(cuuint64_t)w, (cuuint64_t)rows, (cuuint64_t)blocks};
    cuuint64_t strides[2] = {(cuuint64_t)w * (cuuint64_t)blocks * 4u, (cuuint64_t)w * 4u};
    cuuint32_t box[3] = {w, box_rows, box_blocks};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(p), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        t_last_cuda_error = (int)r;
        return OPQ_ERR_CUDA;
    }
    return OPQ_OK;
}

// x [rows, K] bf16 viewed as 3-D {64 (K within a 64-K chunk), rows, K / 64}, box {64, box_rows,
// chunks}, 128-byte swizzle: the chunks land one after the other (needs K % 64 == 0).
opq_status make_x_chunk_map(CUtensorMap *map, const void *x, int64_t rows, int64_t K, uint32_t box_rows,
                            uint32_t chunks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return OPQ_ERR_CUDA;
    cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(K / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)K * 2u, 128u};
    cuuint32_t box[3] = {64u, box_rows, chunks};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(x), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        t_last_cuda_error = (int)r;
        return OPQ_ERR_CUDA;
    }
    return OPQ_OK;
}

opq_status make_u32_map(CUtensorMap *map, const void *p, int64_t rows, int64_t words, uint32_t box_words,
                        uint32_t box_rows, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return OPQ_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)words * 4};
    cuuint32_t box[2] = {box_words, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(p), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        t_last_cuda_error = (int)r;
        return OPQ_ERR_CUDA;
    }
    return OPQ_OK;
}

struct Plan {
    int mode;       // 0 whole tiles, 1 stream-K with a fixed-order fix-up
    int bx;         // activation rows per tile (the MMA N)
    int m_tiles, n_tiles, kblocks;
    int grp;        // 128-K blocks per load group of the chosen tile width
    int ngroups;    // load groups per tile
    int grid;       // CTAs of the linear kernel
    int runs_max;   // mode 1
    int tail_split; // mode 0: 2 = the tiles past the last whole wave run as two half-width runs
    size_t counter_bytes;   // mode 1: the zero-between-calls arrival counters at the workspace start
    size_t ws_bytes;
    int launches;
    bool unsupported;   // a shape no schedule serves: OPQ_ERR_UNSUPPORTED_SHAPE
};

// The schedule depends on the shape alone (a fixed 148-CTA budget), so the
// workspace size and the result bits are the same on every B200.
// Arrival counters occupy a fixed region at the start of every workspace (stream-K: 4 per
// weight tile, at most kCounterTiles tiles; the half-K tail of the wide schedule: 8 per tail
// tile, at most 74 tail tiles), so that no shape's partial sums ever land on counters another
// shape relies on being zero.
constexpr int kCounterTiles = 4096;
constexpr size_t kCounterBytes = (size_t)kCounterTiles * 4u * sizeof(uint32_t);   // 64 KiB
// the half-K tail needs this many 128-K blocks to beat splitting the activation rows
constexpr int kKSplitMinBlocks = 8;

// `wide`: 256-row tiles for every M (the group-wise format has only the wide kernel)
Plan make_plan(int64_t M, int64_t N, int64_t K, bool wide = false) {
    Plan p{};
    p.kblocks = (int)((K + 127) / 128);
    p.n_tiles = (int)((N + 127) / 128);
    if (M <= 128 && !wide) {
        p.bx = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
        // the narrow tiles fetch several 128-K blocks per copy through 3-D views of the planes,
        // which need whole blocks (K % 128 == 0); other K take the one-block-per-copy width
        if (K % 128 != 0) p.bx = 128;
        p.m_tiles = 1;
    } else {
        p.bx = 256;
        p.m_tiles = (int)((M + 255) / 256);
    }
    // blocks per load group: must match the kernel's Cfg<BX>::GRP
    p.grp = p.bx <= 16 ? 4 : (p.bx <= 64 ? 2 : 1);
    p.ngroups = (p.kblocks + p.grp - 1) / p.grp;
    // stream-K (the kernel deals units in 32-bit arithmetic: units x CTAs below 2^31)
    const bool stream_k = M <= 128 && !wide && p.n_tiles <= kCounterTiles &&
                          (int64_t)p.n_tiles * p.ngroups * kPlanSMs < ((int64_t)1 << 31);
    // whole narrow tiles (past stream-K's range) only for whole 128-K blocks: with the sign
    // words copied by cp.async, max-size tests of that schedule faulted (narrow tiles) or
    // returned wrong sums for a few tiles (256-row tiles at M = 8); the entry points refuse it
    p.unsupported = M <= 128 && !wide && !stream_k && K % 128 != 0;
    if (stream_k) {
        p.mode = 1;
        const int64_t U = (int64_t)p.n_tiles * p.ngroups;
        p.grid = (int)(U < kPlanSMs ? U : kPlanSMs);
        const int64_t per = (U + p.grid - 1) / p.grid;
        p.runs_max = (int)((per + p.ngroups - 1) / p.ngroups + 1);
        p.counter_bytes = kCounterBytes;
        p.ws_bytes = p.counter_bytes + (size_t)p.grid * (size_t)p.runs_max * (size_t)p.bx * 128u * sizeof(float);
    } else {
        p.mode = 0;
        const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
        p.grid = (int)(tiles < kPlanSMs ? tiles : kPlanSMs);
        p.runs_max = 1;
        // tiles left after the whole waves: when there are at most half as many as CTAs, each
        // is split over two CTAs, so that the last wave takes about half a tile's time instead
        // of a whole one. 256-row tiles with at least 8 blocks split K (each CTA decodes half
        // the tile's weights; the two fp32 partial sums meet in the workspace); otherwise the
        // activation rows are split (each CTA decodes all of them for half the rows)
        const int64_t tail = tiles - (tiles / p.grid) * p.grid;
        p.tail_split = 1;
        p.counter_bytes = 0;
        p.ws_bytes = 0;
        if (tail > 0 && 2 * tail <= p.grid) {
            if (p.bx == 256 && p.kblocks >= kKSplitMinBlocks) {
                p.tail_split = 3;
                p.counter_bytes = kCounterBytes;
                p.ws_bytes = p.counter_bytes + (size_t)tail * 256u * 128u * sizeof(float);
            } else if (p.bx >= 32 && p.grp == 1) {
                // half-width runs load their activation rows with a 2-D half-height box, so
                // only tiles that fetch one block per copy take them
                p.tail_split = 2;
            }
        }
    }
    p.launches = 1;
    return p;
}

opq_status check_sizes(int64_t N, int64_t K) {
    if (N < 1 || K < 1) return OPQ_ERR_INVALID_ARG;
    if (K % 32 != 0) return OPQ_ERR_UNSUPPORTED_SHAPE;
    if (N > INT32_MAX || K > INT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    return OPQ_OK;
}

constexpr int gs_index(int gs) { return gs == 0 ? 0 : gs == 32 ? 1 : gs == 64 ? 2 : gs == 128 ? 3 : 4; }

// A linear kernel launch that lets the next programmatically launched kernel of the stream start
// its global-memory-free set-up while this one finishes (the kernels wait for their predecessor
// before touching global memory: opq_device.cuh, pdl_wait).
template <class Kern, class... Args>
cudaError_t launch_programmatic(Kern kernel, int grid, int threads, int smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int BX, int GS>
cudaError_t launch_linear(DeviceInfo *di, const Plan &plan, const CUtensorMap &xmap, const CUtensorMap &xhmap,
                          const CUtensorMap &cmap, const CUtensorMap &smap, const opqk::LinearArgs &a,
                          cudaStream_t st) {
    using C = opqk::Cfg<BX>;
    // half-width runs exist only for one block per copy (2-D x boxes); the plan never asks for
    // them otherwise, and a launch that did is refused here
    if (a.tail_split == 2 && C::GRP != 1) return cudaErrorInvalidConfiguration;
    // whole-tile schedules of the narrow kernel only for whole 128-K blocks (signs by TMA)
    if (a.mode == 0 && a.signs_tma == 0) return cudaErrorInvalidConfiguration;
    const int key = BX == 16 ? 0 : BX == 32 ? 1 : BX == 64 ? 2 : 3;
    if (!di->linear_attr[gs_index(GS)][key]) {
        cudaError_t e = cudaFuncSetAttribute(opqk::linear_kernel<BX, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        di->linear_attr[gs_index(GS)][key] = true;
    }
    cudaError_t e = launch_programmatic(opqk::linear_kernel<BX, GS>, plan.grid, C::THREADS, C::SMEM_BYTES, st, xmap,
                                        xhmap, cmap, smap, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// the wide-tile kernel (256 activation rows per tile, whole tiles, one block per copy)
template <int GS, int BITS = 4>
cudaError_t launch_linear_wide(DeviceInfo *di, const Plan &plan, const CUtensorMap &xmap, const CUtensorMap &xhmap,
                               const CUtensorMap &cmap, const CUtensorMap &smap, const opqk::LinearArgs &n,
                               cudaStream_t st) {
    using C = opqk_wide::Cfg<256, BITS>;
    if (plan.mode != 0) return cudaErrorInvalidValue;   // the wide kernel runs whole-tile schedules only
    opqk_wide::LinearArgs a{};
    a.signs = n.signs;
    a.scales = n.scales;
    a.y = n.y;
    a.ws = n.ws;
    a.counters = n.counters;
    a.signs_tma = n.signs_tma;
    a.M = n.M;
    a.N = n.N;
    a.K = n.K;
    a.m_tiles = n.m_tiles;
    a.n_tiles = n.n_tiles;
    a.kblocks = n.kblocks;
    a.mode = n.mode;
    a.tail_split = n.tail_split;
    for (int i = 0; i < 16; ++i) a.lut[i] = n.lut[i];
    a.gmax = n.gmax;
    a.ngk = n.ngk;
    a.bias = n.bias;
    a.act = n.act;
    for (int q = 0; q < 16; ++q) a.lutf[q] = n.lutf[q];
    for (int q = 0; q < 64; ++q) a.lutb[q] = n.lutb[q];
    bool &attr = BITS == 4 ? di->linear_attr[gs_index(GS)][4] : di->bits_attr[BITS == 3 ? 0 : BITS - 4];
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(opqk_wide::wide_kernel<256, GS, BITS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (C::REG_SPLIT) {
            // the kernel's warpgroups trade registers (setmaxnreg) on the assumption that each
            // thread was launched with REG_LAUNCH of them; any other count is refused, not run
            cudaFuncAttributes fa{};
            if ((e = cudaFuncGetAttributes(&fa, opqk_wide::wide_kernel<256, GS, BITS>)) != cudaSuccess) return e;
            if (fa.numRegs != C::REG_LAUNCH) return cudaErrorInvalidConfiguration;
        }
        attr = true;
    }
    cudaError_t e = launch_programmatic(opqk_wide::wide_kernel<256, GS, BITS>, plan.grid, C::THREADS, C::SMEM_BYTES, st,
                                        xmap, xhmap, cmap, smap, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

extern "C" {

int opq_abi_version(void) { return 1; }

int opq_last_cuda_error(void) { return t_last_cuda_error; }

const char *opq_status_string(opq_status s) {
    switch (s) {
        case OPQ_OK: return "OPQ_OK";
        case OPQ_ERR_INVALID_ARG: return "OPQ_ERR_INVALID_ARG";
        case OPQ_ERR_UNSUPPORTED_SHAPE: return "OPQ_ERR_UNSUPPORTED_SHAPE";
        case OPQ_ERR_MISALIGNED: return "OPQ_ERR_MISALIGNED";
        case OPQ_ERR_WORKSPACE: return "OPQ_ERR_WORKSPACE";
        case OPQ_ERR_CUDA: return "OPQ_ERR_CUDA";
        case OPQ_ERR_NOT_DEVICE_MEMORY: return "OPQ_ERR_NOT_DEVICE_MEMORY";
    }
    return "OPQ_ERR_UNKNOWN";
}

// The row-streaming quantize over a list of matrices: validation, then one launch per row-width
// class (one, four or eight warps per row) and per QS_MAX_JOBS matrices of the class. One-warp
// rows at 4 bits use the shared mantissa tables (STAB) when the launch gives each CTA hundreds of
// rows and the 128 tables fit in shared memory beside a ring of at least 8 rows: each table holds at most dz + 1 <= 128 log2(1/t_1) + 131
// entries (t_1 = (1/30)^(1/alpha); the 128 accounts for the max's mantissa), which caps it
// for alpha >= ~0.7; the kernel itself checks every table against its stride.
extern "C++" {
template <int G, int BITS, bool STAB>
static opq_status launch_quant_stream_v(DeviceInfo *di, const opq_quant_job *jobs, const std::vector<int64_t> &idx,
                                        const opqk::QuantParams &qp, const double *tl, int slot_bytes, int stab_bytes,
                                        int stab_stride, cudaStream_t st) {
    using C = opqk::QsCfg<G, STAB>;
    int nslots = (C::RING_MAX - stab_bytes) / slot_bytes;
    if (nslots > opqk::QS_MAX_SLOTS) nslots = opqk::QS_MAX_SLOTS;
    if (nslots < 2) return OPQ_ERR_UNSUPPORTED_SHAPE;
    const int smem = opqk::QS_OFF_RING + stab_bytes + nslots * slot_bytes;
    const int gi = G == 1 ? 0 : (G == 4 ? 1 : 2);
    bool &attr = STAB ? di->stream_quant_stab_attr : di->stream_quant_attr[gi][BITS - 3];
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(opqk::quantize_stream_kernel<G, BITS, STAB>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             opqk::QS_OFF_RING + C::RING_MAX);
        if (e != cudaSuccess) return cuda_fail(e);
        attr = true;
    }
    static thread_local opqk::QsParams P;   // ~7 KB: kept off the stack
    for (size_t c0 = 0; c0 < idx.size(); c0 += opqk::QS_MAX_JOBS) {
        std::memset(&P, 0, sizeof P);
        P.qp = qp;
        for (int k = 0; k < 64; ++k) P.tl[k] = tl[k];
        P.nslots = nslots;
        P.slot_bytes = slot_bytes;
        P.stab_bytes = stab_bytes;
        P.stab_stride = stab_stride;
        const size_t n = idx.size() - c0 < (size_t)opqk::QS_MAX_JOBS ? idx.size() - c0 : (size_t)opqk::QS_MAX_JOBS;
        int64_t rows = 0;
        for (size_t i = 0; i < n; ++i) {
            const opq_quant_job &J = jobs[idx[c0 + i]];
            opqk::QsJob &q = P.job[i];
            q.w = J.w;
            q.codes = J.codes;
            q.signs = J.signs;
            q.scales = J.scales;
            q.ldw = J.ldw;
            q.N = (int32_t)J.N;
            q.K = (int32_t)J.K;
            q.row_begin = rows;
            rows += J.N;
        }
        P.njobs = (int32_t)n;
        P.rows = rows;
        const int64_t groups = rows < (int64_t)di->sms * C::NG ? rows : (int64_t)di->sms * C::NG;
        const int grid = (int)((groups + C::NG - 1) / C::NG);
        opqk::quantize_stream_kernel<G, BITS, STAB><<<grid, opqk::QS_THREADS, smem, st>>>(P);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return OPQ_OK;
}

template <int G, int BITS>
static opq_status launch_quant_stream(DeviceInfo *di, const opq_quant_job *jobs, const std::vector<int64_t> &idx,
                                      const opqk::QuantParams &qp, const double *tl, cudaStream_t st) {
    int64_t kmax = 0;
    for (int64_t i : idx) kmax = jobs[i].K > kmax ? jobs[i].K : kmax;
    // one slot holds one row of the widest matrix of the class
    const int slot_bytes = (int)((2 * kmax + 127) / 128 * 128);
    int64_t rows = 0;
    for (int64_t i : idx) rows += jobs[i].N;
    // building the 128 tables costs a CTA about as much as building its own for 128 rows, so the
    // shared tables serve launches that give every CTA many more rows than that (a whole model)
    if constexpr (G == 1 && BITS == 4) if (rows >= 512 * (int64_t)di->sms) {
        const double t1 = qp.alpha_is_one ? 1.0 / 30.0 : qp.t[1];
        const double dz_bound = std::ceil(-128.0 * std::log2(t1)) + 131.0;
        const int stride = (int)((dz_bound + 4.0) / 16.0 + 1.0) * 16;   // >= 4 ((dz + 4) / 4) for dz <= dz_bound
        const int stab_bytes = (256 + 128 * stride + 127) / 128 * 128;
        using CS = opqk::QsCfg<1, true>;
        if (stab_bytes <= 136 * 1024 && (CS::RING_MAX - stab_bytes) / slot_bytes >= 8)
            return launch_quant_stream_v<1, 4, true>(di, jobs, idx, qp, tl, slot_bytes, stab_bytes, stride, st);
    }
    return launch_quant_stream_v<G, BITS, false>(di, jobs, idx, qp, tl, slot_bytes, 0, 0, st);
}

template <int BITS>
static opq_status launch_quant_classes(DeviceInfo *di, const opq_quant_job *jobs, const std::vector<int64_t> (&cls)[3],
                                       const opqk::QuantParams &qp, const double *tl, cudaStream_t st) {
    opq_status s = OPQ_OK;
    if (!cls[0].empty() && (s = launch_quant_stream<1, BITS>(di, jobs, cls[0], qp, tl, st)) != OPQ_OK) return s;
    if (!cls[1].empty() && (s = launch_quant_stream<4, BITS>(di, jobs, cls[1], qp, tl, st)) != OPQ_OK) return s;
    if (!cls[2].empty() && (s = launch_quant_stream<8, BITS>(di, jobs, cls[2], qp, tl, st)) != OPQ_OK) return s;
    return OPQ_OK;
}
}  // extern "C++"

// `bits` bits per magnitude code (4: the card's nibble format; 3, 5, 6: per-row bit streams)
static opq_status quantize_jobs(const opq_quant_job *jobs, int64_t count, float alpha, void *stream, int bits = 4) {
    if (jobs == nullptr || count < 1) return OPQ_ERR_INVALID_ARG;
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    for (int64_t i = 0; i < count; ++i) {
        const opq_quant_job &J = jobs[i];
        opq_status s = check_sizes(J.N, J.K);
        if (s != OPQ_OK) return s;
        if (J.K > 32768) return OPQ_ERR_UNSUPPORTED_SHAPE;
        if (J.ldw < J.K || J.ldw % 8 != 0) return OPQ_ERR_INVALID_ARG;
    }
    for (int64_t i = 0; i < count; ++i) {
        opq_status s = check_ptrs({jobs[i].w, jobs[i].codes, jobs[i].signs, jobs[i].scales});
        if (s != OPQ_OK) return s;
    }
    DeviceInfo *di = nullptr;
    opq_status s = device_info(&di);
    if (s != OPQ_OK) return s;
    opqk::QuantParams qp{};
    const double inv = 1.0 / (double)alpha;
    for (int k = 1; k < 16; ++k) qp.t[k] = std::pow(((double)k - 0.5) / 15.0, inv);
    qp.alpha_is_one = (alpha == 1.0f) ? 1 : 0;
    double tl[64] = {};
    const int L = (1 << bits) - 1;
    for (int k = 1; k <= L; ++k) tl[k] = std::pow(((double)k - 0.5) / (double)L, inv);
    std::vector<int64_t> cls[3];
    for (int64_t i = 0; i < count; ++i) {
        const int g = opqk::qs_group_warps(jobs[i].K);
        cls[g == 1 ? 0 : (g == 4 ? 1 : 2)].push_back(i);
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (bits) {
        case 3: return launch_quant_classes<3>(di, jobs, cls, qp, tl, st);
        case 5: return launch_quant_classes<5>(di, jobs, cls, qp, tl, st);
        case 6: return launch_quant_classes<6>(di, jobs, cls, qp, tl, st);
        default: return launch_quant_classes<4>(di, jobs, cls, qp, tl, st);
    }
}

// group-wise format: group size 32, 64, 128 or 256 dividing K
static opq_status check_group(int64_t K, int64_t gs) {
    if (gs != 32 && gs != 64 && gs != 128 && gs != 256) return OPQ_ERR_INVALID_ARG;
    if (K % gs != 0) return OPQ_ERR_UNSUPPORTED_SHAPE;
    return OPQ_OK;
}

opq_status opq_quantize_batched(const opq_quant_job *jobs, int64_t count, float alpha, void *stream) {
    return quantize_jobs(jobs, count, alpha, stream);
}

opq_status opq_quantize(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, float alpha, uint32_t *codes,
                        uint32_t *signs, float *scales, void *stream) {
    const opq_quant_job job = {w, N, K, ldw, codes, signs, scales};
    return quantize_jobs(&job, 1, alpha, stream);
}

opq_status opq_quantize_grouped(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t group_size,
                                float alpha, uint32_t *codes, uint32_t *signs, uint16_t *gmax, void *stream) {
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if ((s = check_group(K, group_size)) != OPQ_OK) return s;
    if (ldw < K || ldw % 8 != 0) return OPQ_ERR_INVALID_ARG;
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    if ((s = check_ptrs({w, codes, signs, gmax})) != OPQ_OK) return s;
    opqk::QuantParams qp{};
    const double inv = 1.0 / (double)alpha;
    qp.t[0] = 0.0;
    for (int k = 1; k < 16; ++k) qp.t[k] = std::pow(((double)k - 0.5) / 15.0, inv);
    qp.alpha_is_one = (alpha == 1.0f) ? 1 : 0;
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != OPQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // one warp per row, 8 rows per block
    const int64_t blocks = (N + 7) / 8;
    const int grid = (int)(blocks < (int64_t)di->sms * 8 ? blocks : (int64_t)di->sms * 8);
    switch (group_size) {
        case 32: opqk::quantize_grouped_kernel<32><<<grid, 256, 0, st>>>(w, N, K, ldw, qp, codes, signs, gmax); break;
        case 64: opqk::quantize_grouped_kernel<64><<<grid, 256, 0, st>>>(w, N, K, ldw, qp, codes, signs, gmax); break;
        case 128: opqk::quantize_grouped_kernel<128><<<grid, 256, 0, st>>>(w, N, K, ldw, qp, codes, signs, gmax); break;
        default: opqk::quantize_grouped_kernel<256><<<grid, 256, 0, st>>>(w, N, K, ldw, qp, codes, signs, gmax); break;
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? OPQ_OK : cuda_fail(e);
}

opq_status opq_dequantize_grouped(const uint32_t *codes, const uint32_t *signs, const uint16_t *gmax, int64_t N,
                                  int64_t K, int64_t group_size, float alpha, uint16_t *w_out, void *stream) {
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if ((s = check_group(K, group_size)) != OPQ_OK) return s;
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    if ((uint64_t)N * (uint64_t)(K / 8) >= (1ull << 40)) return OPQ_ERR_UNSUPPORTED_SHAPE;
    if ((s = check_ptrs({codes, signs, gmax, w_out})) != OPQ_OK) return s;
    opqk::DequantParams dp{};
    const double inv = 1.0 / (double)alpha;
    for (int q = 0; q < 16; ++q) dp.lut[q] = std::pow((double)q / 15.0, inv);
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != OPQ_OK) return s;
    uint64_t blocks = ((uint64_t)N + 7) / 8;
    const uint64_t cap = (uint64_t)di->sms * 16;
    if (blocks > cap) blocks = cap;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint32_t rows = (uint32_t)N, chunks = (uint32_t)(K / 32);
    switch (group_size) {
        case 32: opqk::dequantize_grouped_kernel<32><<<(int)blocks, 256, 0, st>>>(codes, signs, gmax, rows, chunks, dp, w_out); break;
        case 64: opqk::dequantize_grouped_kernel<64><<<(int)blocks, 256, 0, st>>>(codes, signs, gmax, rows, chunks, dp, w_out); break;
        case 128: opqk::dequantize_grouped_kernel<128><<<(int)blocks, 256, 0, st>>>(codes, signs, gmax, rows, chunks, dp, w_out); break;
        default: opqk::dequantize_grouped_kernel<256><<<(int)blocks, 256, 0, st>>>(codes, signs, gmax, rows, chunks, dp, w_out); break;
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? OPQ_OK : cuda_fail(e);
}

opq_status opq_quantize_bits(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int32_t bits, float alpha,
                             uint32_t *codes, uint32_t *signs, float *scales, void *stream) {
    if (bits < 3 || bits > 6) return OPQ_ERR_INVALID_ARG;
    const opq_quant_job job = {w, N, K, ldw, codes, signs, scales};
    return quantize_jobs(&job, 1, alpha, stream, bits);
}

opq_status opq_dequantize_bits(const uint32_t *codes, const uint32_t *signs, const float *scales, int64_t N, int64_t K,
                               int32_t bits, float alpha, uint16_t *w_out, void *stream) {
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if (bits < 3 || bits > 6) return OPQ_ERR_INVALID_ARG;
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    if ((uint64_t)N * (uint64_t)(K / 8) >= (1ull << 40)) return OPQ_ERR_UNSUPPORTED_SHAPE;
    if ((s = check_ptrs({codes, signs, scales, w_out})) != OPQ_OK) return s;
    const int L = (1 << bits) - 1;
    opqk::BitsDequantParams dp{};
    const double inv = 1.0 / (double)alpha;
    for (int q = 0; q <= L; ++q) dp.lut[q] = std::pow((double)q / (double)L, inv);
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != OPQ_OK) return s;
    uint64_t blocks = ((uint64_t)N + 7) / 8;
    const uint64_t cap = (uint64_t)di->sms * 16;
    if (blocks > cap) blocks = cap;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const uint32_t rows = (uint32_t)N, chunks = (uint32_t)(K / 32);
    switch (bits) {
        case 3: opqk::dequantize_bits_kernel<3><<<(int)blocks, 256, 0, st>>>(codes, signs, scales, rows, chunks, dp, w_out); break;
        case 4: opqk::dequantize_bits_kernel<4><<<(int)blocks, 256, 0, st>>>(codes, signs, scales, rows, chunks, dp, w_out); break;
        case 5: opqk::dequantize_bits_kernel<5><<<(int)blocks, 256, 0, st>>>(codes, signs, scales, rows, chunks, dp, w_out); break;
        default: opqk::dequantize_bits_kernel<6><<<(int)blocks, 256, 0, st>>>(codes, signs, scales, rows, chunks, dp, w_out); break;
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? OPQ_OK : cuda_fail(e);
}

opq_status opq_alpha_search_workspace_size(int64_t N, size_t *bytes) {
    if (!bytes || N < 1 || N > INT32_MAX) return OPQ_ERR_INVALID_ARG;
    *bytes = (size_t)N * 2u * sizeof(double);
    return OPQ_OK;
}

opq_status opq_alpha_search(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t group_size,
                            const float *alphas, int32_t count, double *snr_db, float *best_alpha, void *workspace,
                            size_t workspace_bytes, void *stream) {
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if (group_size != 0 && (s = check_group(K, group_size)) != OPQ_OK) return s;
    if (ldw < K || ldw % 8 != 0) return OPQ_ERR_INVALID_ARG;
    if (!alphas || !snr_db || !best_alpha || count < 1) return OPQ_ERR_INVALID_ARG;
    for (int32_t i = 0; i < count; ++i)
        if (!alpha_ok(alphas[i])) return OPQ_ERR_INVALID_ARG;
    if ((s = check_ptrs({w})) != OPQ_OK) return s;
    if (!workspace || workspace_bytes < (size_t)N * 2u * sizeof(double)) return OPQ_ERR_WORKSPACE;
    if ((s = check_ptrs({workspace})) != OPQ_OK) return s;
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != OPQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    double *err = reinterpret_cast<double *>(workspace);
    double *sig = err + N;
    std::vector<double> h((size_t)N * 2u);
    const int64_t blocks = (N + 7) / 8;
    const int grid = (int)(blocks < (int64_t)di->sms * 8 ? blocks : (int64_t)di->sms * 8);
    int best = 0;
    for (int32_t i = 0; i < count; ++i) {
        const float alpha = alphas[i];
        opqk::ErrorParams ep{};
        const double inv = 1.0 / (double)alpha;
        ep.qp.t[0] = 0.0;
        for (int k = 1; k < 16; ++k) ep.qp.t[k] = std::pow(((double)k - 0.5) / 15.0, inv);
        ep.qp.alpha_is_one = (alpha == 1.0f) ? 1 : 0;
        for (int q = 0; q < 16; ++q) ep.lutf[q] = (float)std::pow((double)q / 15.0, inv);
        switch (group_size) {
            case 0: opqk::quant_error_kernel<0><<<grid, 256, 0, st>>>(w, N, K, ldw, ep, err, sig); break;
            case 32: opqk::quant_error_kernel<32><<<grid, 256, 0, st>>>(w, N, K, ldw, ep, err, sig); break;
            case 64: opqk::quant_error_kernel<64><<<grid, 256, 0, st>>>(w, N, K, ldw, ep, err, sig); break;
            case 128: opqk::quant_error_kernel<128><<<grid, 256, 0, st>>>(w, N, K, ldw, ep, err, sig); break;
            default: opqk::quant_error_kernel<256><<<grid, 256, 0, st>>>(w, N, K, ldw, ep, err, sig); break;
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaMemcpyAsync(h.data(), err, (size_t)N * 2u * sizeof(double), cudaMemcpyDeviceToHost, st);
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e);
        double es = 0.0, ss = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            es += h[(size_t)n];
            ss += h[(size_t)(N + n)];
        }
        snr_db[i] = es == 0.0 ? HUGE_VAL : 10.0 * std::log10(ss / es);
        if (snr_db[i] > snr_db[best]) best = i;
    }
    *best_alpha = alphas[best];
    return OPQ_OK;
}

// The dequantize over a list of matrices: validation of every descriptor first, then one launch
// per DQ_MAX_JOBS matrices (one warp per row, four rows per block, at most 32 blocks per SM).
static opq_status dequantize_jobs(const opq_dequant_job *jobs, int64_t count, float alpha, void *stream) {
    if (jobs == nullptr || count < 1) return OPQ_ERR_INVALID_ARG;
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    for (int64_t i = 0; i < count; ++i) {
        const opq_dequant_job &J = jobs[i];
        opq_status s = check_sizes(J.N, J.K);
        if (s != OPQ_OK) return s;
        if ((uint64_t)J.N * (uint64_t)(J.K / 8) >= (1ull << 40) || J.N > UINT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    }
    for (int64_t i = 0; i < count; ++i) {
        opq_status s = check_ptrs({jobs[i].codes, jobs[i].signs, jobs[i].scales, jobs[i].w_out});
        if (s != OPQ_OK) return s;
    }
    DeviceInfo *di = nullptr;
    opq_status s = device_info(&di);
    if (s != OPQ_OK) return s;
    static thread_local opqk::DqParams P;   // ~6 KB: kept off the stack
    const double inv = 1.0 / (double)alpha;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int64_t c0 = 0; c0 < count; c0 += opqk::DQ_MAX_JOBS) {
        std::memset(&P, 0, sizeof P);
        for (int q = 0; q < 16; ++q) P.dp.lut[q] = std::pow((double)q / 15.0, inv);
        const int64_t n = count - c0 < opqk::DQ_MAX_JOBS ? count - c0 : opqk::DQ_MAX_JOBS;
        int64_t rows = 0;
        for (int64_t i = 0; i < n; ++i) {
            const opq_dequant_job &J = jobs[c0 + i];
            opqk::DqJob &q = P.job[i];
            q.codes = J.codes;
            q.signs = J.signs;
            q.scales = J.scales;
            q.out = J.w_out;
            q.row_begin = rows;
            q.N = (uint32_t)J.N;
            q.chunks = (uint32_t)(J.K / 32);
            rows += J.N;
        }
        P.njobs = (int32_t)n;
        P.rows = rows;
        uint64_t blocks = ((uint64_t)rows + 3) / 4;
        const uint64_t cap = (uint64_t)di->sms * 32;
        if (blocks > cap) blocks = cap;
        opqk::dequantize_kernel<<<(int)blocks, 128, 0, st>>>(P);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return OPQ_OK;
}

opq_status opq_dequantize(const uint32_t *codes, const uint32_t *signs, const float *scales, int64_t N, int64_t K,
                          float alpha, uint16_t *w_out, void *stream) {
    const opq_dequant_job job = {codes, signs, scales, N, K, w_out};
    return dequantize_jobs(&job, 1, alpha, stream);
}

opq_status opq_dequantize_batched(const opq_dequant_job *jobs, int64_t count, float alpha, void *stream) {
    return dequantize_jobs(jobs, count, alpha, stream);
}

opq_status opq_linear_workspace_size(int64_t M, int64_t N, int64_t K, size_t *bytes) {
    if (!bytes) return OPQ_ERR_INVALID_ARG;
    if (M < 1) return OPQ_ERR_INVALID_ARG;
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if (M > INT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    const Plan p = make_plan(M, N, K);
    if (p.unsupported) return OPQ_ERR_UNSUPPORTED_SHAPE;
    *bytes = p.ws_bytes;
    return OPQ_OK;
}

opq_status opq_linear_plan(int64_t M, int64_t N, int64_t K, int *path, int *ctas, int *launches) {
    if (M < 1) return OPQ_ERR_INVALID_ARG;
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if (M > INT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    const Plan p = make_plan(M, N, K);
    if (p.unsupported) return OPQ_ERR_UNSUPPORTED_SHAPE;
    if (path) *path = p.mode;
    if (ctas) *ctas = p.grid;
    if (launches) *launches = p.launches;
    return OPQ_OK;
}

// the kernel the plan picked, for group size GS (0 = per-row scales)
extern "C++" {
template <int GS>
static cudaError_t launch_any(DeviceInfo *di, const Plan &plan, const CUtensorMap &xmap, const CUtensorMap &xhmap,
                              const CUtensorMap &cmap, const CUtensorMap &smap, const opqk::LinearArgs &a,
                              cudaStream_t st) {
    switch (plan.bx) {
        case 16: return launch_linear<16, GS>(di, plan, xmap, xhmap, cmap, smap, a, st);
        case 32: return launch_linear<32, GS>(di, plan, xmap, xhmap, cmap, smap, a, st);
        case 64: return launch_linear<64, GS>(di, plan, xmap, xhmap, cmap, smap, a, st);
        case 128: return launch_linear<128, GS>(di, plan, xmap, xhmap, cmap, smap, a, st);
        default: return launch_linear_wide<GS>(di, plan, xmap, xhmap, cmap, smap, a, st);
    }
}
}  // extern "C++"

// the per-row format (scales, gs = 0) or the group-wise one (gmax, gs = 32 .. 256)
static opq_status linear_impl(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                              const float *scales, const uint16_t *gmax, int64_t gs, int64_t N, float alpha,
                              const uint16_t *bias, int activation, uint16_t *y, void *workspace,
                              size_t workspace_bytes, void *stream) {
    if (M < 1) return OPQ_ERR_INVALID_ARG;
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if (gs > 0 && (s = check_group(K, gs)) != OPQ_OK) return s;
    if (M > INT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    if (activation != OPQ_ACT_NONE && activation != OPQ_ACT_SILU && activation != OPQ_ACT_GELU_TANH)
        return OPQ_ERR_INVALID_ARG;
    if ((s = check_ptrs({x, codes, signs, gs > 0 ? (const void *)gmax : (const void *)scales, y})) != OPQ_OK)
        return s;
    if (bias && (s = check_ptrs({bias})) != OPQ_OK) return s;
    const Plan plan = make_plan(M, N, K);
    if (plan.unsupported) return OPQ_ERR_UNSUPPORTED_SHAPE;
    if (plan.ws_bytes > 0) {
        if (workspace == nullptr || workspace_bytes < plan.ws_bytes) return OPQ_ERR_WORKSPACE;
        if ((s = check_ptrs({workspace})) != OPQ_OK) return s;
    }
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != OPQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    opqk::LinearArgs a{};
    a.signs = signs;
    a.scales = scales;
    a.y = y;
    a.counters = reinterpret_cast<uint32_t *>(workspace);
    a.ws = plan.ws_bytes ? reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + plan.counter_bytes)
                         : nullptr;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.m_tiles = plan.m_tiles;
    a.n_tiles = plan.n_tiles;
    a.kblocks = plan.kblocks;
    a.ngroups = plan.ngroups;
    a.mode = plan.mode;
    a.runs_max = plan.runs_max;
    a.tail_split = plan.mode == 0 ? plan.tail_split : 1;
    lut_bf16(alpha, a.lut);
    a.gmax = gmax;
    a.ngk = gs > 0 ? (int)(K / gs) : 0;
    a.bias = bias;
    a.act = activation;
    {
        const double inv = 1.0 / (double)alpha;
        for (int q = 0; q < 16; ++q) a.lutf[q] = (float)std::pow((double)q / 15.0, inv);
    }

    CUtensorMap xmap, xhmap, cmap, smap;
    // the sign plane's rows are 16-byte aligned (a TMA requirement) when K % 128 == 0; otherwise the
    // kernel copies the sign words with cp.async
    a.signs_tma = (K % 128 == 0) ? 1 : 0;
    if (plan.grp > 1) {
        // load groups of plan.grp blocks per copy (K % 128 == 0 here)
        const int64_t kb = K / 128;
        if ((s = make_x_chunk_map(&xmap, x, M, K, (uint32_t)plan.bx, 2u * (uint32_t)plan.grp)) != OPQ_OK) return s;
        if ((s = make_u32_block_map(&cmap, codes, N, 16u, kb, 128u, (uint32_t)plan.grp, CU_TENSOR_MAP_SWIZZLE_64B)) !=
            OPQ_OK)
            return s;
        if ((s = make_u32_block_map(&smap, signs, N, 4u, kb, 128u, (uint32_t)plan.grp, CU_TENSOR_MAP_SWIZZLE_NONE)) !=
            OPQ_OK)
            return s;
    } else {
        if ((s = make_x_map(&xmap, x, M, K, (uint32_t)plan.bx)) != OPQ_OK) return s;
        if ((s = make_u32_map(&cmap, codes, N, K / 8, 16u, 128u, CU_TENSOR_MAP_SWIZZLE_64B)) != OPQ_OK) return s;
        if (a.signs_tma) {
            if ((s = make_u32_map(&smap, signs, N, K / 32, 4u, 128u, CU_TENSOR_MAP_SWIZZLE_NONE)) != OPQ_OK) return s;
        } else {
            smap = cmap;   // not read by the kernel
        }
    }
    if (a.tail_split == 2) {
        if ((s = make_x_map(&xhmap, x, M, K, (uint32_t)plan.bx / 2)) != OPQ_OK) return s;
    } else {
        xhmap = xmap;   // not read by the kernel
    }
    cudaError_t e;
    switch (gs) {
        case 0: e = launch_any<0>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
        case 32: e = launch_any<32>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
        case 64: e = launch_any<64>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
        case 128: e = launch_any<128>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
        default: e = launch_any<256>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
    }
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaGetLastError();
    return e == cudaSuccess ? OPQ_OK : cuda_fail(e);
}

opq_status opq_linear(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                      const float *scales, int64_t N, float alpha, uint16_t *y, void *workspace,
                      size_t workspace_bytes, void *stream) {
    return linear_impl(x, M, K, codes, signs, scales, nullptr, 0, N, alpha, nullptr, OPQ_ACT_NONE, y, workspace,
                       workspace_bytes, stream);
}

opq_status opq_linear_fused(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                            const float *scales, int64_t N, float alpha, const uint16_t *bias, int activation,
                            uint16_t *y, void *workspace, size_t workspace_bytes, void *stream) {
    return linear_impl(x, M, K, codes, signs, scales, nullptr, 0, N, alpha, bias, activation, y, workspace,
                       workspace_bytes, stream);
}

opq_status opq_linear_grouped(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                              const uint16_t *gmax, int64_t N, int64_t group_size, float alpha, uint16_t *y,
                              void *workspace, size_t workspace_bytes, void *stream) {
    if (group_size == 0) return OPQ_ERR_INVALID_ARG;
    return linear_impl(x, M, K, codes, signs, nullptr, gmax, group_size, N, alpha, nullptr, OPQ_ACT_NONE, y,
                       workspace, workspace_bytes, stream);
}

opq_status opq_linear_grouped_fused(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                                    const uint32_t *signs, const uint16_t *gmax, int64_t N, int64_t group_size,
                                    float alpha, const uint16_t *bias, int activation, uint16_t *y, void *workspace,
                                    size_t workspace_bytes, void *stream) {
    if (group_size == 0) return OPQ_ERR_INVALID_ARG;
    return linear_impl(x, M, K, codes, signs, nullptr, gmax, group_size, N, alpha, bias, activation, y, workspace,
                       workspace_bytes, stream);
}

static opq_status check_bits_linear(int64_t M, int64_t N, int64_t K, int32_t bits) {
    if (M < 1) return OPQ_ERR_INVALID_ARG;
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if (bits < 3 || bits > 6) return OPQ_ERR_INVALID_ARG;
    if (M > INT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    // a 128-K block of a row is 4 bits words, copied whole by the tensor copies
    if (bits != 4 && K % 128 != 0) return OPQ_ERR_UNSUPPORTED_SHAPE;
    return OPQ_OK;
}

opq_status opq_linear_bits_workspace_size(int64_t M, int64_t N, int64_t K, int32_t bits, size_t *bytes) {
    if (!bytes) return OPQ_ERR_INVALID_ARG;
    opq_status s = check_bits_linear(M, N, K, bits);
    if (s != OPQ_OK) return s;
    const Plan p = bits == 4 ? make_plan(M, N, K) : make_plan(M, N, K, true);
    if (p.unsupported) return OPQ_ERR_UNSUPPORTED_SHAPE;
    *bytes = p.ws_bytes;
    return OPQ_OK;
}

opq_status opq_linear_bits(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                           const float *scales, int64_t N, int32_t bits, float alpha, uint16_t *y, void *workspace,
                           size_t workspace_bytes, void *stream) {
    opq_status s = check_bits_linear(M, N, K, bits);
    if (s != OPQ_OK) return s;
    if (bits == 4) return opq_linear(x, M, K, codes, signs, scales, N, alpha, y, workspace, workspace_bytes, stream);
    if (!alpha_ok(alpha)) return OPQ_ERR_INVALID_ARG;
    if ((s = check_ptrs({x, codes, signs, scales, y})) != OPQ_OK) return s;
    const Plan plan = make_plan(M, N, K, true);
    if (plan.ws_bytes > 0) {
        if (workspace == nullptr || workspace_bytes < plan.ws_bytes) return OPQ_ERR_WORKSPACE;
        if ((s = check_ptrs({workspace})) != OPQ_OK) return s;
    }
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != OPQ_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    opqk::LinearArgs a{};
    a.signs = signs;
    a.scales = scales;
    a.y = y;
    a.counters = reinterpret_cast<uint32_t *>(workspace);
    a.ws = plan.ws_bytes ? reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) + plan.counter_bytes)
                         : nullptr;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.m_tiles = plan.m_tiles;
    a.n_tiles = plan.n_tiles;
    a.kblocks = plan.kblocks;
    a.ngroups = plan.ngroups;
    a.mode = plan.mode;
    a.runs_max = plan.runs_max;
    a.tail_split = plan.tail_split;
    a.signs_tma = 1;
    a.act = OPQ_ACT_NONE;
    {
        const int L = (1 << bits) - 1;
        const double inv = 1.0 / (double)alpha;
        for (int q = 0; q <= L; ++q) a.lutb[q] = host_bf16(std::pow((double)q / (double)L, inv));
    }
    CUtensorMap xmap, xhmap, cmap, smap;
    if ((s = make_x_map(&xmap, x, M, K, (uint32_t)plan.bx)) != OPQ_OK) return s;
    if ((s = make_u32_map(&cmap, codes, N, K * bits / 32, 4u * (uint32_t)bits, 128u, CU_TENSOR_MAP_SWIZZLE_NONE)) !=
        OPQ_OK)
        return s;
    if ((s = make_u32_map(&smap, signs, N, K / 32, 4u, 128u, CU_TENSOR_MAP_SWIZZLE_NONE)) != OPQ_OK) return s;
    if (a.tail_split == 2) {
        if ((s = make_x_map(&xhmap, x, M, K, (uint32_t)plan.bx / 2)) != OPQ_OK) return s;
    } else {
        xhmap = xmap;   // not read by the kernel
    }
    cudaError_t e;
    switch (bits) {
        case 3: e = launch_linear_wide<0, 3>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
        case 5: e = launch_linear_wide<0, 5>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
        default: e = launch_linear_wide<0, 6>(di, plan, xmap, xhmap, cmap, smap, a, st); break;
    }
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaGetLastError();
    return e == cudaSuccess ? OPQ_OK : cuda_fail(e);
}

opq_status opq_linear_grouped_workspace_size(int64_t M, int64_t N, int64_t K, int64_t group_size, size_t *bytes) {
    if (!bytes) return OPQ_ERR_INVALID_ARG;
    if (M < 1) return OPQ_ERR_INVALID_ARG;
    opq_status s = check_sizes(N, K);
    if (s != OPQ_OK) return s;
    if ((s = check_group(K, group_size)) != OPQ_OK) return s;
    if (M > INT32_MAX) return OPQ_ERR_UNSUPPORTED_SHAPE;
    const Plan p = make_plan(M, N, K);
    if (p.unsupported) return OPQ_ERR_UNSUPPORTED_SHAPE;
    *bytes = p.ws_bytes;
    return OPQ_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free linear: the split-K scratch lives in a static device array.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {
// Scratch for opq_linear_noalloc only. In host code `g_noalloc_scratch` names a
// host-side shadow, not the device array: kernels get the device address looked
// up with cudaGetSymbolAddress (per device, with that device current).
static __device__ __align__(256) float g_noalloc_scratch[OPQ_NOALLOC_SCRATCH_BYTES / sizeof(float)];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {nullptr};

opq_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= 64) return OPQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return OPQ_OK;
}
}  // namespace

extern "C" opq_status opq_device_error(void *stream, uint32_t *err) {
    if (!err) return OPQ_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    uint32_t v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, opqdev::g_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemcpyToSymbol(opqdev::g_error, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e);
    if (v & opqdev::kErrWaitTimeout) {
        // A call that gave up waiting can leave arrival counters or published flags set. In a
        // caller's workspace the caller zeroes them; the allocation-free linear's counters sit
        // in the library's static array, so they are cleared here (a memset, no allocation).
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return cuda_fail(e);
        void *p = nullptr;
        if (dev >= 0 && dev < 64) {
            std::lock_guard<std::mutex> lk(g_noalloc_mu);
            p = g_noalloc_ptr[dev];
        }
        if (p != nullptr) {
            e = cudaMemsetAsync(p, 0, kCounterBytes, st);
            if (e != cudaSuccess) return cuda_fail(e);
            e = cudaStreamSynchronize(st);
            if (e != cudaSuccess) return cuda_fail(e);
        }
    }
    *err = v;
    return OPQ_OK;
}

extern "C" opq_status opq_set_wait_limit_ns(uint64_t ns) {
    const uint64_t v = ns == 0 ? opqdev::kWaitLimitNs : ns;
    cudaError_t e = cudaMemcpyToSymbol(opqdev::g_wait_limit_ns, &v, sizeof v);
    return e == cudaSuccess ? OPQ_OK : cuda_fail(e);
}

extern "C" opq_status opq_linear_noalloc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                                         const uint32_t *signs, const float *scales, int64_t N, float alpha,
                                         uint16_t *y, void *stream) {
    size_t need = 0;
    opq_status s = opq_linear_workspace_size(M, N, K, &need);
    if (s != OPQ_OK) return s;
    if (need > (size_t)OPQ_NOALLOC_SCRATCH_BYTES) return OPQ_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0 && (s = noalloc_scratch(&scratch)) != OPQ_OK) return s;
    return opq_linear(x, M, K, codes, signs, scales, N, alpha, y, scratch,
                      need > 0 ? (size_t)OPQ_NOALLOC_SCRATCH_BYTES : 0, stream);
}
