/*
 * opq.h — C ABI of the B200 (sm_100a) OPQ library, libopq.so.
 *
 * OPQ (Optimal Power Quantization) as described on the "OPQ INT4 Z-Image"
 * model card: per output row n of a weight matrix W[N, K],
 *     u = |w| / max_k |w[n, k]|,   v = u^alpha,   q = round(15 v)  (ties to even),
 *     w' = sign(w) * (q / 15)^(1 / alpha) * max_k |w[n, k]|
 * ("OPQ principle"), stored as 4-bit magnitudes packed 8 per uint32 and 1-bit
 * signs packed 32 per uint32 ("Technical details / storage format"), decoded
 * for inference as sign * (q/15)^(1/alpha) * max ("inference decoding").
 * This library keeps one fp32 scale (the row's max |w|) per output row where
 * the card keeps one fp16 max per group of 128.
 *
 * Packed format of an N x K weight (K a multiple of 32), all row-major:
 *   codes  uint32 [N, K/8]   element (n, 8j+i) is bits 4i..4i+3 of codes[n, j]
 *   signs  uint32 [N, K/32]  element (n, 32j+i) is bit i of signs[n, j]; 1 = negative
 *   scales float  [N]        max_k |w[n, k]| (exact: a bf16 value)
 * bf16 tensors are passed as their 16-bit patterns (uint16_t).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or managed memory of
 *     the current device); host pointers are rejected with
 *     OPQ_ERR_NOT_DEVICE_MEMORY before anything is launched.
 *   - Ownership stays with the caller; the library allocates no device memory.
 *   - Every pointer must be 16-byte aligned (OPQ_ERR_MISALIGNED otherwise).
 *   - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *     stream). The return value reports argument errors (checked before any
 *     launch) and launch errors; execution errors surface at the caller's next
 *     synchronisation, and device-side wait time-outs are reported by
 *     opq_device_error().
 *   - alpha must be finite and > 0. Non-finite weights are accepted without
 *     trapping; their codes and scales are unspecified.
 *   - Sizes are int64_t; N, K, M must be >= 1 and K % 32 == 0.
 */
#ifndef OPQ_H
#define OPQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum opq_status {
    OPQ_OK = 0,
    OPQ_ERR_INVALID_ARG = 1,        /* null pointer, non-positive size, bad alpha, bad ldw */
    OPQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 32 != 0, or a size beyond the supported range */
    OPQ_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
    OPQ_ERR_WORKSPACE = 4,          /* workspace missing or smaller than opq_linear_workspace_size */
    OPQ_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed (see opq_last_cuda_error) */
    OPQ_ERR_NOT_DEVICE_MEMORY = 6   /* a tensor pointer is not device-accessible memory */
} opq_status;

/*
 * opq_quantize — steps "normalise, power transform, quantize, pack" of the
 * card's "OPQ principle" and "storage format", one output row at a time.
 *   w       bf16 [N, ldw] device, row-major; columns 0..K-1 of each row are quantized
 *   N, K    rows (output features) and columns (input features); K % 32 == 0
 *   ldw     row stride of w in elements, ldw >= K and ldw % 8 == 0
 *   alpha   the power (the card's optimum for Z-Image is 0.73)
 *   codes   uint32 [N, K/8] device, written
 *   signs   uint32 [N, K/32] device, written
 *   scales  float [N] device, written (max |w| of the row; 0 for an all-zero row,
 *           whose codes are all 0)
 * Codes are exactly the round-half-even of 15 (|w|/max)^alpha, decided by
 * comparing |w| against per-row thresholds max * ((k - 1/2)/15)^(1/alpha)
 * formed in fp64; the output is deterministic run to run.
 */
opq_status opq_quantize(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, float alpha,
                        uint32_t *codes, uint32_t *signs, float *scales, void *stream);

/*
 * opq_quantize_batched — opq_quantize over a list of matrices in one pass: the card's
 * whole-model quantization ("Quantize and save": every linear layer of the
 * transformer) as one stream through HBM instead of one launch per matrix.
 *   jobs    HOST array of `count` descriptors (count >= 1), read before the call
 *           returns; each names a bf16 weight and its output planes, all device
 *           memory, with the meaning, layout and limits of opq_quantize's arguments
 *           (K % 32 == 0, K <= 32768, ldw >= K, ldw % 8 == 0, 16-byte aligned)
 *   alpha   the power, shared by every matrix of the call
 * Outputs are bit-identical to opq_quantize on each matrix. The work is dealt to
 * one CTA per SM by rows (matrices of up to 128 per launch); a job's output planes
 * must not overlap another job's. An invalid descriptor fails the whole call before
 * anything is launched.
 */
typedef struct opq_quant_job {
    const uint16_t *w;   /* bf16 [N, ldw] */
    int64_t N, K, ldw;
    uint32_t *codes;     /* [N, K/8] */
    uint32_t *signs;     /* [N, K/32] */
    float *scales;       /* [N] */
} opq_quant_job;
opq_status opq_quantize_batched(const opq_quant_job *jobs, int64_t count, float alpha, void *stream);

/*
 * opq_dequantize — the card's "inference decoding": w' = sign * (q/15)^(1/alpha) * max.
 *   codes, signs, scales  packed weight as produced by opq_quantize (device)
 *   N, K                  as for opq_quantize
 *   alpha                 the power used to quantize
 *   w_out                 bf16 [N, K] device, row-major, written
 * The product (q/15)^(1/alpha) * max is formed in fp64 and rounded once to
 * bf16 (round to nearest even); q = 0 with sign 1 gives -0.0.
 */
opq_status opq_dequantize(const uint32_t *codes, const uint32_t *signs, const float *scales,
                          int64_t N, int64_t K, float alpha, uint16_t *w_out, void *stream);

/*
 * opq_dequantize_batched — opq_dequantize over a list of matrices in one pass (the
 * inverse of opq_quantize_batched: every linear layer of a model decoded in one stream).
 *   jobs    HOST array of `count` descriptors (count >= 1), read before the call
 *           returns; each names a packed weight (device codes, signs, scales as
 *           produced by opq_quantize, N, K with opq_dequantize's limits) and its bf16
 *           output w_out [N, K] (device, 16-byte aligned)
 *   alpha   the power used to quantize, shared by every matrix of the call
 * Outputs are bit-identical to opq_dequantize on each matrix. The rows of up to 128
 * matrices per launch form one sequence dealt to the warps; a job's output must not
 * overlap another job's. An invalid descriptor fails the whole call before anything is
 * launched.
 */
typedef struct opq_dequant_job {
    const uint32_t *codes;   /* [N, K/8] */
    const uint32_t *signs;   /* [N, K/32] */
    const float *scales;     /* [N] */
    int64_t N, K;
    uint16_t *w_out;         /* bf16 [N, K] */
} opq_dequant_job;
opq_status opq_dequantize_batched(const opq_dequant_job *jobs, int64_t count, float alpha, void *stream);

/*
 * Group-wise format — the card's own storage ("Technical details / storage
 * format": one float16 max shared by every 128 weights; its configuration also
 * lists group sizes 32, 64 and 256). Row n's weights k = g*GS .. g*GS + GS - 1
 * form group g; u = |w| / gmax[n, g] with gmax the group's max |w| stored as
 * IEEE float16 (round to nearest even, saturating at 65504), the stored value
 * being the one both quantization and decoding use. Codes and signs are packed
 * exactly as in the per-row format:
 *   codes  uint32   [N, K/8]
 *   signs  uint32   [N, K/32]
 *   gmax   float16  [N, K/GS] (passed as 16-bit patterns)
 * group_size must be 32, 64, 128 or 256 (OPQ_ERR_INVALID_ARG otherwise) and
 * divide K (OPQ_ERR_UNSUPPORTED_SHAPE otherwise). A group whose stored max is
 * 0 has all-zero codes; weights above a max that rounded down in float16's
 * subnormal range code to 15.
 *
 * opq_quantize_grouped — as opq_quantize, one max per group; any K (no
 * register-resident row).
 */
opq_status opq_quantize_grouped(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t group_size,
                                float alpha, uint32_t *codes, uint32_t *signs, uint16_t *gmax, void *stream);

/*
 * opq_dequantize_grouped — w'[n, k] = bf16(sign * (q/15)^(1/alpha) * gmax[n, k / GS]),
 * the product formed in fp64 and rounded once (round to nearest even).
 */
opq_status opq_dequantize_grouped(const uint32_t *codes, const uint32_t *signs, const uint16_t *gmax, int64_t N,
                                  int64_t K, int64_t group_size, float alpha, uint16_t *w_out, void *stream);

/*
 * opq_linear_grouped — y = x W'^T with W' in the group-wise format: each decoded
 * weight is bf16(sign * (q/15)^(1/alpha) * gmax) (the product formed in fp32 from
 * fp32 magnitudes, then rounded to bf16) and enters the bf16 tensor-core product
 * with fp32 accumulation; y is the sum rounded once to bf16. Arguments as for
 * opq_linear, with gmax and group_size in place of scales, and the same
 * schedule as opq_linear for the shape; the workspace is sized by
 * opq_linear_grouped_workspace_size and follows opq_linear's workspace rules.
 */
opq_status opq_linear_grouped(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                              const uint32_t *signs, const uint16_t *gmax, int64_t N, int64_t group_size,
                              float alpha, uint16_t *y, void *workspace, size_t workspace_bytes, void *stream);
opq_status opq_linear_grouped_workspace_size(int64_t M, int64_t N, int64_t K, int64_t group_size, size_t *bytes);

/*
 * Fused epilogue — the OPQLinear layers replace nn.Linear modules, which carry a
 * bias, and in the transformer's feed-forward blocks an activation follows.
 * opq_linear_fused / opq_linear_grouped_fused are opq_linear / opq_linear_grouped
 * with, per output, v = sum * scale (per-row format; the group-wise sum carries its
 * scales already) + bias[n], then the activation, in fp32, rounded once to bf16:
 *   bias        bf16 [N] device (16-byte aligned), or NULL for none
 *   activation  OPQ_ACT_NONE, OPQ_ACT_SILU (v / (1 + e^-v)) or OPQ_ACT_GELU_TANH
 *               (0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))); anything else is
 *               OPQ_ERR_INVALID_ARG
 * Both activations are evaluated with the GPU's hardware tanh approximation (SiLU as
 * v (1/2 + tanh(v/2)/2)): the output's extra error is at most about 2.5e-4 |v|.
 * Workspace and schedule as for the unfused calls.
 */
#define OPQ_ACT_NONE 0
#define OPQ_ACT_SILU 1
#define OPQ_ACT_GELU_TANH 2
opq_status opq_linear_fused(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                            const float *scales, int64_t N, float alpha, const uint16_t *bias, int activation,
                            uint16_t *y, void *workspace, size_t workspace_bytes, void *stream);
opq_status opq_linear_grouped_fused(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                                    const uint32_t *signs, const uint16_t *gmax, int64_t N, int64_t group_size,
                                    float alpha, const uint16_t *bias, int activation, uint16_t *y, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * Other bit widths — the card's configuration lists 3, 4, 5 and 6 bits per
 * magnitude; its storage section describes 4. With `bits` bits there are
 * L = 2^bits - 1 levels, q = round(L u^alpha) (ties to even) and
 * w' = sign * (q/L)^(1/alpha) * max, one fp32 max per row. The codes of a row
 * form one little-endian bit stream: element k at bits k*bits .. k*bits+bits-1
 * of the row's K*bits/32 uint32 words (for 4 bits: nibble k % 8 of word k / 8,
 * the per-row format above). Signs and scales as in the per-row format.
 *   codes  uint32 [N, K*bits/32];  bits 3..6 (OPQ_ERR_INVALID_ARG otherwise)
 * opq_quantize_bits takes the arguments and limits of opq_quantize (K % 32 == 0,
 * K <= 32768, ldw >= K, ldw % 8 == 0, w 16-byte aligned) and runs the same
 * row-streaming kernel at the given width.
 */
opq_status opq_quantize_bits(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int32_t bits, float alpha,
                             uint32_t *codes, uint32_t *signs, float *scales, void *stream);
opq_status opq_dequantize_bits(const uint32_t *codes, const uint32_t *signs, const float *scales, int64_t N, int64_t K,
                               int32_t bits, float alpha, uint16_t *w_out, void *stream);

/*
 * opq_linear_bits — the OPQLinear forward at any of the card's widths (its
 * configuration lists OPQ_BITS 3, 4, 5, 6): y = x W'^T with each decoded weight
 * sign * bf16((q/L)^(1/alpha)), L = 2^bits - 1, in a bf16 tensor-core product with
 * fp32 accumulation; y = bf16(sum * scale[n]), as opq_linear.
 *   x, M, K, y, workspace, workspace_bytes, stream   as for opq_linear
 *   codes, signs, scales, N   the planes of opq_quantize_bits at `bits`
 *   bits        3..6 (OPQ_ERR_INVALID_ARG otherwise); 4 runs opq_linear
 * Widths 3, 5 and 6 need K % 128 == 0 (OPQ_ERR_UNSUPPORTED_SHAPE otherwise) and run
 * 256-activation-row tiles for every M; the workspace is sized by
 * opq_linear_bits_workspace_size and follows opq_linear's rules.
 */
opq_status opq_linear_bits_workspace_size(int64_t M, int64_t N, int64_t K, int32_t bits, size_t *bytes);
opq_status opq_linear_bits(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes, const uint32_t *signs,
                           const float *scales, int64_t N, int32_t bits, float alpha, uint16_t *y, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * opq_alpha_search — the card's alpha is a per-model choice in 0.3 .. 1.0 (its
 * "OPQ configuration"; "why alpha = 0.73": a flat optimum on Z-Image weights). For
 * each candidate alpha this quantizes W (per-row format when group_size is 0,
 * else group-wise with that group size) and measures the SNR of the decoded
 * weights against W, 10 log10(sum w^2 / sum (w - w')^2) with w' = sign *
 * (q/15)^(1/alpha) * max in fp32, summed in fp64 in a fixed order. Nothing is
 * written but the results; the call synchronises `stream`.
 *   alphas       HOST float [count], each finite and > 0; count >= 1
 *   snr_db       HOST double [count], written (+HUGE_VAL for an exact reconstruction)
 *   best_alpha   HOST float, written: the first alpha with the largest SNR
 *   workspace    device scratch of opq_alpha_search_workspace_size(N) bytes
 */
opq_status opq_alpha_search_workspace_size(int64_t N, size_t *bytes);
opq_status opq_alpha_search(const uint16_t *w, int64_t N, int64_t K, int64_t ldw, int64_t group_size,
                            const float *alphas, int32_t count, double *snr_db, float *best_alpha, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * opq_linear_workspace_size — device scratch bytes opq_linear needs for an
 * M x K by (N x K)^T product (0 when the chosen kernel needs none).
 */
opq_status opq_linear_workspace_size(int64_t M, int64_t N, int64_t K, size_t *bytes);

/*
 * opq_linear — y = x W'^T with W' decoded from the packed planes (the card's
 * OPQLinear forward: decode w' = sign * (q/15)^(1/alpha) * max, then matmul).
 *   x          bf16 [M, K] device, row-major (leading dimension K)
 *   M, K       activation rows and the reduction length (K % 32 == 0). M <= 128 with
 *              more than 4096 128-row weight tiles (N > 524288), or with
 *              ceil(N/128) x (load groups per tile) x 148 >= 2^31, needs K % 128 == 0
 *              (OPQ_ERR_UNSUPPORTED_SHAPE otherwise, also from the workspace size and
 *              the plan)
 *   codes, signs, scales   packed W [N, K] (device)
 *   N          output features
 *   alpha      the power used to quantize
 *   y          bf16 [M, N] device, row-major (leading dimension N), written
 *   workspace  device scratch of at least opq_linear_workspace_size(M, N, K) bytes
 *              (may be NULL when that size is 0). It must be zero-filled before its
 *              first use (e.g. one cudaMemset after allocation); every completed call
 *              leaves it valid for the next one (its leading arrival counters back at
 *              zero), for any shape. Calls sharing one workspace must not overlap on
 *              the GPU.
 * Arithmetic: each decoded weight sign * bf16((q/15)^(1/alpha)) enters a bf16
 * tensor-core product with fp32 accumulation; the row scale is applied to the
 * fp32 sum, which is then rounded once to bf16. Deterministic: the same inputs
 * give bitwise-identical y (split-K partial sums are added in a fixed order).
 */
opq_status opq_linear(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                      const uint32_t *signs, const float *scales, int64_t N, float alpha,
                      uint16_t *y, void *workspace, size_t workspace_bytes, void *stream);

/*
 * opq_linear_plan — the schedule opq_linear uses for this shape (it depends on the
 * shape alone, so workspace sizes and result bits do not vary between B200s):
 *   *path      0 = whole 128-weight-row x 256-activation-row tiles, one persistent CTA
 *              per SM; 1 = stream-K: the (tile, 128-K block) sequence cut into one
 *              contiguous range per CTA, followed by a fixed-order fix-up kernel
 *   *ctas      CTAs of the main kernel
 *   *launches  kernels launched per opq_linear call
 * Any output pointer may be NULL.
 */
opq_status opq_linear_plan(int64_t M, int64_t N, int64_t K, int *path, int *ctas, int *launches);

/*
 * opq_linear_noalloc — opq_linear without a caller-provided workspace. The paper
 * has no counterpart; this entry point exists for callers that cannot allocate
 * device memory themselves: code embedded in a host runtime that owns the GPU's
 * memory pool and forbids foreign cudaMalloc calls after start-up, or code whose
 * fixed operator signature has no slot for a scratch buffer.
 *   Arguments and results are those of opq_linear (x, codes, signs, scales, y are
 *   still the caller's device buffers); the split-K partial sums go to a static
 *   device array of OPQ_NOALLOC_SCRATCH_BYTES (16 MiB) inside libopq.so, which
 *   every GPU that loads the library holds until the process exits.
 *   - Shapes whose opq_linear_workspace_size exceeds OPQ_NOALLOC_SCRATCH_BYTES are
 *     rejected with OPQ_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress, with that device current); make that first
 *     call before any stream capture on the device.
 *   - All calls share the one array and it keeps the last call's contents. Its
 *     leading arrival counters must be zero when a call starts: the array is zero
 *     when the library loads and every completed call leaves them at zero again.
 *     A call whose bounded wait gave up (opq_device_error reports
 *     OPQ_DEVERR_WAIT_TIMEOUT) can leave them set; opq_device_error clears them
 *     when it reports that error, so read it before the next call of this kind.
 *     Calls that overlap on the GPU (different streams, or different host threads
 *     without ordering) race on the array and give wrong results.
 *   - No device memory is allocated or freed by this call.
 */
#define OPQ_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
opq_status opq_linear_noalloc(const uint16_t *x, int64_t M, int64_t K, const uint32_t *codes,
                              const uint32_t *signs, const float *scales, int64_t N, float alpha,
                              uint16_t *y, void *stream);

/*
 * opq_device_error — reads and clears the library's device-side error word on
 * the current device (synchronises `stream`). 0 = no error; otherwise a bitmask
 * of OPQ_DEVERR_* recorded by a kernel that returned early, leaving its output
 * invalid: WAIT_TIMEOUT when a bounded wait on a barrier gave up, SMEM_ALIGN when
 * the dynamic shared-memory window did not start on the 1 KiB boundary that the
 * 128-byte-swizzled tensor-core operand stages need.
 * After a WAIT_TIMEOUT a caller-provided linear workspace must be zero-filled
 * again before its next use; the arrival counters of opq_linear_noalloc's static
 * array are zeroed by this call itself (a memset on `stream`, synchronised; no
 * opq_linear_noalloc call may be in flight on another stream meanwhile).
 */
#define OPQ_DEVERR_WAIT_TIMEOUT 1u
#define OPQ_DEVERR_SMEM_ALIGN 2u
opq_status opq_device_error(void *stream, uint32_t *err);

/*
 * opq_set_wait_limit_ns — the time after which a kernel's bounded wait on a
 * barrier or a flag gives up (records OPQ_DEVERR_WAIT_TIMEOUT, lets its own copies
 * in flight land, frees its tensor memory and returns) on the current device;
 * ns = 0 restores the default of 4 s. Every wait in a healthy call ends within
 * that call's own run time, so the limit only bounds how long a broken
 * protocol (for example a workspace that was not zeroed) can hold the GPU; tests
 * shorten it to see a time-out quickly. The value is written with a
 * synchronous copy to device memory and is read by kernels launched after the
 * call returns; do not change it while library kernels run on other streams.
 */
opq_status opq_set_wait_limit_ns(uint64_t ns);

/* Human-readable name of a status. */
const char *opq_status_string(opq_status s);

/* Last CUDA error code (cudaError_t) seen by this thread inside the library, 0 if none. */
int opq_last_cuda_error(void);

/* ABI version of this header: 1. */
int opq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OPQ_H */
