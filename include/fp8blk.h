/*
 * fp8blk -- the block-FP8 linear layer on NVIDIA B200 (sm_100a).
 *
 * Format (FastVideo PR #1829, "MiniMax H3: block-FP8 text encoder on Hopper,
 * its converter, and a 4xH100 FastH3 profile", section "Changes", converter
 * bullet): a linear's weight W[N][K] (nn.Linear order: N outputs, K inputs)
 * is stored as E4M3 codes q[N][K] plus one float weight_scale_inv per
 * 128 x 128 block, s[ceil(N/128)][ceil(K/128)]. Element (n, k) belongs to
 * block (n/128, k/128) and stands for E4M3(q[n][k]) * s[n/128][k/128]
 * (section "Purpose" and the tests bullet of "Changes": the dequantizer is
 * the code times its block's scale, broadcast over the block).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device.
 *    The caller owns every buffer; the library allocates nothing (the linear
 *    calls take a caller-provided workspace) and never synchronizes.
 *  - Matrices are row-major with an explicit leading dimension ("ld"),
 *    counted in elements. Scale grids are dense row-major.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream). Argument errors are reported synchronously,
 *    before anything is launched; a failed launch returns FP8BLK_ERR_CUDA; a
 *    fault inside a kernel shows up at the caller's next synchronization.
 *  - The device must have compute capability 10.x (B200 class); otherwise
 *    FP8BLK_ERR_UNSUPPORTED_DEVICE. There is no fallback path.
 *  - Every tensor pointer must be 16-byte aligned (scale pointers: 4-byte).
 *  - A size of 0 is valid: nothing is read and (except the K = 0 linear, which
 *    writes y = 0) nothing is written.
 *  - Inputs must be finite; NaN and infinity are outside the contract.
 *  - Calls are reentrant; concurrent calls on different streams are safe as
 *    long as they do not share output or workspace buffers.
 */
#ifndef FP8BLK_H
#define FP8BLK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8BLK_EXPORT __attribute__((visibility("default")))
#else
#define FP8BLK_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp8blk_status {
  FP8BLK_OK = 0,
  FP8BLK_ERR_INVALID_ARG = 1,        /* negative size, ld too small, NULL pointer  */
  FP8BLK_ERR_ALIGNMENT = 2,          /* pointer or leading dimension misaligned    */
  FP8BLK_ERR_UNSUPPORTED_DEVICE = 3, /* current device is not compute capability 10.x */
  FP8BLK_ERR_WORKSPACE = 4,          /* workspace NULL or smaller than required    */
  FP8BLK_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed       */
  FP8BLK_ERR_TIMEOUT = 6             /* a kernel gave up waiting (device error word set) */
} fp8blk_status;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA headers. */
typedef void* fp8blk_stream;

/* ---------------------------------------------------------------------------
 * (1) Converter: BF16 weight -> E4M3 codes + weight_scale_inv.
 * FastVideo PR #1829, section "Changes", converter bullet (E4M3 codes with a
 * float weight_scale_inv grid of shape [N/128, K/128]). For each 128 x 128 block:
 *   amax = max |W| over the block's in-bounds elements (ragged edge blocks
 *          are not padded with anything but zeros),
 *   s    = amax / 448            (float division, round to nearest even),
 *   q    = E4M3(W / s)           (float division, then round to nearest even
 *                                 with saturation to +-448);
 * a block whose elements are all +-0 gets s = 0 and codes 0x00 / 0x80 that
 * keep each element's sign.
 *   w         : BF16 [N][ldw], ldw >= K, ldw % 8 == 0           (input)
 *   q         : uint8 [N][ldq], ldq >= K, ldq % 16 == 0         (output; columns
 *               K..ldq-1 are not written)
 *   scale_inv : float [ceil(N/128)][ceil(K/128)], dense          (output)
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_quantize_weight(const void* w, int64_t N, int64_t K, int64_t ldw,
                                     uint8_t* q, int64_t ldq, float* scale_inv,
                                     fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * (2) Dequantizer: E4M3 codes + scales -> BF16 weight.
 * FastVideo PR #1829, section "Purpose" (the Hopper route materializes the
 * BF16 weight) and the tests bullet of "Changes" (bit-exact against the
 * scale broadcast over each block):
 *   w[n][k] = BF16( float(E4M3(q[n][k])) * s[n/128][k/128] )
 * with one float multiply and one round-to-nearest-even to BF16.
 *   q         : uint8 [N][ldq], ldq >= K, ldq % 16 == 0          (input)
 *   scale_inv : float [ceil(N/128)][ceil(K/128)]                  (input)
 *   w         : BF16 [N][ldw], ldw >= K, ldw % 8 == 0            (output)
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_dequantize(const uint8_t* q, int64_t ldq, const float* scale_inv,
                                int64_t N, int64_t K, void* w, int64_t ldw,
                                fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * Activation quantizer (the first stage of fp8blk_linear_w8a8, exposed so its
 * output can be checked and reused). The Blackwell route of FastVideo PR
 * #1829 quantizes activations before its groupwise GEMM (section "Changes",
 * loader bullet); groups are 1 x 128 along K with the converter's recipe:
 *   sx[g][m] = max_{k in group g} |x[m][k]| / 448,  qx[m][k] = E4M3(x[m][k] / sx[g][m])
 *   x   : BF16 [M][ldx], ldx >= K, ldx % 8 == 0                   (input)
 *   qx  : uint8 [M][ldqx], ldqx >= K, ldqx % 16 == 0              (output)
 *   sx  : float [ceil(K/128)][ldsx], ldsx >= M, ldsx % 4 == 0     (output; note the
 *         group-major layout: the M scales of one K-group are contiguous)
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx,
                                  uint8_t* qx, int64_t ldqx, float* sx, int64_t ldsx,
                                  fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * (3) Linear, BF16 activations x block-FP8 weight ("W8A16"):
 *   y[m][n] = BF16( sum_kb s[n/128][kb] * P_kb[m][n] ),
 *   P_kb[m][n] = sum_{k in slab kb} x[m][k] * E4M3(q[n][k])   (FP32)
 * i.e. y = x . dequant(W)^T (FastVideo PR #1829, "Purpose": the same
 * computation as the Blackwell groupwise GEMM), with the block scale applied to
 * the FP32 partial of each 128-wide K slab and FP32 accumulation across
 * slabs. Tensor cores see the exact BF16 image of each E4M3 code.
 *   x : BF16 [M][ldx], ldx >= K, ldx % 8 == 0                        (input)
 *   q : uint8 [N][ldq], ldq >= K, ldq % 16 == 0; scale_inv as above  (input)
 *   y : BF16 [M][ldy], ldy >= N, ldy % 8 == 0; must not alias the inputs (output)
 *   workspace : 256-byte aligned; its contents on entry do not matter and
 *               are scratch on return.
 *     - M <= 128: fp8blk_workspace_size(0, M, N, K) bytes are required. The
 *       slabs are split evenly over the SMs (stream-K) and the workspace
 *       holds the FP32 partials of tiles split between SMs (at most
 *       160 x 2 x BT x 128 x 4 bytes, BT the token tile: 16, 32, 64 or 128).
 *     - M > 128: optional. Tiles of 256 tokens run whole, one per SM at a
 *       time; when the last wave of tiles would leave at least 15% of the SM
 *       time idle and the workspace holds fp8blk_workspace_size(0, M, N, K)
 *       bytes, that wave's slabs are split evenly over the SMs instead
 *       (partials of [256][128] floats, two per SM). NULL or a smaller
 *       workspace runs every tile whole.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_linear_w8a16(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                                  const float* scale_inv, void* y, int64_t ldy,
                                  int64_t M, int64_t N, int64_t K,
                                  void* workspace, size_t workspace_bytes,
                                  fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * (4) Linear with FP8 activations ("W8A8"): x is first quantized per 1 x 128
 * K-group (see fp8blk_quantize_act) into the workspace, then
 *   y[m][n] = BF16( sum_kb sx[kb][m] * s[n/128][kb] * P_kb[m][n] ),
 *   P_kb[m][n] = sum_{k in slab kb} E4M3(qx[m][k]) * E4M3(q[n][k])  (FP32)
 * on E4M3 x E4M3 tensor cores. Arguments as for fp8blk_linear_w8a16, with
 * workspace >= fp8blk_workspace_size(1, M, N, K). Workspace layout (so the
 * quantized activations can be inspected): qx uint8 [M][round_up(K, 16)] at
 * offset 0, then sx float [ceil(K/128)][round_up(M, 128)] at the next
 * 256-byte boundary.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_linear_w8a8(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                                 const float* scale_inv, void* y, int64_t ldy,
                                 int64_t M, int64_t N, int64_t K,
                                 void* workspace, size_t workspace_bytes,
                                 fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * W8A8 linear without a workspace argument. (The pages have no counterpart:
 * this is a calling convenience of this library.) For callers that cannot
 * allocate device memory -- e.g. a runtime that plans every buffer before it
 * starts serving and forbids allocation afterwards, or host code that must
 * not call cudaMalloc because it can synchronize the device and stall other
 * streams. Computes exactly what fp8blk_linear_w8a8 computes, with the same
 * arguments minus the workspace; its scratch is a fixed array of
 * FP8BLK_NOALLOC_SCRATCH_BYTES built into the library, present on every GPU
 * that loads it until the process exits. The call itself allocates nothing.
 *  - Limit: the problem must satisfy fp8blk_workspace_size(1, M, N, K) <=
 *    FP8BLK_NOALLOC_SCRATCH_BYTES (M * round_up(K, 16) bytes of codes plus the
 *    scales; e.g. M = 2048 at K = 5120); larger problems return
 *    FP8BLK_ERR_WORKSPACE before anything is launched.
 *  - The first call on a device (with that device current) looks up the
 *    array's device address once; make that first call before any stream
 *    capture (a first call on a capturing stream returns INVALID_ARG).
 *  - All calls share the one array: calls that can overlap on the GPU (on
 *    different streams, or from different threads) race on it and must be
 *    ordered by the caller.
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, WORKSPACE (too large), CUDA.
 * ------------------------------------------------------------------------- */
#define FP8BLK_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
FP8BLK_EXPORT fp8blk_status fp8blk_linear_w8a8_noalloc(const void* x, int64_t ldx, const uint8_t* q,
                                                       int64_t ldq, const float* scale_inv, void* y,
                                                       int64_t ldy, int64_t M, int64_t N, int64_t K,
                                                       fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * W8A8 linear on activations already quantized by fp8blk_quantize_act, so
 * that sibling linears reading the same x (Q, K and V; gate and up) quantize
 * it once (FastVideo PR #1829, "Changes": the Blackwell route quantizes the
 * activations before the groupwise GEMM). Computes
 *   y[m][n] = BF16( sum_kb sx[kb][m] * s[n/128][kb] * P_kb[m][n] )
 * exactly as fp8blk_linear_w8a8 does after its own quantization step.
 *   qx : uint8 [M][ldqx], ldqx >= K, ldqx % 16 == 0, 16-byte aligned (input)
 *   sx : float [ceil(K/128)][ldsx], ldsx >= M, 4-byte aligned          (input)
 *   q, scale_inv, y, M, N, K : as for fp8blk_linear_w8a8.
 * No workspace. Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_linear_w8a8_quantized(const uint8_t* qx, int64_t ldqx,
                                                         const float* sx, int64_t ldsx,
                                                         const uint8_t* q, int64_t ldq,
                                                         const float* scale_inv, void* y,
                                                         int64_t ldy, int64_t M, int64_t N,
                                                         int64_t K, fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * A sequence of linears on device weights, launched back to back so that each
 * GEMM starts streaming its weights while the kernels before it finish
 * (programmatic dependent launch). This is the decode-time case: the weight
 * stream is the whole cost, and the linears of a layer follow one another.
 * Each job computes exactly what fp8blk_linear_w8a16 (mode 0) or
 * fp8blk_linear_w8a8 (mode 1) computes from the same arguments, in job order;
 * a job's x may be an earlier job's y, and a job's y may overwrite an
 * earlier job's x. The caller promises that no job writes another job's
 * weights (q, scale_inv): weights are read before the previous job has
 * finished. The first job waits for all earlier work on `stream`.
 *   jobs      : njobs job descriptions (host memory), each as for the linear
 *               calls (device pointers)
 *   workspace : DEVICE, at least the largest fp8blk_workspace_size(mode, M,
 *               N, K) over the jobs (the jobs use it one after another)
 * Every job is checked before anything is launched.
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
typedef struct fp8blk_linear_args {
  int32_t mode;              /* 0 = W8A16, 1 = W8A8 */
  const void* x;             /* BF16 [M][ldx] */
  int64_t ldx;
  const uint8_t* q;          /* E4M3 codes [N][ldq] */
  int64_t ldq;
  const float* scale_inv;    /* [ceil(N/128)][ceil(K/128)] */
  void* y;                   /* BF16 [M][ldy] */
  int64_t ldy;
  int64_t M, N, K;
} fp8blk_linear_args;

FP8BLK_EXPORT fp8blk_status fp8blk_linear_sequence(const fp8blk_linear_args* jobs, int64_t njobs,
                                                   void* workspace, size_t workspace_bytes,
                                                   fp8blk_stream stream);

/* ---------------------------------------------------------------------------
 * Layerwise FP8 weight streaming (FastVideo PR #1829, "Purpose": the FP8
 * checkpoint is what keeps the encoder resident, and what an offloaded
 * encoder moves instead of BF16 weights; the page reports both the memory
 * and the offload time of the two forms). Runs a sequence of linears whose
 * codes and scales live in HOST memory through a ring of `nslots` device
 * weight slots: job i's weights are copied into slot i % nslots on `copy`
 * while earlier jobs run on `compute`; job i's linear runs on `compute` once
 * its copy has landed, and a slot is refilled only after the linear that
 * read it has finished. Each job computes exactly what fp8blk_linear_w8a16
 * (mode 0) or fp8blk_linear_w8a8 (mode 1) computes from the same weights on
 * the device.
 *   jobs[i].q_host     : uint8 [N][ldq] in HOST memory (pinned, or the
 *                        copies are not asynchronous), ldq >= K, ldq % 16 == 0
 *   jobs[i].scale_host : float [ceil(N/128)][ceil(K/128)] in HOST memory
 *   jobs[i].x, ldx, y, ldy, M, N, K : DEVICE activations and output, as for
 *                        the linear calls (x read, y written on `compute`)
 *   slots      : DEVICE, nslots consecutive slots of slot_bytes each;
 *                256-byte aligned, slot_bytes % 256 == 0 and
 *                slot_bytes >= fp8blk_stream_slot_bytes(N, K, ldq) of every
 *                job (codes at the start of a slot, scales after them)
 *   workspace  : DEVICE, as for the linear calls, at least the largest
 *                fp8blk_workspace_size(mode, M, N, K) over the jobs
 *   compute, copy : streams (the same stream twice is valid: no overlap)
 *   events     : 2 * nslots cudaEvent_t created by the caller (timing
 *                disabled is best); the library only records and waits on them
 * The copies of a call start after the work already enqueued on `compute`,
 * so consecutive calls may share slots and events.
 * Everything is enqueued asynchronously: on return nothing need have run.
 * Every job is checked before anything is enqueued; a CUDA error while
 * enqueuing returns FP8BLK_ERR_CUDA with the jobs before it enqueued.
 * Errors: INVALID_ARG, ALIGNMENT, WORKSPACE, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
typedef struct fp8blk_linear_job {
  int32_t mode;              /* 0 = W8A16, 1 = W8A8 */
  const uint8_t* q_host;     /* host codes [N][ldq] */
  const float* scale_host;   /* host scales [ceil(N/128)][ceil(K/128)] */
  int64_t ldq;
  const void* x;             /* device BF16 activations [M][ldx] */
  int64_t ldx;
  void* y;                   /* device BF16 output [M][ldy] */
  int64_t ldy;
  int64_t M, N, K;
} fp8blk_linear_job;

/* A cudaEvent_t, passed as an opaque pointer. */
typedef void* fp8blk_event;

/* Bytes of one weight slot for an N x K linear with code pitch ldq: the
 * codes rounded up to 256 bytes, then the scales, rounded up to 256. Pure
 * host function; 0 for negative sizes or ldq < K. */
FP8BLK_EXPORT size_t fp8blk_stream_slot_bytes(int64_t N, int64_t K, int64_t ldq);

FP8BLK_EXPORT fp8blk_status fp8blk_streamed_linears(const fp8blk_linear_job* jobs, int64_t njobs,
                                                    void* slots, size_t slot_bytes, int32_t nslots,
                                                    void* workspace, size_t workspace_bytes,
                                                    fp8blk_stream compute, fp8blk_stream copy,
                                                    fp8blk_event* events);

/* Workspace bytes for a linear: mode 0 = W8A16, 1 = W8A8. Pure host function;
 * returns 0 for an invalid mode or negative sizes. */
FP8BLK_EXPORT size_t fp8blk_workspace_size(int mode, int64_t M, int64_t N, int64_t K);

/* ---------------------------------------------------------------------------
 * Element codec of the converter, exposed for verification: codes[i] =
 * E4M3(v[i]) with round-to-nearest-even and saturation to +-448 (NaN -> 0x7F),
 * the same device routine the converter and the activation quantizer use.
 *   v : float [n] (device, 16-byte aligned); codes : uint8 [n] (device, 16-byte aligned)
 * Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------- */
FP8BLK_EXPORT fp8blk_status fp8blk_encode_e4m3(const float* v, int64_t n, uint8_t* codes, fp8blk_stream stream);

/* Self-test of the failure-detection path: launches one warp that waits, with
 * the kernels' own bounded wait, on an mbarrier phase that nothing completes.
 * After limit_cycles SM cycles (1000 <= limit_cycles <= 4e9; a few million is
 * about a millisecond) the wait gives up, sets flag 16 in the error word and
 * the kernel returns, leaving the context usable: fp8blk_read_device_error
 * then reports FP8BLK_ERR_TIMEOUT with word 16. No fault, trap or hang.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
FP8BLK_EXPORT fp8blk_status fp8blk_selftest_wait_timeout(int64_t limit_cycles, fp8blk_stream stream);

/* Reads and clears the current device's error word (bit flags set by a kernel
 * whose bounded wait ran out: 1 load, 2 MMA, 4 epilogue, 8 weight expansion,
 * 16 the self-test above).
 * Synchronizes the device. *word receives the flags; returns FP8BLK_ERR_TIMEOUT
 * when any flag was set, FP8BLK_OK when none, FP8BLK_ERR_CUDA on a CUDA error. */
FP8BLK_EXPORT fp8blk_status fp8blk_read_device_error(uint32_t* word);

/* Human-readable name of a status code (static storage). */
FP8BLK_EXPORT const char* fp8blk_status_string(fp8blk_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
FP8BLK_EXPORT int fp8blk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BLK_H */
