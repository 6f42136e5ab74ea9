/*
 * qlora.h -- C ABI of libqlora.so: blockwise NF4 storage with double
 * quantization and the LoRA linear on top of it, forward and backward, for
 * NVIDIA B200 (sm_100a).
 *
 * The method (web pages, cited by title and section):
 *   - "QLoRA: efficient finetuning of quantized LLMs", Abstract: gradients are
 *     backpropagated through a frozen 4-bit quantized model into low-rank
 *     adapters; (a) the NF4 data type, (b) double quantization of the
 *     quantization constants.
 *   - "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
 *     goes": the base is kept in 4 bits, quantized a single time before
 *     training, and expanded to 16-bit inside every forward and backward pass;
 *     gradients flow through the dequantized weights into the adapters, which
 *     stay 16-bit.  Section "NormalFloat, double quantization, paged
 *     optimizers": 16 levels at normal quantiles; one scaling constant per
 *     block; those constants in turn stored in 8 bits, scaled by a further,
 *     coarser level of constants.
 *   - "Qlora 4 Bit Quantization With Nf4 Fp4 Data Types And Lora Adapters",
 *     entry "4-bit quantization with nf4 data type for llm weight
 *     compression": block-wise absmax scaling plus double quantization.
 *
 * Conventions for every call
 *   - Every pointer argument named as "device" is CUDA device memory owned by
 *     the caller.  The library never allocates or frees device memory; the
 *     linear calls take a caller-provided workspace whose size is returned by
 *     qlora_workspace_bytes() (at least qlora_workspace_min_bytes(); its
 *     contents on entry do not matter).
 *   - bf16 tensors are passed as uint16_t bit patterns.  All tensors are dense
 *     row-major and every device pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; no call synchronizes the stream, except
 *     qlora_device_status().
 *   - Argument errors are detected on the host and returned before anything is
 *     enqueued.  Errors only the device can see (a non-finite weight handed to
 *     the quantizer, a pipeline wait that exceeded its bound) are latched in a
 *     device status word; read and clear it with qlora_device_status().
 *   - Outputs are overwritten, never accumulated into.
 *   - The debug build of the library (libqlora_debug.so, compiled with
 *     QLORA_BOUNDS_CHECK) checks the global-memory indices of the quantizer,
 *     the dequantizer and the few-token forward against their buffers; a miss
 *     latches QLORA_ERR_BOUNDS and skips the access instead of trapping.
 *   - The library caches per-device state on first use (the device addresses
 *     of its status word and scratch array, its side streams and events); do
 *     not reset a device (cudaDeviceReset) after calling the library on it.
 *
 * Fixed format: block = 64 consecutive elements of the flat row-major weight,
 * group = 256 consecutive blocks.  codes: element 2j in the low nibble of byte
 * j, 2j+1 in the high nibble (an unused final high nibble is 0).
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad rank/scale   */
  QLORA_ERR_UNSUPPORTED_SHAPE = 2, /* e.g. cols % 64 != 0 for the linear           */
  QLORA_ERR_MISALIGNED = 3,        /* a device pointer not 16-byte aligned         */
  QLORA_ERR_NONFINITE = 4,         /* device: non-finite weight seen by quantizer  */
  QLORA_ERR_DEVICE_TIMEOUT = 5,    /* device: a pipeline wait exceeded its bound   */
  QLORA_ERR_CUDA = 6,              /* a CUDA runtime/driver call failed            */
  QLORA_ERR_WORKSPACE = 7,         /* workspace missing or smaller than required   */
  QLORA_ERR_BOUNDS = 8             /* device, debug build only: an index outside its
                                      buffer was caught and the access skipped     */
} qlora_status;

/* The frozen base weight W [rows=N (out), cols=K (in)] in NF4 + double quant.
 * All three arrays are device memory owned by the caller.
 *   codes       : ceil(rows*cols/2) bytes
 *   absmax_q    : ceil(rows*cols/64) bytes, one 8-bit constant per block
 *   group_scale : ceil(rows*cols/16384) fp32, one per group of 256 blocks, and
 *                 with QLORA_DQ_SIGNED one more fp32 after them: the offset mu
 *                 (qlora_group_scale_bytes_dq gives the size)               */
/* 4-bit code tables.  NF4 is the method's type; the other two are the plain
 * 4-bit float and integer types the pages compare it against (the same
 * storage, block constants and kernels, another 16-entry table):
 *   QLORA_FORMAT_NF4   levels at normal quantiles (qlora_nf4_codebook)
 *   QLORA_FORMAT_FP4   e2m1 float: +-{0, 0.5, 1, 1.5, 2, 3, 4, 6} / 6, codes
 *                      0..7 negative (code 7 = -0), 8..15 positive (code 8 = +0;
 *                      nearest-level encoding with ties to the lower index never
 *                      emits code 8)
 *   QLORA_FORMAT_INT4  symmetric integer grid: level[c] = fl32((c - 8) / 7) */
#define QLORA_FORMAT_NF4 0
#define QLORA_FORMAT_FP4 1
#define QLORA_FORMAT_INT4 2

/* Two readings of the 8-bit block constants ("NormalFloat, double
 * quantization, paged optimizers": the per-block constants are themselves
 * stored in 8 bits under a coarser set of constants; the 8-bit format is not
 * given).  a_b is the exact fp32 absmax of block b, g its group of 256 blocks.
 *   QLORA_DQ_PLAIN   unsigned codes, no offset:
 *                      S_g = fl32(max_g a_b / 255),
 *                      q_b = min(255, rne(fl32(a_b / S_g)))      (0 if S_g = 0),
 *                      a'_b = fl32(q_b * S_g)
 *   QLORA_DQ_SIGNED  signed codes around the tensor-wide mean constant:
 *                      mu = fl32(fl64(fl64(exact sum of all a_b) / n_blocks)),
 *                      c_b = fl32(a_b - mu),  S_g = fl32(max_g |c_b| / 127),
 *                      q_b = clamp(rne(fl32(c_b / S_g)), -127, 127) (0 if S_g = 0),
 *                      stored as its int8 bit pattern; a'_b = fl32(fl32(q_b * S_g) + mu).
 *                    The sum is exact (integer arithmetic), so mu, and with it
 *                    every stored byte, does not depend on the order of work. */
#define QLORA_DQ_PLAIN 0
#define QLORA_DQ_SIGNED 1

typedef struct {
  int64_t rows;
  int64_t cols;
  uint8_t *codes;
  uint8_t *absmax_q;
  float *group_scale;
  int32_t format;     /* QLORA_FORMAT_*; 0 (NF4) for a zero-initialised struct */
  int32_t dq;         /* QLORA_DQ_*; 0 (plain) for a zero-initialised struct   */
} qlora_nf4_weight;

/* Sizes in bytes of the three arrays for a rows x cols weight.
 * qlora_group_scale_bytes is the QLORA_DQ_PLAIN size; qlora_group_scale_bytes_dq
 * takes the variant (4 bytes more for QLORA_DQ_SIGNED; 0 for an unknown one). */
size_t qlora_codes_bytes(int64_t rows, int64_t cols);
size_t qlora_absmax_bytes(int64_t rows, int64_t cols);
size_t qlora_group_scale_bytes(int64_t rows, int64_t cols);
size_t qlora_group_scale_bytes_dq(int64_t rows, int64_t cols, int dq);

/* Element types of the weight handed to the quantizer. */
#define QLORA_DTYPE_F32 0    /* IEEE binary32                                   */
#define QLORA_DTYPE_BF16 1   /* bfloat16 bit patterns (uint16_t)                */

/* qlora_quantize_nf4 -- quantize the weights once, up front (in out->format;
 * NF4 unless the caller chose another table; block constants as out->dq).
 * ("Where the memory goes": the base never changes, so it is quantized once,
 * from the 16-bit or 32-bit form it was trained in.)
 *   W     : device [out->rows * out->cols] elements of `dtype`, flat row-major.
 *   dtype : QLORA_DTYPE_F32 or QLORA_DTYPE_BF16 (QLORA_ERR_INVALID_ARG for any
 *           other value).  A bf16 weight is widened to fp32, which is exact,
 *           so it gives the same result as its fp32 copy.
 *   out   : rows/cols set by the caller; codes/absmax_q/group_scale receive the
 *           result.  Any rows*cols >= 1 is accepted (last block/group partial).
 * Per block b: a_b = max|w| (exact fp32); n = fl32(w / a_b) (n = 0 if a_b = 0);
 * code = index of the nearest level of the table, ties to the lower index.
 * The block constants a_b are then stored as QLORA_DQ_* describes.
 * QLORA_DQ_SIGNED needs a workspace: this call returns QLORA_ERR_WORKSPACE for
 * it; use qlora_quantize_nf4_ws.
 * A non-finite weight latches QLORA_ERR_NONFINITE (outputs then undefined). */
qlora_status qlora_quantize_nf4(const void *W, int dtype, const qlora_nf4_weight *out, void *stream);

/* Workspace bytes qlora_quantize_nf4_ws needs (0 for QLORA_DQ_PLAIN; for
 * QLORA_DQ_SIGNED 128 + 4 bytes per block, rounded up to 256). */
size_t qlora_quantize_workspace_bytes(int64_t rows, int64_t cols, int dq);

/* qlora_quantize_nf4_ws -- qlora_quantize_nf4 with a caller-owned device
 * workspace (16-byte aligned, ws_bytes >= qlora_quantize_workspace_bytes;
 * ws may be NULL when that is 0).  For QLORA_DQ_SIGNED it holds the fp32 block
 * constants between the pass that finds them and the pass that codes them
 * against mu, and the exact sum (ten 64-bit words of 32-bit digits, cleared
 * by the call).  rows*cols < 2^38 for QLORA_DQ_SIGNED
 * (QLORA_ERR_UNSUPPORTED_SHAPE beyond). */
qlora_status qlora_quantize_nf4_ws(const void *W, int dtype, const qlora_nf4_weight *out, void *ws,
                                   size_t ws_bytes, void *stream);

/* qlora_dequantize -- W' = bf16(fl32(v_code * a'_b)) into a device bf16 buffer
 * of rows*cols elements, row-major, a'_b the dequantized block constant of
 * w->dq.  ("Where the memory goes": the 16-bit form each pass works with.)
 * Bit-exact by construction. */
qlora_status qlora_dequantize(const qlora_nf4_weight *w, uint16_t *W_out, void *stream);

/* Operation ids for qlora_workspace_bytes(): the linear on a packed weight,
 * and on a dense bf16 weight (qlora_linear_*_dense / _materialized). */
#define QLORA_OP_FWD 0
#define QLORA_OP_BWD 1
#define QLORA_OP_FWD_DENSE 2
#define QLORA_OP_BWD_DENSE 3

/* Workspace bytes for the linear calls at the given sizes, with every kernel
 * path enabled (0 never means "no workspace" for the linear; it is at least
 * 256).  When the fused GEMMs run on CTA pairs (M > 128, or a dense weight)
 * the last part of this workspace holds the stream-K tail of those GEMMs: the
 * fp32 pieces of output tiles that several clusters share when the tiles do
 * not fill whole waves of the device (up to 80 MB for M > 256).  That part is
 * optional: a workspace of qlora_workspace_min_bytes() bytes or more is
 * accepted, and below qlora_workspace_bytes() the GEMMs run without the tail
 * split (same results to rounding, slower when the last wave is partial).
 * Returns 0 for an unknown op or sizes below 1. */
size_t qlora_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r);
size_t qlora_workspace_min_bytes(int op, int64_t M, int64_t N, int64_t K, int r);

/* qlora_linear_fwd -- Y = X W'^T + s (X A^T) B^T   (W' = dequantized base).
 * ("QLoRA" Abstract; "Where the memory goes".)
 *   w      : the NF4 weight, rows = N, cols = K; K % 64 == 0.
 *   X      : device bf16 [M, K];  A : device bf16 [r, K];  B : device bf16 [N, r]
 *   r      : 8 <= r <= 256, r % 8 == 0;  s : the adapter scale alpha / r (finite).
 *   Y      : device bf16 [M, N] (output).
 *   H_out  : optional device fp32 [M, r]; receives H = X A^T for the backward.
 *   ws     : device workspace, 16-byte aligned, of ws_bytes >= qlora_workspace_min_bytes(FWD, ...)
 *            (qlora_workspace_bytes(FWD, ...) for the stream-K tail); QLORA_ERR_WORKSPACE below.
 * N % 8 == 0.  M >= 1.  M <= 16 runs the memory-bound dequant-GEMV path; larger M runs the
 * tensor-core fused dequant-GEMM with the adapter term as an extra K segment of
 * the same accumulation.  fp32 accumulation; Y rounded once to bf16. */
qlora_status qlora_linear_fwd(const qlora_nf4_weight *w, const uint16_t *X, int64_t M,
                              const uint16_t *A, const uint16_t *B, int r, float s,
                              uint16_t *Y, float *H_out, void *ws, size_t ws_bytes,
                              void *stream);

/* qlora_linear_bwd -- gradients of the linear; the frozen W' gets none.
 *   G  = s dY B                 (fp32, internal)
 *   dX = dY W' + G A            device bf16 [M, K]
 *   dA = G^T X                  device fp32 [r, K]
 *   dB = s dY^T (X A^T)         device fp32 [N, r]
 * ("QLoRA" Abstract: gradients flow through the frozen 4-bit model into the
 * adapters; "Where the memory goes": through the dequantized weights.)
 * dB and dA run on a library-owned low-priority stream (one per host thread
 * and device, forked from and joined back into `stream` by events, so the
 * call stays stream-ordered and capturable) beside the dgrad GEMM.
 *   H_saved : optional device fp32 [M, r] from qlora_linear_fwd; NULL makes the
 *             call recompute X A^T.
 * Same shape rules as the forward; M >= 1.  Workspace as for the forward, with
 * QLORA_OP_BWD. */
qlora_status qlora_linear_bwd(const qlora_nf4_weight *w, const uint16_t *X, const uint16_t *dY,
                              int64_t M, const uint16_t *A, const uint16_t *B, int r, float s,
                              const float *H_saved, uint16_t *dX, float *dA, float *dB,
                              void *ws, size_t ws_bytes, void *stream);

/* ---- Linear on a base weight from any quantizer ----------------------------
 * ("ModuLoRA", abstract: a quantization-agnostic backward that materializes the
 * low-precision weights of a black-box quantization module in each pass.)
 * The base W' arrives as a dense bf16 matrix [N, K] (device, row-major) that
 * the caller's dequantizer produced; the same fused tensor-core GEMM, adapter
 * products and precision rules as qlora_linear_fwd / qlora_linear_bwd apply
 * (the operand is copied into the GEMM's shared-memory ring instead of being
 * decoded; the pair kernel serves every M).  With W' = qlora_dequantize(w) the
 * results equal the packed calls' bit for bit whenever those take the pair
 * kernel (M > 128).  Workspace: qlora_workspace_bytes(QLORA_OP_FWD_DENSE /
 * QLORA_OP_BWD_DENSE, M, N, K, r), at least qlora_workspace_min_bytes of the
 * same op.  Shape rules as for the packed calls. */
qlora_status qlora_linear_fwd_dense(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X, int64_t M,
                                    const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y, float *H_out,
                                    void *ws, size_t ws_bytes, void *stream);
qlora_status qlora_linear_bwd_dense(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X, const uint16_t *dY,
                                    int64_t M, const uint16_t *A, const uint16_t *B, int r, float s,
                                    const float *H_saved, uint16_t *dX, float *dA, float *dB, void *ws,
                                    size_t ws_bytes, void *stream);

/* The black-box boundary itself: `materialize(ctx, W_out, N, K, stream)`
 * enqueues, on `stream`, whatever writes the bf16 base weight [N, K] into the
 * device buffer W_out and returns QLORA_OK (any other status aborts the call
 * and is returned).  The _materialized calls run it into the caller's scratch
 * buffer W_scratch (2 N K bytes, 16-byte aligned) and then the dense linear, so
 * the full-precision weight exists only for the duration of one pass. */
typedef qlora_status (*qlora_materialize_fn)(void *ctx, uint16_t *W_out, int64_t N, int64_t K, void *stream);
qlora_status qlora_linear_fwd_materialized(qlora_materialize_fn materialize, void *ctx, uint16_t *W_scratch,
                                           int64_t N, int64_t K, const uint16_t *X, int64_t M, const uint16_t *A,
                                           const uint16_t *B, int r, float s, uint16_t *Y, float *H_out, void *ws,
                                           size_t ws_bytes, void *stream);
qlora_status qlora_linear_bwd_materialized(qlora_materialize_fn materialize, void *ctx, uint16_t *W_scratch,
                                           int64_t N, int64_t K, const uint16_t *X, const uint16_t *dY, int64_t M,
                                           const uint16_t *A, const uint16_t *B, int r, float s,
                                           const float *H_saved, uint16_t *dX, float *dA, float *dB, void *ws,
                                           size_t ws_bytes, void *stream);

/* Size of the library-owned scratch array used by qlora_linear_fwd_noalloc(). */
#define QLORA_STATIC_SCRATCH_BYTES (8u << 20)

/* qlora_linear_fwd_noalloc -- the same forward as qlora_linear_fwd, for
 * callers that cannot allocate device memory (code running where cudaMalloc
 * is unavailable or forbidden: custom allocator hooks, runtimes with a memory
 * map fixed at start-up, plugin hosts that own every allocation).  The pages
 * have no counterpart of this call; it is a deployment convenience.
 *   Arguments as qlora_linear_fwd, minus the workspace.  The scratch is a
 *   QLORA_STATIC_SCRATCH_BYTES array inside the library, held on every GPU that
 *   loads the library until the process exits; the call allocates and frees
 *   nothing.
 *   Returns QLORA_ERR_WORKSPACE (nothing enqueued) when
 *   qlora_workspace_min_bytes(QLORA_OP_FWD, M, N, K, r) exceeds
 *   QLORA_STATIC_SCRATCH_BYTES.  That minimum grows with M r and does not
 *   depend on N or K: at r = 64 it is about 2.4 KB per token (the adapter
 *   product's fp32 partial sums, in whole 128-token tiles), so M <= 3413 fits
 *   (M = 2048, r = 64 fits; M = 4096, r = 64 does not); at r = 256, M <= 862.
 *   The fused GEMM always runs without its stream-K tail here (that optional
 *   workspace region is about 80 MB for M > 128), so a partial last wave of
 *   tiles is not split.
 *   The first call on a device looks up the array's device address; make that
 *   first call before any stream capture.  Every call shares the one array
 *   (it keeps the previous call's contents; nothing needs clearing), so calls
 *   that overlap on the GPU race: serialize them on one stream.  Like every
 *   entry point here, it must not be called from a stream host callback
 *   (cudaLaunchHostFunc), where CUDA calls are not allowed. */
qlora_status qlora_linear_fwd_noalloc(const qlora_nf4_weight *w, const uint16_t *X, int64_t M,
                                      const uint16_t *A, const uint16_t *B, int r, float s,
                                      uint16_t *Y, float *H_out, void *stream);

/* The 16 NF4 levels (ascending, fp32) as the library computes them on the
 * host: standard-normal quantiles at 8 positive and 7 negative equally spaced
 * probabilities from d = 1 - (1/32 + 1/30)/2 to 1/2, plus an exact 0,
 * normalised to [-1, 1].  ("NormalFloat, double quantization, paged
 * optimizers": 16 levels at normal quantiles.)  out: host float[16]. */
qlora_status qlora_nf4_codebook(float *out);

/* The 16 fp32 levels of any QLORA_FORMAT_* table (ascending), and the 15 fp32
 * decision thresholds the quantizer compares against: code = #{ i : n >
 * thresh[i] }, thresh[i] = the midpoint of level[i] and level[i+1] rounded
 * toward -inf (for two equal levels, the next threshold).  levels: host
 * float[16]; thresh: host float[15] or NULL.  QLORA_ERR_INVALID_ARG for an
 * unknown format or a NULL levels pointer. */
qlora_status qlora_format_codebook(int format, float *levels, float *thresh);

/* ---- Low-rank plus quantized decomposition ------------------------------
 * ("LQ-LoRA: Low-rank Plus Quantized Matrix Decomposition for Efficient
 * Language Model Finetuning", abstract: an iterative algorithm splits each
 * pretrained matrix into a high-precision low-rank part and a quantized part;
 * finetuning keeps the quantized part fixed and trains the low-rank one.)
 *
 * qlora_lq_decompose -- W ~ W'(Q) + L1 L2.  Starts from the principal rank-r
 * part of W, then `iters` rounds of
 *     E = fl32(fl64(W) - P)  (P = L1 L2 summed in fp64 over j = 0 .. r-1),
 *     Q = qlora_quantize_nf4(E) in Q->format / Q->dq,
 *     L1 L2 = rank-r approximation of R = fl32(W - W'(Q)).
 * The rank-r step is randomized subspace iteration on R: Y = orth(R Omega),
 * `power` times Y = orth(R orth(R^T Y)), B = Y^T R, B B^T = U diag(lam) U^T
 * (lam descending), s = sqrt(lam[:r]), L1 = Y U_r diag(sqrt(s)),
 * L2 = diag(1/sqrt(s)) U_r^T B; components with s_i <= 1e-12 s_0 are zero.
 * orth() is Cholesky QR done twice; the l x l steps run in fp64.
 *   W     : device fp32 [N, K] (N = Q->rows, K = Q->cols), not modified.
 *   Q     : the weight header; its arrays receive the final quantized part
 *           (sized for Q->dq, as for qlora_quantize_nf4).
 *   L1    : device fp32 [N, r];  L2 : device fp32 [r, K]  (outputs).
 *   Omega : device fp32 [K, l] Gaussian test matrix (the random numbers the
 *           method draws; the caller supplies them).  r <= l <= 96, l a
 *           multiple of 4 (16-byte rows),
 *           N >= l, K >= l.  0 <= power <= 16, 1 <= iters <= 1000.
 *   err   : device fp64 [2 iters]: err[2t] = ||W - W' - L1 L2||_F / ||W||_F
 *           after round t's quantization, err[2t+1] after its rank-r step.
 *   ws    : device workspace of qlora_lq_workspace_bytes(N, K, r, l, Q->dq)
 *           bytes (about 4 N K + 8 (N + K) l bytes).
 * Every reduction is split over CTAs with parts added in a fixed order: the
 * same inputs give the same bits.  Returns QLORA_ERR_UNSUPPORTED_SHAPE for
 * N < l, K < l or K % 64 != 0 (the rank-r step walks whole 64-element blocks). */
size_t qlora_lq_workspace_bytes(int64_t rows, int64_t cols, int r, int l, int dq);

/* qlora_lq_quantize_residual -- one quantization step of the decomposition:
 * Q = qlora_quantize_nf4(fl32(fl64(W) - P)), P = L1 L2 summed in fp64 over
 * j = 0 .. r-1 (each product of two fp32 values is exact in fp64).  W fp32
 * [N, K], L1 fp32 [N, r], L2 fp32 [r, K] (device); Q as for the quantizer.
 * ws: qlora_lq_workspace_bytes(N, K, r, 0, Q->dq) bytes or more.  Bit-exact. */
qlora_status qlora_lq_quantize_residual(const float *W, const float *L1, const float *L2, int r,
                                        const qlora_nf4_weight *Q, void *ws, size_t ws_bytes, void *stream);

/* qlora_lq_lowrank -- one rank-r step: L1 L2 ~ R with R = fl32(W - W'(Q)), or
 * R = W when Q is NULL, by the randomized subspace iteration described above
 * (Omega [cols, l], `power` rounds).  rows/cols give W's shape (and must match
 * Q's).  ws: qlora_lq_workspace_bytes(rows, cols, r, l, dq) bytes or more. */
qlora_status qlora_lq_lowrank(const float *W, int64_t rows, int64_t cols, const qlora_nf4_weight *Q,
                              const float *Omega, int l, int power, int r, float *L1, float *L2, void *ws,
                              size_t ws_bytes, void *stream);

qlora_status qlora_lq_decompose(const float *W, const qlora_nf4_weight *Q, float *L1, float *L2, int r,
                                const float *Omega, int l, int power, int iters, double *err, void *ws,
                                size_t ws_bytes, void *stream);

/* Synchronize `stream`, return the latched device status and clear it. */
qlora_status qlora_device_status(void *stream);

/* Human-readable name of a status code (static string). */
const char *qlora_status_string(qlora_status st);

/* Upper bound, in GPU clock cycles, on every pipeline wait inside the
 * library's kernels (default 2e9, about one second).  Returns the old value. */
uint64_t qlora_set_wait_limit(uint64_t cycles);

/* When the fused GEMM's pair tiles leave a last, partial wave of cluster slots,
 * the K-steps of those tiles can be split evenly over all slots (stream-K; the
 * clusters sharing a tile add their fp32 pieces in a fixed order, so results
 * repeat bit for bit).  Each split costs its clusters about 33 K-steps of
 * drain, piece traffic and refill (measured on B200), so AUTO splits only when
 * a cluster's share plus that cost is shorter than a whole tile plus its own
 * fill and drain (about 8 K-steps); ALWAYS splits whenever the last wave is
 * partial; OFF never splits.  The split needs the workspace's optional tail
 * (qlora_workspace_bytes).  Returns the previous mode, or -1 (mode unchanged)
 * for an unknown one.  Process-wide; takes effect at the next launch. */
#define QLORA_STREAM_K_OFF 0
#define QLORA_STREAM_K_AUTO 1
#define QLORA_STREAM_K_ALWAYS 2
int qlora_set_stream_k(int mode);

/* Self-test of the bounded wait: launches one block that waits on a barrier
 * nothing ever signals, with a bound of `cycles`.  The wait must give up and
 * latch QLORA_ERR_DEVICE_TIMEOUT (read it with qlora_device_status()). */
qlora_status qlora_selftest_wait_timeout(uint64_t cycles, void *stream);

/* Kernel timing for benchmarks.  While enabled, the library records a CUDA
 * event pair on the launch stream around each of its own kernel launches and
 * counts the launches, per kind:
 *   0 all kernels, 1 fused dequant-GEMM forward, 2 fused dequant-GEMM dgrad,
 *   3 adapter (low-rank) GEMMs and their reductions, 4 quantizer,
 *   5 dequantizer, 6 dequant-GEMV; the decomposition (qlora_lq_*): 7 the
 *   residual products R M and R^T Y, 8 the low-rank residual and error
 *   kernel, 9 Cholesky and triangular inverse, 10 Jacobi eigen-decomposition,
 *   11 Gram, small-factor and split-sum kernels.
 * While recording, the backward keeps every launch on the caller's stream
 * (no side stream), so each event pair times its kernel alone.
 * qlora_profile_enable(1) clears the records; qlora_profile_read()
 * synchronizes the device and returns the summed event time (ms) and the
 * launch count of one kind.  Not thread-safe; off by default. */
void qlora_profile_enable(int on);
qlora_status qlora_profile_read(int kind, double *ms_total, int64_t *launches);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
