/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so, the sm_100a (B200) hot path of a
 * QLoRA linear layer:
 *   (1) blockwise NF4 quantization of a frozen fp32 weight W0,
 *   (2) double quantization (DQ) of the per-block constants,
 *   (3) doubleDequant to BF16, and the fused forward / backward of
 *           Y = X * doubleDequant(W0)^T + s * (X A^T) B^T.
 *
 * The method is described on these web pages (cited per entry point):
 *   "LoRA 与 QLoRA" (whoami-wesleyyou.top): section LoRA, section QLoRA
 *       "1. NF4" and "2. Double Quantization (DQ)".
 *   "QLoRA: Efficient Finetuning of Quantized LLMs", deck "3 QLoRA Finetuning"
 *       (learn.ifs.name), cards 1-4.
 *   jjjymmm.cn 2024/03 QLoRA post: "4-bit NormalFloat(NF4)", "Double
 *       Quantization", "QLoRA" (doubleDequant).
 *   "QLoRA：4-bit 量化与显存账" (finetune.xph.ink kp-007): the
 *       BitsAndBytesConfig flag set (load_in_4bit, nf4, use_double_quant,
 *       compute dtype bf16) that this ABI mirrors.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers, owned by the caller.  The library
 *   never allocates, frees or synchronises; every call enqueues its kernels on
 *   `stream` (a cudaStream_t passed as void*; NULL = legacy default stream) and
 *   returns.  Outputs are overwritten, never accumulated into.
 * - BF16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 * - Layouts are row-major and dense.  Tokens are the leading dimension of the
 *   activations: X [n][din], Y [n][dout], dY [n][dout], dX [n][din],
 *   U = X A^T [n][r].  Weights: W0 [dout][din] (rows = dout, cols = din),
 *   A [r][din], B [dout][r], dA [r][din] fp32, dB [dout][r] fp32.
 * - NF4 storage of a [rows][cols] weight, numel = rows*cols, flattened
 *   row-major, blocks of 64 consecutive elements (nb = numel/64):
 *     codes  uint8 [numel/2]: element 2i in the HIGH nibble of byte i,
 *                             element 2i+1 in the low nibble;
 *     absmax fp32  [nb]     : a_j = max |w| over block j (plain NF4);
 *     qabs   int8  [nb]     : DQ code rhat_j of a_j;
 *     dq_scale fp32 [ng]    : DQ step b_g per group of 256 blocks,
 *                             ng = ceil(nb/256);
 *     dq_mean fp32 [1]      : mu, the mean of all a_j.
 * - Synchronous argument errors are returned BEFORE anything is launched:
 *   NULL pointers (QLN_ERR_NULL), bad sizes (QLN_ERR_SHAPE), pointers not
 *   16-byte aligned (QLN_ERR_ALIGN), workspace too small (QLN_ERR_WORKSPACE),
 *   current device not sm_100 (QLN_ERR_ARCH).  A failed launch returns
 *   QLN_ERR_CUDA (cudaGetLastError).  Kernels that wait (on TMA barriers, on
 *   a thread-block cluster, on the grid-wide barrier of the single-launch
 *   double quantization) give up after a bounded time and write
 *   QLN_ERR_TIMEOUT into the int32 status word at byte offset 0 of the
 *   workspace; read it after the stream has synchronised (0 = QLN_OK).  Each
 *   workspace call clears it.
 * - Bytes 4..255 of a double-quantization workspace hold a generation word,
 *   a counter and two banks for the exact sum of mu.  Zero-fill a workspace
 *   once before its first use and leave it to the library afterwards: each
 *   call sums into the bank the generation selects, zeroes the other one and
 *   advances the generation, so every call finds what it needs zeroed (also
 *   across CUDA graph replays).  After a call that reported QLN_ERR_TIMEOUT,
 *   zero the first 256 bytes again.  The linear forward and backward keep no state in the
 *   workspace between calls.
 * - No entry point creates streams or events or synchronises the host: each
 *   enqueues its kernels on the caller's stream, in order, and returns.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLN_API __attribute__((visibility("default")))
#else
#define QLN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QLN_OK = 0,
    QLN_ERR_NULL = 1,      /* a required pointer is NULL                       */
    QLN_ERR_SHAPE = 2,     /* a size is out of range or not a multiple of 64   */
    QLN_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned                 */
    QLN_ERR_WORKSPACE = 4, /* ws_bytes below qln_workspace_bytes(...)          */
    QLN_ERR_ARCH = 5,      /* current device is not compute capability 10.x    */
    QLN_ERR_CUDA = 6,      /* a CUDA runtime call or launch failed             */
    QLN_ERR_TIMEOUT = 7,   /* device side: a bounded barrier wait gave up      */
    QLN_ERR_INTERNAL = 8   /* device side: an internal consistency check failed*/
} qln_status;

/* Formats of the 8-bit double-quantized block constants (qabs). */
enum { QLN_DQ_INT8 = 0, QLN_DQ_E4M3 = 1 };

/* Element types of the weights given to nf4_quantize_ex. */
enum { QLN_DTYPE_F32 = 0, QLN_DTYPE_BF16 = 1, QLN_DTYPE_F16 = 2 };

/* Workspace-sized operations (qln_workspace_bytes `op`). */
enum { QLN_OP_DOUBLE_QUANT = 1, QLN_OP_LINEAR_FWD = 2, QLN_OP_LINEAR_BWD = 3, QLN_OP_QUANTIZE_DQ_BATCH = 4 };

/* An NF4 weight as stored by nf4_quantize (+ nf4_double_quant).  All pointers
 * are device pointers owned by the caller.  With qabs != NULL the weight is
 * double-quantized (qabs, dq_scale, dq_mean are used, absmax is ignored);
 * with qabs == NULL the plain fp32 absmax is used (bnb_4bit_use_double_quant
 * off).  cols must be a multiple of 64, so blocks never straddle rows.
 * dq_format says how qabs is stored: QLN_DQ_INT8 (0, signed int8, as written
 * by nf4_double_quant) or QLN_DQ_E4M3 (1, OCP FP8 E4M3 codes, as written by
 * nf4_double_quant_ex with that format); a zero-initialized struct is INT8. */
typedef struct {
    const uint8_t *codes;
    const float *absmax;
    const int8_t *qabs;
    const float *dq_scale;
    const float *dq_mean;
    int64_t rows; /* dout */
    int64_t cols; /* din  */
    int32_t dq_format;
} qln_nf4_weight;

/*
 * nf4_quantize -- blockwise NF4 quantization.
 * Defined by: jjjymmm.cn "4-bit NormalFloat(NF4)" (divide by the block
 * ABSMAX, snap to the nearest quant-book entry); "LoRA 与 QLoRA" section 2
 * (a_j = max |W_j| per block of 64); deck "3 QLoRA Finetuning" cards 2-3 (the
 * asymmetric 16-entry NormalFloat book with an exact zero and ends at +-1).
 *   W      [numel] fp32 in : weights, flattened row-major.
 *   codes  [numel/2] u8 out, absmax [numel/64] fp32 out.
 * Per element x = fp32(w / a_j) (IEEE division, round to nearest) and the
 * code is the nearest of the 16 entries, ties to the lower code; a block with
 * a_j == 0 gets code 7 (the exact zero) throughout.  Non-finite inputs are
 * not checked (undefined codes).
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE if numel <= 0 or numel % 64 != 0;
 * QLN_ERR_ALIGN if W or codes is not 16-byte aligned (absmax: 4-byte).
 */
QLN_API qln_status nf4_quantize(const float *W, int64_t numel, uint8_t *codes, float *absmax,
                        void *stream);

/*
 * nf4_quantize_ex -- nf4_quantize for 16-bit weights and for any numel.
 * Checkpoints usually hold 16-bit weights ("LoRA 与 QLoRA", QLoRA usage notes:
 * load the 16-bit model, then quantize).  Every bf16 or fp16 value is exactly
 * an fp32 value, and that value is what gets quantized, so the result equals
 * nf4_quantize of the weights widened to fp32, bit for bit.
 *   W      [numel] in, element type `dtype` (QLN_DTYPE_F32, _BF16, _F16),
 *          flattened row-major; numel >= 1, any value.
 *   codes  [ceil(numel/2)] u8 out; absmax [ceil(numel/64)] fp32 out.
 * Tails: the last block holds the numel mod 64 remaining weights (its absmax
 * is over those); for odd numel the low nibble of the last byte is 7, the
 * code a zero weight gets -- the same bytes as quantizing W zero-padded to
 * whole blocks.  No byte of codes past ceil(numel/2) is written.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE if numel <= 0 or dtype is unknown;
 * QLN_ERR_ALIGN if W or codes is not 16-byte aligned (absmax: 4-byte).
 */
QLN_API qln_status nf4_quantize_ex(const void *W, int32_t dtype, int64_t numel, uint8_t *codes, float *absmax,
                                   void *stream);

/*
 * nf4_double_quant -- quantize the block constants to 8 bits.
 * Defined by: "LoRA 与 QLoRA" section 2 (r_j = (a_j - mu)/b, 8-bit rhat_j,
 * ahat_j = mu + b rhat_j, mu and b stored in 32 bits); deck card 4 and
 * jjjymmm.cn "Double Quantization" (blocks of 256 constants).
 *   absmax   [nb] fp32 in;  qabs [nb] int8 out;  dq_scale [ceil(nb/256)] fp32
 *   out;  dq_mean [1] fp32 out.
 * mu = the binary32 value nearest to the exact mean (1/nb) sum_j a_j, ties
 * to even: the sum is formed exactly in integer arithmetic, so mu does not
 * depend on the order of summation, the grid or the device.  Per group g:
 * d_j = fp32(a_j - mu), b_g = fp32(max|d_j| / 127),
 * rhat_j = clamp(rint(fp32(d_j / b_g)), -127, 127) (ties to even), 0 when
 * b_g == 0.  The last group may be partial.
 *   ws / ws_bytes: device scratch of at least
 *   qln_workspace_bytes(QLN_OP_DOUBLE_QUANT, nb, 0, 0, 0) (= 256) bytes,
 *   256-byte aligned: a status word at offset 0 (QLN_OK, or QLN_ERR_TIMEOUT
 *   when a bounded device wait gave up), the counters of the single-launch
 *   path's grid barrier and the exact sum.  Zero it once before the first
 *   call and then leave it to the library (zero it anew after a
 *   QLN_ERR_TIMEOUT).
 * Weights of up to about 310 M parameters take a single cooperative launch
 * whose CTAs meet at a grid-wide barrier: every CTA is resident at once, so a
 * kernel on another stream can only delay it, and a wait longer than 2 s
 * ends with QLN_ERR_TIMEOUT in the status word instead of a hang.  Larger
 * weights take two launches that do not wait on one another.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE if nb <= 0 or nb > 2^25 (numel above
 * 2^31); QLN_ERR_WORKSPACE; QLN_ERR_ALIGN if absmax is not 16-byte aligned or
 * ws is not 256-byte aligned.
 */
QLN_API qln_status nf4_double_quant(const float *absmax, int64_t nb, int8_t *qabs, float *dq_scale,
                            float *dq_mean, void *ws, size_t ws_bytes, void *stream);

/*
 * nf4_double_quant_ex -- nf4_double_quant with a choice of 8-bit format.
 * The pages disagree on the 8-bit format of the quantized constants: deck
 * "3 QLoRA Finetuning" card 4 says 8-bit floats, jjjymmm.cn "Double
 * Quantization" says INT8.  dq_format QLN_DQ_INT8 is nf4_double_quant;
 * QLN_DQ_E4M3 stores OCP FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, largest finite value 448, no infinities):
 *   b_g = fp32(max|d_j| / 448), rhat_j = E4M3(fp32(d_j / b_g)) rounded to
 *   nearest-even and saturated to +-448; code 0 when b_g == 0.
 * mu is the same as for INT8.  Set qln_nf4_weight.dq_format to the same value
 * when the result is used.  qabs [nb] bytes out; other arguments, workspace
 * and errors as nf4_double_quant, plus QLN_ERR_SHAPE for an unknown format.
 */
QLN_API qln_status nf4_double_quant_ex(const float *absmax, int64_t nb, int32_t dq_format, void *qabs,
                                       float *dq_scale, float *dq_mean, void *ws, size_t ws_bytes, void *stream);

/*
 * nf4_quantize_dq -- nf4_quantize_ex followed by nf4_double_quant_ex, as one
 * call with the same bits.  Defined by the two passages those entry points
 * cite: "LoRA 与 QLoRA" section QLoRA (blockwise NF4 with absmax, then the
 * double quantization of the block constants).
 *   W [numel] of dtype in; codes [ceil(numel/2)], absmax [nb], qabs [nb],
 *   dq_scale [ceil(nb/256)], dq_mean [1] out, nb = ceil(numel/64); dq_format
 *   QLN_DQ_INT8 or QLN_DQ_E4M3 (as nf4_double_quant_ex).
 * The two steps are enqueued back to back, the second as a programmatic
 * dependent of the first, with the double quantization's launch shapes (its
 * single cooperative launch where that fits).  W must be finite (mu of
 * non-finite constants is not defined).
 *   ws / ws_bytes: a double-quantization workspace (qln_workspace_bytes
 *   QLN_OP_DOUBLE_QUANT, 256 bytes), zeroed once before the first call and
 *   then left to the library; byte 0 is the status word.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE (numel <= 0 or above 2^31, unknown
 * dtype or format); QLN_ERR_ALIGN (W, codes, absmax 16-byte; ws 256-byte);
 * QLN_ERR_WORKSPACE; QLN_ERR_ARCH.
 */
QLN_API qln_status nf4_quantize_dq(const void *W, int32_t dtype, int64_t numel, int32_t dq_format, uint8_t *codes,
                                   float *absmax, void *qabs, float *dq_scale, float *dq_mean, void *ws,
                                   size_t ws_bytes, void *stream);

/* One weight of nf4_quantize_dq_batch: the arguments of nf4_quantize_dq. */
typedef struct {
    const void *W;     /* [numel] weights of dtype, 16-byte aligned */
    int64_t numel;     /* 1 .. 2^31 */
    int32_t dtype;     /* QLN_DTYPE_F32, _BF16 or _F16 */
    int32_t dq_format; /* QLN_DQ_INT8 or QLN_DQ_E4M3 */
    uint8_t *codes;    /* [ceil(numel/2)] out, 16-byte aligned */
    float *absmax;     /* [nb] out, nb = ceil(numel/64), 16-byte aligned */
    void *qabs;        /* [nb] out (int8 or E4M3 codes) */
    float *dq_scale;   /* [ceil(nb/256)] out */
    float *dq_mean;    /* [1] out */
} qln_quant_job;

/*
 * nf4_quantize_dq_batch -- nf4_quantize_dq of njobs weights in one call, the
 * same bits as calling it for each job in order.  This is how a whole model is
 * quantized for QLoRA ("LoRA 与 QLoRA" section QLoRA: every frozen weight
 * stored as NF4 with double-quantized constants).
 * When no job's outputs overlap another job's buffers, the quantize launches
 * run back to back (each one starts while the one before it drains) and the
 * double quantization of all jobs follows in two launches per 128 jobs (the
 * exact sums, then the groups), so that its latency is paid once per call
 * rather than once per weight.  Otherwise each weight's quantize is followed
 * by its own two double-quantization launches before the next weight's, as
 * separate calls would run.  Either way every launch reads only what earlier
 * launches completed, so the jobs' buffers may be laid out in any way that
 * separate nf4_quantize_dq calls allow.
 *   ws / ws_bytes: qln_workspace_bytes(QLN_OP_QUANTIZE_DQ_BATCH, njobs, 0, 0,
 *   0) = 256 * njobs bytes, 256-byte aligned, zeroed once before the first
 *   call and then left to the library (job i uses bytes 256 i .. 256 i + 255
 *   as its double-quantization scratch); byte 0 holds QLN_OK afterwards (no
 *   launch of this call waits on anything).
 * Errors: QLN_ERR_NULL (jobs, ws, or a job pointer); QLN_ERR_SHAPE (njobs < 1
 * or above 2^20, or a job's sizes, dtype or format); QLN_ERR_ALIGN;
 * QLN_ERR_WORKSPACE; QLN_ERR_ARCH.  Every job is checked before anything is
 * launched.
 */
QLN_API qln_status nf4_quantize_dq_batch(const qln_quant_job *jobs, int32_t njobs, void *ws, size_t ws_bytes,
                                         void *stream);

/*
 * nf4_double_quant_noalloc -- nf4_double_quant without a caller workspace.
 * The pages describe nothing like it: it exists for callers that cannot
 * allocate device memory at the point where they quantize -- for example a
 * runtime that reserves all device memory up front in its own pool and
 * forbids further cudaMalloc, or a plugin that only receives tensors from a
 * host framework and has no allocator of its own.  It computes exactly what
 * nf4_double_quant computes (the same bits) and allocates nothing:
 * it calls no cudaMalloc, cudaFree or other allocating routine.
 *   Scratch: a 256-byte array at file scope in the library (a generation
 *   word, a counter and the exact sum of mu), present on every GPU that loads it
 *   until the process exits.  It always takes the two-launch path, whose
 *   kernels never wait on one another.
 *   Limit: nb <= 2^25 block constants, as nf4_double_quant; larger nb returns
 *   QLN_ERR_SHAPE before anything is launched.
 *   Set-up: the first call in a CUDA context looks up the array's device
 *   address (cudaGetSymbolAddress, with that device current) and caches it
 *   with the context; make that first call before any stream capture in that
 *   context.
 *   Sharing: every call uses the same array; each leaves the part the next
 *   call sums into zeroed, so nothing carries over from call to call.  Calls
 *   that overlap on the GPU (e.g. on two unordered streams) race on it and
 *   must be serialised by the caller.
 * Arguments and outputs as nf4_double_quant.  Errors: QLN_ERR_NULL,
 * QLN_ERR_SHAPE, QLN_ERR_ALIGN, QLN_ERR_ARCH, QLN_ERR_CUDA.
 */
QLN_API qln_status nf4_double_quant_noalloc(const float *absmax, int64_t nb, int8_t *qabs, float *dq_scale,
                                            float *dq_mean, void *stream);

/*
 * nf4_dequant -- doubleDequant of a whole weight to BF16.
 * Defined by: jjjymmm.cn "QLoRA" (restore the quantization constant first,
 * then dequantize the weight with it; a code dequantizes to its quant-book
 * value); deck card 1 (weights are dequantized to BFloat16 for the matmul).
 *   out [rows*cols] bf16 (uint16) out:  w' = bf16_RN(fp32(ahat_j * c[q])),
 *   ahat_j = fp32(mu + fp32(b_g * rhat_j)) with DQ, a_j without.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE (rows, cols <= 0, cols % 64);
 * QLN_ERR_ALIGN (codes, out).
 */
QLN_API qln_status nf4_dequant(const qln_nf4_weight *w, uint16_t *out, void *stream);

/*
 * nf4_dequant_flat -- nf4_dequant of a flat weight of any numel (as written
 * by nf4_quantize_ex).  w->rows and w->cols are ignored; blocks are 64
 * consecutive weights of the flat array and the last may be partial.
 *   out [numel] bf16 (uint16) out; nothing past numel is written.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE if numel <= 0; QLN_ERR_ALIGN (codes,
 * out: 16-byte).
 */
QLN_API qln_status nf4_dequant_flat(const qln_nf4_weight *w, int64_t numel, uint16_t *out, void *stream);

/*
 * qlora_linear_fwd -- fused QLoRA linear forward.
 * Defined by: "LoRA 与 QLoRA" section LoRA (y = W0 x + s B(A x); A x is
 * formed first, BA never is) and section QLoRA "1. NF4" (4-bit weight ->
 * dequant -> BF16 -> GEMM); jjjymmm.cn "QLoRA" (the forward dequantizes W
 * twice, from NF4 to BF16, and multiplies with BF16 X).
 *   X [n][din] bf16 in, A [r][din] bf16 in, B [dout][r] bf16 in, s scale,
 *   Y [n][dout] bf16 out = bf16_RN(X W'^T + s U B^T) with fp32 accumulation,
 *   U_out [n][r] bf16 out (nullable): U = bf16_RN(X A^T), unscaled, for reuse
 *   by qlora_linear_bwd.
 * W' is decoded tile by tile on chip and never written to HBM.  For n <= 32
 * the whole call is one launch of thread-block clusters (U, the weight
 * stream and the adapter term); its split-K sums are folded in an order fixed
 * by the shape, so results do not depend on timing or on the device's SM
 * count.
 *   ws: at least qln_workspace_bytes(QLN_OP_LINEAR_FWD, dout, din, n, r)
 *   bytes, 256-byte aligned; byte 0 holds the device status word afterwards.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE (n < 1; r not a multiple of 8 in
 * 8..128; rows (dout) or cols (din) not a multiple of 64); QLN_ERR_ALIGN
 * (16-byte: codes, X, A, B, Y, U_out; ws 256-byte); QLN_ERR_WORKSPACE;
 * QLN_ERR_ARCH.
 */
QLN_API qln_status qlora_linear_fwd(const qln_nf4_weight *w, const uint16_t *X, int64_t n,
                            const uint16_t *A, const uint16_t *B, int32_t r, float s,
                            uint16_t *Y, uint16_t *U_out, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * qlora_linear_bwd -- fused QLoRA linear backward.
 * Defined by: deck card 1 (gradients flow through the dequantized weights;
 * only the adapters receive updates); "LoRA 与 QLoRA" section LoRA (W0 fixed,
 * only A and B trained); jjjymmm.cn "QLoRA" (backward updates only the LoRA
 * factors).  For Y = X W'^T + s (X A^T) B^T and upstream gradient dY:
 *   G  = dY B                 [n][r]    (kept in the workspace, bf16)
 *   dX = dY W' + s G A        [n][din]  bf16 out
 *   dA = s G^T X              [r][din]  fp32 out
 *   dB = s dY^T U             [dout][r] fp32 out, U = X A^T
 * U (nullable) is the U_out of the matching forward; when NULL it is
 * recomputed.  W0 gets no gradient.
 * ws: at least qln_workspace_bytes(QLN_OP_LINEAR_BWD, dout, din, n, r) bytes.
 * Errors: as qlora_linear_fwd, plus QLN_ERR_NULL for dY, dX, dA, dB.
 */
QLN_API qln_status qlora_linear_bwd(const qln_nf4_weight *w, const uint16_t *X, int64_t n,
                            const uint16_t *A, const uint16_t *B, int32_t r, float s,
                            const uint16_t *dY, const uint16_t *U, uint16_t *dX, float *dA,
                            float *dB, void *ws, size_t ws_bytes, void *stream);

/* AdamW hyper-parameters (fp32, as the update computes in fp32). */
typedef struct {
    float lr;
    float beta1;
    float beta2;
    float eps;
    float weight_decay;
} qln_adamw_config;

/* qln_adamw_step flags. */
enum { QLN_ADAMW_PAGE_IN = 1, QLN_ADAMW_PAGE_OUT = 2 };

/*
 * qln_adamw_step -- one AdamW update of a LoRA factor (the paged optimizer).
 * Defined by: deck "3 QLoRA Finetuning" card 5 (paged optimizers keep the
 * optimizer states in NVIDIA unified memory, paged out to CPU RAM when the
 * GPU runs short and paged back for the update) and card 1 (only the adapter
 * parameters are updated); "LoRA 与 QLoRA" QLoRA usage notes
 * (paged_adamw_32bit).  The pages do not write AdamW out; this is the
 * published one (Loshchilov & Hutter, ICLR 2019), decay first:
 *   m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;  p = p (1 - lr wd);
 *   p = p - (lr / (1 - b1^t)) m / (sqrt(v / (1 - b2^t)) + eps),
 * evaluated in fp32 per element (bias corrections in binary64).
 *   param  [n] fp32 in/out: the factor's master copy (A or B, flattened).
 *   grad   [n] fp32 in: its gradient (dA or dB from qlora_linear_bwd).
 *   m, v   [n] fp32 in/out: the 32-bit AdamW states, zero before step 1.
 *   param_bf16 [n] bf16 out or NULL: RN(param) after the update, the copy the
 *          forward reads.
 *   step   device pointer to the step number t >= 1 being taken (read by the
 *          kernel, so a captured CUDA graph can be replayed step after step
 *          while the caller increments it).
 *   step   values below 1 are taken as 1.
 *   flags  QLN_ADAMW_PAGE_IN: operands that live in managed memory are
 *          prefetched to the current device before the update;
 *          QLN_ADAMW_PAGE_OUT: m and v, if managed, are prefetched back to
 *          host RAM after it.  Memory of any other kind is left alone.  The
 *          prefetches are stream operations of their own: pass 0 while the
 *          stream is being captured into a CUDA graph.
 * Any pointer may be managed (cudaMallocManaged) or device memory.
 * Errors: QLN_ERR_NULL; QLN_ERR_SHAPE if n <= 0; QLN_ERR_ALIGN if param,
 * grad, m or v is not 16-byte aligned (param_bf16: 8-byte).
 */
QLN_API qln_status qln_adamw_step(float *param, const float *grad, float *m, float *v, uint16_t *param_bf16,
                                  int64_t n, const qln_adamw_config *cfg, const int64_t *step, int32_t flags,
                                  void *stream);

/* Device workspace, in bytes, that `op` needs for these sizes (nb for
 * QLN_OP_DOUBLE_QUANT and the job count for QLN_OP_QUANTIZE_DQ_BATCH are
 * passed as `rows`).  Returns 0 for an unknown op. */
QLN_API size_t qln_workspace_bytes(int32_t op, int64_t rows, int64_t cols, int64_t n, int32_t r);

/* The 16 NF4 values (fp32, ascending) the kernels snap to and decode with. */
QLN_API void qln_codebook(float out16[16]);

/* Human-readable name of a status code (static string). */
QLN_API const char *qln_status_str(qln_status st);

/* ABI version: (major << 16) | minor. */
QLN_API int32_t qln_version(void);

/* Number of kernels this library has enqueued since it was loaded, over all
 * threads and devices (a host-side counter; cudaMemsetAsync of the status word
 * is not counted).  For accounting of launches in benchmarks. */
QLN_API uint64_t qln_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
