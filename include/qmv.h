/*
 * qmv.h -- C ABI of libqmv.so: the weight-quantized matrix-vector product on
 * NVIDIA B200 (sm_100a).
 *
 *     y[m, n] = sum_k x[m, k] * dequant(W)[n, k]      0 <= m < M <= 8
 *
 * The operation and its formats are the ones defined on these pages:
 *  - MLX "quantized_nax.h" (mlx 1.0.0 source page): affine group quantization,
 *    w = scale * q + bias per group of `group_size` codes along K; pack geometry
 *    in get_pack_factor / get_bytes_per_pack (3- and 5-bit codes 8 to a pack of
 *    3 / 5 bytes, 6-bit codes 4 to a pack of 3 bytes, 2/4/8-bit codes 8/bits to
 *    a byte); codes read least significant bit first inside a pack (qdot,
 *    dequantize); scales and biases stored [N, K / group_size] in the dtype of x.
 *  - wh-iron "kernel-op coverage audit", section "Quantization precision
 *    coverage", Track 1 table: MXFP4 (E2M1 codes, E8M0 scale per 32),
 *    NVFP4 (E2M1 codes, E4M3 scale per 16, FP32 global scale), MXFP8 (E4M3
 *    codes, E8M0 scale per 32); 4-bit codes two to a byte, low nibble first.
 *  - MLX pull request "affine_qmv_fast_rows / fp_qmv_fast_rows": the user call
 *    (packed w, scales, biases, bits, group size / mode, NVFP4 global scale),
 *    output sizes N that are not a multiple of the row tile, and the bias term
 *    built from a sum(x) widened to fp32 element by element.
 *
 * Conventions shared by every entry point
 *  - All array pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or keeps them.  Layouts are row-major and dense:
 *      x        [M, K]          dtype
 *      w_packed [N, K*bits/8]   bytes (affine); [N, K/2] (FP4); [N, K] (FP8)
 *      scales   [N, K/group]    dtype (affine);  uint8 [N, K/block] (FP modes)
 *      biases   [N, K/group]    dtype (affine only)
 *      y        [M, N]          dtype
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *    asynchronous on that stream: it validates its arguments on the host, then
 *    enqueues kernels; it never synchronizes.  Kernels are launched with
 *    programmatic dependent launch, so they may start while the previous kernel
 *    in the stream drains.  They read x (and write y) only after that kernel
 *    has finished, but they begin fetching the WEIGHTS (w_packed, scales,
 *    biases) at once: the kernel launched immediately before the call on the
 *    same stream must not write them.  (Weights written by an earlier kernel,
 *    by a copy, or on another stream ordered by an event are fine.)
 *  - Calls are thread-safe for distinct streams.
 *  - Return value: QMV_OK, or a negative qmv_status.  Argument errors are
 *    detected before any launch (nothing is enqueued).  QMV_ECUDA means a launch
 *    failed; qmv_last_cuda_error() gives the cudaError_t of the last such
 *    failure on the calling thread.
 *  - M == 0 or N == 0 is a no-op returning QMV_OK; K == 0 writes y = 0.
 */
#ifndef QMV_H
#define QMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { QMV_F32 = 0, QMV_F16 = 1, QMV_BF16 = 2 } qmv_dtype;

typedef enum { QMV_MXFP4 = 0, QMV_NVFP4 = 1, QMV_MXFP8_E4M3 = 2 } qmv_fp_mode;

/* The symmetric block-scaled formats of the wh-iron kernel-op coverage audit,
 * section "Quantization precision coverage", Track 1 table (30 formats):
 * element / block along K / block-scale type (/ global).
 *   NVFP4  E2M1 / 16 / E4M3 / FP32 global    MXFP4  E2M1 / 32 / E8M0
 *   MXFP8_E4M3  E4M3 / 32 / E8M0            MXFP8_E5M2  E5M2 / 32 / E8M0
 *   NVFP8  E4M3 / 16 / FP32                 FP4 (legacy) E2M1 / 32 / FP32
 *   FP8_E4M3 (legacy) E4M3 / 32 / FP32      FP8_E5M2 (legacy) E5M2 / 32 / FP32
 *   INTb   signed b-bit / 64 / FP32         MXINTb signed b-bit / 32 / E8M0
 *   *_F16  the FP32-scaled formats above with an IEEE binary16 scale. */
typedef enum {
    QMV_FMT_NVFP4 = 0, QMV_FMT_MXFP4 = 1, QMV_FMT_MXFP8_E4M3 = 2, QMV_FMT_MXFP8_E5M2 = 3,
    QMV_FMT_NVFP8 = 4, QMV_FMT_FP4 = 5, QMV_FMT_FP8_E4M3 = 6, QMV_FMT_FP8_E5M2 = 7,
    QMV_FMT_INT2 = 8, QMV_FMT_INT3 = 9, QMV_FMT_INT4 = 10, QMV_FMT_INT5 = 11, QMV_FMT_INT6 = 12,
    QMV_FMT_INT8 = 13,
    QMV_FMT_MXINT2 = 14, QMV_FMT_MXINT3 = 15, QMV_FMT_MXINT4 = 16, QMV_FMT_MXINT5 = 17,
    QMV_FMT_MXINT6 = 18, QMV_FMT_MXINT8 = 19,
    QMV_FMT_NVFP8_F16 = 20, QMV_FMT_FP4_F16 = 21, QMV_FMT_FP8_E4M3_F16 = 22, QMV_FMT_FP8_E5M2_F16 = 23,
    QMV_FMT_INT2_F16 = 24, QMV_FMT_INT3_F16 = 25, QMV_FMT_INT4_F16 = 26, QMV_FMT_INT5_F16 = 27,
    QMV_FMT_INT6_F16 = 28, QMV_FMT_INT8_F16 = 29,
    QMV_FMT_COUNT = 30
} qmv_format;

typedef enum {
    QMV_OK = 0,
    QMV_EINVAL = -1,        /* bad size, null pointer, K not a multiple of the group/block */
    QMV_EUNSUPPORTED = -2,  /* bits, group_size, mode or dtype outside the supported set */
    QMV_EALIGN = -3,        /* a pointer is not aligned to its element (w_packed: 4 bytes) */
    QMV_ECUDA = -4          /* a CUDA launch or device query failed */
} qmv_status;

#define QMV_MAX_M 8

/*
 * qmv_affine -- affine group-quantized qmv.
 *   x, y      dtype elements, [M, K] and [M, N]
 *   w_packed  [N, K*bits/8] bytes; each row is a stream of packs as described
 *             above (4 bytes alignment required; 16 bytes enables the wide-load
 *             path when K is a multiple of its chunk)
 *   scales,   [N, K/group_size] dtype elements
 *   biases
 *   bits in {2,3,4,5,6,8}; group_size in {32,64,128}; K % group_size == 0;
 *   1 <= M <= 8 (0 allowed as a no-op); dtype a qmv_dtype.
 * Each output is  sum over groups g of  scale[n,g] * sum_{k in g} x[m,k]*q[n,k]
 *                                     + bias[n,g]  * sum_{k in g} x[m,k],
 * accumulated in fp32 (sum(x) widened per element) and rounded once to dtype.
 */
int qmv_affine(const void* x, const void* w_packed, const void* scales, const void* biases,
               void* y, int M, int N, int K, int bits, int group_size, int dtype,
               void* stream);

/*
 * qmv_affine_batched -- `batch` independent affine problems in one launch
 * (MLX quantized_nax.h, adjust_matrix_offsets: one batch index per grid z).
 * w_packed, scales, biases and y are contiguous [batch, ...] stacks of the
 * single-problem layouts.  x_batched = 1: x is [batch, M, K]; 0: one x [M, K]
 * shared by every batch entry.  1 <= batch <= 65535.
 */
int qmv_affine_batched(const void* x, const void* w_packed, const void* scales,
                       const void* biases, void* y, int M, int N, int K, int bits,
                       int group_size, int dtype, int batch, int x_batched, void* stream);

/*
 * qmv_fp -- block-scaled FP qmv.
 *   mode QMV_MXFP4:      w_packed [N, K/2] E2M1 codes (low nibble = even k),
 *                        scales [N, K/32] E8M0 bytes; K % 32 == 0
 *   mode QMV_NVFP4:      w_packed [N, K/2] E2M1 codes, scales [N, K/16] E4M3 bytes,
 *                        global_scale: DEVICE pointer to one float (required);
 *                        K % 16 == 0 (a 16-code tail block when K % 32 == 16)
 *   mode QMV_MXFP8_E4M3: w_packed [N, K] E4M3 codes, scales [N, K/32] E8M0 bytes;
 *                        K % 32 == 0
 *   global_scale must be NULL for the MX modes.
 * Output: sum over blocks of  scale_blk * sum_{k in blk} x[m,k] * elem[n,k]
 * (times the global scale for NVFP4), fp32 accumulation, one rounding to dtype.
 * NaN codes (E4M3 0x7F/0xFF, E8M0 0xFF) propagate as NaN.
 */
int qmv_fp(const void* x, const void* w_packed, const void* scales, const float* global_scale,
           void* y, int M, int N, int K, int mode, int dtype, void* stream);

/* qmv_fp_batched -- batched form of qmv_fp; layouts as in qmv_affine_batched.
 * For NVFP4 global_scale points to `batch` floats (one per weight tensor). */
int qmv_fp_batched(const void* x, const void* w_packed, const void* scales,
                   const float* global_scale, void* y, int M, int N, int K, int mode,
                   int dtype, int batch, int x_batched, void* stream);

/*
 * qmv_block_scaled -- qmv for any Track-1 format (qmv_format above; wh-iron
 * kernel-op coverage audit, "Quantization precision coverage").
 *   w_packed  [N, K*b/8] bytes, b = 4 (E2M1), 8 (E4M3 / E5M2) or the int width;
 *             each row an LSB-first stream of b-bit codes (4-bit: low nibble =
 *             even k; 8-bit: one byte per code; signed ints two's complement);
 *             4-byte alignment required, 16 enables 16-byte loads
 *   scales    [N, K/block] of the format's scale type: E8M0 / E4M3 bytes,
 *             float (4-byte aligned) or IEEE half (2-byte aligned)
 *   global_scale  NVFP4 only: DEVICE pointer to one float (required); NULL for
 *             every other format
 *   K % block == 0 (so K % 32 == 16 is valid for the 16-blocks: NVFP4, NVFP8);
 *   1 <= M <= 8 (0 a no-op); x and y dtype elements as in qmv_affine.
 * Output: sum over blocks of  scale_blk * sum_{k in blk} x[m,k] * elem[n,k]
 * (times the global for NVFP4), fp32 accumulation, one rounding to dtype.
 * Signed ints are read as offset binary q + 2^(b-1) with the bias term
 * -2^(b-1) * scale * sum(x) (sum(x) widened per element).  NaN and infinite
 * codes (E4M3 0x7F/0xFF, E5M2 exponent 31, E8M0 0xFF) propagate.
 * Errors: format outside qmv_format -> QMV_EUNSUPPORTED; K % block, a missing
 * or extra global_scale, null pointers -> QMV_EINVAL; misaligned w_packed or
 * scales -> QMV_EALIGN.
 */
int qmv_block_scaled(const void* x, const void* w_packed, const void* scales, const float* global_scale,
                     void* y, int M, int N, int K, int format, int dtype, void* stream);

/* qmv_block_scaled_batched -- batched form; layouts as in qmv_affine_batched
 * (for NVFP4 global_scale points to `batch` floats). */
int qmv_block_scaled_batched(const void* x, const void* w_packed, const void* scales,
                             const float* global_scale, void* y, int M, int N, int K, int format,
                             int dtype, int batch, int x_batched, void* stream);

/* qmv_dequant_block_scaled_f32 -- check kernel: w_out [N, K] fp32 (16-byte
 * aligned) = element * scale rounded once (NVFP4: (element * E4M3) * global). */
int qmv_dequant_block_scaled_f32(const void* w_packed, const void* scales, const float* global_scale,
                                 float* w_out, int N, int K, int format, void* stream);

/* qmv_format_info -- layout facts of a qmv_format, for sizing buffers: bits
 * per code, codes per block scale, bytes per block scale, and whether a
 * global scale is taken.  Any output pointer may be NULL.  Returns QMV_OK or
 * QMV_EUNSUPPORTED. */
int qmv_format_info(int format, int* element_bits, int* block, int* scale_bytes, int* has_global);

/*
 * qmv_quantize_affine -- affine quantizer (wh-iron kernel-op coverage audit,
 * "quantized (affine_quantize / affine_dequantize)" row: quantize kernels for
 * every width; the pages do not state their arithmetic, this is the plainest
 * reading consistent with w = scale * q + bias, MLX quantized_nax.h).
 *   w         [N, K] row-major in dtype (finite values)
 *   w_packed  [N, K*bits/8] bytes out, the layout qmv_affine reads (LSB-first
 *             packs: 2/4/8-bit 8/bits codes per byte, 3/5-bit 8 codes per 3/5
 *             bytes, 6-bit 4 codes per 3 bytes)
 *   scales, biases  [N, K/group_size] in dtype, out
 * For each group of group_size consecutive weights of a row: bias = min,
 * scale = (max - min) / (2^bits - 1), both rounded to dtype (to nearest, ties
 * to even); q = rint((w - bias) / scale), the difference and the quotient each
 * one fp32 operation on the rounded values (ties to even), clamped to
 * [0, 2^bits - 1]; q = 0 when the rounded scale is 0 or the quotient is NaN.
 * (The kernel multiplies by one reciprocal per group and divides only where
 * that could change a code: the codes are those of the division.)
 * bits in {2,3,4,5,6,8}, group_size in {32,64,128}, K % group_size == 0.
 * Alignment: w, scales, biases to their element size, w_packed to 4 bytes
 * (QMV_EALIGN otherwise); 16-byte aligned rows of w are read 16 bytes at a
 * time.  Asynchronous on `stream`; the caller owns every buffer.  Returns
 * QMV_OK or a status as for qmv_affine.
 */
int qmv_quantize_affine(const void* w, void* w_packed, void* scales, void* biases, int N, int K,
                        int bits, int group_size, int dtype, void* stream);

/*
 * qmv_affine_gather -- expert-indexed (MoE) qmv: for each token t,
 *     y[t] = x[t] * dequant(W[expert_ids[t]])^T
 * (wh-iron kernel-op coverage audit, "gather_qmv / gather_qmm" row; DS4
 * moe.metal, kernel_mul_mv_id: an ids tensor selects each slot's routed expert
 * on the device, with no per-expert dispatch from the host).
 *   w_packed  [n_experts, N, K*bits/8] bytes, a stack of qmv_affine matrices
 *   scales,   [n_experts, N, K/group_size] dtype
 *   biases
 *   expert_ids DEVICE int32 [n_tokens] (4-byte aligned), read on the GPU; an
 *             id outside [0, n_experts) makes that token's y rows NaN (nothing
 *             out of bounds is read)
 *   x         [n_tokens, M, K] (x_batched = 1) or one [M, K] for every token
 *   y         [n_tokens, M, N]
 *   1 <= n_tokens <= 65535, n_experts >= 1; other arguments as qmv_affine.
 * Runs on the CUDA-core kernels (row-tiled, or few-rows for small N), launched
 * without programmatic dependent launch so that ids written by the previous
 * kernel in the stream are complete.  Same accumulation and rounding as
 * qmv_affine.
 */
int qmv_affine_gather(const void* x, const void* w_packed, const void* scales, const void* biases,
                      const int* expert_ids, void* y, int M, int N, int K, int bits, int group_size,
                      int dtype, int n_tokens, int n_experts, int x_batched, void* stream);

/*
 * qmv_affine_swiglu -- decode gate + up projection fused with the SwiGLU
 * activation (DS4 moe.metal: kernel_mul_mv_id_q4_K_pair_swiglu_f32, the
 * paired gate / up matvec whose lanes derive the routed SwiGLU input, and
 * kernel_dsv4_moe_swiglu_weight for the activation; wh-iron kernel-op
 * coverage audit, "moe routed-expert decode fuse" row: the activation fused
 * into the gate / up qmv epilogue).  For every x row m and output n:
 *     g = sum_k x[m,k] * dequant(W_gate)[n,k],  u = same with W_up,
 *     if clamp > 1e-6:  g = min(g, clamp),  u = min(max(u, -clamp), clamp),
 *     mid[m, n] = g / (1 + exp(-g)) * u * route_weight[m],
 * with g and u accumulated in fp32 exactly as qmv_affine does, the
 * activation in fp32 and one rounding of mid to dtype.  gate and up are not
 * written.
 *   w_gate, s_gate, b_gate   the gate matrix, as qmv_affine's w_packed,
 *   w_up, s_up, b_up         scales, biases (same N, K, bits, group_size)
 *   route_weight  DEVICE pointer to M floats (one per x row, read after the
 *                 previous kernel in the stream completes), or NULL for 1
 *   mid           [M, N] dtype
 *   clamp         >= 0 (QMV_EINVAL if negative or NaN); at or below 1e-6 no
 *                 clamping
 * Other arguments, alignment and errors as qmv_affine; both matrices take
 * the wide-load path when both are 16-byte aligned.  Runs the row-tiled
 * CUDA-core kernel over the 2N interleaved gate / up rows, so each warp holds
 * both sums of its outputs.
 */
int qmv_affine_swiglu(const void* x, const void* w_gate, const void* s_gate, const void* b_gate,
                      const void* w_up, const void* s_up, const void* b_up, const float* route_weight,
                      void* mid, int M, int N, int K, int bits, int group_size, int dtype, float clamp,
                      void* stream);

/*
 * qmv_affine_qkv -- the Q, K and V projections of one x in one launch
 * (wh-iron kernel-op coverage audit, "batched_qkv_qgemv" row: Q / K / V
 * 4-bit qGEMV in one dispatch, output concatenated [Q | K | V]; K and V have
 * the same size, grouped-query attention).
 *   w_q, s_q, b_q   [Nq, ...]  the Q matrix, as qmv_affine's w_packed, scales,
 *   w_k, s_k, b_k   [Nkv, ...] biases (all three share K, bits, group_size)
 *   w_v, s_v, b_v   [Nkv, ...]
 *   y               [M, Nq + 2 Nkv] dtype: y[m, 0:Nq] = x W_q^T, then K, then V
 * Each output as qmv_affine computes it; the row-tiled CUDA-core kernel reads
 * each output row from its own matrix.  Nq, Nkv >= 0; a matrix with no rows
 * may be NULL.  Other arguments, alignment and errors as qmv_affine.
 */
int qmv_affine_qkv(const void* x, const void* w_q, const void* s_q, const void* b_q, const void* w_k,
                   const void* s_k, const void* b_k, const void* w_v, const void* s_v, const void* b_v,
                   void* y, int M, int Nq, int Nkv, int K, int bits, int group_size, int dtype,
                   void* stream);

/*
 * qmv_affine_rms_norm -- RMSNorm of x fused into the affine qmv (wh-iron
 * kernel-op coverage audit, "rms_norm_qgemv" row):
 *     y[m, n] = sum_k xh[m, k] * dequant(W)[n, k],
 *     xh[m, k] = x[m, k] * gamma[k] / sqrt(mean_k x[m, k]^2 + eps),
 * xh kept in fp32 (never rounded to dtype): the sum of squares and the
 * products in fp32, then qmv_affine's accumulation and one rounding of y.
 *   gamma   [K] dtype (device)
 *   eps     >= 0 and finite (QMV_EINVAL otherwise)
 * Other arguments, alignment and errors as qmv_affine (gamma aligned to its
 * element).  Runs the row-tiled CUDA-core kernel: every block first reduces
 * the sums of squares of the M x rows (read after the previous kernel in the
 * stream completes), then stages xh instead of x.
 */
int qmv_affine_rms_norm(const void* x, const void* gamma, float eps, const void* w_packed,
                        const void* scales, const void* biases, void* y, int M, int N, int K, int bits,
                        int group_size, int dtype, void* stream);

/*
 * qmv_qmm_affine -- small-M quantized matmul, y = x * dequant(W)^T for up to
 * QMV_QMM_MAX_M x rows (the qmm family of MLX quantized_nax.h and of the
 * wh-iron audit, M-batched prefill).  Arguments and layouts as qmv_affine,
 * with 1 <= M <= 64 (0 allowed as a no-op).  M <= 8 is qmv_affine.  More
 * rows, 4-bit codes with bf16 / f16 x, K a multiple of 8 groups, 16-byte
 * aligned weights, scales and biases: chunks of 16 or 32 rows through the
 * per-group tensor-core ring kernel (every decoded weight feeds all rows of
 * the chunk).  Otherwise, for N <= 5120 with bf16 x, 16-byte aligned x,
 * weights, scales and biases, K a multiple of 64 and K / group_size a
 * multiple of 8, ONE launch of the tensor-memory kernel (tcgen05: each weight
 * decoded once for all rows, the rows are the MMA's N, K split over a
 * thread-block cluster) when x fits its shared memory; otherwise chunks of 32
 * or 16 rows through the tensor-core ring kernel where it takes that many (x
 * rows times groups of a 128-code super-block at most 32, N > 64, 16-byte
 * aligned weights), else chunks of QMV_MAX_M.  Chunks run back to back on
 * `stream` (a weight matrix that fits in L2 is read from HBM once).  Every
 * argument is checked before the first launch.  Same accumulation and
 * rounding as qmv_affine.
 */
#define QMV_QMM_MAX_M 64
int qmv_qmm_affine(const void* x, const void* w_packed, const void* scales, const void* biases,
                   void* y, int M, int N, int K, int bits, int group_size, int dtype, void* stream);

/*
 * qmv_qvm_affine -- qvm: x times an affine weight matrix stored [K, N]
 * (MLX quantized_nax.h, qouter: result[j] += x * (scale * q_j + bias) over a
 * packed row; the wh-iron audit's qvm family, "x.W with W [K, N]").
 *   x         [M, K] dtype
 *   w_packed  [K, N*bits/8] bytes: row k packs the codes of output columns
 *             0..N-1 exactly like a qmv_affine row (LSB-first packs); 16-byte
 *             aligned
 *   scales,   [K, N/group_size] dtype (grouped along N)
 *   biases
 *   y         [M, N] dtype
 *   workspace NULL, or a device buffer of qmv_qvm_workspace_bytes(M, N) bytes,
 *             16-byte aligned, ALL ZERO before its first use (cudaMemset
 *             once); every call returns it to zero.  With it, K is split over
 *             several blocks whose fp32 partial sums meet there (the order of
 *             that final fp32 sum varies between runs); without it, each 1024
 *             columns are summed by a single block (few blocks for small N).
 *             Calls that share a workspace must not overlap on the GPU (one
 *             stream, or ordered by events).
 *   bits in {2,3,4,5,6,8}; group_size in {32,64,128}; N % group_size == 0;
 *   1 <= M <= 8 (0 allowed as a no-op); K >= 0 (K == 0 writes y = 0).
 * y[m, n] = sum_k x[m,k] * (scale[k, n/group_size] * q[k,n] + bias[k, n/group_size]),
 * accumulated in fp32 and rounded once to dtype.  Alignment: x, y, scales,
 * biases to their element (QMV_EALIGN otherwise).  Asynchronous on `stream`;
 * no programmatic dependent launch.  Returns QMV_OK or a status as for
 * qmv_affine.
 */
int qmv_qvm_affine(const void* x, const void* w_packed, const void* scales, const void* biases,
                   void* y, int M, int N, int K, int bits, int group_size, int dtype,
                   void* workspace, void* stream);

/* Bytes of the qmv_qvm_affine workspace for M x rows and N columns (0 for a
 * negative size).  Host-only. */
size_t qmv_qvm_workspace_bytes(int M, int N);

/*
 * qmv_qvm_affine_noalloc -- qmv_qvm_affine for callers that cannot allocate
 * device memory.  The pages have no counterpart; this is a library addition.
 * Some callers must not allocate at all: a plugin whose host framework owns
 * every device byte through its own pool and forbids driver allocations, or a
 * latency-critical decode loop that cannot afford the device synchronization
 * that cudaMalloc / cudaFree may imply.  They cannot hand qmv_qvm_affine a
 * workspace; this call uses a fixed scratch array of
 * QMV_QVM_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that
 * loads it, until the process exits, and allocates nothing.
 *   Arguments, layouts and result as qmv_qvm_affine without `workspace`.
 *   Limit: qmv_qvm_workspace_bytes(M, N) <= QMV_QVM_NOALLOC_SCRATCH_BYTES
 *   (M = 1 with N up to 261888, M = 8 with N up to 32736); larger sizes
 *   return QMV_EUNSUPPORTED before any launch.
 *   The first call on a device looks up the scratch's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.  The address is kept for the life of the process: calls after a
 *   cudaDeviceReset() of that device are not supported (the module reloads
 *   and the array may move).  Each call clears the part of the scratch it uses on `stream`,
 *   then launches.  Every call, on every stream, shares the one array:
 *   calls that overlap on the GPU race and give wrong results, so order them
 *   (one stream, or events).
 *   A failure of the address lookup or of the clearing returns QMV_ECUDA
 *   without updating qmv_last_cuda_error; a failed kernel launch updates it.
 */
#define QMV_QVM_NOALLOC_SCRATCH_BYTES (1u << 20)
int qmv_qvm_affine_noalloc(const void* x, const void* w_packed, const void* scales,
                           const void* biases, void* y, int M, int N, int K, int bits,
                           int group_size, int dtype, void* stream);

/*
 * qmv_quantize_fp -- block-scaled FP quantizer (wh-iron kernel-op coverage
 * audit, "fp_quantized (fp4/fp8 quant + dequant)" row: a per-group max
 * scale and mantissa rounding, saturating with no NaN or infinity; the pages
 * give no formula for the scale, this is the reading used).
 *   w        [N, K] row-major in dtype (finite values)
 *   mode QMV_MXFP4:      w_packed [N, K/2] E2M1 codes (low nibble = even k),
 *                        scales [N, K/32] E8M0 bytes; K % 32 == 0
 *   mode QMV_MXFP8_E4M3: w_packed [N, K] E4M3 codes, scales [N, K/32] E8M0
 *   mode QMV_NVFP4:      w_packed [N, K/2] E2M1 codes, scales [N, K/16] E4M3
 *                        bytes, global_scale: DEVICE pointer to one float g
 *                        (required, normal and > 0); K % 16 == 0
 *   global_scale must be NULL for the MX modes.
 * MX: E8M0 byte = clamp(floor(log2(amax)) - emax + 127, 0, 254) per block
 * (emax 2 for E2M1, 8 for E4M3; 0 when amax is 0), element w * 2^(127 - byte).
 * NVFP4: scale = nearest E4M3 to amax / (6 g), element w / (scale * g), both
 * in fp32.  Each code is the nearest element, ties to the even code,
 * saturating at the largest finite element (6 or 448); the sign bit is set
 * for negative elements.  The output is the layout qmv_fp reads.  Alignment:
 * w to its element (QMV_EALIGN otherwise); 16-byte aligned w and w_packed use
 * vector loads and stores.  Asynchronous on `stream`; caller-owned buffers.
 */
int qmv_quantize_fp(const void* w, void* w_packed, void* scales, const float* global_scale, int N, int K,
                    int mode, int dtype, void* stream);

/*
 * qmv_dequant_affine_f32 -- check kernel: w_out[n*K + k] = fp32 value of
 * scale * q + bias, computed with one rounding (fmaf) from the stored dtype
 * scale / bias.  Uses the same device decoders as qmv_affine.  w_out is a
 * caller-owned device buffer of N*K floats.
 */
int qmv_dequant_affine_f32(const void* w_packed, const void* scales, const void* biases,
                           float* w_out, int N, int K, int bits, int group_size, int dtype,
                           void* stream);

/*
 * qmv_dequant_fp_f32 -- check kernel: w_out[n*K + k] = elem * scale (MX), or
 * (elem * e4m3_scale) * global (NVFP4, one rounding), in fp32.
 */
int qmv_dequant_fp_f32(const void* w_packed, const void* scales, const float* global_scale,
                       float* w_out, int N, int K, int mode, void* stream);

/* Human-readable text of a qmv_status. */
const char* qmv_status_string(int status);

/* cudaError_t of the last QMV_ECUDA returned on this thread (0 if none). */
int qmv_last_cuda_error(void);

/*
 * qmv_describe_plan -- the launch the picker would choose for these sizes,
 * written as text into buf (at most buflen bytes, NUL-terminated).  `family`
 * is 0 for affine (bits, group_size used), 1 + qmv_fp_mode, or 100 + a
 * qmv_format (bits and group_size ignored).  M up to 8 is
 * qmv's plan; 9..64 (affine) is qmv_qmm_affine's ("path=umma ...", or
 * "path=chunked<rows> chunks=<n>" and the plan of one chunk).  Host-only; no CUDA call except
 * cached device-property and occupancy queries.  Returns QMV_OK or an
 * argument error.
 */
int qmv_describe_plan(int family, int M, int N, int K, int bits, int group_size, int dtype,
                      int w_align16, char* buf, int buflen);

/*
 * qmv_device_fault -- the fault word of the current device.  Kernels that
 * stream weights through a shared-memory ring wait on barriers with a bound
 * (about one second); a wait that expires ORs a nonzero code into this word
 * (1: a consumer warp gave up on a ring stage, 2: the producer warp gave up on
 * a free stage, 4: the producer gave up waiting for its own copies) and the
 * call that hit it leaves y undefined.  Writes the word to *code and, if clear != 0,
 * resets it to zero.  Synchronous: it waits for the device's pending work
 * (cudaMemcpyFromSymbol).  Returns QMV_OK, QMV_EINVAL (code NULL) or QMV_ECUDA.
 */
int qmv_device_fault(unsigned int* code, int clear);

/*
 * qmv_force_config -- benchmarking / testing knob: pin the launch shape used
 * by every later call in this process.  path: 8 = per-group tensor-core
 * kernel with the weight ring (affine 4-bit, f16 / bf16 x, up to 32 x rows,
 * K a multiple of 8 groups), 7 = tensor-memory (tcgen05) kernel (qmm), 6 =
 * CUDA-core kernel with the weight ring (one bf16 x row), 5 = few-rows
 * latency kernel, 4 =
 * tensor-core kernel with the weight ring, 3 = tensor-core kernel (4 and 3 for
 * affine formats; paths fall back to automatic where their size rules do not
 * hold), 1 = CUDA-core kernel with wide (16-byte) chunk loads, 0 = CUDA-core
 * kernel with 4-byte chunks, -1 = automatic; rows_per_warp in {1,2,4} or -1
 * (CUDA-core kernel); warps_k (warps that split K inside a block) and
 * warps_rows (16-row tiles per block) up to 12 each, or -1; the weight-ring
 * kernels run warps_k * warps_rows in {8, 12} compute warps (path 8: 8 or 16,
 * warps_k in {1, 2, 4, 8}) and a producer warp.
 * Unsupported combinations fall back to automatic for that field.
 * NOT FOR PRODUCTION USE: this is process-wide state for the parity tests and
 * the benchmark's sweeps; it is not thread-safe with concurrent calls and
 * overrides the picker for every caller in the process.  (Likewise the
 * environment variable QMV_PDL=0, read once per process, turns programmatic
 * dependent launch off; it exists for A/B timing only.)
 */
void qmv_force_config(int path, int rows_per_warp, int warps_k, int warps_rows);

/*
 * qmv_test_skip_last_copy -- NOT FOR PRODUCTION USE (tests of the bounded
 * waits).  While enabled (nonzero), every launch of a weight-ring kernel
 * (paths "tcb" and "tcf") has the producer warp of block (0, 0) skip its final
 * ring stage: no expected-bytes arrival and no tensor copy.  That block's
 * consumer warps then give up their bounded wait on the stage (about 1 s) and
 * OR code 1 into the fault word, the producer gives up its wait for its own
 * copies on it and ORs code 4, and the kernel returns normally with undefined
 * output; no copy is left in flight, and the context stays usable.  Process
 * global, not thread-safe; 0 restores normal launches.
 */
void qmv_test_skip_last_copy(int enable);

#ifdef __cplusplus
}
#endif

#endif /* QMV_H */
