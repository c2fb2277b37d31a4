/*
 * sp24.h -- C ABI of the B200 (sm_100a) 2:4 structured-sparse FP8 GEMM library.
 *
 * The library implements the hot path of 2:4 structured sparsity with FP8
 * for the linear and FFN layers of an LLM:
 *   1. magnitude 2:4 pruning along K, ties to the lower index
 *      ("Deploying 2:4 Sparsity with FP8 on Hopper: A Production Cookbook",
 *       pipeline step 4 and Practical Example 1);
 *   2. compression into an [N, K/2] values array plus 2-bit index metadata
 *      (the cookbook, pipeline step 2; "La Densite Dynamique et les Noyaux
 *       Non Structures", §Lacunes des noyaux);
 *   3. per-tensor dynamic E4M3 quantisation with scale = amax / 448
 *      (the cookbook, pipeline steps 3 and 6);
 *   4. the sparse GEMM Y[M,N] = X[M,K] . W^T with fp32 accumulation, both
 *      scales applied and bf16 output;
 * and the (2N-2):2N extension for 6:8 ("SlideSparse: Fast and Flexible
 * (2N-2):2N Structured Sparsity", Resumen tecnico §2 Metodologia): each
 * 8-group is split into three overlapping stride-2 windows that are each
 * 2:4 over a lifted K' = 1.5 K, and the activation lift is fused into the
 * FP8 quantisation pass.  Beyond that path: the fused quantise + GEMM forms
 * for decode, per-token and per-channel scales, the general (2N-2):2N
 * decomposition for N = 3 and 5, INT8 W8A8 and FP4 (quantisers and the
 * sparse GEMMs; each declared with its own citation below).
 *
 * Conventions for every entry point
 * ---------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller; the library
 *   never allocates.  Matrices are row-major with K contiguous.  Every
 *   tensor pointer must be 16-byte aligned (SP24_ERR_ALIGN otherwise).
 * - bf16 tensors are IEEE bfloat16 bit patterns (uint16); E4M3 tensors are
 *   OCP FP8 E4M3 ("FN": no infinities, 0x7F/0xFF = NaN, max 448) bytes.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL means the
 *   legacy default stream) and returns an int status (SP24_OK or a negative
 *   SP24_ERR_*).  Arguments are validated on the host before any launch;
 *   there is no silent dense or CPU fallback.
 * - Scales are device floats (dequantisation scales: real = code * scale), so
 *   dynamic scaling never forces a host synchronisation.
 * - `workspace` is device scratch of at least sp24_workspace_size(...)
 *   bytes (never less than 256).  It must be zero-filled before its FIRST
 *   use.  Its first 256 bytes (and, for a split-K GEMM, its tile counters)
 *   hold counters that every call returns to zero; the rest is scratch that
 *   a call rewrites before reading.  So one buffer can serve any sequence of
 *   calls, as long as calls sharing it never run concurrently.  After a call
 *   that reported SP24_STATUS_TIMEOUT the counters may be left nonzero (a
 *   late arrival can count into a tile its owner gave up on): zero-fill the
 *   workspace again before its next use, or a later call may read partial
 *   sums that are not ready.
 * - `status` (nullable) is a device int32 that kernels OR error bits into:
 *   SP24_STATUS_NONFINITE when an input holds NaN/Inf (the method is defined
 *   for finite inputs only; a NaN input element is encoded as 0x7F whatever
 *   its sign).  Read it after synchronising the stream.
 * - The library is for sm_100a (B200).  On any other device the entry
 *   points return SP24_ERR_ARCH.
 *
 * Compressed weight layout (shared by every GEMM entry point)
 * ------------------------------------------------------------
 *   values[n, 2g + t] = t-th kept element (ascending index) of group g of row n
 *   meta[n, b]        = nibble(2b) | nibble(2b + 1) << 4
 *   nibble(g)         = i0 | i1 << 2, 0 <= i0 < i1 <= 3, the in-group indices
 *                       of the two kept elements of group g.
 */
#ifndef SP24_H
#define SP24_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sp24_stream_t; /* identical to cudaStream_t */

/* Return codes */
#define SP24_OK 0
#define SP24_ERR_NULL (-1)      /* a required pointer is NULL */
#define SP24_ERR_SHAPE (-2)     /* a dimension breaks the shape rules of the call */
#define SP24_ERR_ALIGN (-3)     /* a pointer is not 16-byte aligned */
#define SP24_ERR_DTYPE (-4)     /* unknown dtype code */
#define SP24_ERR_CUDA (-5)      /* CUDA launch/runtime error, see sp24_last_cuda_error() */
#define SP24_ERR_WORKSPACE (-6) /* workspace missing or smaller than required */
#define SP24_ERR_ARCH (-7)      /* current device is not sm_100 */

/* Device status bits (OR-ed into *status by the kernels) */
#define SP24_STATUS_NONFINITE 1 /* an input element was NaN or Inf */
#define SP24_STATUS_TIMEOUT 2   /* a pipeline wait hit its iteration limit */

/* dtype codes */
#define SP24_DTYPE_E4M3 0
#define SP24_DTYPE_BF16 1

/* op codes for sp24_workspace_size */
#define SP24_OP_QUANTIZE 0
#define SP24_OP_PRUNE_COMPRESS 1
#define SP24_OP_SLIDE68_DECOMPOSE 2
#define SP24_OP_SLIDE68_LIFT 3
#define SP24_OP_GEMM 4
#define SP24_OP_GEMM_DENSE 5
#define SP24_OP_GEMM_PACKED 6
#define SP24_OP_QUANTIZE_GEMM_PACKED 7 /* K = the columns of X */
#define SP24_OP_LIFT_GEMM_PACKED 8     /* K = the columns of X (the GEMM runs over 3K/2) */
#define SP24_OP_GEMM_FP4 9

/*
 * Weight path, 2:4.  W: bf16 [N, K].  For every row and every group of 4
 * contiguous K-values the two largest |w| are kept (equal magnitudes go to the
 * lower index; -0 equals +0).  Pruning ranks the bf16 magnitudes before any
 * quantisation.
 *   out_dtype = SP24_DTYPE_E4M3: w_scale <- amax|W| / 448 (1.0 when amax = 0),
 *     values <- E4M3(w / w_scale) of the kept elements (u8 [N, K/2]; the
 *     quotient is one correctly rounded fp32 division, then round to nearest
 *     even with saturation to +-448), pruned_dense (nullable) <- u8 [N, K]
 *     with the same codes at kept positions and 0x00 elsewhere.
 *   out_dtype = SP24_DTYPE_BF16: values <- the kept bf16 values (u16 [N, K/2]),
 *     w_scale is ignored (may be NULL), pruned_dense (nullable) <- bf16 [N, K].
 * meta <- u8 [N, K/8] in the layout above.
 * Shape rules: N >= 1, K >= 8, K % 8 == 0.
 */
int sp24_prune_compress(const void *W, int N, int K, int out_dtype, void *values,
                        uint8_t *meta, float *w_scale, void *pruned_dense, void *workspace,
                        size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * Per-tensor dynamic E4M3 quantisation (the cookbook, pipeline step 3).
 * X: bf16 [rows, cols] -> q: u8 [rows, cols], scale <- amax|X| / 448 (1.0 when
 * amax = 0), q = E4M3(x / scale) as above.  Also used for the weights of the
 * dense FP8 comparison GEMM.  Shape rules: rows >= 1, cols >= 1, cols % 16 == 0.
 * A decode-sized X (rows * cols <= 131072) is done by one thread-block
 * cluster that leaves the workspace untouched and lets the next kernel on
 * `stream` launch at once (it must wait for this one before reading q or
 * scale, as every kernel of this library does).
 */
int fp8_quantize_pertensor(const void *X, int64_t rows, int64_t cols, uint8_t *q, float *scale,
                           void *workspace, size_t ws_bytes, int32_t *status,
                           sp24_stream_t stream);

/*
 * Weight path, 6:8 through 2:4 windows (SlideSparse, §2 "Descomposicion de
 * Ventana Deslizante").  W: bf16 [N, K].  Each group of 8 contiguous K-values
 * keeps its six largest |w| (ties to the lower index).  Window j = 0, 1, 2 of
 * group g covers positions 2j .. 2j+3; in that order each window takes the two
 * lowest-index kept positions in its range not taken by an earlier window.  A
 * position p taken by window j goes to expanded column 12g + 4j + (p - 2j) of
 * W' [N, K' = 3K/2], which is then 2:4 and stored compressed:
 * values [N, 3K/4] (E4M3 codes with w_scale as for 2:4, or bf16) and
 * meta [N, 3K/16].  Shape rules: N >= 1, K % 16 == 0.
 */
int slide68_decompose(const void *W, int N, int K, int out_dtype, void *values, uint8_t *meta,
                      float *w_scale, void *workspace, size_t ws_bytes, int32_t *status,
                      sp24_stream_t stream);

/*
 * Activation lift fused with per-tensor E4M3 quantisation (SlideSparse, §2
 * "Levantamiento de Activacion").  X: bf16 [M, K] -> q_lifted: u8 [M, 3K/2]
 * with q_lifted[m, 12g + 4j + r] = E4M3(X[m, 8g + 2j + r] / scale), scale <-
 * amax|X| / 448.  Shape rules: M >= 1, K % 16 == 0.  M * K <= 131072: one
 * thread-block cluster, as for fp8_quantize_pertensor.
 */
int slide68_lift(const void *X, int M, int K, uint8_t *q_lifted, float *scale, void *workspace,
                 size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * Sparse GEMM Y[M, N] = bf16( x_scale * w_scale * sum_k X[m, k] * W[n, k] ),
 * accumulated in fp32 over the kept K positions only, on the 5th-generation
 * tensor cores (sparse tcgen05 MMA, accumulators in tensor memory).
 *   dtype = SP24_DTYPE_E4M3: Xq u8 [M, K], w_values u8 [N, K/2] (E4M3), scales
 *     are device floats (NULL means 1.0).
 *   dtype = SP24_DTYPE_BF16: Xq bf16 [M, K], w_values bf16 [N, K/2], scales
 *     ignored (may be NULL).
 * w_meta u8 [N, K/8]; Y bf16 [M, N].  K is the K of the compressed operand
 * (for 6:8 weights pass K' = 3K/2 and the lifted activations).
 * The kernel is persistent (at most one CTA per SM).  With many output tiles
 * each CTA takes whole tiles and needs no workspace.  With few tiles (decode
 * shapes) the (tile, K-block) work is split evenly over the CTAs (stream-K):
 * tiles shared by several CTAs are finished by the CTA holding their first
 * K-block, which adds the others' fp32 partials in a fixed order, so the
 * output is deterministic.  That needs sp24_workspace_size(SP24_OP_GEMM, ...)
 * bytes of workspace: a 16 KB prefix of counters (zero before the first
 * use, zero again after every call) followed by the partial tiles.
 * Shape rules: M >= 1, N % 128 == 0, K % 128 == 0 (both dtypes).
 * Y must not alias any input.
 */
int sp24_gemm(const void *Xq, const float *x_scale, const void *w_values, const uint8_t *w_meta,
              const float *w_scale, void *Y, int M, int N, int K, int dtype, void *workspace,
              size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * Tile-packed 2:4 E4M3 weights ("tile-aligned packing" of the compressed
 * values and metadata, as the roadmap page's §Lacunes des noyaux advises).
 * The canonical layout stores every row's values and metadata contiguously,
 * so one 128-row x 128-K GEMM stage touches 128 separate 64-byte and 16-byte
 * pieces; the packed layout makes each such stage one contiguous 10240-byte
 * block, read with a single bulk copy.  packed (u8, N*K/2 + N*K/8 bytes):
 * block (t, kb) at byte ((t * K/128) + kb) * 10240 holds, for rows
 * r = 0..127 of tile t, the 64 value bytes of K-block kb with 16-byte chunk c
 * stored at chunk position c ^ ((r >> 1) & 3), followed by the 128 rows x 16
 * metadata bytes of K-block kb.  It is a pure permutation of the canonical
 * bytes.  Shape rules: N % 128 == 0, K % 128 == 0.
 */
int sp24_pack_weights(const uint8_t *values, const uint8_t *meta, int N, int K, void *packed,
                      sp24_stream_t stream);

/*
 * The E4M3 2:4 weight path of sp24_prune_compress written straight into the
 * tile-packed layout: packed receives, byte for byte, what
 * sp24_pack_weights would make of the values and metadata that
 * sp24_prune_compress(W, N, K, SP24_DTYPE_E4M3, ...) computes, without the
 * canonical arrays ever being stored; w_scale <- amax|W| / 448 as there.
 * packed: u8, N*K/2 + N*K/8 bytes.  Workspace: sp24_workspace_size(
 * SP24_OP_PRUNE_COMPRESS, ...).  Shape rules: N % 128 == 0, K % 128 == 0,
 * N * K <= 2^38.
 */
int sp24_prune_compress_packed(const void *W, int N, int K, void *packed, float *w_scale,
                               void *workspace, size_t ws_bytes, int32_t *status,
                               sp24_stream_t stream);

/*
 * The E4M3 path of slide68_decompose written straight into the tile-packed
 * layout of the lifted 2:4 operand (K' = 3K/2): packed receives, byte for
 * byte, what sp24_pack_weights(values, meta, N, K') would make of the values
 * and metadata that slide68_decompose(W, N, K, SP24_DTYPE_E4M3, ...)
 * computes; w_scale <- amax|W| / 448.  packed: u8, N*K'/2 + N*K'/8 bytes.
 * Workspace: sp24_workspace_size(SP24_OP_SLIDE68_DECOMPOSE, ...).
 * Shape rules: N % 128 == 0, K % 256 == 0, N * K <= 2^38.
 */
int slide68_decompose_packed(const void *W, int N, int K, void *packed, float *w_scale,
                             void *workspace, size_t ws_bytes, int32_t *status,
                             sp24_stream_t stream);

/*
 * sp24_gemm (E4M3) with tile-packed weights (sp24_pack_weights); same result
 * within the GEMM tolerance (split tiles may sum their K ranges in another
 * order).  Workspace from sp24_workspace_size(SP24_OP_GEMM_PACKED, M, N, K,
 * 0).  When N % 256 == 0 and M is above 128 (prefill- and down-projection-
 * sized calls) the kernel launches clusters of two CTAs (one 256-row MMA
 * over two SMs); everywhere else one CTA per SM at most.
 */
int sp24_gemm_packed(const void *Xq, const float *x_scale, const void *packed,
                     const float *w_scale, void *Y, int M, int N, int K, void *workspace,
                     size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * Per-tensor activation quantisation and the packed sparse GEMM, for small
 * token counts (decode).  Computes exactly what
 *   fp8_quantize_pertensor(X, M, K, Xq, x_scale, ...) followed by
 *   sp24_gemm_packed(Xq, x_scale, packed, w_scale, Y, M, N, K, ...)
 * computes: Xq u8 [M, K] <- E4M3(x / x_scale), x_scale <- amax|X| / 448
 * (1.0 when amax = 0), Y bf16 [M, N]; Xq and x_scale are outputs (the codes
 * can feed further GEMMs of the same X).  X: bf16 [M, K].  When M * K <=
 * 8192 it is ONE launch: every CTA of the GEMM quantises all of X itself and
 * starts its tensor-core work on the codes while the packed weights already
 * stream in.  Otherwise the quantiser runs first (one thread-block cluster up
 * to M * K = 131072) and the GEMM, launched right behind it, streams its
 * weights while it runs.  Workspace:
 * sp24_workspace_size(SP24_OP_QUANTIZE_GEMM_PACKED, M, N, K, 0) (its first
 * 8 KB hold the quantiser's counters, zero before the first use and after
 * every call).
 * Shape rules: 1 <= M <= 256, N % 128 == 0, K % 128 == 0.  Xq and Y must not
 * alias X or each other.  SP24_STATUS_NONFINITE is set as by
 * fp8_quantize_pertensor.
 */
int sp24_quantize_gemm_packed(const void *X, int M, int N, int K, const void *packed,
                              const float *w_scale, uint8_t *Xq, float *x_scale, void *Y,
                              void *workspace, size_t ws_bytes, int32_t *status,
                              sp24_stream_t stream);

/*
 * The same with the SlideSparse activation lift (SlideSparse, §2
 * "Levantamiento de Activacion"): what slide68_lift(X, M, K, Xq_lifted,
 * x_scale, ...) followed by sp24_gemm_packed over K' = 3K/2 against 6:8
 * weights from slide68_decompose_packed computes.  X: bf16 [M, K];
 * Xq_lifted u8 [M, 3K/2]; packed over K'.  Workspace:
 * sp24_workspace_size(SP24_OP_LIFT_GEMM_PACKED, M, N, K, 0).
 * Shape rules: 1 <= M <= 256, N % 128 == 0, K % 256 == 0.
 */
int slide68_lift_gemm_packed(const void *X, int M, int N, int K, const void *packed,
                             const float *w_scale, uint8_t *Xq_lifted, float *x_scale, void *Y,
                             void *workspace, size_t ws_bytes, int32_t *status,
                             sp24_stream_t stream);

/*
 * INT8 W8A8 with 2:4 weights (the cookbook, Comparison Tables: the "INT8
 * W8A8" recipe; SlideSparse, §3 "Contribuciones Clave": INT8 among the
 * supported precisions).  Symmetric per-tensor scales: s = amax / 127 (1.0
 * for an all-zero tensor), q = clamp(round_half_even(RN_fp32(x / s)),
 * -127, 127).
 * int8_quantize_pertensor: X bf16 [rows, cols] (cols % 16 == 0) -> q int8
 *   [rows, cols], *scale <- s.
 * sp24_prune_compress_int8: W bf16 [N, K] (K % 8 == 0) -> the 2:4 selection
 *   of sp24_prune_compress (two largest |w| per group of 4, ties to the lower
 *   index) in the canonical layout with INT8 codes: values int8 [N, K/2],
 *   meta [N, K/8], *w_scale <- s.
 * Pointers are device pointers, 16-byte aligned (scale: 4-byte).  Workspace:
 * sp24_workspace_size(SP24_OP_QUANTIZE or SP24_OP_PRUNE_COMPRESS, ...)
 * (256 bytes of counters, zero before and after the call).  Errors as for
 * the E4M3 calls; SP24_STATUS_NONFINITE when the input holds Inf or NaN.
 */
int int8_quantize_pertensor(const void *X, int64_t rows, int64_t cols, int8_t *q, float *scale, void *workspace,
                            size_t ws_bytes, int32_t *status, sp24_stream_t stream);
int sp24_prune_compress_int8(const void *W, int N, int K, int8_t *values, uint8_t *meta, float *w_scale,
                             void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream);
/*
 * The INT8 W8A8 sparse GEMM: Y[M, N] = x_scale * w_scale * (Xq . W^T), the
 * integer products summed exactly in the tensor cores' s32 accumulators
 * (kind::i8) and converted to fp32 in the epilogue, bf16 out.  Xq: int8
 * [M, K] from int8_quantize_pertensor; packed: sp24_pack_weights applied to
 * the values (int8, as bytes) and metadata of sp24_prune_compress_int8;
 * scales: one device float each.  Shape rules, workspace
 * (sp24_workspace_size(SP24_OP_GEMM_PACKED, M, N, K, 0)) and errors as for
 * sp24_gemm_packed.
 */
int sp24_gemm_int8_packed(const int8_t *Xq, const float *x_scale, const void *packed, const float *w_scale,
                          void *Y, int M, int N, int K, void *workspace, size_t ws_bytes, int32_t *status,
                          sp24_stream_t stream);

/*
 * FP4 (OCP E2M1) with 2:4 weights (SlideSparse, §3 "Contribuciones Clave":
 * FP4 among the supported precisions).  The pages give no format; the rule
 * is the per-tensor E4M3 one on the E2M1 grid (magnitudes 0, 0.5, 1, 1.5,
 * 2, 3, 4, 6): s = amax / 6 (1.0 for an all-zero tensor), code =
 * E2M1(RN_fp32(x / s)) to the nearest grid value, ties to the even code,
 * saturating at 6, the sign kept on a value that rounds to zero (code 8);
 * no block scales.  Codes are 4 bits (bit 3 the sign), packed two per byte,
 * element 2i in the low nibble of byte i.
 * fp4_quantize_pertensor: X bf16 [rows, cols] (cols % 32 == 0) -> q u8
 *   [rows, cols / 2], *scale <- s.
 * sp24_prune_compress_fp4: W bf16 [N, K] (K % 64 == 0) -> the 2:4 selection
 *   of sp24_prune_compress in the canonical layout with FP4 codes: values
 *   [N, K/2] codes = u8 [N, K/4], meta [N, K/8], *w_scale <- s.
 * Pointers are device pointers, 16-byte aligned (scale: 4-byte).  Workspace:
 * sp24_workspace_size(SP24_OP_QUANTIZE or SP24_OP_PRUNE_COMPRESS, ...)
 * (256 bytes of counters, zero before and after the call).  Errors as for
 * the E4M3 calls; SP24_STATUS_NONFINITE when the input holds Inf or NaN.
 */
int fp4_quantize_pertensor(const void *X, int64_t rows, int64_t cols, uint8_t *q, float *scale, void *workspace,
                           size_t ws_bytes, int32_t *status, sp24_stream_t stream);
int sp24_prune_compress_fp4(const void *W, int N, int K, uint8_t *values, uint8_t *meta, float *w_scale,
                            void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream);
/*
 * The FP4 sparse GEMM: Y[M, N] = x_scale * w_scale * (Xq . W^T) on the
 * tensor cores (tcgen05.mma.sp kind::f8f6f4 with E2M1 operands, fp32
 * accumulation), bf16 out.  Xq: u8 [M, K / 2] from fp4_quantize_pertensor;
 * values u8 [N, K / 4] and meta [N, K / 8] from sp24_prune_compress_fp4;
 * scales: one device float each.  Shape rules: M >= 1, N % 128 == 0,
 * K % 256 == 0.  Xq and values must be 32-byte aligned (the 4-bit tensor
 * maps), meta and Y 16-byte aligned.  Workspace:
 * sp24_workspace_size(SP24_OP_GEMM_FP4, M, N, K, 0) (zero-filled before the
 * first use, its counters zero again after every call, as for sp24_gemm).
 */
int sp24_gemm_fp4(const uint8_t *Xq, const float *x_scale, const uint8_t *w_values, const uint8_t *w_meta,
                  const float *w_scale, void *Y, int M, int N, int K, void *workspace, size_t ws_bytes,
                  int32_t *status, sp24_stream_t stream);

/*
 * The general (2N-2):2N case through 2:4 windows (SlideSparse, §2
 * "Descomposicion de Ventana Deslizante": N-1 overlapping windows of 4 with
 * stride 2 per 2N-group, expansion (2N-2)/N), for n = N = 3 (4:6), 4 (6:8,
 * the same results as slide68_decompose / slide68_lift) or 5 (8:10).  Each
 * 2n-group keeps its 2n-2 largest |w| (ties to the lower index); window j
 * (positions 2j .. 2j+3) takes, for j = 0 .. n-2 in turn, the two
 * lowest-index kept positions of its range not taken by an earlier window;
 * position p of group g taken by window j goes to column 4((n-1)g + j) +
 * (p - 2j) of W' [N, K' = K (2n-2)/n], stored 2:4-compressed with E4M3
 * codes and the per-tensor w_scale: values [N, K'/2], meta [N, K'/8].
 * slide_lift: X bf16 [M, K] -> q_lifted u8 [M, K'],
 * q_lifted[m, 4((n-1)g + j) + r] = E4M3(X[m, 2n g + 2j + r] / scale), scale
 * <- amax|X| / 448.  Workspace: sp24_workspace_size(SP24_OP_SLIDE68_DECOMPOSE
 * or SP24_OP_SLIDE68_LIFT, ...) (256 bytes of counters).  Shape rules:
 * 3 <= n <= 5, K % 2n == 0, K' % 16 == 0, rows * K % 8 == 0; the GEMM over
 * K' (sp24_gemm, or sp24_gemm_packed after sp24_pack_weights) further needs
 * K' % 128 == 0.
 */
int slide_decompose(const void *W, int N, int K, int n, uint8_t *values, uint8_t *meta, float *w_scale,
                    void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream);
int slide_lift(const void *X, int M, int K, int n, uint8_t *q_lifted, float *scale, void *workspace,
               size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * Finer-grained scales (SlideSparse, §2 "Pipeline de Implementacion": its
 * fused quantiser scales each token; the roadmap, §Interaction avec la
 * quantification: finer scales for outlier layers).  The per-tensor rule of
 * fp8_quantize_pertensor applied to each row on its own.
 *
 * Per-token quantisation: X bf16 [rows, cols] -> q u8 [rows, cols] and
 * scales f32 [rows]: scales[m] = amax|X[m, :]| / 448 (1.0 for an all-zero
 * row), q[m, k] = E4M3(X[m, k] / scales[m]) (correctly rounded fp32
 * quotient, then round to nearest even with saturation).  No workspace.
 * SP24_STATUS_NONFINITE when a row holds NaN/Inf.  Shape rules: rows >= 1,
 * cols % 8 == 0.
 */
int fp8_quantize_pertoken(const void *X, int64_t rows, int64_t cols, uint8_t *q, float *scales,
                          int32_t *status, sp24_stream_t stream);

/*
 * Per-channel 2:4 weight path: the selection of sp24_prune_compress (two
 * largest |w| of each 4, ties to the lower index) with one scale per output
 * channel: w_scales[n] = amax|W[n, :]| / 448 (1.0 for an all-zero row),
 * values u8 [N, K/2] = E4M3 codes of the kept elements of row n divided by
 * w_scales[n], meta u8 [N, K/8] in the canonical layout (sp24_pack_weights
 * makes the tile-packed form).  No workspace.  Shape rules: N >= 1,
 * K % 8 == 0.
 */
int sp24_prune_compress_perchannel(const void *W, int N, int K, uint8_t *values, uint8_t *meta,
                                   float *w_scales, int32_t *status, sp24_stream_t stream);

/*
 * sp24_gemm_packed with scale vectors: Y[m, n] = bf16( x_scale(m) *
 * w_scale(n) * sum_k Xq[m, k] * W[n, k] ), where x_scale(m) = x_scales[m]
 * when x_per_token (M floats), else x_scales[0], and w_scale(n) =
 * w_scales[n] when w_per_channel (N floats), else w_scales[0].  Workspace,
 * layouts and shape rules as sp24_gemm_packed; both scale pointers are
 * required.
 */
int sp24_gemm_packed_scaled(const void *Xq, const float *x_scales, int x_per_token, const void *packed,
                            const float *w_scales, int w_per_channel, void *Y, int M, int N, int K,
                            void *workspace, size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * Dense FP8 GEMM of the same kernel family (comparison baseline for the
 * sparse speedup): Y[M, N] = bf16( x_scale * w_scale * sum_k Xq[m,k] Wq[n,k] )
 * with Xq u8 [M, K], Wq u8 [N, K] (E4M3, e.g. the pruned_dense output of
 * sp24_prune_compress).  Shape rules: M >= 1, N % 128 == 0, K % 128 == 0.
 */
int fp8_gemm_dense(const uint8_t *Xq, const float *x_scale, const uint8_t *Wq,
                   const float *w_scale, void *Y, int M, int N, int K, void *workspace,
                   size_t ws_bytes, int32_t *status, sp24_stream_t stream);

/*
 * fp8_quantize_pertensor for callers that cannot allocate device memory (the
 * pages have no counterpart: this is a deployment convenience).  Engines and
 * plugin hosts that own every device allocation, or hot loops that cannot
 * afford the implicit synchronisation of cudaMalloc/cudaFree, may have no
 * workspace to pass.  This entry point computes exactly what
 * fp8_quantize_pertensor computes (same arguments except the workspace) and
 * keeps the scratch of its amax reduction in a 256-byte static device array
 * inside the library instead; every GPU that loads the library holds those
 * bytes until the process exits.  It calls no allocating routine.
 *   - A decode-sized X (rows * cols <= 131072) uses no scratch at all (one
 *     thread-block cluster, as fp8_quantize_pertensor).
 *   - A larger X looks up the array's device address (cudaGetSymbolAddress)
 *     on every call, with that device current; make the first such call on
 *     a device before any stream capture (it loads the module).
 *   - Such a call clears the array's counters on `stream` before using them
 *     (a copy between the previous kernel and the quantiser, which then
 *     cannot start beside that kernel).  All calls share the one array, so
 *     calls that overlap on the GPU (other streams, other threads) race:
 *     serialise them.
 *   - The scratch needed does not grow with the tensor; a configuration whose
 *     need exceeded the array would be rejected with SP24_ERR_WORKSPACE.
 * Shape rules and errors as fp8_quantize_pertensor.
 */
int fp8_quantize_pertensor_static(const void *X, int64_t rows, int64_t cols, uint8_t *q,
                                  float *scale, int32_t *status, sp24_stream_t stream);

/* Bytes of workspace the op needs for these sizes (0 is a valid answer). */
size_t sp24_workspace_size(int op, int64_t M, int64_t N, int64_t K, int dtype);

/* Human-readable text for a return code. */
const char *sp24_status_str(int code);

/* The last cudaError_t seen by a call that returned SP24_ERR_CUDA (per thread). */
int sp24_last_cuda_error(void);

/*
 * Test hook: E4M3 encoding of fp32 values with the same device routine the
 * quantisation kernels use (round to nearest even, saturate to +-448, sign of
 * zero kept).  v: f32 [n] -> out: u8 [n].  n >= 0.
 */
int sp24_debug_e4m3_encode(const float *v, uint8_t *out, int64_t n, sp24_stream_t stream);

/* Library version string. */
const char *sp24_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SP24_H */
