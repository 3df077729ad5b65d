/*
 * fp4.h -- C ABI of libfp4.so: block-scaled FP4 quantization and block-scaled
 * FP4 GEMMs on NVIDIA B200 (sm_100a).
 *
 * The method (sources are page titles and sections):
 *   - "Pre-addestramento di Modelli Linguistici di Grandi Dimensioni con MXFP4",
 *     Metodologia: MXFP4 on the Fprop, Dgrad and Wgrad GEMMs of every linear
 *     layer, stabilised by deterministic 16x16 / 32x32 Hadamard rotations
 *     (H16 / H32), with stochastic rounding and randomised Hadamard as the
 *     alternatives studied.
 *   - "Ripensare il Bias di Shrinkage nel Pretraining di LLM in FP4",
 *     Problematica and Metodologia 1-2: the E2M1 grid under round-to-nearest-
 *     even, the uniform UFP4 grid (levels k*s, k in [-7, 7]), random Hadamard
 *     on all three GEMMs, stochastic rounding on the upstream gradient.
 *   - "TetraJet-v2", section 2.A: NVFP4 = E2M1 in 16-element groups with an
 *     8-bit (E4M3) scale; the double-block variant, a 128-element outer block
 *     with an FP32 scale over 16-element inner blocks; stochastic rounding in
 *     the backward pass; 1x16 weight groups re-quantized along the transposed
 *     axis for the backward GEMMs.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers of the current CUDA device, owned
 *     and allocated by the caller; the library allocates no memory and keeps
 *     no per-call state.
 *   - `stream` is a cudaStream_t passed as void* (NULL: the legacy default
 *     stream).  Calls are asynchronous on it: outputs are valid once the
 *     stream has reached the call.
 *   - Argument, shape and alignment errors are returned synchronously and
 *     nothing is launched.  A failed launch returns FP4_ERR_CUDA.  A bounded
 *     device-side wait that ran out (a GEMM pipeline hand-off, a ring wait
 *     or the grid barrier of the row-axis quantizer) is reported by
 *     fp4_last_error() as FP4_ERR_TIMEOUT.
 *   - Pointers to tensor data must be 16-byte aligned.
 *
 * Quantized tensor ("K-major view")
 *   A quantized tensor has L lines of K elements each, quantized along the
 *   line.  For axis = 1 the lines are the rows of the [R, C] input (L = R,
 *   K = C); for axis = 0 they are its columns (L = C, K = R), so the output is
 *   the transposed tensor, as the Dgrad / Wgrad operands need.
 *     codes   uint8 [L, K/2]: 4-bit codes, element 2j in the low nibble of
 *             byte j.  Code = sign << 3 | magnitude index; E2M1 magnitudes
 *             {0, .5, 1, 1.5, 2, 3, 4, 6}, UFP4 magnitudes k = 0..7.
 *     scales  one byte per block of the line (block 32 for MXFP4: E8M0, value
 *             2^(byte - 127); block 16 for NVFP4/UFP4: E4M3), in the tiled
 *             layout below.
 *     outer   float [L, K/128] row-major (double block only).
 *     tensor_scale  one float (NVFP4/UFP4 without double block).
 *   Element value = q * s_block (MXFP4), q * s_block * tensor_scale (NVFP4,
 *   UFP4), q * s_block * outer[l][k/128] (double block).
 *
 * Tiled scale layout (the layout the tcgen05 block-scaled MMA reads): with
 * nb = K / block scale bytes per line, the byte of line l, block b is at
 *     ((l / 128) * ceil(nb / 4) + b / 4) * 512
 *       + (l % 32) * 16 + ((l % 128) / 32) * 4 + (b % 4)
 * and the buffer holds fp4_scales_bytes(L, K, format) bytes (L rounded up to
 * 128 and nb to 4).  Padding bytes are never written.
 */
#ifndef FP4_H
#define FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size */
    FP4_ERR_UNSUPPORTED_SHAPE = 2, /* a size breaks the shape rules */
    FP4_ERR_MISALIGNED = 3,        /* a pointer or leading dimension is not 16-byte aligned */
    FP4_ERR_WORKSPACE = 4,         /* workspace missing or too small */
    FP4_ERR_NO_DEVICE = 5,         /* no CUDA device, or not a B200-class (sm_100) device */
    FP4_ERR_CUDA = 6,              /* a CUDA runtime call failed */
    FP4_ERR_TIMEOUT = 7,           /* a device-side wait gave up (reported by fp4_last_error) */
    FP4_ERR_UNSUPPORTED = 8        /* a valid combination this build does not implement */
} fp4_status_t;

typedef enum { FP4_MXFP4 = 0, FP4_NVFP4 = 1, FP4_UFP4 = 2 } fp4_format_t;
typedef enum { FP4_RTNE = 0, FP4_SR = 1 } fp4_rounding_t;
typedef enum {
    FP4_ROT_NONE = 0,
    FP4_ROT_H16 = 1,   /* deterministic 16x16 Sylvester Hadamard, scaled by 1/4 */
    FP4_ROT_H32 = 2,   /* deterministic 32x32, scaled by binary32(1/sqrt(32)) */
    FP4_ROT_RH16 = 3,  /* random signs then H16 */
    FP4_ROT_RH32 = 4   /* random signs then H32 */
} fp4_rotation_t;
typedef enum { FP4_IN_F32 = 0, FP4_IN_BF16 = 1 } fp4_in_dtype_t;
typedef enum { FP4_OUT_F32 = 0, FP4_OUT_BF16 = 1 } fp4_out_dtype_t;

/*
 * fp4_scales_bytes -- size in bytes of the tiled scale buffer of a quantized
 * tensor with `lines` lines of K elements in `format` (0 for an empty tensor).
 */
size_t fp4_scales_bytes(int64_t lines, int64_t K, fp4_format_t format);

/*
 * fp4_quantize_workspace_size -- device workspace fp4_quantize needs for this
 * format / amax choice: 256 bytes when the tensor amax is computed internally
 * (NVFP4 or UFP4, no double block, tensor_amax == NULL), otherwise 0.
 * Returns FP4_ERR_INVALID_ARG for a bad format or a null `bytes`.
 */
fp4_status_t fp4_quantize_workspace_size(fp4_format_t format, int double_block,
                                         int amax_given, size_t* bytes);

/*
 * fp4_amax -- amax of the rotated tensor: max |y| over all elements, where y
 * is x rotated on every aligned n-block along the quantization axis (no
 * rotation: max |x|).  This is the amax the NVFP4 / UFP4 tensor scale
 * amax / (Q * 448) is taken from ("TetraJet-v2" 2.A: the tensor-wide amax that
 * the double block avoids); calling it separately lets a caller combine the
 * amax of several shards (a max all-reduce) before quantizing each shard.
 *
 *   x         device, [rows, ld] row-major, `cols` <= ld valid columns
 *   rotation  rotation along the axis; its size must divide the axis length
 *   seed      selects the random signs of FP4_ROT_RH16 / RH32
 *   amax_out  device, one float, overwritten
 * Empty input (rows or cols == 0) writes 0.
 */
fp4_status_t fp4_amax(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols,
                      int64_t ld, fp4_rotation_t rotation, int axis, uint64_t seed,
                      float* amax_out, void* stream);

/*
 * fp4_rotate -- the rotation of fp4_quantize's step 2 alone, as a separate
 * pass: y = c_n * H_n * (d . x) on every aligned n-block of each row, in
 * binary32 with the same operation order, stored in the input's type (bf16:
 * rounded to nearest even).  "Ripensare il Bias di Shrinkage nel Pretraining
 * di LLM in FP4", Efficienza: the pages time a separate rotation kernel
 * followed by the quantizer against the fused quantizer; this call is that
 * separate kernel.
 *
 *   x, in_dtype, rows, cols, ld   input [rows, ld] row-major (as fp4_quantize)
 *   rotation        FP4_ROT_H16 / H32 / RH16 / RH32 (not NONE); n divides cols
 *   axis            must be 1 (rows); any other value returns FP4_ERR_UNSUPPORTED
 *   seed            the random signs of RH16 / RH32
 *   y, ldy          device, [rows, ldy] of the input's type, ldy >= cols,
 *                   16-byte aligned; may not overlap x
 */
fp4_status_t fp4_rotate(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                        fp4_rotation_t rotation, int axis, uint64_t seed, void* y, int64_t ldy, void* stream);

/*
 * fp4_quantize -- fused rotate / amax / scale / round / pack of one tensor.
 *
 * Steps, on every line of K elements along `axis`:
 *   1. load and widen to binary32 (bf16 -> f32 is exact);
 *   2. rotation (optional): x <- d . x (random signs: bit j of word 0 of
 *      Philox4x32-10(key = seed, counter = (0, 0, 0, 1)), set = -1), then the
 *      Sylvester butterfly in binary32 for h = 1, 2, ..., n/2, then times
 *      c_n (c_16 = 0.25, c_32 = binary32(1/sqrt 32));
 *   3. scale per block, with m the block amax:
 *      MXFP4 (block 32): e = clamp(floor(log2 m) - 2, -127, 127) (m = 0:
 *        -127), byte e + 127, v = x * 2^-e;
 *      NVFP4 / UFP4 (block 16, Q = 6 / 7): s_t = A / (Q * 448) from the
 *        tensor amax A (1 if that is 0: A = 0 or an underflowing quotient),
 *        s_b = E4M3_rne_satfinite((m / Q) / s_t),
 *        v = x / (s_b * s_t); s_b = 0 gives signed zero codes;
 *      double block (NVFP4 only): s_o = m128 / 2688 per 128-element chunk of
 *        the line (1 if that is 0) replaces s_t;
 *   4. round |v| onto the grid (clamped to the top level), sign from x:
 *      FP4_RTNE: nearest, ties to the even magnitude index;
 *      FP4_SR: up from the level below with probability (|v| - lo)/(hi - lo),
 *        using word (i mod 4) of Philox4x32-10(key = seed, counter =
 *        (lo32(i/4), hi32(i/4), tensor_id, 0)) for input element (r, c),
 *        i = r * cols + c: up iff (word >> 8) * 2^-24 < (|v| - lo)/(hi - lo);
 *   5. pack two codes per byte and store codes and scales.
 *
 * Arguments
 *   x, in_dtype, rows, cols, ld   input [rows, ld] row-major, `cols` valid
 *                                 columns; ld * sizeof(element) % 16 == 0
 *   format, rounding, rotation    as above
 *   axis            1: lines are rows (K = cols); 0: lines are columns
 *                   (K = rows), i.e. the transposed tensor is written
 *   double_block    NVFP4 only: FP32 outer scale per 128 elements
 *   seed, tensor_id SR stream and random signs (tensor_id only for SR)
 *   tensor_amax     optional device float: the rotated-tensor amax to build
 *                   s_t from (e.g. the max over shards); NULL = computed here,
 *                   which needs the workspace.  On the row axis (axis = 1)
 *                   the amax pass and the quantize pass then run as one
 *                   cooperative launch whose CTAs meet at a grid barrier (the
 *                   second read of x mostly hits L2); on axis 0 they are two
 *                   launches
 *   codes           device uint8 [L, K/2]
 *   scales          device, fp4_scales_bytes(L, K, format) bytes, tiled layout
 *   outer_scales    device float [L, K/128] (double block), else ignored
 *   tensor_scale    device float, receives s_t (NVFP4/UFP4, no double block)
 *   workspace       device, >= fp4_quantize_workspace_size() bytes, 16-byte
 *                   aligned; contents are scratch
 * Shape rules: K % block == 0 (32 MXFP4, 16 NVFP4/UFP4), K % n == 0 for a
 * rotation of size n, K % 128 == 0 for double block; L may be anything >= 0.
 */
fp4_status_t fp4_quantize(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols,
                          int64_t ld, fp4_format_t format, fp4_rounding_t rounding,
                          fp4_rotation_t rotation, int axis, int double_block,
                          uint64_t seed, uint32_t tensor_id, const float* tensor_amax,
                          uint8_t* codes, uint8_t* scales, float* outer_scales,
                          float* tensor_scale, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * fp4_quantize_both_axes -- fp4_quantize of one tensor along both axes in a
 * single pass over it.  Every linear layer needs each of its tensors along
 * both axes: X along its rows for Fprop and along its columns for Wgrad, W
 * along its rows for Fprop and its columns for Dgrad, dY along its rows for
 * Dgrad and its columns for Wgrad ("Pre-addestramento di Modelli Linguistici
 * di Grandi Dimensioni con MXFP4", Metodologia: the three GEMMs of a linear;
 * "TetraJet-v2" 2.A: the 1x16 groups re-aligned for the transposed operand).
 * The results are exactly those of two fp4_quantize calls with the internal
 * tensor amax:
 *   rows:    axis = 1, rounding_rows, tensor_id_rows -> codes_rows [rows, cols/2],
 *            scales_rows (fp4_scales_bytes(rows, cols, format)), tensor_scale_rows
 *   columns: axis = 0, rounding_cols, tensor_id_cols -> codes_cols [cols, rows/2],
 *            scales_cols (fp4_scales_bytes(cols, rows, format)), tensor_scale_cols
 * with the same format, rotation and seed.  Each axis has its own rotated
 * amax and tensor scale.  The tensor is read once from HBM for both amax
 * passes and once more (mostly from L2) for both quantize passes, in one
 * cooperative launch whose CTAs meet at a bounded grid barrier.
 *
 *   x, in_dtype, rows, cols, ld   as fp4_quantize; in_dtype must be FP4_IN_BF16
 *   format          FP4_NVFP4 or FP4_UFP4 (no double block)
 *   rotation        FP4_ROT_NONE or FP4_ROT_H16
 *   workspace       device, >= 256 bytes (fp4_quantize_workspace_size with the
 *                   internal amax), 16-byte aligned; contents are scratch
 * Shape rules: rows % 16 == 0, cols % 64 == 0.  Valid combinations outside the
 * ones above (f32 input, MXFP4, other rotations) return FP4_ERR_UNSUPPORTED:
 * use two fp4_quantize calls.  Other errors as fp4_quantize; nothing is
 * launched on an error.  A grid-barrier or ring wait that runs out sets
 * FP4_ERR_TIMEOUT for fp4_last_error (the outputs are then not valid).
 */
fp4_status_t fp4_quantize_both_axes(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols,
                                    int64_t ld, fp4_format_t format, fp4_rotation_t rotation, uint64_t seed,
                                    fp4_rounding_t rounding_rows, uint32_t tensor_id_rows, uint8_t* codes_rows,
                                    uint8_t* scales_rows, float* tensor_scale_rows,
                                    fp4_rounding_t rounding_cols, uint32_t tensor_id_cols, uint8_t* codes_cols,
                                    uint8_t* scales_cols, float* tensor_scale_cols, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * fp4_requantize -- re-quantize an already quantized tensor along the other
 * axis.  "TetraJet-v2", section 2.A: the backward pass estimates with X^, the
 * dequantized forward operand, rather than X ("aligning the tensors"), and the
 * 1x16 weight groups need a matching alignment for the transposed weight.  The
 * Dgrad / Wgrad operand is therefore the forward tensor's dequantized values
 * quantized along the transposed axis, not the original bf16 tensor.
 *
 * The source is a quantized tensor of `lines` lines with K elements each,
 * read as the logical matrix X^ [lines, K].  Each element of X^ is the
 * dequantized value rounded once to binary32: RN(q * s_block * s_ref), with
 * s_ref the tensor scale, the outer scale (double block) or 1 (MXFP4).  The
 * product q * s_block is exact in binary32.  The result is what fp4_quantize
 * gives for that binary32 X^ with axis = 0: K lines of `lines` elements, with
 * the same rotation, scale, rounding and SR-counter rules (element (r, c) of
 * X^ has index i = r * K + c).  The source must not be rotated: undoing a
 * rotation along the source axis is not part of this call.
 *
 * Arguments
 *   src_codes, src_scales, src_outer, src_tensor_scale, lines, K,
 *   src_format, src_double_block   the source, laid out as fp4_quantize
 *                                  writes it (src_outer for double block,
 *                                  src_tensor_scale for NVFP4 / UFP4 without it)
 *   format ... workspace_bytes     the result, as in fp4_quantize, for an
 *                                  input of `lines` rows and K columns on axis 0
 * Shape rules: K % 16 == 0 and K % (source block) == 0 (128 for a double-block
 * source); `lines` % (result block) == 0, % rotation size, % 128 for a
 * double-block result.  src_codes and codes 16-byte aligned.  Errors as
 * fp4_quantize; nothing is launched on an error.
 */
fp4_status_t fp4_requantize(const uint8_t* src_codes, const uint8_t* src_scales, const float* src_outer,
                            const float* src_tensor_scale, int64_t lines, int64_t K, fp4_format_t src_format,
                            int src_double_block, fp4_format_t format, fp4_rounding_t rounding,
                            fp4_rotation_t rotation, int double_block, uint64_t seed, uint32_t tensor_id,
                            const float* tensor_amax, uint8_t* codes, uint8_t* scales, float* outer_scales,
                            float* tensor_scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fp4_mxnorm_quantize -- MXNorm fused with the FP4 cast.  "MXNorm: Reusing
 * MXFP block scales for efficient tensor normalisation", 2. Metodologia: the
 * inverse RMS of each row t is estimated from the absolute maxima m_tk of the
 * row's K blocks -- the maxima the cast's block scales come from --
 *     rho_t = c * ((1/K) sum_k m_tk^p)^(-1/p),   p = 1 or 2,
 * and the normalised row y = x * rho_t is what gets quantized (the norm's
 * gain is folded into the next layer's weight, as the page does).
 *
 * Arithmetic: m_tk in binary32 over blocks of 32 (MXFP4) or 16 (NVFP4 /
 * UFP4); the sum of m_tk^p in binary64, pairwise in block order (the sum of a
 * range is the sum of its two halves, split at the largest power of two
 * below its length); the mean, the square root (p = 2) and c / g correctly
 * rounded in binary64, then rounded once to binary32 and saturated at the
 * largest finite binary32 (an all-zero row: rho = 1); y = RN32(x * rho_t).
 * y is then quantized along the rows exactly as fp4_quantize would quantize
 * it with no rotation: MXFP4 block scales, or the NVFP4 / UFP4 block scales
 * under the tensor scale of y's amax (max_t RN(max|x_t| rho_t)).
 *
 *   x, in_dtype, rows, cols, ld  input [rows, ld] row-major, cols valid;
 *                 cols % 32 (MXFP4) or % 16 (NVFP4, UFP4) == 0, cols <= 16384
 *   p, c          the mean's order (1 or 2) and the constant c(p, B) > 0
 *                 (finite): the page takes it from a Monte Carlo simulation;
 *                 for rows of i.i.d. Gaussian values E[M^p]^(1/p), M the
 *                 maximum of B independent |N(0, 1)|, makes rho_t tend to
 *                 1 / RMS (about 2.35 for p = 1 and 2.39 for p = 2, B = 32)
 *   seed, tensor_id   stochastic rounding, as fp4_quantize (element i = r * cols + c)
 *   codes, scales, tensor_scale   the quantized y, as fp4_quantize on axis 1
 *   rho           device float [rows]: rho_t (for the backward pass)
 *   workspace     NVFP4 / UFP4: >= 256 bytes, 16-byte aligned (the amax of
 *                 y); MXFP4 needs none
 * MXFP4 runs one kernel; NVFP4 / UFP4 a statistics kernel (rho, amax of y)
 * and then the cast.  Errors as fp4_quantize.
 */
fp4_status_t fp4_mxnorm_quantize(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                                 fp4_format_t format, fp4_rounding_t rounding, int p, float c, uint64_t seed,
                                 uint32_t tensor_id, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                 float* rho, void* workspace, size_t workspace_bytes, void* stream);

/*
 * OutControl ("TetraJet-v2", 2.C): a few activation channels carry outliers
 * and do so consistently, so the top p% of the channels (the columns of the
 * activation, i.e. the GEMM's contraction index), chosen once in a short
 * calibration window, are kept in FP8 for the forward and backward passes and
 * the rest stays FP4.  The split of a [rows, cols] operand:
 *   FP4 part   the operand with those channels set to +0, quantized to NVFP4
 *              along the rows exactly as fp4_quantize does (so the outliers
 *              no longer set its tensor and block scales);
 *   FP8 part   the operand's channels, gathered in list order into
 *              [rows, k8] E4M3 codes (sign in bit 7, zero past the list) under
 *              one FP32 tensor scale s8 = amax / 448 (1 if that is 0):
 *              code = E4M3_rne_satfinite(RN(x / s8)).
 * Both GEMM operands are split with the same channel list, and
 *     C = a4 b4 (FP4 product) + s8A s8B (FP8 product)
 * runs in one kernel (fp4_gemm_outctl).
 */

/*
 * fp4_channel_amax -- the calibration statistic: amax_out[c] = max_r |x[r, c]|
 * for a [rows, ld] row-major input (device float [cols], overwritten).  The
 * caller picks its top channels from it.
 */
fp4_status_t fp4_channel_amax(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                              float* amax_out, void* stream);

/* fp4_outctl_workspace_size -- workspace bytes of fp4_outctl_quantize for `cols` columns. */
fp4_status_t fp4_outctl_workspace_size(int64_t cols, size_t* bytes);

/*
 * fp4_outctl_quantize -- the OutControl split of one operand (above).
 *   x, in_dtype, rows, cols, ld   input [rows, ld] row-major; cols % 16 == 0
 *   channels, n_channels  device int32 [n_channels], ascending, unique, in
 *                 [0, cols) (an index outside is skipped and reported by
 *                 fp4_last_error as FP4_ERR_INVALID_ARG)
 *   k8            columns of the FP8 part: n_channels <= k8, k8 % 128 == 0
 *   rounding, rotation, seed, tensor_id   of the FP4 part, as fp4_quantize
 *   codes, scales, tensor_scale   the FP4 part, as fp4_quantize on axis 1
 *   codes8        device uint8 [rows, k8], 16-byte aligned
 *   scale8        device float, receives s8
 *   workspace     >= fp4_outctl_workspace_size(cols) bytes, 16-byte aligned
 */
fp4_status_t fp4_outctl_quantize(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols, int64_t ld,
                                 const int32_t* channels, int64_t n_channels, int64_t k8, fp4_rounding_t rounding,
                                 fp4_rotation_t rotation, uint64_t seed, uint32_t tensor_id, uint8_t* codes,
                                 uint8_t* scales, float* tensor_scale, uint8_t* codes8, float* scale8,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * fp4_gemm_outctl -- C = a4 b4 sum_k qA qB sA sB + s8A s8B sum_k8 eA eB for the
 * split operands A [M, K] / [M, K8] and B [N, K] / [N, K8] of
 * fp4_outctl_quantize: the NVFP4 product and the E4M3 product (tcgen05
 * kind::f8f6f4) accumulate in two TMEM accumulators of one tile, and each
 * output element is formed and rounded once.
 *   c, out_dtype, ldc   as fp4_gemm
 * Shape rules: M, N, K multiples of 128 (K > 0), K8 a multiple of 128 (0: no
 * FP8 part, the FP8 pointers may be NULL); code pointers 16-byte aligned.
 */
fp4_status_t fp4_gemm_outctl(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_tensor_scale,
                             const uint8_t* b_codes, const uint8_t* b_scales, const float* b_tensor_scale,
                             const uint8_t* a8_codes, const float* a8_scale, const uint8_t* b8_codes,
                             const float* b8_scale, int64_t M, int64_t N, int64_t K, int64_t K8, void* c,
                             fp4_out_dtype_t out_dtype, int64_t ldc, void* stream);

/*
 * fp4_quantize_noalloc -- fp4_quantize for NVFP4 / UFP4 with the tensor scale
 * taken from an internal amax, for callers that cannot allocate device
 * memory: code running where cudaMalloc is unavailable or forbidden (a plug-in
 * whose host framework owns every device allocation, a real-time loop that may
 * not touch the allocator) and so cannot supply the 256-byte workspace
 * fp4_quantize asks for.  The pages have no counterpart to this call; it only
 * changes where the scratch lives.
 *
 * The scratch is a static device array of 256 bytes inside libfp4.so (two
 * 32-bit words are used: the amax and a grid-barrier count); every GPU that
 * loads the library holds one copy
 * until the process exits.  A request needing more scratch than that returns
 * FP4_ERR_WORKSPACE (every NVFP4 / UFP4 shape needs exactly the 256 bytes).
 * The caller still owns x, codes, scales and tensor_scale, with the layouts,
 * shape rules and steps of fp4_quantize (double_block = 0, tensor_amax NULL).
 * MXFP4 needs no scratch and returns FP4_ERR_UNSUPPORTED here: use
 * fp4_quantize with no workspace.
 *
 * The first call on a device resolves the array's device address on that
 * device (cudaGetSymbolAddress), so make it before any stream capture.  Every
 * call shares the one array and leaves its amax there; each call clears the
 * words before accumulating into them.  Calls that overlap on the GPU (other
 * streams, other threads, concurrent graph launches) race on them and
 * must be serialized by the caller.  Allocates nothing; errors as
 * fp4_quantize, checked before anything is launched.
 */
fp4_status_t fp4_quantize_noalloc(const void* x, fp4_in_dtype_t in_dtype, int64_t rows, int64_t cols,
                                  int64_t ld, fp4_format_t format, fp4_rounding_t rounding,
                                  fp4_rotation_t rotation, int axis, uint64_t seed, uint32_t tensor_id,
                                  uint8_t* codes, uint8_t* scales, float* tensor_scale, void* stream);

/*
 * fp4_gemm_workspace_size -- device workspace fp4_gemm needs: for UFP4 the
 * two operands rewritten as E2M1 parts (see fp4_gemm), about 2 (M + N) K
 * bytes of codes plus their scales; 0 for MXFP4 and NVFP4.  Returns
 * FP4_ERR_INVALID_ARG for a bad format or size or a null `bytes`.
 */
fp4_status_t fp4_gemm_workspace_size(fp4_format_t format, int double_block, int64_t M, int64_t N, int64_t K,
                                     size_t* bytes);

/*
 * fp4_gemm -- block-scaled FP4 GEMM on tcgen05 tensor cores:
 *     C[i, j] = alpha_ij * sum_k qA[i, k] qB[j, k] sA[i, k/blk] sB[j, k/blk]
 * with A [M, K] and B [N, K] quantized tensors in the K-major view (lines
 * along K) of the same format, as fp4_quantize writes them:
 *   MXFP4:  alpha = 1, blk = 32 (E8M0 scales);
 *   NVFP4:  alpha = a_tensor_scale * b_tensor_scale, blk = 16 (E4M3);
 *   UFP4:   as NVFP4, with q the uniform levels k in [-7, 7] ("Ripensare il
 *           Bias di Shrinkage nel Pretraining di LLM in FP4", Metodologia 2).
 *           The tensor cores take E2M1 codes only, and 5 and 7 are not E2M1
 *           values; but every level is a1 + a2 with a1 in {0,1,2,3,4,4,6,6}
 *           and a2 in {0,0,0,0,0,1,0,1} (both E2M1 under the same block
 *           scale), so A B^T = A1 B1^T + A1 B2^T + A2 B1^T + A2 B2^T exactly.
 *           The call writes [A1 A2 A1 A2] and [B1 B1 B2 B2] into the workspace
 *           (one pass over each operand) and runs one NVFP4 GEMM over 4 K:
 *           four times the tensor-core work of an NVFP4 GEMM;
 *   double block: alpha varies per 128-element K chunk:
 *           a_outer[i, k/128] * b_outer[j, k/128].
 * This is the Fprop (Y = X W^T), Dgrad (dX = dY W: B = W quantized on
 * axis 0) and Wgrad (dW = dY^T X: both quantized on axis 0) GEMM of a linear
 * layer ("Pre-addestramento ... con MXFP4", Metodologia).  Rotations cancel
 * in the contraction only if both operands used the same rotation and seed;
 * the GEMM applies no inverse rotation.
 *
 *   c         device, [M, ldc] row-major, fp32 or bf16, ldc >= N
 *   workspace device, >= fp4_gemm_workspace_size() bytes, 16-byte aligned
 *             (UFP4 only; NULL and 0 otherwise); contents are scratch
 * Shape rules: M % 128 == 0, N % 128 == 0, K % 128 == 0; ldc * size % 16 == 0.
 * The accumulation is FP32 on the tensor cores.
 */
fp4_status_t fp4_gemm(fp4_format_t format, int double_block,
                      const uint8_t* a_codes, const uint8_t* a_scales,
                      const float* a_outer, const float* a_tensor_scale,
                      const uint8_t* b_codes, const uint8_t* b_scales,
                      const float* b_outer, const float* b_tensor_scale,
                      int64_t M, int64_t N, int64_t K,
                      void* c, fp4_out_dtype_t out_dtype, int64_t ldc,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * fp4_last_error -- synchronizes `stream` and returns (and clears) the device
 * error word the kernels set: FP4_ERR_TIMEOUT when a bounded wait gave up (a
 * GEMM pipeline hand-off, a quantizer ring wait or its grid barrier; the kernel
 * then lets its own copies in flight land, frees what it holds and exits; its
 * outputs are not valid), FP4_OK otherwise, FP4_ERR_CUDA if the
 * synchronization failed.
 */
fp4_status_t fp4_last_error(void* stream);

/* fp4_status_string -- a static, human-readable name of a status code. */
const char* fp4_status_string(fp4_status_t status);

/*
 * fp4_set_wait_limit -- iteration limit of the bounded device-side waits of
 * later calls (default 2^20 polls, far above any legitimate wait): a GEMM
 * hand-off polls at most this many times, a quantizer ring wait 16 times as
 * many and the quantizer's grid barrier 4 times as many (32 ns sleeps).  A
 * test can lower it to make a wait run out without hanging the GPU.  0
 * restores the default.  Process-wide; not synchronized with calls in flight
 * on other host threads.
 */
void fp4_set_wait_limit(uint32_t polls);

/*
 * fp4_set_gemm_cta_pairs -- whether later fp4_gemm calls (MXFP4, NVFP4 and
 * UFP4; not the double block) with M and N multiples of 256 run on CTA pairs:
 * 256 x 256 output tiles shared by two SMs through tcgen05 cta_group::2, each
 * SM loading its own A rows and half of B (nonzero, the default), or on single
 * CTAs with 128 x 256 tiles (0).  The products are the same block-scaled dot
 * products either way.  Process-wide; not synchronized with calls in flight on
 * other host threads.
 */
void fp4_set_gemm_cta_pairs(int enable);

#ifdef __cplusplus
}
#endif

#endif /* FP4_H */
