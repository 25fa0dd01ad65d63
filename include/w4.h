/*
 * w4.h -- C ABI of libw4: group-wise INT4 weight quantization and the W4A16
 * product on NVIDIA B200 (sm_100a).
 *
 * The method (web pages on LLM quantization, "page N" below):
 *   page 5, ai-infra.cypggs.com .../model-quantization/02-core-ideas, section 2.2:
 *     symmetric  q = clip(round(x/s), -8, 7),       s = max|x| / 7
 *     asymmetric q = clip(round(x/s) + zp, 0, 15),  s = (max - min) / 15,
 *                zp = round(-min/s)
 *     dequantize x^ = (q - zp) * s, rounding is round-to-nearest-even.
 *   page 2, learn.longtimenohack.com .../quantization.html, item (1) group
 *     quantization: rows are cut into groups of g weights that share one fp16
 *     scale and an integer zero-point (g = 128 gives 4.125 bits per weight).
 *   page 3, blog.freezetheflame.cc .../quantization-deep-dive.html, section 1.2
 *     (dequantize fused into the GEMM so weights stay 4-bit in memory), 2.2
 *     (per-group scales have shape [C_out, num_groups]), 5.3 (the smoothing
 *     vector s is folded into the weights offline, W * s, and the activations
 *     are divided by s upstream).
 *   page 5 section 2.4 and page 1 (AWQ): X' = X/s, W' = W * diag(s) leaves
 *     X W^T unchanged.
 *
 * Exact semantics (fixed where the pages leave a step open):
 *   w'   = fl32(float(w[n][k]) * s[k])        (w' = float(w) when s == NULL)
 *   sym  : amax = max|w'| over the group, s32 = fl32(amax / 7)
 *   asym : mn = min(0, min w'), mx = max(0, max w'), s32 = fl32(fl32(mx - mn) / 15)
 *   s16  = fp16_rne(s32), saturated to 65504 (the stored scale)
 *   zp   = sym: 8;  asym: clip(rint(fl32(-mn / s16)), 0, 15)   (0 when s16 == 0)
 *   u    = sym: clip(rint(fl32(w' / s16)), -8, 7) + 8
 *          asym: clip(rint(fl32(w' / s16)) + zp, 0, 15)
 *          (the zero code, 8 or 0, when s16 == 0); rint = round half to even
 *   w^   = bf16_rne(float(u - zp) * float(s16))   (the product is exact in fp32)
 *   Y[m][n] = bf16_rne(sum_k x[m][k] * w^[n][k]) with fp32 accumulation.
 *
 * Packed layout, version W4_LAYOUT_VERSION (all arrays row-major, C order):
 *   qweight  uint32 [N][K/8]:   word c of row n holds elements k = 8c..8c+7;
 *            bits [4i, 4i+4) hold u of element 8c+2i and bits [16+4i, 16+4i+4)
 *            hold u of element 8c+2i+1 (i = 0..3): even elements in the low
 *            half-word, odd elements in the high half-word.
 *   scales   fp16 [N][K/g]:     s16 of group j = k/g.
 *   qzeros   uint32 [N][ceil(K/g/8)], asymmetric mode only: bits [4(j%8), 4(j%8)+4)
 *            of word j/8 hold zp of group j; unused nibbles are 0.
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned unless stated otherwise; the library allocates no device memory
 *     and keeps no state between calls (except w4a16_gemm_noalloc's fixed
 *     scratch array, described there).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream).  Calls are asynchronous: the library never synchronizes.
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and returns W4_ERR_INVALID_ARG or
 *     W4_ERR_UNSUPPORTED.  A launch failure returns W4_ERR_CUDA.  No exception
 *     crosses the ABI and the library never aborts the process.
 *   - Inputs must be finite; NaN/Inf inputs give unspecified codes.
 *   - There is no CPU fallback: a shape the kernels do not cover is rejected.
 */
#ifndef W4_H
#define W4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4_LAYOUT_VERSION 1

/* A cudaStream_t (the runtime's stream handle type); NULL = default stream. */
typedef struct CUstream_st *w4_stream_t;

typedef enum {
    W4_OK = 0,
    W4_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad group or mode   */
    W4_ERR_UNSUPPORTED = 2,   /* well-formed request outside what the kernels cover     */
    W4_ERR_CUDA = 3           /* a CUDA runtime call or launch failed                   */
} w4_status;

typedef enum { W4_SYM = 0, W4_ASYM = 1 } w4_mode;

/*
 * W4_WEIGHTS_STATIC -- a flag OR-ed into the `mode` argument of w4a16_gemm and
 * w4a16_gemm_noalloc (never of w4_quant_pack), and the `flags` of w4_mx_gemm.  It declares that the packed
 * weight, its scales and its zero-points are NOT written by the kernel that
 * immediately precedes this call on `stream` -- the usual case for model
 * weights quantized once at load time.  The product may then start reading
 * the weight before that kernel has finished (programmatic dependent launch;
 * only the activations wait for it), so in a decode loop the weight stream of
 * one layer overlaps the tail of the previous kernel.  The results are the
 * same bits as without the flag.  If the declaration is false (the weight is
 * quantized by the kernel right before this call, on the same stream), the
 * result is undefined.  The tensor-core path (M > 16) ignores the flag.
 */
#define W4_WEIGHTS_STATIC 0x100

/*
 * W4_OUT_F32 -- a flag OR-ed into the `mode` argument of w4a16_gemm and
 * w4a16_gemm_noalloc: Y is fp32 [M][N] (4-byte aligned) and holds the fp32
 * sums themselves, not their bf16 rounding.  Used by a row-parallel (k-split)
 * product, whose partial sums are added across devices before the one bf16
 * rounding (w4_f32_to_bf16).
 */
#define W4_OUT_F32 0x200

/*
 * W4_REPACKED -- a flag OR-ed into the `mode` argument of w4a16_gemm and
 * w4a16_gemm_noalloc: `qweight` is in the layout that w4_repack writes (the
 * GEMV's 16-channel x 256-k boxes stored one after another), not the canonical
 * [N][K/8].  The codes are the same, and so is every bit of Y.  Served by the
 * GEMV only: M <= 16 and K % 256 == 0, else W4_ERR_UNSUPPORTED.
 */
#define W4_REPACKED 0x400

/* Block-scaled FP4 kinds for w4_fp4_quant. */
typedef enum { W4_NVFP4 = 0, W4_MXFP4 = 1 } w4_fp4_kind;

/*
 * w4_quant_pack -- fold, group-quantize and pack a bf16 weight matrix.
 *   (page 5 section 2.2 formulas; page 2 group quantization; page 3 sections
 *    2.2 and 5.3 for the scale shape and the fold)
 *   W        bf16 [N][K], row k-contiguous, 32-byte aligned.
 *   N, K     N >= 1; K >= 8, K % group == 0.
 *   group    32, 64 or 128.
 *   mode     W4_SYM or W4_ASYM.
 *   s        fp32 [K] smoothing vector folded into W (w' = w * s[k]), or NULL.
 *   qweight  out, uint32 [N][K/8] (layout above).
 *   scales   out, fp16 [N][K/group]; only 2-byte alignment required.
 *   qzeros   out, uint32 [N][ceil(K/group/8)]; must be NULL in W4_SYM mode and
 *            non-NULL in W4_ASYM mode; only 4-byte alignment required.
 * Every output byte is written; outputs must not overlap inputs.
 */
w4_status w4_quant_pack(const void *W, int64_t N, int64_t K, int group, int mode, const float *s,
                        uint32_t *qweight, void *scales, uint32_t *qzeros, w4_stream_t stream);

/*
 * w4a16_workspace_bytes -- device scratch that w4a16_gemm needs for this
 * shape (split-K partial sums and tile counters), 0 if none.  The workspace
 * must be zero-filled before its first use with a given shape; every
 * successful call leaves it zero-filled again, so one zeroed buffer can be
 * reused across calls on the same stream.
 */
size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K, int group);

/*
 * w4a16_gemm -- Y = X . W^T with W^ dequantized on the fly from the packed
 * layout (page 3 section 1.2: dequantize fused into the GEMM; page 5 section
 * 2.2: x^ = (q - zp) * s).
 *   X        bf16 [M][K] activations, already divided by the smoothing vector
 *            when one was folded into W (page 3 section 5.3).
 *   M, N, K  M >= 1, N >= 1, K % group == 0, K >= group.
 *   qweight, scales, qzeros, group, mode: as produced by w4_quant_pack
 *            (qzeros NULL in W4_SYM mode).
 *   Y        out, bf16 [M][N] (fp32 [M][N], 4-byte aligned, with W4_OUT_F32).
 *   workspace, workspace_bytes: device scratch of at least
 *            w4a16_workspace_bytes(M, N, K, group) bytes (may be NULL when
 *            that is 0); 256-byte aligned.
 *   mode     W4_SYM or W4_ASYM, optionally OR-ed with W4_WEIGHTS_STATIC,
 *            W4_OUT_F32 and W4_REPACKED.
 * Paths: M <= 16 runs the GEMV (codes streamed to shared memory by TMA,
 * dequantized in registers, mma.sync); larger M runs the tcgen05 kernel
 * (dequantized weights in tensor memory, activations in shared memory, fp32
 * accumulation in tensor memory).
 */
w4_status w4a16_gemm(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                     const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                     void *workspace, size_t workspace_bytes, w4_stream_t stream);

/*
 * w4_awq_workspace_bytes -- device scratch that w4_awq_search needs for a
 * grid of n_alpha points (0 for malformed arguments).  It holds, among
 * others, the scale vector of every alpha (n_alpha * K fp32) and X divided by
 * each of them (n_alpha * M * K bf16).
 */
size_t w4_awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int mode, int n_alpha);

/*
 * w4_awq_search -- the AWQ smoothing-scale search (page 2, AWQ section, the
 * awq_search_scale listing: a grid search over alpha for the per-input-channel
 * scale s that minimises the error of the quantized layer on calibration data).
 *   W        bf16 [N][K] weight, 32-byte aligned.
 *   X        bf16 [M][K] calibration activations, 16-byte aligned; every input
 *            channel must have a nonzero mean magnitude.
 *   group, mode: as for w4_quant_pack.
 *   n_alpha  grid size, 2..4096: alpha_i = i / (n_alpha - 1) in fp64.
 *   losses   out, fp64 [n_alpha] device array (8-byte aligned).
 *   best     out, int device scalar: the first index of the smallest loss.
 *   s_best   out, fp32 [K] device array (16-byte aligned): s for that alpha,
 *            ready to pass to w4_quant_pack (and to divide X by upstream).
 *   workspace / workspace_bytes: w4_awq_workspace_bytes(M, N, K, group, mode,
 *            n_alpha) bytes, 256-byte aligned, contents need not be initialised.
 * For each alpha: act[k] = mean_m |x[m][k]| (fp64); s = act^alpha /
 * mean_k act^alpha in fp64, rounded once to fp32; Q = w4_quant_pack(W, s);
 * Y_q = w4a16_gemm(bf16(X / s), Q) (the product (W^ / s) X^T as the W4A16
 * path computes it); loss = mean over all M x N outputs of
 * (Y_ref - Y_q)^2 in fp64, with Y_ref = X W^T accumulated in fp32.
 * Asynchronous on `stream`; errors as for the other entry points.
 */
w4_status w4_awq_search(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                        int n_alpha, double *losses, int *best, float *s_best, void *workspace,
                        size_t workspace_bytes, w4_stream_t stream);

/*
 * w4a16_gemm_noalloc -- w4a16_gemm for callers that cannot allocate device
 * memory (a host whose allocator owns all device memory, a real-time host
 * that freezes its memory map after start-up, a plug-in that only receives its
 * input and output buffers).  The pages have no counterpart to this entry point: it only
 * changes where the split-K scratch lives.
 *   Arguments, results and errors are those of w4a16_gemm without the
 *   workspace.  The split-K scratch is a library-owned device array of
 *   W4_NOALLOC_SCRATCH_BYTES bytes that every GPU which loads the library
 *   holds until the process exits; shapes whose w4a16_workspace_bytes
 *   exceeds it are rejected with W4_ERR_UNSUPPORTED before anything is
 *   launched.  No device memory is allocated or freed.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture on the device.
 *   Each call first clears the array's split-K counters with
 *   cudaMemsetAsync on `stream`.  All calls share the array: calls ordered
 *   on one stream are safe, calls whose work overlaps on the GPU (unordered
 *   streams, several host threads) race and give wrong results.
 */
#define W4_NOALLOC_SCRATCH_BYTES (16u << 20)

w4_status w4a16_gemm_noalloc(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                             const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                             w4_stream_t stream);

/*
 * w4_fp4_quant -- block-scaled FP4 quantization of a bf16 weight matrix.
 *   (page 2, the Blackwell FP4 paragraph: E2M1 values, blocks of 16 sharing an
 *    FP8 E4M3 scale with amax mapped to 6; page 3 section 4.3: MXFP4, blocks of
 *    32 sharing an E8M0 scale, two FP4 values per byte; page 5 section 2.1:
 *    the E2M1 set {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6} and E4M3)
 *   Exact semantics, per block of B consecutive weights of a row:
 *     amax = max |w| over the block
 *     W4_NVFP4 (B = 16): scale code = e4m3_rne_satfinite(fl32(amax / 6));
 *                        s = its value (0 when it rounds to 0)
 *     W4_MXFP4 (B = 32): e = clamp(floor(log2 amax) - 2, -127, 127) (-127 for
 *                        an all-zero block); scale code = e + 127 (E8M0); s = 2^e
 *     code = e2m1_rne_satfinite(fl32(w / s)) for s > 0, else 0: the nearest
 *            E2M1 value, ties to the even fraction bit, magnitudes above 6
 *            giving 6; the sign bit is w / s's sign bit
 *     w^   = e2m1(code) * s (exact; the pages' snippet multiplies by 6.0 a
 *            second time, which would map amax to 36, and is not followed)
 *   W        bf16 [N][K], finite, 16-byte aligned (codes of a block holding
 *            an infinity or NaN are unspecified).
 *   N, K     N >= 1, K >= B, K % B == 0.
 *   kind     W4_NVFP4 or W4_MXFP4.
 *   codes    out, uint8 [N][K/2], 16-byte aligned: element 2i of a row in the
 *            low nibble of byte i, element 2i+1 in the high nibble.
 *   scales   out, uint8 [N][K/B]: E4M3 codes (NVFP4) or E8M0 codes (MXFP4).
 * Every output byte is written; outputs must not overlap inputs.
 * Errors: W4_ERR_INVALID_ARG for a NULL or misaligned pointer, an unknown
 * kind, N < 1, or K not a positive multiple of B; W4_ERR_CUDA if the launch
 * fails.  Asynchronous on `stream`.
 */
w4_status w4_fp4_quant(const void *W, int64_t N, int64_t K, int kind, uint8_t *codes, uint8_t *scales,
                       w4_stream_t stream);

/*
 * w4_repacked_words -- 32-bit words of the repacked layout of an [N][K/8]
 * packed weight: ceil(N/16) * 16 * K/8 (0 unless K % 256 == 0).
 */
size_t w4_repacked_words(int64_t N, int64_t K);

/*
 * w4_repack -- the offline repack of a packed weight into the GEMV's box
 * order (a layout-specialised copy in the spirit of page 3 section 3.1's
 * Marlin, which reorders INT4 weights offline into the tiles its kernel
 * reads; the codes themselves are unchanged).  Word kw of channel n goes to
 *   (((n/16) * (K/256) + kw/32) * 16 + n % 16) * 32 + kw % 32,
 * so that each 16-channel x 256-k box the GEMV loads is 2 KB of contiguous
 * memory; the channels that pad N to a multiple of 16 are written as 0.
 *   qweight  uint32 [N][K/8] (w4_quant_pack layout), 16-byte aligned.
 *   N, K     N >= 1, K >= 256; K % 256 != 0 gives W4_ERR_UNSUPPORTED.
 *   out      out, w4_repacked_words(N, K) words, 16-byte aligned; scales and
 *            zero-points keep their layout.
 * Errors as for w4_quant_pack.  Asynchronous on `stream`.
 */
w4_status w4_repack(const uint32_t *qweight, int64_t N, int64_t K, uint32_t *out, w4_stream_t stream);

/*
 * w4_gptq_workspace_bytes -- device scratch that w4_gptq needs (0 for
 * malformed arguments): about 16 K^2 + 8 N K bytes (the Hessian, its
 * factor's inverse and an fp64 copy of W).
 */
size_t w4_gptq_workspace_bytes(int64_t N, int64_t K, int group);

/*
 * w4_gptq -- GPTQ: INT4 codes chosen column by column with Hessian-weighted
 * error feedback, in the packed layout of w4_quant_pack (page 5 section 2.5,
 * the column update with the upper Cholesky factor of the inverse Hessian;
 * page 3 section 3.1, the Hessian and its damping; page 2, GPTQ section).
 * Exact semantics (fp64 unless stated), for calibration rows X [M][K]:
 *   H      = 2 X^T X + lambda I,  lambda = 0.01 trace(X^T X) / K
 *   U      = upper triangular with H^-1 = U^T U  (U = I if trace(X^T X) = 0)
 *   for j = 0 .. K-1, on every row independently:
 *     if j % group == 0: the group's s16 and zp from fl32 of the group's
 *        current values, by w4_quant_pack's rules (no smoothing vector)
 *     u_j  = w4_quant_pack's code of fl32(w_j) on that grid
 *     e    = (w_j - (u_j - zp) s16) / U[j][j];   w_k -= e U[j][k] for k > j
 *   The result equals that definition up to the rounding order of fp64 sums
 *   (the later columns are updated 32 columns at a time); a code can differ
 *   only where a value lies within that rounding of a decision boundary.
 *   W        bf16 [N][K];  X bf16 [M][K] calibration activations.
 *   N, K, M  N >= 1, M >= 1, K >= 32, K % group == 0, K <= 16384.
 *   group, mode, qweight, scales, qzeros: as for w4_quant_pack.
 *   workspace, workspace_bytes: w4_gptq_workspace_bytes(N, K, group) bytes,
 *            256-byte aligned; contents need not be initialised.
 * About 3 K / 32 + 2 K / group kernel launches.  Errors as for w4_quant_pack;
 * W4_ERR_UNSUPPORTED for K > 16384.  Asynchronous on `stream`.
 */
w4_status w4_gptq(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                  uint32_t *qweight, void *scales, uint32_t *qzeros, void *workspace, size_t workspace_bytes,
                  w4_stream_t stream);

/*
 * w4_f32_to_bf16 -- dst[i] = bf16_rne(src[i]) for i < n: the one rounding of a
 * product whose fp32 partial sums were added across devices.
 *   src  fp32 [n], 4-byte aligned;  dst  out, bf16 [n], 2-byte aligned.
 * Errors: W4_ERR_INVALID_ARG for NULL, misaligned or n < 1; W4_ERR_CUDA if the
 * launch fails.  Asynchronous on `stream`.
 */
w4_status w4_f32_to_bf16(const float *src, int64_t n, void *dst, w4_stream_t stream);

/*
 * MX scale layouts (for the E8M0 scales of w4_mxfp8_quant, w4_mx_scale_layout
 * and w4_mx_gemm; R rows, K columns, one scale per 32-element block kb):
 *   W4_MX_SCALES_ROWS  uint8 [R][K/32], byte r * (K/32) + kb.
 *   W4_MX_SCALES_MMA   the tensor-core layout: ceil(R/128) bands of 128 rows,
 *                      each band K/128 atoms of 512 bytes in k order; the
 *                      scale of (r, kb) is the byte at
 *                        ((r/128) * (K/128) + kb/4) * 512
 *                          + (r % 32) * 16 + ((r % 128) / 32) * 4 + kb % 4.
 *                      Size ceil(R/128) * 128 * (K/32) bytes; the bytes of
 *                      rows R.. of the last band are written as 0.
 */
#define W4_MX_SCALES_ROWS 0
#define W4_MX_SCALES_MMA 1

/*
 * w4_mxfp8_quant -- MXFP8 quantization of bf16 activations.
 *   (page 3 section 4.3: activations kept at FP8 beside FP4 weights, one
 *    E8M0 scale per block of 32 elements; page 5 section 2.1 and page 3
 *    section 4.1: the E4M3 format)
 *   Exact semantics, per block of 32 consecutive elements of a row:
 *     amax = max |x| over the block
 *     e    = clamp(floor(log2 amax) - 8, -127, 127) (-127 for an all-zero
 *            block); scale code = e + 127 (E8M0); s = 2^e
 *     code = e4m3_rne_satfinite(fl32(x / s)): round to nearest even, finite
 *            magnitudes above 448 giving 448 (a block's largest elements clip
 *            when amax lies in [1.75, 2) * 2^(e+8)); the sign follows x / s
 *     x^   = e4m3(code) * s (exact)
 *   X        bf16 [M][K], finite, 16-byte aligned.
 *   M, K     M >= 1, K >= 32, K % 32 == 0; K % 128 == 0 for W4_MX_SCALES_MMA.
 *   codes    out, uint8 [M][K] E4M3 codes, 16-byte aligned.
 *   scales   out, E8M0 codes in `scale_layout` (W4_MX_SCALES_ROWS: [M][K/32];
 *            W4_MX_SCALES_MMA: see above, 16-byte aligned).
 * Every output byte is written; outputs must not overlap inputs.
 * Errors: W4_ERR_INVALID_ARG for a NULL or misaligned pointer, a bad size or
 * layout; W4_ERR_CUDA if the launch fails.  Asynchronous on `stream`.
 */
w4_status w4_mxfp8_quant(const void *X, int64_t M, int64_t K, uint8_t *codes, uint8_t *scales, int scale_layout,
                         w4_stream_t stream);

/*
 * w4_mx_scale_layout -- copy E8M0 scales from W4_MX_SCALES_ROWS to
 * W4_MX_SCALES_MMA (a permutation of bytes, plus the zero rows that pad the
 * last band).  Used once per weight: w4_fp4_quant(W4_MXFP4) writes rows.
 *   src      uint8 [R][K/32], 4-byte aligned.
 *   R, K     R >= 1, K >= 128, K % 128 == 0.
 *   dst      out, ceil(R/128) * 128 * (K/32) bytes, 16-byte aligned.
 * Errors as for w4_mxfp8_quant.
 */
w4_status w4_mx_scale_layout(const uint8_t *src, int64_t R, int64_t K, uint8_t *dst, w4_stream_t stream);

/*
 * w4_mx_gemm -- Y = X^ . W^^T for MXFP8 activations and MXFP4 weights on the
 * block-scaled tensor cores (page 3 section 4.3: FP4 weights times FP8
 * activations, E8M0 scales per 32; page 2, the Blackwell FP4 paragraph: the
 * block-scaled format feeds the tensor cores directly).
 *   Y[m][n] = bf16_rne(sum_k x^[m][k] * w^[n][k]) with x^ from
 *   w4_mxfp8_quant, w^ from w4_fp4_quant(W4_MXFP4) (w^ = e2m1(code) * 2^e),
 *   accumulated by the tensor cores in fp32; a split of k across CTAs adds
 *   its fp32 partial sums in a fixed order, so results repeat bit for bit.
 *   x_codes  uint8 [M][K] E4M3 codes, 16-byte aligned.
 *   x_scales E8M0, W4_MX_SCALES_MMA layout for M rows, 16-byte aligned.
 *   M, N, K  M >= 1, N >= 1, K >= 128, K % 128 == 0.
 *   w_codes  uint8 [N][K/2] MXFP4 codes (w4_fp4_quant layout), 32-byte aligned.
 *   w_scales E8M0, W4_MX_SCALES_MMA layout for N rows, 16-byte aligned.
 *   Y        out, bf16 [M][N], 2-byte aligned.
 *   flags    0 or W4_WEIGHTS_STATIC (as for w4a16_gemm: the weight codes and
 *            scales are not written by the kernel right before this call on
 *            `stream`, so their stream may start before it finishes).
 * Needs no workspace.  Errors: W4_ERR_INVALID_ARG for a NULL or misaligned
 * pointer, a bad size or flag; W4_ERR_UNSUPPORTED for shapes past 32-bit
 * indexing; W4_ERR_CUDA if the launch fails.  Asynchronous on `stream`.
 */
w4_status w4_mx_gemm(const uint8_t *x_codes, const uint8_t *x_scales, int64_t M, int64_t N, int64_t K,
                     const uint8_t *w_codes, const uint8_t *w_scales, void *Y, int flags, w4_stream_t stream);

/* Text for a status code; never NULL. */
const char *w4_status_string(int status);

/* W4_LAYOUT_VERSION of the library that was loaded. */
int w4_layout_version(void);

/*
 * w4_set_wait_limit_ns -- the time after which a kernel's wait for a copy, an
 * MMA or another warp gives up, records a code (see w4_device_error) and ends
 * the kernel early; 0 restores the default of 200 ms, far above any
 * legitimate wait.  This exists to test the failure path: a test lowers the
 * limit so that a wait runs out, checks the recorded code and that the next
 * call is correct.  Waits that let a kernel's own copies and MMAs finish
 * before it exits always keep the default.  Process-wide; read at each launch.
 */
void w4_set_wait_limit_ns(uint64_t ns);

/*
 * w4_test_stall_first_wait -- for tests of the failure path only: while `on`
 * is nonzero, each warp's first wait for a copy (in w4_quant_pack,
 * w4a16_gemm and w4_mx_gemm) targets a barrier that nothing completes, so that it runs out
 * after the limit set by w4_set_wait_limit_ns and the kernel takes its failure
 * path; the copies it issued still land (they are drained with the default
 * limit).  0 (the default) turns it off.  Process-wide; read at each launch.
 */
void w4_test_stall_first_wait(int on);

/*
 * w4_device_error -- read and clear the library's device-side error word.
 * Kernels that wait on barriers give every wait an iteration limit; a wait
 * that runs out records a nonzero code here and the kernel returns early
 * instead of hanging.  This call synchronizes the device.  *code receives 0
 * when no wait has run out since the last call.
 */
w4_status w4_device_error(int *code);

#ifdef __cplusplus
}
#endif

#endif /* W4_H */
