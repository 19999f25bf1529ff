/*
 * mx.h -- C ABI of the B200 (sm_100a) microscaling library: MX / NVFP4 quantisation,
 * dequantisation and the MX block-scaled matmul.
 *
 * Sources (page title, section):
 *   [Q]  "MXFP4 と NVFP4 は何が違うのか調べてみた"
 *        §1 "E2M1 という共通土台": E2M1 values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and mirrors; max 6.
 *        §2 "MXFP4 はブロック32と E8M0": blocks of 32 share one E8M0 scale (bias 127,
 *           0xFF = NaN, no Inf); MXFP8 = E4M3 or E5M2 elements; RNE cast; the scale
 *           rounding is left to the implementation.
 *        §3 "NVFP4 はブロック16と E4M3、そして二段目": blocks of 16, unsigned E4M3 block
 *           scale (max 448), FP32 per-tensor scale = tensor amax / (6 * 448).
 *        §4 "同じ E2M1 でも、別仕様である" / "精度の差はどこから出るか": the OCP floor
 *           rule (scaled block max in [4, 8), clipped at 6) and the no-clip rule
 *           (scaled block max in (3, 6]).
 *        §6 "DeepSeek-V4 の入れ子構造": training needs the weight in both orientations.
 *        §7 "ハードウェアの対応状況": Blackwell's 5th-generation tensor cores consume
 *           MXFP8/MXFP4 natively; MX scale application is an exponent add.
 *   [P4] gpt-oss MXFP4 explainer, section "MXFP4": the direct cast vs the scaled cast.
 *
 * Conventions for every entry point:
 *   - Ownership: the caller allocates and owns every buffer.  Device pointers must be
 *     device (or managed) memory of the current CUDA device.  The library keeps, per
 *     device, only a small scratch array for NVFP4 partial maxima (allocated on the
 *     first NVFP4 call on that device) and a static watchdog flag.
 *   - NVFP4 calls on one device (mx_quantize with MX_FMT_NVFP4, mx_quantize_train with
 *     MX_FMT_NVFP4, mx_quantize_nvfp4_2d, mx_quantize_mx_nvfp4) share that scratch array:
 *     calls whose GPU work overlaps -- on two streams with no ordering between them -- race on it and may
 *     produce a wrong per-tensor scale.  Issue them on one stream, or order the streams
 *     with events.  The MX formats use no scratch and may overlap freely.
 *   - Execution: every call only validates its arguments on the host and enqueues
 *     kernels on `stream` (0 = the legacy default stream); it returns before the GPU
 *     work finishes.  Nothing is written to any output before the work runs.
 *   - Errors: arguments are validated before any launch.  A non-MX_OK status means no
 *     kernel was launched, except MX_ERR_CUDA, which reports a failed launch (the CUDA
 *     error code is kept per host thread, see mx_last_cuda_error).  Empty inputs
 *     (rows == 0 or cols == 0) are valid and launch nothing.
 *   - bf16 is IEEE binary16-brain (1/8/7), stored as 2-byte little-endian words.
 *   - Element codes are packed densely along each row: code i occupies bits
 *     [w*i, w*i + w) of the row read as a little-endian bit string, w the code width.
 *     FP8 / INT8: one byte per code; FP6: four codes per three bytes (16 per 12 bytes);
 *     FP4: two per byte, the even element index in the low nibble.
 *   - Overflow saturates to the format maximum (448 E4M3, 57344 E5M2, 6 E2M1); a
 *     block holding a NaN or Inf gets the NaN scale (0xFF E8M0, 0x7F UE4M3) and
 *     element codes 0.
 */
#ifndef MX_H_
#define MX_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle; the same type as cudaStream_t. */
struct CUstream_st;
typedef struct CUstream_st *mx_stream_t;

typedef enum {
    MX_OK = 0,
    MX_ERR_ARG = 1,      /* null pointer, unknown enum, unsupported combination */
    MX_ERR_SHAPE = 2,    /* negative size, or a size that is not a multiple of the block/tile */
    MX_ERR_ALIGN = 3,    /* a pointer that is not aligned as the call requires */
    MX_ERR_LAYOUT = 4,   /* scale-layout mask empty, unknown, or missing its second buffer */
    MX_ERR_CUDA = 5,     /* a CUDA launch or driver call failed; see mx_last_cuda_error */
    MX_ERR_TIMEOUT = 6   /* a bounded device wait gave up (watchdog); see mx_watchdog_status */
} mx_status;

typedef enum {
    MX_FMT_E4M3 = 0,     /* MXFP8, E4M3 elements, block 32, E8M0 scale */
    MX_FMT_E5M2 = 1,     /* MXFP8, E5M2 elements, block 32, E8M0 scale */
    MX_FMT_E2M1 = 2,     /* MXFP4, E2M1 elements, block 32, E8M0 scale */
    MX_FMT_NVFP4 = 3,    /* NVFP4, E2M1 elements, block 16, UE4M3 scale, fp32 tensor scale */
    MX_FMT_E2M3 = 4,     /* MXFP6, E2M3 elements (max 7.5), block 32, E8M0 scale */
    MX_FMT_E3M2 = 5,     /* MXFP6, E3M2 elements (max 28), block 32, E8M0 scale */
    MX_FMT_INT8 = 6      /* MXINT8, int8 q read as q / 64 (-127 .. 127), block 32, E8M0 scale */
} mx_fmt;
/* Storage (w bits per code, packed densely along a row): FP8 and INT8 w = 8; FP6 w = 6,
 * so MXFP6 costs 6 + 8/32 = 6.25 bits per element; FP4 w = 4, even element low. */

typedef enum {
    MX_AXIS_ROW = 0,     /* blocks run along a row (contiguous elements) */
    MX_AXIS_COL = 1      /* blocks run down a column; output is the transposed matrix */
} mx_axis;

typedef enum {
    MX_SCALE_FLOOR_OCP = 0,    /* s = floor(log2 amax) - emax_elem ([Q] §4, OCP example) */
    MX_SCALE_CEIL_RECIPE = 1   /* smallest s with amax <= max_elem * 2^s (no clipping, [Q] §4) */
} mx_scale_rounding;

typedef enum {
    MX_LAYOUT_ROWMAJOR = 1,    /* scales[r * S + c], S = blocks per output row */
    MX_LAYOUT_TCGEN05 = 2      /* tcgen05 tiling: 128-row x 4-column atoms of 512 bytes */
} mx_scale_layout;             /* used as a bit mask where a call accepts both */

/*
 * Byte size of a scale buffer for an output of `rows` rows and `scale_cols` scales per
 * row in `layout` (exactly one bit).  ROWMAJOR: rows * scale_cols.  TCGEN05:
 * ceil(rows/128) * ceil(scale_cols/4) * 512; inside an atom, scale (r, c) sits at byte
 * (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4), atoms ordered row-block-major; pad bytes
 * are written as 0 by the quantisers.  Returns -1 for invalid arguments.  Host only.
 */
int64_t mx_scale_bytes(int64_t rows, int64_t scale_cols, mx_scale_layout layout);

/*
 * mx_quantize -- quantise a bf16 matrix to MXFP8 / MXFP6 / MXFP4 / MXINT8 / NVFP4
 * ([Q] §2 and its MX family table, §3, §4).
 *   src_bf16    device, rows x cols bf16 row-major, 16-byte aligned.
 *   fmt         MX_FMT_E4M3 / E5M2 / E2M3 / E3M2 / E2M1 / INT8 (block 32, E8M0) or
 *               MX_FMT_NVFP4 (block 16).
 *   axis        ROW: blocks along rows; output rows x cols, scales rows x cols/B.
 *               COL: blocks down columns; output is the transposed matrix cols x rows
 *               (K-major for a weight-gradient matmul), scales cols x rows/B.
 *               NVFP4 supports ROW only.
 *   rounding    shared-exponent rule (ignored for NVFP4).
 *   out_elems   device, 16-byte aligned; out_rows x (out_cols * w / 8) bytes: w = 8
 *               (FP8, INT8), 6 (FP6), 4 (FP4).
 *   out_scales  device; first scale layout (the lower set bit of `layout`).
 *   layout      ROWMAJOR, TCGEN05 or both; with both, out_scales gets ROWMAJOR and
 *               out_scales_alt gets TCGEN05 (else out_scales_alt must be NULL).
 *   global_scale  NVFP4 only (else NULL): device fp32, written with g = amax / 2688,
 *               the per-tensor decode scale (1.0 when the tensor is all zero).
 *   Shape rule: the blocked dimension (cols for ROW, rows for COL) is a multiple of the
 *   block (32, or 16 for NVFP4), else MX_ERR_SHAPE.
 */
mx_status mx_quantize(const void *src_bf16, int64_t rows, int64_t cols, mx_fmt fmt, mx_axis axis,
                      mx_scale_rounding rounding, void *out_elems, uint8_t *out_scales,
                      mx_scale_layout layout, uint8_t *out_scales_alt, float *global_scale,
                      mx_stream_t stream);

/*
 * mx_quantize_nvfp4_noalloc -- NVFP4 quantisation that never allocates device memory.
 * The pages have no counterpart to this call; it exists for callers of this library.
 *
 * mx_quantize(fmt = MX_FMT_NVFP4) needs a small scratch buffer (one partial maximum
 * per CTA of its tensor-maximum pass), which the library allocates with cudaMalloc on the first
 * NVFP4 call on each device.  Callers that cannot allow a cudaMalloc -- a serving loop
 * that reserves all device memory at start-up and must not take the implicit device
 * synchronisation or the out-of-memory risk of an allocation on its request path, or a
 * host framework that owns all device memory through its own allocator -- call this
 * variant instead.  It runs the same kernels and produces bit-identical outputs, with the
 * scratch in a fixed static device array of MX_NOALLOC_MAX_PARTIALS fp32 values (4 KiB)
 * that every GPU loading the library holds until the process exits.
 *
 * Arguments are those of mx_quantize with fmt = MX_FMT_NVFP4 and axis = ROW (cols a
 * multiple of 16, global_scale required, same layouts, alignment and ownership).
 * The caller still allocates every input and output.
 *   - The first call on each device performs a one-time set-up on that device (it
 *     queries the SM count and looks up the static array's device address with
 *     cudaGetSymbolAddress; neither allocates).  Make that first call before any stream
 *     capture on that device.
 *   - Limit: the call needs one scratch slot per CTA of its maximum pass, that is
 *     min(ceil(rows * cols / 8192), 3 x the SM count) slots.  A call that would need more
 *     than MX_NOALLOC_MAX_PARTIALS returns MX_ERR_SHAPE without launching (on a 148-SM
 *     B200 the count never exceeds 444).
 *   - Every call shares the one array, which keeps the previous call's contents.  Each
 *     call writes every partial-maximum slot it later reads, so nothing carries over.
 *     Calls whose GPU work overlaps (for example on two streams without ordering between
 *     them) race on the array and may produce wrong results.  Order such calls on one
 *     stream.
 */
#define MX_NOALLOC_MAX_PARTIALS 1024
mx_status mx_quantize_nvfp4_noalloc(const void *src_bf16, int64_t rows, int64_t cols, void *out_elems,
                                    uint8_t *out_scales, mx_scale_layout layout, uint8_t *out_scales_alt,
                                    float *global_scale, mx_stream_t stream);

/*
 * mx_quantize_train -- the training-side row-wise quantiser ([Q] §4: the 4-bit pre-training
 * recipe applies a 16 x 16 random Hadamard transform to the inputs of the weight gradient
 * and rounds gradients stochastically; [Q] §8: stochastic rounding is a P3109 mode).
 * Same outputs as mx_quantize(axis = ROW) for fmt E4M3, E5M2, E2M1 or NVFP4, with:
 *   rht16       1: every 16 consecutive elements of a row are first replaced by
 *               H16 D x / 4 (D = diag of signs: bit i of rht_signs set negates element i;
 *               H16 the Sylvester Hadamard matrix), computed by radix-2 butterflies
 *               (strides 1, 2, 4, 8) in fp32 round-to-nearest and rounded to bf16; the
 *               quantiser (scales, NVFP4 tensor scale included) sees those values.  0: none.
 *               Applying the same transform to both operands along K leaves A * B^T
 *               unchanged (H16 D / 4 is orthogonal).
 *   sr_random   NULL: round to nearest even.  Else device, rows x cols random bytes (one per
 *               element, 16-byte aligned): a scaled value strictly between its representable
 *               neighbours lo < |y| < hi becomes hi when 256 (|y| - lo) > r (hi - lo), else
 *               lo (probability of rounding up ceil(256 f) / 256, f the position between
 *               them); values at or beyond the maximum saturate.  Scales are unchanged.
 * Other arguments, shapes, layouts and errors as mx_quantize(axis = ROW).
 */
mx_status mx_quantize_train(const void *src_bf16, int64_t rows, int64_t cols, mx_fmt fmt,
                            mx_scale_rounding rounding, int rht16, unsigned rht_signs,
                            const uint8_t *sr_random, void *out_elems, uint8_t *out_scales,
                            mx_scale_layout layout, uint8_t *out_scales_alt, float *global_scale,
                            mx_stream_t stream);

/*
 * mx_quantize_nvfp4_2d -- NVFP4 with two-dimensional 16 x 16 blocks, for weights ([Q] §4:
 * the 4-bit pre-training recipe scales weights in two-dimensional blocks, so that a weight
 * and its transpose quantise identically).  Same steps as mx_quantize(fmt = NVFP4) with the
 * block maximum taken over 16 rows x 16 columns; each block's UE4M3 scale is written to all
 * 16 of its rows in the usual 1 x 16 layouts (rows x cols/16), so mx_dequantize and mx_gemm
 * consume the result unchanged.  Arguments as mx_quantize with fmt = NVFP4, axis = ROW;
 * rows and cols are multiples of 16 (else MX_ERR_SHAPE).
 */
mx_status mx_quantize_nvfp4_2d(const void *src_bf16, int64_t rows, int64_t cols, void *out_elems,
                               uint8_t *out_scales, mx_scale_layout layout, uint8_t *out_scales_alt,
                               float *global_scale, mx_stream_t stream);

/*
 * mx_quantize_mx_nvfp4 -- row-wise MX quantisation (any MX format) and NVFP4 quantisation
 * of the same bf16 tensor in one call, the two encodings of one weight that [Q] §4
 * ("同じ E2M1 でも、別仕様である") compares.  The input is read from memory once for both
 * maxima: the MX pass also reduces the tensor's finite |x| maximum, so the NVFP4 pass runs
 * without a maximum pass of its own (it re-reads the input, from L2 when it fits there).
 * Results are bit-identical to mx_quantize(fmt, ROW, rounding, mx_*) followed by
 * mx_quantize(NVFP4, ROW, nv_*).
 *   fmt, rounding, mx_elems, mx_scales, mx_layout, mx_scales_alt
 *                 the MX output, as mx_quantize(axis = ROW); cols % 32 == 0.
 *   nv_elems, nv_scales, nv_layout, nv_scales_alt, global_scale
 *                 the NVFP4 output, as mx_quantize(fmt = NVFP4).
 * Uses the NVFP4 partial-maxima scratch (the ordering rule above applies).
 */
mx_status mx_quantize_mx_nvfp4(const void *src_bf16, int64_t rows, int64_t cols, mx_fmt fmt,
                               mx_scale_rounding rounding, void *mx_elems, uint8_t *mx_scales,
                               mx_scale_layout mx_layout, uint8_t *mx_scales_alt, void *nv_elems,
                               uint8_t *nv_scales, mx_scale_layout nv_layout, uint8_t *nv_scales_alt,
                               float *global_scale, mx_stream_t stream);

/*
 * mx_quantize_dual -- one pass over a bf16 matrix producing both orientations ([Q] §6:
 * training needs the row-wise copy for the forward matmul and the column-wise copy for
 * the weight-gradient matmul).  The input is read once.
 *   row_elems / row_scales   as mx_quantize(axis = ROW).
 *   col_elems / col_scales   as mx_quantize(axis = COL): cols x rows, scales cols x rows/32.
 *   layout      ROWMAJOR, TCGEN05 or both (bitwise or), used for both orientations.  With
 *               one layout, row_scales / col_scales are in it and the two *_alt pointers
 *               must be NULL; with both, row_scales / col_scales are ROWMAJOR and
 *               row_scales_alt / col_scales_alt (device, non-NULL) TCGEN05 -- all four
 *               are written by the same single pass.
 *   fmt         any MX format (E4M3, E5M2, E2M3, E3M2, E2M1, INT8).  rows and cols are
 *               multiples of 32.
 */
mx_status mx_quantize_dual(const void *src_bf16, int64_t rows, int64_t cols, mx_fmt fmt,
                           mx_scale_rounding rounding, void *row_elems, uint8_t *row_scales,
                           void *col_elems, uint8_t *col_scales, mx_scale_layout layout,
                           uint8_t *row_scales_alt, uint8_t *col_scales_alt, mx_stream_t stream);

/*
 * mx_dequantize -- codes and scales back to bf16 ([Q] §7: MX is an exponent add,
 * x = dec(q) * 2^(s - 127), exact before the bf16 rounding; NVFP4 is
 * (dec(q) * dec(sb)) * g in fp32).  A NaN scale makes the whole block NaN ([Q] §2).
 *   elems, scales  device, as produced by mx_quantize(axis = ROW) for a rows x cols tensor.
 *   global_scale   NVFP4 only: device fp32 g (else NULL).
 *   layout         exactly one of ROWMAJOR / TCGEN05 (the layout of `scales`).
 *   out_bf16       device, rows x cols bf16, 16-byte aligned; round to nearest even.
 */
mx_status mx_dequantize(const void *elems, const uint8_t *scales, const float *global_scale,
                        int64_t rows, int64_t cols, mx_fmt fmt, mx_scale_layout layout,
                        void *out_bf16, mx_stream_t stream);

/*
 * mx_cast -- the direct cast of [P4] "MXFP4": each bf16 value cast to the element format
 * with no block scale (RNE, saturating).  NaN becomes 0x7F|sign (E4M3, E5M2) or the
 * signed maximum 0x7|sign (E2M1) / 0x1F|sign (E2M3, E3M2), formats without NaN.  INT8
 * needs a scale and is not a cast target (MX_ERR_ARG).
 *   n           element count (even for E2M1, a multiple of 4 for FP6: whole bytes of
 *               packed codes); src and out 16-byte aligned.
 */
mx_status mx_cast(const void *src_bf16, int64_t n, mx_fmt fmt, void *out_elems, mx_stream_t stream);

/*
 * One operand of the block-scaled matmul: a rows x K matrix of codes, K-major (each row
 * holds K consecutive codes, packed as the quantisers write them), with its block scales in the TCGEN05
 * layout exactly as mx_quantize(axis = ROW, layout = TCGEN05) writes them: E8M0 per 32
 * along K (rows x K/32) for the MX formats, UE4M3 per 16 along K (rows x K/16) for NVFP4.
 *   global_scale  NVFP4 only: device pointer to the operand's fp32 per-tensor scale g (as
 *                 written by mx_quantize); NULL for MX operands.
 */
typedef struct {
    const void *elems;
    const uint8_t *scales;
    mx_fmt fmt;
    const float *global_scale;
} mx_operand;

/*
 * mx_gemm -- C = A * B^T with block scaling ([Q] §7; mixed MXFP4 x MXFP8 per [Q] §2 and
 * §6; FP4 x FP4 per [Q] §7's FP4 tensor-core rate and §3's NVFP4 two-level scale):
 *   MX:    C[m, n] = sum_k dec(A[m,k]) 2^(sA[m,k/32]-127) dec(B[n,k]) 2^(sB[n,k/32]-127)
 *   NVFP4: C[m, n] = gA gB sum_k dec(A[m,k]) dec(sA[m,k/16]) dec(B[n,k]) dec(sB[n,k/16])
 * accumulated in fp32 on the tensor cores (the NVFP4 product gA gB is applied to the fp32
 * sum), written as bf16 (RNE).
 *   Format pairs (A, B): A in {E4M3, E5M2, E2M3, E3M2} with B in {E4M3, E5M2, E2M3, E3M2,
 *   E2M1} (FP8 / FP6 run at the FP8 rate, [Q] §7) -- e.g. activations x MXFP4 weights --
 *   and (E2M1, E2M1), (NVFP4, NVFP4) at the FP4 rate; any other pair (INT8 has no
 *   block-scaled tensor-core form), or a global_scale that is missing for NVFP4 or
 *   present for MX, is MX_ERR_ARG.
 *   C_bf16      device, M x N row-major bf16, 16-byte aligned.
 *   Shapes: M and N multiples of 128; K a multiple of 128 (8-bit A) or 256 (FP4 x FP4)
 *   (else MX_ERR_SHAPE).
 *   Alignment: elems 32-byte aligned, scales 16-byte aligned, global scales 4-byte aligned
 *   (else MX_ERR_ALIGN).
 */
mx_status mx_gemm(mx_operand A, mx_operand B, void *C_bf16, int64_t M, int64_t N, int64_t K,
                  mx_stream_t stream);

/*
 * mx_mxfp4_to_fp8_blocks -- the nested blocks of [Q] §6 ("DeepSeek-V4 の入れ子構造"): an
 * MXFP4 weight (1 x 32 tiles, E8M0 scales) re-expressed as FP8 E4M3 with one scale per
 * 128 x 128 block, the block scaling FP8 training keeps; a block holds 4 x 128 = 512 tiles.
 * Per block: s_max = the largest tile exponent (scale code - 127) among tiles that are not
 * NaN and hold a nonzero code; block scale S = 2^(s_max - 6) (the largest FP4 value
 * 6 * 2^s_max becomes 384; 1.0 for a block without such a tile); every element becomes
 * the RNE-saturating E4M3 code of dec(q) * 2^(s_tile - 127) / S; a NaN tile gives 0x7F
 * codes.  block_exact = 1 when every element of the block decodes back to its FP4 value
 * (the lossless condition of the pages; it always holds when no nonzero tile is more than
 * 14 binades below s_max), else 0.
 *   elems         device, rows x cols/2 packed E2M1 (even element in the low nibble),
 *                 16-byte aligned, as mx_quantize(E2M1, ROW) writes it.
 *   scales        device, rows x cols/32 E8M0, ROWMAJOR layout.
 *   rows, cols    multiples of 128 (else MX_ERR_SHAPE).
 *   out_fp8       device, rows x cols E4M3 codes, 16-byte aligned.
 *   block_scales  device, (rows/128) x (cols/128) fp32 (powers of two), 4-byte aligned.
 *   block_exact   device, (rows/128) x (cols/128) bytes.
 */
mx_status mx_mxfp4_to_fp8_blocks(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                                 void *out_fp8, float *block_scales, uint8_t *block_exact, mx_stream_t stream);

/* Human-readable name of a status code (static string). */
const char *mx_status_string(mx_status status);

/* The CUDA error code (cudaError_t value) behind the last MX_ERR_CUDA on this host thread. */
int mx_last_cuda_error(void);

/*
 * Watchdog: the pipelined kernels bound every wait on a barrier; a wait that gives up
 * records a nonzero code in a device flag and the kernel returns early.  This call
 * synchronises the current device, reads the flag (0 = no timeout) into *code and, if
 * `clear`, resets it.  Returns MX_ERR_TIMEOUT if the flag was set, MX_OK otherwise.
 * While the flag is set, pipelined kernels give up their waits at once (so one stuck
 * CTA cannot stall a whole grid); outputs of calls made while it is set are undefined.
 * Clear it to resume normal operation.
 */
mx_status mx_watchdog_status(int *code, int clear);

/*
 * Watchdog self-test (a diagnostic, not part of the pages' method): enqueues on `stream`
 * one kernel whose single wait -- the same bounded barrier wait the pipelined kernels use
 * -- is on a barrier that nothing ever arrives at.  After `limit_us` microseconds of
 * device time (1 .. 100000, else MX_ERR_ARG) the wait gives up, records code 9 in the
 * watchdog flag and the kernel returns normally: no fault, no trap, the context stays
 * usable.  mx_watchdog_status then reports MX_ERR_TIMEOUT with *code == 9; clear the flag
 * before further calls (see above).  Allocates nothing.
 */
mx_status mx_watchdog_selftest(uint32_t limit_us, mx_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MX_H_ */
