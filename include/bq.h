/*
 * bq.h -- C ABI of the B200 (sm_100a) group-wise MinMax weight quantizer and
 * weight-only linear layer.
 *
 * The method (GreenBitAI article "只需单卡 RTX 3090，低比特量化训练就能实现
 * LLaMA-3 8B 全参微调", paragraph on the quantizer): classic Group-wise MinMax
 * quantization, used only as INT4 with group size 128 and INT2 with group
 * size 64, mixed per layer (Layer-mix) or per output-channel block
 * (Channel-mix).  Per group of `group` consecutive weights of one row
 * ("大模型量化实战：从原理到4-bit部署的完整指南", section 2.2; "低比特量化 /
 * Low-bit Quantization", sections "Group Quantization" and "Zero Point"):
 *
 *     lo = min(min x, 0)     hi = max(max x, 0)          (range widened to 0)
 *     s  = (hi - lo) / (2^b - 1)                          fp32, round to nearest even
 *     z  = round(-lo / s)                                 half to even, 0 <= z <= 2^b-1
 *     q  = clamp(round(x / s) + z, 0, 2^b - 1)            x/s one fp32 division
 *     dequant(q) = (q - z) * s
 *     an all-zero group stores s = 0, z = 0, q = 0
 *
 * and the weight-only linear layer y = x . dequant(W)^T (survey "A Survey of
 * Low-bit Large Language Models", section 6.2 weight-only: dequantize, then a
 * 16-bit matmul; "大模型量化实战" section 3.3: dequantize and multiply in one
 * fused kernel).  No dequantized weight is ever written by the linear layer.
 * Its input gradient dx = dy . dequant(W) (bq_linear_grad_input) reads the
 * same packed weights in place.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - W is [rows, cols] row-major: rows = N = output channels, cols = K = input
 *    channels.  Groups run along cols inside one row.
 *  - Every buffer pointer is a DEVICE pointer unless the argument says "host".
 *    The caller owns and allocates every buffer; the library never allocates
 *    or frees memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued asynchronously; argument errors are returned
 *    synchronously before anything is enqueued.
 *  - Pointers to W, x, y, packed codes and dequantized output must be 16-byte
 *    aligned; scales and zeros 4-byte and 1-byte aligned, except for
 *    bq_linear and bq_linear_grad_input, which read them with bulk copies
 *    and need 16-byte alignment.
 *  - Conditions only the device can see (a non-finite weight, a wait that
 *    gave up) set a device status word; read it with bq_device_status().
 *  - On a CUDA launch failure the entry point returns BQ_ERR_CUDA.
 *  - Every entry point may be called from several host threads and for
 *    several devices in one process (kernel attributes are set per device).
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BQ_OK = 0,
    BQ_ERR_NULL = 1,        /* a required pointer is NULL */
    BQ_ERR_SHAPE = 2,       /* sizes are inconsistent or not multiples of a tile */
    BQ_ERR_ALIGN = 3,       /* a pointer is not aligned as required */
    BQ_ERR_UNSUPPORTED = 4, /* bits / group / layout / dtype combination not supported */
    BQ_ERR_WORKSPACE = 5,   /* reserved */
    BQ_ERR_NONFINITE = 6,   /* device: a weight is NaN/Inf, or a group's fp32 scale overflows */
    BQ_ERR_TIMEOUT = 7,     /* device: a bounded wait inside a kernel gave up */
    BQ_ERR_CUDA = 8         /* a CUDA runtime call or launch failed */
} bq_status;

typedef enum { BQ_F16 = 0, BQ_BF16 = 1, BQ_F32 = 2 } bq_dtype;

/*
 * Packed-code layouts.  Both hold b-bit codes, b in {2, 4}; a matrix takes
 * rows * cols * b / 8 bytes in either layout.
 *
 * BQ_LAYOUT_CANONICAL: row-major; code k of a row is field k mod (32/b) of
 *   little-endian 32-bit word k / (32/b) of that row, fields numbered from the
 *   least significant bit.  Needs cols * b % 32 == 0.
 *
 * BQ_LAYOUT_INTERLEAVED: the layout the linear kernels read.  The matrix is
 *   cut into 512-byte tiles of 16 rows by T columns (T = 64 for 4-bit, 128 for
 *   2-bit).  Rows are grouped in blocks of 128 (the last block may be shorter:
 *   R_b = its rows / 16 tiles high).  Block b starts at byte
 *   b * 128 * cols * bits / 8 and stores its tiles column-block major: tile
 *   (row tile t of the block, column block kt) at 512 * (kt * R_b + t) from
 *   the block start, so a run of column blocks of a whole block is one
 *   contiguous range.
 *   Inside a tile, 16-byte "lane" L (0..31) serves rows r = L/4 and r + 8 and,
 *   in every run of 16 columns, the column pairs (2c, 2c+1) and (2c+8, 2c+9),
 *   c = L % 4.  Slot i of a run is (row r, low pair), (row r+8, low pair),
 *   (row r, high pair), (row r+8, high pair) for i = 0..3.
 *     4-bit: 32-bit word j of the lane holds run j; slot i keeps its even
 *            column in nibble i and its odd column in nibble i + 4.
 *     2-bit: word j holds runs 2j (fields 0..3, 8..11) and 2j+1 (fields
 *            4..7, 12..15); slot i of run 2j+h keeps its even column in field
 *            4h + i and its odd column in field 4h + i + 8.
 *   Scales and zeros of the interleaved layout are stored 128-row-block
 *   major, then by group, then by row: group g of row n (G = cols / group
 *   groups per row) at index 128 * G * (n / 128) + g * R + n % 128, R = rows
 *   of n's block, so a block's metadata over a run of groups is contiguous.
 *   (Canonical layout: row-major [rows, cols/group].)
 *   Needs rows % 16 == 0 and cols % T == 0.  With this order a lane's 16-byte
 *   load is already in the register order of a 16x8x16 bf16 tensor-core
 *   fragment, and one AND/OR with a magic exponent turns two codes into a
 *   bf16x2 pair.
 */
typedef enum { BQ_LAYOUT_CANONICAL = 0, BQ_LAYOUT_INTERLEAVED = 1 } bq_layout;

/* Bytes of packed codes for a rows x cols matrix at `bits` (no metadata). */
size_t bq_packed_bytes(int64_t rows, int64_t cols, int bits);

/* Number of groups (= number of scales = number of zeros). */
size_t bq_group_count(int64_t rows, int64_t cols, int group);

/*
 * Mixed precision (Layer-mix / Channel-mix, GreenBitAI article, paragraph on
 * the mixed-precision search space).  A bit map assigns one width to every
 * block of 128 consecutive rows: 4 (group 128) or 2 (group 64).  Layer-mix
 * is the special case of one width per matrix.  A mixed matrix stores its
 * blocks one after the other in row order: block i's packed codes start at
 * byte code_off[i] and its scales / zeros at element group_off[i], each
 * block laid out as an independent 128 x cols matrix.
 *
 * bq_mixed_offsets: host-side helper.  bit_map (host, rows/128 entries);
 * code_off and group_off (host, rows/128 + 1 entries each) receive the
 * running sums; the last entries are the totals.  Needs rows % 128 == 0.
 */
bq_status bq_mixed_offsets(const uint8_t *bit_map, int64_t rows, int64_t cols,
                           int64_t *code_off, int64_t *group_off);

/*
 * bq_quantize: quantize W and pack the codes.
 *   W        [rows, cols] of wtype (BQ_F16 or BQ_BF16), 16-byte aligned
 *   bits     4 or 2
 *   group    production: 128 with bits 4, 64 with bits 2.  Also accepted for
 *            tests: any of 16, 32, 64, 128, 256 dividing cols (canonical layout
 *            also 8).
 *   layout   BQ_LAYOUT_CANONICAL or BQ_LAYOUT_INTERLEAVED (shape rules above)
 *   packed   [bq_packed_bytes(rows, cols, bits)] bytes, 16-byte aligned
 *   scales   rows * cols/group fp32, in the layout's metadata order (above)
 *   zeros    rows * cols/group uint8, same order
 * A non-finite weight, or a group whose scale overflows fp32, sets
 * BQ_ERR_NONFINITE in the device status word; that group's outputs are then
 * unspecified.
 */
bq_status bq_quantize(const void *W, bq_dtype wtype, int64_t rows, int64_t cols,
                      int bits, int group, bq_layout layout,
                      void *packed, float *scales, uint8_t *zeros, void *stream);

/*
 * bq_quantize_mixed: quantize with a per-128-row-block width.
 *   bit_map  DEVICE array of rows/128 bytes, each 4 or 2 (any other value sets
 *            BQ_ERR_UNSUPPORTED in the device status word and skips the block)
 *   packed / scales / zeros: sized by the totals of bq_mixed_offsets(); the
 *            device computes each block's offsets from bit_map itself.
 */
bq_status bq_quantize_mixed(const void *W, bq_dtype wtype, int64_t rows, int64_t cols,
                            const uint8_t *bit_map, bq_layout layout,
                            void *packed, float *scales, uint8_t *zeros, void *stream);

/*
 * bq_dequantize: W_out[rows, cols] = (q - z) * s, computed in fp32 and
 * rounded once to otype (BQ_F32, BQ_F16 or BQ_BF16).  A test / inspection
 * utility; the linear layer never calls it.
 *   bit_map  NULL for a uniform matrix (bits, group used), else a DEVICE
 *            bit map as in bq_quantize_mixed (bits and group ignored).
 */
bq_status bq_dequantize(const void *packed, const float *scales, const uint8_t *zeros,
                        const uint8_t *bit_map, int bits, int group,
                        int64_t rows, int64_t cols, bq_layout layout,
                        void *W_out, bq_dtype otype, void *stream);

/*
 * bq_quantize_symmetric: the symmetric abs-max scheme ("大模型量化实战",
 * section 2.3: s = x_absmax / 127 at 8 bits, zero point fixed at 0), per
 * group like bq_quantize:
 *     s = max |x| / (2^(b-1) - 1)          fp32, one IEEE division
 *     q = round(x / s) + 2^(b-1)           half to even; 1 <= q <= 2^b - 1
 *     z = 2^(b-1) (stored in `zeros`, so dequant(q) = (q - z) * s as above)
 *     an all-zero group stores s = 0 and every code equal to z
 * Same arguments, layouts, outputs and errors as bq_quantize; the result is
 * consumed unchanged by bq_dequantize and bq_linear.
 */
bq_status bq_quantize_symmetric(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                                bq_layout layout, void *packed, float *scales, uint8_t *zeros, void *stream);

/*
 * bq_quantize_f16s: the asymmetric MinMax scheme of bq_quantize with the
 * group scales stored as binary16 -- a storage format that cuts the
 * metadata from 5 to 3 bytes per group (INT2 g64: from 24% to 16% of the
 * linear layer's bytes).  s is computed as in bq_quantize, rounded to the
 * nearest binary16 (ties to even; a positive s below the binary16 range
 * becomes 2^-24, one above it sets BQ_ERR_NONFINITE), and z and the codes
 * are then computed from that stored s16 with bq_quantize's steps, so
 * dequant(q) = (q - z) * s16 ("大模型量化实战", section 2.2 formulas; "低比特
 * 量化", Zero Point).  A code that round(x / s16) + z pushes past 2^b - 1
 * is clamped.  Only the linear layer's pairs: bits 4 with group 128, bits 2
 * with group 64 (others BQ_ERR_UNSUPPORTED).
 *   scales   binary16 bit patterns, same count and order as bq_quantize's
 *            fp32 scales, 2-byte aligned (16-byte for bq_linear_f16s)
 * Other arguments, layouts, outputs and errors as bq_quantize.
 */
bq_status bq_quantize_f16s(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                           bq_layout layout, void *packed, uint16_t *scales, uint8_t *zeros, void *stream);

/*
 * bq_fake_quantize: W_out = dequant(quant(W)) in one pass, without storing
 * codes, scales or zeros -- the forward of quantization-aware training
 * ("大模型量化实战", section 5.2: a FakeQuantize module simulates
 * round(x/s) + z in the forward pass; "A Survey of Low-bit Large Language
 * Models", section 8.1).
 *   W       [rows, cols] of wtype (BQ_F16 / BQ_BF16), 16-byte aligned
 *   groups  `group` consecutive elements along cols (cols % group == 0;
 *           group in {8, 16, 32, 64, 128, 256}); bits 2 or 4
 *   W_out   [rows, cols] of otype (BQ_F16, BQ_BF16 or BQ_F32), 16-byte aligned;
 *           element (q - z) * s computed in fp32 and rounded once to otype, so
 *           W_out equals bq_dequantize(bq_quantize(W)) bit for bit
 * A non-finite weight sets BQ_ERR_NONFINITE in the device status (its group's
 * outputs are unspecified).
 */
bq_status bq_fake_quantize(const void *W, bq_dtype wtype, int64_t rows, int64_t cols, int bits, int group,
                           void *W_out, bq_dtype otype, void *stream);

/*
 * bq_linear: y[M, N] = x[M, K] . dequant(W)^T.
 *   x        [M, K] of xtype (BQ_BF16 or BQ_F16), 16-byte aligned rows (K % 8 == 0)
 *   packed / scales / zeros: from bq_quantize in BQ_LAYOUT_INTERLEAVED; all
 *            three 16-byte aligned (they are read with bulk copies)
 *   bit_map  NULL for a uniform matrix (bits, group used; production pairs
 *            (4, 128) and (2, 64), tests also group 32 and 256), else a DEVICE
 *            bit map as in bq_quantize_mixed (bits, group ignored)
 *   y        [M, N] of xtype, written in full (K == 0: zeros, x not read;
 *            M == 0 or N == 0: nothing is done)
 * Products are accumulated in fp32 per group on exact (q - z) operands, then
 * scaled by the group's fp32 s and summed in fp32; y is rounded once.
 * M <= 16 runs the decode kernel (split-K dequant-GEMV on tensor cores);
 * larger M runs the prefill kernel.  Needs N % 16 == 0 and K % 256 == 0 at
 * 4 bits, K % 512 == 0 at 2 bits; with a bit map N % 128 == 0 and
 * K % 512 == 0.
 */
bq_status bq_linear(const void *x, bq_dtype xtype, int64_t M, int64_t K,
                    const void *packed, const float *scales, const uint8_t *zeros,
                    const uint8_t *bit_map, int bits, int group, int64_t N,
                    bq_layout layout, void *y, void *stream);

/*
 * bq_linear_workspace_bytes: device workspace that lets bq_linear_ws split
 * the K dimension of the tensor-core kernel (M >= 64) for this shape; 0
 * when no split is planned (bq_linear_ws then does what bq_linear does).
 * A split is planned when the output tiles (128 weight rows x 256 tokens)
 * would occupy fewer than half of the SMs: SK CTAs (2..8, filling one wave)
 * then share each tile, each over a K range of whole code stages (256
 * columns at 4 bits, 512 at 2 bits or under a width map).  The workspace
 * holds their fp32 partial tiles (128 KB per CTA) and one counter per tile.
 *   mixed    nonzero for a width map (bits then ignored)
 * Returns 0 for shapes the tensor-core kernel does not take.
 */
size_t bq_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int bits, int mixed);

/*
 * bq_linear_ws: bq_linear with a DEVICE workspace for the split-K plan of
 * bq_linear_workspace_bytes.  A NULL or smaller workspace disables the split
 * (the result is then bq_linear's).  With a split, each CTA stores its
 * partial tile and counts its arrival; the CTA that arrives last adds the
 * partials in rank order and writes y, so y is deterministic (it can differ
 * from bq_linear's in the last bits: another fp32 summation order).  The
 * library resets the counters it uses at each call (on `stream`, before the
 * kernel); two calls in flight at the same time must not share a workspace.
 *   workspace  256-byte aligned (BQ_ERR_ALIGN otherwise)
 * Other arguments, rules and errors as bq_linear.  No page describes a
 * split of the contraction: it is a scheduling choice of this library.
 */
bq_status bq_linear_ws(const void *x, bq_dtype xtype, int64_t M, int64_t K,
                       const void *packed, const float *scales, const uint8_t *zeros,
                       const uint8_t *bit_map, int bits, int group, int64_t N,
                       bq_layout layout, void *y, void *workspace, size_t workspace_bytes, void *stream);

/*
 * bq_linear_f16s: bq_linear for weights from bq_quantize_f16s (binary16
 * scales, uniform width, bits 4 with group 128 or bits 2 with group 64; no
 * bit map).  The binary16 scale is exact in fp32, so the products are
 * those of bq_linear with the same scale values.  Arguments, shape rules,
 * alignment and errors as bq_linear.
 */
bq_status bq_linear_f16s(const void *x, bq_dtype xtype, int64_t M, int64_t K,
                         const void *packed, const uint16_t *scales, const uint8_t *zeros,
                         int bits, int group, int64_t N, bq_layout layout, void *y, void *stream);

/*
 * bq_linear_grad_input: dx[M, K] = dy[M, N] . dequant(W), the gradient of
 * bq_linear's output with respect to its input -- the backward pass of the
 * layer when training in the quantized weight space (GreenBitAI article: the
 * Bitorch Engine paragraph on gradients of low-bit tensors, and the Q-SFT
 * paragraph).  W [N, K] is read in place; no dequantized copy is formed.
 *   dy       [M, N] of dtype (BQ_BF16 or BQ_F16), 16-byte aligned
 *   packed / scales / zeros: W from bq_quantize or bq_quantize_symmetric in
 *            BQ_LAYOUT_INTERLEAVED, all three 16-byte aligned
 *   bit_map  NULL for a uniform matrix (bits, group as in bq_linear), else a
 *            DEVICE width map as in bq_quantize_mixed (W from
 *            bq_quantize_mixed; bits, group ignored; N % 128 == 0; an entry
 *            other than 4 or 2 sets BQ_ERR_UNSUPPORTED in the device status
 *            and that block contributes nothing)
 *   dx       [M, K] of dtype, written in full (N == 0: zeros, dy not read;
 *            M == 0 or K == 0: nothing is done)
 * dx[m, k] = sum_n dy[m, n] s[n, g] (q[n, k] - z[n, g]) on tensor cores with
 * fp32 accumulation: (q - z) enters exactly, dy[m, n] s[n, g] is rounded once
 * to tf32 (relative error at most 2^-11), dx is rounded once to dtype.  Runs
 * in passes of at most 16 tokens, each reading W once.  Needs N % 16 == 0,
 * K % 128 == 0 and K % group == 0.
 */
bq_status bq_linear_grad_input(const void *dy, bq_dtype dtype, int64_t M, int64_t N,
                               const void *packed, const float *scales, const uint8_t *zeros,
                               const uint8_t *bit_map, int bits, int group, int64_t K,
                               bq_layout layout, void *dx, void *stream);

/*
 * Options.
 *
 * BQ_OPT_LINEAR_OVERLAP (process-wide, default 0 or the value of the
 * environment variable BQ_OVERLAP):
 *   0  bq_linear launches plainly.
 *   1  bq_linear uses programmatic dependent launch: it lets the next kernel
 *      in the stream start launching early and waits for the previous kernel
 *      to complete before reading any input or writing y.  Hides launch gaps
 *      in back-to-back layers; results are identical.
 *   2  as 1, and the decode kernel may start streaming packed codes, scales
 *      and zeros BEFORE the previous kernel in the stream has completed.  Only
 *      valid when that kernel does not write them (static weights, e.g. a
 *      decode step); x is always read after the wait.
 * bq_set_option returns BQ_ERR_UNSUPPORTED for an unknown option or value.
 */
typedef enum { BQ_OPT_LINEAR_OVERLAP = 0 } bq_option;
bq_status bq_set_option(int option, int value);
int bq_get_option(int option);

/*
 * bq_device_status: synchronize `stream`, return the first error recorded by
 * a kernel since the last call (BQ_OK if none) and clear it.
 */
bq_status bq_device_status(void *stream);

/*
 * bq_check_division: diagnostic.  The quantizer rounds x / s from a quotient
 * computed by two Markstein refinements of x * RN(1/s) (P. Markstein, IBM J.
 * Res. Dev. 34(1), 1990) rather than an IEEE division.  This entry point
 * compares that quotient (with `refinements` = 1 or 2 steps) bit for bit
 * against the IEEE division (a zero quotient of either sign counts as equal:
 * x = -0 gives +0 after refinement, and both round to the same code) for
 * every fp32 divisor whose bit pattern lies in
 * [s_bits_begin, s_bits_end) and every fp16 numerator with |x| < 64.
 *   result  DEVICE array of 4 uint64, zeroed by the caller: [0] mismatches,
 *           [1] pairs checked, [2] / [3] bit patterns of the first mismatch
 *           found (divisor, fp16 numerator).
 */
bq_status bq_check_division(uint32_t s_bits_begin, uint32_t s_bits_end, int refinements,
                            unsigned long long *result, void *stream);

/*
 * bq_check_const_division: diagnostic.  The quantizer computes the group
 * scale s = (hi - lo) / (2^b - 1) (and the symmetric scale max|x| /
 * (2^(b-1) - 1)) by the same refinement with the constant r = RN(1/D), for
 * 2^-100 <= |x| <= 2^120, and by the IEEE division outside that range.  This
 * entry point compares that quotient bit for bit against the IEEE division
 * by `divisor` (3, 7 or 15; others return BQ_ERR_UNSUPPORTED) for every fp32
 * bit pattern in [x_bits_begin, x_bits_end) (NaN inputs compare equal when
 * both results are NaN).
 *   result  DEVICE array of 4 uint64, zeroed by the caller: [0] mismatches,
 *           [1] values checked, [2] bit pattern of the first mismatch found,
 *           [3] the divisor it was found for.
 */
bq_status bq_check_const_division(int divisor, uint32_t x_bits_begin, uint32_t x_bits_end,
                                  unsigned long long *result, void *stream);

/*
 * bq_selftest_bounded_wait: diagnostic of the failure path of the kernels'
 * bounded waits.  Launches one small kernel on `stream` that waits, with the
 * same routine every kernel of the library uses, on a shared-memory barrier
 * phase that nothing ever completes, giving up after `limit` polls (1 to
 * 2^20).  The kernel then records BQ_ERR_TIMEOUT in the device status word
 * and returns normally; nothing hangs and the context stays usable.  The next
 * bq_device_status() returns BQ_ERR_TIMEOUT (and clears it).
 */
bq_status bq_selftest_bounded_wait(uint32_t limit, void *stream);

/* Human-readable name of a status code (static string). */
const char *bq_status_string(bq_status status);

/* Library version string, for logs. */
const char *bq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
