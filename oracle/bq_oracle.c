/*
 * bq_oracle.c -- plain, slow CPU oracle for the group-wise asymmetric MinMax
 * weight quantizer and the weight-only linear layer that consumes its output.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA
 * path.
 *
 * Sources (web pages, cited by title and section):
 *   [GB]  "只需单卡 RTX 3090，低比特量化训练就能实现 LLaMA-3 8B 全参微调"
 *         (GreenBitAI article) -- the paragraph that fixes the quantizer:
 *         classic Group-wise MinMax, INT4 with group 128 and INT2 with
 *         group 64; the paragraph on Layer-mix / Channel-mix.
 *   [LBQ] "低比特量化 / Low-bit Quantization" -- table "What is Low-bit
 *         Quantization" (INT4 0~15, INT2 0~3), sections "Group Quantization"
 *         and "Zero Point" (value = (code - zero_point) * scale).
 *   [4BG] "大模型量化实战：从原理到4-bit部署的完整指南" -- section 2.2
 *         (Q(x) = round(x/s) + z, s = range / number of levels - 1,
 *         z = round(0 - x_min/s), z kept inside the integer range).
 *
 * Readings where the pages leave a step open (each is also listed in the
 * design notes of the repository):
 *   R1  the group range is widened to contain 0: lo' = min(min x, 0),
 *       hi' = max(max x, 0).  Identical to the literal formula whenever the
 *       group straddles 0; guarantees 0 <= z <= 2^b - 1.
 *   R2  an all-zero group has s = 0; it stores s = 0, z = 0, q = 0.
 *   R3  "round" is round-half-to-even applied to the fp32 quotient x/s
 *       (one IEEE division, round-to-nearest-even), and z is added as an
 *       integer afterwards; s = (hi' - lo') / (2^b - 1) in fp32,
 *       z = round(-lo'/s) likewise.  Codes are clamped to [0, 2^b - 1].
 *   R4  scales are fp32, zeros are uint8.
 *   R5  groups run along the input dimension K inside one output row.
 *   R8  a non-finite input, or a group whose fp32 scale overflows, is an error.
 *   R14 fp16 group scales (a storage format of the same scheme): s is
 *       computed as in R1-R3, then rounded to the nearest binary16 (ties to
 *       even); a positive s that rounds to zero takes the smallest positive
 *       binary16 (2^-24), one that rounds to infinity is an error (R8).  z and
 *       the codes are then computed from the stored binary16 scale exactly as
 *       R3 prescribes, so (q - z) * s16 is the reconstruction.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared.
 * -ffp-contract=off keeps every multiply and add separately rounded, so the
 * fp32 steps below are exactly the ones written.
 *
 * Parity status: every function here is pinned by tests that do not retype
 * its formulas (hand-worked examples, exact rational brute force, closed
 * forms, library conversions); see tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <fenv.h>

#define BQO_OK 0
#define BQO_ERR_NONFINITE 1
#define BQO_ERR_ARG 2

/* ------------------------------------------------------------------ */
/* Element decoding.                                                   */
/* ------------------------------------------------------------------ */

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Decoded by its definition; every binary16 value is exact in binary32. */
float bqo_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    float mag;
    if (e == 0) {
        mag = ldexpf((float)f, -24);                  /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        mag = (f == 0) ? INFINITY : NAN;
    } else {
        mag = ldexpf((float)(1024 + f), e - 25);      /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of a binary32 word. */
float bqo_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float v;
    memcpy(&v, &u, 4);
    return v;
}

/* binary32 -> binary16, round to nearest, ties to even, from the format's
 * definition: 10 fraction bits, exponent bias 15, subnormals below 2^-14
 * with a fixed step of 2^-24, values at or above 65520 (halfway between the
 * largest finite 65504 and 2^16) round to infinity. */
uint16_t bqo_f32_to_f16(float v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    float a = fabsf(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7e00u);
    if (a >= 65520.0f) return (uint16_t)(sign | 0x7c00u);
    /* the step (unit in the last place) of binary16 at a */
    int e;
    frexpf(a, &e);                     /* a = m * 2^e, 0.5 <= m < 1 */
    int ulp_exp = e - 11;              /* 11 significant bits */
    if (ulp_exp < -24) ulp_exp = -24;  /* subnormal step */
    /* a / step is exact in binary32 (a scaled by a power of two); round it
     * to an integer, half to even */
    float n = nearbyintf(ldexpf(a, -ulp_exp));
    double r = ldexp((double)n, ulp_exp);   /* the rounded magnitude, exact */
    if (r == 0.0) return sign;
    int re;
    frexp(r, &re);
    if (re - 1 < -14) {                /* subnormal: fraction = r / 2^-24 */
        return (uint16_t)(sign | (uint16_t)ldexp(r, 24));
    }
    if (re - 1 > 15) return (uint16_t)(sign | 0x7c00u);
    /* normal: r = (1 + f/1024) * 2^(re-1) */
    uint16_t exp_field = (uint16_t)(re - 1 + 15);
    uint16_t frac = (uint16_t)(ldexp(r, -(re - 1) + 10) - 1024.0);
    return (uint16_t)(sign | (exp_field << 10) | frac);
}

static float decode(uint16_t h, int wtype)
{
    return wtype == 0 ? bqo_f16_to_f32(h) : bqo_bf16_to_f32(h);
}

/* ------------------------------------------------------------------ */
/* One group: [GB] MinMax quantizer with [4BG] s.2.2 arithmetic.        */
/* ------------------------------------------------------------------ */

/* f16_scale = 1: reading R14, the scale stored as binary16 (one rounding
 * step inserted after s is computed; z and the codes then use it). */
static int quantize_group_minmax(const float *x, int g, int bits, int f16_scale,
                                 float *s_out, int *z_out, uint8_t *q_out)
{
    if (g <= 0 || bits < 1 || bits > 8) return BQO_ERR_ARG;
    const int qmax = (1 << bits) - 1;

    /* min and max of the group (exact) */
    float lo = x[0], hi = x[0];
    for (int i = 0; i < g; ++i) {
        if (!isfinite(x[i])) return BQO_ERR_NONFINITE;
        if (x[i] < lo) lo = x[i];
        if (x[i] > hi) hi = x[i];
    }
    /* R1: the range always contains zero */
    if (lo > 0.0f) lo = 0.0f;
    if (hi < 0.0f) hi = 0.0f;

    /* s = (max - min) / (2^b - 1), fp32 */
    float range = hi - lo;
    float s = range / (float)qmax;
    if (!isfinite(s)) return BQO_ERR_NONFINITE;

    /* R2: all-zero group */
    if (s == 0.0f) {
        *s_out = 0.0f;
        *z_out = 0;
        memset(q_out, 0, (size_t)g);
        return BQO_OK;
    }

    /* R14: round the scale to binary16 and work with the stored value */
    if (f16_scale) {
        s = bqo_f16_to_f32(bqo_f32_to_f16(s));
        if (s == 0.0f) s = ldexpf(1.0f, -24);
        if (!isfinite(s)) return BQO_ERR_NONFINITE;
    }

    /* z = round(-min / s), half to even (the default rounding mode) */
    float zq = -lo / s;
    int z = (int)nearbyintf(zq);

    /* q = clamp(round(x / s) + z, 0, 2^b - 1) */
    for (int i = 0; i < g; ++i) {
        float t = x[i] / s;
        int r = (int)nearbyintf(t);
        int q = r + z;
        if (q < 0) q = 0;
        if (q > qmax) q = qmax;
        q_out[i] = (uint8_t)q;
    }
    *s_out = s;
    *z_out = z;
    return BQO_OK;
}

int bqo_quantize_group(const float *x, int g, int bits,
                       float *s_out, int *z_out, uint8_t *q_out)
{
    return quantize_group_minmax(x, g, bits, 0, s_out, z_out, q_out);
}

/* R14: the MinMax scheme with the scale stored as binary16. */
int bqo_quantize_group_s16(const float *x, int g, int bits,
                           float *s_out, int *z_out, uint8_t *q_out)
{
    return quantize_group_minmax(x, g, bits, 1, s_out, z_out, q_out);
}

/* Symmetric abs-max scheme ("大模型量化实战", section 2.3: s = x_absmax /
 * (2^(b-1) - 1) -- 127 at 8 bits -- and z fixed at 0, codes round(x / s)).
 * Readings: applied per group like the MinMax scheme; codes are stored
 * offset by 2^(b-1) (z = 2^(b-1)) so that the unsigned storage and
 * dequant(q) = (q - z) * s of the MinMax scheme apply unchanged; the same
 * rounding as R3 (one fp32 division, half to even); an all-zero group
 * stores s = 0 and every code equal to z.
 *   s = max |x| / (2^(b-1) - 1)
 *   q = clamp(round(x / s) + 2^(b-1), 0, 2^b - 1)                            */
int bqo_quantize_group_sym(const float *x, int g, int bits,
                           float *s_out, int *z_out, uint8_t *q_out)
{
    if (g <= 0 || bits < 2 || bits > 8) return BQO_ERR_ARG;
    const int qmax = (1 << bits) - 1;
    const int z = 1 << (bits - 1);

    float amax = 0.0f;
    for (int i = 0; i < g; ++i) {
        if (!isfinite(x[i])) return BQO_ERR_NONFINITE;
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s = amax / (float)(z - 1);
    if (!isfinite(s)) return BQO_ERR_NONFINITE;
    if (s == 0.0f) {
        *s_out = 0.0f;
        *z_out = z;
        memset(q_out, z, (size_t)g);
        return BQO_OK;
    }
    for (int i = 0; i < g; ++i) {
        int q = (int)nearbyintf(x[i] / s) + z;
        q_out[i] = (uint8_t)(q < 0 ? 0 : (q > qmax ? qmax : q));
    }
    *s_out = s;
    *z_out = z;
    return BQO_OK;
}

/* Whole matrix W[rows, cols] (row-major, fp16 when wtype == 0, bf16 when
 * wtype == 1), groups of `group` consecutive elements along cols (R5).
 * Only rows [r0, r1) are processed so that callers may split rows across
 * threads.  Outputs: codes[rows*cols] unpacked, scales/zeros[rows*(cols/group)]. */
int bqo_quantize_scheme(const uint16_t *W, int wtype, int64_t rows, int64_t cols,
                        int bits, int group, int scheme, int64_t r0, int64_t r1,
                        uint8_t *codes, float *scales, uint8_t *zeros);

int bqo_quantize(const uint16_t *W, int wtype, int64_t rows, int64_t cols,
                 int bits, int group, int64_t r0, int64_t r1,
                 uint8_t *codes, float *scales, uint8_t *zeros)
{
    return bqo_quantize_scheme(W, wtype, rows, cols, bits, group, 0, r0, r1, codes, scales, zeros);
}

/* scheme 0: asymmetric MinMax (bqo_quantize_group); 1: symmetric abs-max
 * (bqo_quantize_group_sym); 2: asymmetric MinMax with binary16 scales
 * (bqo_quantize_group_s16; the scales are written as the binary32 values of
 * the stored binary16 numbers). */
int bqo_quantize_scheme(const uint16_t *W, int wtype, int64_t rows, int64_t cols,
                        int bits, int group, int scheme, int64_t r0, int64_t r1,
                        uint8_t *codes, float *scales, uint8_t *zeros)
{
    if (scheme < 0 || scheme > 2) return BQO_ERR_ARG;
    if (group <= 0 || cols % group != 0 || r0 < 0 || r1 > rows) return BQO_ERR_ARG;
    if (group > 4096) return BQO_ERR_ARG;
    if (fegetround() != FE_TONEAREST) return BQO_ERR_ARG;
    const int64_t G = cols / group;
    float buf[4096];
    for (int64_t n = r0; n < r1; ++n) {
        for (int64_t j = 0; j < G; ++j) {
            const uint16_t *src = W + n * cols + j * group;
            for (int i = 0; i < group; ++i) buf[i] = decode(src[i], wtype);
            float s;
            int z;
            uint8_t *q = codes + n * cols + j * group;
            int rc = scheme == 1 ? bqo_quantize_group_sym(buf, group, bits, &s, &z, q)
                   : scheme == 2 ? bqo_quantize_group_s16(buf, group, bits, &s, &z, q)
                                 : bqo_quantize_group(buf, group, bits, &s, &z, q);
            if (rc) return rc;
            scales[n * G + j] = s;
            zeros[n * G + j] = (uint8_t)z;
        }
    }
    return BQO_OK;
}

/* ------------------------------------------------------------------ */
/* Bit packing.                                                        */
/* ------------------------------------------------------------------ */

/* Canonical layout: each row is a run of little-endian 32-bit words; code k
 * of a row sits at bit position bits*(k mod (32/bits)) of word k/(32/bits).
 * Equivalently: byte (k*bits)/8 of the row, bit (k*bits)%8 of that byte. */
static void canonical_position(int64_t n, int64_t k, int64_t cols, int bits,
                               int64_t *byte_off, int *bit_off)
{
    const int per_word = 32 / bits;
    int64_t row_bytes = cols * bits / 8;
    int64_t word = k / per_word;
    int bit_in_word = bits * (int)(k % per_word);
    *byte_off = n * row_bytes + word * 4 + bit_in_word / 8;
    *bit_off = bit_in_word % 8;
}

/* Interleaved (tiled) layout used by the linear kernels.
 *
 * The matrix is cut into tiles of 16 rows by T columns (T = 64 for 4-bit,
 * T = 128 for 2-bit); every tile is 512 bytes.  Rows are grouped in blocks
 * of 128 (8 tiles high; the last block may hold fewer, R_b = its rows / 16).
 * Block b starts at byte b * 128 * cols * bits / 8 and stores its tiles
 * column-block major: tile (row tile t of the block, column block kt) at
 * 512 * (kt * R_b + t) from the block start, so one column block of a whole
 * 128-row block is contiguous.  Inside a tile, "lane" L in 0..31 owns bytes
 * [16L, 16L + 16) = four 32-bit words.  Lane L serves rows r = L/4 and r + 8
 * of the tile and, within each run of 16 columns, the column pairs (2c, 2c+1)
 * and (2c+8, 2c+9) with c = L % 4.  The four (row, column pair) slots of one
 * run of 16 columns are numbered
 *     slot 0: row r,   columns 2c, 2c+1
 *     slot 1: row r+8, columns 2c, 2c+1
 *     slot 2: row r,   columns 2c+8, 2c+9
 *     slot 3: row r+8, columns 2c+8, 2c+9
 * 4-bit: word j (0..3) holds the 16-column run j; slot i puts its even column
 *        in nibble i and its odd column in nibble i + 4.
 * 2-bit: word j (0..3) holds the 16-column runs 2j and 2j+1; run 2j+h, slot i
 *        puts its even column in 2-bit field 4h + i and its odd column in
 *        field 4h + i + 8.
 * Fields are numbered from the least significant bit of the little-endian
 * 32-bit word. */
static int64_t block_rows(int64_t n, int64_t rows)
{
    int64_t b = n / 128;
    int64_t left = rows - b * 128;
    return left < 128 ? left : 128;
}

static void interleaved_position(int64_t n, int64_t k, int64_t rows, int64_t cols, int bits,
                                 int64_t *byte_off, int *bit_off)
{
    const int64_t T = (bits == 4) ? 64 : 128;
    int64_t b = n / 128;
    int64_t Rb = block_rows(n, rows) / 16;   /* row tiles in this block */
    int64_t t = (n % 128) / 16;              /* row tile inside the block */
    int64_t kt = k / T;
    int rr = (int)(n % 16);
    int kk = (int)(k % T);
    int r = rr % 8, upper_row = rr / 8;
    int run = kk / 16;               /* 16-column run inside the tile */
    int kq = kk % 16;
    int high_half = kq / 8;          /* columns 8..15 of the run */
    int c = (kq % 8) / 2;
    int odd = kq % 2;
    int lane = 4 * r + c;
    int slot = upper_row + 2 * high_half;
    int word, field;
    if (bits == 4) {
        word = run;
        field = slot + 4 * odd;
    } else {
        word = run / 2;
        field = 4 * (run % 2) + slot + 8 * odd;
    }
    int bit_in_word = field * bits;
    int64_t block_start = b * 128 * cols * bits / 8;
    *byte_off = block_start + (kt * Rb + t) * 512 + lane * 16 + word * 4 + bit_in_word / 8;
    *bit_off = bit_in_word % 8;
}

static void position(int layout, int64_t n, int64_t k, int64_t rows, int64_t cols, int bits,
                     int64_t *byte_off, int *bit_off)
{
    if (layout == 0) canonical_position(n, k, cols, bits, byte_off, bit_off);
    else interleaved_position(n, k, rows, cols, bits, byte_off, bit_off);
}

/* Byte offset and bit offset of element (n, k) of a rows x cols matrix:
 * exported so tests can check the map against hand-derived positions. */
void bqo_code_position(int layout, int64_t n, int64_t k, int64_t rows, int64_t cols, int bits,
                       int64_t *byte_off, int *bit_off)
{
    position(layout, n, k, rows, cols, bits, byte_off, bit_off);
}

int bqo_pack(const uint8_t *codes, int64_t rows, int64_t cols, int bits,
             int layout, uint8_t *out)
{
    if (bits != 2 && bits != 4) return BQO_ERR_ARG;
    if (layout == 1) {
        const int64_t T = (bits == 4) ? 64 : 128;
        if (rows % 16 != 0 || cols % T != 0) return BQO_ERR_ARG;
    } else if ((cols * bits) % 8 != 0) {
        return BQO_ERR_ARG;
    }
    memset(out, 0, (size_t)(rows * cols * bits / 8));
    const int mask = (1 << bits) - 1;
    for (int64_t n = 0; n < rows; ++n) {
        for (int64_t k = 0; k < cols; ++k) {
            int64_t byte_off;
            int bit_off;
            position(layout, n, k, rows, cols, bits, &byte_off, &bit_off);
            out[byte_off] |= (uint8_t)((codes[n * cols + k] & mask) << bit_off);
        }
    }
    return BQO_OK;
}

int bqo_unpack(const uint8_t *packed, int64_t rows, int64_t cols, int bits,
               int layout, uint8_t *codes)
{
    if (bits != 2 && bits != 4) return BQO_ERR_ARG;
    const int mask = (1 << bits) - 1;
    for (int64_t n = 0; n < rows; ++n) {
        for (int64_t k = 0; k < cols; ++k) {
            int64_t byte_off;
            int bit_off;
            position(layout, n, k, rows, cols, bits, &byte_off, &bit_off);
            codes[n * cols + k] = (uint8_t)((packed[byte_off] >> bit_off) & mask);
        }
    }
    return BQO_OK;
}

/* Metadata layout.  Canonical: scales / zeros are [rows, cols/group],
 * row-major.  Interleaved: 128-row-block major, then group, then row, so the
 * metadata of one 128-row block over a run of groups is contiguous: element
 * (n, g) of a matrix with G groups per row sits at index
 * 128 * G * (n / 128) + g * R + n % 128, where R is the number of rows of
 * n's block (128, or fewer in a last partial block). */
int64_t bqo_meta_index(int layout, int64_t n, int64_t g, int64_t rows, int64_t G)
{
    if (layout == 0) return n * G + g;
    return 128 * G * (n / 128) + g * block_rows(n, rows) + n % 128;
}

void bqo_pack_meta_f32(const float *in, int64_t rows, int64_t G, int layout, float *out)
{
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t g = 0; g < G; ++g) out[bqo_meta_index(layout, n, g, rows, G)] = in[n * G + g];
}

void bqo_pack_meta_u8(const uint8_t *in, int64_t rows, int64_t G, int layout, uint8_t *out)
{
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t g = 0; g < G; ++g) out[bqo_meta_index(layout, n, g, rows, G)] = in[n * G + g];
}

/* ------------------------------------------------------------------ */
/* Dequantization and the weight-only linear layer.                    */
/* ------------------------------------------------------------------ */

/* [LBQ] "Zero Point": value = (code - zero_point) * scale, here in fp64 over
 * rows [r0, r1). */
void bqo_dequant_f64(const uint8_t *codes, const float *scales, const uint8_t *zeros,
                     int64_t rows, int64_t cols, int group, int64_t r0, int64_t r1,
                     double *out)
{
    const int64_t G = cols / group;
    for (int64_t n = r0; n < r1 && n < rows; ++n)
        for (int64_t k = 0; k < cols; ++k) {
            int64_t j = k / group;
            out[n * cols + k] = (double)((int)codes[n * cols + k] - (int)zeros[n * G + j])
                                * (double)scales[n * G + j];
        }
}

/* Same, rounded once to fp32 (what a dequantize-to-fp32 call returns). */
void bqo_dequant_f32(const uint8_t *codes, const float *scales, const uint8_t *zeros,
                     int64_t rows, int64_t cols, int group, float *out)
{
    const int64_t G = cols / group;
    for (int64_t n = 0; n < rows; ++n)
        for (int64_t k = 0; k < cols; ++k) {
            int64_t j = k / group;
            float d = (float)((int)codes[n * cols + k] - (int)zeros[n * G + j]);
            out[n * cols + k] = d * scales[n * G + j];
        }
}

/* y[m, n] = sum_k x[m, k] * dequant(W)[n, k] in fp64, k ascending, for output
 * channels n in [n0, n1).  x is [M, K] doubles, y is [M, N] doubles. */
void bqo_linear_f64(const double *x, int64_t M, int64_t K,
                    const uint8_t *codes, const float *scales, const uint8_t *zeros,
                    int64_t N, int group, int64_t n0, int64_t n1,
                    double *wrow /* scratch of K doubles */, double *y)
{
    const int64_t G = K / group;
    for (int64_t n = n0; n < n1 && n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t j = k / group;
            wrow[k] = (double)((int)codes[n * K + k] - (int)zeros[n * G + j])
                      * (double)scales[n * G + j];
        }
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += x[m * K + k] * wrow[k];
            y[m * N + n] = acc;
        }
    }
}

/* Input gradient of the same layer: the backward pass that training in the
 * quantized weight space needs ([GB], the Bitorch Engine paragraph on
 * gradients of low-bit tensors, and the Q-SFT paragraph).  With
 * y = x . dequant(W)^T, the gradient with respect to x is dx = dy . dequant(W):
 *   dx[m, k] = sum_n dy[m, n] * dequant(W)[n, k]   in fp64, n ascending,
 * for input columns k in [k0, k1).  dy is [M, N] doubles, dx is [M, K]. */
void bqo_linear_grad_input_f64(const double *dy, int64_t M, int64_t N,
                               const uint8_t *codes, const float *scales, const uint8_t *zeros,
                               int64_t K, int group, int64_t k0, int64_t k1,
                               double *wcol /* scratch of N doubles */, double *dx)
{
    const int64_t G = K / group;
    for (int64_t k = k0; k < k1 && k < K; ++k) {
        const int64_t j = k / group;
        for (int64_t n = 0; n < N; ++n)
            wcol[n] = (double)((int)codes[n * K + k] - (int)zeros[n * G + j])
                      * (double)scales[n * G + j];
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) acc += dy[m * N + n] * wcol[n];
            dx[m * K + k] = acc;
        }
    }
}

/* Decode an fp16 (wtype 0) or bf16 (wtype 1) array to doubles. */
void bqo_decode_f64(const uint16_t *src, int wtype, int64_t count, double *dst)
{
    for (int64_t i = 0; i < count; ++i) dst[i] = (double)decode(src[i], wtype);
}

/* Round a double straight to the nearest bfloat16 (8 significant bits,
 * exponent range of binary32, ties to even) and return its bit pattern.
 * v = m * 2^e with 0.5 <= |m| < 1; the bf16 quantum at that exponent is
 * 2^(e-8), or 2^-133 below the normal range.  The rounded value is exactly
 * representable in binary32, so the final conversion is exact. */
uint16_t bqo_f64_to_bf16(double v)
{
    if (isnan(v)) return 0x7fc0;
    double r;
    if (v == 0.0 || isinf(v)) {
        r = v;
    } else {
        int e;
        frexp(v, &e);
        int qexp = e - 8;
        if (qexp < -133) qexp = -133;
        r = ldexp(nearbyint(ldexp(v, -qexp)), qexp);
        if (fabs(r) > 3.3895313892515355e38) r = v > 0 ? INFINITY : -INFINITY;
    }
    float f = (float)r;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}
