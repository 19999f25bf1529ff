/*
 * mx_oracle.c -- plain, slow, CPU reference of microscaling (MX) quantisation,
 * NVFP4 quantisation, dequantisation and the block-scaled matmul.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant generator with the CUDA
 * path: every codec here is written out from the format definitions with integer
 * bit manipulation and exact double arithmetic, one plain loop per block.
 *
 * Sources (cited by page title and section):
 *   [Q]  "MXFP4 と NVFP4 は何が違うのか調べてみた" (qiita.com)
 *        Q§1 "E2M1 という共通土台"               -- E2M1 value set, no Inf/NaN, max 6
 *        Q§2 "MXFP4 はブロック32と E8M0"           -- block 32, E8M0 (bias 127, 0xFF NaN,
 *                                                     no Inf), MX family table, RNE rule,
 *                                                     scale rounding left open
 *        Q§3 "NVFP4 はブロック16と E4M3、そして二段目" -- block 16, unsigned E4M3 scale
 *                                                     (max 448), FP32 per-tensor scale
 *                                                     = amax / (6 * 448)
 *        Q§4 "同じ E2M1 でも、別仕様である", sub-section "精度の差はどこから出るか"
 *                                                  -- floor school (scaled max in [4,8),
 *                                                     clip above 6) vs no-clip school
 *                                                     (scaled max in (3,6])
 *        Q§7 "ハードウェアの対応状況"               -- scale application: MX is an
 *                                                     exponent add; NVFP4 an FP8 multiply
 *                                                     then an FP32 multiply
 *        Q§8 "その後の標準化はどこへ向かっているか", sub-section "適合性検証という新しい層"
 *                                                  -- E4M3 overflow: saturate or NaN is
 *                                                     implementation-defined
 *   [P4] gpt-oss MXFP4 explainer (m.lxslee.cn repost), section "MXFP4"
 *                                                  -- worked example of a direct cast and
 *                                                     of a shared-scale cast
 *
 * Readings taken where the pages are silent (each is also listed in the design notes):
 *   - overflow saturates to +-max (Q§8 allows either; saturate is chosen);
 *   - +-Inf saturates to +-max; a NaN element (direct cast only) becomes the format's
 *     NaN code with its sign for E4M3/E5M2 (0x7F|s) and +-6 (0x7|s) for E2M1, which
 *     has no NaN (Q§1);
 *   - a 32-block that holds a NaN or Inf gets scale 0xFF and all element codes 0
 *     (Q§2: a NaN scale makes the whole block NaN, so the codes carry nothing);
 *   - an all-zero block gets s = -127 (E8M0 code 0x00) after the clamp;
 *   - the sign of a zero result is kept (-tiny -> 0x80 for FP8, 0x8 for FP4);
 *   - element codes are stored densely, code i of a row at bits [w*i, w*i + w) of the
 *     row read as a little-endian bit string: FP4 two per byte (even index low), FP6
 *     four per three bytes, FP8 / INT8 one per byte (the pages give no memory layout;
 *     dense packing keeps MXFP6 at its 6.25 bits per element);
 *   - column-wise output is the transposed matrix (cols x rows), blocks along rows;
 *   - NVFP4 step order: see mxo_quantize_nvfp4.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

/* Format identifiers (shared numbering with the public ABI enum, an interface only). */
enum { F_E4M3 = 0, F_E5M2 = 1, F_E2M1 = 2, F_NVFP4 = 3, F_E2M3 = 4, F_E3M2 = 5, F_INT8 = 6 };
/* Extra code kinds for mxo_decode / mxo_encode. */
enum { K_E4M3 = 0, K_E5M2 = 1, K_E2M1 = 2, K_UE4M3 = 3, K_E8M0 = 4, K_BF16 = 5, K_E2M3 = 6, K_E3M2 = 7,
       K_INT8 = 8 };
enum { R_FLOOR = 0, R_CEIL = 1 };

/* ------------------------------------------------------------------------- */
/* Format parameters, written from the definitions.                          */
/*   E2M1: 1 sign, 2 exponent, 1 mantissa bit, bias 1, no Inf/NaN, max 6  (Q§1) */
/*   E4M3: 1 sign, 4 exponent, 3 mantissa bits, bias 7, S.1111.111 = NaN,     */
/*         no Inf, max 448 (Q§3 "最大448")                                     */
/*   E5M2: 1 sign, 5 exponent, 2 mantissa bits, bias 15, IEEE-like Inf/NaN,   */
/*         max 1.75 * 2^15 = 57344                                            */
/*   E8M0: 8 exponent bits, bias 127, 0xFF = NaN, no Inf (Q§2)                */
/*   MXFP6 / MXINT8 element formats (Q§2 lists them as MX family members with */
/*   6.25 and 8.25 effective bits; their parameters are the OCP MX ones):     */
/*   E2M3: 1 sign, 2 exponent, 3 mantissa bits, bias 1, no Inf/NaN, max 7.5   */
/*   E3M2: 1 sign, 3 exponent, 2 mantissa bits, bias 3, no Inf/NaN, max 28    */
/*   INT8: two's complement q with an implicit factor 2^-6 (value q/64),      */
/*         symmetric range -127 .. 127 (max 127/64)                           */
/* ------------------------------------------------------------------------- */
typedef struct {
    int ebits, mbits, bias;
    int has_sign;
    int nan_all_ones;   /* E4M3: only exponent=all-ones & mantissa=all-ones is NaN */
    int ieee_special;   /* E5M2: exponent all-ones is Inf/NaN */
} fmt_t;

static fmt_t fmt_of(int kind) {
    fmt_t f;
    memset(&f, 0, sizeof f);
    switch (kind) {
    case K_E4M3:  f.ebits = 4; f.mbits = 3; f.bias = 7;  f.has_sign = 1; f.nan_all_ones = 1; break;
    case K_UE4M3: f.ebits = 4; f.mbits = 3; f.bias = 7;  f.has_sign = 0; f.nan_all_ones = 1; break;
    case K_E5M2:  f.ebits = 5; f.mbits = 2; f.bias = 15; f.has_sign = 1; f.ieee_special = 1; break;
    case K_E2M1:  f.ebits = 2; f.mbits = 1; f.bias = 1;  f.has_sign = 1; break;
    case K_E2M3:  f.ebits = 2; f.mbits = 3; f.bias = 1;  f.has_sign = 1; break;
    case K_E3M2:  f.ebits = 3; f.mbits = 2; f.bias = 3;  f.has_sign = 1; break;
    case K_BF16:  f.ebits = 8; f.mbits = 7; f.bias = 127; f.has_sign = 1; f.ieee_special = 1; break;
    default: break;
    }
    return f;
}

/* Decode one code of a sign/exponent/mantissa format to its exact value. */
static double decode_sem(fmt_t f, unsigned code) {
    unsigned nbits = (unsigned)(f.has_sign + f.ebits + f.mbits);
    unsigned mmask = (1u << f.mbits) - 1u;
    unsigned emask = (1u << f.ebits) - 1u;
    unsigned sign = f.has_sign ? (code >> (nbits - 1)) & 1u : 0u;
    unsigned e = (code >> f.mbits) & emask;
    unsigned m = code & mmask;
    double v;
    if (f.nan_all_ones && e == emask && m == mmask) return sign ? -NAN : NAN;
    if (f.ieee_special && e == emask) return m ? (sign ? -NAN : NAN) : (sign ? -INFINITY : INFINITY);
    if (e == 0) v = ldexp((double)m, 1 - f.bias - f.mbits);             /* subnormal */
    else        v = ldexp((double)((1u << f.mbits) | m), (int)e - f.bias - f.mbits);
    return sign ? -v : v;
}

/* Largest finite magnitude and its code (without sign). */
static unsigned max_code(fmt_t f) {
    unsigned emask = (1u << f.ebits) - 1u, mmask = (1u << f.mbits) - 1u;
    if (f.nan_all_ones) return (emask << f.mbits) | (mmask - 1u);       /* S.1111.110 */
    if (f.ieee_special) return ((emask - 1u) << f.mbits) | mmask;        /* S.11110.11 */
    return (emask << f.mbits) | mmask;                   /* no specials: all ones (E2M1 0.11.1) */
}

/* Split a finite positive double into integer significand M and exponent x:  a = M * 2^x. */
static void split_double(double a, uint64_t *M, int *x) {
    uint64_t bits;
    memcpy(&bits, &a, 8);
    int ef = (int)((bits >> 52) & 0x7FF);
    uint64_t frac = bits & ((1ull << 52) - 1);
    if (ef == 0) { *M = frac; *x = -1074; }
    else         { *M = frac | (1ull << 52); *x = ef - 1075; }
}

static int bitlen64(uint64_t v) { int n = 0; while (v) { n++; v >>= 1; } return n; }

/*
 * Round-to-nearest-even of a finite value onto the format's finite grid, saturating
 * at the largest finite magnitude (Q§2: the OCP text requires roundTiesToEven for the
 * cast; Q§8: saturation is one of the two allowed overflow behaviours).
 * The rounding is done on the integer significand with a remainder (guard/sticky)
 * compare, never through floating-point arithmetic.
 */
static unsigned encode_sem(fmt_t f, double v, int saturate_to_inf /* bf16 only */) {
    unsigned nbits = (unsigned)(f.has_sign + f.ebits + f.mbits);
    unsigned sign_bit = f.has_sign ? (1u << (nbits - 1)) : 0u;
    unsigned sign = (f.has_sign && signbit(v)) ? sign_bit : 0u;
    unsigned mc = max_code(f);
    double maxval = decode_sem(f, mc);
    if (isnan(v)) return 0; /* callers decide NaN handling before calling */
    double a = fabs(v);
    if (!saturate_to_inf && a >= maxval) return sign | mc;
    if (a == 0.0) return sign;
    uint64_t M; int x;
    split_double(a, &M, &x);
    int E = x + bitlen64(M) - 1;                     /* floor(log2 a) */
    int emin = 1 - f.bias;                           /* exponent of the smallest normal */
    int Eq = E > emin ? E : emin;
    int qe = Eq - f.mbits;                           /* grid quantum is 2^qe in this binade */
    uint64_t q;
    int k = qe - x;                                  /* right shift that lands on the grid */
    if (k <= 0) {
        q = M << (-k);
    } else if (k >= 63) {
        q = 0;                                       /* far below half a quantum */
    } else {
        uint64_t rem = M & ((1ull << k) - 1), half = 1ull << (k - 1);
        q = M >> k;
        if (rem > half || (rem == half && (q & 1u))) q += 1;
    }
    if (q == 0) return sign;
    /* q * 2^qe is the rounded magnitude; q <= 2^(mbits+1). */
    unsigned e_field, m_field;
    if (q < (1ull << f.mbits)) {                    /* subnormal */
        e_field = 0; m_field = (unsigned)q;
    } else if (q == (1ull << (f.mbits + 1))) {      /* carried into the next binade */
        e_field = (unsigned)(Eq + 1 + f.bias); m_field = 0;
    } else {
        e_field = (unsigned)(Eq + f.bias); m_field = (unsigned)(q - (1ull << f.mbits));
    }
    unsigned emask = (1u << f.ebits) - 1u;
    if (saturate_to_inf) {
        /* bf16: overflow past the largest finite value rounds to Inf (IEEE RNE). */
        if (e_field >= emask) return sign | (emask << f.mbits);
        return sign | (e_field << f.mbits) | m_field;
    }
    unsigned code = (e_field << f.mbits) | m_field;
    if (decode_sem(f, code) > maxval || isnan(decode_sem(f, code))) code = mc;
    return sign | code;
}

/* ------------------------------------------------------------------------- */
/* Public scalar codecs                                                       */
/* ------------------------------------------------------------------------- */

/* E8M0: 2^(c-127) for c in 0..254; 0xFF is NaN; no Inf (Q§2). */
static double decode_e8m0(unsigned c) { return c == 0xFFu ? NAN : ldexp(1.0, (int)c - 127); }

double mxo_decode(int kind, unsigned code) {
    if (kind == K_E8M0) return decode_e8m0(code & 0xFFu);
    if (kind == K_INT8) return ldexp((double)(int8_t)(uint8_t)code, -6);
    return decode_sem(fmt_of(kind), code);
}

/* Direct cast of one value (no block scale), saturating RNE, with the NaN reading above. */
unsigned mxo_encode(double v, int kind) {
    fmt_t f = fmt_of(kind);
    if (kind == K_BF16) {
        if (isnan(v)) return 0x7FC0u | (signbit(v) ? 0x8000u : 0u);
        if (isinf(v)) return v > 0 ? 0x7F80u : 0xFF80u;
        return encode_sem(f, v, 1);
    }
    if (kind == K_INT8) {
        /* round half to even onto the integers q/64, saturating symmetrically at +-127 */
        if (isnan(v)) return 0u;
        double q = v * 64.0;                             /* exact: a power-of-two multiply */
        long iq = fabs(q) >= 127.5 ? (q > 0 ? 127 : -127) : (long)rint(q);
        if (iq > 127) iq = 127;
        if (iq < -127) iq = -127;
        return (unsigned)(uint8_t)(int8_t)iq;
    }
    if (isnan(v)) {
        unsigned nbits = (unsigned)(f.has_sign + f.ebits + f.mbits);
        unsigned s = signbit(v) ? (1u << (nbits - 1)) : 0u;
        if (kind == K_E2M1 || kind == K_E2M3 || kind == K_E3M2)
            return s | max_code(f);                      /* no NaN in E2M1 / FP6: +-max */
        if (kind == K_UE4M3) return 0x7Fu;
        return s | 0x7Fu;                                /* E4M3 / E5M2 NaN */
    }
    return encode_sem(f, v, 0);
}

/* bf16 bits -> exact double. */
static double bf16_value(uint16_t b) { return decode_sem(fmt_of(K_BF16), b); }

/* fp32 -> bf16 bits, round to nearest even (used after the NVFP4 fp32 products). */
static uint16_t f32_to_bf16(float y) { return (uint16_t)mxo_encode((double)y, K_BF16); }

/* ------------------------------------------------------------------------- */
/* Shared-scale exponent (Q§4 "精度の差はどこから出るか"; Q§2 last paragraph)   */
/* ------------------------------------------------------------------------- */

/* Exponent of the element format's largest binade and its largest finite value. */
static int emax_of(int fmt) {
    switch (fmt) {
    case F_E4M3: return 8;     /* 448   = 1.75   x 2^8  */
    case F_E5M2: return 15;    /* 57344 = 1.75   x 2^15 */
    case F_E2M3: return 2;     /* 7.5   = 1.875  x 2^2  */
    case F_E3M2: return 4;     /* 28    = 1.75   x 2^4  */
    case F_INT8: return 0;     /* 127/64 = 1.984375 x 2^0 */
    default:     return 2;     /* E2M1: 6 = 1.5 x 2^2 */
    }
}
static int elem_kind(int fmt);
static double maxval_of(int fmt) {
    if (fmt == F_INT8) return 127.0 / 64.0;
    fmt_t f = fmt_of(elem_kind(fmt));
    return decode_sem(f, max_code(f));
}

/*
 * Shared exponent s for a block whose largest magnitude is amax (finite, >= 0).
 *   floor school (OCP example): s = floor(log2 amax) - emax_elem; the scaled block
 *     maximum then lies in [2^emax, 2^(emax+1)) -- [4, 8) for E2M1 -- and whatever is
 *     above the format maximum is clipped by the cast.
 *   ceil school (no clipping): s = the smallest integer with amax <= max_elem * 2^s;
 *     the scaled maximum then lies in (max/2, max] -- (3, 6] for E2M1.
 * Both are clamped to the E8M0 range [-127, 127]; amax = 0 gives -127.
 * floor(log2 amax) comes from frexp (amax = f 2^e with f in [0.5, 1), so it is e - 1);
 * the smallest s is found by exact comparison against max_elem * 2^s, searching
 * upwards from a value known to be too small.
 */
int mxo_scale_exponent(double amax, int fmt, int rounding) {
    int s, e;
    if (amax == 0.0) return -127;
    (void)frexp(amax, &e);
    int E = e - 1;                                   /* floor(log2 amax) */
    if (rounding == R_FLOOR) {
        s = E - emax_of(fmt);
    } else {
        double mx = maxval_of(fmt);
        s = E - emax_of(fmt) - 2;                    /* amax > max * 2^s here */
        while (!(amax <= ldexp(mx, s))) s++;
    }
    if (s < -127) s = -127;
    if (s > 127) s = 127;
    return s;
}

/* ------------------------------------------------------------------------- */
/* MX block quantisation (Q§2, Q§4): block of 32, E8M0 scale, RNE+saturate.   */
/* ------------------------------------------------------------------------- */

static int elem_kind(int fmt) {
    switch (fmt) {
    case F_E4M3: return K_E4M3;
    case F_E5M2: return K_E5M2;
    case F_E2M3: return K_E2M3;
    case F_E3M2: return K_E3M2;
    case F_INT8: return K_INT8;
    default:     return K_E2M1;
    }
}
/* Element formats of the MX family (block 32, E8M0 scale): E4M3, E5M2, E2M1, E2M3, E3M2, INT8. */
static int mx_fmt_ok(int fmt) { return (fmt >= F_E4M3 && fmt <= F_E2M1) || (fmt >= F_E2M3 && fmt <= F_INT8); }

/* Quantise one block of n bf16 values; writes n codes (one per entry) and returns the
 * E8M0 scale byte. */
static unsigned quantize_block_mx(const uint16_t *x, int n, int fmt, int rounding, unsigned *codes) {
    double amax = 0.0;
    int nonfinite = 0;
    for (int i = 0; i < n; i++) {
        double v = bf16_value(x[i]);
        if (isnan(v) || isinf(v)) nonfinite = 1;
        else if (fabs(v) > amax) amax = fabs(v);
    }
    if (nonfinite) {                    /* NaN scale: the whole block is NaN (Q§2) */
        for (int i = 0; i < n; i++) codes[i] = 0;
        return 0xFFu;
    }
    int s = mxo_scale_exponent(amax, fmt, rounding);
    for (int i = 0; i < n; i++) {
        double scaled = ldexp(bf16_value(x[i]), -s);    /* exact: a power-of-two multiply */
        codes[i] = mxo_encode(scaled, elem_kind(fmt));
    }
    return (unsigned)(s + 127);
}

/* Width in bits of one stored element code: FP8 and INT8 8, FP6 6, FP4 4.             */
static int code_bits(int fmt) {
    return (fmt == F_E2M1 || fmt == F_NVFP4) ? 4 : (fmt == F_E2M3 || fmt == F_E3M2) ? 6 : 8;
}

/* Element codes are stored densely along a row: code i occupies bits [w*i, w*i + w) of
 * the row's bytes read as one little-endian bit string (w = code width).  For FP4 that
 * is two codes per byte, the even one low; for FP6 four codes per three bytes; for FP8
 * and INT8 one code per byte.  Written bit by bit, the plainest form of that rule. */
static void put_code(uint8_t *row, int64_t i, unsigned code, int bits) {
    for (int b = 0; b < bits; b++) {
        int64_t at = (int64_t)bits * i + b;
        uint8_t m = (uint8_t)(1u << (at % 8));
        if ((code >> b) & 1u) row[at / 8] |= m;
        else                  row[at / 8] &= (uint8_t)~m;
    }
}
static unsigned get_code(const uint8_t *row, int64_t i, int bits) {
    unsigned code = 0;
    for (int b = 0; b < bits; b++) {
        int64_t at = (int64_t)bits * i + b;
        code |= (unsigned)((row[at / 8] >> (at % 8)) & 1u) << b;
    }
    return code;
}

/*
 * MX quantisation of a rows x cols bf16 row-major matrix.
 *   axis 0 (row-wise): blocks of 32 along each row; elems rows x cols, scales rows x cols/32.
 *   axis 1 (col-wise): blocks of 32 down each column; the output is the transposed
 *     matrix: elems cols x rows, scales cols x rows/32.
 * Scales are row-major here; the tcgen05 tiling is a re-indexing of these bytes.
 * Returns 0, or -1 on a shape that is not a multiple of the block.
 */
int mxo_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int axis, int rounding,
                    uint8_t *elems, uint8_t *scales) {
    const int B = 32;
    int bits = code_bits(fmt);
    int64_t out_rows = axis == 0 ? rows : cols, out_cols = axis == 0 ? cols : rows;
    if (!mx_fmt_ok(fmt) || out_cols % B) return -1;
    uint16_t blk[32];
    unsigned codes[32];
    int64_t row_bytes = out_cols * bits / 8;
    memset(elems, 0, (size_t)(out_rows * row_bytes));
    for (int64_t r = 0; r < out_rows; r++) {
        for (int64_t b = 0; b < out_cols / B; b++) {
            for (int i = 0; i < B; i++) {
                int64_t j = b * B + i;   /* position along the quantisation axis */
                blk[i] = axis == 0 ? x[r * cols + j] : x[j * cols + r];
            }
            scales[r * (out_cols / B) + b] = (uint8_t)quantize_block_mx(blk, B, fmt, rounding, codes);
            for (int i = 0; i < B; i++) put_code(elems + r * row_bytes, b * B + i, codes[i], bits);
        }
    }
    return 0;
}

/* Direct element cast with no block scale (the "direct cast" of [P4]). */
int mxo_cast(const uint16_t *x, int64_t n, int fmt, uint8_t *out) {
    int bits = code_bits(fmt);
    if (!mx_fmt_ok(fmt) || fmt == F_INT8 || (n * bits) % 8) return -1;   /* INT8 needs a scale */
    memset(out, 0, (size_t)(n * bits / 8));
    for (int64_t i = 0; i < n; i++) put_code(out, i, mxo_encode(bf16_value(x[i]), elem_kind(fmt)), bits);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* NVFP4 (Q§3, Q§7): E2M1 elements, block 16, unsigned E4M3 block scale,      */
/* FP32 per-tensor scale = tensor amax / (6 * 448).                           */
/* ------------------------------------------------------------------------- */

/*
 * Step order, every operation an IEEE fp32 round-to-nearest operation:
 *   1. amax_t = max |x| over the finite entries of the tensor.
 *   2. g = amax_t / 2688.0f (the per-tensor decode scale, Q§3); g = 1 if amax_t = 0.
 *   3. per 16-block: amax_b over finite entries; a block holding a NaN or Inf gets the
 *      UE4M3 NaN code 0x7F and all element codes 0;
 *      t = amax_b / (6.0f * g);  sb = UE4M3 RNE-saturated code of t.
 *   4. d = dec(sb) * g.  If d == 0 every code is 0; otherwise q_i = E2M1 RNE-saturated
 *      code of the fp32 quotient x_i / d (one IEEE division, round to nearest; a zero
 *      x_i gives a zero of its own sign).  Q§3 defines the element as x over the
 *      two-level scale and Q§7 fixes only the order of the decode multiplies; the
 *      division by the fp32 decode scale d is the plain reading of that definition.
 * g is written to *g_out.  rows x cols row-major; blocks along rows (cols % 16 == 0);
 * elems rows x cols/2 bytes (even index low nibble), scales rows x cols/16.
 */
/* One NVFP4 block of nr rows x 16 columns at (r0, c0) (steps 3-4 above); writes its codes
 * into elems (packed, row pitch cols/2) and returns the UE4M3 scale code. */
static unsigned nvfp4_block(const uint16_t *x, int64_t cols, int64_t r0, int64_t c0, int nr, float g,
                            uint8_t *elems) {
    const int B = 16;
    float amax_b = 0.0f;
    int nonfinite = 0;
    for (int rr = 0; rr < nr; rr++)
        for (int i = 0; i < B; i++) {
            double v = bf16_value(x[(r0 + rr) * cols + c0 + i]);
            if (isnan(v) || isinf(v)) nonfinite = 1;
            else if ((float)fabs(v) > amax_b) amax_b = (float)fabs(v);
        }
    if (nonfinite) {
        for (int rr = 0; rr < nr; rr++)
            for (int i = 0; i < B; i++) put_code(elems + (r0 + rr) * (cols / 2), c0 + i, 0, 4);
        return 0x7Fu;
    }
    volatile float six_g = 6.0f * g;
    volatile float t = amax_b / six_g;
    unsigned sb = mxo_encode((double)t, K_UE4M3);
    volatile float d = (float)decode_sem(fmt_of(K_UE4M3), sb) * g;
    for (int rr = 0; rr < nr; rr++)
        for (int i = 0; i < B; i++) {
            unsigned q = 0;
            if (d != 0.0f) {
                volatile float xi = (float)bf16_value(x[(r0 + rr) * cols + c0 + i]);
                volatile float y = xi / d;
                q = mxo_encode((double)y, K_E2M1);
            }
            put_code(elems + (r0 + rr) * (cols / 2), c0 + i, q, 4);
        }
    return sb;
}

/* Steps 1-2: the per-tensor decode scale g. */
static float nvfp4_global_scale(const uint16_t *x, int64_t n) {
    float amax_t = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        double v = bf16_value(x[i]);
        if (!isnan(v) && !isinf(v) && (float)fabs(v) > amax_t) amax_t = (float)fabs(v);
    }
    volatile float g = amax_t == 0.0f ? 1.0f : amax_t / 2688.0f;
    return g;
}

int mxo_quantize_nvfp4(const uint16_t *x, int64_t rows, int64_t cols, uint8_t *elems,
                       uint8_t *scales, float *g_out) {
    const int B = 16;
    if (cols % B) return -1;
    const float g = nvfp4_global_scale(x, rows * cols);
    *g_out = g;
    memset(elems, 0, (size_t)(rows * cols / 2));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < cols / B; b++)
            scales[r * (cols / B) + b] = (uint8_t)nvfp4_block(x, cols, r, b * B, 1, g, elems);
    return 0;
}

/*
 * Two-dimensional NVFP4 block scaling for weights (Q§4: the 4-bit pre-training recipe
 * uses two-dimensional block scaling for the weights).  The block is 16 x 16: one UE4M3
 * scale per 16 rows x 16 columns, the same steps 1-4 over its 256 entries.  The scales
 * are written in the 1 x 16 layout (rows x cols/16), each 2-D block's code repeated on its
 * 16 rows, so every 1 x 16 consumer (dequantisation, the matmul) reads them unchanged;
 * the transposed matrix quantised the same way gives the transposed codes and scales.
 * rows and cols are multiples of 16.
 */
int mxo_quantize_nvfp4_2d(const uint16_t *x, int64_t rows, int64_t cols, uint8_t *elems,
                          uint8_t *scales, float *g_out) {
    const int B = 16;
    if (cols % B || rows % B) return -1;
    const float g = nvfp4_global_scale(x, rows * cols);
    *g_out = g;
    memset(elems, 0, (size_t)(rows * cols / 2));
    for (int64_t rb = 0; rb < rows / B; rb++)
        for (int64_t b = 0; b < cols / B; b++) {
            const unsigned sb = nvfp4_block(x, cols, rb * B, b * B, B, g, elems);
            for (int rr = 0; rr < B; rr++) scales[(rb * B + rr) * (cols / B) + b] = (uint8_t)sb;
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Dequantisation (Q§7: MX is an exponent add, exact; Q§2: a NaN scale makes  */
/* the whole block NaN).  Output bf16, round to nearest even.                 */
/* ------------------------------------------------------------------------- */

/* rows x cols codes (row-major, blocks of 32 along rows), scales rows x cols/32. */
int mxo_dequantize_mx(const uint8_t *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                      int fmt, uint16_t *out) {
    const int B = 32;
    int bits = code_bits(fmt);
    if (!mx_fmt_ok(fmt) || cols % B) return -1;
    int64_t row_bytes = cols * bits / 8;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t j = 0; j < cols; j++) {
            unsigned s = scales[r * (cols / B) + j / B];
            unsigned q = get_code(elems + r * row_bytes, j, bits);
            double v = s == 0xFFu ? NAN : ldexp(mxo_decode(elem_kind(fmt), q), (int)s - 127);
            out[r * cols + j] = (uint16_t)mxo_encode(v, K_BF16);
        }
    }
    return 0;
}

/* NVFP4: x = (dec(q) * dec(sb)) * g in fp32, then bf16 RNE; sb = 0x7F gives NaN. */
int mxo_dequantize_nvfp4(const uint8_t *elems, const uint8_t *scales, float g, int64_t rows,
                         int64_t cols, uint16_t *out) {
    const int B = 16;
    if (cols % B) return -1;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t j = 0; j < cols; j++) {
            unsigned sb = scales[r * (cols / B) + j / B] & 0x7Fu;
            unsigned q = get_code(elems + r * (cols / 2), j, 4);
            if (sb == 0x7Fu) { out[r * cols + j] = 0x7FC0u; continue; }
            volatile float p = (float)mxo_decode(K_E2M1, q) * (float)mxo_decode(K_UE4M3, sb);
            volatile float y = p * g;
            out[r * cols + j] = f32_to_bf16(y);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* tcgen05 scale-factor tiling (not in the pages; the layout the Blackwell    */
/* block-scaled MMA reads): a rows x scale_cols byte matrix is cut into       */
/* 128-row x 4-column atoms of 512 bytes; inside an atom, entry (r, c) sits   */
/* at (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4); atoms are stored with the */
/* row-block index outer and the column-block index inner; rows pad to 128    */
/* and scale columns to 4, padding bytes are zero.                            */
/* ------------------------------------------------------------------------- */
int64_t mxo_tcgen05_scale_bytes(int64_t rows, int64_t scale_cols) {
    return ((rows + 127) / 128) * ((scale_cols + 3) / 4) * 512;
}
int64_t mxo_tcgen05_scale_offset(int64_t r, int64_t c, int64_t rows, int64_t scale_cols) {
    (void)rows;
    int64_t col_atoms = (scale_cols + 3) / 4;
    int64_t atom = (r / 128) * col_atoms + c / 4;
    return atom * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4);
}

/* ------------------------------------------------------------------------- */
/* Block-scaled matmul reference: C[m,n] = sum_k a(m,k) b(n,k) in fp64 over   */
/* the dequantised operands, a(m,k) = dec(A_q) * 2^(sA-127) and likewise b   */
/* (Q§7 scale application; scales per 32 along K).  An NVFP4 operand decodes */
/* as dec(q) * dec_UE4M3(s) * g with scales per 16 along K and its per-tensor */
/* g (Q§3 two-level scaling).  A is M x K and B is N x K, both K-major,      */
/* scales row-major (K/32 or K/16 per row).  Computes the npairs requested   */
/* (m, n) entries and, for each, sum_k |a b| (the error budget).             */
/* ------------------------------------------------------------------------- */
static double mx_operand_value(const uint8_t *elems, const uint8_t *scales, int fmt, double g,
                               int64_t row, int64_t k, int64_t K) {
    int bits = code_bits(fmt);
    int64_t row_bytes = K * bits / 8;
    unsigned q = get_code(elems + row * row_bytes, k, bits);
    if (fmt == F_NVFP4) {
        unsigned sb = scales[row * (K / 16) + k / 16];
        if (sb == 0x7Fu) return NAN;
        return mxo_decode(K_E2M1, q) * mxo_decode(K_UE4M3, sb) * g;
    }
    unsigned s = scales[row * (K / 32) + k / 32];
    if (s == 0xFFu) return NAN;
    return ldexp(mxo_decode(elem_kind(fmt), q), (int)s - 127);
}

int mxo_gemm_ref(const uint8_t *a_elems, const uint8_t *a_scales, int a_fmt, double a_g,
                 const uint8_t *b_elems, const uint8_t *b_scales, int b_fmt, double b_g,
                 int64_t M, int64_t N, int64_t K, const int64_t *pairs, int64_t npairs,
                 double *c, double *abs_sum) {
    if (K % 32) return -1;
    for (int64_t p = 0; p < npairs; p++) {
        int64_t m = pairs[2 * p], n = pairs[2 * p + 1];
        if (m < 0 || m >= M || n < 0 || n >= N) return -1;
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double a = mx_operand_value(a_elems, a_scales, a_fmt, a_g, m, k, K);
            double b = mx_operand_value(b_elems, b_scales, b_fmt, b_g, n, k, K);
            acc += a * b;
            mag += fabs(a * b);
        }
        c[p] = acc;
        abs_sum[p] = mag;
    }
    return 0;
}

/* The same reference for every entry of the rectangle [m0, m1) x [n0, n1) (c and abs_sum
 * row-major, (m1 - m0) x (n1 - n0)): the rows involved are decoded once into double
 * buffers, then each entry is the same k = 0 .. K-1 sum as above. */
int mxo_gemm_ref_block(const uint8_t *a_elems, const uint8_t *a_scales, int a_fmt, double a_g,
                       const uint8_t *b_elems, const uint8_t *b_scales, int b_fmt, double b_g,
                       int64_t M, int64_t N, int64_t K, int64_t m0, int64_t m1, int64_t n0, int64_t n1,
                       double *c, double *abs_sum, double *a_rows, double *b_rows) {
    if (K % 32 || m0 < 0 || m1 > M || m0 > m1 || n0 < 0 || n1 > N || n0 > n1) return -1;
    for (int64_t m = m0; m < m1; m++)
        for (int64_t k = 0; k < K; k++) a_rows[(m - m0) * K + k] = mx_operand_value(a_elems, a_scales, a_fmt, a_g, m, k, K);
    for (int64_t n = n0; n < n1; n++)
        for (int64_t k = 0; k < K; k++) b_rows[(n - n0) * K + k] = mx_operand_value(b_elems, b_scales, b_fmt, b_g, n, k, K);
    for (int64_t m = m0; m < m1; m++)
        for (int64_t n = n0; n < n1; n++) {
            const double *a = a_rows + (m - m0) * K, *b = b_rows + (n - n0) * K;
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; k++) {
                acc += a[k] * b[k];
                mag += fabs(a[k] * b[k]);
            }
            c[(m - m0) * (n1 - n0) + (n - n0)] = acc;
            abs_sum[(m - m0) * (n1 - n0) + (n - n0)] = mag;
        }
    return 0;
}

/* tcgen05 tiling of a whole row-major scale matrix, and back (plain loops over the offset
 * function above; padding bytes of `tiled` are written 0). */
int mxo_to_tcgen05_layout(const uint8_t *rowmajor, int64_t rows, int64_t scale_cols, uint8_t *tiled) {
    memset(tiled, 0, (size_t)mxo_tcgen05_scale_bytes(rows, scale_cols));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < scale_cols; c++)
            tiled[mxo_tcgen05_scale_offset(r, c, rows, scale_cols)] = rowmajor[r * scale_cols + c];
    return 0;
}
int mxo_from_tcgen05_layout(const uint8_t *tiled, int64_t rows, int64_t scale_cols, uint8_t *rowmajor) {
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < scale_cols; c++)
            rowmajor[r * scale_cols + c] = tiled[mxo_tcgen05_scale_offset(r, c, rows, scale_cols)];
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Nested blocks (Q§6 "DeepSeek-V4 の入れ子構造"): an MXFP4 weight (1 x 32      */
/* sub-blocks, E8M0 scales) re-expressed as FP8 E4M3 with one scale per      */
/* 128 x 128 block, which holds 4 x 128 = 512 of the 1 x 32 sub-blocks.  The  */
/* conversion is lossless while the sub-block scales inside a block do not    */
/* spread too far; the pages give the condition (a bound on the ratio of the  */
/* largest to the smallest sub-block scale) but not the bound.  Written out:  */
/*   s_max  = the largest sub-block exponent (code - 127) among sub-blocks     */
/*            that are not NaN and hold a nonzero code;                        */
/*   S      = 2^(s_max - 6): the largest FP4 value 6 * 2^s_max maps to 384,    */
/*            inside E4M3 (max 448);                                           */
/*   each element: FP8 code = RNE-saturating E4M3 encoding of                  */
/*            dec_E2M1(q) * 2^(s_b - s_max + 6) (exact in double);             */
/*   exact  <=> every nonzero element is representable: with E2M1 values      */
/*            {1, 1.5} x 2^k (k >= -1) and E4M3's smallest step 2^-9 this is   */
/*            s_max - s_b <= 14 for every sub-block holding a nonzero code     */
/*            (the ratio bound 2^14); all-zero and NaN sub-blocks are exempt.  */
/* A NaN sub-block (scale 0xFF) gives E4M3 NaN codes 0x7F.  A block with no    */
/* nonzero finite element gets S = 1.                                          */
/* The oracle decides exactness by comparing values (decode both and check    */
/* equality), not by the bound, so a test can check the bound against it.     */
/* elems: rows x cols/2 packed E2M1; scales: rows x cols/32 row-major E8M0;   */
/* out: rows x cols E4M3 codes; block_scale / exact: (rows/128) x (cols/128). */
/* ------------------------------------------------------------------------- */
int mxo_mxfp4_to_fp8_blocks(const uint8_t *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                            uint8_t *out, float *block_scale, uint8_t *exact) {
    if (rows % 128 || cols % 128) return -1;
    const int64_t S = cols / 32, BC = cols / 128;
    for (int64_t br = 0; br < rows / 128; br++) {
        for (int64_t bc = 0; bc < BC; bc++) {
            int smax = INT32_MIN;
            for (int64_t r = br * 128; r < br * 128 + 128; r++) {
                for (int64_t b = bc * 4; b < bc * 4 + 4; b++) {
                    unsigned sc = scales[r * S + b];
                    if (sc == 0xFFu) continue;
                    int nonzero = 0;
                    for (int64_t j = b * 32; j < b * 32 + 32; j++)
                        if (mxo_decode(K_E2M1, get_code(elems + r * (cols / 2), j, 4)) != 0.0) nonzero = 1;
                    if (nonzero && (int)sc - 127 > smax) smax = (int)sc - 127;
                }
            }
            if (smax == INT32_MIN) smax = 6;                /* no nonzero finite element: S = 1 */
            block_scale[br * BC + bc] = (float)ldexp(1.0, smax - 6);
            int ok = 1;
            for (int64_t r = br * 128; r < br * 128 + 128; r++) {
                for (int64_t j = bc * 128; j < bc * 128 + 128; j++) {
                    unsigned sc = scales[r * S + j / 32];
                    unsigned q = get_code(elems + r * (cols / 2), j, 4);
                    unsigned code;
                    if (sc == 0xFFu) {
                        code = 0x7Fu;
                    } else {
                        double v = ldexp(mxo_decode(K_E2M1, q), (int)sc - 127 - (smax - 6));
                        code = mxo_encode(v, K_E4M3);
                        if (mxo_decode(K_E4M3, code) != v) ok = 0;   /* -0 == +0 counts as equal */
                    }
                    out[r * cols + j] = (uint8_t)code;
                }
            }
            exact[br * BC + bc] = (uint8_t)ok;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* 16 x 16 random Hadamard transform (Q§4: the 4-bit pre-training recipe      */
/* applies a 16 x 16 random Hadamard transform to the inputs of the weight    */
/* gradient).  The pages name the transform but not its form; reading:        */
/*   for every 16 consecutive elements x of a row: y = H16 D x / 4, with      */
/*   D = diag(+-1) from a 16-bit sign mask (bit i set: element i negated) and */
/*   H16 the Sylvester Hadamard matrix (H1 = [1], H2n = [[Hn, Hn], [Hn, -Hn]]),*/
/*   so that H16 D / 4 is orthogonal; computed as the radix-2 butterfly      */
/*   (strides 1, 2, 4, 8; (a, b) -> (a + b, a - b)) in fp32 round-to-nearest, */
/*   the 1/4 applied last (exact), and the result rounded to bf16 (the       */
/*   tensor's type) before it is quantised.                                  */
/* ------------------------------------------------------------------------- */
static void rht16(const uint16_t *x, unsigned sign_mask, uint16_t *y) {
    volatile float v[16];
    for (int i = 0; i < 16; i++) {
        float f = (float)bf16_value(x[i]);
        v[i] = ((sign_mask >> i) & 1u) ? -f : f;
    }
    for (int h = 1; h < 16; h <<= 1)
        for (int i = 0; i < 16; i += 2 * h)
            for (int j = i; j < i + h; j++) {
                volatile float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    for (int i = 0; i < 16; i++) {
        volatile float q = v[i] * 0.25f;
        y[i] = f32_to_bf16(q);
    }
}

/* The transform of a rows x cols bf16 matrix (cols % 16 == 0), row by row. */
int mxo_rht16(const uint16_t *x, int64_t rows, int64_t cols, unsigned sign_mask, uint16_t *out) {
    if (cols % 16) return -1;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c += 16) rht16(x + r * cols + c, sign_mask & 0xFFFFu, out + r * cols + c);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Stochastic rounding of the element cast (Q§4: the 4-bit pre-training      */
/* recipe rounds gradients stochastically; Q§8: P3109 defines stochastic     */
/* rounding).  The pages fix no procedure; reading, with one random byte r    */
/* (0..255) per element, passed in by the caller:                            */
/*   |y| >= the format maximum  -> the maximum (saturation, as the RNE cast); */
/*   otherwise lo = the largest representable magnitude <= |y| and hi the    */
/*   next one; |y| == lo -> lo; else hi when 256 (|y| - lo) > r (hi - lo),    */
/*   lo otherwise -- probability ceil(256 f) / 256 of rounding up for         */
/*   f = (|y| - lo) / (hi - lo), unbiased to 1/256 of a step;                 */
/*   the sign is that of y (a zero result keeps it).                         */
/* lo and hi are found by scanning the decoded code table (no arithmetic     */
/* shortcut), the comparison is exact in double.                            */
/* ------------------------------------------------------------------------- */
static unsigned encode_sr(double y, int kind, unsigned r) {
    fmt_t f = fmt_of(kind);
    unsigned nbits = (unsigned)(f.has_sign + f.ebits + f.mbits);
    unsigned sign = signbit(y) ? (1u << (nbits - 1)) : 0u;
    unsigned mc = max_code(f);
    double a = fabs(y);
    if (a >= decode_sem(f, mc)) return sign | mc;
    unsigned lo_c = 0, hi_c = mc;
    double lo = 0.0, hi = decode_sem(f, mc);
    for (unsigned c = 0; c <= mc; c++) {          /* magnitudes increase with the code */
        double v = decode_sem(f, c);
        if (isnan(v) || isinf(v)) continue;
        if (v <= a && v >= lo) { lo = v; lo_c = c; }
        if (v > a && v < hi) { hi = v; hi_c = c; }
    }
    if (a == lo) return sign | lo_c;
    return sign | ((256.0 * (a - lo) > (double)r * (hi - lo)) ? hi_c : lo_c);
}

/* Row-wise MX quantisation with stochastic rounding of the element cast (E4M3, E5M2, E2M1;
 * the scale is the deterministic shared exponent); rnd: rows x cols random bytes. */
int mxo_quantize_mx_sr(const uint16_t *x, int64_t rows, int64_t cols, int fmt, int rounding,
                       const uint8_t *rnd, uint8_t *elems, uint8_t *scales) {
    const int B = 32;
    if (!(fmt == F_E4M3 || fmt == F_E5M2 || fmt == F_E2M1) || cols % B) return -1;
    int bits = code_bits(fmt);
    int64_t row_bytes = cols * bits / 8;
    memset(elems, 0, (size_t)(rows * row_bytes));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < cols / B; b++) {
            const uint16_t *blk = x + r * cols + b * B;
            double amax = 0.0;
            int nonfinite = 0;
            for (int i = 0; i < B; i++) {
                double v = bf16_value(blk[i]);
                if (isnan(v) || isinf(v)) nonfinite = 1;
                else if (fabs(v) > amax) amax = fabs(v);
            }
            if (nonfinite) {
                scales[r * (cols / B) + b] = 0xFF;
                continue;                               /* codes stay 0 */
            }
            int s = mxo_scale_exponent(amax, fmt, rounding);
            scales[r * (cols / B) + b] = (uint8_t)(s + 127);
            for (int i = 0; i < B; i++) {
                double scaled = ldexp(bf16_value(blk[i]), -s);
                put_code(elems + r * row_bytes, b * B + i,
                         encode_sr(scaled, elem_kind(fmt), rnd[r * cols + b * B + i]), bits);
            }
        }
    return 0;
}

/* NVFP4 with stochastic rounding of the element cast: steps 1-4 of the NVFP4 path, the
 * E2M1 code of the fp32 quotient x_i / d rounded stochastically (the UE4M3 block scale
 * stays RNE). */
int mxo_quantize_nvfp4_sr(const uint16_t *x, int64_t rows, int64_t cols, const uint8_t *rnd,
                          uint8_t *elems, uint8_t *scales, float *g_out) {
    const int B = 16;
    if (cols % B) return -1;
    const float g = nvfp4_global_scale(x, rows * cols);
    *g_out = g;
    memset(elems, 0, (size_t)(rows * cols / 2));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t b = 0; b < cols / B; b++) {
            const uint16_t *blk = x + r * cols + b * B;
            float amax_b = 0.0f;
            int nonfinite = 0;
            for (int i = 0; i < B; i++) {
                double v = bf16_value(blk[i]);
                if (isnan(v) || isinf(v)) nonfinite = 1;
                else if ((float)fabs(v) > amax_b) amax_b = (float)fabs(v);
            }
            if (nonfinite) { scales[r * (cols / B) + b] = 0x7F; continue; }
            volatile float six_g = 6.0f * g;
            volatile float t = amax_b / six_g;
            unsigned sb = mxo_encode((double)t, K_UE4M3);
            volatile float d = (float)decode_sem(fmt_of(K_UE4M3), sb) * g;
            scales[r * (cols / B) + b] = (uint8_t)sb;
            for (int i = 0; i < B; i++) {
                unsigned q = 0;
                if (d != 0.0f) {
                    volatile float xi = (float)bf16_value(blk[i]);
                    volatile float y = xi / d;
                    q = encode_sr((double)y, K_E2M1, rnd[r * cols + b * B + i]);
                }
                put_code(elems + r * (cols / 2), b * B + i, q, 4);
            }
        }
    return 0;
}
