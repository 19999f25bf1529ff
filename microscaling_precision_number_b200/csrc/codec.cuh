// codec.cuh -- device-side element and scale codecs for the MX kernels (sm_100a).
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §1 "E2M1 という共通土台": E2M1 has 15 values, max 6, no Inf/NaN.
//     §2 "MXFP4 はブロック32と E8M0": E8M0 = 2^(c-127), 0xFF NaN; roundTiesToEven cast.
//     §3 "NVFP4 はブロック16と E4M3、そして二段目": UE4M3 block scale, max 448.
//     §4 "精度の差はどこから出るか": floor rule s = floor(log2 amax) - emax_elem
//        (scaled max in [2^emax, 2^(emax+1))), and the no-clip rule (one step larger
//        when the floor rule would clip).
//
// Every rounding is done by the hardware cvt.rn.satfinite conversions (round to nearest
// even, saturate to the largest finite value); scale exponents come from the bf16
// exponent field by integer arithmetic, and scales are applied as exact power-of-two
// fp32 multiplies.
#pragma once
#include <cstdint>

namespace mxk {

enum : int { FMT_E4M3 = 0, FMT_E5M2 = 1, FMT_E2M1 = 2, FMT_NVFP4 = 3, FMT_E2M3 = 4, FMT_E3M2 = 5, FMT_INT8 = 6 };

// Exponent of the largest binade of the element format (448 = 1.75 * 2^8,
// 57344 = 1.75 * 2^15, 6 = 1.5 * 2^2, 7.5 = 1.875 * 2^2, 28 = 1.75 * 2^4,
// INT8 127/64 = 1.984375 * 2^0) and 128 x the significand of its maximum.
__host__ __device__ constexpr int emax_elem(int fmt) {
    return fmt == FMT_E4M3 ? 8 : fmt == FMT_E5M2 ? 15 : fmt == FMT_E3M2 ? 4 : fmt == FMT_INT8 ? 0 : 2;
}
__host__ __device__ constexpr int max_sig128(int fmt) {
    return fmt == FMT_E2M1 ? 192 : fmt == FMT_E2M3 ? 240 : fmt == FMT_INT8 ? 254 : 224;
}
// Stored width of one element code.  Codes are packed densely along a row: code i at bits
// [w*i, w*i + w) of the row read as a little-endian bit string -- FP4 two per byte (even
// index low), FP6 four per three bytes (16 per 12 bytes, the packed form that the TMA
// 16U6_ALIGN16B type expands for the tensor cores), FP8 / INT8 one per byte.
__host__ __device__ constexpr int code_bits(int fmt) {
    return (fmt == FMT_E2M1 || fmt == FMT_NVFP4) ? 4 : (fmt == FMT_E2M3 || fmt == FMT_E3M2) ? 6 : 8;
}
__host__ __device__ constexpr bool is_fp6(int fmt) { return fmt == FMT_E2M3 || fmt == FMT_E3M2; }

// Four FP6 codes held one per byte (low 6 bits) -> their 24 packed bits, and back.
__device__ __forceinline__ uint32_t fp6_pack4(uint32_t w) {
    return (w & 0x3Fu) | ((w >> 2) & 0xFC0u) | ((w >> 4) & 0x3F000u) | ((w >> 6) & 0xFC0000u);
}
__device__ __forceinline__ uint32_t fp6_unpack4(uint32_t p) {
    return (p & 0x3Fu) | ((p << 2) & 0x3F00u) | ((p << 4) & 0x3F0000u) | ((p << 6) & 0x3F000000u);
}
// 4k codes held one per byte (k words) -> 3k packed words (k a multiple of 4: 16 codes ->
// 12 bytes), and back.
template <int W>
__device__ __forceinline__ void fp6_pack(const uint32_t (&w)[W], uint32_t (&o)[W * 3 / 4]) {
    static_assert(W % 4 == 0, "whole 16-code groups");
#pragma unroll
    for (int g = 0; g < W / 4; g++) {
        const uint32_t p0 = fp6_pack4(w[4 * g]), p1 = fp6_pack4(w[4 * g + 1]);
        const uint32_t p2 = fp6_pack4(w[4 * g + 2]), p3 = fp6_pack4(w[4 * g + 3]);
        o[3 * g] = p0 | (p1 << 24);
        o[3 * g + 1] = (p1 >> 8) | (p2 << 16);
        o[3 * g + 2] = (p2 >> 16) | (p3 << 8);
    }
}
template <int W>
__device__ __forceinline__ void fp6_unpack(const uint32_t (&o)[W * 3 / 4], uint32_t (&w)[W]) {
#pragma unroll
    for (int g = 0; g < W / 4; g++) {
        const uint32_t a = o[3 * g], b = o[3 * g + 1], c = o[3 * g + 2];
        w[4 * g] = fp6_unpack4(a & 0xFFFFFFu);
        w[4 * g + 1] = fp6_unpack4((a >> 24) | ((b & 0xFFFFu) << 8));
        w[4 * g + 2] = fp6_unpack4((b >> 16) | ((c & 0xFFu) << 16));
        w[4 * g + 3] = fp6_unpack4(c >> 8);
    }
}

// E8M0 code from the block maximum given as |x| bf16 bits (0 .. 0x7FFF).  Any
// magnitude >= 0x7F80 (Inf or NaN) yields the NaN scale 0xFF.  A zero block yields
// s = -127 (code 0).  The exponent is clamped to [-127, 127].
template <int FMT, bool CEIL>
__device__ __noinline__ uint32_t e8m0_from_amax_bits_rare(uint32_t a) {
    if (a >= 0x7F80u) return 0xFFu;
    if (a == 0u) return 0u;
    int ef = (int)(a >> 7), mant = (int)(a & 0x7Fu);
    int E, nm;
    if (ef > 0) {            // normal: amax = (128 + mant)/128 * 2^(ef-127)
        E = ef - 127;
        nm = 128 | mant;
    } else {                 // subnormal: amax = mant * 2^-133
        int msb = 31 - __clz(mant);
        E = -133 + msb;
        nm = mant << (7 - msb);
    }
    int s = E - emax_elem(FMT);
    if (CEIL && nm > max_sig128(FMT)) s += 1;   // floor rule would clip: one binade up
    s = s < -127 ? -127 : (s > 127 ? 127 : s);
    return (uint32_t)(s + 127);
}

// Common case, a normal block maximum (0x80 <= a < 0x7F80): the code is the biased
// exponent field minus emax_elem (plus one under the no-clip rule when the maximum's
// significand exceeds the element format's largest), clamped to [0, 254] (the upper
// clamp only binds for INT8, whose emax_elem is 0).  Zero, subnormal and Inf/NaN maxima
// take the general path above (the two agree on every normal a).
template <int FMT, bool CEIL>
__device__ __forceinline__ uint32_t e8m0_from_amax_bits(uint32_t a) {
    if (__builtin_expect(a - 0x80u >= 0x7F00u, 0)) return e8m0_from_amax_bits_rare<FMT, CEIL>(a);
    int code = (int)(a >> 7) - emax_elem(FMT);
    if (CEIL) code += (int)((a & 0x7Fu) > (uint32_t)(max_sig128(FMT) - 128));
    if constexpr (emax_elem(FMT) == 0) code = code > 254 ? 254 : code;
    return (uint32_t)(code < 0 ? 0 : code);
}

// fp32 value 2^-(code-127), the multiplier that brings a block into the element range.
__device__ __forceinline__ float e8m0_inverse_multiplier(uint32_t code) {
    return code <= 253u ? __uint_as_float((254u - code) << 23) : __uint_as_float(0x00400000u);
}

// fp32 value 2^(code-127) for dequantisation (code 0 is the fp32 subnormal 2^-127).
__device__ __forceinline__ float e8m0_multiplier(uint32_t code) {
    return code >= 1u ? __uint_as_float(code << 23) : __uint_as_float(0x00400000u);
}

// bf16 pair packed in a 32-bit word (element 2i in the low half) -> two fp32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per-halfword |x| maximum over a 16-byte chunk of eight bf16 values.
__device__ __forceinline__ uint32_t abs_max_bf16x8(const uint4 &v) {
    uint32_t m = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    m = __vmaxu2(m, __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return m;
}
__device__ __forceinline__ uint32_t hmax(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

// Same, ignoring Inf/NaN lanes (magnitude >= 0x7F80 treated as 0): NVFP4 tensor amax.
__device__ __forceinline__ uint32_t finite_abs_max_bf16x8(const uint4 &v) {
    uint32_t a0 = v.x & 0x7FFF7FFFu, a1 = v.y & 0x7FFF7FFFu, a2 = v.z & 0x7FFF7FFFu, a3 = v.w & 0x7FFF7FFFu;
    a0 &= __vcmpltu2(a0, 0x7F807F80u);
    a1 &= __vcmpltu2(a1, 0x7F807F80u);
    a2 &= __vcmpltu2(a2, 0x7F807F80u);
    a3 &= __vcmpltu2(a3, 0x7F807F80u);
    return __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
}

// ---- hardware conversions (round to nearest even, satfinite) ---------------------------
// Two fp32 -> two byte codes in one 16-bit word, `lo` in the low byte: FP8, FP6 (6-bit
// code in the low bits of its byte) by the hardware conversion; INT8 as the MXINT8
// element (the value times 64, rounded half to even, saturated to -127 .. 127).
template <int FMT>
__device__ __forceinline__ uint32_t cvt_fp8x2(float lo, float hi) {
    if constexpr (FMT == FMT_INT8) {
        int32_t a, b;
        asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(a) : "f"(__fmul_rn(lo, 64.0f)));
        asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(b) : "f"(__fmul_rn(hi, 64.0f)));
        a = max(a, -127);
        b = max(b, -127);
        return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8);
    } else {
        uint16_t r;
        if constexpr (FMT == FMT_E4M3)
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
        else if constexpr (FMT == FMT_E5M2)
            asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
        else if constexpr (FMT == FMT_E2M3)
            asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
        else
            asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
        return (uint32_t)r;
    }
}

// Eight fp32 -> eight E2M1 codes in one 32-bit word (element i in nibble i).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&x)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
    return r;
}

// Eight fp32 -> eight FP8 codes (uint2, element i in byte i).
template <int FMT>
__device__ __forceinline__ uint2 cvt_fp8x8(const float (&x)[8]) {
    uint2 r;
    r.x = cvt_fp8x2<FMT>(x[0], x[1]) | (cvt_fp8x2<FMT>(x[2], x[3]) << 16);
    r.y = cvt_fp8x2<FMT>(x[4], x[5]) | (cvt_fp8x2<FMT>(x[6], x[7]) << 16);
    return r;
}

// Two byte codes (16-bit word, element 2i low) -> two fp32, exact (FP8 / FP6 via f16x2;
// INT8 as q / 64).
template <int FMT>
__device__ __forceinline__ void fp8x2_to_f32(uint32_t codes16, float &lo, float &hi) {
    if constexpr (FMT == FMT_INT8) {
        lo = __fmul_rn((float)(int8_t)(codes16 & 0xFFu), 0.015625f);
        hi = __fmul_rn((float)(int8_t)((codes16 >> 8) & 0xFFu), 0.015625f);
        return;
    }
    uint32_t h2;
    uint16_t c = (uint16_t)codes16;
    if constexpr (FMT == FMT_E4M3)
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    else if constexpr (FMT == FMT_E5M2)
        asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(c));
    else if constexpr (FMT == FMT_E2M3)
        asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    else
        asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h2) : "h"(c));
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h2));
}

// Eight E2M1 codes (nibble i = element i) -> four f16x2 words (element 2i low), exact.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(codes));
}

// f16x2 word -> two fp32 (low half in lo), exact.
__device__ __forceinline__ void f16x2_to_f32(uint32_t h2, float &lo, float &hi) {
    asm("{\n\t.reg .f16 l, hh;\n\tmov.b32 {l, hh}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, hh;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h2));
}

// Eight E2M1 codes (nibble i = element i) -> eight fp32, exact.
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t codes, float (&y)[8]) {
    uint32_t h[4];
    e2m1x8_to_f16x2(codes, h);
#pragma unroll
    for (int i = 0; i < 4; i++) f16x2_to_f32(h[i], y[2 * i], y[2 * i + 1]);
}

// Two fp32 -> bf16x2 word (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// UE4M3 code (0 .. 0x7E) -> fp32, exact (the NVFP4 block scale; [Q] §3 unsigned E4M3).
__device__ __forceinline__ float ue4m3_to_f32(uint32_t code) {
    float lo, hi;
    fp8x2_to_f32<FMT_E4M3>(code & 0x7Fu, lo, hi);
    return lo;
}


}  // namespace mxk
