// tiling.cuh -- index and packed-arithmetic helpers shared by the streaming and the
// TMA-staged quantisers: a host-computed divider, the tcgen05 scale-tile offset, packed
// fp32 pairs (sm_100a mul.rn.f32x2) and the packed bf16 block maximum.
#pragma once
#include <cstdint>

namespace mxk {

// ---- host-computed divider: q = n / d for n < 2^31 --------------------------------------
// m = ceil(2^(31+l) / d) with l = ceil(log2 d); then n / d = (n * m) >> (31 + l) for every
// n < 2^31 (the round-up error of m times n stays below one unit of the quotient).
struct FastDiv {
    uint32_t d, mul, shift;
};

inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f{d, 0u, 0u};
    if (d <= 1) return f;
    uint32_t l = 0;
    while ((1ull << l) < d) l++;                       // ceil(log2 d)
    const uint32_t p = 31 + l;
    f.mul = (uint32_t)(((1ull << p) + d - 1) / d);
    f.shift = p - 32;
    return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
    return f.d <= 1 ? n : (__umulhi(n, f.mul) >> f.shift);
}

// tcgen05 tiling offset of scale (r, c) with S scale columns (col_atoms = ceil(S/4)):
// 512-byte atoms of 128 rows x 4 scale columns, row-block major; inside an atom, row r
// sits at (r % 32) * 16 + ((r / 32) % 4) * 4 and column c at c % 4.
__device__ __forceinline__ uint32_t tc_offset(uint32_t r, uint32_t c, uint32_t col_atoms) {
    return (((r >> 7) * col_atoms + (c >> 2)) << 9) | ((r & 31u) << 4) | (((r >> 5) & 3u) << 2) | (c & 3u);
}

// ---- packed fp32 pairs (two IEEE round-to-nearest products per instruction) ---------------
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    return r;
}
__device__ __forceinline__ uint64_t splat2(float a) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(a));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ void unpack2(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// Eight bf16 (one uint4) times a scalar, as eight fp32 (element i in x[i]).
__device__ __forceinline__ void scale8(const uint4 &v, uint64_t s2, float (&x)[8]) {
    unpack2(mul2(bf16x2_to_f32x2(v.x), s2), x[0], x[1]);
    unpack2(mul2(bf16x2_to_f32x2(v.y), s2), x[2], x[3]);
    unpack2(mul2(bf16x2_to_f32x2(v.z), s2), x[4], x[5]);
    unpack2(mul2(bf16x2_to_f32x2(v.w), s2), x[6], x[7]);
}

// Eight bf16 (one uint4) divided by d, returned NEGATED: x[i] = -RN(v_i / d), the
// correctly rounded fp32 quotient, with nr2 = -RN(1/d) and d2 = d in both lanes.
// Markstein's FMA-corrected quotient (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with y = RN(1/d)
// and q = RN(v y), the remainder e = v - q d is exact in one FMA and RN(q + e y) is the
// IEEE quotient, provided no step underflows -- the caller guarantees d >= 2^-100 and
// needs the exact quotient only where it is >= 1/8, i.e. for |v| >= 2^-103.  Working with
// -q (q' = RN(-v y), e = RN(q' d + v), result RN(e (-y) + q')) keeps the sign of a zero v,
// which the positive form would lose in e; callers flip the sign back on the codes.
__device__ __forceinline__ void neg_quotient8(const uint4 &v, uint64_t nr2, uint64_t d2, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint64_t X = bf16x2_to_f32x2(w[i]);
        const uint64_t Q = mul2(X, nr2);
        const uint64_t E = fma2(Q, d2, X);
        unpack2(fma2(E, nr2, Q), x[2 * i], x[2 * i + 1]);
    }
}

// ---- packed bf16 block maximum ------------------------------------------------------------
// Per-half max(|a|, |b|) in one instruction.  The sign of each result half is the xor of
// the operands' signs (ignored: the caller masks it off at the end); a NaN in either
// operand gives the canonical NaN 0x7FFF, so a block holding a NaN ends with a magnitude
// >= 0x7F80 exactly as the integer maximum of |bits| would.  For all other values the
// order of magnitudes equals the order of the 15-bit |bits| patterns (subnormals kept).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

}  // namespace mxk
