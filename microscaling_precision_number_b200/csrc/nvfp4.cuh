// nvfp4.cuh -- the NVFP4 element step shared by the streaming, 2-D and training
// quantisers: E2M1 codes of x / d, d = dec(sb) g the block's decode scale.
//
// Source: "MXFP4 と NVFP4 は何が違うのか調べてみた", §3 "NVFP4 はブロック16と E4M3、そして
// 二段目" (an element is x over the two-level scale, UE4M3 per 16 times the FP32 tensor
// scale).  The element is the round-to-nearest-even E2M1 code of the correctly rounded
// fp32 quotient RN(x / d).
#pragma once
#include <cstdint>

#include "codec.cuh"
#include "tiling.cuh"

namespace mxk {

// Smallest d for which the quotient takes Markstein's corrected form (neg_quotient8);
// below it the IEEE division is used.
constexpr float kQuotFastMin = 0x1p-100f;

// E2M1 codes of sixteen bf16 (v0: elements 0-7, v1: 8-15) divided by d, round to nearest
// even on the correctly rounded fp32 quotient RN(x / d), as two words (element i in nibble
// i of its word).  nr = -RN(1/d), or 0 when d < 2^-100 (IEEE division); d > 0.  The
// quotients are formed negated (see neg_quotient8) and the code signs flipped back.
// ROUND(x) may replace the quotients before the cast (stochastic rounding).
struct NoRound {
    __device__ __forceinline__ void operator()(float (&)[8], int) const {}
};
template <typename Round = NoRound>
__device__ __forceinline__ void nvfp4_codes16(const uint4 &v0, const uint4 &v1, float d, float nr, uint32_t &q0,
                                              uint32_t &q1, Round round = {}) {
    float x[2][8];
    if (__builtin_expect(nr != 0.0f, 1)) {
        const uint64_t nr2 = splat2(nr), d2 = splat2(d);
        neg_quotient8(v0, nr2, d2, x[0]);
        neg_quotient8(v1, nr2, d2, x[1]);
    } else {
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int i = 0; i < 8; i++) {
            x[i >> 2][2 * (i & 3)] = __fdiv_rn(-bf16_lo(w[i]), d);
            x[i >> 2][2 * (i & 3) + 1] = __fdiv_rn(-bf16_hi(w[i]), d);
        }
    }
    round(x[0], 0);
    round(x[1], 1);
    q0 = cvt_e2m1x8(x[0]) ^ 0x88888888u;
    q1 = cvt_e2m1x8(x[1]) ^ 0x88888888u;
}

// Per-tensor constants of the NVFP4 block math, derived once per CTA from g.
struct Nvfp4Consts {
    float six_g;      // 6 g (fp32 RN)
    float y;          // RN(1 / six_g)
    bool fast;        // six_g >= 2^-80: t = amax_b / six_g may use the corrected quotient
};

// Per-code element divisors: qtab[sb] = {d, -RN(1/d)} with d = RN(dec(sb) g).  The second
// entry is 0 when d < 2^-100 (the quotients then take the IEEE division) and the code 0x7F
// (only NaN blocks, whose codes are zero) gets {0, 0}.
__device__ __forceinline__ Nvfp4Consts nvfp4_consts(float g, float2 *qtab) {
    Nvfp4Consts c;
    c.six_g = __fmul_rn(6.0f, g);
    c.y = __frcp_rn(c.six_g);
    c.fast = c.six_g >= 0x1p-80f;
    if (threadIdx.x < 128) {
        const float d = threadIdx.x < 0x7Fu ? __fmul_rn(ue4m3_to_f32(threadIdx.x), g) : 0.0f;
        qtab[threadIdx.x] = make_float2(d, d >= kQuotFastMin ? -__frcp_rn(d) : 0.0f);
    }
    __syncthreads();
    return c;
}

// RN(amax_b / six_g): with FAST, Markstein's corrected quotient from the precomputed
// reciprocal (q0 = RN(a y), r = a - q0 six_g exact by FMA, t = RN(q0 + r y)).  It is the
// IEEE quotient for every numerator a >= 2^-100; with six_g >= 2^-80 every block whose
// quotient can reach the smallest UE4M3 subnormal has such a numerator, and smaller
// quotients encode to 0 either way.  Otherwise the IEEE division.
template <bool FAST>
__device__ __forceinline__ float nvfp4_block_quotient(float a, const Nvfp4Consts &cst) {
    if constexpr (FAST) {
        const float q0 = __fmul_rn(a, cst.y);
        return __fmaf_rn(__fmaf_rn(-q0, cst.six_g, a), cst.y, q0);
    } else {
        return __fdiv_rn(a, cst.six_g);
    }
}

}  // namespace mxk
