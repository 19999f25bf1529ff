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

}  // namespace mxk
