// train.cu -- the training-side variant of the row-wise quantisers: an optional 16 x 16
// random Hadamard transform of the input and optional stochastic rounding of the element
// cast, for MXFP8 / MXFP4 (block 32, E8M0) and NVFP4 (block 16, UE4M3 + fp32 tensor scale).
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §4 "精度の差はどこから出るか": the 4-bit pre-training recipe applies a 16 x 16 random
//        Hadamard transform to the inputs of the weight gradient and rounds gradients
//        stochastically.
//     §8 "その後の標準化はどこへ向かっているか": stochastic rounding is among the rounding
//        modes P3109 defines.
//
// Transform: every 16 consecutive elements of a row become H16 D x / 4 (D: sign flips from
// a 16-bit mask, H16: the Sylvester Hadamard matrix), computed as the radix-2 butterfly
// (strides 1, 2, 4, 8) in fp32 round-to-nearest, then rounded to bf16; the quantiser then
// sees those bf16 values.  Stochastic rounding: with the element's random byte r (passed
// in, one per element), a value strictly between its two representable neighbours lo < |y|
// < hi rounds to hi when 256 (|y| - lo) > r (hi - lo), else to lo; |y| at or above the
// maximum saturates; the sign is kept.  Scales are computed exactly as in the RNE path.
// One thread per 32-element MX block or per two 16-element NVFP4 blocks (two transform
// groups either way), consecutive threads on adjacent blocks (coalesced), grid-stride
// loops; NVFP4 takes a maximum pass and a quantisation pass.
#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"
#include "nvfp4.cuh"
#include "ptx.cuh"
#include "tiling.cuh"

namespace mxk {

namespace {
constexpr int kTrainThreads = 256;
}  // namespace

// ---- 16 x 16 random Hadamard transform of 16 bf16 (two uint4, element order) ---------------
// D's sign flips as xor masks on the packed bf16 words (bit 15 / 31 of word i of the
// first or second uint4 flips element 2i / 2i + 1 of that half), computed once per thread.
struct RhtSigns {
    uint32_t w[8];
};
__device__ __forceinline__ RhtSigns rht_signs(uint32_t signs) {
    RhtSigns m;
#pragma unroll
    for (int i = 0; i < 8; i++)
        m.w[i] = (((signs >> (2 * i)) & 1u) << 15) | (((signs >> (2 * i + 1)) & 1u) << 31);
    return m;
}

__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The transform runs on two groups at once (a: one group's elements 0-7 and 8-15, b:
// another's): lane 0 of every packed fp32 pair holds group a, lane 1 group b, so all four
// butterfly stages (x_j, x_j+h) <- (x_j + x_j+h, x_j - x_j+h) for h = 1, 2, 4, 8 and the
// x 1/4 run as packed pairs, each lane with the scalar round-to-nearest of one group.
__device__ __forceinline__ void rht16x2_stages(const uint4 &a0, const uint4 &a1, const uint4 &b0, const uint4 &b1,
                                               const RhtSigns &sm, uint64_t (&Q)[16]) {
    const uint32_t wa[8] = {a0.x ^ sm.w[0], a0.y ^ sm.w[1], a0.z ^ sm.w[2], a0.w ^ sm.w[3],
                            a1.x ^ sm.w[4], a1.y ^ sm.w[5], a1.z ^ sm.w[6], a1.w ^ sm.w[7]};
    const uint32_t wb[8] = {b0.x ^ sm.w[0], b0.y ^ sm.w[1], b0.z ^ sm.w[2], b0.w ^ sm.w[3],
                            b1.x ^ sm.w[4], b1.y ^ sm.w[5], b1.z ^ sm.w[6], b1.w ^ sm.w[7]};
#pragma unroll
    for (int i = 0; i < 8; i++) {
        Q[2 * i] = pack2(bf16_lo(wa[i]), bf16_lo(wb[i]));
        Q[2 * i + 1] = pack2(bf16_hi(wa[i]), bf16_hi(wb[i]));
    }
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
        for (int j = 0; j < 16; j++)
            if ((j & h) == 0) {
                const uint64_t t = Q[j];
                Q[j] = add2(t, Q[j + h]);
                Q[j + h] = sub2(t, Q[j + h]);
            }
}

__device__ __forceinline__ void rht16x2(uint4 &a0, uint4 &a1, uint4 &b0, uint4 &b1, const RhtSigns &sm) {
    uint64_t Q[16];
    rht16x2_stages(a0, a1, b0, b1, sm, Q);
    const uint64_t quarter = splat2(0.25f);
    float A[16], B[16];
#pragma unroll
    for (int j = 0; j < 16; j++) unpack2(mul2(Q[j], quarter), A[j], B[j]);
    a0 = make_uint4(f32x2_to_bf16x2(A[0], A[1]), f32x2_to_bf16x2(A[2], A[3]), f32x2_to_bf16x2(A[4], A[5]),
                    f32x2_to_bf16x2(A[6], A[7]));
    a1 = make_uint4(f32x2_to_bf16x2(A[8], A[9]), f32x2_to_bf16x2(A[10], A[11]), f32x2_to_bf16x2(A[12], A[13]),
                    f32x2_to_bf16x2(A[14], A[15]));
    b0 = make_uint4(f32x2_to_bf16x2(B[0], B[1]), f32x2_to_bf16x2(B[2], B[3]), f32x2_to_bf16x2(B[4], B[5]),
                    f32x2_to_bf16x2(B[6], B[7]));
    b1 = make_uint4(f32x2_to_bf16x2(B[8], B[9]), f32x2_to_bf16x2(B[10], B[11]), f32x2_to_bf16x2(B[12], B[13]),
                    f32x2_to_bf16x2(B[14], B[15]));
}

// Largest finite |y| over the two groups' butterfly outputs y, before the x 1/4.  The
// transformed element is RN_bf16(y / 4): y / 4 is exact (y is a multiple of 2^-133, the
// bf16 spacing at the bottom, and cannot overflow), and for finite y it stays finite in
// bf16 (|y / 4| < 2^126).  Rounding is monotone, so the largest finite transformed
// magnitude is RN_bf16(m / 4) with m the value returned here; NaNs drop out of fmaxf, and
// an infinite y (an infinite input, or an fp32 overflow inside the butterfly) sends the
// group pair down the rare path that skips it.
__device__ __forceinline__ float rht16x2_absmax(const uint4 &a0, const uint4 &a1, const uint4 &b0, const uint4 &b1,
                                                const RhtSigns &sm) {
    uint64_t Q[16];
    rht16x2_stages(a0, a1, b0, b1, sm, Q);
    float y[32];
#pragma unroll
    for (int j = 0; j < 16; j++) unpack2(Q[j], y[2 * j], y[2 * j + 1]);
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; j++) m = fmaxf(m, fabsf(y[j]));
    if (__builtin_expect(m == __int_as_float(0x7F800000), 0)) {
        m = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; j++)
            if (fabsf(y[j]) != __int_as_float(0x7F800000)) m = fmaxf(m, fabsf(y[j]));
    }
    return m;
}

// ---- stochastic rounding onto the element grid ----------------------------------------------
// Rounds y to lo or hi, its representable neighbours, with random byte r; carry is
// 2^w - 1 - r 2^(w - 8) (see carry_term).  At or above the format's smallest normal 2^emin,
// the grid step of |y|'s binade is bit w = 23 - mbits of its fp32 pattern, so the w low bits
// L are |y| - lo in units of 2^-w grid steps, and 256 (|y| - lo) > r (hi - lo) reads
// L > r 2^(w - 8): exactly when L + carry carries into bit w.  Adding carry and clearing the
// w low bits gives lo or hi (a carry out of the mantissa steps into the next binade, as the
// grid does).  Below 2^emin the grid has the fixed subnormal step 2^(emin - mbits), which is
// also the step of the binade [2^emin, 2^(emin + 1)]: |y| + 2^emin rounded toward +infinity
// lands there, and rounding up to the next fp32 keeps the decision (L is then the ceiling
// of the exact distance, compared strictly against an integer); subtracting 2^emin is
// exact.  The sign is kept.  A result above the format's maximum (|y| at or above it rounds
// to the maximum or past it, up to the next power of two; Inf stays Inf) is brought to the
// maximum by the saturating conversion that every caller applies next.
template <int FMT> constexpr int kSrMbits = FMT == FMT_E4M3 ? 3 : (FMT == FMT_E5M2 ? 2 : 1);
template <int FMT> constexpr int kSrShift = 23 - kSrMbits<FMT> - 8;
template <int FMT>
__device__ __forceinline__ float sr_value(float y, uint32_t carry) {
    constexpr int emin = FMT == FMT_E4M3 ? -6 : (FMT == FMT_E5M2 ? -14 : 0);   // smallest normal exponent
    constexpr uint32_t low = (1u << (23 - kSrMbits<FMT>)) - 1u;
    constexpr float minnorm = emin >= 0 ? (float)(1 << emin) : 1.0f / (float)(1 << -emin);
    // s = 1 below 2^emin, else 0, from one saturating FMA on the FMA pipe (the integer and
    // compare steps of this routine fill the ALU pipe): (2^emin - |y|) 2^100 is at least
    // 2^(emin + 76) >= 1 whenever it is positive.  Adding and subtracting s 2^emin is exact
    // or, for the shift into the subnormal binade, the rounding toward +infinity.
    const float s = __saturatef(__fmaf_rn(-fabsf(y), 0x1p100f, minnorm * 0x1p100f));
    const float ap = __fmaf_ru(s, minnorm, fabsf(y));
    // the integer add written as a multiply-add (measured faster: the ALU pipe, not the
    // FMA pipe, holds these kernels)
    uint32_t t;
    asm("mad.lo.u32 %0, %1, 1, %2;" : "=r"(t) : "r"(carry), "r"(__float_as_uint(ap)));
    const float v = __fmaf_rn(-s, minnorm, __uint_as_float(t & ~low));
    return copysignf(v, y);
}

// The carry term 2^w - 1 - r 2^(w - 8) for the random byte r = byte K of word (w - 8 = SH):
// the byte by one permute, the rest by one integer multiply-add.
template <int SH, int K>
__device__ __forceinline__ uint32_t carry_term(uint32_t word) {
    const uint32_t r = __byte_perm(word, 0u, 0x4440u | K);
    uint32_t x;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(x) : "r"(r), "r"(0u - (1u << SH)), "r"((1u << (SH + 8)) - 1u));
    return x;
}

template <int FMT, bool SR>
__device__ __forceinline__ void round8(float (&x)[8], const uint8_t *rnd) {
    if constexpr (SR) {
        constexpr int sh = kSrShift<FMT>;
        const uint2 rb = *reinterpret_cast<const uint2 *>(rnd);
        x[0] = sr_value<FMT>(x[0], carry_term<sh, 0>(rb.x));
        x[1] = sr_value<FMT>(x[1], carry_term<sh, 1>(rb.x));
        x[2] = sr_value<FMT>(x[2], carry_term<sh, 2>(rb.x));
        x[3] = sr_value<FMT>(x[3], carry_term<sh, 3>(rb.x));
        x[4] = sr_value<FMT>(x[4], carry_term<sh, 0>(rb.y));
        x[5] = sr_value<FMT>(x[5], carry_term<sh, 1>(rb.y));
        x[6] = sr_value<FMT>(x[6], carry_term<sh, 2>(rb.y));
        x[7] = sr_value<FMT>(x[7], carry_term<sh, 3>(rb.y));
    }
}

// ---- row-wise MX with transform / stochastic rounding --------------------------------------
template <int FMT, bool CEIL, bool RM, bool TC, bool RHT, bool SR>
__global__ void __launch_bounds__(kTrainThreads)
mx_train_kernel(const uint8_t *__restrict__ src, uint32_t n_blocks, FastDiv divS, uint32_t col_atoms,
                uint32_t signs, const uint8_t *__restrict__ rnd, uint8_t *__restrict__ elems,
                uint8_t *__restrict__ sc_rm, uint8_t *__restrict__ sc_tc) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const RhtSigns sm = rht_signs(signs);
    for (uint32_t blk = blockIdx.x * kTrainThreads + threadIdx.x; blk < n_blocks; blk += gridDim.x * kTrainThreads) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src + (size_t)blk * 64);
        uint4 v[4] = {p[0], p[1], p[2], p[3]};
        if constexpr (RHT) rht16x2(v[0], v[1], v[2], v[3], sm);
        uint32_t a = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(v[0].x, v[0].y), absmax_bf16x2(v[0].z, v[0].w)),
                                   absmax_bf16x2(absmax_bf16x2(v[1].x, v[1].y), absmax_bf16x2(v[1].z, v[1].w)));
        a = absmax_bf16x2(a, absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(v[2].x, v[2].y), absmax_bf16x2(v[2].z, v[2].w)),
                                           absmax_bf16x2(absmax_bf16x2(v[3].x, v[3].y), absmax_bf16x2(v[3].z, v[3].w))));
        const uint32_t code = e8m0_from_amax_bits<FMT, CEIL>(max(a & 0x7FFFu, (a >> 16) & 0x7FFFu));
        const uint64_t mul2x = splat2(e8m0_inverse_multiplier(code));
        const bool nan_blk = code == 0xFFu;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            float x[8];
            scale8(v[j], mul2x, x);
            round8<FMT, SR>(x, rnd + (size_t)blk * 32 + 8 * j);
            if constexpr (FMT == FMT_E2M1) {
                out_store(reinterpret_cast<uint32_t *>(elems) + (size_t)blk * 4 + j, nan_blk ? 0u : cvt_e2m1x8(x));
            } else {
                const uint2 q = cvt_fp8x8<FMT>(x);
                out_store(reinterpret_cast<uint2 *>(elems) + (size_t)blk * 4 + j, nan_blk ? make_uint2(0u, 0u) : q);
            }
        }
        if constexpr (RM) out_store(sc_rm + blk, (uint8_t)code);
        if constexpr (TC) {
            const uint32_t r = fdiv(blk, divS);
            out_store(sc_tc + tc_offset(r, blk - r * divS.d, col_atoms), (uint8_t)code);
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- NVFP4 with transform / stochastic rounding ---------------------------------------------
// Pass 1: per-CTA finite maximum of the (transformed) tensor.
template <bool RHT>
__global__ void __launch_bounds__(kTrainThreads)
nvfp4_train_amax_kernel(const uint8_t *__restrict__ src, uint32_t n_groups, uint32_t signs,
                        float *__restrict__ partials) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ uint32_t warp_u[kTrainThreads / 32];
    uint32_t acc = 0;       // without the transform: bf16 magnitude bits, two lanes
    float accf = 0.0f;      // with it: the largest finite butterfly output, before the x 1/4
    const RhtSigns sm = rht_signs(signs);
    // kUnroll groups per trip, all loads issued before the first transform
    constexpr uint32_t kUnroll = 2;
    const uint32_t stride = gridDim.x * kTrainThreads;
    uint32_t gi = blockIdx.x * kTrainThreads + threadIdx.x;
    for (; gi + (kUnroll - 1) * stride < n_groups; gi += kUnroll * stride) {
        uint4 v[kUnroll][2];
#pragma unroll
        for (uint32_t u = 0; u < kUnroll; u++) {
            const uint4 *p = reinterpret_cast<const uint4 *>(src + (size_t)(gi + u * stride) * 32);
            v[u][0] = p[0];
            v[u][1] = p[1];
        }
        if constexpr (RHT) {
#pragma unroll
            for (uint32_t u = 0; u < kUnroll; u += 2)
                accf = fmaxf(accf, rht16x2_absmax(v[u][0], v[u][1], v[u + 1][0], v[u + 1][1], sm));
        } else {
#pragma unroll
            for (uint32_t u = 0; u < kUnroll; u++) {
                acc = __vmaxu2(acc, finite_abs_max_bf16x8(v[u][0]));
                acc = __vmaxu2(acc, finite_abs_max_bf16x8(v[u][1]));
            }
        }
    }
    for (; gi < n_groups; gi += stride) {
        const uint4 *p = reinterpret_cast<const uint4 *>(src + (size_t)gi * 32);
        const uint4 v0 = p[0], v1 = p[1];
        if constexpr (RHT) {
            accf = fmaxf(accf, rht16x2_absmax(v0, v1, v0, v1, sm));   // one group, in both lanes
        } else {
            acc = __vmaxu2(acc, finite_abs_max_bf16x8(v0));
            acc = __vmaxu2(acc, finite_abs_max_bf16x8(v1));
        }
    }
    uint32_t m;
    if constexpr (RHT) m = f32x2_to_bf16x2(__fmul_rn(accf, 0.25f), 0.0f) & 0xFFFFu;
    else m = max(acc & 0xFFFFu, acc >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) warp_u[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kTrainThreads / 32; w++) r = max(r, warp_u[w]);
        out_store(partials + blockIdx.x, __uint_as_float(r << 16));
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Pass 2: g from the partial maxima, then two consecutive 16-element blocks per thread (so
// the transform runs on both at once).  The block scale and the quotient follow the RNE
// path's fp32 steps (t = amax_b / (6 g) and RN(x / (dec(sb) g)), both correctly rounded,
// from the per-tensor constants and the per-code divisor table); the element cast is RNE or
// stochastic.
template <bool RM, bool TC, bool RHT, bool SR>
__global__ void __launch_bounds__(kTrainThreads)
nvfp4_train_quant_kernel(const uint8_t *__restrict__ src, uint32_t n_blocks, FastDiv divS, uint32_t col_atoms,
                         uint32_t signs, const uint8_t *__restrict__ rnd, const float *__restrict__ partials,
                         int n_partials, float *__restrict__ g_out, uint8_t *__restrict__ elems,
                         uint8_t *__restrict__ sc_rm, uint8_t *__restrict__ sc_tc) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float red[kTrainThreads / 32];
    __shared__ float2 qtab[128];
    float a = 0.0f;
    for (int i = threadIdx.x; i < n_partials; i += kTrainThreads) a = fmaxf(a, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    a = 0.0f;
    for (int w = 0; w < kTrainThreads / 32; w++) a = fmaxf(a, red[w]);
    const float g = a == 0.0f ? 1.0f : __fdiv_rn(a, 2688.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) out_store(g_out, g);
    const Nvfp4Consts cst = nvfp4_consts(g, qtab);
    const RhtSigns sm = rht_signs(signs);
    const uint32_t n_pairs = (n_blocks + 1) / 2;
    for (uint32_t pi = blockIdx.x * kTrainThreads + threadIdx.x; pi < n_pairs; pi += gridDim.x * kTrainThreads) {
        const uint32_t blk0 = 2 * pi;
        const bool two = blk0 + 1 < n_blocks;
        const uint4 *p = reinterpret_cast<const uint4 *>(src + (size_t)blk0 * 32);
        uint4 v[4];
        v[0] = p[0];
        v[1] = p[1];
        v[2] = two ? p[2] : v[0];
        v[3] = two ? p[3] : v[1];
        if constexpr (RHT) rht16x2(v[0], v[1], v[2], v[3], sm);
        uint32_t q[4], sbs[2];
#pragma unroll
        for (int b = 0; b < 2; b++) {
            const uint4 &v0 = v[2 * b], &v1 = v[2 * b + 1];
            const uint32_t am = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(v0.x, v0.y), absmax_bf16x2(v0.z, v0.w)),
                                              absmax_bf16x2(absmax_bf16x2(v1.x, v1.y), absmax_bf16x2(v1.z, v1.w)));
            const uint32_t m = max(am & 0x7FFFu, (am >> 16) & 0x7FFFu);
            const bool special = m >= 0x7F80u;
            const float tq = cst.fast ? nvfp4_block_quotient<true>(__uint_as_float(m << 16), cst)
                                      : nvfp4_block_quotient<false>(__uint_as_float(m << 16), cst);
            uint32_t sb = cvt_fp8x2<FMT_E4M3>(tq, 0.0f) & 0x7Fu;
            const float2 dn = qtab[sb];
            const float d = special ? 0.0f : dn.x;
            if (special) sb = 0x7Fu;
            // the quotients arrive negated; stochastic rounding is odd-symmetric, so it
            // commutes with the sign flip applied to the codes
            const uint8_t *rb = rnd + (size_t)(blk0 + b) * 16;
            nvfp4_codes16(v0, v1, d, dn.y, q[2 * b], q[2 * b + 1],
                          [&](float (&x)[8], int j) { round8<FMT_E2M1, SR>(x, rb + 8 * j); });
            if (special || d == 0.0f) q[2 * b] = q[2 * b + 1] = 0u;
            sbs[b] = sb;
        }
        if (two) {
            out_store(reinterpret_cast<uint4 *>(elems) + pi, make_uint4(q[0], q[1], q[2], q[3]));
        } else {
            out_store(reinterpret_cast<uint2 *>(elems) + blk0, make_uint2(q[0], q[1]));
        }
#pragma unroll
        for (int b = 0; b < 2; b++) {
            if (b == 1 && !two) break;
            const uint32_t blk = blk0 + b;
            if constexpr (RM) out_store(sc_rm + blk, (uint8_t)sbs[b]);
            if constexpr (TC) {
                const uint32_t rr = fdiv(blk, divS);
                out_store(sc_tc + tc_offset(rr, blk - rr * divS.d, col_atoms), (uint8_t)sbs[b]);
            }
        }
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- launchers ---------------------------------------------------------------------------
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTrainThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Grid of the quantisation kernels: up to 8 CTAs per SM (more than fit at once at their
// register counts; measured faster on the 16384 x 14336 gradient than one resident wave).
static int train_grid(uint64_t items, int num_sms) {
    uint64_t g = (items + kTrainThreads - 1) / kTrainThreads;
    const uint64_t cap = (uint64_t)num_sms * 8;
    if (g > cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

// Grid of the NVFP4 maximum pass: one wave of the CTAs that fit on the SMs at once (the
// kernel's registers set that), fewer when there are fewer items than threads.
template <auto Kernel>
static int resident_grid(uint64_t items, int num_sms) {
    static const int per_sm = [] {
        int n = 0;
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, kTrainThreads, 0) == cudaSuccess && n > 0 ? n
                                                                                                                 : 1;
    }();
    uint64_t g = (items + kTrainThreads - 1) / kTrainThreads;
    const uint64_t cap = (uint64_t)num_sms * (uint64_t)per_sm;
    if (g > cap) g = cap;
    return g < 1 ? 1 : (int)g;
}

template <int FMT, bool CEIL, bool RHT, bool SR>
static cudaError_t launch_mx_train_t(const uint8_t *src, uint32_t nb, FastDiv f, uint32_t ca, uint32_t signs,
                                     const uint8_t *rnd, uint8_t *e, uint8_t *rm, uint8_t *tc, int num_sms,
                                     cudaStream_t st) {
    if (rm && tc)
        return launch_pdl(mx_train_kernel<FMT, CEIL, true, true, RHT, SR>, train_grid(nb, num_sms), st, src, nb, f, ca, signs, rnd, e, rm, tc);
    if (rm)
        return launch_pdl(mx_train_kernel<FMT, CEIL, true, false, RHT, SR>, train_grid(nb, num_sms), st, src, nb, f, ca, signs, rnd, e, rm, tc);
    return launch_pdl(mx_train_kernel<FMT, CEIL, false, true, RHT, SR>, train_grid(nb, num_sms), st, src, nb, f, ca, signs, rnd, e, rm, tc);
}

template <int FMT, bool CEIL>
static cudaError_t launch_mx_train_f(bool rht, bool sr, const uint8_t *src, uint32_t nb, FastDiv f, uint32_t ca,
                                     uint32_t signs, const uint8_t *rnd, uint8_t *e, uint8_t *rm, uint8_t *tc,
                                     int num_sms, cudaStream_t st) {
    if (rht && sr) return launch_mx_train_t<FMT, CEIL, true, true>(src, nb, f, ca, signs, rnd, e, rm, tc, num_sms, st);
    if (rht) return launch_mx_train_t<FMT, CEIL, true, false>(src, nb, f, ca, signs, rnd, e, rm, tc, num_sms, st);
    if (sr) return launch_mx_train_t<FMT, CEIL, false, true>(src, nb, f, ca, signs, rnd, e, rm, tc, num_sms, st);
    return launch_mx_train_t<FMT, CEIL, false, false>(src, nb, f, ca, signs, rnd, e, rm, tc, num_sms, st);
}

template <bool RHT, bool SR>
static cudaError_t launch_nvfp4_train_t(const uint8_t *src, uint32_t nb, FastDiv f, uint32_t ca, uint32_t signs,
                                        const uint8_t *rnd, float *partials, int max_partials, float *g, uint8_t *e,
                                        uint8_t *rm, uint8_t *tc, int num_sms, cudaStream_t st) {
    int grid1 = resident_grid<nvfp4_train_amax_kernel<RHT>>(nb, num_sms);
    if (grid1 > max_partials) grid1 = max_partials;
    cudaError_t err = launch_pdl(nvfp4_train_amax_kernel<RHT>, grid1, st, src, nb, signs, partials);
    if (err != cudaSuccess) return err;
    const int grid2 = train_grid((nb + 1) / 2, num_sms);
    const float *cp = partials;
    if (rm && tc)
        return launch_pdl(nvfp4_train_quant_kernel<true, true, RHT, SR>, grid2, st, src, nb, f, ca, signs, rnd, cp, grid1,
                          g, e, rm, tc);
    if (rm)
        return launch_pdl(nvfp4_train_quant_kernel<true, false, RHT, SR>, grid2, st, src, nb, f, ca, signs, rnd, cp, grid1,
                          g, e, rm, tc);
    return launch_pdl(nvfp4_train_quant_kernel<false, true, RHT, SR>, grid2, st, src, nb, f, ca, signs, rnd, cp, grid1,
                          g, e, rm, tc);
}

cudaError_t launch_quantize_train(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil, bool rht,
                                  uint32_t signs, const uint8_t *rnd, float *partials, int max_partials, float *g,
                                  void *elems, uint8_t *rm, uint8_t *tc, int num_sms, cudaStream_t st) {
    const uint8_t *s8 = static_cast<const uint8_t *>(src);
    uint8_t *e8 = static_cast<uint8_t *>(elems);
    const bool sr = rnd != nullptr;
    {
        const int64_t B = fmt == FMT_NVFP4 ? 16 : 32, S = cols / B;
        const OutRange out[5] = {{elems, (uint64_t)(rows * cols * code_bits(fmt) / 8)}, {rm, (uint64_t)(rows * S)},
                                 {tc, (uint64_t)((rows + 127) / 128) * ((S + 3) / 4) * 512}, {g, 4},
                                 {partials, (uint64_t)max_partials * 4}};
        const cudaError_t e = set_out_ranges(out, st);
        if (e != cudaSuccess) return e;
    }
    if (fmt == FMT_NVFP4) {
        const uint32_t nb = (uint32_t)(rows * cols / 16), S = (uint32_t)(cols / 16);
        const FastDiv f = make_fastdiv(S);
        const uint32_t ca = (S + 3) / 4;
        if (rht && sr) return launch_nvfp4_train_t<true, true>(s8, nb, f, ca, signs, rnd, partials, max_partials, g, e8, rm, tc, num_sms, st);
        if (rht) return launch_nvfp4_train_t<true, false>(s8, nb, f, ca, signs, rnd, partials, max_partials, g, e8, rm, tc, num_sms, st);
        if (sr) return launch_nvfp4_train_t<false, true>(s8, nb, f, ca, signs, rnd, partials, max_partials, g, e8, rm, tc, num_sms, st);
        return launch_nvfp4_train_t<false, false>(s8, nb, f, ca, signs, rnd, partials, max_partials, g, e8, rm, tc, num_sms, st);
    }
    const uint32_t nb = (uint32_t)(rows * cols / 32), S = (uint32_t)(cols / 32);
    const FastDiv f = make_fastdiv(S);
    const uint32_t ca = (S + 3) / 4;
    switch (fmt * 2 + (ceil ? 1 : 0)) {
    case FMT_E4M3 * 2 + 0: return launch_mx_train_f<FMT_E4M3, false>(rht, sr, s8, nb, f, ca, signs, rnd, e8, rm, tc, num_sms, st);
    case FMT_E4M3 * 2 + 1: return launch_mx_train_f<FMT_E4M3, true>(rht, sr, s8, nb, f, ca, signs, rnd, e8, rm, tc, num_sms, st);
    case FMT_E5M2 * 2 + 0: return launch_mx_train_f<FMT_E5M2, false>(rht, sr, s8, nb, f, ca, signs, rnd, e8, rm, tc, num_sms, st);
    case FMT_E5M2 * 2 + 1: return launch_mx_train_f<FMT_E5M2, true>(rht, sr, s8, nb, f, ca, signs, rnd, e8, rm, tc, num_sms, st);
    case FMT_E2M1 * 2 + 0: return launch_mx_train_f<FMT_E2M1, false>(rht, sr, s8, nb, f, ca, signs, rnd, e8, rm, tc, num_sms, st);
    case FMT_E2M1 * 2 + 1: return launch_mx_train_f<FMT_E2M1, true>(rht, sr, s8, nb, f, ca, signs, rnd, e8, rm, tc, num_sms, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace mxk
