// nested.cu -- MXFP4 (1 x 32 E2M1 tiles, E8M0 scales) re-expressed as FP8 E4M3 with one
// power-of-two scale per 128 x 128 block.
//
// Source (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §6 "DeepSeek-V4 の入れ子構造": FP8 training keeps 128 x 128 block scaling; each such
//        block holds 4 x 128 = 512 MXFP4 1 x 32 tiles, and the FP4 -> FP8 dequantisation is
//        lossless while the ratio of the largest to the smallest tile scale in a block stays
//        under a bound (E4M3's two extra exponent bits absorb the fine-grained scales).
//
// Per 128 x 128 block: s_max = largest tile exponent among tiles that are finite and hold
// a nonzero code; block scale S = 2^(s_max - 6) (the largest FP4 value 6 * 2^s_max lands
// on 384, inside E4M3); each element becomes the RNE-saturating E4M3 code of
// dec(q) * 2^(s_tile - s_max + 6); the block is flagged exact when every element decodes
// back to its FP4 value (a tile scale at most 14 binades below s_max always is).  NaN tiles
// give E4M3 NaN codes.  One CTA per block, one thread per 64-element half row (two tiles).
//
// Exactness without a round trip: with d = s_tile - s_max + 6 <= 6 a nonzero product
// v * 2^d (v = k / 2, k in {1, 2, 3, 4, 6, 8, 12}) stays within 384, so it is an E4M3
// value iff it is a multiple of E4M3's smallest subnormal 2^-9, i.e. iff d + 8 + tz(k) >= 0
// (tz: trailing zero bits).  Every code is therefore exact for d >= -8; at d = -9 the
// magnitudes 0.5 and 1.5 (E2M1 magnitude codes 1, 3) fail, at -10 also 1 and 3 (codes 2,
// 5), at -11 everything but 4 (code 6), and below -11 every nonzero code.  Those sets are
// tested on the packed codes with bit operations (b0, b1, b2: the magnitude bits of every
// nibble).
#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"

namespace mxk {

namespace {
constexpr int kNestThreads = 256;
constexpr int kNoScale = -100000;
}  // namespace

// Whether the 32 codes of a tile (four words) all survive the move to the E4M3 grid at
// exponent offset d (rule above).
__device__ __forceinline__ bool tile_exact(int d, const uint32_t *w) {
    if (d >= -8) return true;
    uint32_t bad = 0u;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const uint32_t b0 = w[k] & 0x11111111u, b1 = (w[k] >> 1) & 0x11111111u, b2 = (w[k] >> 2) & 0x11111111u;
        uint32_t f;
        if (d == -9) f = b0 & ~b2;                                        // magnitudes 1, 3
        else if (d == -10) f = (~b2 & (b0 | b1)) | (b2 & b0 & ~b1);      // 1, 2, 3, 5
        else if (d == -11) f = (b0 | b1 | b2) & ~(~b0 & b1 & b2);         // all nonzero but 6
        else f = b0 | b1 | b2;                                            // every nonzero code
        bad |= f;
    }
    return bad == 0u;
}

// WIDE (codes and output 32-byte aligned, scales 2-byte aligned): each thread's 32 bytes of
// codes in one 256-bit load, its two tile scales in one 16-bit load and its 64 output codes
// in two 256-bit stores, halving the load / store instructions of the narrow form.
template <bool WIDE>
__global__ void __launch_bounds__(kNestThreads)
mxfp4_to_fp8_blocks_kernel(const uint8_t *__restrict__ elems, const uint8_t *__restrict__ scales, int64_t cols,
                           uint32_t blocks_c, uint8_t *__restrict__ out, float *__restrict__ block_scale,
                           uint8_t *__restrict__ block_exact) {
    __shared__ __align__(16) int warp_max[kNestThreads / 32];
    static_assert(kNestThreads / 32 == 8, "the block maximum reads the eight warp maxima as two int4");
    const uint32_t blk = blockIdx.x;
    const uint32_t br = blk / blocks_c, bc = blk - br * blocks_c;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t R = (int64_t)br * 128 + (tid >> 1);           // this thread's row
    const int64_t c0 = (int64_t)bc * 128 + 64 * (tid & 1);      // its first column (two tiles)
    const int64_t S = cols / 32;

    // 64 packed E2M1 codes (32 bytes) and the two tile scales
    uint32_t w[8], sc[2];
    if constexpr (WIDE) {
        asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                     : "l"(elems + ((R * cols + c0) >> 1)));
        const uint32_t s2 = *reinterpret_cast<const uint16_t *>(scales + R * S + (c0 >> 5));
        sc[0] = s2 & 0xFFu;
        sc[1] = s2 >> 8;
    } else {
        const uint4 *src = reinterpret_cast<const uint4 *>(elems + ((R * cols + c0) >> 1));
        const uint4 p0 = src[0], p1 = src[1];
        w[0] = p0.x, w[1] = p0.y, w[2] = p0.z, w[3] = p0.w, w[4] = p1.x, w[5] = p1.y, w[6] = p1.z, w[7] = p1.w;
        sc[0] = scales[R * S + (c0 >> 5)];
        sc[1] = scales[R * S + (c0 >> 5) + 1];
    }

    // largest exponent among finite tiles holding a nonzero code (E2M1 magnitude bits 0-2)
    int m = kNoScale;
#pragma unroll
    for (int t = 0; t < 2; t++) {
        const bool nonzero = ((w[4 * t] | w[4 * t + 1] | w[4 * t + 2] | w[4 * t + 3]) & 0x77777777u) != 0u;
        if (sc[t] != 0xFFu && nonzero) m = max(m, (int)sc[t] - 127);
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);                       // one redux instruction per warp
    if (lane == 0) warp_max[warp] = m;
    __syncthreads();
    const int4 wa = *reinterpret_cast<const int4 *>(&warp_max[0]), wb = *reinterpret_cast<const int4 *>(&warp_max[4]);
    int smax = max(max(max(wa.x, wa.y), max(wa.z, wa.w)), max(max(wb.x, wb.y), max(wb.z, wb.w)));
    if (smax == kNoScale) smax = 6;                               // no nonzero finite element: S = 1

    bool exact = true;
    uint32_t o[16];                                               // 64 E4M3 codes
#pragma unroll
    for (int t = 0; t < 2; t++) {
        const int d = (int)sc[t] - 127 - smax + 6;                // tile exponent relative to S
        exact = exact && (sc[t] == 0xFFu || tile_exact(d, &w[4 * t]));
        // 2^d as an f16 pair, exact for -24 <= d <= 6 (f16 subnormals below 2^-14); 0 below
        // 2^-24, where every product (at most 6 * 2^-25) encodes to E4M3 zero anyway; capped
        // at 2^6, which larger d reach only for tiles whose codes are all zero.  An E2M1 value
        // has at most 2 significant bits, so every product that can encode to a nonzero E4M3
        // code (>= 2^-10) is exact in f16, and the smaller ones encode to a zero of the same
        // sign through f16 as through fp32: the codes are the fp32 path's, with one packed
        // f16 product and one packed conversion per element pair.
        const int dh = d > 6 ? 6 : d;
        const uint32_t fb = dh >= -14 ? (uint32_t)(dh + 15) << 10 : (dh >= -24 ? 1u << (dh + 24) : 0u);
        const uint32_t f2 = fb | (fb << 16);
#pragma unroll
        for (int k = 0; k < 4; k++) {                             // 8 codes per word
            uint32_t h[4], c[4];
            e2m1x8_to_f16x2(w[4 * t + k], h);
#pragma unroll
            for (int i = 0; i < 4; i++) {
                uint32_t p;
                uint16_t q2;
                asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(h[i]), "r"(f2));
                asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(q2) : "r"(p));
                c[i] = q2;
            }
            o[8 * t + 2 * k] = sc[t] == 0xFFu ? 0x7F7F7F7Fu : (c[0] | (c[1] << 16));    // NaN tile: E4M3 NaN
            o[8 * t + 2 * k + 1] = sc[t] == 0xFFu ? 0x7F7F7F7Fu : (c[2] | (c[3] << 16));
        }
    }
    if constexpr (WIDE) {
#pragma unroll
        for (int i = 0; i < 2; i++) {
            uint8_t *p = out + R * cols + c0 + 32 * i;
            if (out_ok(p, 32))
                asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                             ::"l"(p), "r"(o[8 * i]), "r"(o[8 * i + 1]), "r"(o[8 * i + 2]), "r"(o[8 * i + 3]),
                             "r"(o[8 * i + 4]), "r"(o[8 * i + 5]), "r"(o[8 * i + 6]), "r"(o[8 * i + 7])
                             : "memory");
        }
    } else {
        uint4 *dst = reinterpret_cast<uint4 *>(out + R * cols + c0);
#pragma unroll
        for (int i = 0; i < 4; i++) out_store(dst + i, make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
    }
    const int all_exact = __syncthreads_and(exact ? 1 : 0);
    if (tid == 0) {
        const int e = smax - 6;                                   // S = 2^e, e in [-133, 121]
        out_store(block_scale + blk,
                  e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << (e + 149)));
        out_store(block_exact + blk, (uint8_t)all_exact);
    }
}

cudaError_t launch_mxfp4_to_fp8_blocks(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                                       void *out, float *block_scale, uint8_t *block_exact, cudaStream_t st) {
    const int64_t n_blocks = (rows / 128) * (cols / 128);
    if (n_blocks <= 0) return cudaSuccess;
    if (n_blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const OutRange rng[3] = {{out, (uint64_t)(rows * cols)}, {block_scale, (uint64_t)n_blocks * 4},
                             {block_exact, (uint64_t)n_blocks}};
    const cudaError_t e = set_out_ranges(rng, st);
    if (e != cudaSuccess) return e;
    const bool wide = ((reinterpret_cast<uintptr_t>(elems) | reinterpret_cast<uintptr_t>(out)) & 31u) == 0 &&
                      (reinterpret_cast<uintptr_t>(scales) & 1u) == 0;
    auto k = wide ? mxfp4_to_fp8_blocks_kernel<true> : mxfp4_to_fp8_blocks_kernel<false>;
    k<<<(unsigned)n_blocks, kNestThreads, 0, st>>>(static_cast<const uint8_t *>(elems), scales, cols,
                                                    (uint32_t)(cols / 128), static_cast<uint8_t *>(out), block_scale,
                                                    block_exact);
    return cudaGetLastError();
}

}  // namespace mxk
