// quant.cu -- streaming (HBM-bound) kernels: row-wise MX quantiser, NVFP4 quantiser,
// direct cast, dequantisers, tcgen05 scale padding.
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §2 "MXFP4 はブロック32と E8M0": one E8M0 scale per 32 contiguous elements; NaN scale
//        = whole block NaN; RNE cast.
//     §3 "NVFP4 はブロック16と E4M3、そして二段目": 16-element blocks, unsigned E4M3 block
//        scale, FP32 tensor scale = tensor amax / (6 * 448).
//     §4 "精度の差はどこから出るか": floor and no-clip shared-exponent rules.
//     §7 "ハードウェアの対応状況": MX scale application is an exponent add (exact);
//        NVFP4 applies an FP8 then an FP32 multiply.
//   gpt-oss MXFP4 explainer, section "MXFP4": the direct cast (no scale).
//
// Layout of work: a "chunk" is 16 bytes of bf16 input (8 elements).  Four consecutive
// lanes hold one 32-element MX block (two lanes one 16-element NVFP4 block); the block
// maximum is reduced with xor shuffles.  Every load is a coalesced 16-byte vector load
// and every code store is a contiguous 8-byte (FP8) or 4-byte (FP4) vector store, so a
// warp moves 512 contiguous input bytes per load instruction.  Grids are a multiple of
// the SM count and each thread keeps kUnroll independent loads in flight.
#include "codec.cuh"
#include "internal.h"

namespace mxk {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }

static int grid_for(int64_t n_chunks, int num_sms, int per_sm = 8) {
    int64_t want = (n_chunks + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
    int64_t cap = (int64_t)num_sms * per_sm;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    return (int)want;
}

// ---------------------------------------------------------------------------------------
// Row-wise MX quantiser: E4M3 / E5M2 / E2M1, floor or no-clip scale rule.
// ---------------------------------------------------------------------------------------
template <int FMT, bool CEIL, bool RM, bool TC>
__global__ void __launch_bounds__(kThreads)
quant_rows_mx_kernel(const uint4 *__restrict__ src, int64_t n_chunks, int64_t scale_cols,
                     uint8_t *__restrict__ elems, uint8_t *__restrict__ sc_rm,
                     uint8_t *__restrict__ sc_tc) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t warp0 = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31);
    for (int64_t base = warp0; base < n_chunks; base += stride * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
            const int64_t c = base + u * stride + lane;
            v[u] = c < n_chunks ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
            const int64_t c = base + u * stride + lane;
            uint32_t m = hmax(abs_max_bf16x8(v[u]));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if (c >= n_chunks) continue;
            const uint32_t code = e8m0_from_amax_bits<FMT, CEIL>(m);
            const float mul = e8m0_inverse_multiplier(code);
            float x[8];
            x[0] = __fmul_rn(bf16_lo(v[u].x), mul); x[1] = __fmul_rn(bf16_hi(v[u].x), mul);
            x[2] = __fmul_rn(bf16_lo(v[u].y), mul); x[3] = __fmul_rn(bf16_hi(v[u].y), mul);
            x[4] = __fmul_rn(bf16_lo(v[u].z), mul); x[5] = __fmul_rn(bf16_hi(v[u].z), mul);
            x[6] = __fmul_rn(bf16_lo(v[u].w), mul); x[7] = __fmul_rn(bf16_hi(v[u].w), mul);
            if constexpr (FMT == FMT_E2M1) {
                uint32_t q = cvt_e2m1x8(x);
                if (code == 0xFFu) q = 0u;
                reinterpret_cast<uint32_t *>(elems)[c] = q;
            } else {
                uint2 q = cvt_fp8x8<FMT>(x);
                if (code == 0xFFu) q = make_uint2(0u, 0u);
                reinterpret_cast<uint2 *>(elems)[c] = q;
            }
            if ((lane & 3) == 0) {
                const int64_t blk = c >> 2;
                if constexpr (RM) sc_rm[blk] = (uint8_t)code;
                if constexpr (TC) {
                    const int64_t r = blk / scale_cols;
                    sc_tc[tcgen05_scale_offset(r, blk - r * scale_cols, scale_cols)] = (uint8_t)code;
                }
            }
        }
    }
}

template <int FMT, bool CEIL>
static cudaError_t quant_rows_dispatch_layout(const void *src, int64_t n_chunks, int64_t S,
                                              void *elems, uint8_t *rm, uint8_t *tc, int grid,
                                              cudaStream_t st) {
    const uint4 *s = static_cast<const uint4 *>(src);
    uint8_t *e = static_cast<uint8_t *>(elems);
    if (rm && tc)
        quant_rows_mx_kernel<FMT, CEIL, true, true><<<grid, kThreads, 0, st>>>(s, n_chunks, S, e, rm, tc);
    else if (rm)
        quant_rows_mx_kernel<FMT, CEIL, true, false><<<grid, kThreads, 0, st>>>(s, n_chunks, S, e, rm, tc);
    else
        quant_rows_mx_kernel<FMT, CEIL, false, true><<<grid, kThreads, 0, st>>>(s, n_chunks, S, e, rm, tc);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows_mx(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil,
                                 void *elems, uint8_t *rm, uint8_t *tc, int num_sms,
                                 cudaStream_t st) {
    const int64_t n_chunks = rows * cols / 8, S = cols / 32;
    const int grid = grid_for(n_chunks, num_sms);
    switch (fmt * 2 + (ceil ? 1 : 0)) {
    case FMT_E4M3 * 2 + 0: return quant_rows_dispatch_layout<FMT_E4M3, false>(src, n_chunks, S, elems, rm, tc, grid, st);
    case FMT_E4M3 * 2 + 1: return quant_rows_dispatch_layout<FMT_E4M3, true>(src, n_chunks, S, elems, rm, tc, grid, st);
    case FMT_E5M2 * 2 + 0: return quant_rows_dispatch_layout<FMT_E5M2, false>(src, n_chunks, S, elems, rm, tc, grid, st);
    case FMT_E5M2 * 2 + 1: return quant_rows_dispatch_layout<FMT_E5M2, true>(src, n_chunks, S, elems, rm, tc, grid, st);
    case FMT_E2M1 * 2 + 0: return quant_rows_dispatch_layout<FMT_E2M1, false>(src, n_chunks, S, elems, rm, tc, grid, st);
    case FMT_E2M1 * 2 + 1: return quant_rows_dispatch_layout<FMT_E2M1, true>(src, n_chunks, S, elems, rm, tc, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------------------------------
// tcgen05 tiling pad: write 0 to every byte of the padded buffer that holds no scale.
// ---------------------------------------------------------------------------------------
__global__ void tcgen05_pad_kernel(uint8_t *__restrict__ sc, int64_t rows, int64_t S, int64_t total) {
    const int64_t col_atoms = (S + 3) >> 2;
    for (int64_t off = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; off < total;
         off += (int64_t)gridDim.x * blockDim.x) {
        const int64_t atom = off >> 9;
        const int w = (int)(off & 511);
        const int64_t rb = atom / col_atoms, cb = atom - rb * col_atoms;
        const int64_t r = rb * 128 + (w >> 4) + ((w >> 2) & 3) * 32;
        const int64_t c = cb * 4 + (w & 3);
        if (r >= rows || c >= S) sc[off] = 0;
    }
}

cudaError_t launch_tcgen05_pad(uint8_t *sc, int64_t rows, int64_t S, cudaStream_t st) {
    if (rows % 128 == 0 && S % 4 == 0) return cudaSuccess;   // no padding bytes
    const int64_t total = ((rows + 127) / 128) * ((S + 3) / 4) * 512;
    int64_t grid = (total + 255) / 256;
    if (grid > 4096) grid = 4096;
    tcgen05_pad_kernel<<<(int)grid, 256, 0, st>>>(sc, rows, S, total);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// NVFP4 pass 1: finite |x| maximum per CTA.
// ---------------------------------------------------------------------------------------
int nvfp4_partials_count(int64_t n, int num_sms) { return grid_for(n / 8, num_sms, 4); }

__global__ void __launch_bounds__(kThreads)
nvfp4_amax_kernel(const uint4 *__restrict__ src, int64_t n_chunks, float *__restrict__ partials) {
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    uint32_t m = 0;
    for (int64_t base = (int64_t)blockIdx.x * kThreads + threadIdx.x; base < n_chunks;
         base += stride * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
            const int64_t c = base + u * stride;
            v[u] = c < n_chunks ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; u++) m = __vmaxu2(m, finite_abs_max_bf16x8(v[u]));
    }
    m = hmax(m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ uint32_t warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kThreads / 32; w++) r = max(r, warp_max[w]);
        partials[blockIdx.x] = __uint_as_float(r << 16);
    }
}

cudaError_t launch_nvfp4_amax(const void *src, int64_t n, float *partials, int n_partials,
                              cudaStream_t st) {
    nvfp4_amax_kernel<<<n_partials, kThreads, 0, st>>>(static_cast<const uint4 *>(src), n / 8, partials);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// NVFP4 pass 2.  Every CTA reduces the partial maxima itself (same order, same value),
// so no grid-wide synchronisation or atomics are needed; CTA 0 publishes g.
//   g = amax_t / 2688 (1 if amax_t = 0);  per 16-block: t = amax_b / (6 g),
//   sb = UE4M3(t) (RNE, saturating), d = dec(sb) g, q = E2M1(x * (1/d)).
// ---------------------------------------------------------------------------------------
template <bool RM, bool TC>
__global__ void __launch_bounds__(kThreads)
nvfp4_quant_kernel(const uint4 *__restrict__ src, int64_t n_chunks, int64_t scale_cols,
                   const float *__restrict__ partials, int n_partials, float *__restrict__ g_out,
                   uint8_t *__restrict__ elems, uint8_t *__restrict__ sc_rm,
                   uint8_t *__restrict__ sc_tc) {
    __shared__ float warp_max[kThreads / 32];
    float a = 0.0f;
    for (int i = threadIdx.x; i < n_partials; i += kThreads) a = fmaxf(a, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
    __syncthreads();
    a = 0.0f;
    for (int w = 0; w < kThreads / 32; w++) a = fmaxf(a, warp_max[w]);
    const float g = a == 0.0f ? 1.0f : __fdiv_rn(a, 2688.0f);
    const float six_g = __fmul_rn(6.0f, g);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;

    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t warp0 = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31);
    for (int64_t base = warp0; base < n_chunks; base += stride * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
            const int64_t c = base + u * stride + lane;
            v[u] = c < n_chunks ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; u++) {
            const int64_t c = base + u * stride + lane;
            uint32_t m = hmax(abs_max_bf16x8(v[u]));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            if (c >= n_chunks) continue;
            uint32_t sb, q = 0u;
            if (m >= 0x7F80u) {
                sb = 0x7Fu;                                   // UE4M3 NaN: block is NaN
            } else {
                const float t = __fdiv_rn(__uint_as_float(m << 16), six_g);
                sb = cvt_fp8x2<FMT_E4M3>(t, 0.0f) & 0xFFu;    // t >= 0: sign bit stays 0
                const float d = __fmul_rn(ue4m3_to_f32(sb), g);
                if (d != 0.0f) {
                    const float r = __frcp_rn(d);
                    const float in[8] = {bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y), bf16_hi(v[u].y),
                                         bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w), bf16_hi(v[u].w)};
                    float x[8];
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        x[i] = __fmul_rn(in[i], r);
                        if (x[i] != x[i]) x[i] = in[i];           // 0 * Inf: keep the signed zero
                    }
                    q = cvt_e2m1x8(x);
                }
            }
            reinterpret_cast<uint32_t *>(elems)[c] = q;
            if ((lane & 1) == 0) {
                const int64_t blk = c >> 1;
                if constexpr (RM) sc_rm[blk] = (uint8_t)sb;
                if constexpr (TC) {
                    const int64_t r = blk / scale_cols;
                    sc_tc[tcgen05_scale_offset(r, blk - r * scale_cols, scale_cols)] = (uint8_t)sb;
                }
            }
        }
    }
}

cudaError_t launch_nvfp4_quant(const void *src, int64_t rows, int64_t cols, const float *partials,
                               int n_partials, float *g, void *elems, uint8_t *rm, uint8_t *tc,
                               int num_sms, cudaStream_t st) {
    const int64_t n_chunks = rows * cols / 8, S = cols / 16;
    const int grid = grid_for(n_chunks, num_sms);
    const uint4 *s = static_cast<const uint4 *>(src);
    uint8_t *e = static_cast<uint8_t *>(elems);
    if (rm && tc)
        nvfp4_quant_kernel<true, true><<<grid, kThreads, 0, st>>>(s, n_chunks, S, partials, n_partials, g, e, rm, tc);
    else if (rm)
        nvfp4_quant_kernel<true, false><<<grid, kThreads, 0, st>>>(s, n_chunks, S, partials, n_partials, g, e, rm, tc);
    else
        nvfp4_quant_kernel<false, true><<<grid, kThreads, 0, st>>>(s, n_chunks, S, partials, n_partials, g, e, rm, tc);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Direct cast (no block scale): RNE + saturation by the hardware conversion; NaN is
// mapped explicitly (0x7F|s for FP8, 0x7|s for E2M1, which has no NaN).
// ---------------------------------------------------------------------------------------
template <int FMT>
__device__ __forceinline__ void cast8(const uint4 &v, uint8_t *out, int64_t c) {
    const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    if constexpr (FMT == FMT_E2M1) {
        uint32_t q = cvt_e2m1x8(x);
#pragma unroll
        for (int i = 0; i < 8; i++)
            if (x[i] != x[i]) q = (q & ~(0xFu << (4 * i))) | ((0x7u | (__float_as_uint(x[i]) >> 31 << 3)) << (4 * i));
        reinterpret_cast<uint32_t *>(out)[c] = q;
    } else {
        uint2 q = cvt_fp8x8<FMT>(x);
        uint32_t w[2] = {q.x, q.y};
#pragma unroll
        for (int i = 0; i < 8; i++)
            if (x[i] != x[i]) {
                const uint32_t nanc = 0x7Fu | (__float_as_uint(x[i]) >> 31 << 7);
                w[i >> 2] = (w[i >> 2] & ~(0xFFu << (8 * (i & 3)))) | (nanc << (8 * (i & 3)));
            }
        reinterpret_cast<uint2 *>(out)[c] = make_uint2(w[0], w[1]);
    }
}

template <int FMT>
__global__ void __launch_bounds__(kThreads)
cast_kernel(const uint4 *__restrict__ src, int64_t n_chunks, const uint16_t *__restrict__ tail_src,
            int tail, uint8_t *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x; c < n_chunks; c += stride)
        cast8<FMT>(ld_stream(src + c), out, c);
    if (tail && blockIdx.x == 0 && threadIdx.x == 0) {
        // the last n % 8 elements, packed the same way, in one thread
        uint16_t t16[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int i = 0; i < tail; i++) t16[i] = tail_src[i];
        uint4 v;
        v.x = t16[0] | ((uint32_t)t16[1] << 16); v.y = t16[2] | ((uint32_t)t16[3] << 16);
        v.z = t16[4] | ((uint32_t)t16[5] << 16); v.w = t16[6] | ((uint32_t)t16[7] << 16);
        alignas(8) uint8_t tmp[8];
        cast8<FMT>(v, tmp, 0);
        const int nbytes = FMT == FMT_E2M1 ? tail / 2 : tail;
        uint8_t *dst = out + (FMT == FMT_E2M1 ? n_chunks * 4 : n_chunks * 8);
        for (int i = 0; i < nbytes; i++) dst[i] = tmp[i];
    }
}

cudaError_t launch_cast(const void *src, int64_t n, int fmt, void *out, int num_sms, cudaStream_t st) {
    const int64_t n_chunks = n / 8;
    const int tail = (int)(n % 8);
    const int grid = grid_for(n_chunks > 0 ? n_chunks : 1, num_sms);
    const uint4 *s = static_cast<const uint4 *>(src);
    const uint16_t *ts = static_cast<const uint16_t *>(src) + n_chunks * 8;
    uint8_t *o = static_cast<uint8_t *>(out);
    switch (fmt) {
    case FMT_E4M3: cast_kernel<FMT_E4M3><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    case FMT_E5M2: cast_kernel<FMT_E5M2><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    case FMT_E2M1: cast_kernel<FMT_E2M1><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Dequantisers.  MX: x = dec(q) * 2^(s-127), the product is exact in fp32 and the only
// rounding is fp32 -> bf16 (RNE).  A 0xFF scale yields NaN for the whole block.
// NVFP4: (dec(q) * dec(sb)) * g in fp32, then bf16; sb = 0x7F yields NaN.
// ---------------------------------------------------------------------------------------
template <int FMT, bool TC>
__global__ void __launch_bounds__(kThreads)
dequant_mx_kernel(const uint8_t *__restrict__ elems, const uint8_t *__restrict__ scales,
                  int64_t n_chunks, int64_t scale_cols, uint4 *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t warp0 = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31);
    for (int64_t base = warp0; base < n_chunks; base += stride) {
        const int64_t c = base + lane;
        const bool ok = c < n_chunks;
        uint32_t s = 0;
        if (ok && (lane & 3) == 0) {
            const int64_t blk = c >> 2;
            if constexpr (TC) {
                const int64_t r = blk / scale_cols;
                s = scales[tcgen05_scale_offset(r, blk - r * scale_cols, scale_cols)];
            } else {
                s = scales[blk];
            }
        }
        s = __shfl_sync(0xffffffffu, s, lane & ~3);
        if (!ok) continue;
        const float mul = s == 0xFFu ? __uint_as_float(0x7FC00000u) : e8m0_multiplier(s);
        float y[8];
        if constexpr (FMT == FMT_E2M1) {
            e2m1x8_to_f32(reinterpret_cast<const uint32_t *>(elems)[c], y);
        } else {
            const uint2 q = reinterpret_cast<const uint2 *>(elems)[c];
            fp8x2_to_f32<FMT>(q.x & 0xFFFFu, y[0], y[1]);
            fp8x2_to_f32<FMT>(q.x >> 16, y[2], y[3]);
            fp8x2_to_f32<FMT>(q.y & 0xFFFFu, y[4], y[5]);
            fp8x2_to_f32<FMT>(q.y >> 16, y[6], y[7]);
        }
        uint4 o;
        o.x = f32x2_to_bf16x2(__fmul_rn(y[0], mul), __fmul_rn(y[1], mul));
        o.y = f32x2_to_bf16x2(__fmul_rn(y[2], mul), __fmul_rn(y[3], mul));
        o.z = f32x2_to_bf16x2(__fmul_rn(y[4], mul), __fmul_rn(y[5], mul));
        o.w = f32x2_to_bf16x2(__fmul_rn(y[6], mul), __fmul_rn(y[7], mul));
        out[c] = o;
    }
}

template <bool TC>
__global__ void __launch_bounds__(kThreads)
dequant_nvfp4_kernel(const uint8_t *__restrict__ elems, const uint8_t *__restrict__ scales,
                     const float *__restrict__ g_ptr, int64_t n_chunks, int64_t scale_cols,
                     uint4 *__restrict__ out) {
    const float g = *g_ptr;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t warp0 = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31);
    for (int64_t base = warp0; base < n_chunks; base += stride) {
        const int64_t c = base + lane;
        const bool ok = c < n_chunks;
        uint32_t s = 0;
        if (ok && (lane & 1) == 0) {
            const int64_t blk = c >> 1;
            if constexpr (TC) {
                const int64_t r = blk / scale_cols;
                s = scales[tcgen05_scale_offset(r, blk - r * scale_cols, scale_cols)];
            } else {
                s = scales[blk];
            }
        }
        s = __shfl_sync(0xffffffffu, s, lane & ~1) & 0x7Fu;
        if (!ok) continue;
        const float sbv = s == 0x7Fu ? __uint_as_float(0x7FC00000u) : ue4m3_to_f32(s);
        float y[8];
        e2m1x8_to_f32(reinterpret_cast<const uint32_t *>(elems)[c], y);
        uint4 o;
        o.x = f32x2_to_bf16x2(__fmul_rn(__fmul_rn(y[0], sbv), g), __fmul_rn(__fmul_rn(y[1], sbv), g));
        o.y = f32x2_to_bf16x2(__fmul_rn(__fmul_rn(y[2], sbv), g), __fmul_rn(__fmul_rn(y[3], sbv), g));
        o.z = f32x2_to_bf16x2(__fmul_rn(__fmul_rn(y[4], sbv), g), __fmul_rn(__fmul_rn(y[5], sbv), g));
        o.w = f32x2_to_bf16x2(__fmul_rn(__fmul_rn(y[6], sbv), g), __fmul_rn(__fmul_rn(y[7], sbv), g));
        out[c] = o;
    }
}

cudaError_t launch_dequant_mx(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                              int fmt, bool tc, void *out, int num_sms, cudaStream_t st) {
    const int64_t n_chunks = rows * cols / 8, S = cols / 32;
    int64_t grid = (n_chunks + kThreads - 1) / kThreads;
    if (grid > (int64_t)num_sms * 16) grid = (int64_t)num_sms * 16;
    const uint8_t *e = static_cast<const uint8_t *>(elems);
    uint4 *o = static_cast<uint4 *>(out);
#define MXK_DQ(F, T) dequant_mx_kernel<F, T><<<(int)grid, kThreads, 0, st>>>(e, scales, n_chunks, S, o)
    switch (fmt) {
    case FMT_E4M3: if (tc) MXK_DQ(FMT_E4M3, true); else MXK_DQ(FMT_E4M3, false); break;
    case FMT_E5M2: if (tc) MXK_DQ(FMT_E5M2, true); else MXK_DQ(FMT_E5M2, false); break;
    case FMT_E2M1: if (tc) MXK_DQ(FMT_E2M1, true); else MXK_DQ(FMT_E2M1, false); break;
    default: return cudaErrorInvalidValue;
    }
#undef MXK_DQ
    return cudaGetLastError();
}

cudaError_t launch_dequant_nvfp4(const void *elems, const uint8_t *scales, const float *g,
                                 int64_t rows, int64_t cols, bool tc, void *out, int num_sms,
                                 cudaStream_t st) {
    const int64_t n_chunks = rows * cols / 8, S = cols / 16;
    int64_t grid = (n_chunks + kThreads - 1) / kThreads;
    if (grid > (int64_t)num_sms * 16) grid = (int64_t)num_sms * 16;
    const uint8_t *e = static_cast<const uint8_t *>(elems);
    uint4 *o = static_cast<uint4 *>(out);
    if (tc) dequant_nvfp4_kernel<true><<<(int)grid, kThreads, 0, st>>>(e, scales, g, n_chunks, S, o);
    else    dequant_nvfp4_kernel<false><<<(int)grid, kThreads, 0, st>>>(e, scales, g, n_chunks, S, o);
    return cudaGetLastError();
}

}  // namespace mxk
