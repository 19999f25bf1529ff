// quant.cu -- the direct cast (no block scale) and the tcgen05 scale-padding kernel.
//
// Sources (page title, section):
//   gpt-oss MXFP4 explainer, section "MXFP4": the direct cast of bf16 values to FP4 with
//   no shared scale (the page's first example).
//   "MXFP4 と NVFP4 は何が違うのか調べてみた" §2 "MXFP4 はブロック32と E8M0": the cast
//   rounds to nearest even; overflow saturates (the reading taken for the
//   implementation-defined overflow of §8 "適合性検証という新しい層").
//
// A "chunk" is 16 bytes of bf16 input (8 elements); each thread converts whole chunks
// with the hardware cvt.rn.satfinite conversions and writes 8 (FP8), 6 (FP6, packed) or
// 4 (FP4) bytes.
#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"

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
        if (r >= rows || c >= S) out_store(sc + off, (uint8_t)0);
    }
}

cudaError_t launch_tcgen05_pad(uint8_t *sc, int64_t rows, int64_t S, cudaStream_t st) {
    if (rows % 128 == 0 && S % 4 == 0) return cudaSuccess;   // no padding bytes
    const int64_t total = ((rows + 127) / 128) * ((S + 3) / 4) * 512;
    int64_t grid = (total + 255) / 256;
    if (grid > 4096) grid = 4096;
    const OutRange rng[1] = {{sc, (uint64_t)total}};
    const cudaError_t e = set_out_ranges(rng, st);
    if (e != cudaSuccess) return e;
    tcgen05_pad_kernel<<<(int)grid, 256, 0, st>>>(sc, rows, S, total);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Watchdog self-test: one thread waits, with the library's bounded wait and a short limit,
// on a shared-memory barrier that expects one arrival and never gets it.  The wait gives
// up after limit_ns, records WD_SELFTEST in the watchdog flag and the kernel returns; no
// copy or other asynchronous work is in flight, so nothing needs draining.
// ---------------------------------------------------------------------------------------
__global__ void watchdog_selftest_kernel(uint64_t limit_ns, int *watchdog) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    (void)mbar_wait_bounded(&bar, 0u, watchdog, WD_SELFTEST, limit_ns);
}

cudaError_t launch_watchdog_selftest(uint64_t limit_ns, int *watchdog, cudaStream_t st) {
    watchdog_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, watchdog);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Direct cast (no block scale): RNE + saturation by the hardware conversion; NaN is
// mapped explicitly (0x7F|s for FP8; the signed maximum for E2M1 and FP6, which have no
// NaN: 0x7|s, 0x1F|s).
// ---------------------------------------------------------------------------------------
// st(p, v): the store of the codes -- bounds-checked for the output buffer (GLOBAL), plain
// for the tail's local staging buffer.
template <bool GLOBAL, typename T>
__device__ __forceinline__ void st(T *p, T v) {
    if constexpr (GLOBAL) out_store(p, v);
    else *p = v;
}

template <int FMT, bool GLOBAL = true>
__device__ __forceinline__ void cast8(const uint4 &v, uint8_t *out, int64_t c) {
    const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    if constexpr (FMT == FMT_E2M1) {
        uint32_t q = cvt_e2m1x8(x);
#pragma unroll
        for (int i = 0; i < 8; i++)
            if (x[i] != x[i]) q = (q & ~(0xFu << (4 * i))) | ((0x7u | (__float_as_uint(x[i]) >> 31 << 3)) << (4 * i));
        st<GLOBAL>(reinterpret_cast<uint32_t *>(out) + c, q);
    } else {
        uint2 q = cvt_fp8x8<FMT>(x);
        uint32_t w[2] = {q.x, q.y};
#pragma unroll
        for (int i = 0; i < 8; i++)
            if (x[i] != x[i]) {
                const uint32_t nanc = (FMT == FMT_E2M3 || FMT == FMT_E3M2)
                                          ? 0x1Fu | (__float_as_uint(x[i]) >> 31 << 5)
                                          : 0x7Fu | (__float_as_uint(x[i]) >> 31 << 7);
                w[i >> 2] = (w[i >> 2] & ~(0xFFu << (8 * (i & 3)))) | (nanc << (8 * (i & 3)));
            }
        if constexpr (is_fp6(FMT)) {
            // 8 codes packed into 6 bytes at 6c: a 4-byte and a 2-byte store, in the order
            // that keeps each aligned (6c is 4-aligned for even c, 2 more for odd c)
            const uint32_t p0 = fp6_pack4(w[0]), p1 = fp6_pack4(w[1]);
            const uint32_t lo = p0 | (p1 << 24), hi = p1 >> 8;      // 48 bits
            uint8_t *d = out + c * 6;
            if ((c & 1) == 0) {
                st<GLOBAL>(reinterpret_cast<uint32_t *>(d), lo);
                st<GLOBAL>(reinterpret_cast<uint16_t *>(d + 4), (uint16_t)hi);
            } else {
                st<GLOBAL>(reinterpret_cast<uint16_t *>(d), (uint16_t)lo);
                st<GLOBAL>(reinterpret_cast<uint32_t *>(d + 2), (lo >> 16) | (hi << 16));
            }
        } else {
            st<GLOBAL>(reinterpret_cast<uint2 *>(out) + c, make_uint2(w[0], w[1]));
        }
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
        cast8<FMT, false>(v, tmp, 0);
        const int nbytes = tail * code_bits(FMT) / 8;                 // FP6: tail is 4
        uint8_t *dst = out + n_chunks * code_bits(FMT);
        for (int i = 0; i < nbytes; i++) out_store(dst + i, tmp[i]);
    }
}

cudaError_t launch_cast(const void *src, int64_t n, int fmt, void *out, int num_sms, cudaStream_t st) {
    const int64_t n_chunks = n / 8;
    const int tail = (int)(n % 8);
    const int grid = grid_for(n_chunks > 0 ? n_chunks : 1, num_sms);
    const uint4 *s = static_cast<const uint4 *>(src);
    const uint16_t *ts = static_cast<const uint16_t *>(src) + n_chunks * 8;
    uint8_t *o = static_cast<uint8_t *>(out);
    const OutRange rng[1] = {{out, (uint64_t)(n * code_bits(fmt) / 8)}};
    const cudaError_t e = set_out_ranges(rng, st);
    if (e != cudaSuccess) return e;
    switch (fmt) {
    case FMT_E4M3: cast_kernel<FMT_E4M3><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    case FMT_E5M2: cast_kernel<FMT_E5M2><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    case FMT_E2M1: cast_kernel<FMT_E2M1><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    case FMT_E2M3: cast_kernel<FMT_E2M3><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    case FMT_E3M2: cast_kernel<FMT_E3M2><<<grid, kThreads, 0, st>>>(s, n_chunks, ts, tail, o); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace mxk
