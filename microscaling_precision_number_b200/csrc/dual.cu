// dual.cu -- TMA-staged MX quantiser that reads each bf16 element once and writes the
// row-wise copy, the column-wise (transposed) copy, or both.
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §2 "MXFP4 はブロック32と E8M0": 32-element blocks, E8M0 scale, RNE cast.
//     §4 "精度の差はどこから出るか": floor and no-clip shared-exponent rules.
//     §6 "DeepSeek-V4 の入れ子構造": training uses the weight both as is and transposed;
//        quantising both orientations from one read avoids re-quantising a transposed copy.
//
// Design: persistent CTAs (a multiple of the SM count) walk 32-row x 128-column bf16
// tiles.  One thread streams tiles into a 4-deep shared-memory ring with 2-D TMA loads
// (each stage completes an mbarrier); all 256 threads then
//   - row pass: four lanes per 32-element row block (16-byte shared loads, xor-shuffle
//     maximum), contiguous 8-byte code stores;
//   - column pass: two threads per column (16 rows each, maxima exchanged through shared
//     memory), each writing 16 contiguous codes of the transposed output.
// Every barrier wait is bounded (watchdog); on a timeout the CTA drains its own TMA loads
// (bounded) and returns.
#include <cuda.h>
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace mxk {

namespace {
constexpr int kDualThreads = 256;
constexpr int kTileR = 32, kTileC = 128;
constexpr int kTileBytes = kTileR * kTileC * 2;   // 8 KiB of bf16
constexpr int kStages = 4;
}  // namespace

template <int FMT, bool CEIL, bool ROW, bool COL, bool TC>
__global__ void __launch_bounds__(kDualThreads)
quant_dual_kernel(const __grid_constant__ CUtensorMap tmap, int64_t rows, int64_t cols,
                  uint8_t *__restrict__ row_elems, uint8_t *__restrict__ row_sc,
                  uint8_t *__restrict__ col_elems, uint8_t *__restrict__ col_sc, int *watchdog) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t full_bar[kStages];
    __shared__ uint32_t s_amax[kDualThreads];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int64_t tiles_c = (cols + kTileC - 1) / kTileC;
    const int64_t n_tiles = tiles_c * (rows / kTileR);
    const int64_t row_S = cols / 32, col_S = rows / 32;

    if (tid == 0) {
        prefetch_tensormap(&tmap);
        for (int s = 0; s < kStages; s++) mbar_init(&full_bar[s], 1);
        fence_barrier_init();
    }
    __syncthreads();

    auto issue = [&](int64_t t, int s) {
        const int64_t tr = t / tiles_c, tcl = t - tr * tiles_c;
        mbar_arrive_expect_tx(&full_bar[s], kTileBytes);
        tma_load_2d(smem + s * kTileBytes, &tmap, (int32_t)(tcl * kTileC), (int32_t)(tr * kTileR), &full_bar[s]);
    };
    if (tid == 0)
        for (int s = 0; s < kStages; s++) {
            const int64_t t = blockIdx.x + (int64_t)s * gridDim.x;
            if (t < n_tiles) issue(t, s);
        }

    int it = 0;
    bool failed = false;
    for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
        const int s = it % kStages;
        const uint32_t phase = (uint32_t)(it / kStages) & 1u;
        const bool ok = mbar_wait_bounded(&full_bar[s], phase, watchdog, WD_DUAL_FULL);
        if (__syncthreads_or(!ok)) { failed = true; break; }

        const uint8_t *tile = smem + s * kTileBytes;
        const int64_t tr = t / tiles_c, tcl = t - tr * tiles_c;
        const int64_t r0 = tr * kTileR, c0 = tcl * kTileC;

        if constexpr (ROW) {
#pragma unroll
            for (int k = 0; k < 2; k++) {
                const int j = tid + k * kDualThreads;       // 16-byte chunk within the tile
                const int rr = j >> 4, c8 = j & 15;
                const uint4 v = *reinterpret_cast<const uint4 *>(tile + rr * (kTileC * 2) + c8 * 16);
                uint32_t m = hmax(abs_max_bf16x8(v));
                m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
                m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
                const int64_t col = c0 + c8 * 8;
                if (col < cols) {
                    const uint32_t code = e8m0_from_amax_bits<FMT, CEIL>(m);
                    const float mul = e8m0_inverse_multiplier(code);
                    float x[8];
                    x[0] = __fmul_rn(bf16_lo(v.x), mul); x[1] = __fmul_rn(bf16_hi(v.x), mul);
                    x[2] = __fmul_rn(bf16_lo(v.y), mul); x[3] = __fmul_rn(bf16_hi(v.y), mul);
                    x[4] = __fmul_rn(bf16_lo(v.z), mul); x[5] = __fmul_rn(bf16_hi(v.z), mul);
                    x[6] = __fmul_rn(bf16_lo(v.w), mul); x[7] = __fmul_rn(bf16_hi(v.w), mul);
                    const int64_t e = (r0 + rr) * cols + col;          // element index, multiple of 8
                    if constexpr (FMT == FMT_E2M1) {
                        uint32_t q = cvt_e2m1x8(x);
                        if (code == 0xFFu) q = 0u;
                        reinterpret_cast<uint32_t *>(row_elems)[e >> 3] = q;
                    } else {
                        uint2 q = cvt_fp8x8<FMT>(x);
                        if (code == 0xFFu) q = make_uint2(0u, 0u);
                        reinterpret_cast<uint2 *>(row_elems)[e >> 3] = q;
                    }
                    if ((lane & 3) == 0) {
                        const int64_t R = r0 + rr, b = col >> 5;
                        if constexpr (TC) row_sc[tcgen05_scale_offset(R, b, row_S)] = (uint8_t)code;
                        else row_sc[R * row_S + b] = (uint8_t)code;
                    }
                }
            }
        }

        if constexpr (COL) {
            const int c = tid & (kTileC - 1), h = tid >> 7;     // column, 16-row half
            uint32_t w[8];                                       // 16 bf16, two per word
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const uint32_t lo = *reinterpret_cast<const uint16_t *>(tile + (16 * h + 2 * i) * (kTileC * 2) + c * 2);
                const uint32_t hi = *reinterpret_cast<const uint16_t *>(tile + (16 * h + 2 * i + 1) * (kTileC * 2) + c * 2);
                w[i] = lo | (hi << 16);
                m = max(m, max(lo & 0x7FFFu, hi & 0x7FFFu));
            }
            s_amax[tid] = m;
            __syncthreads();
            m = max(s_amax[c], s_amax[c + kTileC]);
            const int64_t col = c0 + c;
            if (col < cols) {
                const uint32_t code = e8m0_from_amax_bits<FMT, CEIL>(m);
                const float mul = e8m0_inverse_multiplier(code);
                float x0[8], x1[8];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    x0[2 * i] = __fmul_rn(bf16_lo(w[i]), mul);
                    x0[2 * i + 1] = __fmul_rn(bf16_hi(w[i]), mul);
                    x1[2 * i] = __fmul_rn(bf16_lo(w[i + 4]), mul);
                    x1[2 * i + 1] = __fmul_rn(bf16_hi(w[i + 4]), mul);
                }
                const int64_t e = col * rows + r0 + 16 * h;        // element index, multiple of 16
                if constexpr (FMT == FMT_E2M1) {
                    uint2 q = make_uint2(cvt_e2m1x8(x0), cvt_e2m1x8(x1));
                    if (code == 0xFFu) q = make_uint2(0u, 0u);
                    reinterpret_cast<uint2 *>(col_elems)[e >> 4] = q;
                } else {
                    const uint2 qa = cvt_fp8x8<FMT>(x0), qb = cvt_fp8x8<FMT>(x1);
                    uint4 q = make_uint4(qa.x, qa.y, qb.x, qb.y);
                    if (code == 0xFFu) q = make_uint4(0u, 0u, 0u, 0u);
                    reinterpret_cast<uint4 *>(col_elems)[e >> 4] = q;
                }
                if (h == 0) {
                    if constexpr (TC) col_sc[tcgen05_scale_offset(col, tr, col_S)] = (uint8_t)code;
                    else col_sc[col * col_S + tr] = (uint8_t)code;
                }
            }
        }

        __syncthreads();   // stage s and s_amax are free again
        if (tid == 0) {
            const int64_t tn = t + (int64_t)kStages * gridDim.x;
            if (tn < n_tiles) issue(tn, s);
        }
    }

    if (failed && tid == 0) {
        // Drain: wait (bounded) for the loads this CTA still has in flight.
        for (int k = 0; k < kStages; k++) {
            const int j = it + k;
            const int64_t t = blockIdx.x + (int64_t)j * gridDim.x;
            if (t >= n_tiles) break;
            (void)mbar_wait_bounded(&full_bar[j % kStages], (uint32_t)(j / kStages) & 1u, nullptr, 0, kDrainLimitNs);
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

template <int FMT, bool CEIL>
static void launch_dual_t(const CUtensorMap &tm, int grid, size_t smem, int64_t rows, int64_t cols,
                          uint8_t *re, uint8_t *rs, uint8_t *ce, uint8_t *cs, bool tc, int *wd,
                          cudaStream_t st) {
#define MXK_DUAL(R, C, T) quant_dual_kernel<FMT, CEIL, R, C, T><<<grid, kDualThreads, smem, st>>>(tm, rows, cols, re, rs, ce, cs, wd)
    const bool row = re != nullptr, col = ce != nullptr;
    if (row && col) { if (tc) MXK_DUAL(true, true, true); else MXK_DUAL(true, true, false); }
    else if (row)   { if (tc) MXK_DUAL(true, false, true); else MXK_DUAL(true, false, false); }
    else            { if (tc) MXK_DUAL(false, true, true); else MXK_DUAL(false, true, false); }
#undef MXK_DUAL
}

cudaError_t launch_quant_dual(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil,
                              void *row_elems, uint8_t *row_sc, void *col_elems, uint8_t *col_sc,
                              bool tc, int *watchdog, int num_sms, cudaStream_t st) {
    auto encode = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tm;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {kTileC, kTileR};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(src), gdim, gstride, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int64_t n_tiles = ((cols + kTileC - 1) / kTileC) * (rows / kTileR);
    int64_t grid = (int64_t)num_sms * 4;
    if (grid > n_tiles) grid = n_tiles;
    const size_t smem = (size_t)kStages * kTileBytes + 128;
    uint8_t *re = static_cast<uint8_t *>(row_elems), *ce = static_cast<uint8_t *>(col_elems);
    switch (fmt * 2 + (ceil ? 1 : 0)) {
    case FMT_E4M3 * 2 + 0: launch_dual_t<FMT_E4M3, false>(tm, (int)grid, smem, rows, cols, re, row_sc, ce, col_sc, tc, watchdog, st); break;
    case FMT_E4M3 * 2 + 1: launch_dual_t<FMT_E4M3, true>(tm, (int)grid, smem, rows, cols, re, row_sc, ce, col_sc, tc, watchdog, st); break;
    case FMT_E5M2 * 2 + 0: launch_dual_t<FMT_E5M2, false>(tm, (int)grid, smem, rows, cols, re, row_sc, ce, col_sc, tc, watchdog, st); break;
    case FMT_E5M2 * 2 + 1: launch_dual_t<FMT_E5M2, true>(tm, (int)grid, smem, rows, cols, re, row_sc, ce, col_sc, tc, watchdog, st); break;
    case FMT_E2M1 * 2 + 0: launch_dual_t<FMT_E2M1, false>(tm, (int)grid, smem, rows, cols, re, row_sc, ce, col_sc, tc, watchdog, st); break;
    case FMT_E2M1 * 2 + 1: launch_dual_t<FMT_E2M1, true>(tm, (int)grid, smem, rows, cols, re, row_sc, ce, col_sc, tc, watchdog, st); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace mxk
