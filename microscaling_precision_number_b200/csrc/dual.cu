// dual.cu -- TMA-staged MX quantiser that reads each bf16 element once and writes the
// column-wise (transposed) copy, alone or together with the row-wise copy.
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §2 "MXFP4 はブロック32と E8M0": 32-element blocks, E8M0 scale, RNE cast.
//     §4 "精度の差はどこから出るか": floor and no-clip shared-exponent rules.
//     §6 "DeepSeek-V4 の入れ子構造": training uses the weight both as is and transposed;
//        quantising both orientations from one read avoids re-quantising a transposed copy.
//
// Design:
//   - persistent CTAs, one per SM, walk 32-row x 256-column bf16 tiles.  A producer warp
//     loads each tile as four 32 x 64 boxes (2-D TMA, 128-byte swizzle) into a 7-stage
//     ring (112 KiB in flight per SM; 8 stages for the column-only form, see kStagesOf)
//     guarded by full / empty mbarriers.  Measured on the
//     16384 x 4096 and 16384 x 14336 inputs, 7 stages beat both shallower (4, 6) and
//     deeper rings (8, 10, 12, 13), and one CTA per SM beat two or three CTAs with
//     shallower rings;
//   - warp specialisation over the same stage: warps 0-3 run the column pass (one warp
//     per box, one lane per column pair, 32-bit shared loads), warps 4-7 the row pass (one
//     lane per 32-element row block, four 16-byte shared loads).  The swizzle makes both
//     access patterns bank-conflict free.  With only the column output requested, warps
//     4-7 run the column pass too, on alternate tiles;
//   - block maxima with the packed bf16 |max| instruction (the column pass reduces two
//     columns per instruction), scales by the same exponent arithmetic as every other
//     quantiser, products as packed fp32 pairs, codes by cvt.rn.satfinite;
//   - each lane writes whole 32-byte sectors (one 256-bit store per FP8 block when the
//     output is 32-byte aligned).
// Every barrier wait is bounded (watchdog); the producer drains its own loads before the
// CTA exits, whatever happened.
#include <cuda.h>
#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tiling.cuh"

namespace mxk {

namespace {
constexpr int kBoxC = 64;                            // bf16 columns per box = one 128-byte swizzle row
constexpr int kBoxes = 4;
constexpr int kTileR = 32, kTileC = kBoxC * kBoxes;  // 32 x 256 tile
constexpr int kBoxBytes = kTileR * kBoxC * 2;        // 4 KiB
constexpr int kTileBytes = kBoxBytes * kBoxes;       // 16 KiB
// Ring depth: 7 stages when both orientations are written (every consumer warp takes every
// tile), 8 when only the column-wise output is (the two warp groups take alternate tiles).
// With alternating groups the depth must be even: each stage then belongs to one group,
// whose waits on it follow its phases one by one.  With an odd depth a group's next use of
// a stage is two phases after its last one, and a parity wait cannot tell "two phases on"
// from "the phase the other group is still waiting for": it would pass early.
template <bool ROW> constexpr int kStagesOf = ROW ? 7 : 8;
constexpr int kMaxStages = 8;
constexpr int kProducerWarp = 8;
constexpr int kDualThreads = 32 * (kProducerWarp + 1);
constexpr int kCtasPerSm = 1;
template <bool ROW> constexpr size_t kDualSmem = (size_t)kStagesOf<ROW> * kTileBytes + 1024;   // + alignment
}  // namespace

// 32 bytes at p (w, or zeros when `zero`): one 256-bit store when p is 32-byte aligned,
// else two 16-byte stores.  The rare zero case is a separate store, not a per-word select.
__device__ __forceinline__ void store32(uint8_t *p, const uint32_t (&w)[8], bool v8, bool zero) {
    if (!out_ok(p, 32)) return;
    if (__builtin_expect(zero, 0)) {
        reinterpret_cast<uint4 *>(p)[0] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4 *>(p)[1] = make_uint4(0u, 0u, 0u, 0u);
    } else if (v8) {
        asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                     ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                     : "memory");
    } else {
        reinterpret_cast<uint4 *>(p)[0] = make_uint4(w[0], w[1], w[2], w[3]);
        reinterpret_cast<uint4 *>(p)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// The 32 codes (one per byte in w) of the block that starts at element e of an output:
// FP8 / INT8 as 32 bytes (store32), FP6 packed into 24 bytes (three 8-byte stores; e is a
// multiple of 32, so the address is 8-byte aligned).
template <int FMT>
__device__ __forceinline__ void store_codes(uint8_t *base, uint64_t e, const uint32_t (&w)[8], bool v8, bool zero) {
    if constexpr (is_fp6(FMT)) {
        uint32_t o[6];
        fp6_pack<8>(w, o);
        uint2 *p = reinterpret_cast<uint2 *>(base + e * 3 / 4);
#pragma unroll
        for (int i = 0; i < 3; i++) out_store(p + i, zero ? make_uint2(0u, 0u) : make_uint2(o[2 * i], o[2 * i + 1]));
    } else {
        store32(base + e, w, v8, zero);
    }
}

// Tile order: bands of kBand column tiles, row-tile major inside a band, so that the tiles
// in flight at any moment span many rows of few columns.  The transposed output of a
// column then grows by long contiguous runs (and the row-wise output by kBand x 256-byte
// runs) instead of 32-byte pieces scattered over every column of the matrix.
constexpr uint32_t kBand = 4;
struct TileOrder {
    FastDiv band_tiles;     // tiles per full band (tiles_r * kBand)
    uint32_t n_full;        // tiles in the full bands
    FastDiv last_w;         // width of the last, narrower band (tiles_c % kBand), if any
    uint32_t last_c0;       // its first column tile
};

__device__ __forceinline__ void tile_coords(uint32_t t, const TileOrder &o, uint32_t &tr, uint32_t &tcl) {
    if (t < o.n_full) {
        const uint32_t b = fdiv(t, o.band_tiles), in = t - b * o.band_tiles.d;
        tr = in / kBand;
        tcl = b * kBand + in % kBand;
    } else {
        const uint32_t in = t - o.n_full;
        tr = fdiv(in, o.last_w);
        tcl = o.last_c0 + (in - tr * o.last_w.d);
    }
}

// Byte offset of a swizzled 16-byte chunk: row r (128 bytes) of a 1024-byte-aligned box,
// logical chunk c; the 128-byte swizzle stores it at chunk c ^ (r % 8).
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c) { return r * 128u + ((c ^ (r & 7u)) << 4); }

// Where the scales of one orientation go: a row-major array of S scales per row and/or
// the tcgen05 tiling with `atoms` 4-column atoms per 128 rows (either pointer may be null
// according to the RM / TC template flags).
struct ScaleOut {
    uint8_t *rm;
    uint8_t *tc;
    uint32_t S, atoms;
};
template <bool RM, bool TC>
__device__ __forceinline__ void put_scale(const ScaleOut &o, uint32_t r, uint32_t c, uint32_t code) {
    if constexpr (RM) out_store(o.rm + (uint64_t)r * o.S + c, (uint8_t)code);
    if constexpr (TC) out_store(o.tc + tc_offset(r, c, o.atoms), (uint8_t)code);
}

// Column pass: columns col, col + 1 (box-relative pair q) over the tile's 32 rows.
template <int FMT, bool CEIL, bool RM, bool TC>
__device__ __forceinline__ void column_pair(const uint8_t *box, uint32_t q, uint32_t col, uint32_t rows,
                                            uint32_t r0, uint32_t tr, uint8_t *__restrict__ col_elems,
                                            const ScaleOut &col_sc, bool v8) {
    uint32_t w[32];                                      // row r: bf16 of col (low) and col + 1 (high)
#pragma unroll
    for (int r = 0; r < 32; r++)
        w[r] = *reinterpret_cast<const uint32_t *>(box + swz(r, q >> 2) + ((q & 3u) << 2));
    uint32_t m[16];
#pragma unroll
    for (int i = 0; i < 16; i++) m[i] = absmax_bf16x2(w[2 * i], w[2 * i + 1]);
#pragma unroll
    for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
        for (int i = 0; i < n; i++) m[i] = absmax_bf16x2(m[i], m[i + n]);
    const uint32_t code_lo = e8m0_from_amax_bits<FMT, CEIL>(m[0] & 0x7FFFu);
    const uint32_t code_hi = e8m0_from_amax_bits<FMT, CEIL>((m[0] >> 16) & 0x7FFFu);
    const uint64_t s_lo = splat2(e8m0_inverse_multiplier(code_lo));
    const uint64_t s_hi = splat2(e8m0_inverse_multiplier(code_hi));
    const uint64_t e0 = (uint64_t)col * rows + r0;       // first element of column col in the output

    if constexpr (FMT == FMT_E2M1) {
        uint32_t o_lo[4], o_hi[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {                    // rows 8k .. 8k + 7
            float x[8], y[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const uint32_t a = w[8 * k + 2 * i], b = w[8 * k + 2 * i + 1];
                unpack2(mul2(pack2(__uint_as_float(a << 16), __uint_as_float(b << 16)), s_lo), x[2 * i], x[2 * i + 1]);
                unpack2(mul2(pack2(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(b & 0xFFFF0000u)), s_hi),
                        y[2 * i], y[2 * i + 1]);
            }
            o_lo[k] = cvt_e2m1x8(x);
            o_hi[k] = cvt_e2m1x8(y);
        }
        // a NaN scale makes the whole block NaN: its codes are stored as 0
        uint4 *p = reinterpret_cast<uint4 *>(col_elems + (e0 >> 1));
        out_store(p, code_lo == 0xFFu ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(o_lo[0], o_lo[1], o_lo[2], o_lo[3]));
        out_store(p + (rows >> 5), code_hi == 0xFFu ? make_uint4(0u, 0u, 0u, 0u)     // next column: rows / 2 bytes on
                                                    : make_uint4(o_hi[0], o_hi[1], o_hi[2], o_hi[3]));
    } else {
        uint32_t o_lo[8], o_hi[8];
#pragma unroll
        for (int i = 0; i < 16; i++) {                   // rows 2i, 2i + 1
            const uint32_t a = w[2 * i], b = w[2 * i + 1];
            float x0, x1, y0, y1;
            unpack2(mul2(pack2(__uint_as_float(a << 16), __uint_as_float(b << 16)), s_lo), x0, x1);
            unpack2(mul2(pack2(__uint_as_float(a & 0xFFFF0000u), __uint_as_float(b & 0xFFFF0000u)), s_hi), y0, y1);
            const uint32_t cl = cvt_fp8x2<FMT>(x0, x1), ch = cvt_fp8x2<FMT>(y0, y1);
            if (i & 1) { o_lo[i >> 1] |= cl << 16; o_hi[i >> 1] |= ch << 16; }
            else       { o_lo[i >> 1] = cl;        o_hi[i >> 1] = ch; }
        }
        store_codes<FMT>(col_elems, e0, o_lo, v8, code_lo == 0xFFu);        // NaN scale: codes 0
        store_codes<FMT>(col_elems, e0 + rows, o_hi, v8, code_hi == 0xFFu);
    }
    put_scale<RM, TC>(col_sc, col, tr, code_lo);
    put_scale<RM, TC>(col_sc, col + 1, tr, code_hi);
}

// Row pass: the 32-element block of tile row r starting at box-relative chunk 4h.
template <int FMT, bool CEIL, bool RM, bool TC>
__device__ __forceinline__ void row_block(const uint8_t *box, uint32_t r, uint32_t h, uint32_t col, uint32_t cols,
                                          uint32_t R, uint8_t *__restrict__ row_elems, const ScaleOut &row_sc,
                                          bool v8) {
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; k++) v[k] = *reinterpret_cast<const uint4 *>(box + swz(r, 4u * h + k));
    uint32_t m[8];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        m[2 * k] = absmax_bf16x2(v[k].x, v[k].y);
        m[2 * k + 1] = absmax_bf16x2(v[k].z, v[k].w);
    }
#pragma unroll
    for (int n = 4; n >= 1; n >>= 1)
#pragma unroll
        for (int i = 0; i < n; i++) m[i] = absmax_bf16x2(m[i], m[i + n]);
    const uint32_t code = e8m0_from_amax_bits<FMT, CEIL>(max(m[0] & 0x7FFFu, (m[0] >> 16) & 0x7FFFu));
    const uint64_t s2 = splat2(e8m0_inverse_multiplier(code));
    const uint64_t e0 = (uint64_t)R * cols + col;

    if constexpr (FMT == FMT_E2M1) {
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            float x[8];
            scale8(v[k], s2, x);
            o[k] = cvt_e2m1x8(x);
        }
        out_store(reinterpret_cast<uint4 *>(row_elems + (e0 >> 1)),
                  code == 0xFFu ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(o[0], o[1], o[2], o[3]));   // NaN scale: codes 0
    } else {
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            float x[8];
            scale8(v[k], s2, x);
            const uint2 q = cvt_fp8x8<FMT>(x);
            o[2 * k] = q.x;
            o[2 * k + 1] = q.y;
        }
        store_codes<FMT>(row_elems, e0, o, v8, code == 0xFFu);             // NaN scale: codes 0
    }
    put_scale<RM, TC>(row_sc, R, col >> 5, code);
}

// ROW: also write the row-wise output.  RM / TC: write the scales in the row-major layout,
// the tcgen05 tiling, or both (one pass either way).
template <int FMT, bool CEIL, bool ROW, bool RM, bool TC>
__global__ void __launch_bounds__(kDualThreads, kCtasPerSm)
quant_dual_kernel(const __grid_constant__ CUtensorMap tmap, uint32_t rows, uint32_t cols, uint32_t n_tiles,
                  TileOrder order, uint8_t *__restrict__ row_elems, ScaleOut row_sc,
                  uint8_t *__restrict__ col_elems, ScaleOut col_sc, int v8, int *watchdog) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int kStages = kStagesOf<ROW>;
    static_assert(ROW || kStages % 2 == 0, "alternating consumer groups need an even ring depth");
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];

    const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t G = gridDim.x;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmap);
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], ROW ? 8 : 4);          // consumer warps per tile
        }
        fence_barrier_init();
    }
    // Programmatic dependent launch: the set-up above overlaps the previous kernel's tail;
    // nothing is read or written in global memory before that kernel has completed.  The
    // next kernel may then be launched at once (its CTAs start as ours retire).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();

    uint32_t issued = 0;
    if (warp == kProducerWarp) {
        if (lane == 0) {
            for (uint32_t t = blockIdx.x; t < n_tiles; t += G, ++issued) {
                const uint32_t s = issued % kStages;
                if (issued >= kStages &&
                    !mbar_wait_bounded(&empty[s], (issued / kStages - 1) & 1u, watchdog, WD_DUAL_EMPTY))
                    break;
                uint32_t tr, tcl;
                tile_coords(t, order, tr, tcl);
                mbar_arrive_expect_tx(&full[s], kTileBytes);
#pragma unroll
                for (int j = 0; j < kBoxes; j++)
                    tma_load_2d(smem + s * kTileBytes + j * kBoxBytes, &tmap, (int32_t)(tcl * kTileC + j * kBoxC),
                                (int32_t)(tr * kTileR), &full[s]);
            }
        }
    } else {
        const uint32_t grp = warp >> 2, j = warp & 3;    // warp group, box
        const bool row_pass = ROW && grp == 1;
        uint32_t it = 0;
        for (uint32_t t = blockIdx.x; t < n_tiles; t += G, ++it) {
            if (!ROW && (it & 1u) != grp) continue;       // column-only: groups alternate tiles
            const uint32_t s = it % kStages;
            const bool ok = mbar_wait_bounded(&full[s], (it / kStages) & 1u, watchdog, WD_DUAL_FULL);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
            uint32_t tr, tcl;
            tile_coords(t, order, tr, tcl);
            const uint32_t r0 = tr * kTileR, c0 = tcl * kTileC + j * kBoxC;
            const uint8_t *box = smem + s * kTileBytes + j * kBoxBytes;
            if (row_pass) {
                const uint32_t h = lane & 1u, col = c0 + 32u * h;
                if (col < cols) {
                    row_block<FMT, CEIL, RM, TC>(box, lane >> 1, h, col, cols, r0 + (lane >> 1), row_elems, row_sc,
                                                 v8 != 0);
                    row_block<FMT, CEIL, RM, TC>(box, 16 + (lane >> 1), h, col, cols, r0 + 16 + (lane >> 1),
                                                 row_elems, row_sc, v8 != 0);
                }
            } else {
                const uint32_t col = c0 + 2u * lane;
                if (col < cols)
                    column_pair<FMT, CEIL, RM, TC>(box, lane, col, rows, r0, tr, col_elems, col_sc, v8 != 0);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
    __syncthreads();
    if (warp == kProducerWarp && lane == 0) {
        // Wait (bounded, short) for the last load issued into each stage.  On the normal
        // path every one of them has been consumed and this returns at once; after a
        // timeout it keeps the CTA alive until its own copies have landed.
        for (uint32_t s = 0; s < kStages && s < issued; s++) {
            const uint32_t last = s + ((issued - 1 - s) / kStages) * kStages;
            (void)mbar_wait_bounded(&full[s], (last / kStages) & 1u, nullptr, 0, kDrainLimitNs);
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

template <int FMT, bool CEIL, bool ROW, bool RM, bool TC>
static cudaError_t launch_dual_k(const CUtensorMap &tm, int grid, uint32_t rows, uint32_t cols, uint32_t n_tiles,
                                 TileOrder order, uint8_t *re, const ScaleOut &rs, uint8_t *ce, const ScaleOut &cs,
                                 int v8, int *wd, cudaStream_t st) {
    auto k = quant_dual_kernel<FMT, CEIL, ROW, RM, TC>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDualSmem<ROW>);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kDualThreads);
    cfg.dynamicSmemBytes = kDualSmem<ROW>;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, tm, rows, cols, n_tiles, order, re, rs, ce, cs, v8, wd);
}

template <int FMT, bool CEIL, bool ROW>
static cudaError_t launch_dual_l(const CUtensorMap &tm, int grid, uint32_t rows, uint32_t cols, uint32_t n_tiles,
                                 TileOrder d, uint8_t *re, const ScaleOut &rs, uint8_t *ce, const ScaleOut &cs,
                                 int v8, int *wd, cudaStream_t st) {
    if (cs.rm && cs.tc)
        return launch_dual_k<FMT, CEIL, ROW, true, true>(tm, grid, rows, cols, n_tiles, d, re, rs, ce, cs, v8, wd, st);
    if (cs.rm)
        return launch_dual_k<FMT, CEIL, ROW, true, false>(tm, grid, rows, cols, n_tiles, d, re, rs, ce, cs, v8, wd, st);
    return launch_dual_k<FMT, CEIL, ROW, false, true>(tm, grid, rows, cols, n_tiles, d, re, rs, ce, cs, v8, wd, st);
}

template <int FMT, bool CEIL>
static cudaError_t launch_dual_t(bool row, const CUtensorMap &tm, int grid, uint32_t rows, uint32_t cols,
                                 uint32_t n_tiles, TileOrder d, uint8_t *re, const ScaleOut &rs, uint8_t *ce,
                                 const ScaleOut &cs, int v8, int *wd, cudaStream_t st) {
    return row ? launch_dual_l<FMT, CEIL, true>(tm, grid, rows, cols, n_tiles, d, re, rs, ce, cs, v8, wd, st)
               : launch_dual_l<FMT, CEIL, false>(tm, grid, rows, cols, n_tiles, d, re, rs, ce, cs, v8, wd, st);
}

cudaError_t launch_quant_dual(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil,
                              void *row_elems, uint8_t *row_rm, uint8_t *row_tc, void *col_elems, uint8_t *col_rm,
                              uint8_t *col_tc, int *watchdog, int num_sms, cudaStream_t st) {
    // Preconditions (checked by the caller): rows % 32 == 0, cols % 8 == 0 (cols % 32 == 0
    // with the row-wise output), 16-byte aligned source and outputs, column output present
    // with at least one scale layout; the row-wise output, when present, gets the same
    // scale layouts as the column-wise one.
    if (!col_elems || (!col_rm && !col_tc)) return cudaErrorInvalidValue;
    const bool row = row_elems != nullptr;
    if (row && ((row_rm != nullptr) != (col_rm != nullptr) || (row_tc != nullptr) != (col_tc != nullptr)))
        return cudaErrorInvalidValue;
    auto encode = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tm;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {kBoxC, kTileR};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(src), gdim, gstride, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const uint32_t tiles_c = (uint32_t)((cols + kTileC - 1) / kTileC);
    const uint32_t n_tiles = tiles_c * (uint32_t)(rows / kTileR);
    const int grid = (int)(n_tiles < (uint32_t)(kCtasPerSm * num_sms) ? n_tiles : (uint32_t)(kCtasPerSm * num_sms));
    const uint32_t tiles_r = (uint32_t)(rows / kTileR);
    TileOrder d;
    d.band_tiles = make_fastdiv(tiles_r * kBand);
    d.n_full = tiles_c / kBand * kBand * tiles_r;
    d.last_w = make_fastdiv(tiles_c % kBand ? tiles_c % kBand : 1);
    d.last_c0 = tiles_c / kBand * kBand;
    // scale-array geometry: scales per row (row-major) and 4-column atoms (tcgen05)
    const uint32_t row_S = (uint32_t)(cols / 32), col_S = (uint32_t)(rows / 32);
    const ScaleOut rs{row_rm, row_tc, row_S, (row_S + 3) / 4};
    const ScaleOut cs{col_rm, col_tc, col_S, (col_S + 3) / 4};
    const uint64_t code_bytes = (uint64_t)(rows * cols * code_bits(fmt) / 8);
    const uint64_t row_tc_bytes = (uint64_t)((rows + 127) / 128) * ((row_S + 3) / 4) * 512;
    const uint64_t col_tc_bytes = (uint64_t)((cols + 127) / 128) * ((col_S + 3) / 4) * 512;
    const OutRange out[6] = {{row_elems, code_bytes}, {row_rm, (uint64_t)rows * row_S}, {row_tc, row_tc_bytes},
                             {col_elems, code_bytes}, {col_rm, (uint64_t)cols * col_S}, {col_tc, col_tc_bytes}};
    const cudaError_t re_err = set_out_ranges(out, st);
    if (re_err != cudaSuccess) return re_err;
    uint8_t *re = static_cast<uint8_t *>(row_elems), *ce = static_cast<uint8_t *>(col_elems);
    const int v8 = ((reinterpret_cast<uintptr_t>(re) | reinterpret_cast<uintptr_t>(ce)) & 31u) == 0;
    const uint32_t R = (uint32_t)rows, C = (uint32_t)cols;
    switch (fmt * 2 + (ceil ? 1 : 0)) {
    case FMT_E4M3 * 2 + 0: return launch_dual_t<FMT_E4M3, false>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E4M3 * 2 + 1: return launch_dual_t<FMT_E4M3, true>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E5M2 * 2 + 0: return launch_dual_t<FMT_E5M2, false>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E5M2 * 2 + 1: return launch_dual_t<FMT_E5M2, true>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E2M1 * 2 + 0: return launch_dual_t<FMT_E2M1, false>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E2M1 * 2 + 1: return launch_dual_t<FMT_E2M1, true>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E2M3 * 2 + 0: return launch_dual_t<FMT_E2M3, false>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E2M3 * 2 + 1: return launch_dual_t<FMT_E2M3, true>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E3M2 * 2 + 0: return launch_dual_t<FMT_E3M2, false>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_E3M2 * 2 + 1: return launch_dual_t<FMT_E3M2, true>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_INT8 * 2 + 0: return launch_dual_t<FMT_INT8, false>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    case FMT_INT8 * 2 + 1: return launch_dual_t<FMT_INT8, true>(row, tm, grid, R, C, n_tiles, d, re, rs, ce, cs, v8, watchdog, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace mxk
