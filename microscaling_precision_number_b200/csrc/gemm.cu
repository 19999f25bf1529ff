// gemm.cu -- MX block-scaled matmul on the sm_100a 5th-generation tensor cores.
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §2 "MXFP4 はブロック32と E8M0": MXFP8 (E4M3) and MXFP4 (E2M1) share the 32-element
//        block and the E8M0 scale, which is what makes MXFP4 weights x MXFP8 activations
//        (W4A8) convenient.
//     §7 "ハードウェアの対応状況": Blackwell's 5th-generation tensor cores run MX formats
//        natively; applying an E8M0 scale is an exponent add (no multiplier, no rounding);
//        B200 dense peaks FP8 4.5 / FP4 9 PFLOPS.
//
// C[m, n] = sum_k dec(A[m,k]) 2^(sA-127) * dec(B[n,k]) 2^(sB-127), fp32 accumulation in
// tensor memory, bf16 output.  A: M x K E4M3 codes, B: N x K E4M3 or E2M1 codes, both
// K-major; scales per 32 along K in the tcgen05 tiling (512-byte atoms of 128 rows x 4
// scale columns).
//
// Kernel structure: persistent CTAs (one per SM, 11 warps), 128 x 256 output tiles
// (128 x 128 when N is not a multiple of 256):
//   warp 8  TMA producer: per 128-wide K step, 2-D TMA loads of the A tile (128 x 128 B)
//           and the B tile (256 x 128 B, E2M1 expanded by the TMA to one byte per
//           element) with 128-byte swizzle, plus bulk copies of the matching scale atoms
//           (1 for A, 2 for B) into a 4-stage shared-memory ring (mbarrier "full"); the
//           ring runs on across tile boundaries.
//   warp 10 scale copier: copies the stage's scale atoms into tensor memory
//           (tcgen05.cp 32x128b.warpx4) and commits to the stage's "sf_ready" barrier.
//   warp 9  TMEM allocator and MMA issuer: waits on "sf_ready", issues four
//           tcgen05.mma.kind::mxf8f6f4.block_scale (K = 32 each; the scale byte of each
//           is selected by the scale-factor id in the instruction descriptor), and
//           releases the stage with tcgen05.commit on its "empty" barrier; a finished
//           tile is signalled on "acc_full".
//   The three issuing warps run their loops converged and issue from one elected lane.
//   warps 0-7  epilogue: two warps per 32-lane TMEM quadrant (one per column half) load
//           the fp32 accumulator (tcgen05.ld), convert to bf16 in registers, release the
//           accumulator on "acc_empty" -- the next tile's MMAs start now -- and then
//           store their row segments with 16-byte global stores.
// All waits are bounded by the watchdog; tensor memory is always released.
#include <cuda.h>
#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace mxk {

namespace {
constexpr int kBM = 128, kBK = 128;                      // tile rows; bytes of K per row per stage
constexpr int kStages = 4;
constexpr int kEpilogueWarps = 8;                  // two per TMEM lane quadrant
constexpr int kProducerWarp = 8, kMmaWarp = 9, kSfWarp = 10;
constexpr int kGemmThreads = 352;
constexpr int kABytes = kBM * kBK;                       // 16 KiB
constexpr uint32_t kTmemCols = 512;                      // accumulator (<= 256) + scale slots
constexpr uint32_t kSfCol0 = 256;                        // first scale-slot column
template <int BN, int KIND> struct Tile {
    // K elements per stage (128 bytes of codes per row) and scale atoms (512 B: 128 rows x
    // 4 scales) per 128 rows per stage
    static constexpr int kStageK = KIND == KIND_F8F6F4 ? 128 : 256;
    static constexpr int kAtoms = KIND == KIND_F8F6F4 ? 1 : (KIND == KIND_MXF4 ? 2 : 4);
    static constexpr int kBBytes = BN * kBK;             // 32 KiB for BN = 256
    static constexpr int kSfaBytes = 512 * kAtoms;
    static constexpr int kSfbBytes = 512 * kAtoms * (BN / 128);
    // tensor-memory scale columns per stage: B atoms first (4 columns per 128 rows), then A
    static constexpr uint32_t kSfbCols = 4 * kAtoms * (BN / 128);
    static constexpr uint32_t kSfColsPerStage = kSfbCols + 4 * kAtoms;
    static constexpr int kSmemBytes = kStages * (kABytes + kBBytes + kSfaBytes + kSfbBytes) + 1024;
};
static_assert(kSfCol0 + kStages * Tile<256, KIND_NVF4>::kSfColsPerStage <= kTmemCols, "scale slots exceed TMEM");
static_assert(Tile<256, KIND_NVF4>::kSmemBytes + 256 <= 227 * 1024, "shared memory");
}  // namespace

// ---- kernel ------------------------------------------------------------------------------
// Persistent: CTA c processes output tiles c, c + grid, c + 2 grid, ... (row-major over the
// M/128 x N/BN tile grid).  The TMA producer and the MMA issuer run through the K steps of
// consecutive tiles without a break (the shared-memory ring spans tiles).  The epilogue
// drains a finished accumulator into registers, releases it (acc_empty) so that the MMAs
// of the next tile start at once, and then writes its bf16 rows while they run.
// alpha = (*ga) * (*gb) multiplies the accumulator before the bf16 conversion (the NVFP4
// per-tensor scales; ga = gb = nullptr means 1).
template <int BN, int KIND>
__global__ void __launch_bounds__(kGemmThreads, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const uint8_t *__restrict__ a_sc, const uint8_t *__restrict__ b_sc, const float *__restrict__ ga,
               const float *__restrict__ gb, uint16_t *__restrict__ C, int M, int N, int K, uint32_t a_fmt_code,
               uint32_t b_fmt_code, int band, int *watchdog) {
    using T = Tile<BN, KIND>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;                                   // kStages x 16 KiB (1024-aligned)
    constexpr int kBBytes = T::kBBytes, kSfaBytes = T::kSfaBytes, kSfbBytes = T::kSfbBytes;
    uint8_t *sB = sA + kStages * kABytes;                 // kStages x BN x 128 B
    uint8_t *sSFA = sB + kStages * kBBytes;               // kStages x 512 B
    uint8_t *sSFB = sSFA + kStages * kSfaBytes;           // kStages x kAtoms x 512 B per 128 rows of B

    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], sf_ready[kStages], acc_full, acc_empty,
        drain_bar, sf_drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int fail_flag;
    volatile int *fail_sh = &fail_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_kb = K / T::kStageK;
    const int tiles_n = N / BN, tiles_m = M / kBM;
    const int n_tiles = tiles_m * tiles_n;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
            mbar_init(&sf_ready[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, kEpilogueWarps);
        mbar_init(&drain_bar, 1);
        mbar_init(&sf_drain, 1);
        *fail_sh = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(&tmem_base_sh, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    int last_it[kStages];                                 // producer: last ring use armed per stage
    for (int s = 0; s < kStages; s++) last_it[s] = -1;
    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer
        // the whole warp runs the loop (warp-uniform waits); one elected lane issues
        // scale atoms per 128-row block of an operand (the tcgen05 layout's column-atom count)
        const int64_t col_atoms = (int64_t)num_kb * T::kAtoms;
        const uint32_t tx = (KIND == KIND_F8F6F4 ? f8f6f4_packed_bytes(kABytes, a_fmt_code) : kABytes) +
                            (KIND == KIND_F8F6F4 ? f8f6f4_packed_bytes(kBBytes, b_fmt_code) : kBBytes) +
                            kSfaBytes + kSfbBytes;
        int it = 0;
        for (int t = blockIdx.x; t < n_tiles && !warp_failed(fail_sh); t += gridDim.x) {
            int m_blk, n_blk;
            tile_coords(t, tiles_m, tiles_n, band, m_blk, n_blk);
            for (int kb = 0; kb < num_kb; kb++, it++) {
                const int s = it % kStages;
                if (it >= kStages &&
                    !warp_wait(&empty_bar[s], (uint32_t)((it / kStages) - 1) & 1u, watchdog, WD_GEMM_EMPTY)) {
                    *fail_sh = 1;
                    break;
                }
                if (elect_one()) {
                    // E2M1 and FP6 tiles of the mxf8f6f4 kind land in shared memory padded to
                    // one 16-byte group per 16 codes, but the copy completes only the packed
                    // global bytes.  Either way a stage holds 128 bytes of K per row.
                    mbar_arrive_expect_tx(&full_bar[s], tx);
                    tma_load_2d(sA + s * kABytes, &tmA, kb * kBK, m_blk * kBM, &full_bar[s]);
                    tma_load_2d(sB + s * kBBytes, &tmB, kb * kBK, n_blk * BN, &full_bar[s]);
                    // the stage's scale atoms are contiguous in the tcgen05 layout
                    bulk_load(sSFA + s * kSfaBytes, a_sc + ((int64_t)m_blk * col_atoms + (int64_t)kb * T::kAtoms) * 512,
                              kSfaBytes, &full_bar[s]);
#pragma unroll
                    for (int h = 0; h < BN / 128; h++)
                        bulk_load(sSFB + s * kSfbBytes + h * T::kSfaBytes,
                                  b_sc + ((int64_t)((BN / 128) * n_blk + h) * col_atoms + (int64_t)kb * T::kAtoms) * 512,
                                  T::kSfaBytes, &full_bar[s]);
                }
                __syncwarp();
                last_it[s] = it;
            }
        }
    } else if (warp == kSfWarp) {
        // ------------------------------------------------ scale-atom copier
        // Copies each stage's scale atoms into tensor memory as soon as the stage has
        // landed and signals sf_ready[s] once the copies are complete; the MMA issuer waits
        // on sf_ready alone, so the copies (3 to 12 per stage) stay off the MMA warp.  A
        // stage's scale slot is rewritten only after full[s] of its next use, i.e. after
        // the MMAs that read it have completed (empty[s]).
        const uint64_t sfa_d0 = sf_desc(smem_u32(sSFA)), sfb_d0 = sf_desc(smem_u32(sSFB));
        int it = 0;
        for (int t = blockIdx.x; t < n_tiles && !warp_failed(fail_sh); t += gridDim.x) {
            for (int kb = 0; kb < num_kb; kb++, it++) {
                const int s = it % kStages;
                if (!warp_wait(&full_bar[s], (uint32_t)(it / kStages) & 1u, watchdog, WD_GEMM_FULL)) {
                    *fail_sh = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t sfb_t = tmem + kSfCol0 + s * T::kSfColsPerStage;
                const uint32_t sfa_t = sfb_t + T::kSfbCols;
                const uint64_t sfa_d = sfa_d0 + (uint64_t)((s * kSfaBytes) >> 4);
                const uint64_t sfb_d = sfb_d0 + (uint64_t)((s * kSfbBytes) >> 4);
                if (elect_one()) {
#pragma unroll
                    for (int a = 0; a < T::kAtoms; a++) {
                        tc_cp_sf(sfa_t + 4 * a, sfa_d + (uint64_t)(a * 512 / 16));
#pragma unroll
                        for (int h = 0; h < BN / 128; h++)
                            tc_cp_sf(sfb_t + 4 * (a * (BN / 128) + h), sfb_d + (uint64_t)((h * T::kSfaBytes + a * 512) / 16));
                    }
                    tc_commit(&sf_ready[s]);                  // the stage's scales are in tensor memory
                }
                __syncwarp();
            }
        }
        if (elect_one()) tc_commit(&sf_drain);            // completes once every copy above has finished
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer
        // Descriptors are precomputed and advance by offsets >> 4 (the 14-bit start-address
        // field never overflows inside shared memory); the whole warp runs the loop and one
        // elected lane issues each stage's MMAs and its commit.
        const uint64_t a_d0 = smem_desc(smem_u32(sA), 16, 1024, 2), b_d0 = smem_desc(smem_u32(sB), 16, 1024, 2);
        uint32_t idesc[4];
#pragma unroll
        for (int k = 0; k < 4; k++)
            idesc[k] = mma_idesc<kBM, BN, KIND>(
                a_fmt_code, b_fmt_code,
                KIND == KIND_F8F6F4 ? (uint32_t)k : (KIND == KIND_MXF4 ? 2u * (k & 1) : 0u));
        int it = 0, i = 0;
        for (int t = blockIdx.x; t < n_tiles && !warp_failed(fail_sh); t += gridDim.x, i++) {
            if (i > 0 && !warp_wait(&acc_empty, (uint32_t)(i - 1) & 1u, watchdog, WD_GEMM_ACC)) {
                *fail_sh = 1;
                break;
            }
            tc_fence_after();
            for (int kb = 0; kb < num_kb; kb++, it++) {
                const int s = it % kStages;
                // the stage's operands have landed and its scales are in tensor memory
                if (!warp_wait(&sf_ready[s], (uint32_t)(it / kStages) & 1u, watchdog, WD_GEMM_FULL)) {
                    *fail_sh = 1;
                    break;
                }
                tc_fence_after();
                // tensor-memory scale slots of this stage: B atom (a, h) at column
                // sfb_t + 4 (a (BN/128) + h), A atom a at sfa_t + 4 a
                const uint32_t sfb_t = tmem + kSfCol0 + s * T::kSfColsPerStage;
                const uint32_t sfa_t = sfb_t + T::kSfbCols;
                const uint64_t a_d = a_d0 + (uint64_t)((s * kABytes) >> 4);
                const uint64_t b_d = b_d0 + (uint64_t)((s * kBBytes) >> 4);
                // four instructions per stage, each over 32 bytes of K per row (K = 32 for
                // 8-bit codes, 64 for packed 4-bit codes).  Instruction k reads scale atom
                // a and, inside its 32-bit words, the scale byte(s) starting at sf_id:
                // 1X: a = 0, sf_id = k; 2X: a = k / 2, sf_id = 2 (k % 2); 4X: a = k, sf_id = 0.
                if (elect_one()) {
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        const int a = KIND == KIND_F8F6F4 ? 0 : (KIND == KIND_MXF4 ? k >> 1 : k);
                        tc_mma_mx<KIND>(tmem, a_d + (uint64_t)(2 * k), b_d + (uint64_t)(2 * k), idesc[k], sfa_t + 4 * a,
                                        sfb_t + 4 * a * (BN / 128), (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty_bar[s]);
                }
                __syncwarp();
            }
            if (warp_failed(fail_sh)) break;
            if (elect_one()) tc_commit(&acc_full);        // the tile's accumulator is complete
            __syncwarp();
        }
        if (elect_one()) tc_commit(&drain_bar);           // completes once every MMA above has finished
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-7)
        // warp w reads TMEM lanes 32 (w % 4) .. + 31 (rows) and columns of half w / 4
        constexpr int kHalf = BN / 2;
        const int quad = warp & 3, half = warp >> 2;
        const float alpha = (ga && gb) ? __fmul_rn(__ldg(ga), __ldg(gb)) : 1.0f;
        const uint32_t t_base = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * kHalf);
        int i = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, i++) {
            const bool ok = mbar_wait_bounded(&acc_full, (uint32_t)i & 1u, watchdog, WD_GEMM_ACC);
            if (!ok || *fail_sh) { *fail_sh = 1; break; }
            tc_fence_after();
            // the whole row segment comes out of tensor memory first (one wait), so the
            // accumulator is released before the conversion and the stores
            uint32_t r[kHalf / 32][32];
            tmem_ld32_batch<kHalf / 32>(t_base, r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty);       // accumulator may be overwritten now
            int m_blk, n_blk;
            tile_coords(t, tiles_m, tiles_n, band, m_blk, n_blk);
            const int row = m_blk * kBM + quad * 32 + lane;
            uint4 *dst = reinterpret_cast<uint4 *>(C + (int64_t)row * N + (int64_t)n_blk * BN + half * kHalf);
            // evict-first stores: the output must not push operand panels out of L2
#pragma unroll
            for (int j = 0; j < kHalf / 32; j++)
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; e++)
                        o[e] = f32x2_to_bf16x2(__fmul_rn(__uint_as_float(r[j][8 * q + 2 * e]), alpha),
                                               __fmul_rn(__uint_as_float(r[j][8 * q + 2 * e + 1]), alpha));
                    if (out_ok(dst + 4 * j + q, 16)) __stcs(dst + 4 * j + q, make_uint4(o[0], o[1], o[2], o[3]));
                }
        }
    }

    // teardown: on the error path wait (bounded) for every copy this CTA armed and for
    // every MMA it issued, so that no copy or MMA touches shared or tensor memory after
    // they are released
    __syncthreads();
    if (*fail_sh && warp == kProducerWarp && lane == 0) {
        for (int s = 0; s < kStages; s++)
            if (last_it[s] >= 0)
                (void)mbar_wait_bounded(&full_bar[s], (uint32_t)(last_it[s] / kStages) & 1u, nullptr, 0, kDrainLimitNs);
    }
    if (*fail_sh && warp == kMmaWarp && lane == 0) (void)mbar_wait_bounded(&drain_bar, 0u, nullptr, 0, kDrainLimitNs);
    if (warp == kSfWarp && lane == 0) (void)mbar_wait_bounded(&sf_drain, 0u, nullptr, 0, kDrainLimitNs);
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// 2-D tensor map over a rows x K operand: 8-bit codes (one byte per element); E2M1 or FP6
// codes expanded by the copy to a 16-byte group per 16 codes (16U4_ALIGN16B /
// 16U6_ALIGN16B, mxf8f6f4 kind); or packed E2M1 codes read as bytes (4-bit kinds).  Either
// way the box is 128 bytes of shared memory per row.
static bool encode_operand(EncodeTiledFn enc, CUtensorMap *tm, const void *ptr, int64_t rows, int64_t K,
                           int fmt, bool expand, uint32_t box_rows) {
    const int bits = code_bits(fmt);
    const cuuint64_t gdim[2] = {(cuuint64_t)(expand || bits == 8 ? K : K * bits / 8), (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)(K * bits / 8)};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = !expand ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : bits == 6 ? CU_TENSOR_MAP_DATA_TYPE_16U6_ALIGN16B
                                               : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
    const CUresult r = enc(tm, dt, 2,
                           const_cast<void *>(ptr), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int BN, int KIND>
static cudaError_t launch_gemm_k(const CUtensorMap &tmA, const CUtensorMap &tmB, const uint8_t *a_sc,
                                 const uint8_t *b_sc, const float *ga, const float *gb, void *c, int64_t M,
                                 int64_t N, int64_t K, uint32_t a_code, uint32_t b_code, int64_t band, int *watchdog,
                                 int grid, cudaStream_t st) {
    auto k = mx_gemm_kernel<BN, KIND>;
    const OutRange rng[1] = {{c, (uint64_t)(M * N * 2)}};
    cudaError_t e = set_out_ranges(rng, st);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile<BN, KIND>::kSmemBytes);
    if (e != cudaSuccess) return e;
    k<<<grid, kGemmThreads, Tile<BN, KIND>::kSmemBytes, st>>>(tmA, tmB, a_sc, b_sc, ga, gb, static_cast<uint16_t *>(c),
                                                             (int)M, (int)N, (int)K, a_code, b_code, (int)band, watchdog);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const void *a_elems, const uint8_t *a_sc, int a_fmt, const float *ga, const void *b_elems,
                        const uint8_t *b_sc, int b_fmt, const float *gb, void *c, int64_t M, int64_t N, int64_t K,
                        int *watchdog, int num_sms, cudaStream_t st) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return cudaErrorNotSupported;
    int kind;
    if (f8f6f4_code(a_fmt) >= 0 && a_fmt != FMT_E2M1 && f8f6f4_code(b_fmt) >= 0) kind = KIND_F8F6F4;
    else if (a_fmt == FMT_E2M1 && b_fmt == FMT_E2M1) kind = KIND_MXF4;
    else if (a_fmt == FMT_NVFP4 && b_fmt == FMT_NVFP4) kind = KIND_NVF4;
    else return cudaErrorInvalidValue;
    const int stage_k = kind == KIND_F8F6F4 ? 128 : 256;
    if (K % stage_k) return cudaErrorInvalidValue;
    // sub-byte codes are expanded by the copy for the mxf8f6f4 kind only
    const bool a_expand = kind == KIND_F8F6F4 && code_bits(a_fmt) < 8;
    const bool b_expand = kind == KIND_F8F6F4 && code_bits(b_fmt) < 8;
    CUtensorMap tmA, tmB;
    if (!encode_operand(enc, &tmA, a_elems, M, K, a_fmt, a_expand, kBM)) return cudaErrorInvalidValue;
    const bool wide = N % 256 == 0;
    const int bn = wide ? 256 : 128;
    if (!encode_operand(enc, &tmB, b_elems, N, K, b_fmt, b_expand, (uint32_t)bn)) return cudaErrorInvalidValue;
    const int64_t n_tiles = (M / kBM) * (N / bn);
    // band of N-tiles whose B panels (bn rows x K codes) take at most ~48 MB of L2
    const int64_t panel = (int64_t)bn * (K * code_bits(b_fmt) / 8);
    int64_t band = (48ll << 20) / (panel > 0 ? panel : 1);
    if (band < 1) band = 1;
    if (band > N / bn) band = N / bn;
    const int grid = (int)(n_tiles < num_sms ? n_tiles : num_sms);
    const uint32_t a_code = kind == KIND_F8F6F4 ? (uint32_t)f8f6f4_code(a_fmt) : 1u;
    const uint32_t b_code = kind == KIND_F8F6F4 ? (uint32_t)f8f6f4_code(b_fmt) : 1u;
    if (kind == KIND_F8F6F4)
        return wide ? launch_gemm_k<256, KIND_F8F6F4>(tmA, tmB, a_sc, b_sc, nullptr, nullptr, c, M, N, K, a_code, b_code, band, watchdog, grid, st)
                    : launch_gemm_k<128, KIND_F8F6F4>(tmA, tmB, a_sc, b_sc, nullptr, nullptr, c, M, N, K, a_code, b_code, band, watchdog, grid, st);
    if (kind == KIND_MXF4)
        return wide ? launch_gemm_k<256, KIND_MXF4>(tmA, tmB, a_sc, b_sc, nullptr, nullptr, c, M, N, K, a_code, b_code, band, watchdog, grid, st)
                    : launch_gemm_k<128, KIND_MXF4>(tmA, tmB, a_sc, b_sc, nullptr, nullptr, c, M, N, K, a_code, b_code, band, watchdog, grid, st);
    return wide ? launch_gemm_k<256, KIND_NVF4>(tmA, tmB, a_sc, b_sc, ga, gb, c, M, N, K, a_code, b_code, band, watchdog, grid, st)
                : launch_gemm_k<128, KIND_NVF4>(tmA, tmB, a_sc, b_sc, ga, gb, c, M, N, K, a_code, b_code, band, watchdog, grid, st);
}

}  // namespace mxk
