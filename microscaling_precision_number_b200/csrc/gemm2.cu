// gemm2.cu -- the MX block-scaled matmul on CTA pairs (tcgen05 cta_group::2).
//
// Sources (page title, section): as gemm.cu --
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §2 "MXFP4 はブロック32と E8M0", §3 "NVFP4 はブロック16と E4M3、そして二段目",
//     §7 "ハードウェアの対応状況": block-scaled MMA on the 5th-generation tensor cores.
//
// Same product, formats and scale handling as gemm.cu, computed per 256 x 256 output tile
// by a cluster of two CTAs on two SMs:
//   - each CTA loads its own 128 rows of A and its own 128 rows (of 256) of B, plus its A
//     rows' scale atoms and the scale atoms of all 256 B rows, with 2-D TMA loads that all
//     complete on the even CTA's barriers (the `.cta_group::2` form with the peer bit of the
//     barrier address cleared; scale atoms and operand tiles on separate barriers);
//   - the even CTA's MMA thread copies the stage's scale atoms (each CTA's own shared
//     memory into its own tensor memory) and issues tcgen05.mma.cta_group::2 with M = 256:
//     the tensor core of each SM computes its CTA's 128 rows x 256 columns, reading A from
//     its own shared memory and B from both CTAs' shared memory;
//   - commits arrive on the barrier at the same offset in both CTAs (stage release,
//     accumulator ready); both CTAs' epilogues release the accumulator on the even CTA's
//     barrier (remote mbarrier arrive).
// Per SM a K step moves A 16 KiB + half of B 16 KiB instead of 16 + 32 KiB: a third less
// L2 -> SM traffic for the same MMA work, and 5-6 ring stages fit in shared memory.
// Every wait is bounded (watchdog); the pair leaves through a bounded handshake after the
// even CTA has drained its barriers and MMAs, so no copy or MMA touches a CTA that exited.
#include <cuda.h>
#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "umma.cuh"

namespace mxk {

namespace {
constexpr int kHalfRows = 128;                       // rows of A and of B per CTA
constexpr int kPairM = 256, kPairN = 256;            // output tile of the pair
constexpr int kRowBytes = 128;                       // bytes of K per row per stage
constexpr int kABytes = kHalfRows * kRowBytes;       // 16 KiB
constexpr int kBBytes = kHalfRows * kRowBytes;       // 16 KiB (this CTA's half of B)
constexpr int kProducerWarp = 8, kMmaWarp = 9, kSfWarp = 10, kEpilogueWarps = 8;
constexpr int kPairThreads = 352;
constexpr uint32_t kTmemCols = 512, kSfCol0 = 256;
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;       // shared::cluster address of the even CTA's copy

// A pipeline stage holds SUB sub-tiles of 128 bytes of K per row (one 128-byte-swizzled TMA
// box each): 4 x SUB MMAs per stage, so the per-stage barrier wait and commit of the
// issuing thread are shared by more tensor work.
template <int KIND, int SUB> struct Pair {
    static constexpr int kSubK = KIND == KIND_F8F6F4 ? 128 : 256;          // K per sub-tile
    static constexpr int kStageK = kSubK * SUB;
    static constexpr int kSubAtoms = KIND == KIND_F8F6F4 ? 1 : (KIND == KIND_MXF4 ? 2 : 4);
    static constexpr int kAtoms = kSubAtoms * SUB;   // scale atoms per 128 rows per stage
    static constexpr int kSfaBytes = 512 * kAtoms;   // this CTA's 128 A rows
    static constexpr int kSfbBytes = 1024 * kAtoms;  // all 256 B rows
    static constexpr int kAStage = kABytes * SUB, kBStage = kBBytes * SUB;
    static constexpr int kStageBytes = kAStage + kBStage + kSfaBytes + kSfbBytes;
    static constexpr int kStages = (220 * 1024) / kStageBytes > 6 ? 6 : (220 * 1024) / kStageBytes;
    static constexpr uint32_t kSfbCols = 8 * kAtoms;              // B atom (a, h) at 4 (2a + h)
    static constexpr uint32_t kSfColsPerStage = kSfbCols + 4 * kAtoms;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024;
    static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "tensor-memory scale slots");
    static_assert(kSmemBytes + 1024 <= 227 * 1024, "shared memory");
    static_assert(kStages >= 2, "pipeline depth");
};
// Sub-tiles per stage for each kind (the depth of the ring follows from the stage size).
template <int KIND> constexpr int kPairSub = 1;
}  // namespace

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 2-D TMA load into this CTA's shared memory whose completion is counted on the even CTA's
// barrier (same offset).
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const void *tmap, int32_t x, int32_t y,
                                                 uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y),
          "r"(smem_u32(bar) & kPeerBitMask)
        : "memory");
}
// Arrive (release, cluster scope) on the barrier at the same offset in CTA `rank`.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(bar)), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

template <int KIND, int SUB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                    const float *__restrict__ ga, const float *__restrict__ gb, uint16_t *__restrict__ C, int M,
                    int N, int K, uint32_t a_fmt_code, uint32_t b_fmt_code, int band, int *watchdog) {
    using P = Pair<KIND, SUB>;
    constexpr int S = P::kStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;                                  // S x SUB x 16 KiB (1024-aligned)
    uint8_t *sB = sA + S * P::kAStage;                   // S x SUB x 16 KiB
    uint8_t *sSFA = sB + S * P::kBStage;                 // S x kAtoms x 512 B
    uint8_t *sSFB = sSFA + S * P::kSfaBytes;             // S x 2 x kAtoms x 512 B

    __shared__ __align__(8) uint64_t full_bar[S], sf_full[S], empty_bar[S], sf_ready[S], acc_full, acc_empty, drain_bar,
        sf_drain, exit_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int fail_flag;
    volatile int *fail_sh = &fail_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int num_kb = K / P::kStageK;
    const int tiles_n = N / kPairN, tiles_m = M / kPairM;
    const int n_tiles = tiles_m * tiles_n;
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmSA);
        prefetch_tensormap(&tmSB);
        for (int s = 0; s < S; s++) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&sf_full[s], 1);
            mbar_init(&empty_bar[s], 1);
            mbar_init(&sf_ready[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, 2 * kEpilogueWarps);
        mbar_init(&drain_bar, 1);
        mbar_init(&sf_drain, 1);
        mbar_init(&exit_bar, 1);
        *fail_sh = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc<2>(&tmem_base_sh, kTmemCols);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                                  // both CTAs' barriers exist before any remote use
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    int last_it[S];                                      // producer: last ring use armed per stage
    for (int s = 0; s < S; s++) last_it[s] = -1;
    if (warp == kProducerWarp) {
        // ------------------------------------------------ TMA producer (both CTAs)
        // the whole warp runs the loop; one elected lane issues the copies
        const int col_atoms = num_kb * P::kAtoms;            // scale atoms per 128-row block
        const uint32_t tx_ops =
            2u * SUB * ((KIND == KIND_F8F6F4 ? f8f6f4_packed_bytes(kABytes, a_fmt_code) : kABytes) +
                        (KIND == KIND_F8F6F4 ? f8f6f4_packed_bytes(kBBytes, b_fmt_code) : kBBytes));
        const uint32_t tx_sf = 2u * (P::kSfaBytes + P::kSfbBytes);
        int it = 0;
        for (int t = pair; t < n_tiles && !warp_failed(fail_sh); t += n_pairs) {
            int m_blk, n_blk;
            tile_coords(t, tiles_m, tiles_n, band, m_blk, n_blk);
            const int a_row = m_blk * kPairM + (int)rank * kHalfRows;
            const int b_row = n_blk * kPairN + (int)rank * kHalfRows;
            for (int kb = 0; kb < num_kb; kb++, it++) {
                const int s = it % S;
                if (it >= S && !warp_wait(&empty_bar[s], (uint32_t)((it / S) - 1) & 1u, watchdog, WD_GEMM_EMPTY)) {
                    *fail_sh = 1;
                    break;
                }
                if (elect_one()) {
                    if (leader) {
                        mbar_arrive_expect_tx(&sf_full[s], tx_sf);
                        mbar_arrive_expect_tx(&full_bar[s], tx_ops);
                    }
                    // scale atoms first, on their own barrier, so that their copy into tensor
                    // memory overlaps the landing of the operand tiles; atoms as rows of 256
                    // bytes (two per atom), a stage's atoms of one 128-row block contiguous
                    tma_load_2d_pair(sSFA + s * P::kSfaBytes, &tmSA, 0,
                                     2 * ((2 * m_blk + (int)rank) * col_atoms + kb * P::kAtoms), &sf_full[s]);
#pragma unroll
                    for (int h = 0; h < 2; h++)
                        tma_load_2d_pair(sSFB + s * P::kSfbBytes + h * P::kSfaBytes, &tmSB, 0,
                                         2 * ((2 * n_blk + h) * col_atoms + kb * P::kAtoms), &sf_full[s]);
#pragma unroll
                    for (int j = 0; j < SUB; j++) {
                        const int kx = (kb * SUB + j) * kRowBytes;
                        tma_load_2d_pair(sA + s * P::kAStage + j * kABytes, &tmA, kx, a_row, &full_bar[s]);
                        tma_load_2d_pair(sB + s * P::kBStage + j * kBBytes, &tmB, kx, b_row, &full_bar[s]);
                    }
                }
                __syncwarp();
                last_it[s] = it;
            }
        }
    } else if (warp == kSfWarp) {
        // ------------------------------------------------ scale-atom copier (even CTA only)
        // Copies each stage's scale atoms into tensor memory (both CTAs') as soon as they
        // have landed (sf_full[s]: the atoms travel apart from the operand tiles and are
        // issued first, so the copies overlap the tiles' landing), and signals sf_ready[s]
        // once the copies are complete.  The MMA issuer waits on full[s] (operands) and
        // sf_ready[s], so the copies stay off the MMA-issuing warp.  A stage's scale slot is
        // rewritten only after sf_full[s] of its next use, which the producer arms after
        // empty[s], i.e. after the MMAs that read the slot have completed.
        if (leader) {
            const uint64_t sfa_d0 = sf_desc(smem_u32(sSFA)), sfb_d0 = sf_desc(smem_u32(sSFB));
            int it = 0;
            for (int t = pair; t < n_tiles && !warp_failed(fail_sh); t += n_pairs) {
                for (int kb = 0; kb < num_kb; kb++, it++) {
                    const int s = it % S;
                    if (!warp_wait(&sf_full[s], (uint32_t)(it / S) & 1u, watchdog, WD_GEMM_FULL)) {
                        *fail_sh = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfb_t = tmem + kSfCol0 + s * P::kSfColsPerStage;
                    const uint32_t sfa_t = sfb_t + P::kSfbCols;
                    const uint64_t sfa_d = sfa_d0 + (uint64_t)((s * P::kSfaBytes) >> 4);
                    const uint64_t sfb_d = sfb_d0 + (uint64_t)((s * P::kSfbBytes) >> 4);
                    if (elect_one()) {
#pragma unroll
                        for (int a = 0; a < P::kAtoms; a++) {
                            tc_cp_sf<2>(sfa_t + 4 * a, sfa_d + (uint64_t)(a * 512 / 16));
#pragma unroll
                            for (int h = 0; h < 2; h++)
                                tc_cp_sf<2>(sfb_t + 4 * (2 * a + h),
                                            sfb_d + (uint64_t)((h * P::kSfaBytes + a * 512) / 16));
                        }
                        tc_commit_pair_local(&sf_ready[s]);  // the stage's scales are in tensor memory
                    }
                    __syncwarp();
                }
            }
            if (elect_one()) tc_commit_pair_local(&sf_drain);   // completes once every copy has finished
            __syncwarp();
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------ MMA issuer (even CTA only)
        if (leader) {
            // descriptors precomputed and advanced by offsets; the whole warp runs the loop
            // and one elected lane issues each stage's MMAs and its commit
            const uint64_t a_d0 = smem_desc(smem_u32(sA), 16, 1024, 2), b_d0 = smem_desc(smem_u32(sB), 16, 1024, 2);
            uint32_t idesc[4];
#pragma unroll
            for (int k = 0; k < 4; k++)
                idesc[k] = mma_idesc<kPairM, kPairN, KIND>(
                    a_fmt_code, b_fmt_code,
                    KIND == KIND_F8F6F4 ? (uint32_t)k : (KIND == KIND_MXF4 ? 2u * (k & 1) : 0u));
            int it = 0, i = 0;
            for (int t = pair; t < n_tiles && !warp_failed(fail_sh); t += n_pairs, i++) {
                if (i > 0 && !warp_wait(&acc_empty, (uint32_t)(i - 1) & 1u, watchdog, WD_GEMM_ACC)) {
                    *fail_sh = 1;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < num_kb; kb++, it++) {
                    const int s = it % S;
                    // the stage's operands have landed and its scales are in tensor memory
                    if (!warp_wait(&full_bar[s], (uint32_t)(it / S) & 1u, watchdog, WD_GEMM_FULL) ||
                        !warp_wait(&sf_ready[s], (uint32_t)(it / S) & 1u, watchdog, WD_GEMM_FULL)) {
                        *fail_sh = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sfb_t = tmem + kSfCol0 + s * P::kSfColsPerStage;
                    const uint32_t sfa_t = sfb_t + P::kSfbCols;
                    if (elect_one()) {
#pragma unroll
                        for (int j = 0; j < SUB; j++) {
                            const uint64_t a_d = a_d0 + (uint64_t)((s * P::kAStage + j * kABytes) >> 4);
                            const uint64_t b_d = b_d0 + (uint64_t)((s * P::kBStage + j * kBBytes) >> 4);
#pragma unroll
                            for (int k = 0; k < 4; k++) {
                                const int a = j * P::kSubAtoms +
                                              (KIND == KIND_F8F6F4 ? 0 : (KIND == KIND_MXF4 ? k >> 1 : k));
                                tc_mma_mx<KIND, 2>(tmem, a_d + (uint64_t)(2 * k), b_d + (uint64_t)(2 * k), idesc[k],
                                                   sfa_t + 4 * a, sfb_t + 8 * a, (kb > 0 || j > 0 || k > 0) ? 1u : 0u);
                            }
                        }
                        tc_commit_pair(&empty_bar[s]);       // stage s free in both CTAs
                    }
                    __syncwarp();
                }
                if (warp_failed(fail_sh)) break;
                if (elect_one()) tc_commit_pair(&acc_full);  // both halves of the tile are complete
                __syncwarp();
            }
            if (elect_one()) tc_commit_pair(&drain_bar);     // completes once every MMA above has finished
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue (warps 0-7, both CTAs)
        constexpr int kHalf = kPairN / 2;
        const int quad = warp & 3, half = warp >> 2;
        const uint32_t t_base = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(half * kHalf);
        const float alpha = (ga && gb) ? __fmul_rn(__ldg(ga), __ldg(gb)) : 1.0f;
        int i = 0;
        for (int t = pair; t < n_tiles; t += n_pairs, i++) {
            const bool ok = mbar_wait_bounded(&acc_full, (uint32_t)i & 1u, watchdog, WD_GEMM_ACC);
            if (!ok || *fail_sh) { *fail_sh = 1; break; }
            tc_fence_after();
            // the whole row segment comes out of tensor memory first (one wait), so the
            // accumulator is released before the conversion and the stores
            uint32_t r[kHalf / 32][32];
            tmem_ld32_batch<kHalf / 32>(t_base, r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(&acc_empty, 0);   // on the even CTA's barrier
            int m_blk, n_blk;
            tile_coords(t, tiles_m, tiles_n, band, m_blk, n_blk);
            const int row = m_blk * kPairM + (int)rank * kHalfRows + quad * 32 + lane;
            uint4 *dst = reinterpret_cast<uint4 *>(C + (int64_t)row * N + (int64_t)n_blk * kPairN + half * kHalf);
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

    // teardown: the even CTA waits (bounded) for the copies it counted and for every MMA;
    // the odd CTA waits for the MMAs too (they write its tensor memory); then a bounded
    // handshake, so that neither CTA releases tensor memory or exits while the pair's
    // copies or MMAs may still use the other's memory
    __syncthreads();
    // error path: the even CTA's producer (whose record of the armed stages this is) waits
    // for the pair's copies that were counted on its barriers
    if (warp == kProducerWarp && lane == 0 && leader && *fail_sh)
        for (int s = 0; s < S; s++)
            if (last_it[s] >= 0) {
                (void)mbar_wait_bounded(&sf_full[s], (uint32_t)(last_it[s] / S) & 1u, nullptr, 0, kDrainLimitNs);
                (void)mbar_wait_bounded(&full_bar[s], (uint32_t)(last_it[s] / S) & 1u, nullptr, 0, kDrainLimitNs);
            }
    __syncthreads();
    if (warp == kMmaWarp && lane == 0) {
        (void)mbar_wait_bounded(&drain_bar, 0u, nullptr, 0, kDrainLimitNs);
        if (leader) (void)mbar_wait_bounded(&sf_drain, 0u, nullptr, 0, kDrainLimitNs);   // scale copies too
        // the odd CTA's copies complete on the even CTA's barriers, so it stays until the
        // even CTA has drained them: each CTA arrives on the other's exit barrier
        mbar_arrive_remote(&exit_bar, rank ^ 1u);
        (void)mbar_wait_bounded(&exit_bar, 0u, nullptr, 0, 2 * kWaitLimitNs);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc<2>(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// Operand codes: rows x K, 128 bytes of K x 128 rows per box, 128-byte swizzle (as gemm.cu;
// E2M1 / FP6 codes of the mxf8f6f4 kind expanded by the copy to 16-byte groups).
static bool encode_codes(EncodeTiledFn enc, CUtensorMap *tm, const void *ptr, int64_t rows, int64_t K, int fmt,
                         bool expand) {
    const int bits = code_bits(fmt);
    const cuuint64_t gdim[2] = {(cuuint64_t)(expand || bits == 8 ? K : K * bits / 8), (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)(K * bits / 8)};
    const cuuint32_t box[2] = {(cuuint32_t)kRowBytes, (cuuint32_t)kHalfRows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = !expand ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : bits == 6 ? CU_TENSOR_MAP_DATA_TYPE_16U6_ALIGN16B
                                               : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
    return enc(tm, dt, 2,
               const_cast<void *>(ptr), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// tcgen05-tiled scales (rows/128 x col_atoms atoms of 512 B) viewed as 256-byte rows, two
// per atom; a box is the kAtoms consecutive atoms of one 128-row block in one stage.
static bool encode_scales(EncodeTiledFn enc, CUtensorMap *tm, const uint8_t *ptr, int64_t rows, int64_t col_atoms,
                          int atoms_per_box) {
    const cuuint64_t gdim[2] = {256, (cuuint64_t)((rows / 128) * col_atoms * 2)};
    const cuuint64_t gstride[1] = {256};
    const cuuint32_t box[2] = {256, (cuuint32_t)(2 * atoms_per_box)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(ptr), gdim, gstride, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND, int SUB>
static cudaError_t launch_pair_s(EncodeTiledFn enc, const void *a, const uint8_t *a_sc, const float *ga, int a_fmt,
                                 const void *b, const uint8_t *b_sc, const float *gb, int b_fmt, uint32_t a_code,
                                 uint32_t b_code, void *c, int64_t M, int64_t N, int64_t K, int *watchdog,
                                 int num_sms, cudaStream_t st) {
    using P = Pair<KIND, SUB>;
    CUtensorMap tmA, tmB, tmSA, tmSB;
    const int64_t col_atoms = (K / P::kStageK) * P::kAtoms;
    const bool a_expand = KIND == KIND_F8F6F4 && code_bits(a_fmt) < 8;
    const bool b_expand = KIND == KIND_F8F6F4 && code_bits(b_fmt) < 8;
    if (!encode_codes(enc, &tmA, a, M, K, a_fmt, a_expand) ||
        !encode_codes(enc, &tmB, b, N, K, b_fmt, b_expand) ||
        !encode_scales(enc, &tmSA, a_sc, M, col_atoms, P::kAtoms) ||
        !encode_scales(enc, &tmSB, b_sc, N, col_atoms, P::kAtoms))
        return cudaErrorInvalidValue;
    const int64_t n_tiles = (M / kPairM) * (N / kPairN);
    const int64_t panel = (int64_t)kPairN * (K * code_bits(b_fmt) / 8);
    int64_t band = (48ll << 20) / (panel > 0 ? panel : 1);
    if (band < 1) band = 1;
    if (band > N / kPairN) band = N / kPairN;
    int64_t pairs = num_sms / 2;
    if (pairs > n_tiles) pairs = n_tiles;
    if (pairs < 1) pairs = 1;
    auto k = mx_gemm_pair_kernel<KIND, SUB>;
    const OutRange rng[1] = {{c, (uint64_t)(M * N * 2)}};
    cudaError_t e = set_out_ranges(rng, st);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, P::kSmemBytes);
    if (e != cudaSuccess) return e;
    k<<<(unsigned)(2 * pairs), kPairThreads, P::kSmemBytes, st>>>(tmA, tmB, tmSA, tmSB, ga, gb,
                                                                   static_cast<uint16_t *>(c), (int)M, (int)N,
                                                                   (int)K, a_code, b_code, (int)band, watchdog);
    return cudaGetLastError();
}

// The kind's sub-tiles per stage when K is a multiple of the stage's K, else one.
template <int KIND>
static cudaError_t launch_pair_k(EncodeTiledFn enc, const void *a, const uint8_t *a_sc, const float *ga, int a_fmt,
                                 const void *b, const uint8_t *b_sc, const float *gb, int b_fmt, uint32_t a_code,
                                 uint32_t b_code, void *c, int64_t M, int64_t N, int64_t K, int *watchdog,
                                 int num_sms, cudaStream_t st) {
    constexpr int SUB = kPairSub<KIND>;
    if (SUB > 1 && K % Pair<KIND, SUB>::kStageK == 0)
        return launch_pair_s<KIND, SUB>(enc, a, a_sc, ga, a_fmt, b, b_sc, gb, b_fmt, a_code, b_code, c, M, N, K,
                                        watchdog, num_sms, st);
    return launch_pair_s<KIND, 1>(enc, a, a_sc, ga, a_fmt, b, b_sc, gb, b_fmt, a_code, b_code, c, M, N, K, watchdog,
                                  num_sms, st);
}

bool gemm_pair_supported(int64_t M, int64_t N) { return M % kPairM == 0 && N % kPairN == 0; }

cudaError_t launch_gemm_pair(const void *a_elems, const uint8_t *a_sc, int a_fmt, const float *ga,
                             const void *b_elems, const uint8_t *b_sc, int b_fmt, const float *gb, void *c,
                             int64_t M, int64_t N, int64_t K, int *watchdog, int num_sms, cudaStream_t st) {
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return cudaErrorNotSupported;
    if (!gemm_pair_supported(M, N)) return cudaErrorInvalidValue;
    if (f8f6f4_code(a_fmt) >= 0 && a_fmt != FMT_E2M1 && f8f6f4_code(b_fmt) >= 0) {
        if (K % 128) return cudaErrorInvalidValue;
        return launch_pair_k<KIND_F8F6F4>(enc, a_elems, a_sc, nullptr, a_fmt, b_elems, b_sc, nullptr, b_fmt,
                                          (uint32_t)f8f6f4_code(a_fmt), (uint32_t)f8f6f4_code(b_fmt), c, M, N, K,
                                          watchdog, num_sms, st);
    }
    if (K % 256) return cudaErrorInvalidValue;
    if (a_fmt == FMT_E2M1 && b_fmt == FMT_E2M1)
        return launch_pair_k<KIND_MXF4>(enc, a_elems, a_sc, nullptr, a_fmt, b_elems, b_sc, nullptr, b_fmt, 1u, 1u, c,
                                        M, N, K, watchdog, num_sms, st);
    if (a_fmt == FMT_NVFP4 && b_fmt == FMT_NVFP4)
        return launch_pair_k<KIND_NVF4>(enc, a_elems, a_sc, ga, a_fmt, b_elems, b_sc, gb, b_fmt, 1u, 1u, c, M, N, K,
                                        watchdog, num_sms, st);
    return cudaErrorInvalidValue;
}

}  // namespace mxk
