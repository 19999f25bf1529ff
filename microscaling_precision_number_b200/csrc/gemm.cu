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
// Kernel structure (one CTA per 128 x 256 output tile, 6 warps):
//   warp 4  TMA producer: per 128-wide K step, 2-D TMA loads of the A tile (128 x 128 B)
//           and the B tile (256 x 128 B, E2M1 expanded by the TMA to one byte per
//           element) with 128-byte swizzle, plus bulk copies of the matching scale atoms
//           (1 for A, 2 for B) into a 4-stage shared-memory ring (mbarrier "full").
//   warp 5  TMEM allocator and MMA issuer: copies the stage's scale atoms into tensor
//           memory (tcgen05.cp 32x128b.warpx4), then issues four
//           tcgen05.mma.kind::mxf8f6f4.block_scale (K = 32 each; the scale byte of each
//           is selected by the scale-factor id in the instruction descriptor), and
//           releases the stage with tcgen05.commit on its "empty" barrier.
//   warps 0-3  epilogue: tcgen05.ld of the 128 x 256 fp32 accumulator, one TMEM lane
//           (= one output row) per thread, bf16 conversion, 16-byte global stores.
// All waits are bounded by the watchdog; tensor memory is always released.
#include <cuda.h>
#include "codec.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace mxk {

namespace {
constexpr int kBM = 128, kBK = 128;                      // tile rows; kBK in elements (= smem bytes)
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kABytes = kBM * kBK;                       // 16 KiB
constexpr int kSfaBytes = 512;
constexpr uint32_t kTmemCols = 512;                      // accumulator (<= 256) + scale slots
constexpr uint32_t kSfCol0 = 256;                        // first scale-slot column
constexpr uint32_t kSfColsPerStage = 16;                 // B: 8 at +0, A: 4 at +8
template <int BN> struct Tile {
    static constexpr int kBBytes = BN * kBK;             // 32 KiB for BN = 256
    static constexpr int kSfbBytes = 512 * (BN / 128);
    static constexpr int kSmemBytes = kStages * (kABytes + kBBytes + kSfaBytes + kSfbBytes) + 1024;
};
}  // namespace

// ---- tcgen05 wrappers -------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start >> 4 in bits 0-13, leading
// byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45, descriptor version 1 in
// bits 46-47, swizzle mode in 61-63 (2 = 128-byte swizzle, 0 = none).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t swz) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(swz & 7u) << 61;
    return d;
}

// Instruction descriptor for kind::mxf8f6f4 with block scaling: B scale-factor id in
// bits 4-5, A format 7-9, B format 10-12 (E4M3 = 0, E2M1 = 5), K-major A and B, N >> 3
// in 17-22, scale type E8M0 (bit 23 = 1), M >> 4 in 24-28, A scale-factor id in 29-30.
template <int BN>
__device__ __forceinline__ uint32_t mma_idesc(uint32_t b_fmt_code, uint32_t sf_id) {
    uint32_t d = 0;
    d |= (sf_id & 3u) << 4;
    d |= 0u << 7;                         // A: E4M3
    d |= (b_fmt_code & 7u) << 10;
    d |= (uint32_t)(BN >> 3) << 17;
    d |= 1u << 23;                        // UE8M0 scales
    d |= (uint32_t)(kBM >> 4) << 24;
    d |= (sf_id & 3u) << 29;
    return d;
}

__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Copy a 512-byte scale atom (32 rows x 16 bytes, contiguous) into 4 TMEM columns,
// replicated into all four 32-lane sub-partitions.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint32_t saddr) {
    const uint64_t d = smem_desc(saddr, 16, 128, 0);
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- kernel ------------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const uint8_t *__restrict__ a_sc, const uint8_t *__restrict__ b_sc,
               uint16_t *__restrict__ C, int M, int N, int K, uint32_t b_fmt_code, int *watchdog) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;                                   // kStages x 16 KiB (1024-aligned)
    constexpr int kBBytes = Tile<BN>::kBBytes, kSfbBytes = Tile<BN>::kSfbBytes;
    uint8_t *sB = sA + kStages * kABytes;                 // kStages x BN x 128 B
    uint8_t *sSFA = sB + kStages * kBBytes;               // kStages x 512 B
    uint8_t *sSFB = sSFA + kStages * kSfaBytes;           // kStages x 512 B per 128 rows of B

    __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], acc_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int fail_flag;
    volatile int *fail_sh = &fail_flag;
    int last_kb[kStages];                                 // producer: last K step armed per stage

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_blk = blockIdx.x, m_blk = blockIdx.y;
    const int num_kb = K / kBK;

    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        for (int s = 0; s < kStages; s++) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
        mbar_init(&acc_bar, 1);
        *fail_sh = 0;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(&tmem_base_sh, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        for (int s = 0; s < kStages; s++) last_kb[s] = -1;
        if (lane == 0) {
            const int64_t kb128 = K / 128;
            for (int kb = 0; kb < num_kb; kb++) {
                const int s = kb % kStages;
                if (kb >= kStages) {
                    if (!mbar_wait_bounded(&empty_bar[s], (uint32_t)((kb / kStages) - 1) & 1u, watchdog, WD_GEMM_EMPTY)) {
                        *fail_sh = 1;
                        break;
                    }
                }
                if (*fail_sh) break;
                // An E2M1 tile lands in shared memory padded to one byte per element
                // (16U4_ALIGN16B), but the copy completes only the packed global bytes.
                mbar_arrive_expect_tx(&full_bar[s], kABytes + (b_fmt_code == 5u ? kBBytes / 2 : kBBytes) +
                                                        kSfaBytes + kSfbBytes);
                tma_load_2d(sA + s * kABytes, &tmA, kb * kBK, m_blk * kBM, &full_bar[s]);
                tma_load_2d(sB + s * kBBytes, &tmB, kb * kBK, n_blk * BN, &full_bar[s]);
                bulk_load(sSFA + s * kSfaBytes, a_sc + ((int64_t)m_blk * kb128 + kb) * 512, kSfaBytes, &full_bar[s]);
#pragma unroll
                for (int h = 0; h < BN / 128; h++)
                    bulk_load(sSFB + s * kSfbBytes + h * 512,
                              b_sc + ((int64_t)((BN / 128) * n_blk + h) * kb128 + kb) * 512, 512, &full_bar[s]);
                last_kb[s] = kb;
            }
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            for (int kb = 0; kb < num_kb; kb++) {
                const int s = kb % kStages;
                if (!mbar_wait_bounded(&full_bar[s], (uint32_t)(kb / kStages) & 1u, watchdog, WD_GEMM_FULL)) {
                    *fail_sh = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t sfb_t = tmem + kSfCol0 + s * kSfColsPerStage;
                const uint32_t sfa_t = sfb_t + 8;
                tc_cp_sf(sfa_t, smem_u32(sSFA + s * kSfaBytes));
#pragma unroll
                for (int h = 0; h < BN / 128; h++) tc_cp_sf(sfb_t + 4 * h, smem_u32(sSFB + s * kSfbBytes + h * 512));
                const uint32_t a_base = smem_u32(sA + s * kABytes);
                const uint32_t b_base = smem_u32(sB + s * kBBytes);
#pragma unroll
                for (int k = 0; k < kBK / 32; k++) {
                    const uint64_t ad = smem_desc(a_base + k * 32, 16, 1024, 2);
                    const uint64_t bd = smem_desc(b_base + k * 32, 16, 1024, 2);
                    tc_mma_mx(tmem, ad, bd, mma_idesc<BN>(b_fmt_code, (uint32_t)k), sfa_t, sfb_t,
                              (kb > 0 || k > 0) ? 1u : 0u);
                }
                tc_commit(&empty_bar[s]);
            }
            tc_commit(&acc_bar);   // completes when every MMA issued above has finished
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 0-3)
        const bool ok = mbar_wait_bounded(&acc_bar, 0u, watchdog, WD_GEMM_ACC);
        tc_fence_after();
        if (ok && !*fail_sh) {
            const int row = m_blk * kBM + warp * 32 + lane;
            uint16_t *crow = C + (int64_t)row * N + (int64_t)n_blk * BN;
            const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
            for (int j = 0; j < BN / 32; j++) {
                uint32_t r[32];
                tmem_ld32(t_row + j * 32, r);
                uint4 *dst = reinterpret_cast<uint4 *>(crow + j * 32);
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint4 o;
                    o.x = f32x2_to_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
                    o.y = f32x2_to_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
                    o.z = f32x2_to_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
                    o.w = f32x2_to_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
                    dst[q] = o;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*fail_sh && warp == 4 && lane == 0) {
        // Error path: wait (bounded) for the loads this CTA armed, and for the MMAs it
        // issued (the final commit above), before shared and tensor memory go away.
        for (int s = 0; s < kStages; s++)
            if (last_kb[s] >= 0) (void)mbar_wait_bounded(&full_bar[s], (uint32_t)(last_kb[s] / kStages) & 1u, nullptr, 0, kDrainLimitNs);
        (void)mbar_wait_bounded(&acc_bar, 0u, nullptr, 0, kDrainLimitNs);
    }
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static bool encode_operand(EncodeTiledFn enc, CUtensorMap *tm, const void *ptr, int64_t rows, int64_t K,
                           bool fp4, uint32_t box_rows) {
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)(fp4 ? K / 2 : K)};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(tm, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                           const_cast<void *>(ptr), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm(const void *a_elems, const uint8_t *a_sc, const void *b_elems, const uint8_t *b_sc,
                        int b_fmt, void *c, int64_t M, int64_t N, int64_t K, int *watchdog, int num_sms,
                        cudaStream_t st) {
    (void)num_sms;
    auto enc = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap tmA, tmB;
    const bool fp4 = b_fmt == FMT_E2M1;
    if (!encode_operand(enc, &tmA, a_elems, M, K, false, kBM)) return cudaErrorInvalidValue;
    const bool wide = N % 256 == 0;
    const int bn = wide ? 256 : 128;
    if (!encode_operand(enc, &tmB, b_elems, N, K, fp4, (uint32_t)bn)) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)(N / bn), (unsigned)(M / kBM));
    cudaError_t e;
    if (wide) {
        e = cudaFuncSetAttribute(mx_gemm_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile<256>::kSmemBytes);
        if (e != cudaSuccess) return e;
        mx_gemm_kernel<256><<<grid, kGemmThreads, Tile<256>::kSmemBytes, st>>>(
            tmA, tmB, a_sc, b_sc, static_cast<uint16_t *>(c), (int)M, (int)N, (int)K, fp4 ? 5u : 0u, watchdog);
    } else {
        e = cudaFuncSetAttribute(mx_gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, Tile<128>::kSmemBytes);
        if (e != cudaSuccess) return e;
        mx_gemm_kernel<128><<<grid, kGemmThreads, Tile<128>::kSmemBytes, st>>>(
            tmA, tmB, a_sc, b_sc, static_cast<uint16_t *>(c), (int)M, (int)N, (int)K, fp4 ? 5u : 0u, watchdog);
    }
    return cudaGetLastError();
}

}  // namespace mxk
