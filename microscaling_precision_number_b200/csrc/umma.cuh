// umma.cuh -- tcgen05 (5th-generation tensor core) wrappers shared by the block-scaled
// matmul kernels: tensor-memory allocation, descriptors, the three block-scaled MMA kinds,
// scale-factor copies into tensor memory, accumulator loads, and the banded tile order.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace mxk {

// MMA kinds: E4M3 x {E4M3, E2M1 expanded to bytes} with E8M0 scales per 32 (one scale
// per row per K = 32 instruction); E2M1 x E2M1 packed with E8M0 scales per 32 (two per
// K = 64 instruction); E2M1 x E2M1 packed with UE4M3 scales per 16 (four per K = 64).
enum : int { KIND_F8F6F4 = 0, KIND_MXF4 = 1, KIND_NVF4 = 2 };

// mxf8f6f4 operand format code of an element format (E4M3 0, E5M2 1, E2M3 3, E3M2 4,
// E2M1 5), or -1 when the format is not an operand of that kind.
__host__ __device__ constexpr int f8f6f4_code(int fmt) {
    return fmt == 0 ? 0 : fmt == 1 ? 1 : fmt == 4 ? 3 : fmt == 5 ? 4 : fmt == 2 ? 5 : -1;
}

// Global bytes behind `smem_bytes` of an mxf8f6f4 operand tile.  FP4 (code 5) and FP6
// (codes 3, 4) are stored packed and the copy expands each 16 codes to a 16-byte group in
// shared memory (16U4_ALIGN16B: 8 code bytes; 16U6_ALIGN16B: 12); the copy's transaction
// count is the packed size.
__host__ __device__ constexpr uint32_t f8f6f4_packed_bytes(uint32_t smem_bytes, uint32_t code) {
    return code == 5u ? smem_bytes / 2 : (code == 3u || code == 4u) ? smem_bytes / 4 * 3 : smem_bytes;
}

// ---- tcgen05 wrappers -------------------------------------------------------------------
// Tensor-memory allocation by one full warp.  With CG = 2 the instruction is collective
// over the CTA pair: the warp with the same index in both CTAs executes it, and both pass
// the same shared-memory offset for the returned address.
template <int CG = 1>
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    if constexpr (CG == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    } else {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
}
template <int CG = 1>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    if constexpr (CG == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
    else
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive once on `bar` when every tcgen05 operation this thread issued before has
// completed.  The pair form arrives on the barrier at the same offset in each CTA of the
// pair (mask 0b11).
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
// Pair form without multicast: arrives on `bar` in the issuing CTA only.
__device__ __forceinline__ void tc_commit_pair_local(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    const uint16_t mask = 3;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(mask) : "memory");
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

// Instruction descriptor for the block-scaled kinds: B scale-factor id (first scale byte
// of the 32-bit tensor-memory word) in bits 4-5, A format 7-9, B format 10-12 (mxf8f6f4:
// E4M3 = 0, E5M2 = 1, E2M3 = 3, E3M2 = 4, E2M1 = 5; mxf4 / mxf4nvf4: E2M1 = 1), K-major A and B, N >> 3 in 17-22, scale
// type in bit 23 (1 = UE8M0, 0 = UE4M3), M >> 4 in 24-28, A scale-factor id in 29-30,
// bit 31 = 0 (dense K of 32 for 8-bit kinds, 64 for 4-bit kinds).
template <int BM, int BN, int KIND>
__device__ __forceinline__ uint32_t mma_idesc(uint32_t a_fmt_code, uint32_t b_fmt_code, uint32_t sf_id) {
    const uint32_t a_fmt = KIND == KIND_F8F6F4 ? a_fmt_code : 1u;
    const uint32_t b_fmt = KIND == KIND_F8F6F4 ? b_fmt_code : 1u;
    uint32_t d = 0;
    d |= (sf_id & 3u) << 4;
    d |= a_fmt << 7;
    d |= (b_fmt & 7u) << 10;
    d |= (uint32_t)(BN >> 3) << 17;
    d |= (KIND == KIND_NVF4 ? 0u : 1u) << 23;
    d |= (uint32_t)(BM >> 4) << 24;
    d |= (sf_id & 3u) << 29;
    return d;
}

template <int KIND, int CG = 1>
__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    if constexpr (KIND == KIND_F8F6F4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::%7.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "n"(CG)
            : "memory");
    } else if constexpr (KIND == KIND_MXF4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::%7.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "n"(CG)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::%7.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "n"(CG)
            : "memory");
    }
}

// Copy a 512-byte scale atom (32 rows x 16 bytes, contiguous) into 4 TMEM columns,
// replicated into all four 32-lane sub-partitions.
// With CG = 2 (issued by the pair's MMA thread) each CTA's atom at the same shared-memory
// offset goes to the same columns of that CTA's own tensor memory.
// Shared-memory descriptor of a scale atom (512 bytes, no swizzle) at saddr.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) { return smem_desc(saddr, 16, 128, 0); }

// The copy with a ready descriptor d (the MMA loops advance one base descriptor by
// offsets >> 4 instead of rebuilding it on the issuing thread's critical path).
template <int CG = 1>
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t d) {
    if constexpr (CG == 1)
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
    else
        asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// NJ x 32 columns (columns taddr + 32 j) with one wait for all of them: a single
// 128-column load when NJ = 4 (measured 0.5-2% faster matmuls than four 32-column loads,
// the accumulator hand-off being on the per-tile critical path), else NJ 32-column loads
// back to back.  The empty asm statements after the wait tie every loaded register to it,
// so no use of r can be scheduled before the data has landed.
template <int NJ>
__device__ __forceinline__ void tmem_ld32_batch(uint32_t taddr, uint32_t (&r)[NJ][32]) {
    if constexpr (NJ == 4) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, "
            "%21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, "
            "%40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, "
            "%59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, "
            "%78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, "
            "%97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, "
            "%114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];"
            : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]),
              "=r"(r[0][6]), "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]),
              "=r"(r[0][12]), "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]), "=r"(r[0][16]), "=r"(r[0][17]),
              "=r"(r[0][18]), "=r"(r[0][19]), "=r"(r[0][20]), "=r"(r[0][21]), "=r"(r[0][22]), "=r"(r[0][23]),
              "=r"(r[0][24]), "=r"(r[0][25]), "=r"(r[0][26]), "=r"(r[0][27]), "=r"(r[0][28]), "=r"(r[0][29]),
              "=r"(r[0][30]), "=r"(r[0][31]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]),
              "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]), "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]),
              "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]), "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15]),
              "=r"(r[1][16]), "=r"(r[1][17]), "=r"(r[1][18]), "=r"(r[1][19]), "=r"(r[1][20]), "=r"(r[1][21]),
              "=r"(r[1][22]), "=r"(r[1][23]), "=r"(r[1][24]), "=r"(r[1][25]), "=r"(r[1][26]), "=r"(r[1][27]),
              "=r"(r[1][28]), "=r"(r[1][29]), "=r"(r[1][30]), "=r"(r[1][31]), "=r"(r[2][0]), "=r"(r[2][1]),
              "=r"(r[2][2]), "=r"(r[2][3]), "=r"(r[2][4]), "=r"(r[2][5]), "=r"(r[2][6]), "=r"(r[2][7]),
              "=r"(r[2][8]), "=r"(r[2][9]), "=r"(r[2][10]), "=r"(r[2][11]), "=r"(r[2][12]), "=r"(r[2][13]),
              "=r"(r[2][14]), "=r"(r[2][15]), "=r"(r[2][16]), "=r"(r[2][17]), "=r"(r[2][18]), "=r"(r[2][19]),
              "=r"(r[2][20]), "=r"(r[2][21]), "=r"(r[2][22]), "=r"(r[2][23]), "=r"(r[2][24]), "=r"(r[2][25]),
              "=r"(r[2][26]), "=r"(r[2][27]), "=r"(r[2][28]), "=r"(r[2][29]), "=r"(r[2][30]), "=r"(r[2][31]),
              "=r"(r[3][0]), "=r"(r[3][1]), "=r"(r[3][2]), "=r"(r[3][3]), "=r"(r[3][4]), "=r"(r[3][5]),
              "=r"(r[3][6]), "=r"(r[3][7]), "=r"(r[3][8]), "=r"(r[3][9]), "=r"(r[3][10]), "=r"(r[3][11]),
              "=r"(r[3][12]), "=r"(r[3][13]), "=r"(r[3][14]), "=r"(r[3][15]), "=r"(r[3][16]), "=r"(r[3][17]),
              "=r"(r[3][18]), "=r"(r[3][19]), "=r"(r[3][20]), "=r"(r[3][21]), "=r"(r[3][22]), "=r"(r[3][23]),
              "=r"(r[3][24]), "=r"(r[3][25]), "=r"(r[3][26]), "=r"(r[3][27]), "=r"(r[3][28]), "=r"(r[3][29]),
              "=r"(r[3][30]), "=r"(r[3][31])
            : "r"(taddr));
    } else {
#pragma unroll
        for (int j = 0; j < NJ; j++)
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                : "=r"(r[j][0]), "=r"(r[j][1]), "=r"(r[j][2]), "=r"(r[j][3]), "=r"(r[j][4]), "=r"(r[j][5]),
                  "=r"(r[j][6]), "=r"(r[j][7]), "=r"(r[j][8]), "=r"(r[j][9]), "=r"(r[j][10]), "=r"(r[j][11]),
                  "=r"(r[j][12]), "=r"(r[j][13]), "=r"(r[j][14]), "=r"(r[j][15]), "=r"(r[j][16]), "=r"(r[j][17]),
                  "=r"(r[j][18]), "=r"(r[j][19]), "=r"(r[j][20]), "=r"(r[j][21]), "=r"(r[j][22]), "=r"(r[j][23]),
                  "=r"(r[j][24]), "=r"(r[j][25]), "=r"(r[j][26]), "=r"(r[j][27]), "=r"(r[j][28]), "=r"(r[j][29]),
                  "=r"(r[j][30]), "=r"(r[j][31])
                : "r"(taddr + 32u * (uint32_t)j));
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < NJ; j++)
        asm volatile("" : "+r"(r[j][0]), "+r"(r[j][1]), "+r"(r[j][2]), "+r"(r[j][3]), "+r"(r[j][4]), "+r"(r[j][5]), "+r"(r[j][6]), "+r"(r[j][7]), "+r"(r[j][8]), "+r"(r[j][9]), "+r"(r[j][10]), "+r"(r[j][11]), "+r"(r[j][12]), "+r"(r[j][13]), "+r"(r[j][14]), "+r"(r[j][15]), "+r"(r[j][16]), "+r"(r[j][17]), "+r"(r[j][18]), "+r"(r[j][19]), "+r"(r[j][20]), "+r"(r[j][21]), "+r"(r[j][22]), "+r"(r[j][23]), "+r"(r[j][24]), "+r"(r[j][25]), "+r"(r[j][26]), "+r"(r[j][27]), "+r"(r[j][28]), "+r"(r[j][29]), "+r"(r[j][30]), "+r"(r[j][31]));
}

// ---- tile order ------------------------------------------------------------------------------
// Banded raster: N-tiles are grouped into bands of `band` tiles whose B panels fit in L2;
// within a band the tiles run M-major, so concurrently resident CTAs share A panels and the
// band's B panels are read from HBM about once.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int band, int &m_blk, int &n_blk) {
    const int per_band = tiles_m * band;
    const int b = t / per_band;
    const int rem = t - b * per_band;
    const int n0 = b * band;
    const int bw = tiles_n - n0 < band ? tiles_n - n0 : band;   // the last band may be narrower
    m_blk = rem / bw;
    n_blk = n0 + (rem - m_blk * bw);
}

}  // namespace mxk
