// stream.cu -- bulk-copy pipelined streaming kernels: row-wise MX quantiser, NVFP4
// tensor maximum and quantiser, MX / NVFP4 dequantisers.
//
// Sources (page title, section):
//   "MXFP4 と NVFP4 は何が違うのか調べてみた"
//     §2 "MXFP4 はブロック32と E8M0": 32 contiguous elements share one E8M0 scale; a NaN
//        scale makes the whole block NaN; the element cast rounds to nearest even.
//     §3 "NVFP4 はブロック16と E4M3、そして二段目": 16-element blocks with an unsigned
//        E4M3 scale and an FP32 per-tensor scale = tensor amax / (6 * 448).
//     §4 "精度の差はどこから出るか": floor and no-clip shared-exponent rules.
//     §7 "ハードウェアの対応状況": MX scales apply as an exponent add (exact); NVFP4 applies
//        an FP8 multiply then an FP32 multiply.
//
// Every kernel here is HBM-bound.  Structure shared by all of them:
//   - persistent CTAs, a few per SM, walk fixed-size tiles of consecutive blocks;
//   - one thread streams each tile into a 4-stage shared-memory ring with a single 1-D
//     bulk copy (cp.async.bulk, completion on an mbarrier), so each SM keeps >100 KB of
//     loads in flight with almost no issue cost;
//   - one thread owns one quantisation block: the block maximum and the scale are
//     computed once per block, never replicated across lanes;
//   - shared-memory reads of a thread's block are rotated per thread so that every
//     8-thread wavefront touches 8 distinct 16-byte bank groups (conflict-free);
//   - 32-bit indices; the tcgen05 scale offset divides by the scales-per-row count with
//     a precomputed multiply-shift (no integer division instruction).
// Waits are bounded (watchdog); a CTA that gives up drains its own copies and returns.
#include <cstdlib>
#include <mutex>
#include <set>
#include <utility>

#include "checked.cuh"
#include "codec.cuh"
#include "internal.h"
#include "nvfp4.cuh"
#include "ptx.cuh"
#include "tiling.cuh"

namespace mxk {

namespace {
constexpr int kThreads = 256;
constexpr int kStages = 4;
constexpr int kTileBytes = 16384;
constexpr int kCtasPerSm = 3;
}  // namespace

// ---- tile ring ------------------------------------------------------------------------------
struct Ring {
    uint8_t *buf;
    uint64_t *full;
    int *watchdog;
    const uint8_t *src;         // global source of the streamed bytes
    uint32_t tile_bytes;        // bytes per full tile
    uint64_t total_bytes;       // bytes in the whole stream

    __device__ __forceinline__ uint32_t bytes_of(uint32_t t) const {
        const uint64_t off = (uint64_t)t * tile_bytes;
        if (off >= total_bytes) return 0;
        const uint64_t rem = total_bytes - off;
        return rem < tile_bytes ? (uint32_t)rem : tile_bytes;
    }
    __device__ __forceinline__ void issue(uint32_t t, int s) const {
        const uint32_t b = bytes_of(t);
        if (b == 0) {                       // nothing to copy: complete the phase directly
            mbar_arrive(&full[s]);
            return;
        }
        mbar_arrive_expect_tx(&full[s], b);
        bulk_load(buf + s * kTileBytes, src + (uint64_t)t * tile_bytes, b, &full[s]);
    }
};

// Programmatic dependent launch: block until the previous kernel on the stream has
// completed and its writes are visible (a no-op without a programmatic predecessor),
// then let the next kernel's CTAs be scheduled as soon as ours retire.
__device__ __forceinline__ void pdl_wait_and_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Runs body(tile, stage_ptr) over this CTA's tiles with the bulk-copy ring.  `after_issue`
// runs in every thread once the first kStages copies are in flight and before the first
// tile is consumed (a kernel that must wait for its predecessor's results, but not for its
// input, waits there so that its first loads overlap the predecessor's tail).
// A stage is refilled once every warp is done with it.  By default the CTA synchronises
// after each tile and thread 0 refills at once.  With WARP_RELEASE each warp releases the
// stage on an "empty" barrier (ring.full holds kStages full barriers, then kStages empty
// ones) and thread 0 waits for the release, so only warp 0 waits for the slowest warp and
// the others run on into stages already loaded: measured 5-7% faster for the dequantisers
// (their warps drift with the store traffic) but 3-7% slower for the quantisers, where the
// refill then comes later than after a hardware barrier.
struct NoPrologue {
    __device__ __forceinline__ void operator()() const {}
};
template <bool WARP_RELEASE = false, typename Body, typename Prologue = NoPrologue>
__device__ __forceinline__ void stream_tiles(Ring &ring, uint32_t n_tiles, Body body, Prologue after_issue = {}) {
    const int tid = threadIdx.x;
    uint64_t *empty = ring.full + kStages;
    if (tid == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&ring.full[s], 1);
            if constexpr (WARP_RELEASE) mbar_init(&empty[s], kThreads / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();
    uint32_t issued = 0;                                   // tiles issued by thread 0
    if (tid == 0)
        for (int s = 0; s < kStages; s++) {
            const uint32_t t = blockIdx.x + (uint32_t)s * gridDim.x;
            if (t < n_tiles) { ring.issue(t, s); issued++; }
        }
    after_issue();
    uint32_t it = 0;
    for (uint32_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
        const int s = (int)(it % kStages);
        const uint32_t phase = (it / kStages) & 1u;
        // warp-uniform outcome (bodies may use full-warp shuffles)
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&ring.full[s], phase, ring.watchdog, WD_STREAM_FULL));
        if (ok) body(t, ring.buf + s * kTileBytes);
        const uint32_t tn = t + (uint32_t)kStages * gridDim.x;
        if constexpr (WARP_RELEASE) {
            __syncwarp();
            if ((tid & 31) == 0) mbar_arrive(&empty[s]);   // this warp is done with stage s
            if (tid == 0 && tn < n_tiles && *reinterpret_cast<volatile int *>(ring.watchdog) == 0 &&
                mbar_wait_bounded(&empty[s], phase, ring.watchdog, WD_STREAM_EMPTY)) {
                ring.issue(tn, s);
                issued++;
            }
        } else {
            __syncthreads();                               // stage s is free again
            if (tid == 0 && tn < n_tiles && *reinterpret_cast<volatile int *>(ring.watchdog) == 0) {
                ring.issue(tn, s);
                issued++;
            }
        }
    }
    if (tid == 0 && *reinterpret_cast<volatile int *>(ring.watchdog) != 0) {
        // error path: wait (bounded, short) for every copy this CTA issued
        for (uint32_t j = it; j < issued; j++)
            (void)mbar_wait_bounded(&ring.full[j % kStages], (j / kStages) & 1u, nullptr, 0, kDrainLimitNs);
    }
    if constexpr (WARP_RELEASE) __syncthreads();           // warps leave the loop together
}

// |x| maximum (15-bit bf16 magnitude; NaN anywhere gives >= 0x7F80) of a 32-element block
// held as four uint4 / a 16-element block held as two, by the packed bf16 maximum.
__device__ __forceinline__ uint32_t absmax_block32(const uint4 (&v)[4]) {
    uint32_t a = absmax_bf16x2(absmax_bf16x2(v[0].x, v[0].y), absmax_bf16x2(v[0].z, v[0].w));
    uint32_t b = absmax_bf16x2(absmax_bf16x2(v[1].x, v[1].y), absmax_bf16x2(v[1].z, v[1].w));
    uint32_t c = absmax_bf16x2(absmax_bf16x2(v[2].x, v[2].y), absmax_bf16x2(v[2].z, v[2].w));
    uint32_t d = absmax_bf16x2(absmax_bf16x2(v[3].x, v[3].y), absmax_bf16x2(v[3].z, v[3].w));
    const uint32_t m = absmax_bf16x2(absmax_bf16x2(a, b), absmax_bf16x2(c, d));
    return max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
}
__device__ __forceinline__ uint32_t absmax_block16(const uint4 &v0, const uint4 &v1) {
    const uint32_t a = absmax_bf16x2(absmax_bf16x2(v0.x, v0.y), absmax_bf16x2(v0.z, v0.w));
    const uint32_t b = absmax_bf16x2(absmax_bf16x2(v1.x, v1.y), absmax_bf16x2(v1.z, v1.w));
    const uint32_t m = absmax_bf16x2(a, b);
    return max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
}

__device__ __forceinline__ uint32_t amax_words(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __vmaxu2(__vmaxu2(a & 0x7FFF7FFFu, b & 0x7FFF7FFFu), __vmaxu2(c & 0x7FFF7FFFu, d & 0x7FFF7FFFu));
}

// Block-wide maximum of a per-thread |x| maximum (bf16 bits in either half); thread 0
// stores it as fp32.
__device__ __forceinline__ void store_partial(uint32_t acc, float *dst, uint32_t *warp_u) {
    const uint32_t tid = threadIdx.x;
    uint32_t m = hmax(acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) warp_u[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kThreads / 32; w++) r = max(r, warp_u[w]);
        out_store(dst, __uint_as_float(r << 16));
    }
}

// ---------------------------------------------------------------------------------------
// Row-wise MX quantiser: thread = one 32-element block (64 input bytes).
// ---------------------------------------------------------------------------------------
// partials: when non-null, the CTA also reduces the finite |x| maximum of everything it
// read (Inf / NaN excluded) into partials[blockIdx.x] -- the NVFP4 per-tensor maximum of
// the same tensor, so that an NVFP4 quantisation of it needs no maximum pass of its own.
template <int FMT, bool CEIL, bool RM, bool TC>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
mx_rows_kernel(const uint8_t *__restrict__ src, uint32_t n_blocks, FastDiv divS, uint32_t col_atoms,
               uint8_t *__restrict__ elems, uint8_t *__restrict__ sc_rm, uint8_t *__restrict__ sc_tc,
               float *__restrict__ partials, int *watchdog) {
    pdl_wait_and_release();
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[2 * kStages];   // full, then empty barriers
    __shared__ uint32_t warp_u[kThreads / 32];
    Ring ring{reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127)),
              full, watchdog, src, kTileBytes, (uint64_t)n_blocks * 64};
    constexpr uint32_t kBlocksPerTile = kTileBytes / 64;   // 256 = one per thread
    const uint32_t n_tiles = (n_blocks + kBlocksPerTile - 1) / kBlocksPerTile;
    const uint32_t tid = threadIdx.x;
    const uint32_t rot = tid >> 1;                          // bank-group rotation
    uint32_t finite_acc = 0;                                // finite |x| maximum (bf16 bits)

    stream_tiles(ring, n_tiles, [&](uint32_t t, const uint8_t *tile) {
        const uint32_t blk = t * kBlocksPerTile + tid;
        if (blk >= n_blocks) return;
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t c = (j + rot) & 3u;
            v[j] = *reinterpret_cast<const uint4 *>(tile + tid * 64 + c * 16);
        }
        const uint32_t m = absmax_block32(v);
        if (partials) {
            uint32_t f = m;
            if (__builtin_expect(m >= 0x7F80u, 0))          // Inf / NaN in the block: mask them out
                f = hmax(__vmaxu2(__vmaxu2(finite_abs_max_bf16x8(v[0]), finite_abs_max_bf16x8(v[1])),
                                  __vmaxu2(finite_abs_max_bf16x8(v[2]), finite_abs_max_bf16x8(v[3]))));
            finite_acc = max(finite_acc, f);
        }
        const uint32_t code = e8m0_from_amax_bits<FMT, CEIL>(m);
        const uint64_t mul2x = splat2(e8m0_inverse_multiplier(code));
        const bool nan_blk = code == 0xFFu;
        if constexpr (is_fp6(FMT)) {
            // the 32 codes are packed into 24 bytes, so the rotated chunks are put back in
            // order (register selects) before packing
            uint2 q[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                float x[8];
                scale8(v[j], mul2x, x);
                q[j] = cvt_fp8x8<FMT>(x);
            }
            uint32_t w[8];
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const uint32_t j = (c - rot) & 3u;              // q[j] holds chunk c
                const uint2 t = j == 0 ? q[0] : j == 1 ? q[1] : j == 2 ? q[2] : q[3];
                w[2 * c] = t.x;
                w[2 * c + 1] = t.y;
            }
            uint32_t o[6];
            fp6_pack<8>(w, o);
            uint2 *dst = reinterpret_cast<uint2 *>(elems + (size_t)blk * 24);
#pragma unroll
            for (int i = 0; i < 3; i++) out_store(dst + i, nan_blk ? make_uint2(0u, 0u) : make_uint2(o[2 * i], o[2 * i + 1]));
        } else {
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t c = (j + rot) & 3u;             // which 8-element chunk of the block
                float x[8];
                scale8(v[j], mul2x, x);
                if constexpr (FMT == FMT_E2M1) {
                    const uint32_t q = nan_blk ? 0u : cvt_e2m1x8(x);
                    out_store(reinterpret_cast<uint32_t *>(elems) + (size_t)blk * 4 + c, q);
                } else {
                    uint2 q = cvt_fp8x8<FMT>(x);
                    if (nan_blk) q = make_uint2(0u, 0u);
                    out_store(reinterpret_cast<uint2 *>(elems) + (size_t)blk * 4 + c, q);
                }
            }
        }
        if constexpr (RM) out_store(sc_rm + blk, (uint8_t)code);
        if constexpr (TC) {
            const uint32_t r = fdiv(blk, divS);
            out_store(sc_tc + tc_offset(r, blk - r * divS.d, col_atoms), (uint8_t)code);
        }
    });
    if (partials) store_partial(finite_acc, partials + blockIdx.x, warp_u);
}

__device__ __forceinline__ uint32_t finite_mask(uint32_t m) {
    // halfwords >= 0x7F80 (Inf/NaN magnitude) become 0
    return m & __vcmpltu2(m, 0x7F807F80u);
}

// ---------------------------------------------------------------------------------------
// NVFP4 quantisation of one 16 KiB tile (512 blocks of 16; thread = blocks tid, tid+256),
// read from the shared-memory ring.  g is the per-tensor decode scale.
//   per block: t = amax_b / (6 g), sb = UE4M3(t) (RNE, saturating), d = dec(sb) g,
//   q = E2M1(RN(x / d)); a block holding a NaN/Inf gets sb = 0x7F and codes 0.
// ---------------------------------------------------------------------------------------
template <bool RM, bool TC, bool FAST>
__device__ __forceinline__ void nvfp4_quant_tile(const uint8_t *tile, uint32_t t, uint32_t n_blocks,
                                                 const Nvfp4Consts &cst, const float2 *qtab, const FastDiv &divS,
                                                 uint32_t col_atoms, uint8_t *__restrict__ elems,
                                                 uint8_t *__restrict__ sc_rm, uint8_t *__restrict__ sc_tc) {
    // The thread's two blocks (tid, tid + 256) are processed side by side: the common path
    // has no data-dependent branch, so the two dependency chains interleave.
    constexpr uint32_t kBlocksPerTile = kTileBytes / 32;    // 512
    const uint32_t tid = threadIdx.x;
    const uint32_t rot = (tid >> 2) & 1u;
    uint32_t blk[2];
    bool ok[2];
    uint4 v[2][2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
        const uint32_t lb = tid + h * kThreads;
        blk[h] = t * kBlocksPerTile + lb;
        ok[h] = blk[h] < n_blocks;
        // v[h][j] holds 8-element chunk (j + rot) & 1 of the block (rotated shared-memory
        // reads); codes are computed per chunk and stored back at the chunk's position
#pragma unroll
        for (int j = 0; j < 2; j++)
            v[h][j] = ok[h] ? *reinterpret_cast<const uint4 *>(tile + lb * 32 + ((j + rot) & 1u) * 16)
                            : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t sb[2], q[2][2];
    float2 dq[2];
    bool special[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
        const uint32_t m = absmax_block16(v[h][0], v[h][1]);
        special[h] = m >= 0x7F80u;                           // Inf/NaN in the block
        const float tq = nvfp4_block_quotient<FAST>(__uint_as_float(m << 16), cst);
        sb[h] = cvt_fp8x2<FMT_E4M3>(tq, 0.0f) & 0xFFu;     // tq >= 0: sign bit stays 0
        dq[h] = qtab[sb[h] & 0x7Fu];                         // {d, -RN(1/d)}
    }
#pragma unroll
    for (int h = 0; h < 2; h++) {
        nvfp4_codes16(v[h][0], v[h][1], dq[h].x, dq[h].y, q[h][0], q[h][1]);
        if (special[h] || dq[h].x == 0.0f) q[h][0] = q[h][1] = 0u;   // NaN block, or d = 0: codes 0
        if (special[h]) sb[h] = 0x7Fu;                                 // UE4M3 NaN: the block is NaN
    }
#pragma unroll
    for (int h = 0; h < 2; h++) {
        if (!ok[h]) continue;
        // the block's 8 code bytes in element order as one 8-byte store (a warp writes 256
        // contiguous bytes per instruction)
        out_store(reinterpret_cast<uint2 *>(elems) + blk[h],
                  rot ? make_uint2(q[h][1], q[h][0]) : make_uint2(q[h][0], q[h][1]));
        if constexpr (RM) out_store(sc_rm + blk[h], (uint8_t)sb[h]);
        if constexpr (TC) {
            const uint32_t rr = fdiv(blk[h], divS);
            out_store(sc_tc + tc_offset(rr, blk[h] - rr * divS.d, col_atoms), (uint8_t)sb[h]);
        }
    }
}

// Tensor maximum of every CTA's partial maxima (all CTAs compute the same value in the
// same order) and the NVFP4 decode scale g = amax / 2688 (1 when the tensor is all zero).
__device__ __forceinline__ float nvfp4_global_scale(const float *partials, int n_partials, float *warp_max) {
    const uint32_t tid = threadIdx.x;
    float a = 0.0f;
    for (int i = tid; i < n_partials; i += kThreads) a = fmaxf(a, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = a;
    __syncthreads();
    a = 0.0f;
    for (int w = 0; w < kThreads / 32; w++) a = fmaxf(a, warp_max[w]);
    return a == 0.0f ? 1.0f : __fdiv_rn(a, 2688.0f);
}

// Finite |x| maximum of one streamed tile, folded into acc (Inf/NaN excluded).
__device__ __forceinline__ uint32_t finite_amax_tile(const uint8_t *tile, uint32_t nbytes, uint32_t acc) {
    const uint32_t tid = threadIdx.x;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint32_t off = (tid + j * kThreads) * 16;    // consecutive threads, consecutive 16 B
        if (off < nbytes) {
            const uint4 v = *reinterpret_cast<const uint4 *>(tile + off);
            uint32_t m = amax_words(v.x, v.y, v.z, v.w);
            if (__builtin_expect((m & 0x7F800000u) == 0x7F800000u || (m & 0x7F80u) == 0x7F80u, 0)) {
                m = __vmaxu2(__vmaxu2(finite_mask(v.x & 0x7FFF7FFFu), finite_mask(v.y & 0x7FFF7FFFu)),
                             __vmaxu2(finite_mask(v.z & 0x7FFF7FFFu), finite_mask(v.w & 0x7FFF7FFFu)));
            }
            acc = __vmaxu2(acc, m);
        }
    }
    return acc;
}


// ---------------------------------------------------------------------------------------
// NVFP4 as two kernels.  Pass 1: per-CTA maximum of the finite |x| (Inf/NaN excluded).
// Pass 2 (below) starts streaming the input before it waits for pass 1, and normally
// finds it in L2.  A single cooperative kernel that kept each CTA's last tiles in shared
// memory across a grid barrier measured slower at every size (the cooperative launch and
// the barrier cost more than the L2 re-read saves).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
nvfp4_amax_bulk_kernel(const uint8_t *__restrict__ src, uint64_t n_bytes, float *__restrict__ partials,
                       int *watchdog) {
    pdl_wait_and_release();
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[2 * kStages];   // full, then empty barriers
    __shared__ uint32_t warp_u[kThreads / 32];
    Ring ring{reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127)),
              full, watchdog, src, kTileBytes, n_bytes};
    const uint32_t n_tiles = (uint32_t)((n_bytes + kTileBytes - 1) / kTileBytes);
    uint32_t acc = 0;
    stream_tiles(ring, n_tiles, [&](uint32_t t, const uint8_t *tile) {
        acc = finite_amax_tile(tile, ring.bytes_of(t), acc);
    });
    store_partial(acc, partials + blockIdx.x, warp_u);
}

// Pass 2: reads the partial maxima written by pass 1.
template <bool RM, bool TC>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
nvfp4_quant_bulk_kernel(const uint8_t *__restrict__ src, uint32_t n_blocks, FastDiv divS, uint32_t col_atoms,
                        const float *__restrict__ partials, int n_partials, float *__restrict__ g_out,
                        uint8_t *__restrict__ elems, uint8_t *__restrict__ sc_rm, uint8_t *__restrict__ sc_tc,
                        int *watchdog) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[2 * kStages];   // full, then empty barriers
    __shared__ float warp_max[kThreads / 32];
    Ring ring{reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127)),
              full, watchdog, src, kTileBytes, (uint64_t)n_blocks * 32};
    __shared__ float2 qtab[128];
    Nvfp4Consts cst;
    const uint32_t n_tiles = (n_blocks + kTileBytes / 32 - 1) / (kTileBytes / 32);
    // The input is not written by the maximum pass, so the ring starts loading it at once;
    // the partial maxima are read only after the wait on that pass.
    auto after_issue = [&]() {
        pdl_wait_and_release();
        const float g = nvfp4_global_scale(partials, n_partials, warp_max);
        if (blockIdx.x == 0 && threadIdx.x == 0) out_store(g_out, g);
        cst = nvfp4_consts(g, qtab);
    };
    stream_tiles(ring, n_tiles, [&](uint32_t t, const uint8_t *tile) {
        if (cst.fast) nvfp4_quant_tile<RM, TC, true>(tile, t, n_blocks, cst, qtab, divS, col_atoms, elems, sc_rm, sc_tc);
        else nvfp4_quant_tile<RM, TC, false>(tile, t, n_blocks, cst, qtab, divS, col_atoms, elems, sc_rm, sc_tc);
    }, after_issue);
}

// ---------------------------------------------------------------------------------------
// NVFP4 with 16 x 16 weight blocks (two-dimensional block scaling for weights, the 4-bit
// pre-training recipe): second pass after nvfp4_amax_bulk_kernel.  A warp takes a strip of
// 16 horizontally adjacent blocks (16 rows x 256 columns): lane = (row parity, block), so
// every load and store instruction covers one or two whole 512-byte row segments (codes:
// 128 bytes, scales: 16 bytes per row).  Each lane holds its block's 8 rows of one parity
// in registers; the block maximum is its own maximum and its partner lane's (xor 16).
// Every other step is the 1 x 16 path's (same fp32 operations in the same order), and the
// block scale is written to each of the block's 16 rows in the 1 x 16 layouts.
// ---------------------------------------------------------------------------------------
template <bool RM, bool TC>
__global__ void __launch_bounds__(kThreads, 2)
nvfp4_2d_quant_kernel(const uint8_t *__restrict__ src, uint32_t cols, uint32_t rows, FastDiv div_strips,
                      uint32_t col_atoms, const float *__restrict__ partials, int n_partials,
                      float *__restrict__ g_out, uint8_t *__restrict__ elems, uint8_t *__restrict__ sc_rm,
                      uint8_t *__restrict__ sc_tc) {
    __shared__ float warp_max[kThreads / 32];
    __shared__ float2 qtab[128];
    pdl_wait_and_release();
    const float g = nvfp4_global_scale(partials, n_partials, warp_max);
    if (blockIdx.x == 0 && threadIdx.x == 0) out_store(g_out, g);
    const Nvfp4Consts cst = nvfp4_consts(g, qtab);
    const uint32_t lane = threadIdx.x & 31, par = lane >> 4, c = lane & 15;
    const uint32_t S = cols / 16;                                  // blocks (scale columns) per row
    const uint32_t n_tasks = (rows / 16) * div_strips.d;
    const uint32_t warps = gridDim.x * (kThreads / 32);
    // the loop bound is uniform over the warp, so the full-warp shuffle is safe
    for (uint32_t task = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); task < n_tasks; task += warps) {
        const uint32_t rb = fdiv(task, div_strips), cb = (task - rb * div_strips.d) * 16 + c;
        const bool valid = cb < S;
        uint4 v[8][2];
#pragma unroll
        for (int k = 0; k < 8; k++) {
            const uint32_t row = rb * 16 + 2 * k + par;
            const uint4 *p = reinterpret_cast<const uint4 *>(src + ((size_t)row * cols + (size_t)cb * 16) * 2);
            v[k][0] = valid ? p[0] : make_uint4(0u, 0u, 0u, 0u);
            v[k][1] = valid ? p[1] : make_uint4(0u, 0u, 0u, 0u);
        }
        uint32_t m = 0;
#pragma unroll
        for (int k = 0; k < 8; k++) m = max(m, absmax_block16(v[k][0], v[k][1]));
        m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
        const bool special = m >= 0x7F80u;                         // Inf/NaN in the block
        const float a = __uint_as_float(m << 16);
        const float tq = cst.fast ? nvfp4_block_quotient<true>(a, cst) : nvfp4_block_quotient<false>(a, cst);
        uint32_t sb = cvt_fp8x2<FMT_E4M3>(tq, 0.0f) & 0xFFu;
        const float2 dq = qtab[sb & 0x7Fu];
        const bool zero_codes = special || dq.x == 0.0f;
        if (special) sb = 0x7Fu;
        if (!valid) continue;
#pragma unroll
        for (int k = 0; k < 8; k++) {
            uint32_t q[2];
            nvfp4_codes16(v[k][0], v[k][1], dq.x, dq.y, q[0], q[1]);
            if (zero_codes) q[0] = q[1] = 0u;
            const uint32_t row = rb * 16 + 2 * k + par;
            out_store(reinterpret_cast<uint2 *>(elems) + (((size_t)row * cols + (size_t)cb * 16) >> 4), make_uint2(q[0], q[1]));
            if constexpr (RM) out_store(sc_rm + (size_t)row * S + cb, (uint8_t)sb);
            if constexpr (TC) out_store(sc_tc + tc_offset(row, cb, col_atoms), (uint8_t)sb);
        }
    }
}

// ---------------------------------------------------------------------------------------
// Dequantisers: codes streamed through the ring; each thread reads the scale of one block
// (two for NVFP4) directly; the bf16 output is written in 16-byte chunks of 8 elements,
// the lanes of a warp taking consecutive chunks so that every store instruction covers
// 512 contiguous bytes (FP6: thread = one block, 64 bytes).
// ---------------------------------------------------------------------------------------
// Eight fp32 times the scale m (m2 = m in both lanes), each product rounded to fp32 and then
// to bf16: one packed fp32 product per element pair.
__device__ __forceinline__ uint4 scaled_bf16x8(const float (&y)[8], uint64_t m2) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float lo, hi;
        unpack2(mul2(pack2(y[2 * i], y[2 * i + 1]), m2), lo, hi);
        w[i] = f32x2_to_bf16x2(lo, hi);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int FMT, bool TC>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
dequant_mx_bulk_kernel(const uint8_t *__restrict__ elems, const uint8_t *__restrict__ scales,
                       uint32_t n_blocks, FastDiv divS, uint32_t col_atoms, uint4 *__restrict__ out,
                       int *watchdog) {
    pdl_wait_and_release();
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[2 * kStages];   // full, then empty barriers
    constexpr uint32_t kCodeBytes = 32 * code_bits(FMT) / 8;              // per block: 16, 24 or 32
    constexpr uint32_t kBlocksPerTile = kThreads;                          // one per thread
    // Bulk copies move whole 16-byte units; with FP6 (24 bytes a block) and an odd block
    // count the last block is read straight from global memory by its thread.
    const uint32_t ring_blocks = is_fp6(FMT) ? (n_blocks & ~1u) : n_blocks;
    Ring ring{reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127)),
              full, watchdog, elems, kBlocksPerTile * kCodeBytes, (uint64_t)ring_blocks * kCodeBytes};
    const uint32_t n_tiles = (n_blocks + kBlocksPerTile - 1) / kBlocksPerTile;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, wbase = tid & ~31u;
    // this thread's block scale of tile t (0x100 past the end); loaded one tile ahead, so
    // that its latency overlaps the previous tile instead of stalling the current one
    auto scale_of = [&](uint32_t t) -> uint32_t {
        const uint32_t blk = t * kBlocksPerTile + tid;
        if (t >= n_tiles || blk >= n_blocks) return 0x100u;
        if constexpr (TC) {
            const uint32_t r = fdiv(blk, divS);
            return scales[tc_offset(r, blk - r * divS.d, col_atoms)];
        } else {
            return scales[blk];
        }
    };
    uint32_t s_next = scale_of(blockIdx.x);
    stream_tiles<true>(ring, n_tiles, [&](uint32_t t, const uint8_t *tile) {
        const uint32_t blk = t * kBlocksPerTile + tid;
        const uint32_t s = s_next;
        s_next = scale_of(t + gridDim.x);
        // the block scale as an fp32 multiplier (0 past the end, NaN for 0xFF)
        const float mul = s == 0x100u ? 0.0f : s == 0xFFu ? __uint_as_float(0x7FC00000u) : e8m0_multiplier(s);
        if constexpr (is_fp6(FMT)) {
            if (blk >= n_blocks) return;
            uint4 *dst = out + (size_t)blk * 4;
            // 24 bytes = 32 packed codes, as three 8-byte reads (stride 24 B: conflict-free)
            const uint2 *p = blk < ring_blocks ? reinterpret_cast<const uint2 *>(tile + tid * 24)
                                               : reinterpret_cast<const uint2 *>(elems + (size_t)blk * 24);
            const uint2 a = p[0], b = p[1], c = p[2];
            const uint32_t o[6] = {a.x, a.y, b.x, b.y, c.x, c.y};
            uint32_t w[8];
            fp6_unpack<8>(o, w);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                float y[8];
                fp8x2_to_f32<FMT>(w[2 * j] & 0xFFFFu, y[0], y[1]);
                fp8x2_to_f32<FMT>(w[2 * j] >> 16, y[2], y[3]);
                fp8x2_to_f32<FMT>(w[2 * j + 1] & 0xFFFFu, y[4], y[5]);
                fp8x2_to_f32<FMT>(w[2 * j + 1] >> 16, y[6], y[7]);
                out_store(dst + j, scaled_bf16x8(y, splat2(mul)));
            }
        } else {
            // The warp's 32 blocks are 128 chunks of 8 elements; in round j lane l converts
            // chunk 32 j + l, so every store instruction of the warp writes 512 contiguous
            // bytes.  The chunk's block scale comes from its owner lane by a shuffle.
            constexpr uint32_t kChunkBytes = kCodeBytes / 4;               // 4 (FP4) or 8
            const uint8_t *wcodes = tile + wbase * kCodeBytes;
            uint4 *wout = out + ((size_t)t * kBlocksPerTile + wbase) * 4;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const uint32_t q = 32u * j + lane, lb = q >> 2;               // chunk, block in the warp
                const float m = __shfl_sync(0xFFFFFFFFu, mul, (int)lb);
                if (t * kBlocksPerTile + wbase + lb >= n_blocks) continue;
                float y[8];
                if constexpr (FMT == FMT_E2M1) {
                    e2m1x8_to_f32(*reinterpret_cast<const uint32_t *>(wcodes + q * kChunkBytes), y);
                } else {
                    const uint2 c = *reinterpret_cast<const uint2 *>(wcodes + q * kChunkBytes);
                    fp8x2_to_f32<FMT>(c.x & 0xFFFFu, y[0], y[1]);
                    fp8x2_to_f32<FMT>(c.x >> 16, y[2], y[3]);
                    fp8x2_to_f32<FMT>(c.y & 0xFFFFu, y[4], y[5]);
                    fp8x2_to_f32<FMT>(c.y >> 16, y[6], y[7]);
                }
                out_store(wout + q, scaled_bf16x8(y, splat2(m)));
            }
        }
    });
}

template <bool TC>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
dequant_nvfp4_bulk_kernel(const uint8_t *__restrict__ elems, const uint8_t *__restrict__ scales,
                          const float *__restrict__ g_ptr, uint32_t n_blocks, FastDiv divS, uint32_t col_atoms,
                          uint4 *__restrict__ out, int *watchdog) {
    pdl_wait_and_release();
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full[2 * kStages];   // full, then empty barriers
    constexpr uint32_t kBlocksPerTile = 2 * kThreads;                      // 8 code bytes each
    // Bulk copies move whole 16-byte units (block pairs); with an odd block count the
    // last block's 8 code bytes are read straight from global memory by its thread.
    Ring ring{reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127)),
              full, watchdog, elems, kBlocksPerTile * 8, (uint64_t)(n_blocks & ~1u) * 8};
    const uint32_t n_tiles = (n_blocks + kBlocksPerTile - 1) / kBlocksPerTile;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, wbase = 2u * (tid & ~31u);   // warp's first block
    const uint64_t g2 = splat2(*g_ptr);
    const uint32_t ring_blocks = n_blocks & ~1u;
    // this thread's two UE4M3 block scales of tile t (0 past the end), loaded one tile ahead
    auto scales_of = [&](uint32_t t, uint32_t (&sc)[2]) {
#pragma unroll
        for (int b = 0; b < 2; b++) {
            const uint32_t blk = t * kBlocksPerTile + tid * 2 + b;
            sc[b] = 0u;
            if (t < n_tiles && blk < n_blocks) {
                if constexpr (TC) {
                    const uint32_t r = fdiv(blk, divS);
                    sc[b] = scales[tc_offset(r, blk - r * divS.d, col_atoms)];
                } else {
                    sc[b] = scales[blk];
                }
            }
        }
    };
    uint32_t sc_next[2];
    scales_of(blockIdx.x, sc_next);
    stream_tiles<true>(ring, n_tiles, [&](uint32_t t, const uint8_t *tile) {
        // this thread's two blocks' UE4M3 scales as f16x2 words holding dec(sb) twice (0 past
        // the end; code 0x7F decodes to NaN).  dec(q) dec(sb) is exact in f16: at most 6
        // significant bits, magnitudes 2^-10 .. 2688, so the packed f16 product equals the
        // fp32 one and only the product with g rounds.
        const uint32_t sc[2] = {sc_next[0], sc_next[1]};
        scales_of(t + gridDim.x, sc_next);
        uint32_t sbh[2];
#pragma unroll
        for (int b = 0; b < 2; b++) {
            const uint32_t s = sc[b] & 0x7Fu;
            const uint16_t s2 = (uint16_t)(s | (s << 8));
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(sbh[b]) : "h"(s2));
        }
        // The warp's 64 blocks are 128 chunks of 8 elements; in round j lane l converts
        // chunk 32 j + l (block 16 j + l / 2, owned by lane 8 j + l / 4), so every store
        // instruction of the warp writes 512 contiguous bytes.
        const uint32_t wblk = t * kBlocksPerTile + wbase;
        uint4 *wout = out + (size_t)wblk * 2;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t q = 32u * j + lane, lb = q >> 1;
            const uint32_t s0 = __shfl_sync(0xFFFFFFFFu, sbh[0], (int)(lb >> 1));
            const uint32_t s1 = __shfl_sync(0xFFFFFFFFu, sbh[1], (int)(lb >> 1));
            const uint32_t sb = (lb & 1u) ? s1 : s0;
            const uint32_t blk = wblk + lb;
            if (blk >= n_blocks) continue;
            const uint32_t c = blk < ring_blocks
                                   ? *reinterpret_cast<const uint32_t *>(tile + (size_t)(wbase + lb) * 8 + (q & 1u) * 4)
                                   : *reinterpret_cast<const uint32_t *>(elems + (size_t)blk * 8 + (q & 1u) * 4);
            uint32_t h[4];
            e2m1x8_to_f16x2(c, h);
            float y[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                uint32_t p;
                asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(h[i]), "r"(sb));
                f16x2_to_f32(p, y[2 * i], y[2 * i + 1]);
            }
            out_store(wout + q, scaled_bf16x8(y, g2));
        }
    });
}

// ---------------------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------------------
static int stream_grid(uint32_t n_tiles, int num_sms) {
    int64_t g = (int64_t)num_sms * kCtasPerSm;
    if (g > n_tiles) g = n_tiles;
    return g < 1 ? 1 : (int)g;
}
constexpr size_t kStreamSmem = (size_t)kStages * kTileBytes + 128;

// Launch with programmatic dependent launch enabled: the kernel may be scheduled while the
// previous kernel on the stream drains; its first instruction (griddepcontrol.wait) holds it
// until that kernel has completed.  The shared-memory attribute is set once per device and
// kernel.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_smem(void (*kernel)(KArgs...), int grid, size_t smem, cudaStream_t st, Args... args);

template <typename... KArgs, typename... Args>
static cudaError_t launch_stream(void (*kernel)(KArgs...), int grid, cudaStream_t st, Args... args) {
    return launch_pdl_smem(kernel, grid, kStreamSmem, st, args...);
}

// As launch_stream, for kernels without the tile ring (no dynamic shared memory).
template <typename... KArgs, typename... Args>
static cudaError_t launch_direct(void (*kernel)(KArgs...), int grid, cudaStream_t st, Args... args) {
    return launch_pdl_smem(kernel, grid, 0, st, args...);
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_smem(void (*kernel)(KArgs...), int grid, size_t smem, cudaStream_t st, Args... args) {
    static std::mutex mu;
    static std::set<std::pair<int, const void *>> configured;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto key = std::make_pair(dev, reinterpret_cast<const void *>(kernel));
        if (smem > 0 && !configured.count(key)) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            configured.insert(key);
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Bytes of a tcgen05-tiled scale array of rows x S scales (512-byte atoms of 128 x 4).
static uint64_t tc_bytes(int64_t rows, int64_t S) { return (uint64_t)((rows + 127) / 128) * ((S + 3) / 4) * 512; }

bool stream_supported(int64_t rows, int64_t cols) {
    return rows * cols / 16 < ((int64_t)1 << 31);   // block indices fit 31 bits
}

template <int FMT, bool CEIL, bool RM, bool TC>
static cudaError_t launch_rows_t(const void *src, uint32_t n_blocks, FastDiv f, uint32_t col_atoms, void *elems,
                                 uint8_t *rm, uint8_t *tc, float *partials, int grid, int *wd, cudaStream_t st) {
    return launch_stream(mx_rows_kernel<FMT, CEIL, RM, TC>, grid, st, static_cast<const uint8_t *>(src), n_blocks, f,
                         col_atoms, static_cast<uint8_t *>(elems), rm, tc, partials, wd);
}

template <int FMT, bool CEIL>
static cudaError_t launch_rows_layout(const void *src, uint32_t nb, FastDiv f, uint32_t ca, void *elems, uint8_t *rm,
                                      uint8_t *tc, float *p, int grid, int *wd, cudaStream_t st) {
    if (rm && tc) return launch_rows_t<FMT, CEIL, true, true>(src, nb, f, ca, elems, rm, tc, p, grid, wd, st);
    if (rm) return launch_rows_t<FMT, CEIL, true, false>(src, nb, f, ca, elems, rm, tc, p, grid, wd, st);
    return launch_rows_t<FMT, CEIL, false, true>(src, nb, f, ca, elems, rm, tc, p, grid, wd, st);
}

// Grid of the row-wise MX kernel for a rows x cols tensor (its CTA count is also the number
// of partial maxima it writes when asked to).
int stream_rows_grid(int64_t rows, int64_t cols, int num_sms) {
    const uint32_t n_tiles = (uint32_t)((rows * cols / 32 + 255) / 256);
    return stream_grid(n_tiles, num_sms);
}

cudaError_t launch_stream_rows_mx(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil, void *elems,
                                  uint8_t *rm, uint8_t *tc, float *partials, int *wd, int num_sms, cudaStream_t st) {
    const uint32_t n_blocks = (uint32_t)(rows * cols / 32);
    const uint32_t S = (uint32_t)(cols / 32);
    const FastDiv f = make_fastdiv(S);
    const uint32_t ca = (S + 3) / 4;
    const int g = stream_rows_grid(rows, cols, num_sms);
    const OutRange out[4] = {{elems, (uint64_t)(rows * cols * code_bits(fmt) / 8)}, {rm, (uint64_t)(rows * cols / 32)},
                             {tc, tc_bytes(rows, S)}, {partials, (uint64_t)g * 4}};
    cudaError_t e = set_out_ranges(out, st);
    if (e != cudaSuccess) return e;
    switch (fmt * 2 + (ceil ? 1 : 0)) {
    case FMT_E4M3 * 2 + 0: return launch_rows_layout<FMT_E4M3, false>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E4M3 * 2 + 1: return launch_rows_layout<FMT_E4M3, true>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E5M2 * 2 + 0: return launch_rows_layout<FMT_E5M2, false>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E5M2 * 2 + 1: return launch_rows_layout<FMT_E5M2, true>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E2M1 * 2 + 0: return launch_rows_layout<FMT_E2M1, false>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E2M1 * 2 + 1: return launch_rows_layout<FMT_E2M1, true>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E2M3 * 2 + 0: return launch_rows_layout<FMT_E2M3, false>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E2M3 * 2 + 1: return launch_rows_layout<FMT_E2M3, true>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E3M2 * 2 + 0: return launch_rows_layout<FMT_E3M2, false>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_E3M2 * 2 + 1: return launch_rows_layout<FMT_E3M2, true>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_INT8 * 2 + 0: return launch_rows_layout<FMT_INT8, false>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    case FMT_INT8 * 2 + 1: return launch_rows_layout<FMT_INT8, true>(src, n_blocks, f, ca, elems, rm, tc, partials, g, wd, st);
    default: return cudaErrorInvalidValue;
    }
}

// Partial maxima: one per CTA of the streaming maximum pass (kCtasPerSm per SM) or of the
// training quantiser's maximum pass (at most 8 per SM).
int stream_nvfp4_scratch_floats(int num_sms) { return (kCtasPerSm > 8 ? kCtasPerSm : 8) * num_sms; }

template <bool RM, bool TC>
static cudaError_t launch_nvfp4_t(const uint8_t *src, uint32_t nb, FastDiv f, uint32_t ca, float *partials,
                                  int max_partials, int n_given, float *g, uint8_t *elems, uint8_t *rm, uint8_t *tc,
                                  int *wd, int num_sms, cudaStream_t st) {
    const uint32_t n_tiles = (nb + 511) / 512;
    int grid = n_given;
    if (grid == 0) {
        // pass 1: per-CTA maxima
        grid = stream_grid(n_tiles, num_sms);
        if (grid > max_partials) grid = max_partials;
        cudaError_t e = launch_stream(nvfp4_amax_bulk_kernel, grid, st, src, (uint64_t)nb * 32, partials, wd);
        if (e != cudaSuccess) return e;
    }
    // pass 2 (programmatic dependent launch): quantisation
    return launch_stream(nvfp4_quant_bulk_kernel<RM, TC>, stream_grid(n_tiles, num_sms), st, src, nb, f, ca,
                         (const float *)partials, grid, g, elems, rm, tc, wd);
}

template <bool RM, bool TC>
static cudaError_t launch_nvfp4_2d_t(const uint8_t *src, int64_t rows, int64_t cols, float *partials,
                                     int max_partials, float *g, uint8_t *elems, uint8_t *rm, uint8_t *tc, int *wd,
                                     int num_sms, cudaStream_t st) {
    const uint64_t nbytes = (uint64_t)rows * cols * 2;
    const uint32_t n_tiles = (uint32_t)((nbytes + kTileBytes - 1) / kTileBytes);
    int grid = stream_grid(n_tiles, num_sms);
    if (grid > max_partials) grid = max_partials;
    cudaError_t e = launch_stream(nvfp4_amax_bulk_kernel, grid, st, src, nbytes, partials, wd);
    if (e != cudaSuccess) return e;
    // a warp per strip of 16 blocks (16 x 256 elements); 2 CTAs of 8 warps per SM
    const uint32_t bc = (uint32_t)(cols / 16), strips = (bc + 15) / 16;
    const uint32_t n_tasks = (uint32_t)(rows / 16) * strips;
    int grid2 = (int)((n_tasks + kThreads / 32 - 1) / (kThreads / 32));
    if (grid2 > 2 * num_sms) grid2 = 2 * num_sms;
    return launch_direct(nvfp4_2d_quant_kernel<RM, TC>, grid2, st, src, (uint32_t)cols, (uint32_t)rows,
                         make_fastdiv(strips), (bc + 3) / 4, (const float *)partials, grid, g, elems, rm, tc);
}

cudaError_t launch_stream_nvfp4_2d(const void *src, int64_t rows, int64_t cols, float *partials, int max_partials,
                                   float *g, void *elems, uint8_t *rm, uint8_t *tc, int num_sms, int *wd,
                                   cudaStream_t st) {
    const OutRange out[5] = {{elems, (uint64_t)(rows * cols / 2)}, {rm, (uint64_t)(rows * cols / 16)},
                             {tc, tc_bytes(rows, cols / 16)}, {g, 4}, {partials, (uint64_t)max_partials * 4}};
    cudaError_t e = set_out_ranges(out, st);
    if (e != cudaSuccess) return e;
    const uint8_t *s8 = static_cast<const uint8_t *>(src);
    uint8_t *e8 = static_cast<uint8_t *>(elems);
    if (rm && tc) return launch_nvfp4_2d_t<true, true>(s8, rows, cols, partials, max_partials, g, e8, rm, tc, wd, num_sms, st);
    if (rm) return launch_nvfp4_2d_t<true, false>(s8, rows, cols, partials, max_partials, g, e8, rm, tc, wd, num_sms, st);
    return launch_nvfp4_2d_t<false, true>(s8, rows, cols, partials, max_partials, g, e8, rm, tc, wd, num_sms, st);
}

cudaError_t launch_stream_nvfp4(const void *src, int64_t rows, int64_t cols, float *partials, int max_partials,
                                int n_given, float *g, void *elems, uint8_t *rm, uint8_t *tc, int *wd, int num_sms,
                                cudaStream_t st) {
    const uint32_t nb = (uint32_t)(rows * cols / 16), S = (uint32_t)(cols / 16);
    const FastDiv f = make_fastdiv(S);
    const uint32_t ca = (S + 3) / 4;
    const OutRange out[5] = {{elems, (uint64_t)(rows * cols / 2)}, {rm, (uint64_t)(rows * cols / 16)},
                             {tc, tc_bytes(rows, S)}, {g, 4}, {partials, (uint64_t)max_partials * 4}};
    cudaError_t e = set_out_ranges(out, st);
    if (e != cudaSuccess) return e;
    const uint8_t *s8 = static_cast<const uint8_t *>(src);
    uint8_t *e8 = static_cast<uint8_t *>(elems);
    if (rm && tc)
        return launch_nvfp4_t<true, true>(s8, nb, f, ca, partials, max_partials, n_given, g, e8, rm, tc, wd, num_sms, st);
    if (rm)
        return launch_nvfp4_t<true, false>(s8, nb, f, ca, partials, max_partials, n_given, g, e8, rm, tc, wd, num_sms, st);
    return launch_nvfp4_t<false, true>(s8, nb, f, ca, partials, max_partials, n_given, g, e8, rm, tc, wd, num_sms, st);
}

template <int FMT, bool TC>
static cudaError_t launch_dq_t(const void *elems, const uint8_t *scales, uint32_t nb, FastDiv f, uint32_t ca,
                               void *out, int *wd, int num_sms, cudaStream_t st) {
    const uint32_t n_tiles = (nb + kThreads - 1) / kThreads;
    return launch_stream(dequant_mx_bulk_kernel<FMT, TC>, stream_grid(n_tiles, num_sms), st,
                         static_cast<const uint8_t *>(elems), scales, nb, f, ca, static_cast<uint4 *>(out), wd);
}

cudaError_t launch_stream_dequant_mx(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols, int fmt,
                                     bool tc, void *out, int *wd, int num_sms, cudaStream_t st) {
    const uint32_t nb = (uint32_t)(rows * cols / 32), S = (uint32_t)(cols / 32);
    const FastDiv f = make_fastdiv(S);
    const uint32_t ca = (S + 3) / 4;
    const OutRange orng[1] = {{out, (uint64_t)(rows * cols * 2)}};
    cudaError_t e = set_out_ranges(orng, st);
    if (e != cudaSuccess) return e;
    switch (fmt) {
    case FMT_E4M3: return tc ? launch_dq_t<FMT_E4M3, true>(elems, scales, nb, f, ca, out, wd, num_sms, st)
                             : launch_dq_t<FMT_E4M3, false>(elems, scales, nb, f, ca, out, wd, num_sms, st);
    case FMT_E5M2: return tc ? launch_dq_t<FMT_E5M2, true>(elems, scales, nb, f, ca, out, wd, num_sms, st)
                             : launch_dq_t<FMT_E5M2, false>(elems, scales, nb, f, ca, out, wd, num_sms, st);
    case FMT_E2M1: return tc ? launch_dq_t<FMT_E2M1, true>(elems, scales, nb, f, ca, out, wd, num_sms, st)
                             : launch_dq_t<FMT_E2M1, false>(elems, scales, nb, f, ca, out, wd, num_sms, st);
    case FMT_E2M3: return tc ? launch_dq_t<FMT_E2M3, true>(elems, scales, nb, f, ca, out, wd, num_sms, st)
                        : launch_dq_t<FMT_E2M3, false>(elems, scales, nb, f, ca, out, wd, num_sms, st);
    case FMT_E3M2: return tc ? launch_dq_t<FMT_E3M2, true>(elems, scales, nb, f, ca, out, wd, num_sms, st)
                        : launch_dq_t<FMT_E3M2, false>(elems, scales, nb, f, ca, out, wd, num_sms, st);
    case FMT_INT8: return tc ? launch_dq_t<FMT_INT8, true>(elems, scales, nb, f, ca, out, wd, num_sms, st)
                        : launch_dq_t<FMT_INT8, false>(elems, scales, nb, f, ca, out, wd, num_sms, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_stream_dequant_nvfp4(const void *elems, const uint8_t *scales, const float *g, int64_t rows,
                                        int64_t cols, bool tc, void *out, int *wd, int num_sms, cudaStream_t st) {
    const uint32_t nb = (uint32_t)(rows * cols / 16), S = (uint32_t)(cols / 16);
    const FastDiv f = make_fastdiv(S);
    const uint32_t ca = (S + 3) / 4;
    const uint32_t n_tiles = (nb + 2 * kThreads - 1) / (2 * kThreads);
    const int grid = stream_grid(n_tiles, num_sms);
    const OutRange orng[1] = {{out, (uint64_t)(rows * cols * 2)}};
    cudaError_t e = set_out_ranges(orng, st);
    if (e != cudaSuccess) return e;
    const uint8_t *e8 = static_cast<const uint8_t *>(elems);
    uint4 *o = static_cast<uint4 *>(out);
    return tc ? launch_stream(dequant_nvfp4_bulk_kernel<true>, grid, st, e8, scales, g, nb, f, ca, o, wd)
              : launch_stream(dequant_nvfp4_bulk_kernel<false>, grid, st, e8, scales, g, nb, f, ca, o, wd);
}

}  // namespace mxk
