// internal.h -- launchers shared between the kernel files and the C ABI layer.
// Not part of the public interface (see include/mx.h for that).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace mxk {

// ---- stream.cu: bulk-copy pipelined streaming kernels -------------------------------------
// True when the block indices of a rows x cols tensor fit the kernels' 31-bit indexing.
bool stream_supported(int64_t rows, int64_t cols);

// Row-wise MX quantiser (blocks of 32 along rows); row-major and/or tcgen05 scales.  With
// `partials` non-null, each of its stream_rows_grid() CTAs also writes the finite |x|
// maximum of what it read to partials[cta] (the NVFP4 per-tensor maximum's partials).
int stream_rows_grid(int64_t rows, int64_t cols, int num_sms);
cudaError_t launch_stream_rows_mx(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil, void *elems,
                                  uint8_t *sc_rowmajor, uint8_t *sc_tcgen05, float *partials, int *watchdog,
                                  int num_sms, cudaStream_t st);

// NVFP4 scratch: one partial maximum per CTA of the maximum pass (no initial value needed:
// every call writes each slot it later reads).  Returns the float count the launch below
// needs on a device with num_sms SMs.
int stream_nvfp4_scratch_floats(int num_sms);
// NVFP4 quantisation (tensor amax -> g written to *global_scale -> block scales and codes)
// as two kernels; the maximum pass uses at most max_partials CTAs.  n_given > 0: the
// n_given partial maxima are already in `partials` (written by an earlier kernel on the
// stream) and only the quantisation pass runs.
cudaError_t launch_stream_nvfp4(const void *src, int64_t rows, int64_t cols, float *partials, int max_partials,
                                int n_given, float *global_scale, void *elems, uint8_t *sc_rowmajor,
                                uint8_t *sc_tcgen05, int *watchdog, int num_sms, cudaStream_t st);

// NVFP4 with 16 x 16 blocks (rows, cols multiples of 16); scales in the 1 x 16 layouts.
cudaError_t launch_stream_nvfp4_2d(const void *src, int64_t rows, int64_t cols, float *partials, int max_partials,
                                   float *g, void *elems, uint8_t *rm, uint8_t *tc, int num_sms, int *wd,
                                   cudaStream_t st);

cudaError_t launch_stream_dequant_mx(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols, int fmt,
                                     bool tcgen05, void *out, int *watchdog, int num_sms, cudaStream_t st);
cudaError_t launch_stream_dequant_nvfp4(const void *elems, const uint8_t *scales, const float *g, int64_t rows,
                                        int64_t cols, bool tcgen05, void *out, int *watchdog, int num_sms,
                                        cudaStream_t st);

// ---- quant.cu ----------------------------------------------------------------------------------
// Zero the padding bytes of a tcgen05-tiled scale buffer (rows x S scales).
cudaError_t launch_tcgen05_pad(uint8_t *sc, int64_t rows, int64_t S, cudaStream_t st);
// Direct element cast (no block scale).
cudaError_t launch_cast(const void *src, int64_t n, int fmt, void *out, int num_sms, cudaStream_t st);
// One bounded wait on a barrier nothing arrives at (the watchdog's own test).
cudaError_t launch_watchdog_selftest(uint64_t limit_ns, int *watchdog, cudaStream_t st);

// ---- dual.cu -------------------------------------------------------------------------------------
// TMA-staged quantiser producing the column-wise (transposed) output and optionally the
// row-wise one (row_elems non-null), with scales in the row-major layout (*_rm), the
// tcgen05 tiling (*_tc) or both; the row-wise output takes the same layouts.
cudaError_t launch_quant_dual(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil,
                              void *row_elems, uint8_t *row_rm, uint8_t *row_tc, void *col_elems, uint8_t *col_rm,
                              uint8_t *col_tc, int *watchdog, int num_sms, cudaStream_t st);

// ---- gemm.cu -------------------------------------------------------------------------------------
// tcgen05 block-scaled matmul C = alpha A * B^T.  Format pairs: E4M3 x {E4M3, E2M1}
// (K % 128 == 0), E2M1 x E2M1 and NVFP4 x NVFP4 (K % 256 == 0); alpha = (*ga) (*gb) for
// NVFP4, else 1.
cudaError_t launch_gemm(const void *a_elems, const uint8_t *a_sc, int a_fmt, const float *ga, const void *b_elems,
                        const uint8_t *b_sc, int b_fmt, const float *gb, void *c, int64_t M, int64_t N, int64_t K,
                        int *watchdog, int num_sms, cudaStream_t st);

// ---- gemm2.cu: the same matmul on CTA pairs (256 x 256 tiles, tcgen05 cta_group::2) ---------------
bool gemm_pair_supported(int64_t M, int64_t N);
cudaError_t launch_gemm_pair(const void *a_elems, const uint8_t *a_sc, int a_fmt, const float *ga,
                             const void *b_elems, const uint8_t *b_sc, int b_fmt, const float *gb, void *c,
                             int64_t M, int64_t N, int64_t K, int *watchdog, int num_sms, cudaStream_t st);

// ---- train.cu: row-wise MX / NVFP4 with an optional 16 x 16 random Hadamard transform and
// optional stochastic rounding (rnd: one random byte per element, or nullptr for RNE) ----------
cudaError_t launch_quantize_train(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil, bool rht,
                                  uint32_t signs, const uint8_t *rnd, float *partials, int max_partials, float *g,
                                  void *elems, uint8_t *rm, uint8_t *tc, int num_sms, cudaStream_t st);

// ---- nested.cu: MXFP4 -> FP8 E4M3 with 128 x 128 block scales ----------------------------------
cudaError_t launch_mxfp4_to_fp8_blocks(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                                       void *out, float *block_scale, uint8_t *block_exact, cudaStream_t st);

// ---- api.cu --------------------------------------------------------------------------------------
// Driver entry point for cuTensorMapEncodeTiled (resolved once, no libcuda link).
void *tensor_map_encoder();
// Record the CUDA error behind an MX_ERR_CUDA status for mx_last_cuda_error().
void record_cuda_error(cudaError_t e);
// Current device's SM count and watchdog-flag address (set up once per device; no allocation).
cudaError_t device_info(int *num_sms, int **watchdog);

}  // namespace mxk
