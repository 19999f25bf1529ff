// internal.h -- launchers shared between the kernel files and the C ABI layer.
// Not part of the public interface (see include/mx.h for that).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace mxk {

// Row-wise MX quantiser (blocks of 32 along rows); writes row-major and/or tcgen05 scales.
cudaError_t launch_quant_rows_mx(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil,
                                 void *elems, uint8_t *sc_rowmajor, uint8_t *sc_tcgen05,
                                 int num_sms, cudaStream_t st);

// Zero the padding bytes of a tcgen05-tiled scale buffer (rows x S scales).
cudaError_t launch_tcgen05_pad(uint8_t *sc, int64_t rows, int64_t S, cudaStream_t st);

// NVFP4: pass 1 writes one finite |x| maximum per CTA into `partials` (n_partials CTAs).
cudaError_t launch_nvfp4_amax(const void *src, int64_t n, float *partials, int n_partials,
                              cudaStream_t st);
// NVFP4: pass 2 reduces the partials to the tensor amax, writes g, quantises.
cudaError_t launch_nvfp4_quant(const void *src, int64_t rows, int64_t cols, const float *partials,
                               int n_partials, float *global_scale, void *elems,
                               uint8_t *sc_rowmajor, uint8_t *sc_tcgen05, int num_sms,
                               cudaStream_t st);
int nvfp4_partials_count(int64_t n, int num_sms);

cudaError_t launch_cast(const void *src, int64_t n, int fmt, void *out, int num_sms, cudaStream_t st);

cudaError_t launch_dequant_mx(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                              int fmt, bool tcgen05, void *out, int num_sms, cudaStream_t st);
cudaError_t launch_dequant_nvfp4(const void *elems, const uint8_t *scales, const float *g,
                                 int64_t rows, int64_t cols, bool tcgen05, void *out, int num_sms,
                                 cudaStream_t st);

// TMA-staged quantiser producing the row-wise and/or the column-wise (transposed) output.
cudaError_t launch_quant_dual(const void *src, int64_t rows, int64_t cols, int fmt, bool ceil,
                              void *row_elems, uint8_t *row_sc, void *col_elems, uint8_t *col_sc,
                              bool tcgen05, int *watchdog, int num_sms, cudaStream_t st);

// tcgen05 block-scaled matmul C = A * B^T (A: M x K E4M3, B: N x K E4M3 or E2M1).
cudaError_t launch_gemm(const void *a_elems, const uint8_t *a_sc, const void *b_elems,
                        const uint8_t *b_sc, int b_fmt, void *c, int64_t M, int64_t N, int64_t K,
                        int *watchdog, int num_sms, cudaStream_t st);

// Driver entry point for cuTensorMapEncodeTiled (resolved once, no libcuda link).
void *tensor_map_encoder();

// Record the CUDA error behind an MX_ERR_CUDA status for mx_last_cuda_error().
void record_cuda_error(cudaError_t e);

}  // namespace mxk
