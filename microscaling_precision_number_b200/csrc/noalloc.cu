// noalloc.cu -- NVFP4 quantisation for callers that must not allocate device memory.
//
// mx_quantize(fmt = MX_FMT_NVFP4) keeps its scratch (one partial maximum per CTA of the
// tensor-maximum pass) in a buffer that the library allocates with cudaMalloc on the first
// NVFP4 call on each device.  Some callers cannot allow that: a serving loop that
// reserves all device memory up front and must not take the implicit device
// synchronisation (or the out-of-memory risk) of a cudaMalloc on its request path, or a
// host framework that owns every byte of device memory through its own allocator and
// forbids a library from allocating behind its back.  This entry point runs the same
// kernels with the scratch in a fixed, statically sized device array instead, so it
// allocates nothing at any point.
//
// The array lives in this file.  Every GPU that loads the library holds it until the
// process exits.  Host code cannot use the array's name as a device address; its device
// address is obtained once per device with cudaGetSymbolAddress (the set-up below) and
// passed to the kernels.
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/mx.h"
#include "internal.h"

// One partial maximum per CTA of the maximum pass (each call writes every slot it reads).
static __device__ __align__(256) float g_noalloc_scratch[MX_NOALLOC_MAX_PARTIALS];

namespace {

constexpr int kMaxDevices = 64;

struct NoAllocDevice {
    bool ready = false;
    int num_sms = 0;
    int *watchdog = nullptr;     // the library's watchdog flag on this device
    float *scratch = nullptr;    // device address of g_noalloc_scratch on this device
};
NoAllocDevice g_na[kMaxDevices];
std::mutex g_na_mu;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Once per device, with that device current: the SM count and the static array's address.
mx_status noalloc_setup(NoAllocDevice **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { mxk::record_cuda_error(e); return MX_ERR_CUDA; }
    if (dev < 0 || dev >= kMaxDevices) return MX_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_na_mu);
    NoAllocDevice &d = g_na[dev];
    if (!d.ready) {
        e = mxk::device_info(&d.num_sms, &d.watchdog);   // SM count and watchdog address; no allocation
        if (e != cudaSuccess) { mxk::record_cuda_error(e); return MX_ERR_CUDA; }
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) { mxk::record_cuda_error(e); return MX_ERR_CUDA; }
        d.scratch = static_cast<float *>(p);
        d.ready = true;
    }
    *out = &d;
    return MX_OK;
}

}  // namespace

extern "C" mx_status mx_quantize_nvfp4_noalloc(const void *src_bf16, int64_t rows, int64_t cols,
                                               void *out_elems, uint8_t *out_scales,
                                               mx_scale_layout layout, uint8_t *out_scales_alt,
                                               float *global_scale, mx_stream_t stream) {
    if (layout != MX_LAYOUT_ROWMAJOR && layout != MX_LAYOUT_TCGEN05 &&
        layout != (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05))
        return MX_ERR_LAYOUT;
    const bool both = layout == (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05);
    if (both != (out_scales_alt != nullptr)) return MX_ERR_LAYOUT;
    if (rows < 0 || cols < 0 || cols % 16) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!mxk::stream_supported(rows, cols)) return MX_ERR_SHAPE;
    if (!src_bf16 || !out_elems || !out_scales || !global_scale) return MX_ERR_ARG;
    if (!aligned(src_bf16, 16) || !aligned(out_elems, 16) || !aligned(global_scale, 4)) return MX_ERR_ALIGN;

    uint8_t *rm = nullptr, *tc = nullptr;
    if (both) { rm = out_scales; tc = out_scales_alt; }
    else if (layout == MX_LAYOUT_ROWMAJOR) rm = out_scales;
    else tc = out_scales;

    NoAllocDevice *d = nullptr;
    mx_status st = noalloc_setup(&d);
    if (st != MX_OK) return st;
    // One partial maximum per CTA of the maximum pass: min(16 KiB tiles, 3 per SM).
    const int64_t tiles = (rows * cols * 2 + 16383) / 16384;
    const int64_t needed = tiles < 3 * (int64_t)d->num_sms ? tiles : 3 * (int64_t)d->num_sms;
    if (needed > MX_NOALLOC_MAX_PARTIALS) return MX_ERR_SHAPE;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mxk::launch_stream_nvfp4(src_bf16, rows, cols, d->scratch, MX_NOALLOC_MAX_PARTIALS, 0,
                                             global_scale, out_elems, rm, tc, d->watchdog, d->num_sms, s);
    if (e == cudaSuccess && tc) e = mxk::launch_tcgen05_pad(tc, rows, cols / 16, s);
    if (e != cudaSuccess) { mxk::record_cuda_error(e); return MX_ERR_CUDA; }
    return MX_OK;
}
