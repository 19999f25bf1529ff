// api.cu -- the C ABI of include/mx.h: argument validation, per-device state and dispatch
// to the kernels.  Validation happens entirely on the host before any CUDA call, so a
// rejected call never touches the device.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdlib>
#include <mutex>
#include <utility>

#include "../../include/mx.h"
#include "checked.cuh"
#include "internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

__device__ int g_watchdog_flag = 0;

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    int *watchdog = nullptr;     // device address of g_watchdog_flag
    float *partials = nullptr;   // NVFP4 per-CTA maxima (scratch, allocated once)
    int partials_cap = 0;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

mx_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return MX_ERR_CUDA;
}

mx_status device_state(DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return MX_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.watchdog), g_watchdog_flag);
        if (e != cudaSuccess) return cuda_fail(e);
        d.ready = true;
    }
    *out = &d;
    return MX_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool fmt_ok(int f) { return f >= MX_FMT_E4M3 && f <= MX_FMT_INT8; }
bool mx_block_fmt(int f) { return fmt_ok(f) && f != MX_FMT_NVFP4; }
// 8-bit-container element formats of the mxf8f6f4 tensor-core kind
bool f8f6_fmt(int f) { return f == MX_FMT_E4M3 || f == MX_FMT_E5M2 || f == MX_FMT_E2M3 || f == MX_FMT_E3M2; }
int block_of(int f) { return f == MX_FMT_NVFP4 ? 16 : 32; }
bool single_layout(int l) { return l == MX_LAYOUT_ROWMAJOR || l == MX_LAYOUT_TCGEN05; }

}  // namespace

namespace mxk {
void record_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }

cudaError_t device_info(int *num_sms, int **watchdog) {
    DeviceState *d = nullptr;
    if (device_state(&d) != MX_OK) return (cudaError_t)g_last_cuda_error;
    *num_sms = d->num_sms;
    *watchdog = d->watchdog;
    return cudaSuccess;
}

#ifdef MX_CHECKED
cudaError_t set_out_ranges_impl(const OutRange *r, int n, int *flag, cudaStream_t st, CheckState *sym) {
    CheckState h = {};
    h.flag = flag;
    for (int i = 0; i < n; i++) {
        if (!r[i].base) continue;
        const uint64_t lo = reinterpret_cast<uint64_t>(r[i].base);
        h.lo[h.n] = lo;
        h.hi[h.n] = lo + r[i].bytes;
        h.n++;
    }
    // test hook: shorten the last registered range (stores beyond it are then refused)
    if (const char *shrink = std::getenv("MX_CHECKED_SHRINK")) {
        const uint64_t k = std::strtoull(shrink, nullptr, 10);
        if (h.n > 0 && h.hi[h.n - 1] - h.lo[h.n - 1] > k) h.hi[h.n - 1] -= k;
    }
    // pageable source: staged by the runtime before the call returns, so `h` may go
    return cudaMemcpyAsync(sym, &h, sizeof h, cudaMemcpyHostToDevice, st);
}
#endif

void *tensor_map_encoder() {
    static void *fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = p;
    });
    return fn;
}
}  // namespace mxk

extern "C" {

int64_t mx_scale_bytes(int64_t rows, int64_t scale_cols, mx_scale_layout layout) {
    if (rows < 0 || scale_cols < 0) return -1;
    if (layout == MX_LAYOUT_ROWMAJOR) return rows * scale_cols;
    if (layout == MX_LAYOUT_TCGEN05) return ((rows + 127) / 128) * ((scale_cols + 3) / 4) * 512;
    return -1;
}

const char *mx_status_string(mx_status s) {
    switch (s) {
    case MX_OK: return "MX_OK";
    case MX_ERR_ARG: return "MX_ERR_ARG: null pointer, unknown enum or unsupported combination";
    case MX_ERR_SHAPE: return "MX_ERR_SHAPE: negative size or size not a multiple of the block/tile";
    case MX_ERR_ALIGN: return "MX_ERR_ALIGN: pointer not aligned as required";
    case MX_ERR_LAYOUT: return "MX_ERR_LAYOUT: invalid scale layout mask or missing second scale buffer";
    case MX_ERR_CUDA: return "MX_ERR_CUDA: CUDA call failed (see mx_last_cuda_error)";
    case MX_ERR_TIMEOUT: return "MX_ERR_TIMEOUT: a bounded device wait gave up";
    default: return "unknown mx_status";
    }
}

int mx_last_cuda_error(void) { return g_last_cuda_error; }

mx_status mx_watchdog_status(int *code, int clear) {
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e);
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_watchdog_flag, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    if (clear && v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_watchdog_flag, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (code) *code = v;
    return v ? MX_ERR_TIMEOUT : MX_OK;
}

mx_status mx_watchdog_selftest(uint32_t limit_us, mx_stream_t stream) {
    if (limit_us < 1 || limit_us > 100000) return MX_ERR_ARG;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    const cudaError_t e = mxk::launch_watchdog_selftest((uint64_t)limit_us * 1000ull, d->watchdog,
                                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

// One fixed-size scratch per device for the NVFP4 per-CTA partial maxima, allocated on
// first use (every call writes each slot it later reads).
static mx_status nvfp4_scratch(DeviceState *d) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!d->partials) {
        const int nf = mxk::stream_nvfp4_scratch_floats(d->num_sms);
        const cudaError_t e = cudaMalloc(reinterpret_cast<void **>(&d->partials), sizeof(float) * (size_t)nf);
        if (e != cudaSuccess) return cuda_fail(e);
        d->partials_cap = nf;
    }
    return MX_OK;
}

mx_status mx_quantize(const void *src, int64_t rows, int64_t cols, mx_fmt fmt, mx_axis axis,
                      mx_scale_rounding rounding, void *out_elems, uint8_t *out_scales,
                      mx_scale_layout layout, uint8_t *out_scales_alt, float *global_scale,
                      mx_stream_t stream) {
    if (!fmt_ok(fmt) || (axis != MX_AXIS_ROW && axis != MX_AXIS_COL) ||
        (rounding != MX_SCALE_FLOOR_OCP && rounding != MX_SCALE_CEIL_RECIPE))
        return MX_ERR_ARG;
    if (fmt == MX_FMT_NVFP4 && axis != MX_AXIS_ROW) return MX_ERR_ARG;
    if ((fmt == MX_FMT_NVFP4) != (global_scale != nullptr)) return MX_ERR_ARG;
    if (layout != MX_LAYOUT_ROWMAJOR && layout != MX_LAYOUT_TCGEN05 &&
        layout != (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05))
        return MX_ERR_LAYOUT;
    const bool both = layout == (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05);
    if (both != (out_scales_alt != nullptr)) return MX_ERR_LAYOUT;
    if (rows < 0 || cols < 0) return MX_ERR_SHAPE;
    const int B = block_of(fmt);
    if ((axis == MX_AXIS_ROW ? cols : rows) % B) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!mxk::stream_supported(rows, cols)) return MX_ERR_SHAPE;
    if (!src || !out_elems || !out_scales) return MX_ERR_ARG;
    if (!aligned(src, 16) || !aligned(out_elems, 16)) return MX_ERR_ALIGN;
    if (global_scale && !aligned(global_scale, 4)) return MX_ERR_ALIGN;

    uint8_t *rm = nullptr, *tc = nullptr;
    if (both) { rm = out_scales; tc = out_scales_alt; }
    else if (layout == MX_LAYOUT_ROWMAJOR) rm = out_scales;
    else tc = out_scales;

    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    const bool ceil = rounding == MX_SCALE_CEIL_RECIPE;

    if (fmt == MX_FMT_NVFP4) {
        st = nvfp4_scratch(d);
        if (st != MX_OK) return st;
        e = mxk::launch_stream_nvfp4(src, rows, cols, d->partials, 3 * d->num_sms, 0, global_scale, out_elems, rm, tc,
                                     d->watchdog, d->num_sms, s);
        if (e != cudaSuccess) return cuda_fail(e);
        if (tc) {
            e = mxk::launch_tcgen05_pad(tc, rows, cols / 16, s);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return MX_OK;
    }

    if (axis == MX_AXIS_ROW) {
        e = mxk::launch_stream_rows_mx(src, rows, cols, fmt, ceil, out_elems, rm, tc, nullptr, d->watchdog,
                                       d->num_sms, s);
        if (e != cudaSuccess) return cuda_fail(e);
        if (tc) {
            e = mxk::launch_tcgen05_pad(tc, rows, cols / 32, s);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return MX_OK;
    }

    // Column-wise: the TMA-staged kernel with only the transposed output enabled; the
    // requested scale layouts (one or both) are written by the same pass.
    if (cols % 8 != 0) return MX_ERR_SHAPE;    // the TMA row pitch (cols * 2 bytes) must be a multiple of 16
    e = mxk::launch_quant_dual(src, rows, cols, fmt, ceil, nullptr, nullptr, nullptr, out_elems, rm, tc,
                               d->watchdog, d->num_sms, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (tc) {
        e = mxk::launch_tcgen05_pad(tc, cols, rows / 32, s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return MX_OK;
}

mx_status mx_quantize_mx_nvfp4(const void *src, int64_t rows, int64_t cols, mx_fmt fmt,
                               mx_scale_rounding rounding, void *mx_elems, uint8_t *mx_scales,
                               mx_scale_layout mx_layout, uint8_t *mx_scales_alt, void *nv_elems,
                               uint8_t *nv_scales, mx_scale_layout nv_layout, uint8_t *nv_scales_alt,
                               float *global_scale, mx_stream_t stream) {
    if (!mx_block_fmt(fmt)) return MX_ERR_ARG;
    if (rounding != MX_SCALE_FLOOR_OCP && rounding != MX_SCALE_CEIL_RECIPE) return MX_ERR_ARG;
    const int both = MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05;
    for (const auto &[lay, alt] : {std::pair<int, const uint8_t *>{mx_layout, mx_scales_alt},
                                   std::pair<int, const uint8_t *>{nv_layout, nv_scales_alt}}) {
        if (!single_layout(lay) && lay != both) return MX_ERR_LAYOUT;
        if ((lay == both) != (alt != nullptr)) return MX_ERR_LAYOUT;
    }
    if (rows < 0 || cols < 0) return MX_ERR_SHAPE;
    if (cols % 32) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!mxk::stream_supported(rows, cols)) return MX_ERR_SHAPE;
    if (!src || !mx_elems || !mx_scales || !nv_elems || !nv_scales || !global_scale) return MX_ERR_ARG;
    if (!aligned(src, 16) || !aligned(mx_elems, 16) || !aligned(nv_elems, 16)) return MX_ERR_ALIGN;
    if (!aligned(global_scale, 4)) return MX_ERR_ALIGN;
    uint8_t *mrm = mx_layout == MX_LAYOUT_TCGEN05 ? nullptr : mx_scales;
    uint8_t *mtc = mx_layout == MX_LAYOUT_TCGEN05 ? mx_scales : mx_scales_alt;
    uint8_t *nrm = nv_layout == MX_LAYOUT_TCGEN05 ? nullptr : nv_scales;
    uint8_t *ntc = nv_layout == MX_LAYOUT_TCGEN05 ? nv_scales : nv_scales_alt;

    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    st = nvfp4_scratch(d);
    if (st != MX_OK) return st;
    const int n_partials = mxk::stream_rows_grid(rows, cols, d->num_sms);
    if (n_partials > d->partials_cap) return MX_ERR_SHAPE;      // cannot happen: 3 per SM, the scratch holds 8
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the MX pass also leaves the NVFP4 partial maxima; the NVFP4 pass then skips its own
    // maximum pass (programmatic dependent launch orders it after the MX pass)
    cudaError_t e = mxk::launch_stream_rows_mx(src, rows, cols, fmt, rounding == MX_SCALE_CEIL_RECIPE, mx_elems, mrm,
                                               mtc, d->partials, d->watchdog, d->num_sms, s);
    if (e == cudaSuccess)
        e = mxk::launch_stream_nvfp4(src, rows, cols, d->partials, d->partials_cap, n_partials, global_scale, nv_elems,
                                     nrm, ntc, d->watchdog, d->num_sms, s);
    if (e == cudaSuccess && mtc) e = mxk::launch_tcgen05_pad(mtc, rows, cols / 32, s);
    if (e == cudaSuccess && ntc) e = mxk::launch_tcgen05_pad(ntc, rows, cols / 16, s);
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

mx_status mx_quantize_dual(const void *src, int64_t rows, int64_t cols, mx_fmt fmt,
                           mx_scale_rounding rounding, void *row_elems, uint8_t *row_scales,
                           void *col_elems, uint8_t *col_scales, mx_scale_layout layout,
                           uint8_t *row_scales_alt, uint8_t *col_scales_alt, mx_stream_t stream) {
    if (!mx_block_fmt(fmt)) return MX_ERR_ARG;
    if (rounding != MX_SCALE_FLOOR_OCP && rounding != MX_SCALE_CEIL_RECIPE) return MX_ERR_ARG;
    const bool both = layout == (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05);
    if (!single_layout(layout) && !both) return MX_ERR_LAYOUT;
    if (both != (row_scales_alt != nullptr) || both != (col_scales_alt != nullptr)) return MX_ERR_LAYOUT;
    if (rows < 0 || cols < 0) return MX_ERR_SHAPE;
    if (rows % 32 || cols % 32) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!src || !row_elems || !row_scales || !col_elems || !col_scales) return MX_ERR_ARG;
    if (!aligned(src, 16) || !aligned(row_elems, 16) || !aligned(col_elems, 16)) return MX_ERR_ALIGN;
    uint8_t *row_rm = nullptr, *row_tc = nullptr, *col_rm = nullptr, *col_tc = nullptr;
    if (both) {
        row_rm = row_scales; row_tc = row_scales_alt; col_rm = col_scales; col_tc = col_scales_alt;
    } else if (layout == MX_LAYOUT_ROWMAJOR) {
        row_rm = row_scales; col_rm = col_scales;
    } else {
        row_tc = row_scales; col_tc = col_scales;
    }
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mxk::launch_quant_dual(src, rows, cols, fmt, rounding == MX_SCALE_CEIL_RECIPE, row_elems,
                                           row_rm, row_tc, col_elems, col_rm, col_tc, d->watchdog, d->num_sms, s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (row_tc) {
        e = mxk::launch_tcgen05_pad(row_tc, rows, cols / 32, s);
        if (e != cudaSuccess) return cuda_fail(e);
        e = mxk::launch_tcgen05_pad(col_tc, cols, rows / 32, s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return MX_OK;
}

mx_status mx_dequantize(const void *elems, const uint8_t *scales, const float *global_scale,
                        int64_t rows, int64_t cols, mx_fmt fmt, mx_scale_layout layout,
                        void *out_bf16, mx_stream_t stream) {
    if (!fmt_ok(fmt)) return MX_ERR_ARG;
    if ((fmt == MX_FMT_NVFP4) != (global_scale != nullptr)) return MX_ERR_ARG;
    if (!single_layout(layout)) return MX_ERR_LAYOUT;
    if (rows < 0 || cols < 0) return MX_ERR_SHAPE;
    if (cols % block_of(fmt)) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!mxk::stream_supported(rows, cols)) return MX_ERR_SHAPE;
    if (!elems || !scales || !out_bf16) return MX_ERR_ARG;
    if (!aligned(elems, 16) || !aligned(out_bf16, 16)) return MX_ERR_ALIGN;
    if (global_scale && !aligned(global_scale, 4)) return MX_ERR_ALIGN;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool tc = layout == MX_LAYOUT_TCGEN05;
    cudaError_t e = fmt == MX_FMT_NVFP4
                        ? mxk::launch_stream_dequant_nvfp4(elems, scales, global_scale, rows, cols, tc, out_bf16,
                                                           d->watchdog, d->num_sms, s)
                        : mxk::launch_stream_dequant_mx(elems, scales, rows, cols, fmt, tc, out_bf16, d->watchdog,
                                                        d->num_sms, s);
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

mx_status mx_cast(const void *src, int64_t n, mx_fmt fmt, void *out, mx_stream_t stream) {
    if (!mx_block_fmt(fmt) || fmt == MX_FMT_INT8) return MX_ERR_ARG;
    if (n < 0 || (fmt == MX_FMT_E2M1 && n % 2) || ((fmt == MX_FMT_E2M3 || fmt == MX_FMT_E3M2) && n % 4))
        return MX_ERR_SHAPE;                                  // whole bytes of packed codes
    if (n == 0) return MX_OK;
    if (!src || !out) return MX_ERR_ARG;
    if (!aligned(src, 16) || !aligned(out, 16)) return MX_ERR_ALIGN;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    cudaError_t e = mxk::launch_cast(src, n, fmt, out, d->num_sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

mx_status mx_gemm(mx_operand A, mx_operand B, void *C, int64_t M, int64_t N, int64_t K,
                  mx_stream_t stream) {
    const bool f8 = f8f6_fmt(A.fmt) && (f8f6_fmt(B.fmt) || B.fmt == MX_FMT_E2M1);
    const bool mxf4 = A.fmt == MX_FMT_E2M1 && B.fmt == MX_FMT_E2M1;
    const bool nvf4 = A.fmt == MX_FMT_NVFP4 && B.fmt == MX_FMT_NVFP4;
    if (!f8 && !mxf4 && !nvf4) return MX_ERR_ARG;
    if (nvf4 != (A.global_scale != nullptr) || nvf4 != (B.global_scale != nullptr)) return MX_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return MX_ERR_SHAPE;
    if (M % 128 || N % 128 || K % (f8 ? 128 : 256)) return MX_ERR_SHAPE;
    if (M > (int64_t)1 << 30 || N > (int64_t)1 << 30 || K > (int64_t)1 << 30) return MX_ERR_SHAPE;
    if (M == 0 || N == 0) return MX_OK;
    if (!A.elems || !A.scales || !B.elems || !B.scales || !C) return MX_ERR_ARG;
    if (!aligned(A.elems, 32) || !aligned(B.elems, 32) || !aligned(A.scales, 16) || !aligned(B.scales, 16) ||
        !aligned(C, 16) || !aligned(A.global_scale, 4) || !aligned(B.global_scale, 4))
        return MX_ERR_ALIGN;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (K == 0) {
        e = cudaMemsetAsync(C, 0, (size_t)(M * N * 2), s);   // empty sum
        return e == cudaSuccess ? MX_OK : cuda_fail(e);
    }
    // 256 x 256 tiles on CTA pairs when the shape allows (8192^3: 1-3% faster than single
    // CTAs for the 8-bit and MXFP4 kinds, 13% for NVFP4 x NVFP4), else 128 x {256, 128} tiles
    if (mxk::gemm_pair_supported(M, N))
        e = mxk::launch_gemm_pair(A.elems, A.scales, A.fmt, A.global_scale, B.elems, B.scales, B.fmt, B.global_scale,
                                  C, M, N, K, d->watchdog, d->num_sms, s);
    else
        e = mxk::launch_gemm(A.elems, A.scales, A.fmt, A.global_scale, B.elems, B.scales, B.fmt, B.global_scale, C,
                             M, N, K, d->watchdog, d->num_sms, s);
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

mx_status mx_mxfp4_to_fp8_blocks(const void *elems, const uint8_t *scales, int64_t rows, int64_t cols,
                                 void *out_fp8, float *block_scales, uint8_t *block_exact, mx_stream_t stream) {
    if (rows < 0 || cols < 0 || rows % 128 || cols % 128) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if ((rows / 128) * (cols / 128) > 0x7FFFFFFF) return MX_ERR_SHAPE;
    if (!elems || !scales || !out_fp8 || !block_scales || !block_exact) return MX_ERR_ARG;
    if (!aligned(elems, 16) || !aligned(out_fp8, 16) || !aligned(block_scales, 4)) return MX_ERR_ALIGN;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    const cudaError_t e = mxk::launch_mxfp4_to_fp8_blocks(elems, scales, rows, cols, out_fp8, block_scales,
                                                          block_exact, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

mx_status mx_quantize_train(const void *src, int64_t rows, int64_t cols, mx_fmt fmt, mx_scale_rounding rounding,
                            int rht16, unsigned rht_signs, const uint8_t *sr_random, void *out_elems,
                            uint8_t *out_scales, mx_scale_layout layout, uint8_t *out_scales_alt, float *global_scale,
                            mx_stream_t stream) {
    if (fmt != MX_FMT_E4M3 && fmt != MX_FMT_E5M2 && fmt != MX_FMT_E2M1 && fmt != MX_FMT_NVFP4) return MX_ERR_ARG;
    if (rounding != MX_SCALE_FLOOR_OCP && rounding != MX_SCALE_CEIL_RECIPE) return MX_ERR_ARG;
    if (rht16 != 0 && rht16 != 1) return MX_ERR_ARG;
    if ((fmt == MX_FMT_NVFP4) != (global_scale != nullptr)) return MX_ERR_ARG;
    if (layout != MX_LAYOUT_ROWMAJOR && layout != MX_LAYOUT_TCGEN05 &&
        layout != (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05))
        return MX_ERR_LAYOUT;
    const bool both = layout == (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05);
    if (both != (out_scales_alt != nullptr)) return MX_ERR_LAYOUT;
    if (rows < 0 || cols < 0 || cols % block_of(fmt)) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!mxk::stream_supported(rows, cols)) return MX_ERR_SHAPE;
    if (!src || !out_elems || !out_scales) return MX_ERR_ARG;
    if (!aligned(src, 16) || !aligned(out_elems, 16) || !aligned(sr_random, 16) || !aligned(global_scale, 4))
        return MX_ERR_ALIGN;
    uint8_t *rm = nullptr, *tc = nullptr;
    if (both) { rm = out_scales; tc = out_scales_alt; }
    else if (layout == MX_LAYOUT_ROWMAJOR) rm = out_scales;
    else tc = out_scales;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    if (fmt == MX_FMT_NVFP4) {
        st = nvfp4_scratch(d);
        if (st != MX_OK) return st;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mxk::launch_quantize_train(src, rows, cols, fmt, rounding == MX_SCALE_CEIL_RECIPE, rht16 != 0,
                                               rht_signs & 0xFFFFu, sr_random, d->partials, d->partials_cap,
                                               global_scale, out_elems, rm, tc, d->num_sms, s);
    if (e == cudaSuccess && tc) e = mxk::launch_tcgen05_pad(tc, rows, cols / block_of(fmt), s);
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

mx_status mx_quantize_nvfp4_2d(const void *src, int64_t rows, int64_t cols, void *out_elems, uint8_t *out_scales,
                               mx_scale_layout layout, uint8_t *out_scales_alt, float *global_scale,
                               mx_stream_t stream) {
    if (layout != MX_LAYOUT_ROWMAJOR && layout != MX_LAYOUT_TCGEN05 &&
        layout != (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05))
        return MX_ERR_LAYOUT;
    const bool both = layout == (MX_LAYOUT_ROWMAJOR | MX_LAYOUT_TCGEN05);
    if (both != (out_scales_alt != nullptr)) return MX_ERR_LAYOUT;
    if (rows < 0 || cols < 0 || rows % 16 || cols % 16) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;
    if (!mxk::stream_supported(rows, cols)) return MX_ERR_SHAPE;
    if (!src || !out_elems || !out_scales || !global_scale) return MX_ERR_ARG;
    if (!aligned(src, 16) || !aligned(out_elems, 16) || !aligned(global_scale, 4)) return MX_ERR_ALIGN;
    uint8_t *rm = nullptr, *tc = nullptr;
    if (both) { rm = out_scales; tc = out_scales_alt; }
    else if (layout == MX_LAYOUT_ROWMAJOR) rm = out_scales;
    else tc = out_scales;
    DeviceState *d = nullptr;
    mx_status st = device_state(&d);
    if (st != MX_OK) return st;
    st = nvfp4_scratch(d);
    if (st != MX_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = mxk::launch_stream_nvfp4_2d(src, rows, cols, d->partials, d->partials_cap, global_scale,
                                                out_elems, rm, tc, d->num_sms, d->watchdog, s);
    if (e == cudaSuccess && tc) e = mxk::launch_tcgen05_pad(tc, rows, cols / 16, s);
    return e == cudaSuccess ? MX_OK : cuda_fail(e);
}

}  // extern "C"
