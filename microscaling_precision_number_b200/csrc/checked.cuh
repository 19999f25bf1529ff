// checked.cuh -- the bounds-checked build of the kernels (compiled with -DMX_CHECKED).
//
// In that build every global store a kernel makes goes through out_ok(): the address
// range it writes must lie inside one of the output ranges the launcher registered for
// the launch -- extents the launcher computes on the host from the shapes, independently
// of the kernel's own index arithmetic.  A store outside all of them is not made; the
// first such store records kOobCode in the device's watchdog flag (read with
// mx_watchdog_status), so a test sees it without any memory fault.  In the normal build
// out_ok() is a constant true and nothing of this is compiled in.
//
// The registered ranges live in a per-translation-unit device variable, written with a
// stream-ordered copy right before each launch; a checked build is for single-stream test
// runs (two streams launching kernels of the same file at once would share it).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "internal.h"

namespace mxk {

constexpr int kOobCode = 64;                 // watchdog code: a refused out-of-range store
constexpr int kMaxOutRanges = 8;

struct OutRange {
    const void *base;
    uint64_t bytes;
};

#ifdef MX_CHECKED
struct CheckState {
    int *flag;
    int n;
    uint64_t lo[kMaxOutRanges], hi[kMaxOutRanges];
};
static __device__ CheckState g_check;

__device__ __forceinline__ bool out_ok(const void *p, uint32_t nbytes) {
    const uint64_t a = reinterpret_cast<uint64_t>(p);
    for (int i = 0; i < g_check.n; i++)
        if (a >= g_check.lo[i] && a + nbytes <= g_check.hi[i]) return true;
    if (g_check.flag) atomicCAS(g_check.flag, 0, kOobCode);
    return false;
}

// Registers the launch's output ranges (null bases are skipped).  The test-only
// environment variable MX_CHECKED_SHRINK=n shortens the last registered range by n bytes,
// so that a test can watch the checks refuse stores that are in fact inside the buffer.
cudaError_t set_out_ranges_impl(const OutRange *r, int n, int *flag, cudaStream_t st, CheckState *sym);
template <int N>
static inline cudaError_t set_out_ranges(const OutRange (&r)[N], cudaStream_t st) {
    static_assert(N <= kMaxOutRanges, "too many output ranges");
    CheckState *sym = nullptr;
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&sym), g_check);
    if (e != cudaSuccess) return e;
    int nsm = 0, *flag = nullptr;
    e = device_info(&nsm, &flag);
    if (e != cudaSuccess) return e;
    return set_out_ranges_impl(r, N, flag, st, sym);
}
#else
__device__ __forceinline__ bool out_ok(const void *, uint32_t) { return true; }
template <int N>
static inline cudaError_t set_out_ranges(const OutRange (&)[N], cudaStream_t) { return cudaSuccess; }
#endif

// A global store of v at p, bounds-checked in the checked build.
template <typename T>
__device__ __forceinline__ void out_store(T *p, const T &v) {
    if (out_ok(p, sizeof(T))) *p = v;
}

}  // namespace mxk
