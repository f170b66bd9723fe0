// dcheck.cuh -- device-side index checks of the bounds build.
//
// Compiled with -DM3_DEVICE_CHECKS (the library libm3_bounds.so), every
// global-memory access a kernel makes through a plain pointer first checks
// that its element range lies inside the buffer the host validated (extents
// computed from the problem's dims); a failed check skips the access and
// records the site, the first index and the extent of the first failure, and
// counts failures, in device words of the kernel's own translation unit,
// which m3_stream_status reads back (M3_ERR_BOUNDS).  No trap, no assert: the
// kernel runs on and the context stays usable.  Tile copies (TMA) are not
// checked here: the tensor maps carry the extents and the hardware fills
// out-of-range elements.  In the normal build every check is the constant
// `true` and compiles to nothing.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "m3_internal.h"  // DcheckRecord

namespace m3 {
namespace dchk {

// The predicate of every check: elements [i, i + cnt) inside [0, n), without
// forming i + cnt (no overflow for any 64-bit operands with n >= 0).
__host__ __device__ __forceinline__ constexpr bool in_range(long long i, long long cnt, long long n) {
    return i >= 0 && cnt >= 0 && cnt <= n && i <= n - cnt;
}

#ifdef M3_DEVICE_CHECKS
static __device__ unsigned g_count;
static __device__ unsigned g_site;
static __device__ long long g_index, g_extent;

static __device__ __noinline__ void record(unsigned site, long long i, long long n) {
    if (atomicAdd(&g_count, 1u) == 0u) {
        g_site = site;
        g_index = i;
        g_extent = n;
    }
}

// True when elements [i, i + cnt) lie inside [0, n); otherwise records the
// failure and returns false so that the caller skips the access.
__device__ __forceinline__ bool in(unsigned site, long long i, long long cnt, long long n) {
    if (in_range(i, cnt, n)) return true;
    record(site, i, n);
    return false;
}
#else
__device__ __forceinline__ constexpr bool in(unsigned, long long, long long, long long) { return true; }
#endif

}  // namespace dchk
}  // namespace m3

// Defines `cudaError_t NAME(m3::DcheckRecord *r)`, the host reader of this
// translation unit's record: copies it out and clears it (the normal build
// reports nothing).  Call after the work has completed.
#ifdef M3_DEVICE_CHECKS
#define M3_DCHECK_READER(NAME)                                                              \
    cudaError_t NAME(m3::DcheckRecord *r) {                                                 \
        *r = m3::DcheckRecord{0u, 0u, 0, 0};                                                \
        cudaError_t e = cudaMemcpyFromSymbol(&r->count, m3::dchk::g_count, sizeof(unsigned)); \
        if (e != cudaSuccess || r->count == 0u) return e;                                   \
        if ((e = cudaMemcpyFromSymbol(&r->site, m3::dchk::g_site, sizeof(unsigned))) != cudaSuccess) return e; \
        if ((e = cudaMemcpyFromSymbol(&r->index, m3::dchk::g_index, sizeof(long long))) != cudaSuccess)       \
            return e;                                                                       \
        if ((e = cudaMemcpyFromSymbol(&r->extent, m3::dchk::g_extent, sizeof(long long))) != cudaSuccess)     \
            return e;                                                                       \
        const unsigned zero = 0u;                                                           \
        return cudaMemcpyToSymbol(m3::dchk::g_count, &zero, sizeof(unsigned));              \
    }
#else
#define M3_DCHECK_READER(NAME)                    \
    cudaError_t NAME(m3::DcheckRecord *r) {       \
        *r = m3::DcheckRecord{0u, 0u, 0, 0};      \
        return cudaSuccess;                       \
    }
#endif
