// checked.cuh -- index checks of the bounds-checked debug build.
//
// Built with -DNVFP4_BOUNDS_CHECK (build.py, checked=True: libnvfp4_checked.so),
// every guarded global access first checks that the elements it touches,
// [first, first + count), lie inside [0, extent) of the buffer as the call's
// shapes define it.  A failed check skips the access and records the source
// line of the first failure in a flag of this translation unit; nothing traps.
// nvfp4_bounds_status() reads and clears the flags of all translation units.
// Without the macro NVFP4_IN_RANGE is the constant true and the product
// kernels are unchanged.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#ifdef NVFP4_BOUNDS_CHECK
namespace {  // one flag and one check per translation unit
__device__ int tu_bounds_site = 0;  // 0, or the source line of the first failed check
__device__ __forceinline__ bool tu_in_range(int64_t first, int64_t count, int64_t extent, int line) {
    if (first >= 0 && count >= 0 && first <= extent && count <= extent - first) return true;
    atomicCAS(&tu_bounds_site, 0, line);
    return false;
}
}  // namespace
#define NVFP4_IN_RANGE(first, count, extent) \
    (tu_in_range((int64_t)(first), (int64_t)(count), (int64_t)(extent), __LINE__))
// Host side: read and clear this translation unit's flag.
#define NVFP4_DEFINE_BOUNDS_READER(fn)                                                  \
    cudaError_t fn(int *site) {                                                         \
        int v = 0;                                                                      \
        cudaError_t e = cudaMemcpyFromSymbol(&v, tu_bounds_site, sizeof(int));          \
        if (e != cudaSuccess) return e;                                                 \
        *site = v;                                                                      \
        if (v == 0) return cudaSuccess;                                                 \
        const int zero = 0;                                                             \
        return cudaMemcpyToSymbol(tu_bounds_site, &zero, sizeof(int));                  \
    }
#else
#define NVFP4_IN_RANGE(first, count, extent) (true)
#define NVFP4_DEFINE_BOUNDS_READER(fn) \
    cudaError_t fn(int *site) {        \
        *site = 0;                     \
        return cudaSuccess;            \
    }
#endif
