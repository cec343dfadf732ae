// noalloc.cu -- nvfp4_linear_fwd_noalloc: the Fprop call for callers that
// cannot allocate device memory, e.g. code running inside a framework that
// owns every byte of device memory through its own pool (so a side cudaMalloc
// would fail or break its accounting), or latency-critical loops where the
// implicit synchronisation of cudaMalloc/cudaFree would stall other streams.
//
// The scratch that nvfp4_linear_fwd takes from a caller's workspace (status
// word, amax partials, both quantised operands) lives instead in one fixed
// file-scope device buffer of kNoAllocScratchBytes.  Every GPU that loads this
// library holds that buffer until the process exits.
#include <mutex>

#include "internal.h"
#include "nvfp4.h"

namespace {

constexpr size_t kNoAllocScratchBytes = NVFP4_NOALLOC_SCRATCH_BYTES;  // 16 MiB per device

// In host code this name is only a stand-in for the device object: a kernel
// must be given the address from cudaGetSymbolAddress, never the name.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
uint8_t *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the fixed buffer on the current device, looked up once per
// device (with that device current) on the first call there.
nvfp4_status scratch_address(uint8_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
        g_scratch_addr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_scratch_addr[dev];
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_linear_fwd_noalloc(const void *X, const void *W, void *Y, int64_t M, int64_t N,
                                                 int64_t K, nvfp4_dtype dtype, nvfp4_dtype y_dtype,
                                                 cudaStream_t stream) {
    if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_SHAPE;
    // Problems whose scratch (the forward operands only) exceeds the fixed
    // buffer are refused before anything runs.
    if (nvfp4::linear_fwd_workspace_bytes(M, N, K) > kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;
    if (M == 0 || N == 0) return nvfp4_linear_fwd(X, W, Y, M, N, K, dtype, y_dtype, nullptr, 0, stream);
    uint8_t *scratch = nullptr;
    nvfp4_status st = scratch_address(&scratch);
    if (st != NVFP4_OK) return st;
    // Every check nvfp4_linear_fwd makes runs first, so a refused call touches
    // neither the shared buffer nor the stream.
    st = nvfp4::linear_fwd_validate(X, W, Y, M, N, K, dtype, y_dtype, scratch, kNoAllocScratchBytes);
    if (st != NVFP4_OK) return st;
    // The device status word must start at zero; the rest is overwritten before it is read.
    if (cudaMemsetAsync(scratch, 0, nvfp4::kStatusBytes, stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    return nvfp4_linear_fwd(X, W, Y, M, N, K, dtype, y_dtype, scratch, kNoAllocScratchBytes, stream);
}
