// selftest.cu -- exercises the device-timeout path without a fault.
//
// One CTA initialises an mbarrier in shared memory that nothing ever arrives
// on and waits on it with the same bounded loop (try_wait + %globaltimer) the
// GEMM uses, but with a caller-chosen limit.  When the limit passes it records
// NVFP4_ERR_DEVICE_TIMEOUT in the workspace status word and returns, leaving
// the context usable.  The pages have no counterpart: this checks the
// library's own error plumbing.
#include "checked.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

__global__ void wait_timeout_kernel(int *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    uint64_t t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
        uint32_t done;
        // phase 0 never completes: no thread arrives
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\tselp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(b)
            : "memory");
        if (done) return;  // unreachable: reported as success by leaving the status alone
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > limit_ns) break;
    }
    atomicExch(status, 7);  // NVFP4_ERR_DEVICE_TIMEOUT
}

// One check that passes (element 0) and one that fails (element n of an
// n-element range); buf holds n + 1 bytes.
__global__ void bounds_selftest_kernel(uint8_t *buf, int64_t n) {
    if (NVFP4_IN_RANGE(0, 1, n)) buf[0] = 1;
    if (NVFP4_IN_RANGE(n, 1, n)) buf[n] = 1;
}

}  // namespace

cudaError_t launch_selftest_bounds(uint8_t *buf, int64_t n, cudaStream_t s, int *launches) {
    bounds_selftest_kernel<<<1, 1, 0, s>>>(buf, n);
    ++*launches;
    return cudaGetLastError();
}

NVFP4_DEFINE_BOUNDS_READER(read_bounds_selftest)

cudaError_t launch_wait_timeout(int *status, uint64_t limit_ns, cudaStream_t s, int *launches) {
    wait_timeout_kernel<<<1, 1, 0, s>>>(status, limit_ns);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace nvfp4
