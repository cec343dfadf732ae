// gemm.cu -- block-scaled NVFP4 GEMM on the sm_100a tensor cores.
//
// C[M x N] = (A . B^T) * sA * sB with A [M x K], B [N x K] both K-major NVFP4:
// packed E2M1 codes, one E4M3 scale per 16 k (the 128x4 scale atoms written by
// the quantiser), one FP32 tensor scale each.  4-bit GEMMs on Blackwell
// tensor cores: nerdman.de, "Nvidia drueckt KI-Training auf 4 Bit runter",
// section "Was konkret passiert ist"; format: aisight.pl, section
// "Architektura NVFP4 kontra ograniczenia mikroskalowania".
//
// One CTA computes one 128 x 256 tile with warp roles:
//   warp 0 (one lane)  producer: TMA loads of the code tiles (128-byte swizzle)
//                      and bulk copies of the scale atoms into a 4-stage ring;
//   warp 1             allocates TMEM; one lane copies each stage's scales into
//                      TMEM (tcgen05.cp) and issues tcgen05.mma
//                      kind::mxf4nvf4 block16 (K = 64 per instruction) with the
//                      FP32 accumulator in TMEM; tcgen05.commit frees the stage;
//   warps 2..5         epilogue: tcgen05.ld of the accumulator (each warp its
//                      32-lane TMEM quarter), scale by sA*sB, store f32 / bf16.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the CTA
// records NVFP4_ERR_DEVICE_TIMEOUT in the status word, drains its own copies
// and MMAs, frees TMEM and returns.  No TMA multicast is used.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int BM = 128, BN = 256, BK = 256;           // BK in elements (128 bytes of codes)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;                   // 16 KB
constexpr int B_BYTES = BN * BK / 2;                   // 32 KB
constexpr int SFA_BYTES = (BM / 128) * (BK / 64) * 512;  // 2 KB
constexpr int SFB_BYTES = (BN / 128) * (BK / 64) * 512;  // 4 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned for the 128B swizzle");
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;                    // acc 256 + SFA 16 + SFB 32, rounded up
constexpr uint32_t TMEM_SFA = 256, TMEM_SFB = 272;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr int kTimeoutStatus = 7;                      // NVFP4_ERR_DEVICE_TIMEOUT

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1) at bits 7-9 /
// 10-12, K-major, N >> 3 at bits 17-22, UE4M3 scales (bit 23 = 0), M >> 4 at
// bits 24-28, scale-factor byte ids 0, dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false once the limit passes or another role has given up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          bool honour_abort = true) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (honour_abort && *abort_flag) return false;
        if (globaltimer() - t0 > WAIT_LIMIT_NS) {
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// Scale atom (32 rows x 16 bytes in smem) -> 32 TMEM lanes x 4 columns, copied to all four lane quarters.
__device__ __forceinline__ void tc_cp_scales(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa, uint32_t sfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(IDESC), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart (SBO); LBO unused; version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Descriptor of a 512-byte scale atom for tcgen05.cp: 8-row x 16-byte core
// matrices stacked 128 bytes apart (SBO), no swizzle.
__device__ __forceinline__ uint64_t sdesc_scales(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

struct KParams {
    const uint8_t *sfa, *sfb;
    const float *tsa, *tsb;
    void *C;
    int64_t ldc;
    int M, N, K;
    int kb4;          // scale atoms per 128-row tile (= ceil(K / 64))
    int b_rowtiles;   // 128-row tiles of B's scale buffer (= ceil(N / 128))
    int c_bf16;
    int *status;
};

__global__ void __launch_bounds__(THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t bar_full = smem_u32(bars), bar_empty = smem_u32(bars + STAGES),
                   bar_acc = smem_u32(bars + 2 * STAGES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int num_kt = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        mbar_init(bar_acc, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- producer ----------------
        int issued = 0;
        for (int kt = 0; kt < num_kt; ++kt) {
            const int s = kt % STAGES;
            const uint32_t ph = (kt / STAGES) & 1;
            if (!mbar_wait(bar_empty + 8 * s, ph ^ 1, abort_flag)) break;
            const int steps = min(BK / 64, (p.K - kt * BK) / 64);
            const int b_tiles = min(2, p.b_rowtiles - 2 * (int)blockIdx.x);
            const uint32_t bytes = A_BYTES + B_BYTES + steps * 512 * (1 + b_tiles);
            uint8_t *st = smem + s * STAGE_BYTES;
            const uint32_t fb = bar_full + 8 * s;
            mbar_expect_tx(fb, bytes);
            tma_load_2d(smem_u32(st), &map_a, fb, kt * (BK / 2), m0);
            tma_load_2d(smem_u32(st + A_BYTES), &map_b, fb, kt * (BK / 2), n0);
            bulk_load(smem_u32(st + A_BYTES + B_BYTES),
                      p.sfa + ((size_t)blockIdx.y * p.kb4 + (size_t)kt * 4) * 512, steps * 512, fb);
            for (int t = 0; t < b_tiles; ++t)
                bulk_load(smem_u32(st + A_BYTES + B_BYTES + SFA_BYTES + t * 2048),
                          p.sfb + ((size_t)(2 * blockIdx.x + t) * p.kb4 + (size_t)kt * 4) * 512, steps * 512, fb);
            issued = kt + 1;
        }
        // Drain: every issued stage must have landed before the CTA may exit.
        for (int kt = max(0, issued - STAGES); kt < issued; ++kt)
            mbar_wait(bar_full + 8 * (kt % STAGES), (kt / STAGES) & 1, abort_flag, false);
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        for (int kt = 0; kt < num_kt; ++kt) {
            const int s = kt % STAGES;
            const uint32_t ph = (kt / STAGES) & 1;
            if (!mbar_wait(bar_full + 8 * s, ph, abort_flag)) break;
            tc_fence_after();
            const int steps = min(BK / 64, (p.K - kt * BK) / 64);
            const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES, ssfa = sb + B_BYTES, ssfb = ssfa + SFA_BYTES;
            for (int j = 0; j < steps; ++j) {
                tc_cp_scales(tmem + TMEM_SFA + 4 * j, sdesc_scales(ssfa + 512 * j));
                tc_cp_scales(tmem + TMEM_SFB + 8 * j, sdesc_scales(ssfb + 512 * j));
                tc_cp_scales(tmem + TMEM_SFB + 8 * j + 4, sdesc_scales(ssfb + 2048 + 512 * j));
            }
            const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sb);
            for (int j = 0; j < steps; ++j)
                tc_mma(tmem, da + 2 * j, db + 2 * j, tmem + TMEM_SFA + 4 * j, tmem + TMEM_SFB + 8 * j,
                       (kt > 0 || j > 0) ? 1u : 0u);
            tc_commit(bar_empty + 8 * s);
        }
        tc_commit(bar_acc);  // arrives once every MMA issued above has completed
    } else if (warp >= 2) {
        // ---------------- epilogue ----------------
        const int quarter = warp & 3;
        bool ok = mbar_wait(bar_acc, 0, abort_flag, false);
        ok = __all_sync(0xFFFFFFFFu, ok) && !*abort_flag;
        tc_fence_after();
        if (ok) {
            const float scale = __fmul_rn(*p.tsa, *p.tsb);
            const int row = m0 + quarter * 32 + lane;
            const bool row_ok = row < p.M;
#pragma unroll 1
            for (int ch = 0; ch < BN / 32; ++ch) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + ch * 32, r);
                const int col0 = n0 + ch * 32;
                if (!row_ok || col0 >= p.N) continue;
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(__uint_as_float(r[j]), scale);
                if (p.c_bf16) {
                    uint16_t *dst = static_cast<uint16_t *>(p.C) + (int64_t)row * p.ldc + col0;
                    uint32_t w[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[j]) : "f"(v[2 * j + 1]), "f"(v[2 * j]));
                    if (col0 + 32 <= p.N) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            reinterpret_cast<uint4 *>(dst)[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < p.N) dst[j] = (uint16_t)((j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xFFFFu));
                    }
                } else {
                    float *dst = static_cast<float *>(p.C) + (int64_t)row * p.ldc + col0;
                    if (col0 + 32 <= p.N) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            reinterpret_cast<float4 *>(dst)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (col0 + j < p.N) dst[j] = v[j];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
    if (threadIdx.x == 0 && *abort_flag && p.status) atomicExch(p.status, kTimeoutStatus);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D byte view of a codes buffer: [rows x K/2], box = 128 bytes x box_rows, 128B swizzle.
bool make_codes_map(CUtensorMap *map, const uint8_t *codes, int64_t rows, int64_t K, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s, int *launches) {
    const size_t esz = a.c_bf16 ? 2 : 4;
    if (a.M == 0 || a.N == 0) return cudaSuccess;
    if (a.K == 0) {
        ++*launches;
        return cudaMemset2DAsync(a.C, (size_t)a.ldc * esz, 0, (size_t)a.N * esz, (size_t)a.M, s);
    }
    CUtensorMap map_a, map_b;
    if (!make_codes_map(&map_a, a.a_codes, a.M, a.K, BM) || !make_codes_map(&map_b, a.b_codes, a.N, a.K, BN))
        return cudaErrorInvalidValue;
    static bool configured[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    KParams p;
    p.sfa = a.a_scales;
    p.sfb = a.b_scales;
    p.tsa = a.a_ts;
    p.tsb = a.b_ts;
    p.C = a.C;
    p.ldc = a.ldc;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.kb4 = (int)((a.K + 63) / 64);
    p.b_rowtiles = (int)((a.N + 127) / 128);
    p.c_bf16 = a.c_bf16 ? 1 : 0;
    p.status = a.status;
    dim3 grid((unsigned)((a.N + BN - 1) / BN), (unsigned)((a.M + BM - 1) / BM));
    gemm_nvfp4_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(map_a, map_b, p);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace nvfp4
