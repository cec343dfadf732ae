// gemm.cu -- block-scaled NVFP4 (and MXFP4) GEMM on the sm_100a tensor cores.
//
// C[M x N] = (A . B^T) * sA * sB with A [M x K], B [N x K] both K-major NVFP4:
// packed E2M1 codes, one E4M3 scale per 16 k (the 128x4 scale atoms written by
// the quantiser), one FP32 tensor scale each.  4-bit GEMMs on Blackwell
// tensor cores: nerdman.de, "Nvidia drueckt KI-Training auf 4 Bit runter",
// section "Was konkret passiert ist"; format: aisight.pl, section
// "Architektura NVFP4 kontra ograniczenia mikroskalowania" (which also gives
// MXFP4, 32-element blocks with power-of-two scales, as the comparison).
//
// Persistent kernel on CTA pairs (cluster of 2 SMs).  A pair owns a 256 x 256
// output tile at a time: CTA rank r holds A rows [128r, 128r+128) of the tile
// and B rows [128r, 128r+128), and the pair's tensor cores run one
// M=256, N=256, K=64 tcgen05.mma (cta_group::2) per 64-k step, each CTA's
// 128 x 256 FP32 accumulator in its own TMEM.  Warp roles, per CTA:
//   warp 0 (one lane)  producer: TMA loads of this CTA's A and B code tiles
//                      (128-byte swizzle) and scale atoms (A: its 128 rows;
//                      B: all 256 rows) into a 5-stage ring; the code bytes of
//                      both CTAs are counted on the leader's barriers, each
//                      CTA's scale atoms on a barrier of its own;
//   warp 1             allocates TMEM (pair-wide); on the leader one lane issues
//                      the MMAs, four per 256-k stage, reading the stage's
//                      scales from its TMEM slot; tcgen05.commit multicast to
//                      both CTAs frees the stage;
//   warps 11-14        scale writers (both CTAs), one per TMEM lane quarter:
//                      once a stage's scale atoms have landed, each lane loads
//                      its row of every atom from shared memory and writes it
//                      into the stage's TMEM slot with tcgen05.st, in the
//                      layout a tcgen05.cp 32x128b.warpx4 copy of the atom
//                      gives; then the warp arrives on the leader's scale
//                      barrier.  Twelve tcgen05.cp copies per stage from one
//                      warp took ~930 cycles and finished after the code tiles
//                      had landed on most stages; the stores take a fraction
//                      of that and leave the tensor pipe to the MMAs (8192 x
//                      20480 x 5120: 0.356 -> 0.343 ms, interleaved runs);
//   warp 10            waiter (leader): polls the stage's code and scale
//                      barriers and the accumulator-free barrier, and relays
//                      each event to the
//                      MMA warp through a hardware named barrier, so that the
//                      issuing warp never waits on shared memory;
//   warps 2..9         epilogue: two warps per 32-lane TMEM quarter, each
//                      reading 128 accumulator columns (tcgen05.ld), handing
//                      TMEM back to the leader, then scaling by sA*sB and
//                      writing f32 / bf16 through a swizzled 4 KB
//                      shared-memory chunk and a TMA store (32 rows x 128
//                      bytes per chunk; per-row stores from registers cost
//                      several microseconds per tile here).
// TMEM: accumulator columns [0, 256), then one 48-column scale slot per stage.
// Tiles are visited in groups of 8 tile columns so that the pairs running at
// the same time share A and B panels in L2.  Every mbarrier wait is bounded
// (about 2 s of %globaltimer); on expiry the CTA records
// NVFP4_ERR_DEVICE_TIMEOUT in the status word, drains its loads and MMAs,
// frees TMEM and returns.  No TMA load uses cluster multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "checked.cuh"
#include "common.cuh"
#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int BM = 256, BN = 256, BK = 256;   // pair tile; BK in elements (128 bytes of codes)
constexpr int STAGES = 5;
constexpr int A_BYTES = 128 * BK / 2;          // 16 KB: this CTA's 128 A rows
constexpr int B_BYTES = 128 * BK / 2;          // 16 KB: this CTA's 128 B rows
constexpr int SFA_BYTES = (BK / 64) * 512;     // 2 KB: scale atoms of this CTA's A rows
constexpr int SFB_BYTES = 2 * (BK / 64) * 512; // 4 KB: scale atoms of all 256 B rows
constexpr int SF_OFF = A_BYTES + B_BYTES;      // scale atoms inside a stage: A, B rows 0-127, B rows 128-255
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
static_assert(STAGE_BYTES % 1024 == 0, "stages must stay 1024-byte aligned for the 128B swizzle");
constexpr int EPI_WARPS = 8;
constexpr int CHUNK_BYTES = 4096;               // epilogue staging per warp: 32 rows x 128 bytes
constexpr int STAGING_OFF = STAGES * STAGE_BYTES;
constexpr int BAR_OFF = STAGING_OFF + EPI_WARPS * CHUNK_BYTES;
constexpr int BAR_BYTES = 512;
constexpr int SMEM_BYTES = BAR_OFF + BAR_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr int SF_WARPS = 4;                     // scale writers, one per TMEM lane quarter (both CTAs)
constexpr int THREADS = 32 * (11 + SF_WARPS);   // producer, MMA, 8 epilogue warps, waiter, scale writers
constexpr int MMA_WARP = 1, EPI_WARP0 = 2, WAITER_WARP = 10, SF_WARP0 = 11;
// Hardware named barriers (64 threads: the waiter warp and the MMA warp).
constexpr uint32_t NB_ACC = 1;     // accumulator free for the next tile
constexpr uint32_t NB_STAGE0 = 2;  // NB_STAGE0 + s: stage s loaded
constexpr uint32_t NB_EPI = NB_STAGE0 + STAGES;  // the 8 epilogue warps (fused amax reduction)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_SF = 256;              // scale slot of stage s at TMEM_SF + 48 s
constexpr uint32_t SF_SLOT_COLS = 48;          // SFA 4 x 4 columns, then SFB 4 x 8 columns
static_assert(TMEM_SF + STAGES * SF_SLOT_COLS <= TMEM_COLS, "TMEM columns");
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 20000000ull;
constexpr int kTimeoutStatus = 7;              // NVFP4_ERR_DEVICE_TIMEOUT
constexpr int GROUP_N = 8;                     // tile columns per raster group

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1) at bits 7-9 /
// 10-12, K-major, N >> 3 at bits 17-22, UE4M3 scales (bit 23 = 0), M >> 4 at
// bits 24-28 (M = 256 across the pair), scale-factor byte ids 0, dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
// MXFP4 (kind::mxf4, blocks of 32): the same fields with UE8M0 scales (bit 23).
// Each K = 64 step reads two scale bytes per row out of a 4-byte TMEM word; the
// byte they start at (0 or 2) goes in bits 29-30 (A) and 4-5 (B).
constexpr uint32_t IDESC_MX = IDESC | (1u << 23);
__host__ __device__ constexpr uint32_t idesc_mx(uint32_t sf_byte) { return IDESC_MX | (sf_byte << 29) | (sf_byte << 4); }
// Scale atoms (128 rows x 4 bytes) per 256-k stage and 128-row tile: one per 64 k
// for NVFP4 (16-element blocks), one per 128 k for MXFP4 (32-element blocks).
template <bool MX> constexpr int kAtomsPerStage = MX ? 2 : 4;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Arrive on a barrier of the pair (own or peer CTA) with the default semantics
// (release, CTA scope).  It hands TMEM back after tcgen05.wait::ld and
// tcgen05.fence::before_thread_sync: the reads it orders are complete, nothing
// this thread wrote to memory needs to be seen by the waiting CTA, and a
// cluster-scope release here cost ~1800 cycles per tile (~310 with the default).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
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
// The same with cluster-scope acquire, for barriers that CTAs of the pair arrive on.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void named_sync(uint32_t id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }
// Bounded wait, slow path: false once the limit passes or another role of this
// CTA has given up.  Kept out of line so the issue loops stay short.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag, bool honour_abort,
                                            uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (honour_abort && *abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          bool honour_abort = true, uint64_t limit_ns = WAIT_LIMIT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, abort_flag, honour_abort, limit_ns);
}

// Tile load into this CTA's shared memory whose completion bytes are counted
// on the leader's barrier (a shared::cluster address).
__device__ __forceinline__ void tma_load_pair(uint32_t dst, const CUtensorMap *map, uint32_t leader_bar, int x, int y,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(map), "r"(leader_bar), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// The MMA warp runs its loop on all 32 lanes (no divergent branches around the
// issue sequence) and issues each tensor-core instruction from the lanes whose
// `issue` is non-zero -- one lane -- through a PTX predicate.
// Scale atom (32 rows x 16 bytes in smem) -> 32 TMEM lanes x 4 columns, copied to
// all four lane quarters, in both CTAs of the pair (each from its own smem).  The
// tensor-pipe probe below loads its scales this way; the GEMM writes the same
// layout with tcgen05.st.
__device__ __forceinline__ void tc_cp_scales_if(uint32_t issue, uint32_t taddr, uint64_t sdesc) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %0, 0;\n\t"
        "@q tcgen05.cp.cta_group::2.32x128b.warpx4 [%1], %2;\n\t}" ::"r"(issue),
        "r"(taddr), "l"(sdesc)
        : "memory");
}
template <bool MX>
__device__ __forceinline__ void tc_mma_if(uint32_t issue, uint32_t d, uint64_t a, uint64_t b, uint32_t sfa,
                                          uint32_t sfb, uint32_t acc, uint32_t idesc) {
    if (MX)
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "setp.ne.b32 q, %7, 0;\n\t"
            "@q tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb), "r"(issue)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p, q;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "setp.ne.b32 q, %7, 0;\n\t"
            "@q tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
            "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb), "r"(issue)
            : "memory");
}
// Arrives on the barrier at the same offset in both CTAs once every MMA issued so far has completed.
__device__ __forceinline__ void tc_commit_pair_if(uint32_t issue, uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %0, 0;\n\t"
        "@q tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%1], %2;\n\t}" ::"r"(
            issue),
        "r"(bar), "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void tc_commit_self_if(uint32_t issue, uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %0, 0;\n\t"
        "@q tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%1];\n\t}" ::"r"(issue),
        "r"(bar)
        : "memory");
}
// Warp-uniform bounded wait: every lane returns the same answer.
template <bool CLUSTER>
__device__ __forceinline__ bool try_wait_scoped(uint32_t bar, uint32_t parity) {
    return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
}
template <bool CLUSTER>
__device__ __noinline__ bool mbar_wait_warp_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                 bool honour_abort, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (__all_sync(0xFFFFFFFFu, try_wait_scoped<CLUSTER>(bar, parity))) return true;
        const bool aborted = __any_sync(0xFFFFFFFFu, honour_abort && *abort_flag);
        if (aborted) return false;
        if (__any_sync(0xFFFFFFFFu, globaltimer() - t0 > limit_ns)) {
            *abort_flag = 1;
            return false;
        }
    }
}
template <bool CLUSTER = false>
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                               bool honour_abort = true, uint64_t limit_ns = WAIT_LIMIT_NS) {
    if (__all_sync(0xFFFFFFFFu, try_wait_scoped<CLUSTER>(bar, parity))) return true;
    return mbar_wait_warp_slow<CLUSTER>(bar, parity, abort_flag, honour_abort, limit_ns);
}
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 16 / 32 consecutive TMEM columns of this warp's lane quarter from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *w) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
        "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *w) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]), "r"(w[9]),
        "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15]), "r"(w[16]), "r"(w[17]), "r"(w[18]),
        "r"(w[19]), "r"(w[20]), "r"(w[21]), "r"(w[22]), "r"(w[23]), "r"(w[24]), "r"(w[25]), "r"(w[26]), "r"(w[27]),
        "r"(w[28]), "r"(w[29]), "r"(w[30]), "r"(w[31])
        : "memory");
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

// TMA load into this CTA's shared memory, completing on this CTA's own barrier.
__device__ __forceinline__ void tma_load_own(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y,
                                             uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(map), "r"(bar), "r"(x), "r"(y), "l"(policy)
        : "memory");
}
// TMA store of a shared-memory box (bulk async-group completion).
__device__ __forceinline__ void tma_store(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map), "r"(src),
                 "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the TMA engine.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
// Byte offset of 16-byte unit u of row r in a 32-row x 128-byte chunk laid out
// with the TMA 128-byte swizzle (unit index xor row % 8): a warp's 16-byte
// accesses of one unit index cover all banks.
__device__ __forceinline__ uint32_t chunk_off(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

struct KParams {
    const float *tsa, *tsb;
    int M, N, K;
    int kbs;    // scale atoms per 128-row tile (K / 64 for NVFP4, ceil(K / 128) for MXFP4)
    int kfull;  // full 256-k stages (= K / 256)
    int ktail;  // 64-k steps in a last, partial stage (= (K % 256) / 64)
    int c_bf16;
    int tiles_m, tiles_n, num_tiles;
    int *status;
    int epi;          // GEMM_EPI_* (internal.h)
    uint64_t seed;    // Hadamard signs of the fused amax
    float *partials;  // per CTA: max |out| at [cta], max |RHT(out)| at [kMaxPartials + cta]
};

// Tile t -> (tile row, tile column).  Tile columns form bands of GROUP_N; inside
// a band, consecutive t walk along a tile row, then down to the next tile row.
__device__ __forceinline__ void tile_coords(const KParams &p, int t, int &mt, int &nt) {
    const int per_group = p.tiles_m * GROUP_N;
    const int g = t / per_group, r = t - g * per_group;
    const int gw = min(GROUP_N, p.tiles_n - g * GROUP_N);
    mt = r / gw;
    nt = g * GROUP_N + (r - mt * gw);
}

// One epilogue chunk (32 rows x 128 bytes, row = lane) from registers into the
// warp's staging buffer and out through a TMA store.  The previous store of
// this warp must have finished reading the buffer first.
__device__ __forceinline__ void store_chunk(const CUtensorMap *map, uint32_t stg, const uint32_t (&w)[32], int lane,
                                            int x, int y, bool write) {
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 8; ++u) st_shared_v4(stg + chunk_off(lane, u), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    fence_proxy_async();
    __syncwarp();
    if (lane == 0 && write) {
        tma_store(map, stg, x, y);
        bulk_commit();
    }
}

// Running max |v| and max |H16 D v| of one bf16 pair per lane, the transform
// down the 16-row groups held by lanes 0-15 and 16-31 (lower lane a + b, upper
// lane a - b, strides 1, 2, 4, 8): the fused relu^2 epilogue's two amaxes.
__device__ __forceinline__ void amax_pair_rht(uint32_t o, uint32_t row_sign, int lane, float &m0, float &m1) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        float v = k ? bf16hi(o) : bf16lo(o);
        m0 = fmaxf(m0, fabsf(v));
        v = __uint_as_float(__float_as_uint(v) ^ row_sign);
#pragma unroll
        for (int hs = 1; hs < 16; hs <<= 1) {
            const float pv = __shfl_xor_sync(0xFFFFFFFFu, v, hs);
            v = (lane & hs) ? __fsub_rn(pv, v) : __fadd_rn(v, pv);
        }
        m1 = fmaxf(m1, fabsf(v));
    }
}

template <bool MX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                      const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_aux,
                      const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + BAR_OFF);
    const uint32_t bar_full = smem_u32(bars);                    // [S] leader: both CTAs' bytes of a stage
    const uint32_t bar_empty = smem_u32(bars + STAGES);          // [S] each CTA: MMAs reading the stage done
    const uint32_t bar_accf = smem_u32(bars + 2 * STAGES);       // each CTA: accumulator complete
    const uint32_t bar_acce = smem_u32(bars + 2 * STAGES + 1);   // leader: accumulator read (16 epilogue warps)
    const uint32_t bar_drain = smem_u32(bars + 2 * STAGES + 2);  // leader: every MMA done
    const uint32_t bar_epi = smem_u32(bars + 2 * STAGES + 3);    // [8] each CTA: an epilogue warp's aux chunk
    const uint32_t bar_sf = smem_u32(bars + 2 * STAGES + 3 + EPI_WARPS);       // [S] leader: stage's scales in TMEM
    const uint32_t bar_sfull = smem_u32(bars + 3 * STAGES + 3 + EPI_WARPS);    // [S] each CTA: its scale bytes
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * STAGES + 3 + EPI_WARPS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *stop_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);  // waiter -> MMA warp, per tile
    float *red = reinterpret_cast<float *>(tmem_slot + 4);                      // fused amax: 2 x 8 warps

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const int cid = (int)cluster_id_x(), ncl = (int)nclusters_x();
    constexpr int APS = kAtomsPerStage<MX>;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
            mbar_init(bar_sf + 8 * s, 2 * SF_WARPS);  // the scale writers of both CTAs
            mbar_init(bar_sfull + 8 * s, 1);
        }
        mbar_init(bar_accf, 1);
        mbar_init(bar_acce, 2 * EPI_WARPS);
        mbar_init(bar_drain, 1);
        for (int w = 0; w < EPI_WARPS; ++w) mbar_init(bar_epi + 8 * w, 1);
        *abort_flag = 0;
        *stop_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == MMA_WARP) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t smem_base = smem_u32(smem);
    const int num_kt = p.kfull + (p.ktail ? 1 : 0);
    float epi_m0 = 0.0f, epi_m1 = 0.0f;  // epilogue, fused relu^2: max |out|, max |H16 D out| (unscaled)

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer (both CTAs) ----------------
            uint64_t policy;
            asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(policy));
            uint32_t s = 0, ph = 0;
            bool ok = true;
            // Bytes per CTA per stage: the scale atoms complete on a barrier of this CTA,
            // so that its scale writers can move them into TMEM while the codes still land.
            constexpr uint32_t CODES_TX = A_BYTES + B_BYTES, SCALES_TX = 3 * APS * 512;
            for (int t = cid; t < p.num_tiles && ok; t += ncl) {
                int mt, nt;
                tile_coords(p, t, mt, nt);
                const int m0 = mt * BM + 128 * (int)rank, n0 = nt * BN;
                const int ya = (m0 / 128) * p.kbs, yb = (n0 / 128) * p.kbs;
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (!mbar_wait(bar_empty + 8 * s, ph ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = smem_base + s * STAGE_BYTES;
                    const uint32_t full_leader = mapa(bar_full + 8 * s, 0);
                    // Out-of-range rows, columns and atoms are zero-filled and still
                    // counted, so every stage brings exactly CODES_TX + SCALES_TX bytes
                    // per CTA.
                    mbar_expect_tx(bar_sfull + 8 * s, SCALES_TX);
                    if (rank == 0) mbar_expect_tx(bar_full + 8 * s, 2 * CODES_TX);
                    tma_load_own(st + SF_OFF, &map_sfa, bar_sfull + 8 * s, 0, ya + kt * APS, policy);
                    tma_load_own(st + SF_OFF + SFA_BYTES, &map_sfb, bar_sfull + 8 * s, 0, yb + kt * APS, policy);
                    tma_load_own(st + SF_OFF + SFA_BYTES + 2048, &map_sfb, bar_sfull + 8 * s, 0,
                                 yb + p.kbs + kt * APS, policy);
                    tma_load_pair(st, &map_a, full_leader, kt * (BK / 2), m0, policy);
                    tma_load_pair(st + A_BYTES, &map_b, full_leader, kt * (BK / 2), n0 + 128 * (int)rank, policy);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // This CTA's code tiles complete on the leader's barriers, and the leader drains
            // them; its scale atoms on its own, which its scale writers drain.
        }
    } else if (warp == MMA_WARP) {
        if (rank == 0) {
            // ---------------- MMA issuer (leader's warp 1, lane 0 issues) ----------------
            const uint32_t issue = lane == 0 ? 1u : 0u;
            const int kfull = p.kfull, ktail = p.ktail;
            uint32_t s = 0, ph = 0;
            int consumed = 0;
            // Every event this warp waits for comes from the waiter warp through a
            // named barrier: the loop below reads no shared memory per stage.
            for (int t = cid; t < p.num_tiles; t += ncl) {
                named_sync(NB_ACC);
                if (*stop_flag) break;  // written by the waiter before the barrier
                tc_fence_after();
                uint32_t acc = 0;  // the first MMA of a tile overwrites the accumulator
                for (int kt = 0; kt < num_kt; ++kt) {
                    // Stage s has landed and its scales are in TMEM slot s (the waiter saw
                    // the scale writers' barrier complete).
                    named_sync(NB_STAGE0 + s);
                    tc_fence_after();
                    const uint32_t sa = smem_base + s * STAGE_BYTES;
                    const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sa + A_BYTES);
                    const uint32_t sf = tmem + TMEM_SF + SF_SLOT_COLS * s;
                    // Descriptor addresses are in 16-byte units: +2 per 64-k step of codes.
                    // Scales: A atom j at sf + 4 j, B atoms at sf + 16 + 8 j (rows 0-127)
                    // and sf + 20 + 8 j (rows 128-255); MXFP4 atom j serves steps 2j, 2j+1.
                    const int steps = kt < kfull ? 4 : ktail;
                    if (steps == 4) {
                        if (lane == 0) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                if (MX)
                                    tc_mma_if<MX>(1u, tmem, da + 2 * j, db + 2 * j, sf + 4 * (j >> 1),
                                                  sf + 16 + 8 * (j >> 1), (acc | (uint32_t)j) ? 1u : 0u,
                                                  idesc_mx(2u * (uint32_t)(j & 1)));
                                else
                                    tc_mma_if<MX>(1u, tmem, da + 2 * j, db + 2 * j, sf + 4 * j, sf + 16 + 8 * j,
                                                  (acc | (uint32_t)j) ? 1u : 0u, IDESC);
                            }
                        }
                        __syncwarp();
                    } else {
                        for (int j = 0; j < steps; ++j) {
                            if (MX)
                                tc_mma_if<MX>(issue, tmem, da + 2 * j, db + 2 * j, sf + 4 * (j >> 1),
                                              sf + 16 + 8 * (j >> 1), (acc | (uint32_t)j) ? 1u : 0u,
                                              idesc_mx(2u * (uint32_t)(j & 1)));
                            else
                                tc_mma_if<MX>(issue, tmem, da + 2 * j, db + 2 * j, sf + 4 * j, sf + 16 + 8 * j,
                                              (acc | (uint32_t)j) ? 1u : 0u, IDESC);
                        }
                    }
                    acc = 1;
                    tc_commit_pair_if(issue, bar_empty + 8 * s);
                    ++consumed;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                tc_commit_pair_if(issue, bar_accf);
            }
            tc_commit_self_if(issue, bar_drain);
            mbar_wait_warp(bar_drain, 0, abort_flag, false);
            if (*abort_flag) {
                // Stages the producers may still be filling: wait (briefly) for their bytes.
                for (int k = consumed; k < consumed + STAGES; ++k) {
                    mbar_wait_warp(bar_full + 8 * (k % STAGES), (k / STAGES) & 1, abort_flag, false, DRAIN_LIMIT_NS);
                    mbar_wait_warp(bar_sfull + 8 * (k % STAGES), (k / STAGES) & 1, abort_flag, false,
                                   DRAIN_LIMIT_NS);
                }
            }
        }
    } else if (warp == WAITER_WARP) {
        if (rank == 0) {
            // ---------------- waiter (leader only) ----------------
            // Waits on the accumulator-free barrier and, per stage, on its code bytes
            // and on its scale barrier (the scale writers of both CTAs arrive once the
            // stage's scale atoms are in TMEM) in the order the MMA warp consumes them, and relays
            // each through a named barrier.  After
            // a timeout inside a tile it keeps relaying without waiting until the
            // tile ends, then both warps stop.
            // Both warps take the same named barriers in the same order (bar.sync on
            // both sides: neither can run ahead), and leave the tile loop together:
            // the stop decision is written before the per-tile barrier and read by
            // the MMA warp after it.
            uint32_t s = 0, ph = 0;
            int tile_i = 0;
            bool ok = true;
            for (int t = cid; t < p.num_tiles; t += ncl, ++tile_i) {
                if (ok) ok = mbar_wait_warp<true>(bar_acce, (tile_i & 1) ^ 1, abort_flag);
                const bool stop = !ok || *abort_flag;
                if (lane == 0) *stop_flag = stop ? 1 : 0;
                named_sync(NB_ACC);
                if (stop) break;
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (ok) ok = mbar_wait_warp(bar_full + 8 * s, ph, abort_flag);
                    if (ok) ok = mbar_wait_warp<true>(bar_sf + 8 * s, ph, abort_flag);  // writers of both CTAs
                    named_sync(NB_STAGE0 + s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
        }
    } else if (warp >= SF_WARP0 && warp < SF_WARP0 + SF_WARPS) {
        // ---------------- scale writers (both CTAs, warps 11-14) ----------------
        // Warp w writes TMEM lane quarter w % 4 of its CTA.  Once stage s's scale atoms
        // have landed in this CTA (bar_sfull, usually well before the code tiles), lane
        // r loads row r of every atom (16 bytes: the 4-byte words of rows r, r + 32,
        // r + 64, r + 96) and stores it into 4 columns of lane 32 q + r of the stage's
        // TMEM slot -- the layout a 32x128b.warpx4 copy of the atom produces, which the
        // MMA reads -- then arrives on the leader's bar_sf[s] (8 arrivals: four warps in
        // each CTA).  A whole slot is written every stage (MXFP4 stages, and the short
        // last stage, leave some of it unread).  The slot is free: the producer reloads
        // stage s only after the MMAs that read the slot have completed.  These stores
        // do not queue on the tensor pipe as tcgen05.cp copies do (~930 cycles per stage
        // from one warp, on the refill path of every stage).
        const uint32_t q = warp & 3;
        uint32_t s = 0, ph = 0;
        bool ok = true;
        int it = 0;
        for (int t = cid; t < p.num_tiles && ok; t += ncl) {
            for (int kt = 0; kt < num_kt; ++kt, ++it) {
                if (!mbar_wait_warp(bar_sfull + 8 * s, ph, abort_flag)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = smem_base + s * STAGE_BYTES + SF_OFF + (uint32_t)lane * 16u;
                uint32_t w[48];
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // SFA atom j -> columns 4 j .. 4 j + 3
                    const uint4 v = ld_shared_v4(sa + 512u * j);
                    w[4 * j] = v.x, w[4 * j + 1] = v.y, w[4 * j + 2] = v.z, w[4 * j + 3] = v.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // SFB atom j: rows 0-127 -> 16 + 8 j, rows 128-255 -> 20 + 8 j
                    const uint4 lo = ld_shared_v4(sa + SFA_BYTES + 512u * j);
                    const uint4 hi = ld_shared_v4(sa + SFA_BYTES + 2048u + 512u * j);
                    w[16 + 8 * j] = lo.x, w[17 + 8 * j] = lo.y, w[18 + 8 * j] = lo.z, w[19 + 8 * j] = lo.w;
                    w[20 + 8 * j] = hi.x, w[21 + 8 * j] = hi.y, w[22 + 8 * j] = hi.z, w[23 + 8 * j] = hi.w;
                }
                const uint32_t ta = tmem + ((q * 32u) << 16) + TMEM_SF + SF_SLOT_COLS * s;
                tmem_st16(ta, w);
                tmem_st32(ta + 16, w + 16);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(mapa(bar_sf + 8 * s, 0));
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1;
                }
            }
        }
        if (!ok && warp == SF_WARP0) {
            // Stages this CTA's producer may still be filling: wait (briefly) for their atoms.
            for (int k = it; k < it + STAGES; ++k)
                mbar_wait_warp(bar_sfull + 8 * (k % STAGES), (k / STAGES) & 1, abort_flag, false, DRAIN_LIMIT_NS);
        }
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // ---------------- epilogue (both CTAs) ----------------
        // Warp w reads TMEM lane quarter w % 4 (the quarter a warp may access) and
        // columns [128 h, 128 h + 128) of the accumulator, h = (w - 2) / 4; row
        // 32 (w % 4) + lane of this CTA's 128 is the thread's.
        const int ew = warp - EPI_WARP0;
        const uint32_t q = warp & 3;
        const int hh = ew >> 2;
        const uint32_t tbase = tmem + ((q * 32u) << 16) + 128u * (uint32_t)hh;
        const uint32_t stg = smem_base + STAGING_OFF + (uint32_t)ew * CHUNK_BYTES;
        const uint32_t ep_bar = bar_epi + 8 * ew;
        uint32_t ep_phase = 0;
        uint64_t policy;
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
        const float scale = MX ? 1.0f : __fmul_rn(*p.tsa, *p.tsb);  // MXFP4 has no tensor scale
        const uint32_t row_sign = p.epi != GEMM_EPI_PLAIN ? ((rht_sign_bits(p.seed) >> (lane & 15)) & 1u) << 31 : 0u;
        int tile_i = 0;
        for (int t = cid; t < p.num_tiles; t += ncl, ++tile_i) {
            // the tile's coordinates before the wait: off the accumulator hand-off path
            int mt, nt;
            tile_coords(p, t, mt, nt);
            const int row0 = mt * BM + 128 * (int)rank + (int)q * 32;  // this warp's 32 rows
            const int col0 = nt * BN + 128 * hh;                        // and 128 columns
            const bool rows_in = row0 < p.M;
            bool ok = mbar_wait(bar_accf, tile_i & 1, abort_flag);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            tc_fence_after();
            if (p.c_bf16) {
                // All 128 accumulator columns into registers, TMEM handed back, then
                // scaled and packed to bf16, each 64-column chunk out through the
                // staging buffer.
                uint32_t w[2][32];
                {
                    uint32_t r[4][32];
#pragma unroll
                    for (int k = 0; k < 4; ++k) tmem_ld32_nowait(tbase + 32 * k, r[k]);
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(mapa(bar_acce, 0));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            w[k >> 1][16 * (k & 1) + j] = pack_bf16x2(__fmul_rn(__uint_as_float(r[k][2 * j]), scale),
                                                                      __fmul_rn(__uint_as_float(r[k][2 * j + 1]), scale));
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int x = col0 + 64 * c;
                    const bool in = rows_in && x < p.N;
                    if (p.epi == GEMM_EPI_PLAIN) {
                        store_chunk(&map_c, stg, w[c], lane, x, row0, in);
                    } else if (p.epi == GEMM_EPI_RELU2_FWD) {
                        // y, then h = relu(y)^2 with its two amaxes
                        store_chunk(&map_c, stg, w[c], lane, x, row0, in);
                        uint32_t o[32];
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            o[k] = relu2_pair(w[c][k]);
                            amax_pair_rht(o[k], row_sign, lane, epi_m0, epi_m1);
                        }
                        store_chunk(&map_aux, stg, o, lane, x, row0, in);
                    } else {
                        // dY = dh * 2 relu(Y): the forward's Y chunk comes in through the
                        // staging buffer (TMA load), dY leaves through it
                        if (lane == 0) {
                            bulk_wait_read_all();
                            mbar_expect_tx(ep_bar, CHUNK_BYTES);
                            tma_load_own(stg, &map_aux, ep_bar, x, row0, policy);
                        }
                        const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(ep_bar, ep_phase, abort_flag));
                        ep_phase ^= 1;
                        uint32_t o[32];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const uint4 y = ld_shared_v4(stg + chunk_off(lane, u));
                            o[4 * u] = drelu2_pair(w[c][4 * u], y.x);
                            o[4 * u + 1] = drelu2_pair(w[c][4 * u + 1], y.y);
                            o[4 * u + 2] = drelu2_pair(w[c][4 * u + 2], y.z);
                            o[4 * u + 3] = drelu2_pair(w[c][4 * u + 3], y.w);
                        }
#pragma unroll
                        for (int k = 0; k < 32; ++k) amax_pair_rht(o[k], row_sign, lane, epi_m0, epi_m1);
                        store_chunk(&map_c, stg, o, lane, x, row0, in && got);
                    }
                }
            } else {
                // f32: four 32-column chunks, read two at a time; TMEM handed back once
                // the second pair is in registers
#pragma unroll 1
                for (int c = 0; c < 4; c += 2) {
                    uint32_t r[2][32];
                    tmem_ld32_nowait(tbase + 32 * c, r[0]);
                    tmem_ld32_nowait(tbase + 32 * (c + 1), r[1]);
                    tmem_wait_ld();
                    if (c == 2) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_remote(mapa(bar_acce, 0));
                    }
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            r[u][j] = __float_as_uint(__fmul_rn(__uint_as_float(r[u][j]), scale));
                        const int x = col0 + 32 * (c + u);
                        store_chunk(&map_c, stg, r[u], lane, x, row0, rows_in && x < p.N);
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();  // every store of this warp complete before the CTA exits
    }

    if (p.epi != GEMM_EPI_PLAIN && warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // this CTA's partials of the fused amax: warps, then the 8 epilogue warps
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            epi_m0 = fmaxf(epi_m0, __shfl_xor_sync(0xFFFFFFFFu, epi_m0, o));
            epi_m1 = fmaxf(epi_m1, __shfl_xor_sync(0xFFFFFFFFu, epi_m1, o));
        }
        if (lane == 0) {
            red[warp - EPI_WARP0] = epi_m0;
            red[EPI_WARPS + warp - EPI_WARP0] = epi_m1;
        }
        asm volatile("bar.sync %0, %1;" ::"r"(NB_EPI), "r"(32 * EPI_WARPS) : "memory");
        if (warp == EPI_WARP0 && lane == 0) {
            float a = 0.0f, b = 0.0f;
            for (int i = 0; i < EPI_WARPS; ++i) {
                a = fmaxf(a, red[i]);
                b = fmaxf(b, red[EPI_WARPS + i]);
            }
            if (NVFP4_IN_RANGE(blockIdx.x, 1, kMaxPartials)) {
                p.partials[blockIdx.x] = a;
                p.partials[kMaxPartials + blockIdx.x] = __fmul_rn(b, 0.25f);  // max |z / 4| = RN(max |z| / 4)
            }
        }
    }

    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == MMA_WARP) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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

// 2-D byte view of a codes buffer: [rows x K/2], box = 128 bytes x 128 rows, 128B swizzle.
bool make_codes_map(CUtensorMap *map, const uint8_t *codes, int64_t rows, int64_t K) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, 128u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A scale buffer as rows of one 512-byte atom (128 words): [atoms x 128] words,
// box = the atoms of one 256-k stage of one 128-row tile (4 NVFP4, 2 MXFP4).
bool make_scale_map(CUtensorMap *map, const uint8_t *scales, int64_t rows, int64_t kbs, int box_atoms) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int64_t atoms = ((rows + 127) / 128) * kbs;
    cuuint64_t dims[2] = {128u, (cuuint64_t)atoms};
    cuuint64_t strides[1] = {512u};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_atoms};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t *>(scales), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major [rows x cols] output (or the fused epilogue's bf16 companion)
// with leading dimension ld elements: box = 128 bytes x 32 rows, 128B swizzle
// (the epilogue's staging chunk).
bool make_out_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld, bool bf16) {
    auto fn = encode_fn();
    if (!fn) return false;
    const uint32_t esz = bf16 ? 2u : 4u;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * esz};
    cuuint32_t box[2] = {128u / esz, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool MX>
cudaError_t launch_gemm_t(const GemmArgs &a, cudaStream_t s, int *launches) {
    const int kbs = MX ? (int)((a.K + 127) / 128) : (int)(a.K / 64);
    CUtensorMap map_a, map_b, map_sfa, map_sfb, map_c, map_aux;
    if (!make_codes_map(&map_a, a.a_codes, a.M, a.K) || !make_codes_map(&map_b, a.b_codes, a.N, a.K) ||
        !make_scale_map(&map_sfa, a.a_scales, a.M, kbs, kAtomsPerStage<MX>) ||
        !make_scale_map(&map_sfb, a.b_scales, a.N, kbs, kAtomsPerStage<MX>) ||
        !make_out_map(&map_c, a.C, a.M, a.N, a.ldc, a.c_bf16))
        return cudaErrorInvalidValue;
    if (a.epi != GEMM_EPI_PLAIN) {
        if (!make_out_map(&map_aux, a.aux, a.M, a.N, a.ldc, true)) return cudaErrorInvalidValue;
    } else {
        map_aux = map_c;  // unused
    }
    constexpr int kMaxDev = 64;
    static int max_clusters[kMaxDev] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    if (!max_clusters[dev]) {
        e = cudaFuncSetAttribute(gemm_nvfp4_kernel<MX>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        // Pairs that can be resident at once (one CTA per SM).
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)(num_sms() / 2));
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_kernel<MX>, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = num_sms() / 2;
        }
        max_clusters[dev] = n;
    }
    KParams p;
    p.tsa = a.a_ts;
    p.tsb = a.b_ts;
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.kbs = kbs;
    p.kfull = (int)(a.K / BK);
    p.ktail = (int)((a.K % BK) / 64);
    p.c_bf16 = a.c_bf16 ? 1 : 0;
    p.tiles_m = (int)((a.M + BM - 1) / BM);
    p.tiles_n = (int)((a.N + BN - 1) / BN);
    p.num_tiles = p.tiles_m * p.tiles_n;
    p.status = a.status;
    p.epi = a.epi;
    p.seed = a.seed;
    p.partials = a.partials;
    const int pairs = std::min(p.num_tiles, max_clusters[dev]);
    gemm_nvfp4_kernel<MX><<<2 * pairs, THREADS, SMEM_BYTES, s>>>(map_a, map_b, map_sfa, map_sfb, map_c, map_aux, p);
    ++*launches;
    if (a.epi != GEMM_EPI_PLAIN) {
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_amax_reduce2(a.partials, 2 * pairs, a.amax_out, a.amax_rht_out, s, launches);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Tensor-pipe rate probe (measurement only).  Every CTA pair issues `iters`
// rounds of the GEMM's stage -- four M256 N256 K64 block-scaled MMAs with the
// same descriptors -- on one stage of operands resident in shared memory (a
// fixed byte pattern: every byte is a valid pair of E2M1 codes) and scales
// resident in TMEM (all 1.0), with a commit per round as the GEMM has.  The
// issuing thread records the %clock64 cycles from its first MMA to the
// completion of the last.  Shared memory is sized so that one CTA fits per SM.
// ---------------------------------------------------------------------------
constexpr int PROBE_THREADS = 128;
constexpr int PROBE_SMEM = 120 * 1024;  // > half an SM's shared memory: one CTA per SM
static_assert(STAGE_BYTES + 64 + 1024 <= PROBE_SMEM, "probe shared memory");

template <bool MX>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PROBE_THREADS, 1)
    mma_rate_kernel(uint64_t *cycles, int64_t iters, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t *words = reinterpret_cast<uint32_t *>(smem);
    for (int i = threadIdx.x; i < SF_OFF / 4; i += PROBE_THREADS) words[i] = (uint32_t)i * 2654435761u;
    for (int i = threadIdx.x; i < (SFA_BYTES + SFB_BYTES) / 4; i += PROBE_THREADS)
        words[SF_OFF / 4 + i] = MX ? 0x7F7F7F7Fu : 0x38383838u;  // E8M0 / E4M3 encodings of 1.0
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGE_BYTES);
    const uint32_t bar_round = smem_u32(bars), bar_drain = smem_u32(bars + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 3);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    if (threadIdx.x == 0) {
        mbar_init(bar_round, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_proxy_async();  // the operand bytes, written by threads, are read by the tensor cores
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (rank == 0 && warp == 0) {
        const uint32_t issue = lane == 0 ? 1u : 0u;
        const uint32_t sa = smem_u32(smem);
        const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sa + A_BYTES);
        const uint64_t dsa = sdesc_scales(sa + SF_OFF), dsb = sdesc_scales(sa + SF_OFF + SFA_BYTES);
        const uint32_t sf = tmem + TMEM_SF;
        for (int j = 0; j < kAtomsPerStage<MX>; ++j) {  // the MMAs below follow these copies in issue order
            tc_cp_scales_if(issue, sf + 4 * j, dsa + 32 * j);
            tc_cp_scales_if(issue, sf + 16 + 8 * j, dsb + 32 * j);
            tc_cp_scales_if(issue, sf + 20 + 8 * j, dsb + 128 + 32 * j);
        }
        const uint64_t t0 = clock64();
        for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t acc = (it > 0 || j > 0) ? 1u : 0u;
                if (MX)
                    tc_mma_if<MX>(issue, tmem, da + 2 * j, db + 2 * j, sf + 4 * (j >> 1), sf + 16 + 8 * (j >> 1), acc,
                                  idesc_mx(2u * (uint32_t)(j & 1)));
                else
                    tc_mma_if<MX>(issue, tmem, da + 2 * j, db + 2 * j, sf + 4 * j, sf + 16 + 8 * j, acc, IDESC);
            }
            tc_commit_self_if(issue, bar_round);
            __syncwarp();
        }
        tc_commit_self_if(issue, bar_drain);
        const bool ok = mbar_wait_warp(bar_drain, 0, abort_flag, false);
        const uint64_t t1 = clock64();
        if (lane == 0) {
            cycles[cluster_id_x()] = t1 - t0;
            if (!ok) atomicExch(status, kTimeoutStatus);
        }
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
}

template <bool MX>
cudaError_t launch_mma_rate_t(int64_t iters, uint64_t *cycles, int64_t cycles_len, int *pairs_out, int *status,
                              cudaStream_t s, int *launches) {
    cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel<MX>, cudaFuncAttributeMaxDynamicSharedMemorySize, PROBE_SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(num_sms() / 2));
    cfg.blockDim = dim3(PROBE_THREADS);
    cfg.dynamicSmemBytes = PROBE_SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, mma_rate_kernel<MX>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms() / 2;
    }
    if (n > cycles_len) return cudaErrorInvalidValue;
    *pairs_out = n;
    mma_rate_kernel<MX><<<2 * n, PROBE_THREADS, PROBE_SMEM, s>>>(cycles, iters, status);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs &a, cudaStream_t s, int *launches) {
    const size_t esz = a.c_bf16 ? 2 : 4;
    if (a.M == 0 || a.N == 0) return cudaSuccess;
    if (a.K == 0) {
        ++*launches;
        return cudaMemset2DAsync(a.C, (size_t)a.ldc * esz, 0, (size_t)a.N * esz, (size_t)a.M, s);
    }
    return a.mx ? launch_gemm_t<true>(a, s, launches) : launch_gemm_t<false>(a, s, launches);
}

cudaError_t launch_mma_rate(bool mx, int64_t iters, uint64_t *cycles, int64_t cycles_len, int *pairs_out, int *status,
                            cudaStream_t s, int *launches) {
    return mx ? launch_mma_rate_t<true>(iters, cycles, cycles_len, pairs_out, status, s, launches)
              : launch_mma_rate_t<false>(iters, cycles, cycles_len, pairs_out, status, s, launches);
}

NVFP4_DEFINE_BOUNDS_READER(read_bounds_gemm)

}  // namespace nvfp4
