// Thin inline-PTX wrappers for the sm_100a features the kernels use: mbarriers, TMA
// (tiled and im2col loads, tiled stores) and tcgen05 (TMEM allocation, MMA, commit, loads);
// every mbarrier wait is bounded by the SM cycle counter.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace convb200 {

// Device status word bits (one per failure kind). Written with atomicOr, read by the host.
enum : unsigned { kStatusTimeout = 1u, kStatusBounds = 2u };

// ---- bounds-checked debug build ---------------------------------------------------------
// Compiled with -DCONV_DEBUG_BOUNDS, every plain global load or store whose address the kernels
// compute (and every 1-D bulk copy, which no tensor map bounds) is first checked against the
// extent of its tensor: elements [idx, idx + len) of a tensor of `limit` elements. A failed check
// sets kStatusBounds in the status word, records the first failure (site, index, limit) and
// returns false: the caller skips the access -- no assertion, no trap, the context stays usable.
// Tensor-map (TMA) copies need no check: the hardware bounds them. In the normal build the
// check is the constant true and costs nothing.
enum BoundsSite : unsigned {
    kSiteDirectX = 1, kSiteDirectY, kSiteFoldY, kSiteHaloY, kSiteStreamY, kSiteTcBias, kSiteDwY, kSiteDwRegX,
    kSiteDwRegY, kSiteDwTmaY, kSiteDwPlaneX, kSiteDwPlaneY, kSiteDwPwX, kSiteDwPwY, kSiteDwPwGemmX,
    kSiteDwPwGemmW, kSiteDwPwGemmY, kSiteIm2colX, kSiteIm2colA, kSiteDwTmaX, kSiteDwX, kSiteHaloPadBias, kSiteHaloPadY,
    kSiteSelftest = 255
};
#ifdef CONV_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
// [0] claimed flag, [1] site, [2] index, [3] limit of the first failed check
__device__ long long g_bounds_first[4];
__device__ __noinline__ void bounds_record(unsigned site, long long idx, long long limit, unsigned *status) {
    atomicOr(status, kStatusBounds);
    if (atomicCAS(reinterpret_cast<unsigned long long *>(&g_bounds_first[0]), 0ull, 1ull) == 0ull) {
        g_bounds_first[1] = site;
        g_bounds_first[2] = idx;
        g_bounds_first[3] = limit;
    }
}
__device__ __forceinline__ bool in_bounds(long long idx, long long len, long long limit, unsigned site,
                                          unsigned *status) {
    if (idx >= 0 && len >= 0 && idx + len <= limit) return true;
    bounds_record(site, idx, limit, status);
    return false;
}
#else
constexpr bool kDebugBounds = false;
__device__ __forceinline__ bool in_bounds(long long, long long, long long, unsigned, unsigned *) { return true; }
#endif

// Every spin on an mbarrier gives up after this many SM clock cycles (about one second at
// the B200's 1.9-2.0 GHz; longer at lower clocks). The SM-local cycle counter is cheap to read,
// unlike %globaltimer, so the check costs nothing on the fast path.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------
// Programmatic dependent launch
// ---------------------------------------------------------------------------------------
// Every kernel of the library is launched with programmatic stream serialisation allowed: the
// next kernel on the stream may be scheduled while this one finishes. A kernel lets its
// dependents launch as soon as it starts (grid_dependents_launch) and, before its first
// global-memory access, waits until every kernel it depends on has completed and its memory
// operations are visible (grid_dependency_wait) -- so a chain of dependent convolutions keeps
// stream order, and only launch latency and the on-chip prologue (barrier set-up, TMEM
// allocation, tensor-map prefetch) overlap the previous kernel's tail. Both are no-ops for a
// kernel launched without the attribute.
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Completes `bytes` of the barrier's expected transaction count without a copy (a copy that a
// bounds check skipped).
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// One poll of the phase with the given parity (no suspend-time hint: measured on B200, a
// hinted wait resumes late and slows the pipelines several-fold).
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

// Waits for the phase with the given parity to complete. Returns false if the wait ran
// past kWaitLimitCycles; the caller then records the timeout and stops.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
}

// Wait for a role that is not on the critical path (producer, epilogue): between polls the
// warp sleeps for about sleep_ns, so it does not compete with the MMA warp and the tensor
// cores for issue slots and the shared-memory pipe.
__device__ __forceinline__ bool mbar_wait_backoff(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        __nanosleep(sleep_ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
}

__device__ __forceinline__ bool mbar_wait_warp_backoff(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
    uint32_t ready = 0;
    if ((threadIdx.x & 31) == 0) ready = mbar_try_wait(bar, parity) ? 1u : 0u;
    if (__shfl_sync(0xffffffffu, ready, 0)) return true;
    return __all_sync(0xffffffffu, mbar_wait_backoff(bar, parity, sleep_ns));
}

// Whole-warp wait. Fast path: one poll by lane 0 (32 lanes polling one barrier serialise,
// about 15 cycles each). Slow path: every lane polls (measured faster on B200 than one polling
// lane with the others parked). True only if every lane saw the phase complete.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity) {
    uint32_t ready = 0;
    if ((threadIdx.x & 31) == 0) ready = mbar_try_wait(bar, parity) ? 1u : 0u;
    if (__shfl_sync(0xffffffffu, ready, 0)) return true;
    return __all_sync(0xffffffffu, mbar_wait(bar, parity));
}

// ---------------------------------------------------------------------------------------
// Thread-block clusters
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cta address -> the same offset in cluster rank `rank`'s shared memory
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// One arrival on an mbarrier of any CTA of the cluster (`addr` from map_rank), release at
// cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// ---------------------------------------------------------------------------------------
// Proxy fences
// ---------------------------------------------------------------------------------------
// Makes this thread's generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// im2col load of a 4-D NHWC tensor: pixelsPerColumn pixels x channelsPerPixel channels,
// starting at pixel (n, h, w) of the bounding box and channel c, with the filter-tap
// offsets (off_w, off_h) added to every pixel's coordinates.
__device__ __forceinline__ void tma_load_im2col_4d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                                   int c, int w, int h, int n, uint16_t off_w,
                                                   uint16_t off_h) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.im2col.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], {%7, %8};"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c), "r"(w), "r"(h), "r"(n),
          "h"(off_w), "h"(off_h)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int x,
                                            int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Tiled loads of one CTA of a pair (cta_group::2): the data lands in this CTA's shared memory
// at `dst`, the transaction bytes are counted on the mbarrier at `bar_cluster` (an address from
// map_rank: the even CTA's barrier).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster, int x,
                                                 int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster, int x,
                                                 int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// im2col-mode load of one CTA of a pair (cta_group::2): lands in this CTA's shared memory,
// transaction bytes counted on the even CTA's barrier `bar_cluster` (from map_rank).
__device__ __forceinline__ void tma_load_im2col_4d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster,
                                                        int c, int w, int h, int n, uint16_t off_w, uint16_t off_h) {
    asm volatile(
        "cp.async.bulk.tensor.4d.im2col.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], {%7, %8};"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c), "r"(w), "r"(h), "r"(n),
          "h"(off_w), "h"(off_h)
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];"
                 :
                 : "l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until all committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until all committed bulk stores are complete (writes performed).
__device__ __forceinline__ void bulk_wait_group0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor-core MMA
// ---------------------------------------------------------------------------------------
// Whole-warp operation: allocates `ncols` TMEM columns (power of two >= 32) and writes the
// base address to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 or f16 operands, f32 accumulator),
// issued by one thread. `accumulate` = 0 overwrites D.
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same MMA issued by a whole converged warp: only the lane whose `leader` is non-zero
// issues it. An MMA-issuing loop that the whole warp runs, with the MMAs predicated instead of
// placed under a one-lane branch, keeps the warp converged; measured on B200 that issues a
// group of four M=128, N=128 MMAs about twice as fast as the one-lane branch does.
__device__ __forceinline__ void umma_f16_ss_if(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}

// umma_commit by the lane whose `leader` is non-zero, in a converged warp.
__device__ __forceinline__ void umma_commit_if(uint32_t bar, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t"
        "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar),
        "r"(leader)
        : "memory");
}

// ---- CTA pairs (cta_group::2): one MMA spans the two CTAs of a 2-CTA cluster --------------
// Each CTA holds M/2 rows of A and N/2 columns of B at the same shared-memory offsets, and
// receives its M/2 rows x N of the accumulator in its own TMEM. The even CTA issues; TMEM is
// allocated by the same warp of both CTAs with the same destination offset.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_f16_ss_pair_if(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
        : "memory");
}

// Arrives once on the mbarrier at offset `bar` of every CTA in `cta_mask` when the pair MMAs
// this thread issued before have completed.
__device__ __forceinline__ void umma_commit_pair_if(uint32_t bar, uint16_t cta_mask, uint32_t leader) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t"
        "@q tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}"
        ::"r"(bar), "h"(cta_mask), "r"(leader)
        : "memory");
}

// 1 in exactly one lane of the converged warp, 0 in the others.
__device__ __forceinline__ uint32_t elect_one_sync() {
    uint32_t p = 0;
    asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, %1;\n\tselp.b32 %0, 1, 0, P;\n\t}"
                 : "=r"(p)
                 : "r"(0xffffffffu));
    return p;
}

// Arrives once on the mbarrier when every tcgen05 operation this thread issued before has
// completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 TMEM lanes x 16 consecutive 32-bit columns: thread t of the warp receives lane
// (base lane + t), columns col .. col+15.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start address, leading
// and stride byte offsets (all in 16-byte units), descriptor version 1 (bits 46-47) and the
// layout type in bits 61-63 (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// Instruction descriptor for kind::f16 with bf16 A and B, f32 D, dense.
//   bits 4-5 D format (1 = f32); 7-9 A format (1 = bf16); 10-12 B format (1 = bf16);
//   bit 15 A major (0 = K-major); bit 16 B major (1 = MN-major); 17-22 N>>3; 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// The same with an MN-major A operand as well (bit 15).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_amn(int M, int N, bool b_mn_major) {
    return idesc_bf16_f32(M, N, b_mn_major) | (1u << 15);
}

}  // namespace convb200
