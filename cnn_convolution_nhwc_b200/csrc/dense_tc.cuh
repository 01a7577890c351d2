// Dense NHWC forward convolution as an implicit GEMM on the sm_100a tensor cores.
//
// Matrix form (CMU DLSys Lecture 14 notes, section 5 "Generalize the patch matrix to
// channels and batches"; with the stride, zero-padding, dilation and bias variants of
// "Convolution Is Wx+b Moving Across a Signal", which the TMA im2col unit expresses directly:
// element strides for the stride, a bounding box that starts at -pad for the padding, with
// out-of-range pixels read as zeros, and tap offsets scaled by the dilation, each per axis):
// A_col[(n,y,x), (i,j,c)] = X[n, y+i, x+j, c] is the (N*Ho*Wo) x (KH*KW*Cin) patch matrix,
// F_mat is F viewed as (KH*KW*Cin) x Cout, and Y_mat = A_col * F_mat is Y viewed as
// (N*Ho*Wo) x Cout. The notes' closing remark in section 6 -- generate patch fragments as
// needed instead of materialising the matrix -- is what this kernel does: A_col never exists
// in memory. Each 128-row x 64-column block of it is gathered straight from X by one TMA
// im2col load (the hardware form of the overlapping-window view of section 4), for filter
// tap (i, j) and channel block c0, and consumed from shared memory by tcgen05 MMAs. The
// reduction runs tap by tap, which is the sum of KH*KW shifted-slice channel matmuls of
// section 2.
//
// Channel groups (the grouped Conv1D of the Wx+b page's section "Find the same sum in CKE's
// C kernels", on two axes) are independent GEMMs of the same shape: a group has its own three
// tensor maps (X at channel g*Cin_g, F and Y at column g*Cout_g, each with the group's extent,
// so boxes past a group's end read zeros and stores are clipped to it), and the persistent
// tile loop runs over (group, row block, column block).
//
// Roles inside one persistent CTA of 6 warps (each role loop is walked by whole, converged
// warps; a single lane issues the asynchronous instructions):
//   warp 0      TMA loads into a STAGES-deep ring of (A, B) slots;
//   warp 1      allocates TMEM; issues tcgen05.mma (M=128, N=BN, K=16) into one of two TMEM
//               tile buffers -- for BN <= 128 as two partial accumulators that alternate per
//               K=16 step and are added once by the epilogue -- and tcgen05.commit to free
//               ring slots;
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows (warp w reads TMEM lanes
//               32*(w%4) .. +31), round to bf16, 128-byte-swizzled staging in shared
//               memory, TMA store to Y. The two accumulators let tile t+1's MMAs run
//               while tile t is stored.
// Shared-memory operand layouts (both 128-byte swizzled, as TMA writes them):
//   A slot: 128 pixel rows x 64 channels (128 B per row) -- K-major.
//   B slot: BN/64 boxes, each 64 reduction rows x 64 output channels (128 B per row) --
//           MN-major, read in place from the KKIO filter, no repacking.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace convb200 {

struct DenseTcParams {
    int M;          // N * Ho * Wo (GEMM rows of every group)
    int Wo;
    int HoWo;
    int KW;         // taps per filter row (the reduction walks ky outer, kx inner)
    int ncols;      // output channels of one group (Cout / groups)
    int num_cblk;   // ceil(Cin_g / 64), Cin_g = input channels of one group
    int num_kblk;   // KH * KW * num_cblk
    int num_ntiles; // ceil(ncols / BN)
    int tiles_per_group;   // ceil(M / 128) * num_ntiles
    int num_tiles;  // groups of this launch * tiles_per_group
    int groups;     // groups of this launch (tensor maps in use)
    int sh, sw, ph, pw, dh, dw;   // window of output (y, x) starts at (y*sh - ph, x*sw - pw);
                                  // tap (i, j) is dh*i rows and dw*j columns further on
    const float *bias;      // per output channel of this launch's first group (group g's at
                            // bias + g*ncols), added in fp32 before the bf16 rounding; or null
};

// Tensor maps of the groups one launch covers: group g reads X channels g*Cin_g .. +Cin_g
// (map x[g], channel extent Cin_g, so a 64-channel box past the group reads zeros), filter
// columns g*ncols .. +ncols (f[g]) and writes Y columns g*ncols .. +ncols (y[g], stores
// clipped to the group).
constexpr int kTcGroups = 8;   // groups per launch of the grouped instantiation (24 maps, 3 KB)

template <int NG>
struct alignas(64) DenseTcMaps {
    CUtensorMap x[NG];
    CUtensorMap f[NG];
    CUtensorMap y[NG];
};

template <int BN_, int STAGES_>
struct DenseTcCfg {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int BM = 128;
    static constexpr int BK = 64;
    static constexpr int A_BYTES = BM * BK * 2;        // 16 KB
    static constexpr int B_BOX_BYTES = BK * 64 * 2;    // 8 KB: 64 k-rows x 64 channels
    static constexpr int B_BYTES = BK * BN * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int EPI_WARP_BYTES = 32 * BN * 2; // 32 rows x BN channels
    static constexpr int EPI_BYTES = 4 * EPI_WARP_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
    // Two partial accumulators per tile when they fit (BN <= 128): consecutive K=16 steps
    // alternate between them, since back-to-back MMAs into one accumulator wait on each other
    // (measured 99 against 64 cycles per M=128 x N=128 MMA); the epilogue adds the two partial
    // sums once in float32. Times two tile buffers.
    static constexpr int PARTS = BN <= 128 ? 2 : 1;
    static constexpr int TMEM_COLS = 2 * PARTS * BN;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + NUM_BARS * 8 + 16;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*B MN-major*/ true);
    static constexpr uint32_t IDESC_PAIR = idesc_bf16_f32(2 * BM, BN, /*B MN-major*/ true);   // cta_group::2
    // shared memory of the CTA-pair form: each CTA stages its A tile and half of every B slot
    static constexpr int SMEM_BYTES_PAIR = 1024 + STAGES * (A_BYTES + B_BYTES / 2) + EPI_BYTES + NUM_BARS * 8 + 16;
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
    static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS <= 512, "TMEM columns");
    static constexpr uint32_t A_UNITS = A_BYTES >> 4;   // descriptor address field per A slot
    static constexpr uint32_t B_UNITS = B_BYTES >> 4;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// PAIR (one group, BN >= 128): 2-CTA clusters; each CTA stages the A tile of its own 128 rows
// and half of every B slot (its BN/2 output channels); the even CTA issues M = 256 MMAs
// (cta_group::2) that read both CTAs' operands and commit to both CTAs' barriers -- the B bytes
// each SM stages per MMA halve. Its full barriers count both CTAs' bytes; its
// accumulator-empty barriers both CTAs' epilogue warps.
template <class Cfg, int NG, bool PAIR>
__global__ void __launch_bounds__(192, 1)
dense_tc_kernel(const __grid_constant__ DenseTcMaps<NG> maps, const DenseTcParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int BN = Cfg::BN;
    constexpr int STAGES = Cfg::STAGES;
    static_assert(!PAIR || (NG == 1 && BN >= 128), "pairs: one group, at least two 64-channel boxes");
    constexpr int B_CTA = PAIR ? Cfg::B_BYTES / 2 : Cfg::B_BYTES;   // B bytes per slot in this CTA
    constexpr int STAGE_CTA = Cfg::A_BYTES + B_CTA;
    constexpr int TILE_ROWS = PAIR ? 2 * Cfg::BM : Cfg::BM;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;   // 1024-B alignment for the swizzle
    uint8_t *smem = smem_raw + (base - raw_base);

    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * Cfg::A_BYTES;
    uint8_t *sEpi = smem + STAGES * STAGE_CTA;
    const uint32_t bars = base + STAGES * STAGE_CTA + Cfg::EPI_BYTES;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
    auto accf_bar = [&](int b) { return bars + 8u * (2 * STAGES + b); };
    auto acce_bar = [&](int b) { return bars + 8u * (2 * STAGES + 2 + b); };
    const uint32_t done_bar = bars + 8u * (2 * STAGES + 4);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + STAGES * STAGE_CTA +
                                                         Cfg::EPI_BYTES + Cfg::NUM_BARS * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_rank() : 0u;
    auto lead = [&](uint32_t a) { return PAIR ? map_rank(a, 0u) : a; };   // the even CTA's barrier

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), PAIR ? 8 : 4);   // one arrival per epilogue warp (of both CTAs)
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        for (int g = 0; g < p.groups; ++g) {
            prefetch_tensormap(&maps.x[g]);
            prefetch_tensormap(&maps.f[g]);
            prefetch_tensormap(&maps.y[g]);
        }
    }
    if (warp == 1) {
        if constexpr (PAIR) {
            tmem_alloc_pair(smem_u32(tmem_holder), Cfg::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(tmem_holder), Cfg::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) cluster_sync_all();   // both CTAs' barriers and TMEM exist before either is used
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    auto fail = [&]() {
        atomicOr(status, kStatusTimeout);
        *abort_flag = 1;
        if constexpr (PAIR) st_cluster_u32(map_rank(smem_u32(const_cast<int *>(abort_flag)), rank ^ 1u), 1u);
    };
    const int first = static_cast<int>(PAIR ? blockIdx.x >> 1 : blockIdx.x);
    const int step = static_cast<int>(PAIR ? gridDim.x >> 1 : gridDim.x);
    // tile -> (group of this launch, 128-row block, BN-column block)
    auto split = [&](int tile, int &grp, int &mt, int &nt) {
        grp = NG == 1 ? 0 : tile / p.tiles_per_group;
        const int rem = tile - grp * p.tiles_per_group;
        mt = rem / p.num_ntiles;
        nt = rem - mt * p.num_ntiles;
    };

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        // The whole warp walks the loop (it stays converged); lane 0 issues.
        uint32_t it = 0, s = 0, ph = 0;   // ring slot and phase as running counters
        for (int tile = first; tile < p.num_tiles && !*abort_flag; tile += step) {
            int grp, mt, nt;
            split(tile, grp, mt, nt);
            const CUtensorMap *tmX = &maps.x[grp];
            const CUtensorMap *tmF = &maps.f[grp];
            const int m0 = mt * TILE_ROWS + static_cast<int>(rank) * Cfg::BM;   // this CTA's rows
            const int n0 = nt * BN;
            const int img = m0 / p.HoWo;
            const int rem = m0 - img * p.HoWo;
            const int oy = rem / p.Wo;
            const int ox = rem - oy * p.Wo;
            bool ok = true;
            int tap = 0, cb = 0, ky = 0, kx = 0;
            for (int kb = 0; kb < p.num_kblk; ++kb, ++it) {
                if (!mbar_wait_warp(empty_bar(s), ph ^ 1u)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    if constexpr (PAIR) {
                        // both CTAs' A tiles and B halves complete on the even CTA's barrier
                        if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * Cfg::A_BYTES + Cfg::B_BYTES);
                        tma_load_im2col_4d_pair(sA + s * Cfg::A_BYTES, tmX, lead(full_bar(s)), cb * 64,
                                                ox * p.sw - p.pw, oy * p.sh - p.ph, img,
                                                static_cast<uint16_t>(kx * p.dw), static_cast<uint16_t>(ky * p.dh));
#pragma unroll
                        for (int h = 0; h < BN / 128; ++h)
                            tma_load_3d_pair(sB + s * B_CTA + h * Cfg::B_BOX_BYTES, tmF, lead(full_bar(s)),
                                             n0 + static_cast<int>(rank) * (BN / 2) + h * 64, cb * 64, tap);
                    } else {
                        mbar_arrive_expect_tx(full_bar(s), Cfg::STAGE_BYTES);
                        tma_load_im2col_4d(sA + s * Cfg::A_BYTES, tmX, full_bar(s), cb * 64, ox * p.sw - p.pw,
                                           oy * p.sh - p.ph, img, static_cast<uint16_t>(kx * p.dw),
                                           static_cast<uint16_t>(ky * p.dh));
#pragma unroll
                        for (int h = 0; h < BN / 64; ++h)
                            tma_load_3d(sB + s * Cfg::B_BYTES + h * Cfg::B_BOX_BYTES, tmF, full_bar(s),
                                        n0 + h * 64, cb * 64, tap);
                    }
                }
                __syncwarp();
                // next (tap, channel block) in (i, j, c) order
                if (++cb == p.num_cblk) {
                    cb = 0;
                    ++tap;
                    if (++kx == p.KW) { kx = 0; ++ky; }
                }
                if (++s == static_cast<uint32_t>(STAGES)) { s = 0; ph ^= 1u; }
            }
            if (!ok) break;
        }
        // Drain: every load issued has landed before the CTA may exit (in a pair: has been
        // consumed by the pair's MMAs, which the even CTA's commits report to both CTAs).
        const uint32_t j0 = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t j = j0; j < it; ++j) {
            const bool landed = PAIR ? mbar_wait_warp(empty_bar(j % STAGES), (j / STAGES) & 1u)
                                     : mbar_wait_warp(full_bar(j % STAGES), (j / STAGES) & 1u);
            if (!landed) {
                if (lane == 0) fail();
                break;
            }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // The whole warp walks the loop, converged; the MMAs and commits are predicated on one
        // elected lane (all of them, so that each commit tracks every MMA of the warp). The loop
        // is one serial instruction stream, so the ring slot and phase are running counters and
        // the descriptors advance by adding to their address fields (16-byte units).
        // A: K-major, +2 per 16 channels (32 B inside the swizzle atom), 8-row groups 1024 B
        // apart. B: MN-major, +128 per 16 reduction rows (2048 B), 8-row groups 1024 B apart
        // (SBO), 64-channel boxes B_BOX_BYTES apart (LBO).
        const uint32_t leader = elect_one_sync();
        constexpr uint16_t kBoth = 0x3;
        auto commit = [&](uint32_t bar) {
            if constexpr (PAIR) umma_commit_pair_if(bar, kBoth, leader);
            else umma_commit_if(bar, leader);
        };
        const uint64_t a_desc0 = smem_desc_sw128(sA, 16, 1024);
        const uint64_t b_desc0 = smem_desc_sw128(sB, Cfg::B_BOX_BYTES, 1024);
        constexpr uint32_t kBUnits = B_CTA >> 4;
        uint32_t it = 0, local = 0, s = 0, ph = 0;
        // in a pair only the even CTA's MMA warp walks the tiles
        for (int tile = first; rank == 0 && tile < p.num_tiles && !__any_sync(0xffffffffu, *abort_flag != 0);
             tile += step, ++local) {
            const uint32_t b = local & 1u;
            const uint32_t aph = (local >> 1) & 1u;
            // waiting here means the epilogue is the slower role: sleep between polls instead
            // of taking its issue slots
            if (!mbar_wait_warp_backoff(acce_bar(b), aph ^ 1u, 64)) {
                if (lane == 0) fail();
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * (Cfg::PARTS * BN);   // partial p at + p*BN
            bool ok = true;
            for (int kb = 0; kb < p.num_kblk; ++kb, ++it) {
                if (!mbar_wait_warp(full_bar(s), ph)) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = a_desc0 + s * Cfg::A_UNITS;
                const uint64_t bd = b_desc0 + s * kBUnits;
#pragma unroll
                for (int kk = 0; kk < Cfg::BK / 16; ++kk) {
                    const uint32_t part = Cfg::PARTS == 2 ? (kk & 1) : 0;
                    // the first MMA into each partial accumulator of the tile overwrites it
                    const uint32_t acc = (kb != 0 || kk >= Cfg::PARTS) ? 1u : 0u;
                    if constexpr (PAIR)
                        umma_f16_ss_pair_if(d_tmem + part * BN, ad + 2 * kk, bd + 128 * kk, Cfg::IDESC_PAIR, acc,
                                            leader);
                    else
                        umma_f16_ss_if(d_tmem + part * BN, ad + 2 * kk, bd + 128 * kk, Cfg::IDESC, acc, leader);
                }
                commit(empty_bar(s));
                if (++s == static_cast<uint32_t>(STAGES)) { s = 0; ph ^= 1u; }
            }
            if (!ok) break;
            commit(accf_bar(b));
        }
        __syncwarp();
        // All MMAs issued by this warp complete before TMEM is released (in a pair: before the
        // cluster barrier both CTAs pass ahead of their deallocation).
        if (rank == 0) {
            commit(done_bar);
            if (!mbar_wait_warp(done_bar, 0) && lane == 0) fail();
        }
    } else {
        // ------------------------------- Epilogue -----------------------------------
        const int q = warp & 3;   // TMEM lane quarter this warp may access
        uint8_t *stage = sEpi + q * Cfg::EPI_WARP_BYTES;
        const uint32_t stage_s = smem_u32(stage);
        uint32_t local = 0;
        for (int tile = first; tile < p.num_tiles; tile += step, ++local) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t b = local & 1u;
            const uint32_t aph = (local >> 1) & 1u;
            const bool ok = mbar_wait_warp(accf_bar(b), aph);
            if (!ok) { if (lane == 0) fail(); break; }
            tc_fence_after();
            int grp, mt, nt;
            split(tile, grp, mt, nt);
            const int m0 = mt * TILE_ROWS + static_cast<int>(rank) * Cfg::BM;
            const int n0 = nt * BN;
            // the staging buffer is free once the previous tile's stores have read it
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * (Cfg::PARTS * BN);
#pragma unroll 1
            for (int h = 0; h < BN / 64; ++h) {
                uint32_t r[4][16];
#pragma unroll
                for (int g = 0; g < 4; ++g) tmem_ld_32x32b_x16(t_row + h * 64 + g * 16, r[g]);
                tmem_wait_ld();
                if (Cfg::PARTS == 2) {   // the two partial sums (even and odd K=16 steps), added once
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint32_t r2[16];
                        tmem_ld_32x32b_x16(t_row + BN + h * 64 + g * 16, r2);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            r[g][c] = __float_as_uint(__fadd_rn(__uint_as_float(r[g][c]), __uint_as_float(r2[c])));
                    }
                }
                if (p.bias) {   // one fp32 addition per output, before the single rounding
                    const int c0 = n0 + h * 64;
                    const float *bg = p.bias + static_cast<long long>(grp) * p.ncols;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const int col = c0 + u * 16 + c;
                            const bool bok =
                                col < p.ncols && in_bounds(static_cast<long long>(grp) * p.ncols + col, 1,
                                                           static_cast<long long>(p.groups) * p.ncols, kSiteTcBias, status);
                            const float bv = bok ? __ldg(bg + col) : 0.0f;
                            r[u][c] = __float_as_uint(__fadd_rn(__uint_as_float(r[u][c]), bv));
                        }
                }
                const uint32_t row_addr = stage_s + h * 4096 + lane * 128;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const uint32_t c = g * 2 + cc;   // 16-byte chunk = 8 channels
                        const uint32_t* v = &r[g][cc * 8];
                        st_shared_v4(row_addr + ((c ^ (lane & 7)) << 4),
                                     pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1])),
                                     pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3])),
                                     pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5])),
                                     pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7])));
                    }
                }
            }
            // accumulator b may now be overwritten by the MMA warp (of the even CTA)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster(lead(acce_bar(b)));
                else mbar_arrive(acce_bar(b));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                const int row0 = m0 + q * 32;
                if (row0 < p.M) {
#pragma unroll
                    for (int h = 0; h < BN / 64; ++h)
                        if (n0 + h * 64 < p.ncols) tma_store_2d(&maps.y[grp], stage_s + h * 4096, n0 + h * 64, row0);
                    bulk_commit_group();
                }
            }
        }
        if (lane == 0) bulk_wait_group0();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    // neither CTA of a pair leaves while the other may still signal its barriers
    if constexpr (PAIR) cluster_sync_all();
    tc_fence_after();
    if (warp == 1) {
        if constexpr (PAIR) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
        else tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace convb200
