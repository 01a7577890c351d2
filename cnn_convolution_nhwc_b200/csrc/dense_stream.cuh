// Dense NHWC forward convolution for layers whose filter is too large to stay in shared memory:
// the halo implicit GEMM of dense_halo.cuh with 256-row tiles, two TMEM accumulators that share
// every streamed filter slot, and 32-channel halo blocks.
//
// Same operation and flattened-row addressing as dense_halo.cuh (CMU DLSys Lecture 14 notes,
// section 1 "Fix the index contract before optimizing it" for the definition, section 2 "Move the
// channel contraction into matrix multiplication" for the sum of per-tap matrix products): GEMM
// row P = (n*H + y)*W + x of X viewed as [N*H*W][Cin]; tap (i, j) of row P reads row
// P + i*W + j, so a tile of rows P0 .. P0+255 needs the contiguous rows P0 .. P0 + 255 + (K-1)*W
// + K-1 of X, and the A operand of tap (i, j) is that staged halo read from row i*W + j on.
//
// What changes against the halo kernel is the operand traffic per tensor-core cycle when the
// filter has to stream. Each (tap, 32-channel) filter slot -- 32 reduction rows x BN output
// channels -- feeds four MMAs (two K=16 steps into each of two M=128 accumulators, rows 0..127
// and 128..255 of the tile) instead of two, halving the filter bytes per MMA, and each halo
// block serves all K*K taps. The halo is staged 32 channels (64 bytes) per row with the 64-byte
// swizzle so that three halo slots and a deep filter ring fit in shared memory together.
//
// Roles in one persistent CTA of 11 warps (role loops walked by whole converged warps, one lane
// issuing the asynchronous instructions; the producers poll their slots without sleeping -- a
// producer that sleeps between polls refills its slot late and starves the tensor pipe, measured
// at a third of its active cycles):
//   warp 0      TMA: the filter ring, one (tap, channel block) slot at a time;
//   warp 1      TMEM allocation; tcgen05.mma M=128, N=BN, K=16 into the two accumulators of the
//               tile's accumulator pair (two pairs: tile t+1's MMAs run while tile t drains);
//   warps 2..9  epilogue, two warps per TMEM lane quarter taking alternate 64-column chunks of
//               both accumulators: tcgen05.ld, round to bf16, per-warp swizzled staging,
//               coalesced 16-byte stores of the valid rows straight to Y;
//   warp 10     TMA: one halo per (tile, channel block) into a ring of HS slots, running ahead
//               of the filter ring.
#pragma once
#include <cuda_bf16.h>

#include "dense_halo.cuh"
#include "ptx.cuh"

namespace convb200 {

struct DenseStreamParams {
    int rows;          // N * H * W: flattened input positions (GEMM rows computed)
    int H, W, Ho, Wo;
    int K, KK;         // K and K*K
    int Cout;
    int num_cblk;      // ceil(Cin / 32)
    int halo_rows;     // rows per halo slot (n_boxes * box_rows)
    int box_rows;      // rows per TMA box (<= 256, a multiple of 16)
    int n_boxes;
    int halo_bytes;    // halo_rows * 64
    int num_mtiles, num_ntiles, num_tiles;
    int HS;            // halo ring slots
    int BS;            // filter ring slots
};

template <int BN_>
struct DenseStreamCfg {
    static constexpr int BN = BN_;
    static constexpr int BM = 256;                     // two M=128 accumulators per tile
    static constexpr int CB = 32;                      // channels per halo block / filter slot
    static constexpr int B_BOX_BYTES = CB * 64 * 2;    // 32 reduction rows x 64 channels
    static constexpr int B_BYTES = CB * BN * 2;        // one (tap, channel block) filter slot
    static constexpr int NUM_EPI = 8;                  // epilogue warps: two per TMEM lane quarter
    static constexpr int EPI_BYTES = NUM_EPI * 32 * 128;   // per-warp 32 rows x 64 channels staging
    static constexpr int MAX_HS = 4;
    static constexpr int MAX_BS = 24;
    static constexpr int NUM_BARS = 2 * MAX_HS + 2 * MAX_BS + 4 /*acc pairs*/ + 2;
    static constexpr int TMEM_COLS = 4 * BN;           // two accumulator pairs
    static constexpr int THREADS = 32 * (3 + NUM_EPI);   // TMA x2, MMA, epilogue
    static constexpr int HALO_WARP = 2 + NUM_EPI;
    static constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, /*B MN-major*/ true);
    static constexpr uint32_t IDESC_PAIR = idesc_bf16_f32(256, BN, /*B MN-major*/ true);   // cta_group::2
    // shared-memory bytes besides the filter ring and the halo ring
    static constexpr int FIXED_BYTES = 1024 + EPI_BYTES + NUM_BARS * 8 + NUM_EPI * 32 * 8 + 16;
    static_assert(BN == 64 || BN == 128, "two accumulator pairs of BN columns must fit in TMEM");
};

// Shared-memory matrix descriptor for a K-major operand with the 64-byte swizzle (layout type 4):
// rows of 64 bytes, 8-row groups 512 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;                 // leading byte offset (unused when swizzled)
    d |= static_cast<uint64_t>(512u >> 4) << 32;          // stride byte offset: 8 rows x 64 B
    d |= 1ull << 46;
    d |= 4ull << 61;
    return d;
}

template <class Cfg, bool PAIR>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
dense_stream_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmF,
                    __nv_bfloat16 *__restrict__ Y, const DenseStreamParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int BN = Cfg::BN;
    static_assert(!PAIR || BN == 128, "a pair splits the filter slot into two 64-channel boxes");
    constexpr int B_CTA = PAIR ? Cfg::B_BYTES / 2 : Cfg::B_BYTES;   // filter bytes per slot in this CTA
    constexpr int TILE_ROWS = PAIR ? 2 * Cfg::BM : Cfg::BM;          // GEMM rows per (pair) tile
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;   // 1024-B alignment for the swizzles
    uint8_t *smem = smem_raw + (base - raw_base);

    const uint32_t sB = base;                                       // filter ring
    const uint32_t sH = base + p.BS * B_CTA;                        // halo ring
    const uint32_t epi_off = p.BS * B_CTA + p.HS * p.halo_bytes;
    const uint32_t sEpi = base + epi_off;
    const uint32_t bars = sEpi + Cfg::EPI_BYTES;
    constexpr int RH = Cfg::MAX_HS, RB = Cfg::MAX_BS;
    auto hfull = [&](int s) { return bars + 8u * s; };
    auto hempty = [&](int s) { return bars + 8u * (RH + s); };
    auto bfull = [&](int s) { return bars + 8u * (2 * RH + s); };
    auto bempty = [&](int s) { return bars + 8u * (2 * RH + RB + s); };
    auto accf = [&](int b) { return bars + 8u * (2 * RH + 2 * RB + b); };
    auto acce = [&](int b) { return bars + 8u * (2 * RH + 2 * RB + 2 + b); };
    const uint32_t done_bar = bars + 8u * (2 * RH + 2 * RB + 4);
    long long *rowoff_all = reinterpret_cast<long long *>(smem + epi_off + Cfg::EPI_BYTES + Cfg::NUM_BARS * 8);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(rowoff_all + Cfg::NUM_EPI * 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // In a pair the even CTA (rank 0) issues the MMAs for both; its full and accumulator-empty
    // barriers count both CTAs' copies and epilogues. lead(a): barrier a of the even CTA.
    const uint32_t rank = PAIR ? cluster_rank() : 0u;
    auto lead = [&](uint32_t a) { return PAIR ? map_rank(a, 0u) : a; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < RH; ++s) {
            mbar_init(hfull(s), 1);
            mbar_init(hempty(s), 1);
        }
        for (int s = 0; s < RB; ++s) {
            mbar_init(bfull(s), 1);
            mbar_init(bempty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf(b), 1);
            mbar_init(acce(b), (PAIR ? 2 : 1) * Cfg::NUM_EPI);   // one arrival per epilogue warp
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmF);
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
    const int row0 = static_cast<int>(rank) * Cfg::BM;   // this CTA's rows inside the (pair) tile

    // The role loops keep their ring slots and phases as running counters and advance the MMA
    // descriptors by adding to their address fields: the MMA warp is one serial instruction
    // stream, and every instruction of its loop delays the next MMA (a loop with a division per
    // slot was measured at ~440 cycles per 4-MMA slot against ~260 of tensor work). The MMA
    // warp also stays converged (predicated MMAs, no one-lane branch): measured on B200, a loop
    // that waits, fences and issues four M=128, N=128 MMAs per slot takes ~310 cycles per slot
    // that way against ~590 with the MMAs under `if (lane == 0)`.
    if (warp == Cfg::HALO_WARP) {
        // ------------------------------- halo producer ------------------------------
        uint32_t hit = 0, hs = 0, hph = 0;
        bool ok = true;
        for (int t = first; t < p.num_tiles && ok && !*abort_flag; t += step) {
            const int P0 = (t / p.num_ntiles) * TILE_ROWS + row0;
            for (int cb = 0; cb < p.num_cblk; ++cb, ++hit) {
                if (!mbar_wait_warp(hempty(hs), hph ^ 1u)) { ok = false; break; }
                if (lane == 0) {
                    if (rank == 0) mbar_arrive_expect_tx(hfull(hs), (PAIR ? 2 : 1) * p.halo_bytes);
                    for (int bx = 0; bx < p.n_boxes; ++bx) {
                        const uint32_t dst = sH + hs * p.halo_bytes + bx * p.box_rows * 64;
                        if constexpr (PAIR)
                            tma_load_2d_pair(dst, &tmX, lead(hfull(hs)), cb * Cfg::CB, P0 + bx * p.box_rows);
                        else
                            tma_load_2d(dst, &tmX, hfull(hs), cb * Cfg::CB, P0 + bx * p.box_rows);
                    }
                }
                __syncwarp();
                if (++hs == static_cast<uint32_t>(p.HS)) { hs = 0; hph ^= 1u; }
            }
        }
        if (!ok && lane == 0) fail();
        // Drain: every load issued has landed before the CTA may exit (in a pair: has been
        // consumed by the pair's MMAs, which the even CTA's commits report to both CTAs).
        for (uint32_t j = hit > (uint32_t)p.HS ? hit - p.HS : 0u; j < hit; ++j) {
            const bool landed = PAIR ? mbar_wait_warp(hempty(j % p.HS), (j / p.HS) & 1u)
                                     : mbar_wait_warp(hfull(j % p.HS), (j / p.HS) & 1u);
            if (!landed) { if (lane == 0) fail(); break; }
        }
    } else if (warp == 0) {
        // ------------------------------- filter producer ----------------------------
        uint32_t bit = 0, bs = 0, bph = 0;
        bool ok = true;
        for (int t = first; t < p.num_tiles && ok && !*abort_flag; t += step) {
            const int n0 = (t % p.num_ntiles) * BN;
            for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                for (int tap = 0; tap < p.KK; ++tap, ++bit) {
                    if (!mbar_wait_warp(bempty(bs), bph ^ 1u)) { ok = false; break; }
                    if (lane == 0) {
                        if (rank == 0) mbar_arrive_expect_tx(bfull(bs), Cfg::B_BYTES);   // both halves
                        if constexpr (PAIR) {
                            // this CTA's half of the slot: output channels n0 + 64*rank .. + 63
                            tma_load_3d_pair(sB + bs * B_CTA, &tmF, lead(bfull(bs)), n0 + 64 * static_cast<int>(rank),
                                             cb * Cfg::CB, tap);
                        } else {
#pragma unroll
                            for (int h = 0; h < BN / 64; ++h)
                                tma_load_3d(sB + bs * B_CTA + h * Cfg::B_BOX_BYTES, &tmF, bfull(bs), n0 + h * 64,
                                            cb * Cfg::CB, tap);
                        }
                    }
                    __syncwarp();
                    if (++bs == static_cast<uint32_t>(p.BS)) { bs = 0; bph ^= 1u; }
                }
            }
        }
        if (!ok && lane == 0) fail();
        for (uint32_t j = bit > (uint32_t)p.BS ? bit - p.BS : 0u; j < bit; ++j) {
            const bool landed = PAIR ? mbar_wait_warp(bempty(j % p.BS), (j / p.BS) & 1u)
                                     : mbar_wait_warp(bfull(j % p.BS), (j / p.BS) & 1u);
            if (!landed) { if (lane == 0) fail(); break; }
        }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // The whole warp runs the loop, converged; the MMAs and commits are predicated on one
        // elected lane (every commit of this warp comes from that lane, so that each commit
        // tracks all of the warp's MMAs). In a pair only the even CTA's warp issues: M = 256
        // MMAs (128 rows from each CTA) whose commits arrive on the barriers of both CTAs.
        const uint32_t leader = elect_one_sync();
        constexpr uint16_t kBoth = 0x3;
        auto commit = [&](uint32_t bar) {
            if constexpr (PAIR) umma_commit_pair_if(bar, kBoth, leader);
            else umma_commit_if(bar, leader);
        };
        auto mma = [&](uint32_t d, uint64_t a, uint64_t bdesc, uint32_t acc) {
            if constexpr (PAIR) umma_f16_ss_pair_if(d, a, bdesc, Cfg::IDESC_PAIR, acc, leader);
            else umma_f16_ss_if(d, a, bdesc, Cfg::IDESC, acc, leader);
        };
        if (rank == 0) {
            uint32_t local = 0, hs = 0, hph = 0, bs = 0, bph = 0;
            bool ok = true;
            // descriptors differ only in the start-address field (16-byte units): A +4 per 64-byte
            // halo row, +2 per K=16 step, +512 for the second accumulator's rows (128 rows further
            // on); B +B_CTA/16 per filter slot, +128 per K=16 step (16 reduction rows = 2048 B)
            const uint64_t b_desc0 = smem_desc_sw128(sB, Cfg::B_BOX_BYTES, 1024);
            constexpr uint32_t kSlotUnits = B_CTA >> 4;
            const uint32_t row_skip4 = static_cast<uint32_t>(p.W - p.K) * 4u;
            for (int t = first; t < p.num_tiles && ok && !__any_sync(0xffffffffu, *abort_flag != 0);
                 t += step, ++local) {
                const uint32_t b = local & 1u;
                // waiting here means the epilogue is the slower role: sleep between polls
                if (!mbar_wait_warp_backoff(acce(b), ((local >> 1) & 1u) ^ 1u, 64)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d0 = tmem_base + b * (2 * BN);   // rows 0..127 of the CTA's tile
                const uint32_t d1 = d0 + BN;                    // rows 128..255
                for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                    if (!mbar_wait_warp(hfull(hs), hph)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t a_desc0 = smem_desc_sw64(sH + hs * p.halo_bytes);
                    uint32_t row4 = 0;   // (ky*W + kx) * 4: tap (ky, kx) reads the halo from row ky*W + kx on
                    for (int ky = 0; ky < p.K && ok; ++ky, row4 += row_skip4) {
                        for (int kx = 0; kx < p.K; ++kx, row4 += 4u) {
                            if (!mbar_wait_warp(bfull(bs), bph)) { ok = false; break; }
                            tc_fence_after();
                            const uint64_t ad = a_desc0 + row4;
                            const uint64_t bd = b_desc0 + bs * kSlotUnits;
                            const uint32_t acc = (cb | ky | kx) != 0 ? 1u : 0u;
                            mma(d0, ad, bd, acc);
                            mma(d1, ad + 512, bd, acc);
                            mma(d0, ad + 2, bd + 128, 1u);
                            mma(d1, ad + 514, bd + 128, 1u);
                            commit(bempty(bs));
                            if (++bs == static_cast<uint32_t>(p.BS)) { bs = 0; bph ^= 1u; }
                        }
                    }
                    if (!ok) break;
                    commit(hempty(hs));
                    if (++hs == static_cast<uint32_t>(p.HS)) { hs = 0; hph ^= 1u; }
                }
                if (!ok) break;
                commit(accf(b));
            }
            __syncwarp();
            if (!ok && lane == 0) fail();
            // All MMAs issued by this warp complete before TMEM is released (in a pair: before
            // the cluster barrier that both CTAs pass ahead of their deallocation).
            commit(done_bar);
            if (!mbar_wait_warp(done_bar, 0) && lane == 0) fail();
        }
    } else {
        // ------------------------------- Epilogue (warps 2..9) -----------------------
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int eg = (warp - 2) >> 2;     // which of the quarter's two warps: chunks eg, eg + 2, ...
        const uint32_t stage = sEpi + (warp - 2) * 4096;
        long long *rowoff = rowoff_all + (warp - 2) * 32;
        uint32_t local = 0;
        for (int t = first; t < p.num_tiles; t += step, ++local) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t b = local & 1u;
            if (!mbar_wait_warp_backoff(accf(b), (local >> 1) & 1u, 128)) { if (lane == 0) fail(); break; }
            tc_fence_after();
            const int mt = t / p.num_ntiles;
            const int n0 = (t - mt * p.num_ntiles) * BN;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                // this lane's row: flattened input position P -> output row, or -1 if dropped
                {
                    const int P = mt * TILE_ROWS + row0 + half * 128 + q * 32 + lane;
                    long long off = -1;
                    if (P < p.rows) {
                        const int row = P / p.W;
                        const int x = P - row * p.W;
                        const int n = row / p.H;
                        const int y = row - n * p.H;
                        if (x < p.Wo && y < p.Ho)
                            off = ((static_cast<long long>(n) * p.Ho + y) * p.Wo + x) * p.Cout;
                    }
                    rowoff[lane] = off;
                }
                const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * (2 * BN) + half * BN;
#pragma unroll 1
                for (int h = eg; h < BN / 64; h += 2) {
                    uint32_t r[4][16];
#pragma unroll
                    for (int g = 0; g < 4; ++g) tmem_ld_32x32b_x16(t_row + h * 64 + g * 16, r[g]);
                    tmem_wait_ld();
                    // stage this warp's 32 rows x 64 channels (128-byte swizzled rows)
                    const uint32_t row_addr = stage + lane * 128;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const uint32_t c = g * 2 + cc;
                            const uint32_t *v = &r[g][cc * 8];
                            st_shared_v4(row_addr + ((c ^ (lane & 7)) << 4),
                                         halo_pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1])),
                                         halo_pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3])),
                                         halo_pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5])),
                                         halo_pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7])));
                        }
                    }
                    __syncwarp();
                    // coalesced stores: 8 lanes per row, 4 rows per instruction
                    const int col = n0 + h * 64 + (lane & 7) * 8;
                    if (col < p.Cout) {
                        const long long y_elems = 1LL * (p.rows / (p.H * p.W)) * p.Ho * p.Wo * p.Cout;   // bounds checks (debug build)
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int rr = i * 4 + (lane >> 3);
                            const long long off = rowoff[rr];
                            if (off >= 0 && in_bounds(off + col, 8, y_elems, kSiteStreamY, status)) {
                                uint32_t a, bb, c, d;
                                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                             : "=r"(a), "=r"(bb), "=r"(c), "=r"(d)
                                             : "r"(stage + rr * 128 + ((((lane & 7) ^ (rr & 7))) << 4)));
                                uint4 *dst = reinterpret_cast<uint4 *>(Y + off + col);
                                *dst = make_uint4(a, bb, c, d);
                            }
                        }
                    }
                    __syncwarp();
                }
            }
            // the accumulator pair may now be overwritten by the MMA warp (of the even CTA)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR) mbar_arrive_cluster(lead(acce(b)));
                else mbar_arrive(acce(b));
            }
        }
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
