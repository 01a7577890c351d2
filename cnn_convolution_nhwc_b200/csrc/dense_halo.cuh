// Dense NHWC forward convolution as an implicit GEMM over the flattened input grid, on the
// sm_100a tensor cores, loading every input pixel of a tile once ("halo" tiles).
//
// The CMU DLSys Lecture 14 notes (section 2, "Move the channel contraction into matrix
// multiplication") write the convolution as a sum over filter taps (i, j) of shifted input
// slices times the channel matrix F[i, j]. Flatten X to rows P = (n*H + y)*W + x of Cin
// channels. For any P whose (y, x) is a valid output origin (y < Ho, x < Wo), the input pixel
// tap (i, j) needs is row P + i*W + j -- a fixed shift for the whole tile. So a tile of 128
// consecutive rows P0 .. P0+127 needs only the contiguous rows P0 .. P0 + 127 + (K-1)*W + K-1
// of X (its halo): one TMA tiled load per 64-channel block, and the A operand of tap (i, j)
// is the same shared-memory tile read from row i*W + j on. tcgen05 applies the 128-byte
// swizzle from absolute shared-memory address bits, so a K-major SW128 descriptor may start at
// any 128-byte row of the TMA-written tile (base-offset field 0). Rows whose (y, x) is not a
// valid output (the last K-1 columns and rows of every image) are computed and dropped by the
// epilogue: the price of a shift-only addressing, (H*W - Ho*Wo) / (Ho*Wo) extra MMA rows.
//
// Compared with gathering one im2col tile per tap, the operand bytes per tile fall from
// K*K*16 KB to (halo rows)*128 B per channel block, and with the filter resident in shared
// memory the per-tile operand traffic is the halo alone; the SM's TMA engine is then no
// longer the bottleneck.
//
// Roles in one persistent CTA of 10 warps (role loops walked by whole converged warps, one lane
// issuing the asynchronous instructions):
//   warp 0      TMA: the resident filter once (or a ring of per-tap filter slots), then one
//               halo per (tile, channel block) into a ring of HS halo slots;
//   warp 1      TMEM allocation; tcgen05.mma M=128, N=BN, K=16 into one of two accumulators;
//   warps 2..9  epilogue, two warps per TMEM lane quarter taking alternate 64-column chunks:
//               tcgen05.ld, round to bf16, per-warp swizzled staging, coalesced 16-byte stores
//               of the valid rows straight to Y.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace convb200 {

struct DenseHaloParams {
    int rows;          // N * H * W: flattened input positions (GEMM rows computed)
    int H, W, Ho, Wo;
    int K, KK;         // K and K*K
    int Cout;
    int num_cblk;      // ceil(Cin / 64)
    int num_kblk;      // KK * num_cblk, ordered channel block outer, tap inner
    int halo_rows;     // rows per halo buffer (n_boxes * box_rows)
    int box_rows;      // rows per TMA box (<= 256)
    int n_boxes;
    int num_mtiles, num_ntiles, num_tiles;
    int HS;            // halo ring slots
    int BS;            // filter ring slots (streamed filter only)
    int b_region;      // bytes of the filter region (resident: num_kblk slots; else BS slots)
    int halo_bytes;    // halo_rows * 128
    int n_fixed;       // 1: each CTA keeps one N tile (resident filter with several N tiles)
};

template <int BN_, bool BRES_>
struct DenseHaloCfg {
    static constexpr int BN = BN_;
    static constexpr bool BRES = BRES_;
    static constexpr int BM = 128;
    static constexpr int B_BOX_BYTES = 64 * 64 * 2;   // 64 reduction rows x 64 channels
    static constexpr int B_BYTES = 64 * BN * 2;       // one (tap, channel block) filter slot
    static constexpr int NUM_EPI = 8;                 // epilogue warps: two per TMEM lane quarter
    static constexpr int THREADS = 64 + 32 * NUM_EPI;
    static constexpr int EPI_BYTES = NUM_EPI * 32 * 128;   // per-warp 32 rows x 64 channels staging
    static constexpr int MAX_RING = 8;
    static constexpr int NUM_BARS = 2 * MAX_RING /*halo*/ + 2 * MAX_RING /*filter*/ + 4 /*acc*/ + 2;
    // Tiles up to 128 columns wide alternate their MMAs between two partial accumulators (an MMA
    // into the accumulator the previous one wrote waits for it: measured on B200, 99 against 64
    // cycles at N = 128), summed once in the epilogue; two tiles in flight either way.
    static constexpr int PARTS = BN <= 128 ? 2 : 1;
    static constexpr int TMEM_COLS = 2 * PARTS * BN;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*B MN-major*/ true);
    // shared-memory bytes besides the filter region and the halo ring
    static constexpr int FIXED_BYTES = 1024 + EPI_BYTES + NUM_BARS * 8 + NUM_EPI * 32 * 8 + 16;
    static_assert(BN == 64 || BN == 128 || BN == 256, "BN");
};

__device__ __forceinline__ uint32_t halo_pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
dense_halo_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmF,
                  __nv_bfloat16 *__restrict__ Y, const DenseHaloParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int BN = Cfg::BN;
    constexpr bool BRES = Cfg::BRES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;   // 1024-B alignment for the swizzle
    uint8_t *smem = smem_raw + (base - raw_base);

    const uint32_t sB = base;                                 // filter region
    const uint32_t sH = base + p.b_region;                    // halo ring
    const uint32_t epi_off = p.b_region + p.HS * p.halo_bytes;
    const uint32_t sEpi = base + epi_off;
    const uint32_t bars = sEpi + Cfg::EPI_BYTES;
    constexpr int R = Cfg::MAX_RING;
    auto hfull = [&](int s) { return bars + 8u * s; };
    auto hempty = [&](int s) { return bars + 8u * (R + s); };
    auto bfull = [&](int s) { return bars + 8u * (2 * R + s); };
    auto bempty = [&](int s) { return bars + 8u * (3 * R + s); };
    auto accf = [&](int b) { return bars + 8u * (4 * R + b); };
    auto acce = [&](int b) { return bars + 8u * (4 * R + 2 + b); };
    const uint32_t done_bar = bars + 8u * (4 * R + 4);
    long long *rowoff_all = reinterpret_cast<long long *>(smem + epi_off + Cfg::EPI_BYTES + Cfg::NUM_BARS * 8);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(rowoff_all + Cfg::NUM_EPI * 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < R; ++s) {
            mbar_init(hfull(s), 1);
            mbar_init(hempty(s), 1);
            mbar_init(bfull(s), 1);
            mbar_init(bempty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf(b), 1);
            mbar_init(acce(b), Cfg::NUM_EPI);   // one arrival per epilogue warp
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmF);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    auto fail = [&]() {
        atomicOr(status, kStatusTimeout);
        *abort_flag = 1;
    };
    // Tile order: with a resident filter and several N tiles each CTA keeps one N tile.
    const int cta_per_n = p.n_fixed ? static_cast<int>(gridDim.x) / p.num_ntiles : 0;
    const int my_nt = p.n_fixed ? static_cast<int>(blockIdx.x) % p.num_ntiles : 0;
    const int first = p.n_fixed ? static_cast<int>(blockIdx.x) / p.num_ntiles : static_cast<int>(blockIdx.x);
    const int step = p.n_fixed ? cta_per_n : static_cast<int>(gridDim.x);
    const int count = p.n_fixed ? p.num_mtiles : p.num_tiles;
    auto tile_mn = [&](int t, int &mt, int &nt) {
        if (p.n_fixed) { mt = t; nt = my_nt; }
        else { mt = t / p.num_ntiles; nt = t - mt * p.num_ntiles; }
    };

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        uint32_t hit = 0, bit = 0;
        bool ok = true;
        // the resident filter slice of this CTA's N tile, once; issued after the first halo
        // so the first tile's operands arrive together
        auto load_resident_filter = [&]() {
            if (lane == 0) {
                const int n0 = my_nt * BN;
                mbar_arrive_expect_tx(bfull(0), p.num_kblk * Cfg::B_BYTES);
                for (int kb = 0; kb < p.num_kblk; ++kb) {
                    const int cb = kb / p.KK, tap = kb - cb * p.KK;
#pragma unroll
                    for (int h = 0; h < BN / 64; ++h)
                        tma_load_3d(sB + kb * Cfg::B_BYTES + h * Cfg::B_BOX_BYTES, &tmF, bfull(0), n0 + h * 64,
                                    cb * 64, tap);
                }
            }
            __syncwarp();
        };
        bool filter_issued = !BRES;
        for (int t = first; t < count && ok && !*abort_flag; t += step) {
            int mt, nt;
            tile_mn(t, mt, nt);
            const int P0 = mt * Cfg::BM;
            const int n0 = nt * BN;
            for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                const uint32_t hs = hit % p.HS, hph = (hit / p.HS) & 1u;
                if (!mbar_wait_warp_backoff(hempty(hs), hph ^ 1u, 64)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(hfull(hs), p.halo_bytes);
                    for (int bx = 0; bx < p.n_boxes; ++bx)
                        tma_load_2d(sH + hs * p.halo_bytes + bx * p.box_rows * 128, &tmX, hfull(hs), cb * 64,
                                    P0 + bx * p.box_rows);
                }
                __syncwarp();
                ++hit;
                if (!filter_issued) {
                    load_resident_filter();
                    filter_issued = true;
                }
                if (!BRES) {
                    for (int tap = 0; tap < p.KK; ++tap) {
                        const uint32_t bs = bit % p.BS, bph = (bit / p.BS) & 1u;
                        if (!mbar_wait_warp_backoff(bempty(bs), bph ^ 1u, 32)) { ok = false; break; }
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bfull(bs), Cfg::B_BYTES);
#pragma unroll
                            for (int h = 0; h < BN / 64; ++h)
                                tma_load_3d(sB + bs * Cfg::B_BYTES + h * Cfg::B_BOX_BYTES, &tmF, bfull(bs),
                                            n0 + h * 64, cb * 64, tap);
                        }
                        __syncwarp();
                        ++bit;
                    }
                }
            }
        }
        if (!filter_issued) load_resident_filter();
        if (!ok && lane == 0) fail();
        // Drain: every load issued has landed before the CTA may exit.
        if (BRES && !mbar_wait_warp(bfull(0), 0) && lane == 0) fail();
        for (uint32_t j = hit > (uint32_t)p.HS ? hit - p.HS : 0u; j < hit; ++j)
            if (!mbar_wait_warp(hfull(j % p.HS), (j / p.HS) & 1u)) { if (lane == 0) fail(); break; }
        if (!BRES)
            for (uint32_t j = bit > (uint32_t)p.BS ? bit - p.BS : 0u; j < bit; ++j)
                if (!mbar_wait_warp(bfull(j % p.BS), (j / p.BS) & 1u)) { if (lane == 0) fail(); break; }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // The whole warp walks the loop, converged; the MMAs and commits are predicated on one
        // elected lane (all of them, so that each commit tracks every MMA of the warp).
        const uint32_t leader = elect_one_sync();
        uint32_t hit = 0, bit = 0, local = 0;
        bool ok = true;
        if (BRES && !mbar_wait_warp(bfull(0), 0)) ok = false;
        for (int t = first; t < count && ok && !__any_sync(0xffffffffu, *abort_flag != 0); t += step, ++local) {
            const uint32_t b = local & 1u;
            // waiting here means the epilogue is the slower role: sleep between polls instead
            // of taking its issue slots
            if (!mbar_wait_warp_backoff(acce(b), ((local >> 1) & 1u) ^ 1u, 64)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * (Cfg::PARTS * BN);   // partial k at + k*BN
            for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                const uint32_t hs = hit % p.HS, hph = (hit / p.HS) & 1u;
                if (!mbar_wait_warp(hfull(hs), hph)) { ok = false; break; }
                tc_fence_after();
                const uint32_t halo = sH + hs * p.halo_bytes;
                if (BRES) {
                    // filter resident: the whole channel block (all taps x 4 K-steps) back to
                    // back; tap (ky, kx) reads the halo from row ky*W + kx on. Descriptors
                    // differ only in the start-address field (16-byte units): +2 per 16
                    // channels of A, +128 per 16 reduction rows of B
                    const uint64_t a0 = smem_desc_sw128(halo, 16, 1024);
                    uint64_t bd = smem_desc_sw128(sB + cb * p.KK * Cfg::B_BYTES, Cfg::B_BOX_BYTES, 1024);
                    // the tile's first MMA into each partial accumulator overwrites it
                    const uint32_t acc_first = cb != 0 ? 1u : 0u;
                    constexpr uint32_t P1 = Cfg::PARTS == 2 ? BN : 0u;   // the second partial's columns
                    uint32_t row = 0;
                    for (int ky = 0; ky < p.K; ++ky, row += p.W) {
                        for (int kx = 0; kx < p.K; ++kx, bd += Cfg::B_BYTES >> 4) {
                            const uint64_t ad = a0 + static_cast<uint64_t>((row + kx) * 8u);
                            const uint32_t first = (ky | kx) != 0 ? 1u : acc_first;
                            umma_f16_ss_if(d_tmem, ad, bd, Cfg::IDESC, first, leader);
                            umma_f16_ss_if(d_tmem + P1, ad + 2, bd + 128, Cfg::IDESC, Cfg::PARTS == 2 ? first : 1u,
                                           leader);
                            umma_f16_ss_if(d_tmem, ad + 4, bd + 256, Cfg::IDESC, 1u, leader);
                            umma_f16_ss_if(d_tmem + P1, ad + 6, bd + 384, Cfg::IDESC, 1u, leader);
                        }
                    }
                } else {
                    uint32_t row8 = 0;   // (ky*W + kx) * 8: A start of tap (ky, kx), 16-byte units
                    const uint32_t row_skip8 = static_cast<uint32_t>(p.W - p.K) * 8u;
                    const uint64_t a0 = smem_desc_sw128(halo, 16, 1024);
                    const uint64_t b0 = smem_desc_sw128(sB, Cfg::B_BOX_BYTES, 1024);
                    int kx = 0;
                    for (int tap = 0; tap < p.KK; ++tap) {
                        const uint32_t bs = bit % p.BS, bph = (bit / p.BS) & 1u;
                        if (!mbar_wait_warp(bfull(bs), bph)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t ad = a0 + row8;
                        const uint64_t bd = b0 + bs * (Cfg::B_BYTES >> 4);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint32_t part = Cfg::PARTS == 2 ? (kk & 1) : 0;
                            umma_f16_ss_if(d_tmem + part * BN, ad + 2 * kk, bd + 128 * kk, Cfg::IDESC,
                                           ((cb | tap) != 0 || kk >= Cfg::PARTS) ? 1u : 0u, leader);
                        }
                        umma_commit_if(bempty(bs), leader);
                        ++bit;
                        row8 += 8u;
                        if (++kx == p.K) { kx = 0; row8 += row_skip8; }
                    }
                }
                umma_commit_if(hempty(hs), leader);
                ++hit;
            }
            if (!ok) break;
            umma_commit_if(accf(b), leader);
        }
        __syncwarp();
        if (!ok && lane == 0) fail();
        umma_commit_if(done_bar, leader);
        if (!mbar_wait_warp(done_bar, 0) && lane == 0) fail();
    } else {
        // ------------------------------- Epilogue -----------------------------------
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int eg = (warp - 2) >> 2;     // which of the quarter's two warps: chunks eg, eg + 2, ...
        const uint32_t stage = sEpi + (warp - 2) * 4096;
        long long *rowoff = rowoff_all + (warp - 2) * 32;
        uint32_t local = 0;
        for (int t = first; t < count; t += step, ++local) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t b = local & 1u;
            if (!mbar_wait_warp_backoff(accf(b), (local >> 1) & 1u, 128)) { if (lane == 0) fail(); break; }
            tc_fence_after();
            int mt, nt;
            tile_mn(t, mt, nt);
            const int n0 = nt * BN;
            // this lane's row: flattened input position P -> output row, or -1 if dropped
            {
                const int P = mt * Cfg::BM + q * 32 + lane;
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
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * (Cfg::PARTS * BN);
#pragma unroll 1
            for (int h = eg; h < BN / 64; h += 2) {
                uint32_t r[4][16];
#pragma unroll
                for (int g = 0; g < 4; ++g) tmem_ld_32x32b_x16(t_row + h * 64 + g * 16, r[g]);
                if constexpr (Cfg::PARTS == 2) {
                    // the second partial accumulator, added once in fp32
                    uint32_t r2[4][16];
#pragma unroll
                    for (int g = 0; g < 4; ++g) tmem_ld_32x32b_x16(t_row + BN + h * 64 + g * 16, r2[g]);
                    tmem_wait_ld();
#pragma unroll
                    for (int g = 0; g < 4; ++g)
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            r[g][c] = __float_as_uint(__fadd_rn(__uint_as_float(r[g][c]), __uint_as_float(r2[g][c])));
                } else {
                    tmem_wait_ld();
                }
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
                        if (off >= 0 && in_bounds(off + col, 8, y_elems, kSiteHaloY, status)) {
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce(b));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

}  // namespace convb200
