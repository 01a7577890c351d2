// Dense NHWC forward convolution for narrow layers (Cout <= 64, 2 <= K <= 4): the halo
// implicit GEMM with the filter's column taps folded into the MMA's N dimension.
//
// Same operation and flattened-row addressing as dense_halo.cuh (CMU DLSys Lecture 14 notes,
// section 1 "Fix the index contract before optimizing it" for the definition, section 2 "Move
// the channel contraction into matrix multiplication" for the per-tap matrix products). With
// Cout = 64 every tap of the halo kernel is an M=128, N=64 tcgen05.mma, which sm_100a issues at
// about half the tensor rate of N >= 128. Here the K column taps j of one filter row i share
// one MMA of N = 64*K instead:
//
//     D_j[m, o] = sum_i sum_c X[m + i*W, c] * F[i, j, c, o]      (one MMA per (i, 16 channels))
//     Y[m, o]   = D_0[m, o] + D_1[m + 1, o] + ... + D_{K-1}[m + K-1, o]
//
// B of that MMA is the K filter slots (i, 0..K-1) side by side, which the resident filter
// already holds contiguously (one 64-column MN-major box per slot), so the descriptor's
// leading-byte offset steps from one tap to the next. The row shift m + j moves from the A
// operand to the epilogue: a TMEM lane holds one row, so lane r adds group j of row r + j,
// taken from the lane j below by a warp shuffle, or -- for the last K-1 lanes of a warp --
// from the next warp's first lanes through a small shared-memory exchange. A tile computes 128
// rows of D and keeps the first 128 - (K-1) rows of Y; consecutive tiles overlap by K-1 rows.
//
// Summation order per output: fp32 tensor-core sums over (i, c) inside each group j, then the
// groups added in j order in fp32, one rounding to bf16 -- a different order from the other
// kernels, within the same error bound.
//
// Roles: warp 0 TMA, warp 1 TMEM + MMA, then the epilogue warps: 64/CW per TMEM lane quarter,
// CW output channels each (CW = 16: 16 warps, four per SM sub-partition, hiding each other's
// TMEM-load, shuffle and store latencies); the filter is always resident here.
#pragma once
#include <cuda_bf16.h>

#include "dense_halo.cuh"
#include "dense_tc.cuh"
#include "depthwise.cuh"   // FastDiv
#include "ptx.cuh"

namespace convb200 {

struct DenseFoldParams {
    int rows;          // N * H * W: flattened input positions
    int H, W, Ho, Wo;
    int K, KK, Cout;
    int num_cblk;      // ceil(Cin / 64)
    int num_kblk;      // KK * num_cblk filter slots, channel block outer, tap (i, j) inner
    int halo_rows, box_rows, n_boxes, halo_bytes;
    int num_tiles;     // ceil(rows / (128 - (K-1)))
    int HS;            // halo ring slots
    int b_region;      // bytes of the resident filter
    FastDiv div_w, div_h;
};

template <int KF, int CW_ = 16>
struct DenseFoldCfg {
    static constexpr int K = KF;
    static constexpr int NF = 64 * KF;                 // MMA N: K groups of 64 columns
    static constexpr int BM = 128;
    static constexpr int TM = BM - (KF - 1);           // output rows kept per tile
    static constexpr int SLOT_BYTES = 64 * 64 * 2;     // one (tap, channel block) filter slot
    static constexpr int CW = CW_;                     // output channels per epilogue warp
    static constexpr int G = CW / 16;                  // 16-column TMEM chunks per warp
    static constexpr int CPR = CW / 8;                 // 16-byte chunks per staged row
    static constexpr int RPL = 64 / CW;                // staged rows per 128 bytes
    static constexpr int NUM_EPI = 4 * (64 / CW);      // epilogue warps: 4 lane quarters x 64/CW column slices
    static constexpr int THREADS = 64 + 32 * NUM_EPI;
    static constexpr int EPI_BYTES = NUM_EPI * 32 * CW * 2;   // per-warp 32 rows x CW channels staging
    static constexpr int MAX_RING = 8;
    // exchange: lanes 0..j-1 of group j (j >= 1), CW floats each, per warp and tile parity
    static constexpr int XCH_FLOATS = KF * (KF - 1) / 2 * CW;
    static constexpr int XCH_BYTES = 2 * NUM_EPI * XCH_FLOATS * 4;
    static constexpr int NUM_BARS = 2 * MAX_RING /*halo*/ + 4 /*filter rows*/ + 4 /*acc*/ + 2 /*xch*/ + 1;
    static constexpr int TMEM_COLS = 2 * NF <= 256 ? 256 : 512;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BM, NF, /*B MN-major*/ true);
    static constexpr int FIXED_BYTES = 1024 + EPI_BYTES + XCH_BYTES + NUM_BARS * 8 + NUM_EPI * 32 * 8 + 16;
    static_assert(KF >= 2 && KF <= 4, "N = 64*K must stay within 256");
    static_assert(CW == 16 || CW == 32, "CW");
};

// st.shared.v4 executed only where pred != 0 (predicated, no branch)
__device__ __forceinline__ void st_shared_v4_if(uint32_t pred, uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                                uint32_t d) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, %0, 0; @p st.shared.v4.b32 [%1], {%2, %3, %4, %5}; }" ::"r"(pred),
                 "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
dense_fold_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmF,
                  __nv_bfloat16 *__restrict__ Y, const DenseFoldParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int K = Cfg::K;
    constexpr int NF = Cfg::NF;
    constexpr int TM = Cfg::TM;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;   // 1024-B alignment for the swizzle
    uint8_t *smem = smem_raw + (base - raw_base);

    const uint32_t sB = base;                                 // resident filter
    const uint32_t sH = base + p.b_region;                    // halo ring
    const uint32_t epi_off = p.b_region + p.HS * p.halo_bytes;
    const uint32_t sEpi = base + epi_off;
    const uint32_t sX = sEpi + Cfg::EPI_BYTES;                 // row-shift exchange
    const uint32_t bars = sEpi + Cfg::EPI_BYTES + Cfg::XCH_BYTES;
    constexpr int R = Cfg::MAX_RING;
    auto hfull = [&](int s) { return bars + 8u * s; };
    auto hempty = [&](int s) { return bars + 8u * (R + s); };
    auto bfull = [&](int i) { return bars + 8u * (2 * R + i); };   // filter row i resident
    auto accf = [&](int b) { return bars + 8u * (2 * R + 4 + b); };
    auto acce = [&](int b) { return bars + 8u * (2 * R + 6 + b); };
    auto xbar = [&](int b) { return bars + 8u * (2 * R + 8 + b); };
    const uint32_t done_bar = bars + 8u * (2 * R + 10);
    const uint32_t rowoff_all = sEpi + Cfg::EPI_BYTES + Cfg::XCH_BYTES + Cfg::NUM_BARS * 8;   // s64 per row
    uint32_t *tmem_holder =
        reinterpret_cast<uint32_t *>(smem + epi_off + Cfg::EPI_BYTES + Cfg::XCH_BYTES + Cfg::NUM_BARS * 8 +
                                     Cfg::NUM_EPI * 32 * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < R; ++s) {
            mbar_init(hfull(s), 1);
            mbar_init(hempty(s), 1);
        }
        for (int i = 0; i < K; ++i) mbar_init(bfull(i), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf(b), 1);
            mbar_init(acce(b), Cfg::NUM_EPI);   // one arrival per epilogue warp
            mbar_init(xbar(b), Cfg::NUM_EPI);
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
    const int first = static_cast<int>(blockIdx.x);
    const int step = static_cast<int>(gridDim.x);

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        uint32_t hit = 0;
        bool ok = true, filter_issued = false;
        // the filter row by row, each with its own barrier, so the first tile's MMAs for
        // row 0 start while rows 1.. are still in flight
        auto load_filter = [&]() {
            if (lane == 0) {
                for (int i = 0; i < K; ++i) {
                    mbar_arrive_expect_tx(bfull(i), p.num_cblk * K * Cfg::SLOT_BYTES);
                    for (int cb = 0; cb < p.num_cblk; ++cb)
                        for (int j = 0; j < K; ++j)
                            tma_load_3d(sB + (cb * p.KK + i * K + j) * Cfg::SLOT_BYTES, &tmF, bfull(i), 0, cb * 64,
                                        i * K + j);
                }
            }
            __syncwarp();
        };
        for (int t = first; t < p.num_tiles && ok && !*abort_flag; t += step) {
            const int P0 = t * TM;
            for (int cb = 0; cb < p.num_cblk; ++cb) {
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
                if (!filter_issued) {   // after the first halo, so the first tile's operands arrive together
                    load_filter();
                    filter_issued = true;
                }
            }
        }
        if (!filter_issued) load_filter();
        if (!ok && lane == 0) fail();
        // Drain: every load issued has landed before the CTA may exit.
        for (int i = 0; i < K; ++i)
            if (!mbar_wait_warp(bfull(i), 0)) { if (lane == 0) fail(); break; }
        for (uint32_t j = hit > (uint32_t)p.HS ? hit - p.HS : 0u; j < hit; ++j)
            if (!mbar_wait_warp(hfull(j % p.HS), (j / p.HS) & 1u)) { if (lane == 0) fail(); break; }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // The whole warp walks the loop, converged; the MMAs and commits are predicated on one
        // elected lane (all of them, so that each commit tracks every MMA of the warp).
        const uint32_t leader = elect_one_sync();
        uint32_t hit = 0, local = 0;
        bool ok = mbar_wait_warp(bfull(0), 0);
        for (int t = first; t < p.num_tiles && ok && !__any_sync(0xffffffffu, *abort_flag != 0);
             t += step, ++local) {
            const uint32_t b = local & 1u;
            // the epilogue is the slower role: sleep between polls instead of taking its issue slots
            if (!mbar_wait_warp_backoff(acce(b), ((local >> 1) & 1u) ^ 1u, 64)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * NF;
            for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                const uint32_t hs = hit % p.HS, hph = (hit / p.HS) & 1u;
                if (!mbar_wait_warp(hfull(hs), hph)) { ok = false; break; }
                tc_fence_after();
                // filter row i reads the halo from row i*W on (start field in 16-byte units: +8
                // per 128-byte row, +2 per 16 channels); B spans the K slots (i, 0..K-1), 8 KB
                // apart (the leading-byte offset), +128 per 16 channels
                const uint64_t a0 = smem_desc_sw128(sH + hs * p.halo_bytes, 16, 1024);
#pragma unroll
                for (int i = 0; i < K; ++i) {
                    // the first tile's filter rows arrive one by one
                    if (local == 0 && cb == 0 && i > 0) {
                        if (!mbar_wait_warp(bfull(i), 0)) { ok = false; break; }
                        tc_fence_after();
                    }
                    const uint64_t ad = a0 + static_cast<uint64_t>(i * p.W * 8);
                    const uint64_t bd = smem_desc_sw128(sB + (cb * p.KK + i * K) * Cfg::SLOT_BYTES,
                                                        Cfg::SLOT_BYTES, 1024);
                    umma_f16_ss_if(d_tmem, ad, bd, Cfg::IDESC, (cb | i) != 0 ? 1u : 0u, leader);
                    umma_f16_ss_if(d_tmem, ad + 2, bd + 128, Cfg::IDESC, 1u, leader);
                    umma_f16_ss_if(d_tmem, ad + 4, bd + 256, Cfg::IDESC, 1u, leader);
                    umma_f16_ss_if(d_tmem, ad + 6, bd + 384, Cfg::IDESC, 1u, leader);
                }
                if (!ok) break;
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
        // warp e = warp - 2: TMEM lane quarter q = warp % 4 (the quarter a warp may access),
        // output channels CW*h .. CW*h + CW - 1 with h = e / 4
        constexpr int CW = Cfg::CW, G = Cfg::G, CPR = Cfg::CPR, RPL = Cfg::RPL;
        const int e = warp - 2;
        const int q = warp & 3;
        const int h = e >> 2;
        const uint32_t stage = sEpi + e * (32 * CW * 2);
        const uint32_t rowoff = rowoff_all + e * 32 * 8;
        uint32_t local = 0;
        for (int t = first; t < p.num_tiles; t += step, ++local) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t b = local & 1u, par = local & 1u;
            if (!mbar_wait_warp_backoff(accf(b), (local >> 1) & 1u, 128)) { if (lane == 0) fail(); break; }
            tc_fence_after();
            // this lane's row r of the tile: an output if r < TM and (y, x) is a valid origin
            {
                const int r = q * 32 + lane;
                const int P = t * TM + r;
                long long off = -1;
                if (r < TM && P < p.rows) {
                    const int row = fdiv(P, p.div_w);
                    const int x = P - row * p.W;
                    const int n = fdiv(row, p.div_h);
                    const int y = row - n * p.H;
                    if (x < p.Wo && y < p.Ho)
                        off = ((static_cast<long long>(n) * p.Ho + y) * p.Wo + x) * p.Cout;
                }
                asm volatile("st.shared.s64 [%0], %1;" ::"r"(rowoff + 8u * lane), "l"(off) : "memory");
            }
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * NF + h * CW;
            // one round trip to TMEM: all K groups of this warp's CW columns
            uint32_t d[K][G][16];
#pragma unroll
            for (int j = 0; j < K; ++j)
#pragma unroll
                for (int g = 0; g < G; ++g) tmem_ld_32x32b_x16(t_row + j * 64 + g * 16, d[j][g]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce(b));   // accumulator read: the MMA warp may reuse it
            // publish lanes 0..j-1 of groups j >= 1 for the warp of the quarter above
            if (q > 0) {
                const uint32_t my_x = sX + 4u * ((par * 4 + q) * (64 / CW) + h) * Cfg::XCH_FLOATS;
#pragma unroll
                for (int j = 1; j < K; ++j) {
                    const uint32_t pub = lane < j ? 1u : 0u;   // predicated stores: no divergent branch
                    const uint32_t dst = my_x + 4u * (j * (j - 1) / 2 + (lane < j ? lane : 0)) * CW;
#pragma unroll
                    for (int g = 0; g < G; ++g)
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            st_shared_v4_if(pub, dst + 16u * (g * 4 + c), d[j][g][4 * c], d[j][g][4 * c + 1],
                                            d[j][g][4 * c + 2], d[j][g][4 * c + 3]);
                }
            }
            __syncwarp();   // the lanes' exchange stores are ordered before lane 0's release
            if (lane == 0) mbar_arrive(xbar(par));
            const uint32_t next_x = sX + 4u * ((par * 4 + (q < 3 ? q + 1 : q)) * (64 / CW) + h) * Cfg::XCH_FLOATS;
            const bool xok = mbar_wait_warp_backoff(xbar(par), (local >> 1) & 1u, 32);
            const uint32_t row_addr = stage + lane * (CW * 2);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float y[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) y[c] = __uint_as_float(d[0][g][c]);
#pragma unroll
                for (int j = 1; j < K; ++j) {
                    // lanes 32-j .. 31 take row r + j from the next quarter's exchange; every lane
                    // loads (a valid address, mostly a broadcast) and selects, so nothing diverges
                    const bool from_next = lane + j >= 32;
                    const bool from_smem = from_next && q < 3 && xok;
                    const uint32_t src = next_x + 4u * ((j * (j - 1) / 2 + (from_next ? lane + j - 32 : 0)) * CW + g * 16);
                    float xv[16];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const float4 t4 = ld_shared_f4(src + 16u * c4);
                        xv[4 * c4] = t4.x; xv[4 * c4 + 1] = t4.y; xv[4 * c4 + 2] = t4.z; xv[4 * c4 + 3] = t4.w;
                    }
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const float sv = __shfl_down_sync(0xffffffffu, __uint_as_float(d[j][g][c]), j);
                        const float v = from_next ? (from_smem ? xv[c] : 0.0f) : sv;
                        y[c] = __fadd_rn(y[c], v);
                    }
                }
                // 2*CW-byte staging rows, 16-byte chunks swizzled by (row / RPL) % CPR:
                // conflict-free writes (one row per lane) and reads (RPL rows per 8 lanes)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const uint32_t c = g * 2 + cc;
                    const float *v = &y[cc * 8];
                    st_shared_v4(row_addr + ((c ^ ((lane / RPL) % CPR)) << 4), halo_pack_bf16x2(v[0], v[1]),
                                 halo_pack_bf16x2(v[2], v[3]), halo_pack_bf16x2(v[4], v[5]),
                                 halo_pack_bf16x2(v[6], v[7]));
                }
            }
            if (!xok) { if (lane == 0) fail(); break; }
            __syncwarp();
            // coalesced stores: CPR lanes per staged row, 32 / CPR rows per instruction
            const int cc = lane % CPR;
            const int col = h * CW + cc * 8;
            if (col < p.Cout) {
                const long long y_elems = 1LL * (p.rows / (p.H * p.W)) * p.Ho * p.Wo * p.Cout;   // bounds checks (debug build)
#pragma unroll
                for (int i = 0; i < CPR; ++i) {
                    const int rr = i * (32 / CPR) + lane / CPR;
                    long long off;
                    asm volatile("ld.shared.s64 %0, [%1];" : "=l"(off) : "r"(rowoff + 8u * rr));
                    if (off >= 0 && in_bounds(off + col, 8, y_elems, kSiteFoldY, status)) {
                        uint32_t a, bb, c, dd;
                        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(a), "=r"(bb), "=r"(c), "=r"(dd)
                                     : "r"(stage + rr * (CW * 2) + ((cc ^ ((rr / RPL) % CPR)) << 4)));
                        *reinterpret_cast<uint4 *>(Y + off + col) = make_uint4(a, bb, c, dd);
                    }
                }
            }
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
}

}  // namespace convb200
