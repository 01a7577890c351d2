// Dense and grouped NHWC forward convolution with zero padding at stride 1, as an implicit GEMM
// over a padded input band that one tensor copy stages per tile ("padded halo" tiles).
//
// The operation is the general entry's (CMU DLSys Lecture 14 notes, section 1 for the index
// contract; "Convolution Is Wx+b Moving Across a Signal", "Why variants matter" and "Find the
// same sum in CKE's C kernels" for zero padding, dilation, channel groups and the bias): output
// (n, y, x, o) of group g = o / Cout_g sums X[n, y + i*dh - ph, x + j*dw - pw, g*Cin_g + c] *
// F[i, j, c, o] over the taps and the group's channels, positions outside the image reading
// zero, plus the fp32 bias before the single bf16 rounding.
//
// A tile is a band of Rout output rows x Wt output columns of one image. Its inputs are the
// (Rout + dh*(KH-1)) x (Wt + dw*(KW-1)) window starting at (y0 - ph, x0 - pw): one 4-D tensor
// copy per 64-channel block, whose box may start above or left of the image and run past its
// end (the copy engine writes zeros there -- the padding), lands in shared memory as rows of
// Wbox = Wt + dw*(KW-1) pixels, 128 bytes (64 channels) each. Flatten that window: output
// (ry, rx) of the tile is GEMM row r = ry*Wbox + rx, and tap (i, j) reads window row
// r + i*dh*Wbox + j*dw -- a fixed shift for the whole tile, so the A operand of every tap is
// the same shared-memory tile read from that row on, as in the unpadded halo kernel. Rows with
// rx >= Wt (the last dw*(KW-1) columns of each window row) and rows past Rout*Wbox are
// computed and dropped. Each input pixel of a tile is loaded once (the im2col kernel loads it
// once per tap).
//
// The filter slice of the CTA's (group, 64- or 128-column tile) stays resident in shared memory;
// each CTA keeps one such slice and walks the spatial tiles. Consecutive MMAs alternate
// between two partial accumulators (summed once in the epilogue).
//
// Roles in one persistent CTA of 10 warps (role loops walked by whole converged warps):
//   warp 0      TMA: the resident filter once, then one padded window per (tile, channel
//               block) into a ring of HS slots;
//   warp 1      TMEM allocation; tcgen05.mma M=128, N=BN, K=16 (predicated on an elected lane);
//   warps 2..9  epilogue: tcgen05.ld, the two partials and the bias added in fp32, round to
//               bf16, per-warp swizzled staging, coalesced 16-byte stores of the valid rows.
#pragma once
#include <cuda_bf16.h>

#include "dense_halo.cuh"   // halo_pack_bf16x2, st_shared_v4
#include "ptx.cuh"

namespace convb200 {

struct DenseHaloPadParams {
    int H, W, Ho, Wo;
    int Cout;            // all output channels (the row pitch of Y)
    int Cin_g, Cout_g;   // channels of one group
    int KH, KW, dh, dw, ph, pw;
    int Rout, Wt, Wbox, Rin;   // output rows / columns per tile; window width and rows
    int n_rb, n_cb;            // row and column bands per image
    int num_spatial;           // N * n_rb * n_cb
    int num_cblk;              // Cin_g / 64
    int KK, num_kblk;          // KH*KW; KK * num_cblk resident filter slots
    int num_nt;                // column tiles per group: ceil(Cout_g / BN)
    int num_gn;                // groups * num_nt: the CTA's fixed (group, column tile)
    int box_bytes;             // Rin * Wbox * 128: one window (the TMA box)
    int halo_bytes;            // window slot (at least box_bytes and the last tap's reach)
    int HS;                    // window ring slots
    int b_region;              // num_kblk * B_BYTES
    const float *bias;         // per output channel (all Cout) or null
    long long y_elems;         // N * Ho * Wo * Cout (bounds checks of the debug build)
};

template <int BN_>
struct DenseHaloPadCfg {
    static constexpr int BN = BN_;
    static constexpr int BM = 128;
    static constexpr int B_BOX_BYTES = 64 * 64 * 2;   // 64 reduction rows x 64 channels
    static constexpr int B_BYTES = 64 * BN * 2;       // one (tap, channel block) filter slot
    static constexpr int NUM_EPI = 8;
    static constexpr int THREADS = 64 + 32 * NUM_EPI;
    static constexpr int EPI_BYTES = NUM_EPI * 32 * 128;
    static constexpr int MAX_RING = 8;
    static constexpr int NUM_BARS = 2 * MAX_RING + 1 /*filter*/ + 4 /*acc*/ + 1 /*done*/;
    static constexpr int PARTS = 2;
    static constexpr int TMEM_COLS = 2 * PARTS * BN;
    static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*B MN-major*/ true);
    static constexpr int FIXED_BYTES = 1024 + EPI_BYTES + NUM_BARS * 8 + NUM_EPI * 32 * 8 + 16;
    static_assert(BN == 64 || BN == 128, "BN");
};

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        :
        : "r"(dst), "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
dense_halo_pad_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmF,
                      __nv_bfloat16 *__restrict__ Y, const DenseHaloPadParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int BN = Cfg::BN;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;   // 1024-B alignment for the swizzle
    uint8_t *smem = smem_raw + (base - raw_base);

    const uint32_t sB = base;                                 // resident filter
    const uint32_t sH = base + p.b_region;                    // window ring
    const uint32_t epi_off = p.b_region + p.HS * p.halo_bytes;
    const uint32_t sEpi = base + epi_off;
    const uint32_t bars = sEpi + Cfg::EPI_BYTES;
    constexpr int R = Cfg::MAX_RING;
    auto hfull = [&](int s) { return bars + 8u * s; };
    auto hempty = [&](int s) { return bars + 8u * (R + s); };
    const uint32_t bfull = bars + 8u * (2 * R);
    auto accf = [&](int b) { return bars + 8u * (2 * R + 1 + b); };
    auto acce = [&](int b) { return bars + 8u * (2 * R + 3 + b); };
    const uint32_t done_bar = bars + 8u * (2 * R + 5);
    long long *rowoff_all = reinterpret_cast<long long *>(smem + epi_off + Cfg::EPI_BYTES + Cfg::NUM_BARS * 8);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(rowoff_all + Cfg::NUM_EPI * 32);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < R; ++s) {
            mbar_init(hfull(s), 1);
            mbar_init(hempty(s), 1);
        }
        mbar_init(bfull, 1);
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
    // the CTA's fixed (group, column tile) and its spatial tiles
    const int gn = static_cast<int>(blockIdx.x) % p.num_gn;
    const int grp = gn / p.num_nt;
    const int nt = gn - grp * p.num_nt;
    const int first = static_cast<int>(blockIdx.x) / p.num_gn;
    const int step = static_cast<int>(gridDim.x) / p.num_gn;
    const int col0 = grp * p.Cout_g + nt * BN;   // the tile's first output channel
    // spatial tile t -> image, first output row and column
    auto tile_at = [&](int t, int &n, int &y0, int &x0) {
        const int per_img = p.n_rb * p.n_cb;
        n = t / per_img;
        const int rem = t - n * per_img;
        const int rb = rem / p.n_cb;
        y0 = rb * p.Rout;
        x0 = (rem - rb * p.n_cb) * p.Wt;
    };

    if (warp == 0) {
        // ------------------------------- TMA producer -------------------------------
        uint32_t hit = 0;
        bool ok = true;
        bool filter_issued = false;
        for (int t = first; t < p.num_spatial && ok && !*abort_flag; t += step) {
            int n, y0, x0;
            tile_at(t, n, y0, x0);
            for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                const uint32_t hs = hit % p.HS, hph = (hit / p.HS) & 1u;
                if (!mbar_wait_warp_backoff(hempty(hs), hph ^ 1u, 64)) { ok = false; break; }
                if (lane == 0) {
                    // the padded window: channels of the group's block cb, columns from x0 - pw,
                    // rows from y0 - ph (zeros outside the image)
                    mbar_arrive_expect_tx(hfull(hs), static_cast<uint32_t>(p.box_bytes));
                    tma_load_4d(sH + hs * p.halo_bytes, &tmX, hfull(hs), grp * p.Cin_g + cb * 64, x0 - p.pw,
                                y0 - p.ph, n);
                }
                __syncwarp();
                ++hit;
                if (!filter_issued) {
                    // the resident filter slice, once, after the first window
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bfull, static_cast<uint32_t>(p.num_kblk * Cfg::B_BYTES));
                        for (int kb = 0; kb < p.num_kblk; ++kb) {
                            const int c = kb / p.KK, tap = kb - c * p.KK;
#pragma unroll
                            for (int h = 0; h < BN / 64; ++h)
                                tma_load_3d(sB + kb * Cfg::B_BYTES + h * Cfg::B_BOX_BYTES, &tmF, bfull,
                                            col0 + h * 64, c * 64, tap);
                        }
                    }
                    __syncwarp();
                    filter_issued = true;
                }
            }
        }
        if (!ok && lane == 0) fail();
        // Drain: every load issued has landed before the CTA may exit.
        if (filter_issued && !mbar_wait_warp(bfull, 0) && lane == 0) fail();
        for (uint32_t j = hit > (uint32_t)p.HS ? hit - p.HS : 0u; j < hit; ++j)
            if (!mbar_wait_warp(hfull(j % p.HS), (j / p.HS) & 1u)) { if (lane == 0) fail(); break; }
    } else if (warp == 1) {
        // ------------------------------- MMA issuer ---------------------------------
        // converged warp, MMAs and commits predicated on one elected lane
        const uint32_t leader = elect_one_sync();
        uint32_t hit = 0, local = 0;
        bool ok = true;
        bool have_filter = false;
        for (int t = first; t < p.num_spatial && ok && !__any_sync(0xffffffffu, *abort_flag != 0);
             t += step, ++local) {
            const uint32_t b = local & 1u;
            if (!mbar_wait_warp_backoff(acce(b), ((local >> 1) & 1u) ^ 1u, 64)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * (Cfg::PARTS * BN);   // partial k at + k*BN
            for (int cb = 0; cb < p.num_cblk && ok; ++cb) {
                const uint32_t hs = hit % p.HS, hph = (hit / p.HS) & 1u;
                if (!mbar_wait_warp(hfull(hs), hph)) { ok = false; break; }
                if (!have_filter) {
                    if (!mbar_wait_warp(bfull, 0)) { ok = false; break; }
                    have_filter = true;
                }
                tc_fence_after();
                // tap (i, j) reads the window from row i*dh*Wbox + j*dw on (start field in 16-byte
                // units: +8 per 128-byte row, +2 per 16 channels); B +128 per 16 reduction rows
                const uint64_t a0 = smem_desc_sw128(sH + hs * p.halo_bytes, 16, 1024);
                uint64_t bd = smem_desc_sw128(sB + cb * p.KK * Cfg::B_BYTES, Cfg::B_BOX_BYTES, 1024);
                const uint32_t acc_first = cb != 0 ? 1u : 0u;
                for (int i = 0; i < p.KH; ++i) {
                    for (int j = 0; j < p.KW; ++j, bd += Cfg::B_BYTES >> 4) {
                        const uint64_t ad = a0 + static_cast<uint64_t>((i * p.dh * p.Wbox + j * p.dw) * 8);
                        const uint32_t first_mma = (i | j) != 0 ? 1u : acc_first;
                        umma_f16_ss_if(d_tmem, ad, bd, Cfg::IDESC, first_mma, leader);
                        umma_f16_ss_if(d_tmem + BN, ad + 2, bd + 128, Cfg::IDESC, first_mma, leader);
                        umma_f16_ss_if(d_tmem, ad + 4, bd + 256, Cfg::IDESC, 1u, leader);
                        umma_f16_ss_if(d_tmem + BN, ad + 6, bd + 384, Cfg::IDESC, 1u, leader);
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
        for (int t = first; t < p.num_spatial; t += step, ++local) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            const uint32_t b = local & 1u;
            if (!mbar_wait_warp_backoff(accf(b), (local >> 1) & 1u, 128)) { if (lane == 0) fail(); break; }
            tc_fence_after();
            int n, y0, x0;
            tile_at(t, n, y0, x0);
            // this lane's GEMM row r -> output (y0 + ry, x0 + rx), or -1 if dropped
            {
                const int r = q * 32 + lane;
                const int ry = r / p.Wbox;
                const int rx = r - ry * p.Wbox;
                long long off = -1;
                if (ry < p.Rout && rx < p.Wt && y0 + ry < p.Ho && x0 + rx < p.Wo)
                    off = ((static_cast<long long>(n) * p.Ho + y0 + ry) * p.Wo + x0 + rx) * p.Cout + col0;
                rowoff[lane] = off;
            }
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * (Cfg::PARTS * BN);
#pragma unroll 1
            for (int h = eg; h < BN / 64; h += 2) {
                const uint32_t row_addr = stage + lane * 128;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    // one 16-column chunk: both partials, then the bias -- fp32 additions before
                    // the single rounding
                    uint32_t r[16], r2[16];
                    tmem_ld_32x32b_x16(t_row + h * 64 + g * 16, r);
                    tmem_ld_32x32b_x16(t_row + BN + h * 64 + g * 16, r2);
                    tmem_wait_ld();
                    const int colc = nt * BN + h * 64 + g * 16;   // the chunk's first column in the group
                    float v[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) v[c] = __fadd_rn(__uint_as_float(r[c]), __uint_as_float(r2[c]));
                    if (p.bias && colc + 16 <= p.Cout_g &&
                        in_bounds(static_cast<long long>(grp) * p.Cout_g + colc, 16, 1LL * p.Cout, kSiteHaloPadBias,
                                  status)) {
                        // a whole chunk inside the group: four 16-byte loads (the host requires a
                        // 16-byte aligned bias; grp * Cout_g + colc is a multiple of 8)
                        const float4 *b4 = reinterpret_cast<const float4 *>(p.bias + grp * p.Cout_g + colc);
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            const float4 bv = __ldg(b4 + c4);
                            v[4 * c4] = __fadd_rn(v[4 * c4], bv.x);
                            v[4 * c4 + 1] = __fadd_rn(v[4 * c4 + 1], bv.y);
                            v[4 * c4 + 2] = __fadd_rn(v[4 * c4 + 2], bv.z);
                            v[4 * c4 + 3] = __fadd_rn(v[4 * c4 + 3], bv.w);
                        }
                    } else if (p.bias) {
                        // the group's last, partial chunk: the columns inside the group only
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            if (colc + c < p.Cout_g &&
                                in_bounds(static_cast<long long>(grp) * p.Cout_g + colc + c, 1, 1LL * p.Cout,
                                          kSiteHaloPadBias, status))
                                v[c] = __fadd_rn(v[c], __ldg(p.bias + grp * p.Cout_g + colc + c));
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const uint32_t c = g * 2 + cc;
                        const float *w = &v[cc * 8];
                        st_shared_v4(row_addr + ((c ^ (lane & 7)) << 4), halo_pack_bf16x2(w[0], w[1]),
                                     halo_pack_bf16x2(w[2], w[3]), halo_pack_bf16x2(w[4], w[5]),
                                     halo_pack_bf16x2(w[6], w[7]));
                    }
                }
                __syncwarp();
                // coalesced stores: 8 lanes per row, 4 rows per instruction; columns past the
                // group's Cout_g are dropped
                const int colg = nt * BN + h * 64 + (lane & 7) * 8;
                if (colg < p.Cout_g) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = i * 4 + (lane >> 3);
                        const long long off = rowoff[rr];
                        if (off >= 0 && in_bounds(off + h * 64 + (lane & 7) * 8, 8, p.y_elems, kSiteHaloPadY, status)) {
                            uint32_t a, bb, c, d;
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(a), "=r"(bb), "=r"(c), "=r"(d)
                                         : "r"(stage + rr * 128 + ((((lane & 7) ^ (rr & 7))) << 4)));
                            uint4 *dst = reinterpret_cast<uint4 *>(Y + off + h * 64 + (lane & 7) * 8);
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
