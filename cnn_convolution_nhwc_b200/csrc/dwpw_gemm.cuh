// Depthwise K x K followed by pointwise 1 x 1, fused, for small square images (7x7, 14x14):
// the channel-mixing GEMM transposed so that the depthwise stage keeps its row-wise register
// window.
//
// Same block and contract as dwpw.cuh ("Convolution Is Wx+b Moving Across a Signal", section
// "Why variants matter"; the depthwise stage is the OneModel "Depthwise convolution" contract of
// section "What each output is", multiplier 1; the intermediate is rounded to bfloat16 once; the
// pointwise sum is float32 with the pointwise bias added once), for stride 1, "same" padding
// (K-1)/2 and dilation 1. Per image n the pointwise pass is
//     Y_n[o, p] = sum_c F[c, o] * bf16(d[n, c, p]),   p = oy*W + ox,
// a GEMM with M = Cout (A = F read as an MN-major operand straight from its [C][Cout] layout),
// N = the image's pixels (B = the depthwise outputs, MN-major: pixels contiguous) and K = C.
// Written this way the depthwise outputs of one channel -- neighbouring pixels of one plane --
// land next to each other in the B tile, so the depthwise stage is the plane-wise loop of the
// standalone kernels: a thread owns a strip of two neighbouring output columns over a run of
// rows, keeps the K input rows it needs as packed pairs in registers (each input value loaded
// once per run), and applies each tap to both outputs with one f32x2 instruction. TMEM lane o
// then holds output channel o's row of pixels, which is exactly one contiguous range of the NCHW
// output plane y[n, o, :, :].
//
// Work layout, two forms. Channel split: one image per cluster of S CTAs (S = 2 when there are
// at least two channel blocks: rank k takes blocks k, k + S, ...). Row split (14x14, the
// default there): two CTAs per image, no cluster; CTA 2k + h computes output rows 7h .. 7h + 6
// for every channel, so each output's whole channel sum stays in one CTA's accumulator and in
// the channel order of the one-CTA form (the same bits), while the image's MMA N halves
// (208 -> 112 columns) and twice as many CTAs share the images. 16 warps per CTA, the
// channels in blocks of CB. Per block:
//   * x: the block's CB planes of the image are one contiguous range of x, staged into a
//     2-slot ring two blocks ahead: at 14x14 one 2-D tensor copy viewing x as [N*C][P] whose
//     box is wider than a plane (a padded pitch: fewer bank conflicts in the row loads; the
//     row-split form copies a 136-float window holding the input rows its half reads), at
//     7x7 one bulk copy of the whole range; the block's taps arrive by a bulk copy on the same
//     barrier;
//   * F: the block's CB x Cout filter rows, 64-column boxes by TMA into a 3-slot ring (two
//     blocks ahead); columns past Cout arrive as zeros;
//   * every thread computes its strip (zeros padding, exact or fast mode, the depthwise bias),
//     rounds to bf16 and writes the values into the B tile (128-byte swizzled, 64 pixels per
//     box); channels past C write zeros;
//   * after the CTA barrier that publishes the B tile, the issuing warp (at 14x14 the
//     sixteenth warp, which has no depthwise work; at 7x7 warp 0) issues the block's MMAs
//     (M = 128 per 128 output channels, N = pixels rounded up to 16, K = 16) into the image's
//     TMEM accumulators and commits; the B slot is rewritten two blocks later, after that
//     commit.
// After the last block all 16 warps read the accumulators (warp w: TMEM lane quarter w % 4, a
// quarter of the 16-column chunks; the row split stores its 98 pixels of each plane). With S = 2, 16-column chunk j belongs to rank j % 2: each
// rank writes its partial of the chunks it does not own into the owner's receive area through
// distributed shared memory, and the owner adds the two partials (one IEEE addition, so the
// result does not depend on which rank adds), the pointwise bias, and stores y.
//
// Every wait is bounded; a wait that runs out sets the status word and the CTA stops its work
// together (barrier-wide OR), but keeps taking every CTA and cluster barrier of its remaining
// images, so its peer is never left waiting; it drains the copies it issued and waits for its
// MMAs before TMEM is freed.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>
#include <type_traits>

#include "depthwise.cuh"       // dw_finish, dw_tap
#include "depthwise_tma.cuh"   // packed-pair helpers
#include "depthwise_plane.cuh" // bulk_g2s
#include "dense_halo.cuh"      // tma_load_2d
#include "ptx.cuh"

namespace convb200 {

struct DwPwGemmParams {
    int C, Cout;
    int num_tiles;      // images
    int nblk;           // ceil(C / CB)
    int S;              // CTAs of a cluster sharing one image (1, or 2 when nblk >= 2)
    int MT;             // 128-row M tiles: ceil(Cout / 128)
    int fslot;          // bytes of one filter slot: MT * 2 boxes of CB x 64 bf16
    uint32_t idesc;
    uint32_t tmem_cols;
    const float *b_dw;  // [C] or null
    const float *b_pw;  // [Cout] or null
};

// Compile-time geometry per image size: channels per block, strips of two columns, rows per run.
// HALF (14x14): the two CTAs of an image each take half of its output rows and all of its
// channels (64 per block), so that neither holds a partial sum of the other's outputs; its
// plane window depends on the filter size KC_.
template <int HW_, bool HALF_ = false, int KC_ = 3>
struct DwPwGemmGeom {
    static constexpr int HW = HW_;
    static constexpr bool HALF = HALF_;
    static constexpr int KC = KC_;
    static constexpr int P = HW * HW;                      // pixels per image
    static constexpr int ROWS = HALF ? HW / 2 : HW;        // output rows a CTA computes
    static constexpr int PC = ROWS * HW;                   // output pixels a CTA computes
    static constexpr int NPAD = (PC + 15) / 16 * 16;       // MMA N
    static constexpr int NCH = NPAD / 16;                  // 16-column accumulator chunks
    static constexpr int CB = HALF ? 64 : (HW <= 8 ? 48 : 32);   // channels per block
    static constexpr int NSTRIP = (HW + 1) / 2;            // strips of two output columns
    static constexpr int RR = HALF ? ROWS : (HW <= 8 ? 4 : 7);   // output rows per run
    static constexpr int NRUN = (ROWS + RR - 1) / RR;
    static constexpr int UPP = NSTRIP * NRUN;              // work units per plane
    static constexpr int THREADS = 512;
    static constexpr int UNITS = CB * UPP;                 // threads with depthwise work
    // a warp without depthwise work issues the copies and the MMAs; else thread 0 does
    static constexpr bool SPARE = UNITS <= THREADS - 32;
    static constexpr int ISSUER_WARP = SPARE ? THREADS / 32 - 1 : 0;
    // planes whose byte size is a multiple of 16 arrive by one 2-D tensor copy whose box is
    // wider than a plane (the overhang reads zeros), which lays them out at a padded pitch and
    // spreads a warp's row loads over more banks (14x14: 196 -> 204 floats); 7x7 planes (196
    // bytes) arrive as one contiguous range
    static constexpr bool PADX = (P * 4) % 16 == 0;
    // HALF: each CTA copies a window of the flat plane, first float XTOP (top half, negative:
    // the rows above the image) or XBOT (bottom half), both multiples of 4 floats (16 bytes),
    // wide enough that every input row and column its strips read -- the padding rows and
    // columns included -- falls inside; rows outside the image lie outside the tensor and arrive
    // as the copy's zero fill, so only the padding columns need a select
    static constexpr int PADH = (KC - 1) / 2;
    static constexpr int XTOP = HALF ? -((PADH * (HW + 1) + 3) / 4 * 4) : 0;
    static constexpr int XBOT = HALF ? ((ROWS - PADH) * HW - PADH) / 4 * 4 : 0;
    static constexpr int XLAST_TOP = (ROWS + PADH - 1) * HW + HW - 1 + PADH - XTOP;       // last float read
    static constexpr int XLAST_BOT = (2 * ROWS + PADH - 1) * HW + HW - 1 + PADH - XBOT;
    static constexpr int XNEED = ((XLAST_TOP > XLAST_BOT ? XLAST_TOP : XLAST_BOT) + 1 + 3) / 4 * 4;
    // plane pitch in shared memory, floats; 8 mod 32, which spreads the planes of a warp's row
    // loads over more banks (14x14 whole planes: 196 -> 204; HALF windows: 136 (3x3), 168 (5x5))
    static constexpr int XP = HALF ? XNEED + (8 - XNEED % 32 + 32) % 32 : (PADX ? P + 8 : P);
    static constexpr int BOX = CB * 128;                   // one 64-wide box of CB rows, bf16
    static constexpr int NBOXB = (NPAD + 63) / 64;
    static constexpr int BSLOT = NBOXB * BOX;              // B tile: CB rows x NPAD pixels
    static constexpr int XSLOT = (CB * XP * 4 + 127) / 128 * 128;
    static constexpr int CHUNK = 128 * 16 * 4;             // 128 rows x 16 fp32 columns
    static constexpr int NOWN = (NCH + 1) / 2;             // chunks a rank of a 2-CTA cluster owns, at most
    static_assert(UNITS <= THREADS, "one work unit per thread");
    static_assert(!HALF || (HW % 2 == 0 && PADX && SPARE), "halves of an even, 16-byte-row image");
    static_assert(!HALF || ((ROWS - PADH) * HW - PADH >= XBOT && -PADH * (HW + 1) >= XTOP), "windows start early enough");
    static_assert(!PADX || (XP * 4) % 16 == 0, "a tensor-copy box row is a multiple of 16 bytes");
    static_assert(CB % 16 == 0, "K = 16 steps");
};

constexpr int kDwPwGemmFSlots = 3;
constexpr int kDwPwGemmBars = 2 /*xfull*/ + 3 /*ffull*/ + 2 /*mma_done*/ + 1 /*accf*/ + 1 /*drain*/;

// bytes of one block's depthwise taps (CB channels x KK), staged beside its planes
template <class G>
__host__ __device__ constexpr int dwpw_gemm_wslot(int KK) {
    return (G::CB * KK * 4 + 127) / 128 * 128;
}

// shared memory: filter ring, B ring, x ring, taps ring, the receive area of the cluster
// reduction (MT x NOWN chunks), barriers
template <class G>
__host__ __device__ constexpr int dwpw_gemm_recv(int MT, int S) {
    return S > 1 ? MT * G::NOWN * G::CHUNK : 0;
}

template <class G>
__host__ __device__ constexpr int dwpw_gemm_smem(int fslot, int MT, int S, int KK) {
    return 1024 + kDwPwGemmFSlots * fslot + 2 * G::BSLOT + 2 * G::XSLOT + 2 * dwpw_gemm_wslot<G>(KK) +
           dwpw_gemm_recv<G>(MT, S) + kDwPwGemmBars * 8 + 16;
}

// Byte offset of one bf16 value of the B tile: row k (channel in the block), column n (pixel);
// 64 pixels per box, 128-byte rows, 16-byte chunks swizzled by k % 8.
__device__ __forceinline__ uint32_t dwpw_b_offset(int box_bytes, int k, int n) {
    const int box = n >> 6, col = n & 63;
    return static_cast<uint32_t>(box * box_bytes + k * 128 + (((col >> 3) ^ (k & 7)) << 4) + (col & 7) * 2);
}

template <int MODE, int KC, class G>
__global__ void __launch_bounds__(512, 1)
dwpw_gemm_kernel(const float *__restrict__ x, const float *__restrict__ w, const __grid_constant__ CUtensorMap tmF,
                 const __grid_constant__ CUtensorMap tmX, float *__restrict__ y, const DwPwGemmParams p,
                 unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int HW = G::HW;
    constexpr int PAD = (KC - 1) / 2;
    constexpr int WIN = KC + 1;   // input columns of a two-column strip
    static_assert(!G::HALF || G::KC == KC, "the row split's plane window is laid out for this filter size");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw);
    const uint32_t sF = base;
    const uint32_t sB = sF + kDwPwGemmFSlots * p.fslot;
    const uint32_t sX = sB + 2 * G::BSLOT;
    constexpr int KK = KC * KC;
    constexpr int WSLOT = dwpw_gemm_wslot<G>(KK);
    const uint32_t sW = sX + 2 * G::XSLOT;   // the blocks' taps, a 2-slot ring beside x
    const uint32_t sR = sW + 2 * WSLOT;      // receive area of the reduction
    const uint32_t bars = sR + dwpw_gemm_recv<G>(p.MT, p.S);
    auto xfull = [&](int s) { return bars + 8u * s; };
    auto ffull = [&](int s) { return bars + 16u + 8u * s; };
    auto mma_done = [&](int s) { return bars + 40u + 8u * s; };
    const uint32_t accf = bars + 56u;
    const uint32_t drain = bars + 64u;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + (bars - base) + kDwPwGemmBars * 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.S;
    const int rank = S > 1 ? static_cast<int>(cluster_rank()) : 0;
    // HALF: CTA pairs 2k, 2k + 1 take the top and bottom halves of the same images (no cluster)
    const int per = G::HALF ? 2 : S;
    const int half = G::HALF ? static_cast<int>(blockIdx.x & 1u) : 0;
    const int cluster = static_cast<int>(blockIdx.x) / per;
    const int nclusters = static_cast<int>(gridDim.x) / per;
    // HALF: the first output row of this CTA, and the first float of its plane window
    const int row0 = half * G::ROWS;
    const int xbase = G::HALF ? (half ? G::XBOT : G::XTOP) : 0;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) mbar_init(xfull(s), 1);
        for (int s = 0; s < 3; ++s) mbar_init(ffull(s), 1);
        for (int s = 0; s < 2; ++s) mbar_init(mma_done(s), 1);
        mbar_init(accf, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
        prefetch_tensormap(&tmF);
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_holder), p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int my_tiles = p.num_tiles > cluster ? (p.num_tiles - cluster + nclusters - 1) / nclusters : 0;
    const int nb = (p.nblk - rank + S - 1) / S;   // this rank's blocks per image: rank, rank + S, ...
    const int total = my_tiles * nb;
    // block g of this CTA -> image and first channel
    auto block_at = [&](int g, int &n, int &c0) {
        n = cluster + (g / nb) * nclusters;
        c0 = (rank + (g % nb) * S) * G::CB;
    };
    // issuing warp: blocks whose copies are in flight or landed
    int x_issued = 0, f_issued = 0;
    const bool issuer = warp == G::ISSUER_WARP;
    const uint32_t leader = issuer ? elect_one_sync() : 0u;
    auto issue_x = [&](int g) {       // the whole issuing warp
        int n, c0;
        block_at(g, n, c0);
        x_issued = g + 1;
        const int planes = min(G::CB, p.C - c0);
        const float *src = x + (static_cast<long long>(n) * p.C + c0) * G::P;
        // the planes' taps: planes * KK floats from w[c0], a multiple of 16 bytes (C % 4 == 0)
        const uint32_t wbytes = static_cast<uint32_t>(planes * KK * 4);
        // 1-D bulk copies are not bounded by a tensor map: checked in the bounds-checked debug
        // build, where a skipped copy still completes the barrier's byte count
        auto copy_w = [&]() {
            if (in_bounds(static_cast<long long>(c0) * KK, static_cast<long long>(planes) * KK, 1LL * p.C * KK,
                          kSiteDwPwGemmW, status))
                bulk_g2s(sW + (g & 1) * WSLOT, w + static_cast<long long>(c0) * KK, wbytes, xfull(g & 1));
            else
                mbar_complete_tx(xfull(g & 1), wbytes);
        };
        if constexpr (G::PADX) {
            // x viewed as [N*C][P]: a box of XP columns x CB rows (always the full box's bytes;
            // rows past the image's channels are other planes or zeros, never used)
            if (lane == 0) {
                mbar_arrive_expect_tx(xfull(g & 1), static_cast<uint32_t>(G::CB * G::XP * 4) + wbytes);
                tma_load_2d(sX + (g & 1) * G::XSLOT, &tmX, xfull(g & 1), xbase, n * p.C + c0);
                copy_w();
            }
        } else if (lane == 0) {
            const uint32_t bytes = static_cast<uint32_t>(planes * G::P * 4);
            mbar_arrive_expect_tx(xfull(g & 1), bytes + wbytes);
            if (in_bounds((static_cast<long long>(n) * p.C + c0) * G::P, static_cast<long long>(planes) * G::P,
                          1LL * p.num_tiles * p.C * G::P, kSiteDwPwGemmX, status))
                bulk_g2s(sX + (g & 1) * G::XSLOT, src, bytes, xfull(g & 1));
            else
                mbar_complete_tx(xfull(g & 1), bytes);
            copy_w();
        }
        __syncwarp();
    };
    auto issue_f = [&](int g) {       // the whole issuing warp (lane 0 issues)
        int n, c0;
        block_at(g, n, c0);
        f_issued = g + 1;
        if (lane == 0) {
            const uint32_t slot = sF + (g % 3) * p.fslot;
            mbar_arrive_expect_tx(ffull(g % 3), static_cast<uint32_t>(p.fslot));
            for (int b = 0; b < 2 * p.MT; ++b) tma_load_2d(slot + b * G::BOX, &tmF, ffull(g % 3), b * 64, c0);
        }
    };
    // fail: the issuing warp's own waits, or'ed into the CTA at the next block barrier
    bool fail = false;
    if (issuer && total > 0) {
        // the first block's copies alone, and the second block's once its planes have landed:
        // every CTA starts at once, and the first block's bytes need not share HBM with the
        // second's (which then arrive while the first block is computed)
        issue_x(0);
        issue_f(0);
        if (total > 1) {
            if (mbar_wait_warp(xfull(0), 0)) {
                issue_x(1);
                issue_f(1);
            } else {
                fail = true;
            }
        }
    }

    // this thread's work unit inside a block: plane (channel) cl, strip of columns 2s, 2s+1,
    // run of output rows r*RR .. r*RR + RR - 1
    const bool unit_ok = tid < G::UNITS;
    const int cl = tid / G::UPP;
    const int rem = tid - cl * G::UPP;
    const int s = rem % G::NSTRIP;
    const int r = rem / G::NSTRIP;
    const int ox0 = 2 * s;
    const int ix0 = ox0 - PAD;
    const int oy_first = row0 + r * G::RR;   // absolute output row (HALF: inside this CTA's half)
    constexpr int ROWS = G::ROWS;
    bool colok[WIN];
#pragma unroll
    for (int t = 0; t < WIN; ++t) colok[t] = ix0 + t >= 0 && ix0 + t < HW;
    const bool second = ox0 + 1 < HW;   // the strip's second column exists

    // depthwise outputs of block g (channel c0 + cl of the image) into the B slot, bf16
    // (its taps arrive with its planes; its bias bv was loaded before the waits). The rows of
    // a run are one branch-free stretch of code, so that their tap chains -- each output's taps
    // in the page's order -- can interleave; only the B-tile store of a row past the image is
    // skipped.
    constexpr bool ALLROWS = G::RR * G::NRUN == ROWS;   // every run's rows exist
    // The B-tile byte offsets of this unit's outputs are the same in every block: row i of the
    // run at pixel pix = (oy - row0) * HW + ox0 of this CTA's rows (and pix + 1 for odd images,
    // whose pair may straddle a 16-byte chunk)
    auto b_off = [&](int n) { return dwpw_b_offset(G::BOX, cl, n); };
    uint32_t boff[G::RR], boff1[G::RR];
#pragma unroll
    for (int i = 0; i < G::RR; ++i) {
        const int pix = (oy_first + i - row0) * HW + ox0;
        boff[i] = b_off(pix);
        boff1[i] = HW % 2 == 0 ? 0u : b_off(pix + 1);
    }
    auto store_pair = [&](uint8_t *bslot, int i, float a0, float a1) {
        if (ALLROWS || oy_first + i < row0 + ROWS) {
            if constexpr (HW % 2 == 0) {
                // pix even: both columns exist and share a 16-byte chunk
                *reinterpret_cast<__nv_bfloat162 *>(bslot + boff[i]) = __floats2bfloat162_rn(a0, a1);
            } else {
                *reinterpret_cast<__nv_bfloat16 *>(bslot + boff[i]) = __float2bfloat16_rn(a0);
                if (second) *reinterpret_cast<__nv_bfloat16 *>(bslot + boff1[i]) = __float2bfloat16_rn(a1);
            }
        }
    };
    // hb_tag: std::true_type when the depthwise bias is given (a compile-time choice per call,
    // so that the finished rows carry no select)
    auto depthwise_block = [&](int g, int c0, float bv, auto hb_tag) {
        constexpr bool HB = decltype(hb_tag)::value;
        // the finished output: NaN made canonical (exact mode), the bias added once when given
        auto finish = [&](float a, float b) { return dw_finish<MODE, HB>(a, b); };
        uint8_t *bslot = smem + (sB - base) + (g & 1) * G::BSLOT;
        const int c = c0 + cl;
        if (c < p.C) {
            const float *xs = reinterpret_cast<const float *>(smem + (sX - base) + (g & 1) * G::XSLOT) + cl * G::XP;
            const float *ws = reinterpret_cast<const float *>(smem + (sW - base) + (g & 1) * WSLOT) + cl * KK;
            float wr[KK];
#pragma unroll
            for (int t = 0; t < KK; ++t) wr[t] = ws[t];
            uint64_t w2[KC * KC];
#pragma unroll
            for (int t = 0; t < KC * KC; ++t) w2[t] = dw_pack(wr[t], wr[t]);
            // input row iy as KC overlapping pairs (x[t], x[t+1]); rows and columns outside the
            // image read as zeros
            auto load_pairs = [&](int iy, uint64_t (&dst)[KC]) {
                float f[WIN];
                if constexpr (G::HALF) {
                    // the window holds zeros for the rows outside the image; the middle columns
                    // of a strip are always inside it
#pragma unroll
                    for (int t = 0; t < WIN; ++t) {
                        const float v = xs[iy * HW + ix0 + t - xbase];
                        f[t] = (t >= PAD && t <= PAD + 1) || colok[t] ? v : 0.0f;
                    }
                } else {
                    const bool rowok = iy >= 0 && iy < HW;
#pragma unroll
                    for (int t = 0; t < WIN; ++t) f[t] = (rowok && colok[t]) ? xs[iy * HW + ix0 + t - xbase] : 0.0f;
                }
#pragma unroll
                for (int t = 0; t < KC; ++t) dst[t] = dw_pack(f[t], f[t + 1]);
            };
            if constexpr (KC == 3) {
                // every input row of the run held at once (RR + 2 rows of 3 pairs), then tap by
                // tap over the RR rows: RR independent chains per output column
                constexpr int NR = G::RR + KC - 1;
                uint64_t rows[NR][KC];
#pragma unroll
                for (int q = 0; q < NR; ++q) load_pairs(oy_first - PAD + q, rows[q]);
                if constexpr (MODE == 0) {
                    float a0[G::RR], a1[G::RR];
#pragma unroll
                    for (int i = 0; i < G::RR; ++i) a0[i] = a1[i] = 0.0f;
#pragma unroll
                    for (int ky = 0; ky < KC; ++ky)
#pragma unroll
                        for (int kx = 0; kx < KC; ++kx)
#pragma unroll
                            for (int i = 0; i < G::RR; ++i) dw_tap2_exact_split(a0[i], a1[i], w2[ky * KC + kx], rows[i + ky][kx]);
#pragma unroll
                    for (int i = 0; i < G::RR; ++i) store_pair(bslot, i, finish(a0[i], bv), finish(a1[i], bv));
                } else {
                    uint64_t a2[G::RR];
#pragma unroll
                    for (int i = 0; i < G::RR; ++i) a2[i] = dw_pack(0.0f, 0.0f);
#pragma unroll
                    for (int ky = 0; ky < KC; ++ky)
#pragma unroll
                        for (int kx = 0; kx < KC; ++kx)
#pragma unroll
                            for (int i = 0; i < G::RR; ++i) a2[i] = dw_tap2_fast(a2[i], w2[ky * KC + kx], rows[i + ky][kx]);
#pragma unroll
                    for (int i = 0; i < G::RR; ++i) {
                        float a0, a1;
                        dw_unpack(a2[i], a0, a1);
                        store_pair(bslot, i, finish(a0, bv), finish(a1, bv));
                    }
                }
            } else {
                // larger filters: a ring of KC input rows, one output row after another
                uint64_t ring[KC][KC];
#pragma unroll
                for (int q = 0; q < KC - 1; ++q) load_pairs(oy_first - PAD + q, ring[q]);
#pragma unroll
                for (int i = 0; i < G::RR; ++i) {
                    load_pairs(oy_first + i - PAD + KC - 1, ring[(i + KC - 1) % KC]);
                    float a0, a1;
                    if constexpr (MODE == 0) {
                        a0 = 0.0f;
                        a1 = 0.0f;
#pragma unroll
                        for (int ky = 0; ky < KC; ++ky)
#pragma unroll
                            for (int kx = 0; kx < KC; ++kx)
                                dw_tap2_exact_split(a0, a1, w2[ky * KC + kx], ring[(i + ky) % KC][kx]);
                    } else {
                        uint64_t a2 = dw_pack(0.0f, 0.0f);
#pragma unroll
                        for (int ky = 0; ky < KC; ++ky)
#pragma unroll
                            for (int kx = 0; kx < KC; ++kx)
                                a2 = dw_tap2_fast(a2, w2[ky * KC + kx], ring[(i + ky) % KC][kx]);
                        dw_unpack(a2, a0, a1);
                    }
                    store_pair(bslot, i, finish(a0, bv), finish(a1, bv));
                }
            }
        } else {
            // channels past C: zero rows, so that the zero filter rows meet finite values
#pragma unroll
            for (int i = 0; i < G::RR; ++i) store_pair(bslot, i, 0.0f, 0.0f);
        }
    };

    // 16 consecutive pixels of output channel o: acc (+ the cluster peer's partial) + bias -> y
    // (the channel split; the row split stages its tile through shared memory)
    auto store_chunk = [&](float *yrow, int p0, const float (&v)[16], float bp) {
        if (!in_bounds((yrow - y) + p0, min(16, G::P - p0), 1LL * p.num_tiles * p.Cout * G::P, kSiteDwPwGemmY, status))
            return;   // skipped (bounds-checked debug build)
        if constexpr (G::P % 4 == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (p0 + 4 * u < G::P)
                    *reinterpret_cast<float4 *>(yrow + p0 + 4 * u) =
                        make_float4(__fadd_rn(v[4 * u], bp), __fadd_rn(v[4 * u + 1], bp),
                                    __fadd_rn(v[4 * u + 2], bp), __fadd_rn(v[4 * u + 3], bp));
        } else {
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (p0 + u < G::P) yrow[p0 + u] = __fadd_rn(v[u], bp);
        }
    };

    // Every thread walks every tile and every block; after a wait ran out (dead) it skips the
    // work but still takes each CTA and cluster barrier, so neither this CTA nor its cluster
    // peer ever waits for it forever.
    bool dead = false;
    int stop = 0;                      // the first block whose wait ran out
    int g = 0;
    for (int tl = 0; tl < my_tiles; ++tl) {
        const int n = cluster + tl * nclusters;
        for (int j = 0; j < nb; ++j, ++g) {
            const int c0 = (rank + j * S) * G::CB;   // block g = tl * nb + j (block_at without the division)
            bool good = true;
            if (!dead) {
                // the channel's bias first, so that its load overlaps the waits
                float bv = 0.0f;
                const int c = c0 + cl;
                if (unit_ok && c < p.C && p.b_dw) bv = __ldg(p.b_dw + c);
                // the block's planes staged; the B slot's previous MMAs (block g - 2) done
                good = mbar_wait_warp(xfull(g & 1), (g >> 1) & 1);
                if (good && g >= 2) good = mbar_wait_warp(mma_done(g & 1), ((g - 2) >> 1) & 1);
                if (good && unit_ok) {
                    if (p.b_dw)
                        depthwise_block(g, c0, bv, std::true_type{});
                    else
                        depthwise_block(g, c0, bv, std::false_type{});
                }
                fence_proxy_async_smem();   // the B tile's generic writes, visible to the tensor cores
            }
            if (__syncthreads_or(!good || fail) && !dead) {
                dead = true;
                stop = g;
            }
            if (!dead && issuer) {
                // the whole issuing warp, converged; the MMAs and commits are predicated on the
                // elected lane (so are the drain's, so that its commit tracks them all). First the
                // refill of x two blocks ahead, into the slot this block's depthwise stage has just
                // finished reading (the barrier above), so that its copy overlaps the MMAs too
                if (g + 2 < total) issue_x(g + 2);
                if (!mbar_wait_warp(ffull(g % 3), (g / 3) & 1)) {
                    fail = true;
                } else {
                    tc_fence_after();
                    const uint32_t fs = sF + (g % 3) * p.fslot;
                    const uint32_t bs = sB + (g & 1) * G::BSLOT;
                    // descriptors: +128 (2048 B, 16 rows) per K=16 step; A +2*BOX/16 per M tile
                    const uint64_t bd0 = smem_desc_sw128(bs, G::BOX, 1024);
                    const uint64_t ad0 = smem_desc_sw128(fs, G::BOX, 1024);
#pragma unroll
                    for (int kk = 0; kk < G::CB / 16; ++kk)
                        for (int mt = 0; mt < p.MT; ++mt)
                            umma_f16_ss_if(tmem + mt * G::NPAD, ad0 + kk * 128 + mt * (2 * G::BOX >> 4), bd0 + kk * 128,
                                           p.idesc, (j | kk) != 0 ? 1u : 0u, leader);
                    umma_commit_if(mma_done(g & 1), leader);
                    if (j == nb - 1) umma_commit_if(accf, leader);
                    // F two blocks ahead into the slot block g - 1 used, once its MMAs are done
                    if (g + 2 < total) {
                        if (g >= 1 && !mbar_wait_warp(mma_done((g - 1) & 1), ((g - 1) >> 1) & 1)) fail = true;
                        else issue_f(g + 2);
                    }
                }
            }
        }

        // ------------------------------- epilogue of image n -------------------------------
        bool got = true;
        if (!dead) got = mbar_wait_warp(accf, tl & 1);
        if (__syncthreads_or(!got || fail) && !dead) {
            dead = true;
            stop = g;
        }
        tc_fence_after();
        const int q = warp & 3, cg = warp >> 2;   // TMEM lane quarter; a quarter of the chunks
        if (S > 1) {
            // the chunks the peer owns: this rank's partial into the peer's receive area
            if (!dead) {
                const uint32_t peer_r = map_rank(sR, static_cast<uint32_t>(rank ^ 1));
                for (int mt = 0; mt < p.MT; ++mt)
                    for (int jc = cg; jc < G::NCH; jc += 4) {
                        if ((jc & 1) == rank) continue;
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + mt * G::NPAD + jc * 16, v);
                        tmem_wait_ld();
                        const uint32_t dst = peer_r + ((mt * G::NOWN + (jc >> 1)) * 128 + q * 32 + lane) * 64;
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            st_cluster_v4(dst + 16 * u, v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    }
            }
            cluster_sync_all();   // the partials have landed in the owners' receive areas
        }
        if constexpr (G::HALF) {
            // Row split: staged through the B ring (its last MMAs are complete and the next
            // image's depthwise writes come after this epilogue), one tile of 128 output
            // channels x 64 pixels at a time, so that y is written in contiguous runs of a
            // channel's pixels rather than one 8-byte piece per channel. The 16-byte chunks of a
            // staged row are XOR-swizzled by the row: conflict-free column writes and row reads.
            float *stage = reinterpret_cast<float *>(smem + (sB - base));
            static_assert(2 * G::BSLOT >= 128 * 64 * 4, "the staging tile fits the B ring");
            constexpr int NPASS = (G::PC + 63) / 64;
            for (int mt = 0; mt < p.MT; ++mt) {
                const int o = mt * 128 + q * 32 + lane;
                const float bp = (p.b_pw && o < p.Cout) ? __ldg(p.b_pw + o) : 0.0f;
                for (int pass = 0; pass < NPASS; ++pass) {
                    const int jc = pass * 4 + cg;   // this warp's 16-column chunk
                    if (!dead && jc < G::NCH) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + mt * G::NPAD + jc * 16, v);
                        tmem_wait_ld();
                        const int r = q * 32 + lane;
                        float *srow = stage + r * 64;
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int chunk = (cg * 4 + u) ^ (r & 15);
                            *reinterpret_cast<float4 *>(srow + chunk * 4) =
                                make_float4(__fadd_rn(__uint_as_float(v[4 * u]), bp),
                                            __fadd_rn(__uint_as_float(v[4 * u + 1]), bp),
                                            __fadd_rn(__uint_as_float(v[4 * u + 2]), bp),
                                            __fadd_rn(__uint_as_float(v[4 * u + 3]), bp));
                        }
                    }
                    __syncthreads();
                    // 128 staged rows, 16 warps: a warp writes a row's pixels as 8-byte pieces (a
                    // half plane starts 8-byte aligned)
                    const int ncols = min(64, G::PC - pass * 64);
                    if (!dead && 2 * lane < ncols) {
                        for (int rr = warp; rr < 128; rr += 16) {
                            const int oo = mt * 128 + rr;
                            if (oo >= p.Cout) break;
                            const int col = 2 * lane;
                            const float2 val = *reinterpret_cast<const float2 *>(
                                stage + rr * 64 + (((col >> 2) ^ (rr & 15)) << 2) + (col & 3));
                            float *dst = y + (static_cast<long long>(n) * p.Cout + oo) * G::P + row0 * HW + pass * 64 + col;
                            if (in_bounds(dst - y, 2, 1LL * p.num_tiles * p.Cout * G::P, kSiteDwPwGemmY, status))
                                *reinterpret_cast<float2 *>(dst) = val;
                        }
                    }
                    __syncthreads();
                }
            }
        } else if (!dead) {
            for (int mt = 0; mt < p.MT; ++mt) {
                const int o = mt * 128 + q * 32 + lane;
                const float bp = (p.b_pw && o < p.Cout) ? __ldg(p.b_pw + o) : 0.0f;
                float *yrow = y + (static_cast<long long>(n) * p.Cout + (o < p.Cout ? o : 0)) * G::P;
                for (int jc = cg; jc < G::NCH; jc += 4) {
                    if (S > 1 && (jc & 1) != rank) continue;
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + mt * G::NPAD + jc * 16, v);
                    tmem_wait_ld();
                    float sum[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) sum[u] = __uint_as_float(v[u]);
                    if (S > 1) {
                        // the two partials added once (an IEEE sum of two terms: the same bits
                        // whichever rank adds them)
                        const float *rv = reinterpret_cast<const float *>(
                            smem + (sR - base) + ((mt * G::NOWN + (jc >> 1)) * 128 + q * 32 + lane) * 64);
#pragma unroll
                        for (int u = 0; u < 16; ++u) sum[u] = __fadd_rn(sum[u], rv[u]);
                    }
                    if (o < p.Cout) store_chunk(yrow, jc * 16, sum, bp);
                }
            }
        }
        // the receive area is read before the next image's partials land in it (after the last
        // image no partials follow)
        if (S > 1 && tl + 1 < my_tiles) cluster_sync_all();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (dead && issuer) {
        if (lane == 0) atomicOr(status, kStatusTimeout);
        // every copy issued lands, and every MMA issued completes, before the CTA exits
        // (bounded waits): the copies of blocks stop .. issued - 1 were not waited for yet
        for (int jj = stop; jj < x_issued; ++jj) mbar_wait_warp(xfull(jj & 1), (jj >> 1) & 1);
        for (int jj = stop; jj < f_issued; ++jj) mbar_wait_warp(ffull(jj % 3), (jj / 3) & 1);
        umma_commit_if(drain, leader);
        mbar_wait_warp(drain, 0);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, p.tmem_cols);
}

}  // namespace convb200
