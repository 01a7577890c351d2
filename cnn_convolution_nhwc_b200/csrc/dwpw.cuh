// Depthwise K x K followed by pointwise 1 x 1, fused: the depthwise output never goes to HBM.
//
// The block of "Convolution Is Wx+b Moving Across a Signal", section "Why variants matter": a
// depthwise pass (one filter per channel) followed by a pointwise pass that mixes channels. Stage
// one is the OneModel "Depthwise convolution" contract (section "What each output is": acc = +0,
// ky outer, kx inner, padding a real zero that is multiplied, exact mode __fmul_rn then
// __fadd_rn with NaN rewritten as 0x7FC00000, fast mode one __fmaf_rn per tap, the depthwise
// bias one rounded addition), multiplier 1. Stage two is a GEMM on the tensor cores:
//     Y_mat[(n, oy, ox), o] = sum_c bf16(d[n, c, oy, ox]) * F[c, o]   (+ bias_pw[o] in fp32),
// with the depthwise output rounded to bfloat16 (nearest even) as the A operand, F bfloat16
// [C][Cout] as the B operand, float32 accumulation in TMEM, and y written as float32 NCHW.
//
// Work layout. A persistent CTA of 8 warps owns 128 consecutive output pixels of the flattened
// (n, oy, ox) space (a tile may span images) and walks the channels in blocks of 64:
//   * every thread computes 32 depthwise outputs of one pixel (thread t: pixel t % 128, channels
//     (t / 128) * 32 .. +31 of the block; a warp's 32 pixels are consecutive, so each tap's x
//     loads are one coalesced row segment and the weights are warp-uniform) and writes them, as
//     bf16 pairs, into a 128 x 64 A tile laid out exactly as a 128-byte-swizzled K-major TMA
//     tile would be;
//   * thread 0 loads the block's 64 x Cout filter rows by TMA (MN-major, 64-column boxes) and,
//     after the CTA barrier that publishes the A tile, issues the four K = 16 MMAs of the block
//     into one TMEM accumulator of N = Cout (rounded up to 16) columns, then commits to the
//     stage's barrier, which frees that A/B stage two blocks later;
//   * after the last block, all 8 warps read the accumulator (warp w: TMEM lanes 32*(w%4), one
//     half of the 16-column chunks), add the pointwise bias and store y: for each output channel
//     a warp writes 32 consecutive pixels of one NCHW plane.
// Two A/B stages let the tensor cores and the TMA run under the next block's depthwise work.
// Every wait is bounded; the CTA decides to stop with a barrier-wide OR, so all threads leave
// together, and all MMAs complete before TMEM is freed.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "dense_tc.cuh"     // pack_bf16x2
#include "depthwise.cuh"    // dw_tap, dw_finish, FastDiv
#include "ptx.cuh"

namespace convb200 {

struct DwPwParams {
    int C, H, W, Ho, Wo, HoWo;
    int K, stride, pad, dil;   // depthwise geometry (both axes)
    int Cout;                  // multiple of 8, at most 256
    int n_mma;                 // Cout rounded up to 16: the MMA's N
    int n_boxes;               // ceil(Cout / 64): filter boxes per channel block
    int num_kblk;              // ceil(C / 64)
    int M;                     // N * Ho * Wo
    int num_tiles;             // ceil(M / 128)
    uint32_t idesc;
    uint32_t tmem_cols;        // power of two >= max(32, n_mma)
    const float *b_dw;         // [C] or null
    const float *b_pw;         // [Cout] or null
    FastDiv div_howo, div_wo;
};

constexpr int kDwPwThreads = 256;
constexpr int kDwPwA = 128 * 128;      // A stage: 128 pixel rows x 64 channels, bf16 (16 KB)
constexpr int kDwPwBox = 64 * 128;     // one filter box: 64 channel rows x 64 outputs, bf16 (8 KB)
constexpr int kDwPwB = 4 * kDwPwBox;   // B stage: up to 256 outputs
constexpr int kDwPwSmem = 1024 + 2 * kDwPwA + 2 * kDwPwB + 64;

template <int MODE, int KC>
__global__ void __launch_bounds__(kDwPwThreads, 2)
dwpw_kernel(const float *__restrict__ x, const float *__restrict__ w, const __grid_constant__ CUtensorMap tmF,
            float *__restrict__ y, const DwPwParams p, unsigned int *status) {
    const int K = KC ? KC : p.K;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;   // swizzle atoms need 1024-byte alignment
    uint8_t *smem = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + 2 * kDwPwA;
    const uint32_t bars = sB + 2 * kDwPwB;
    auto bfull = [&](uint32_t s) { return bars + 8u * s; };
    auto afree = [&](uint32_t s) { return bars + 16u + 8u * s; };
    const uint32_t accf = bars + 32u;
    const uint32_t done = bars + 40u;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + (bars - base) + 48);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + (bars - base) + 52);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        mbar_init(bfull(0), 1);
        mbar_init(bfull(1), 1);
        mbar_init(afree(0), 1);
        mbar_init(afree(1), 1);
        mbar_init(accf, 1);
        mbar_init(done, 1);
        *abort_flag = 0;
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

    const int r = tid & 127;       // pixel row of the tile for the depthwise stage
    const int half = tid >> 7;     // channels half*32 .. +31 of each block
    const long long plane = static_cast<long long>(p.H) * p.W;
    uint32_t it = 0, ntile = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++ntile) {
        const int m = tile * 128 + r;
        const bool valid = m < p.M;
        int n = 0, oy = 0, ox = 0;
        if (valid) {
            n = fdiv(m, p.div_howo);
            const int pix = m - n * p.HoWo;
            oy = fdiv(pix, p.div_wo);
            ox = pix - oy * p.Wo;
        }
        const int iy0 = oy * p.stride - p.pad, ix0 = ox * p.stride - p.pad;
        const float *xn = x + static_cast<long long>(n) * p.C * plane;
        bool stop = false;
        for (int kb = 0; kb < p.num_kblk; ++kb, ++it) {
            const uint32_t s = it & 1u, use = it >> 1;
            // stage s is free once the MMAs of two blocks ago have read it
            const bool w_ok = it < 2 || mbar_wait(afree(s), (use - 1u) & 1u);
            if (__syncthreads_or(!w_ok || *abort_flag)) { stop = true; break; }
            if (tid == 0) {
                mbar_arrive_expect_tx(bfull(s), static_cast<uint32_t>(p.n_boxes * kDwPwBox));
                for (int h = 0; h < p.n_boxes; ++h)
                    tma_load_3d(sB + s * kDwPwB + h * kDwPwBox, &tmF, bfull(s), h * 64, kb * 64, 0);
            }
            // depthwise outputs of 32 channels at this pixel -> bf16 pairs in row r of A[s]
            uint8_t *arow = smem + s * kDwPwA + r * 128;
#pragma unroll 1
            for (int j = 0; j < 32; j += 2) {
                const int cl = half * 32 + j;
                float v[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = kb * 64 + cl + u;
                    float acc = 0.0f;
                    if (valid && c < p.C) {
                        const float *xp = xn + c * plane;
                        const float *wp = w + c * K * K;
                        if (KC) {   // compile-time filter size: fully unrolled taps
#pragma unroll
                            for (int ky = 0; ky < KC; ++ky) {
                                const int iy = iy0 + ky * p.dil;
                                const bool rok = static_cast<unsigned>(iy) < static_cast<unsigned>(p.H);
#pragma unroll
                                for (int kx = 0; kx < KC; ++kx) {
                                    const int ix = ix0 + kx * p.dil;
                                    const bool in = rok && static_cast<unsigned>(ix) < static_cast<unsigned>(p.W);
                                    const float xv = in ? __ldg(xp + iy * p.W + ix) : 0.0f;
                                    acc = dw_tap<MODE>(acc, __ldg(wp + ky * KC + kx), xv);
                                }
                            }
                        } else {
                            for (int ky = 0; ky < K; ++ky) {
                                const int iy = iy0 + ky * p.dil;
                                const bool rok = static_cast<unsigned>(iy) < static_cast<unsigned>(p.H);
                                for (int kx = 0; kx < K; ++kx) {
                                    const int ix = ix0 + kx * p.dil;
                                    const bool in = rok && static_cast<unsigned>(ix) < static_cast<unsigned>(p.W);
                                    const float xv = in ? __ldg(xp + iy * p.W + ix) : 0.0f;
                                    acc = dw_tap<MODE>(acc, __ldg(wp + ky * K + kx), xv);
                                }
                            }
                        }
                        acc = p.b_dw ? dw_finish<MODE, true>(acc, __ldg(p.b_dw + c)) : dw_finish<MODE, false>(acc, 0.0f);
                    }
                    v[u] = acc;
                }
                const uint32_t chunk = static_cast<uint32_t>(cl >> 3) ^ static_cast<uint32_t>(r & 7);
                *reinterpret_cast<uint32_t *>(arow + (chunk << 4) + (cl & 7) * 2) = pack_bf16x2(v[0], v[1]);
            }
            fence_proxy_async_smem();   // the A tile is read by the tensor cores (async proxy)
            __syncthreads();
            if (tid == 0) {
                if (mbar_wait(bfull(s), use & 1u)) {
                    tc_fence_after();
                    const uint32_t a0 = sA + s * kDwPwA, b0 = sB + s * kDwPwB;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        // A: K-major, 16 channels = 32 B inside the swizzle atom, 8-row groups
                        // 1024 B apart. B: MN-major, 16 channel rows = 2048 B, 64-output boxes
                        // 8 KB apart.
                        const uint64_t ad = smem_desc_sw128(a0 + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b0 + kk * 2048, kDwPwBox, 1024);
                        umma_f16_ss(tmem, ad, bd, p.idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    umma_commit(afree(s));
                } else {
                    atomicOr(status, kStatusTimeout);
                    *abort_flag = 1;
                }
            }
        }
        if (stop) break;
        if (tid == 0) umma_commit(accf);
        const bool a_ok = mbar_wait(accf, ntile & 1u);
        if (__syncthreads_or(!a_ok || *abort_flag)) break;
        tc_fence_after();
        // epilogue: accumulator rows -> y (NCHW float32), plus the pointwise bias
        {
            const int q = warp & 3;                 // TMEM lane quarter of this warp
            const int row = q * 32 + lane;
            const int me = tile * 128 + row;
            const bool ve = me < p.M;
            int ne = 0, pix = 0;
            if (ve) {
                ne = fdiv(me, p.div_howo);
                pix = me - ne * p.HoWo;
            }
            float *yrow = y + static_cast<long long>(ne) * p.Cout * p.HoWo + pix;
            const int nch = p.n_mma >> 4;
            for (int cb = warp >> 2; cb < nch; cb += 2) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + cb * 16, v);
                tmem_wait_ld();
                if (ve) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int o = cb * 16 + j;
                        if (o < p.Cout) {
                            float val = __uint_as_float(v[j]);
                            if (p.b_pw) val = __fadd_rn(val, __ldg(p.b_pw + o));
                            yrow[static_cast<long long>(o) * p.HoWo] = val;
                        }
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();   // the accumulator is free for the next tile's MMAs
    }
    // nothing in flight may outlive the CTA: every MMA issued has completed before TMEM is freed
    if (tid == 0) {
        umma_commit(done);
        if (!mbar_wait(done, 0)) atomicOr(status, kStatusTimeout);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, p.tmem_cols);
}

}  // namespace convb200
