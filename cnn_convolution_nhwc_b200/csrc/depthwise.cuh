// Depthwise forward convolution on NCHW float32 planes, CUDA cores.
//
// Each output follows the OneModel "Depthwise convolution" page, section "What each output
// is": plane oc reads input plane oc / mult; acc = +0; for ky (outer), for kx (inner):
// acc = acc + w[oc,ky,kx] * x_padded[oy*s + ky*d, ox*s + kx*d]; padding is a real zero that is
// multiplied; exact mode rounds the product and then the sum (__fmul_rn, __fadd_rn) and
// rewrites a NaN result as 0x7FC00000; fast mode is one fused multiply-add per tap
// (__fmaf_rn); the bias is one rounded addition afterwards.
//
// Work layout. A CTA takes one job: P consecutive output planes x R output rows x CW output
// columns. It stages the input window those outputs read -- rows iy0 .. iy0+rows_in-1 and
// columns ix0 .. ix0+cols_in-1 of each input plane -- into shared memory with cp.async,
// whose zero-fill form writes a real +0 for every position outside the image, so the tap
// loop has no bounds tests and reads the padding exactly as the page defines it. A thread
// then owns VX neighbouring outputs of one row (the page's "lanes are neighbouring output
// columns", here widened to a register strip): per filter row it reads the strip's input
// window from shared memory once (128-bit loads where the shapes are compile-time) and
// reuses it for all VX outputs and KW taps. Every output is still computed independently in
// the one tap order, so results never depend on the job shape (the page's determinism
// property). Stride and dilation are index arithmetic on the staged window; there are no
// phase planes. Index math is 32-bit and per job or per strip, never per tap.
#pragma once
#include <cstdint>

namespace convb200 {

struct DwParams {
    int Cin, mult, Cout, H, W, KH, KW, stride, pad, dil, Ho, Wo;
    int P, R, CW;               // planes, output rows and output columns per job
    int rows_in, cols_in;       // staged input window per plane
    int pitch;                  // shared-memory row pitch (floats, multiple of 4)
    int n_rbands, n_cbands;
    int num_planes;             // N * Cout
    int w_stride;               // floats reserved per plane for the weights in shared memory
};

template <int MODE>
__device__ __forceinline__ float dw_tap(float acc, float wv, float xv) {
    if (MODE == 0) return __fadd_rn(acc, __fmul_rn(wv, xv));
    return __fmaf_rn(wv, xv, acc);
}

template <int MODE, bool HAS_BIAS>
__device__ __forceinline__ float dw_finish(float acc, const float *bias, int oc) {
    if (MODE == 0 && acc != acc) acc = __int_as_float(0x7FC00000);
    if (HAS_BIAS) {
        acc = __fadd_rn(acc, __ldg(bias + oc));
        if (MODE == 0 && acc != acc) acc = __int_as_float(0x7FC00000);
    }
    return acc;
}

__device__ __forceinline__ void cp_async_f32_zfill(uint32_t dst, const float *src, bool valid) {
    // src-size 0 writes zeros and reads nothing
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// KW_T / S_T: compile-time kernel width and stride with unit dilation (0 = runtime values,
// one output per thread). VX: outputs per thread along a row.
template <int MODE, bool HAS_BIAS, int KW_T, int S_T, int VX>
__global__ void __launch_bounds__(256)
depthwise_kernel(const float *__restrict__ x, const float *__restrict__ w,
                 const float *__restrict__ bias, float *__restrict__ y, const DwParams p) {
    extern __shared__ __align__(16) float sm[];
    const int taps = p.KH * p.KW;
    float *sw = sm;
    float *sx = sm + p.P * p.w_stride;
    const int tile = p.rows_in * p.pitch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

    int job = blockIdx.x;
    const int cb = job % p.n_cbands;
    job /= p.n_cbands;
    const int rb = job % p.n_rbands;
    const int pg = job / p.n_rbands;
    const int plane0 = pg * p.P;
    const int nplanes = min(p.P, p.num_planes - plane0);
    const int oy0 = rb * p.R;
    const int nrows = min(p.R, p.Ho - oy0);
    const int ox0 = cb * p.CW;
    const int ncols = min(p.CW, p.Wo - ox0);
    const int iy0 = oy0 * p.stride - p.pad;
    const int ix0 = ox0 * p.stride - p.pad;

    // ---- stage weights and the zero-padded input window ------------------------------
    for (int e = threadIdx.x; e < nplanes * taps; e += blockDim.x) {
        const int pp = e / taps;
        const int t = e - pp * taps;
        const int oc = (plane0 + pp) % p.Cout;
        sw[pp * p.w_stride + t] = __ldg(w + static_cast<long long>(oc) * taps + t);
    }
    const uint32_t sx_s = static_cast<uint32_t>(__cvta_generic_to_shared(sx));
    for (int pr = warp; pr < nplanes * p.rows_in; pr += nwarps) {
        const int pp = pr / p.rows_in;
        const int r = pr - pp * p.rows_in;
        const int plane = plane0 + pp;
        const int n = plane / p.Cout;
        const int ic = (plane - n * p.Cout) / p.mult;
        const int gy = iy0 + r;
        const bool row_ok = gy >= 0 && gy < p.H;
        const float *xrow = x + (static_cast<long long>(n) * p.Cin + ic) * p.H * static_cast<long long>(p.W) +
                            static_cast<long long>(row_ok ? gy : 0) * p.W;
        const uint32_t srow = sx_s + 4u * (pp * tile + r * p.pitch);
        for (int c = lane; c < p.cols_in; c += 32) {
            const int gx = ix0 + c;
            const bool ok = row_ok && gx >= 0 && gx < p.W;
            cp_async_f32_zfill(srow + 4u * c, ok ? xrow + gx : x, ok);
        }
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- compute: one strip of VX outputs of one row per item --------------------------
    const int strips = (ncols + VX - 1) / VX;
    const int per_plane = nrows * strips;
    const long long HoWo = static_cast<long long>(p.Ho) * p.Wo;
    for (int it = threadIdx.x; it < nplanes * per_plane; it += blockDim.x) {
        const int pp = it / per_plane;
        const int rem = it - pp * per_plane;
        const int r = rem / strips;
        const int ox = (rem - r * strips) * VX;
        const float *ws = sw + pp * p.w_stride;
        const int oc = (plane0 + pp) % p.Cout;
        float *yrow = y + (plane0 + pp) * HoWo + static_cast<long long>(oy0 + r) * p.Wo + ox0 + ox;
        if constexpr (KW_T > 0) {
            constexpr int S = S_T;
            constexpr int WIN = (VX - 1) * S + KW_T;        // inputs one filter row touches
            constexpr int WIN4 = (WIN + 3) / 4;             // 128-bit loads per filter row
            float acc[VX];
#pragma unroll
            for (int v = 0; v < VX; ++v) acc[v] = 0.0f;
            const float *xs = sx + pp * tile + (r * S) * p.pitch + ox * S;
            for (int ky = 0; ky < p.KH; ++ky) {
                float win[WIN4 * 4];
                const float4 *src = reinterpret_cast<const float4 *>(xs + ky * p.pitch);
#pragma unroll
                for (int q = 0; q < WIN4; ++q) {
                    const float4 t4 = src[q];
                    win[4 * q] = t4.x; win[4 * q + 1] = t4.y; win[4 * q + 2] = t4.z; win[4 * q + 3] = t4.w;
                }
#pragma unroll
                for (int kx = 0; kx < KW_T; ++kx) {
                    const float wv = ws[ky * KW_T + kx];
#pragma unroll
                    for (int v = 0; v < VX; ++v) acc[v] = dw_tap<MODE>(acc[v], wv, win[v * S + kx]);
                }
            }
#pragma unroll
            for (int v = 0; v < VX; ++v)
                if (ox + v < ncols) yrow[v] = dw_finish<MODE, HAS_BIAS>(acc[v], bias, oc);
        } else {
            // runtime kernel size, stride and dilation; VX == 1
            const float *xs = sx + pp * tile + (r * p.stride) * p.pitch + ox * p.stride;
            float acc = 0.0f;
            for (int ky = 0; ky < p.KH; ++ky) {
                const float *xr = xs + ky * p.dil * p.pitch;
                for (int kx = 0; kx < p.KW; ++kx) acc = dw_tap<MODE>(acc, ws[ky * p.KW + kx], xr[kx * p.dil]);
            }
            yrow[0] = dw_finish<MODE, HAS_BIAS>(acc, bias, oc);
        }
    }
}

}  // namespace convb200
