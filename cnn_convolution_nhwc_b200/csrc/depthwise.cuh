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
// loop has no bounds tests and reads the padding exactly as the page defines it. Staging
// gives every thread a fixed window column and walks rows (and planes) incrementally, so
// consecutive threads load consecutive addresses and no division happens per element. A
// thread then owns VX neighbouring outputs of one row (the page's "lanes are neighbouring
// output columns", widened to a register strip): per filter row it reads the strip's input
// window from shared memory once (128-bit loads where the shapes are compile-time) and
// reuses it for all VX outputs and KW taps. Every output is computed independently in the one
// tap order, so results never depend on the job shape (the page's determinism property).
// Stride and dilation are index arithmetic on the staged window; there are no phase planes.
#pragma once
#include <cstdint>

#include "ptx.cuh"   // in_bounds (bounds-checked debug build)

namespace convb200 {

// Division by an invariant divisor 1 <= d < 2^31 for dividends 0 <= n < 2^31, by a
// multiply-high and a shift (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): s = ceil(log2 d), m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (umulhi(n, m) + n) >> s.
struct FastDiv {
    uint32_t m, s;
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t s = 0;
    while ((1ull << s) < d) ++s;
    const unsigned long long m = ((1ull << 32) * ((1ull << s) - d)) / d + 1;
    return FastDiv{static_cast<uint32_t>(m), s};
}

__device__ __forceinline__ int fdiv(int n, FastDiv f) {
    return static_cast<int>((__umulhi(static_cast<uint32_t>(n), f.m) + static_cast<uint32_t>(n)) >> f.s);
}

struct DwParams {
    int Cin, mult, Cout, H, W, KH, KW, stride, pad, dil, Ho, Wo;
    int P, R, CW;               // planes, output rows and output columns per job
    int rows_in, cols_in;       // staged input window per plane
    int pitch;                  // shared-memory row pitch (floats, multiple of 4)
    int n_rbands, n_cbands;
    int num_planes;             // N * Cout
    int w_stride;               // floats reserved per plane for the weights in shared memory
    int tc_log2;                // staging threads per window row = 2^tc_log2
    int vec_store;              // 1: rows of y are 16-byte aligned (Wo % 4 == 0, y aligned)
    FastDiv div_cout, div_mult, div_taps, div_cbands, div_rbands;
};

template <int MODE>
__device__ __forceinline__ float dw_tap(float acc, float wv, float xv) {
    if (MODE == 0) return __fadd_rn(acc, __fmul_rn(wv, xv));
    return __fmaf_rn(wv, xv, acc);
}

template <int MODE, bool HAS_BIAS>
__device__ __forceinline__ float dw_finish(float acc, float b) {
    if (MODE == 0 && acc != acc) acc = __int_as_float(0x7FC00000);
    if (HAS_BIAS) {
        acc = __fadd_rn(acc, b);
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

// Shared-memory layout of one job: input-plane offsets (P x int64), bias (P), weights
// (P x w_stride), then the staged windows (P x rows_in x pitch), each part 16-byte aligned.
__host__ __device__ inline int dw_smem_head_floats(int P, int w_stride) {
    return 2 * ((P + 1) & ~1) + ((P + 3) & ~3) + P * w_stride;
}

// KW_T / S_T: compile-time kernel width and stride with unit dilation (0 = runtime values,
// one output per thread). VX: outputs per thread along a row (4 for the compile-time forms).
template <int MODE, bool HAS_BIAS, int KW_T, int S_T, int VX>
__global__ void __launch_bounds__(256)
depthwise_kernel(const float *__restrict__ x, const float *__restrict__ w,
                 const float *__restrict__ bias, float *__restrict__ y, const DwParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    // tensor extents for the bounds-checked debug build
    const long long x_elems = 1LL * (p.num_planes / p.Cout) * p.Cin * p.H * p.W;
    const long long y_elems = 1LL * p.num_planes * p.Ho * p.Wo;
    extern __shared__ __align__(16) float sm[];
    long long *s_inoff = reinterpret_cast<long long *>(sm);
    float *sb = sm + 2 * ((p.P + 1) & ~1);
    float *sw = sb + ((p.P + 3) & ~3);
    float *sx = sm + dw_smem_head_floats(p.P, p.w_stride);
    const int taps = p.KH * p.KW;
    const int tile = p.rows_in * p.pitch;

    const int cb = blockIdx.x - fdiv(blockIdx.x, p.div_cbands) * p.n_cbands;
    const int job = fdiv(blockIdx.x, p.div_cbands);
    const int pg = fdiv(job, p.div_rbands);
    const int rb = job - pg * p.n_rbands;
    const int plane0 = pg * p.P;
    const int nplanes = min(p.P, p.num_planes - plane0);
    const int oy0 = rb * p.R;
    const int nrows = min(p.R, p.Ho - oy0);
    const int ox0 = cb * p.CW;
    const int ncols = min(p.CW, p.Wo - ox0);
    const int iy0 = oy0 * p.stride - p.pad;
    const int ix0 = ox0 * p.stride - p.pad;

    // ---- per-plane tables: input plane offset, bias; then the weights ------------------
    for (int pp = threadIdx.x; pp < nplanes; pp += blockDim.x) {
        const int plane = plane0 + pp;
        const int n = fdiv(plane, p.div_cout);
        const int oc = plane - n * p.Cout;
        const int ic = fdiv(oc, p.div_mult);
        s_inoff[pp] = (static_cast<long long>(n) * p.Cin + ic) * p.H * static_cast<long long>(p.W);
        if (HAS_BIAS) sb[pp] = __ldg(bias + oc);
    }
    for (int e = threadIdx.x; e < nplanes * taps; e += blockDim.x) {
        const int pp = fdiv(e, p.div_taps);
        const int t = e - pp * taps;
        const int plane = plane0 + pp;
        const int oc = plane - fdiv(plane, p.div_cout) * p.Cout;
        sw[pp * p.w_stride + t] = __ldg(w + static_cast<long long>(oc) * taps + t);
    }
    __syncthreads();

    // ---- stage the zero-padded windows: fixed column per thread, rows walk incrementally --
    {
        const uint32_t sx_s = static_cast<uint32_t>(__cvta_generic_to_shared(sx));
        const int tc = 1 << p.tc_log2;
        const int c = threadIdx.x & (tc - 1);
        const int row_step = blockDim.x >> p.tc_log2;
        const int gx = ix0 + c;
        const bool col_ok = c < p.cols_in && gx >= 0 && gx < p.W;
        int pp = 0, r = threadIdx.x >> p.tc_log2;
        while (r >= p.rows_in) { r -= p.rows_in; ++pp; }
        const float *xp = x + (pp < nplanes ? s_inoff[pp] : 0);
        int cur = pp;
        if (c < p.cols_in) {
            while (pp < nplanes) {
                if (pp != cur) { xp = x + s_inoff[pp]; cur = pp; }
                const int gy = iy0 + r;
                const bool ok = col_ok && gy >= 0 && gy < p.H &&
                                in_bounds(s_inoff[pp] + static_cast<long long>(gy) * p.W + gx, 1, x_elems, kSiteDwX, status);
                cp_async_f32_zfill(sx_s + 4u * (pp * tile + r * p.pitch + c),
                                   ok ? xp + static_cast<long long>(gy) * p.W + gx : x, ok);
                r += row_step;
                while (r >= p.rows_in) { r -= p.rows_in; ++pp; }
            }
        }
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- compute: one strip of VX outputs of one row per item --------------------------
    const int strips = (ncols + VX - 1) / VX;
    const int per_plane = nrows * strips;
    const FastDiv d_plane = make_fastdiv(per_plane);
    const FastDiv d_strips = make_fastdiv(strips);
    const long long HoWo = static_cast<long long>(p.Ho) * p.Wo;
    for (int it = threadIdx.x; it < nplanes * per_plane; it += blockDim.x) {
        const int pp = fdiv(it, d_plane);
        const int rem = it - pp * per_plane;
        const int r = fdiv(rem, d_strips);
        const int ox = (rem - r * strips) * VX;
        const float *ws = sw + pp * p.w_stride;
        const float b = HAS_BIAS ? sb[pp] : 0.0f;
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
            for (int v = 0; v < VX; ++v) acc[v] = dw_finish<MODE, HAS_BIAS>(acc[v], b);
            const long long yoff = yrow - y;
            if (VX == 4 && p.vec_store && ox + 4 <= ncols) {
                if (in_bounds(yoff, 4, y_elems, kSiteDwY, status))
                    *reinterpret_cast<float4 *>(yrow) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            } else {
#pragma unroll
                for (int v = 0; v < VX; ++v)
                    if (ox + v < ncols && in_bounds(yoff + v, 1, y_elems, kSiteDwY, status)) yrow[v] = acc[v];
            }
        } else {
            // runtime kernel size, stride and dilation; VX == 1
            const float *xs = sx + pp * tile + (r * p.stride) * p.pitch + ox * p.stride;
            float acc = 0.0f;
            for (int ky = 0; ky < p.KH; ++ky) {
                const float *xr = xs + ky * p.dil * p.pitch;
                for (int kx = 0; kx < p.KW; ++kx) acc = dw_tap<MODE>(acc, ws[ky * p.KW + kx], xr[kx * p.dil]);
            }
            if (in_bounds(yrow - y, 1, y_elems, kSiteDwY, status)) yrow[0] = dw_finish<MODE, HAS_BIAS>(acc, b);
        }
    }
}

}  // namespace convb200
