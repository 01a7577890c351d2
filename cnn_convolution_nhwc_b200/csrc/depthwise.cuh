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
// columns. It stages the input window those outputs read -- rows iy0 .. iy0 + rows_in - 1
// and columns ix0 .. ix0 + cols_in - 1 of the input plane, with every position outside the
// image written as a real +0 -- into shared memory with coalesced loads, so the tap loop
// needs no bounds tests and reads the padding exactly as the page defines it. Threads then
// walk the job's outputs with consecutive threads on neighbouring output columns (the page's
// "lanes are neighbouring output columns"), each output computed independently in the one
// tap order, so the result never depends on the tiling chosen (the page's determinism
// property). Stride and dilation are plain index arithmetic on the staged window. The
// weights of the job's planes are staged once and read as warp-uniform broadcasts.
#pragma once

namespace convb200 {

struct DwParams {
    int Cin, mult, Cout, H, W, KH, KW, stride, pad, dil, Ho, Wo;
    int P, R, CW;               // planes, output rows and output columns per job
    int rows_in, cols_in;       // staged input window per plane
    int n_rbands, n_cbands;
    long long num_planes;       // N * Cout
    int w_stride;               // floats reserved per plane for the weights in shared memory
};

template <int MODE>
__device__ __forceinline__ float dw_tap(float acc, float wv, float xv) {
    if (MODE == 0) return __fadd_rn(acc, __fmul_rn(wv, xv));
    return __fmaf_rn(wv, xv, acc);
}

template <int MODE, bool HAS_BIAS>
__global__ void __launch_bounds__(256)
depthwise_kernel(const float *__restrict__ x, const float *__restrict__ w,
                 const float *__restrict__ bias, float *__restrict__ y, const DwParams p) {
    extern __shared__ float sm[];
    const int taps = p.KH * p.KW;
    float *sw = sm;
    float *sx = sm + p.P * p.w_stride;
    const int tile = p.rows_in * p.cols_in;

    long long job = blockIdx.x;
    const int cb = static_cast<int>(job % p.n_cbands);
    job /= p.n_cbands;
    const int rb = static_cast<int>(job % p.n_rbands);
    const long long pg = job / p.n_rbands;
    const long long plane0 = pg * p.P;
    const int nplanes = static_cast<int>(min(static_cast<long long>(p.P), p.num_planes - plane0));
    const int oy0 = rb * p.R;
    const int nrows = min(p.R, p.Ho - oy0);
    const int ox0 = cb * p.CW;
    const int ncols = min(p.CW, p.Wo - ox0);
    const int iy0 = oy0 * p.stride - p.pad;
    const int ix0 = ox0 * p.stride - p.pad;

    for (int e = threadIdx.x; e < nplanes * taps; e += blockDim.x) {
        const int pp = e / taps;
        const long long oc = (plane0 + pp) % p.Cout;
        sw[pp * p.w_stride + (e - pp * taps)] = w[oc * taps + (e - pp * taps)];
    }
    for (int e = threadIdx.x; e < nplanes * tile; e += blockDim.x) {
        const int pp = e / tile;
        const int rr = (e - pp * tile) / p.cols_in;
        const int cc = e - pp * tile - rr * p.cols_in;
        const long long plane = plane0 + pp;
        const long long n = plane / p.Cout;
        const int ic = static_cast<int>(plane - n * p.Cout) / p.mult;
        const int gy = iy0 + rr;
        const int gx = ix0 + cc;
        float v = 0.0f;
        if (gy >= 0 && gy < p.H && gx >= 0 && gx < p.W)
            v = __ldg(x + ((n * p.Cin + ic) * p.H + gy) * static_cast<long long>(p.W) + gx);
        sx[e] = v;
    }
    __syncthreads();

    const int per_plane = nrows * ncols;
    for (int e = threadIdx.x; e < nplanes * per_plane; e += blockDim.x) {
        const int pp = e / per_plane;
        const int oy = (e - pp * per_plane) / ncols;
        const int ox = e - pp * per_plane - oy * ncols;
        const float *xs = sx + pp * tile + oy * p.stride * p.cols_in + ox * p.stride;
        const float *ws = sw + pp * p.w_stride;
        float acc = 0.0f;
        for (int ky = 0; ky < p.KH; ++ky) {
            const float *xr = xs + ky * p.dil * p.cols_in;
            for (int kx = 0; kx < p.KW; ++kx) acc = dw_tap<MODE>(acc, ws[ky * p.KW + kx], xr[kx * p.dil]);
        }
        if (MODE == 0 && acc != acc) acc = __int_as_float(0x7FC00000);
        const long long plane = plane0 + pp;
        if (HAS_BIAS) {
            acc = __fadd_rn(acc, __ldg(bias + plane % p.Cout));
            if (MODE == 0 && acc != acc) acc = __int_as_float(0x7FC00000);
        }
        y[(plane * p.Ho + (oy0 + oy)) * static_cast<long long>(p.Wo) + ox0 + ox] = acc;
    }
}

}  // namespace convb200
