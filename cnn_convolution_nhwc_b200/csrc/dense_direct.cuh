// Dense NHWC forward convolution on the CUDA cores, one output per thread.
//
// This is the path for shapes the tensor-core kernel cannot address with TMA (Cin or Cout
// not a multiple of 8, tensors below 128 KiB, K > 128) and for the float32 entry point. It
// evaluates the index contract of the CMU DLSys Lecture 14 notes, section 1, directly:
// Y[n,y,x,o] = sum over (i, j, c) of X[n,y+i,x+j,c] * F[i,j,c,o], as float32 fused
// multiply-adds in (i, j, c) order, rounded once to the output type -- and the stride, zero
// padding, dilation and bias variants of "Convolution Is Wx+b Moving Across a Signal" (window
// of output (y, x) at (y*stride - pad, x*stride - pad), taps dil apart, positions outside the
// image skipped as zeros, the bias one fp32 addition before the rounding), with separate
// height and width geometry, KH x KW filters and channel groups (output channel o of group
// g = o / (Cout/groups) sums only input channels g*Cin_g .. +Cin_g, Cin_g = Cin/groups, with
// filter F[i, j, c, o] for the group-local channel c; a Conv1D is the H = KH = 1 case).
// Consecutive threads take consecutive output channels o, so the F row reads are coalesced and
// the X reads are warp-uniform broadcasts (or few-address ones across a group boundary).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"   // in_bounds (bounds-checked debug build)

namespace convb200 {

struct DenseDirectParams {
    int H, W, Cin, Cout, KH, KW, Ho, Wo;
    int Cin_g, Cout_g;      // channels of one group (Cin, Cout when there is one group)
    int sh, sw, ph, pw, dh, dw;   // "Convolution Is Wx+b Moving Across a Signal" variants
    const float *bias;      // per output channel or null; added in fp32 before the rounding
    long long total;        // N * Ho * Wo * Cout
    long long x_elems;      // N * H * W * Cin
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store_out(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

template <typename T>
__global__ void __launch_bounds__(256)
dense_direct_kernel(const T *__restrict__ X, const T *__restrict__ F, T *__restrict__ Y,
                    const DenseDirectParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < p.total;
         idx += stride) {
        long long t = idx;
        const int o = static_cast<int>(t % p.Cout);
        t /= p.Cout;
        const int x = static_cast<int>(t % p.Wo);
        t /= p.Wo;
        const int y = static_cast<int>(t % p.Ho);
        const long long n = t / p.Ho;
        const int cin0 = (o / p.Cout_g) * p.Cin_g;
        float acc = 0.0f;
        for (int i = 0; i < p.KH; ++i) {
            const int r = y * p.sh + i * p.dh - p.ph;
            if (r < 0 || r >= p.H) continue;   // zero padding contributes nothing
            for (int j = 0; j < p.KW; ++j) {
                const int q = x * p.sw + j * p.dw - p.pw;
                if (q < 0 || q >= p.W) continue;
                const long long xoff = ((n * p.H + r) * p.W + q) * p.Cin + cin0;
                if (!in_bounds(xoff, p.Cin_g, p.x_elems, kSiteDirectX, status)) continue;
                const T *xr = X + xoff;
                const T *fr = F + ((static_cast<long long>(i) * p.KW + j) * p.Cin_g) * p.Cout + o;
                for (int c = 0; c < p.Cin_g; ++c)
                    acc = __fmaf_rn(to_f32(xr[c]), to_f32(fr[static_cast<long long>(c) * p.Cout]), acc);
            }
        }
        if (p.bias) acc = __fadd_rn(acc, __ldg(p.bias + o));
        if (in_bounds(idx, 1, p.total, kSiteDirectY, status)) store_out(Y + idx, acc);
    }
}

}  // namespace convb200
