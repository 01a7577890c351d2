// Explicit im2col followed by one GEMM: the comparison path the CMU DLSys Lecture 14 notes
// describe (section 5 "Generalize the patch matrix to channels and batches": patch rows of
// N*Ho*Wo pixels by K*K*Cin values in (i, j, c) order, times the filter viewed as a
// (K*K*Cin) x Cout matrix; section 6 "The dense matrix has a measurable storage bill"; section 7
// "Optimize the whole transformation": time the packing together with the multiplication).
//
// The packing kernel copies, for every output pixel (n, y, x) and tap (i, j), the Cin channels
// X[n, y+i, x+j, :] into row (n, y, x), columns (i*K + j)*Cin .. +Cin of the patch matrix A in
// a caller-provided workspace. Consecutive threads take consecutive 16-byte chunks of A, so the
// writes are fully coalesced and the reads walk contiguous channel runs of X. The GEMM is a
// plain library call (cuBLAS, bf16 operands, fp32 accumulation, bf16 output).
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"   // in_bounds (bounds-checked debug build)

namespace convb200 {

struct Im2colParams {
    int H, W, Cin, K, Ho, Wo;
    int kd;              // K * K * Cin: patch-matrix columns
    int chunk;           // channels per copied chunk: 8 (16 bytes) when Cin % 8 == 0, else 1
    long long chunks;    // M * K * K * Cin / chunk
};

__global__ void __launch_bounds__(256)
im2col_pack_kernel(const __nv_bfloat16 *__restrict__ X, __nv_bfloat16 *__restrict__ A, const Im2colParams p,
                   unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    // tensor extents for the bounds-checked debug build
    const long long a_elems = p.chunks * p.chunk;
    const long long x_elems = (a_elems / p.kd) / (1LL * p.Ho * p.Wo) * p.H * p.W * p.Cin;
    const int per_tap = p.Cin / p.chunk;
    for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < p.chunks; t += stride) {
        long long u = t;
        const int cc = static_cast<int>(u % per_tap);
        u /= per_tap;
        const int tap = static_cast<int>(u % (p.K * p.K));
        const long long m = u / (p.K * p.K);
        const int i = tap / p.K, j = tap - i * p.K;
        const int x = static_cast<int>(m % p.Wo);
        const long long r = m / p.Wo;
        const int y = static_cast<int>(r % p.Ho);
        const long long n = r / p.Ho;
        const long long src = ((n * p.H + (y + i)) * p.W + (x + j)) * p.Cin + static_cast<long long>(cc) * p.chunk;
        const long long dst = m * p.kd + static_cast<long long>(tap) * p.Cin + static_cast<long long>(cc) * p.chunk;
        if (!in_bounds(src, p.chunk, x_elems, kSiteIm2colX, status) ||
            !in_bounds(dst, p.chunk, a_elems, kSiteIm2colA, status))
            continue;   // skipped (bounds-checked debug build)
        if (p.chunk == 8)
            *reinterpret_cast<uint4 *>(A + dst) = __ldg(reinterpret_cast<const uint4 *>(X + src));
        else
            A[dst] = X[src];
    }
}

}  // namespace convb200
