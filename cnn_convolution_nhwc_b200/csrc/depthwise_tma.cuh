// Depthwise forward convolution on NCHW float32 planes: per-warp asynchronous staging into a
// zero-padded shared-memory window, computed from a register window that never moves.
//
// Same contract as depthwise.cuh (the OneModel "Depthwise convolution" page, section "What
// each output is": acc = +0; ky outer, kx inner; padding a real zero that is multiplied; exact
// mode __fmul_rn then __fadd_rn with NaN rewritten as 0x7FC00000; fast mode one __fmaf_rn per
// tap; the bias one rounded addition afterwards), for compile-time K x K, stride S, padding
// PAD = (K-1)/2, dilation 1, multiplier 1.
//
// Work layout. Every warp runs its own pipeline over a list of jobs; a job is ppw planes x Rw
// output rows. The warp stages its next jobs' input windows into a ring of NB shared-memory
// buffers while it computes from the current one. A buffer holds, per plane and staged input
// row, 4 zeros, the row, and zeros up to the pitch Wp, so the compute loop has no bounds tests
// and no shuffles. Rows that are 16-byte multiples arrive as one 3-D TMA box {Wp, rows, planes} whose
// x starts at -4: the copy engine writes every zero of the padding itself (left, right, above,
// below). Other widths are staged only as whole planes: 4-byte cp.async copies of the image
// into buffers whose padding was zeroed once at start (it never changes, since every job
// places its planes identically).
//
// Lane g of a plane owns output columns 4g .. 4g+3 and reads its input window -- input columns
// 4gS - PAD .. 4gS - PAD + 3S + K - 1 -- straight from the buffer with the widest aligned
// shared loads the offset allows. Input rows live in a ring of K register rows indexed by
// (staged row mod K); the row loop is unrolled by K, so every ring index is a compile-time
// constant and advancing the window costs only the S new rows' loads. No CTA-wide barrier:
// warps never wait on each other. Every output is computed independently in the one tap order,
// so results are bit-identical to the other depthwise kernels.
#pragma once
#include <cstdint>

#include "depthwise.cuh"
#include "ptx.cuh"

namespace convb200 {

struct DwTmaParams {
    int H, W, Ho, Wo, C;   // C = Cin = Cout (multiplier 1)
    int lpp, ppw;          // lanes per plane, planes per warp
    int Rw;                // output rows per job (Ho when jobs are whole planes)
    int rows_in;           // staged input rows per plane: (Rw - 1) * S + K
    int Wp;                // buffer row pitch in floats (multiple of 4)
    int nbands;            // row bands per plane group
    int num_planes, num_jobs;
    int box_floats;        // ppw * rows_in * Wp: one staged job
    int buf_floats;        // buffer stride: box_floats rounded up to 128 bytes (TMA destinations
                           // in shared memory must be 128-byte aligned)
    int use_tma;           // 1: TMA box (W % 4 == 0); 0: cp.async copies of whole planes
    int vec_out;           // 1: 128-bit output stores
    int stage_out;         // 1: whole-plane jobs collect their outputs in shared memory and write
                           //    the job's contiguous output range with coalesced stores
    int out_floats;        // per-warp output staging (ppw * Ho * Wo rounded up to 128 bytes)
    int warp_floats;       // per-warp shared memory: nbuf * buf_floats + out_floats
    int nbuf;              // staging buffers per warp (2 .. kDwTmaMaxBuf): jobs staged ahead
    int vec_out_staged;    // 1: y 16-byte aligned (staged copies may use 128-bit stores)
    int stagger;           // 1: a warp's first job is copied alone, the rest of its first NB after it
                           //    (the first jobs' bytes need not share HBM at start)
    FastDiv div_nbands, div_lpp, div_c, div_w;
};

constexpr int kDwWarpsPerCta = 4;
constexpr int kDwTmaMaxBuf = 4;

// N consecutive floats from shared memory starting at base + A (base 16-byte aligned), with
// the widest loads the compile-time offset allows
template <int A, int N>
__device__ __forceinline__ void dw_ld_span(const float *base, float *out) {
    if constexpr (N > 0) {
        if constexpr (A % 4 == 0 && N >= 4) {
            const float4 v = *reinterpret_cast<const float4 *>(base + A);
            out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
            dw_ld_span<A + 4, N - 4>(base, out + 4);
        } else if constexpr (A % 2 == 0 && N >= 2) {
            const float2 v = *reinterpret_cast<const float2 *>(base + A);
            out[0] = v.x; out[1] = v.y;
            dw_ld_span<A + 2, N - 2>(base, out + 2);
        } else {
            out[0] = base[A];
            dw_ld_span<A + 1, N - 1>(base, out + 1);
        }
    }
}

// Packed pairs of float32 (sm_100 f32x2 arithmetic): two neighbouring outputs of a lane advance
// together; each half is an IEEE binary32 operation rounded to nearest, exactly as the scalar
// __fmul_rn / __fmaf_rn, so results are bit-identical to the scalar kernels.
__device__ __forceinline__ uint64_t dw_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void dw_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// Exact-mode tap for two outputs (lo, hi): each product rounded once, then each sum rounded
// once, as the page's rounded multiply then rounded add. The product is formed as fma(w, x, +0),
// which equals the rounded product except that an exact zero product comes out +0 where the
// multiply gives -0. A running sum that starts at +0 is never -0 (a rounded sum is -0 only when
// both terms are), and adding +0 or -0 to it gives the same value, so every sum is bit-identical
// to the page's. One packed fma and one packed add per tap pair, and no multiply: a packed
// multiply whose only use is a packed add was measured to come out fused (one rounding).
__device__ __forceinline__ uint64_t dw_tap2_exact(uint64_t acc, uint64_t w2, uint64_t x2) {
    uint64_t prod, r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(prod) : "l"(w2), "l"(x2), "l"(0ull));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(acc), "l"(prod));
    return r;
}

// Fast-mode tap for two outputs: one packed fused multiply-add.
__device__ __forceinline__ uint64_t dw_tap2_fast(uint64_t acc, uint64_t w2, uint64_t x2) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(w2), "l"(x2), "l"(acc));
    return r;
}

// The same exact-mode tap with the two sums kept as scalars: one packed multiply and two scalar
// rounded additions (bit-identical to dw_tap2_exact; the fused depthwise-pointwise kernel,
// bound by its shared-memory loads, measured faster with this form).
__device__ __forceinline__ void dw_tap2_exact_split(float &lo, float &hi, uint64_t w2, uint64_t x2) {
    uint64_t prod;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(prod) : "l"(w2), "l"(x2));
    float p0, p1;
    dw_unpack(prod, p0, p1);
    lo = __fadd_rn(lo, p0);
    hi = __fadd_rn(hi, p1);
}

// A tap for two outputs held as one packed pair, in either mode.
template <int MODE>
__device__ __forceinline__ uint64_t dw_tap2(uint64_t acc, uint64_t w2, uint64_t x2) {
    if constexpr (MODE == 0)
        return dw_tap2_exact(acc, w2, x2);
    else
        return dw_tap2_fast(acc, w2, x2);
}

template <int MODE, bool HAS_BIAS, int K, int S>
__global__ void __launch_bounds__(32 * kDwWarpsPerCta)
depthwise_tma_kernel(const __grid_constant__ CUtensorMap tmx, const float *__restrict__ x,
                     const float *__restrict__ w, const float *__restrict__ bias, float *__restrict__ y,
                     const DwTmaParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int PAD = (K - 1) / 2;
    constexpr int VX = 4;
    constexpr int OWN = VX * S;
    constexpr int WIN = (VX - 1) * S + K;
    extern __shared__ __align__(128) float sraw[];
    __shared__ __align__(8) uint64_t full_all[kDwWarpsPerCta][kDwTmaMaxBuf];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // the dynamic region is only guaranteed 16-byte alignment: align the buffers to 128 bytes
    const uint32_t raw_s = static_cast<uint32_t>(__cvta_generic_to_shared(sraw));
    float *sbuf = sraw + (((raw_s + 127u) & ~127u) - raw_s) / 4u;
    float *my_buf = sbuf + static_cast<size_t>(warp) * p.warp_floats;
    const int NB = p.nbuf;
    float *sout = my_buf + NB * p.buf_floats;
    const uint32_t buf_s = static_cast<uint32_t>(__cvta_generic_to_shared(my_buf));
    const uint32_t full0 = static_cast<uint32_t>(__cvta_generic_to_shared(&full_all[warp][0]));
    auto full = [&](int b) { return full0 + 8u * b; };

    const int gw = blockIdx.x * kDwWarpsPerCta + warp;
    const int GW = gridDim.x * kDwWarpsPerCta;

    // stage job `job` into buffer `b`
    auto issue = [&](int job, int b) {
        const int pg = fdiv(job, p.div_nbands);
        const int band = job - pg * p.nbands;
        const int plane0 = pg * p.ppw;
        const uint32_t dst = buf_s + 4u * b * p.buf_floats;
        if (p.use_tma) {
            if (lane == 0) {
                // the box always has ppw planes; planes past the tensor arrive as zeros
                const int iy0 = band * p.Rw * S - PAD;
                mbar_arrive_expect_tx(full(b), 4u * p.box_floats);
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                    " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
                    "l"(reinterpret_cast<uint64_t>(&tmx)), "r"(full(b)), "r"(-4), "r"(iy0), "r"(plane0)
                    : "memory");
            }
        } else {
            // whole planes: image element e of plane slot s goes to staged row PAD + e / W,
            // buffer column 4 + e % W; the padding around it is already zero
            const int HW = p.H * p.W;
            for (int s = 0; s < p.ppw; ++s) {
                const int plane = plane0 + s;
                if (plane >= p.num_planes) break;
                const float *src = x + static_cast<long long>(plane) * HW;
                const uint32_t dplane = dst + 4u * (s * p.rows_in + PAD) * p.Wp + 16u;
                for (int e = lane; e < HW; e += 32) {
                    const int r = fdiv(e, p.div_w);
                    if (!in_bounds(static_cast<long long>(plane) * HW + e, 1, 1LL * p.num_planes * HW, kSiteDwTmaX,
                                   status))
                        continue;
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dplane + 4u * (r * p.Wp + e - r * p.W)),
                                 "l"(src + e)
                                 : "memory");
                }
            }
            asm volatile("cp.async.mbarrier.arrive.noinc.shared.b64 [%0];" ::"r"(full(b)) : "memory");
        }
    };

    if (lane == 0) {
        for (int b = 0; b < NB; ++b) mbar_init(full(b), p.use_tma ? 1 : 32);
        fence_barrier_init();
        if (p.use_tma) prefetch_tensormap(&tmx);
    }
    if (!p.use_tma) {   // zero the buffers once: the padding of whole-plane jobs never changes
        float4 *z = reinterpret_cast<float4 *>(my_buf);
        for (int i = lane; i < NB * p.buf_floats / 4; i += 32) z[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    __syncwarp();
    // the warp's first NB jobs go in flight at once, or with p.stagger the first job alone and
    // the rest once it has landed (in the loop): every warp starts at once, and the first jobs'
    // bytes need not share HBM with the next ones' (which then arrive while the first is
    // computed)
    for (int b = 0; b < (p.stagger ? 1 : NB); ++b)
        if (gw + b * GW < p.num_jobs) issue(gw + b * GW, b);

    // lane geometry (fixed for the kernel's life)
    const int ps = fdiv(lane, p.div_lpp);
    const int cg = lane - ps * p.lpp;
    const bool lane_ok = ps < p.ppw;
    const int ox = cg * VX;
    const int c0 = cg * OWN;   // first input column this lane owns: buffer column c0 + 4

    int k = 0;
    bool ok = true;
    for (int job = gw; job < p.num_jobs; job += GW, ++k) {
        const int b = k % NB;
        if (!mbar_wait_warp(full(b), (k / NB) & 1)) { ok = false; break; }
        if (k == 0 && p.stagger)
            for (int bb = 1; bb < NB; ++bb)
                if (gw + bb * GW < p.num_jobs) issue(gw + bb * GW, bb);
        const int pg = fdiv(job, p.div_nbands);
        const int band = job - pg * p.nbands;
        const int oy0 = band * p.Rw;
        const int nrows = min(p.Rw, p.Ho - oy0);
        const int plane = pg * p.ppw + (lane_ok ? ps : 0);
        const bool active = lane_ok && plane < p.num_planes;
        const int c = active ? plane - fdiv(plane, p.div_c) * p.C : 0;
        float wr[K * K];
#pragma unroll
        for (int t = 0; t < K * K; ++t) wr[t] = __ldg(w + c * (K * K) + t);
        const float bv = HAS_BIAS ? __ldg(bias + c) : 0.0f;
        // staged row r of this lane's plane; buffer column c0 + 4 - PAD is input column c0 - PAD
        const float *pb = my_buf + b * p.buf_floats + (lane_ok ? ps : 0) * (p.rows_in * p.Wp) + c0;
        float *yp = y + (static_cast<long long>(active ? plane : 0) * p.Ho + oy0) * p.Wo + ox;

        auto store_row = [&](int i, const float (&acc)[VX]) {
            if (p.stage_out) {   // whole-plane job: row oy0 + i = i of plane slot ps
                if (active) {
                    float *dst = sout + (ps * p.Ho + i) * p.Wo + ox;
#pragma unroll
                    for (int v = 0; v < VX; ++v)
                        if (ox + v < p.Wo) dst[v] = acc[v];
                }
            } else if (active) {
                float *dst = yp + static_cast<long long>(i) * p.Wo;
                if (!in_bounds(dst - y, min(VX, p.Wo - ox), 1LL * p.num_planes * p.Ho * p.Wo, kSiteDwTmaY, status)) {
                    // skipped (bounds-checked debug build)
                } else if (p.vec_out && ox + VX <= p.Wo) {
                    *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                } else {
#pragma unroll
                    for (int v = 0; v < VX; ++v)
                        if (ox + v < p.Wo) dst[v] = acc[v];
                }
            }
        };

        if constexpr (S == 1) {
            // ring of K rows held as the WIN - 1 overlapping pairs (x[t], x[t+1]): outputs
            // (2q, 2q+1) at tap kx read pair 2q + kx, and the weight is a pair (w, w)
            uint64_t w2[K * K];
#pragma unroll
            for (int t = 0; t < K * K; ++t) w2[t] = dw_pack(wr[t], wr[t]);
            uint64_t ring[K][WIN - 1];
            auto load_pairs = [&](int r, uint64_t (&dst)[WIN - 1]) {
                float f[WIN];
                dw_ld_span<4 - PAD, WIN>(pb + r * p.Wp, f);
#pragma unroll
                for (int t = 0; t < WIN - 1; ++t) dst[t] = dw_pack(f[t], f[t + 1]);
            };
#pragma unroll
            for (int r = 0; r < K - 1; ++r) load_pairs(r, ring[r]);
            for (int base = 0; base < nrows; base += K) {
#pragma unroll
                for (int u = 0; u < K; ++u) {
                    const int i = base + u;
                    if (i < nrows) {
                        // staged row i + K - 1 completes the window of output row i (ring slot
                        // of staged row r: (u + r - i) % K, base being a multiple of K)
                        load_pairs(i + K - 1, ring[(u + K - 1) % K]);
                        float acc[VX];
                        {
                            uint64_t a2[VX / 2];
#pragma unroll
                            for (int q = 0; q < VX / 2; ++q) a2[q] = dw_pack(0.0f, 0.0f);
#pragma unroll
                            for (int ky = 0; ky < K; ++ky)
#pragma unroll
                                for (int kx = 0; kx < K; ++kx)
#pragma unroll
                                    for (int q = 0; q < VX / 2; ++q)
                                        a2[q] = dw_tap2<MODE>(a2[q], w2[ky * K + kx], ring[(u + ky) % K][2 * q + kx]);
#pragma unroll
                            for (int q = 0; q < VX / 2; ++q) dw_unpack(a2[q], acc[2 * q], acc[2 * q + 1]);
                        }
#pragma unroll
                        for (int v = 0; v < VX; ++v) acc[v] = dw_finish<MODE, HAS_BIAS>(acc[v], bv);
                        store_row(i, acc);
                    }
                }
            }
        } else {
            float ring[K][WIN];
#pragma unroll
            for (int r = 0; r < K - S; ++r) dw_ld_span<4 - PAD, WIN>(pb + r * p.Wp, ring[r]);
            for (int base = 0; base < nrows; base += K) {
#pragma unroll
                for (int u = 0; u < K; ++u) {
                    const int i = base + u;
                    if (i < nrows) {
                        // staged rows i*S + K - S .. i*S + K - 1 complete the window of output row
                        // i (base is a multiple of K, so row r sits in ring slot (u*S + r - i*S) % K)
#pragma unroll
                        for (int s = 0; s < S; ++s)
                            dw_ld_span<4 - PAD, WIN>(pb + (i * S + K - S + s) * p.Wp, ring[(u * S + K - S + s) % K]);
                        float acc[VX];
#pragma unroll
                        for (int v = 0; v < VX; ++v) {
                            float a = 0.0f;
#pragma unroll
                            for (int ky = 0; ky < K; ++ky)
#pragma unroll
                                for (int kx = 0; kx < K; ++kx)
                                    a = dw_tap<MODE>(a, wr[ky * K + kx], ring[(u * S + ky) % K][v * S + kx]);
                            acc[v] = dw_finish<MODE, HAS_BIAS>(a, bv);
                        }
                        store_row(i, acc);
                    }
                }
            }
        }
        if (p.stage_out) {
            // the job's planes are contiguous in y: copy them out with coalesced stores
            __syncwarp();
            const int plane0 = pg * p.ppw;
            const int nplanes = min(p.ppw, p.num_planes - plane0);
            const int plane_out = p.Ho * p.Wo;
            const int total = nplanes * plane_out;
            float *gdst = y + static_cast<long long>(plane0) * plane_out;
            if (!in_bounds(static_cast<long long>(plane0) * plane_out, total, 1LL * p.num_planes * plane_out,
                           kSiteDwTmaY, status)) {
                // skipped (bounds-checked debug build)
            } else if (p.vec_out_staged && ((plane0 * plane_out) & 3) == 0) {
                const int n4 = total >> 2;
                for (int e = lane; e < n4; e += 32)
                    reinterpret_cast<float4 *>(gdst)[e] = reinterpret_cast<const float4 *>(sout)[e];
                for (int e = (n4 << 2) + lane; e < total; e += 32) gdst[e] = sout[e];
            } else {
                for (int e = lane; e < total; e += 32) gdst[e] = sout[e];
            }
        }
        // every lane is done with buffer b (and the output staging); refill b NB jobs ahead
        __syncwarp();
        if (job + NB * GW < p.num_jobs) issue(job + NB * GW, b);
    }
    if (!ok) {
        if (lane == 0) atomicOr(status, kStatusTimeout);
        // drain: copies still in flight land before the warp exits (bounded waits); with
        // p.stagger a wait that ran out on the first job leaves only that job issued
        for (int kk = k; kk < (k == 0 && p.stagger ? 1 : k + NB); ++kk)
            if (gw + kk * GW < p.num_jobs) mbar_wait_warp(full(kk % NB), (kk / NB) & 1);
    }
}

}  // namespace convb200
