// Depthwise forward convolution for small square planes (7x7, 14x14): a lane owns a plane.
//
// Same contract as depthwise.cuh (the OneModel "Depthwise convolution" page, section "What
// each output is": acc = +0; ky outer, kx inner; padding a real zero that is multiplied; exact
// mode __fmul_rn then __fadd_rn with NaN rewritten as 0x7FC00000; fast mode one __fmaf_rn per
// tap; the bias one rounded addition afterwards), for compile-time plane size HW, K x K, stride
// S, padding (K-1)/2, dilation 1, multiplier 1.
//
// Work layout. With planes this small, "lanes are neighbouring output columns" leaves most of a
// warp idle or spread over many planes with tiny rows. Here one warp takes a job of 32 / LPP
// consecutive planes -- one contiguous range of x -- and stages it into shared memory with a
// single 1-D bulk copy. Each lane then computes a whole plane (LPP = 1) or half of its columns
// (LPP = 2): every output row is WOL independent accumulations (no shuffles, no cross-lane
// data), the rows are fully unrolled with a ring of K input rows in registers, and a plane
// stride that is odd (7x7) keeps the lanes' shared loads in different banks. Outputs go to a
// shared-memory staging area and leave as one contiguous, coalesced range of y. Each warp keeps
// a ring of NB input buffers: its first NB jobs are copied at once, and a buffer is refilled
// with the job NB ahead as soon as the compute has read it.
#pragma once
#include <cstdint>

#include "depthwise.cuh"
#include "depthwise_tma.cuh"   // packed-pair helpers
#include "ptx.cuh"

namespace convb200 {

struct DwPlaneParams {
    int C;               // channels (= planes per image, multiplier 1)
    int num_planes;      // N * C
    int num_jobs;        // ceil(num_planes / planes per job)
    int in_floats;       // one input buffer (planes per job * HW * HW, rounded to 32 floats)
    int out_floats;      // per-warp output staging (planes per job * HO * WO, rounded to 32 floats)
    int nbuf;            // input buffers per warp (1 .. kDwPlaneMaxBuf): jobs staged ahead
    int vec_y;           // 1: y 16-byte aligned
    FastDiv div_c;
};

constexpr int kDwPlaneWarps = 4;
constexpr int kDwPlaneMaxBuf = 4;

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

template <int MODE, bool HAS_BIAS, int K, int S, int HW>
__global__ void __launch_bounds__(32 * kDwPlaneWarps)
depthwise_plane_kernel(const float *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias,
                       float *__restrict__ y, const DwPlaneParams p, unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int PAD = (K - 1) / 2;
    constexpr int HO = (HW + 2 * PAD - K) / S + 1;
    constexpr int WO = HO;
    constexpr int LPP = HW <= 8 ? 1 : 2;            // lanes per plane
    constexpr int PPJ = 32 / LPP;                   // planes per job
    constexpr int WOL = (WO + LPP - 1) / LPP;       // output columns per lane
    constexpr int WINC = (WOL - 1) * S + K;         // input columns a lane reads per row
    extern __shared__ __align__(128) float sraw[];
    __shared__ __align__(8) uint64_t full_all[kDwPlaneWarps][kDwPlaneMaxBuf];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int NB = p.nbuf;
    float *sin0 = sraw + static_cast<size_t>(warp) * (NB * p.in_floats + p.out_floats);
    float *sout = sin0 + NB * p.in_floats;
    const uint32_t sin_s = static_cast<uint32_t>(__cvta_generic_to_shared(sin0));
    const uint32_t bar0 = static_cast<uint32_t>(__cvta_generic_to_shared(&full_all[warp][0]));
    auto bar = [&](int b) { return bar0 + 8u * b; };
    const int gw = blockIdx.x * kDwPlaneWarps + warp;
    const int GW = gridDim.x * kDwPlaneWarps;

    // stage job `job` into buffer b: its planes are one contiguous range of x; the 16-byte
    // multiple goes by one bulk copy, the last 0..3 floats by lane 0
    auto issue = [&](int job, int b) {
        const int plane0 = job * PPJ;
        const int nplanes = min(PPJ, p.num_planes - plane0);
        const uint32_t total = static_cast<uint32_t>(nplanes * HW * HW);
        const uint32_t bulk = total & ~3u;
        const float *src = x + static_cast<long long>(plane0) * (HW * HW);
        if (lane == 0) {
            // the job's range of x, checked in the bounds-checked debug build (a skipped copy
            // still completes the barrier's byte count)
            const bool in = in_bounds(static_cast<long long>(plane0) * (HW * HW), total,
                                      1LL * p.num_planes * (HW * HW), kSiteDwPlaneX, status);
            float *dst = sin0 + b * p.in_floats;
            if (in)
                for (uint32_t e = bulk; e < total; ++e) dst[e] = src[e];
            mbar_arrive_expect_tx(bar(b), 4u * bulk);
            if (bulk) {
                if (in) bulk_g2s(sin_s + 4u * b * p.in_floats, src, 4u * bulk, bar(b));
                else mbar_complete_tx(bar(b), 4u * bulk);
            }
        }
    };

    if (lane == 0) {
        for (int b = 0; b < NB; ++b) mbar_init(bar(b), 1);
        fence_barrier_init();
    }
    __syncwarp();
    // the warp's first NB jobs go in flight at once
    for (int b = 0; b < NB; ++b)
        if (gw + b * GW < p.num_jobs) issue(gw + b * GW, b);

    const int slot = lane / LPP;          // plane slot of this lane in the job
    const int part = lane - slot * LPP;   // column part
    const int ox0 = part * WOL;
    const int ix0 = ox0 * S - PAD;        // first input column this lane reads

    int k = 0;
    bool ok = true;
    for (int job = gw; job < p.num_jobs; job += GW, ++k) {
        const int b = k % NB;
        const float *pb = sin0 + b * p.in_floats + slot * (HW * HW);
        const int plane0 = job * PPJ;
        const int plane = plane0 + slot;
        const bool active = plane < p.num_planes;
        const int c = active ? plane - fdiv(plane, p.div_c) * p.C : 0;
        // the plane's weights load while the bulk copy is in flight
        float wr[K * K];
#pragma unroll
        for (int t = 0; t < K * K; ++t) wr[t] = __ldg(w + c * (K * K) + t);
        const float bv = HAS_BIAS ? __ldg(bias + c) : 0.0f;
        if (!mbar_wait_warp(bar(b), (k / NB) & 1)) { ok = false; break; }

        // input row iy (compile-time) of this lane's columns; zeros outside the plane
        auto load_row = [&](int iy, float (&row)[WINC]) {
#pragma unroll
            for (int t = 0; t < WINC; ++t) {
                const int col = ix0 + t;
                row[t] = (iy >= 0 && iy < HW && col >= 0 && col < HW) ? pb[iy * HW + col] : 0.0f;
            }
        };
        auto store_row = [&](int oy, const float (&acc)[WOL]) {
#pragma unroll
            for (int v = 0; v < WOL; ++v)
                if (ox0 + v < WO) sout[slot * (HO * WO) + oy * WO + ox0 + v] = acc[v];
        };
        if constexpr (S == 1) {
            // stride 1: the ring holds each row as its WINC - 1 overlapping pairs (x[t], x[t+1]);
            // outputs (2q, 2q+1) at tap kx read pair 2q + kx (packed f32x2 arithmetic, the same
            // roundings as the scalar path)
            uint64_t w2[K * K];
#pragma unroll
            for (int t = 0; t < K * K; ++t) w2[t] = dw_pack(wr[t], wr[t]);
            uint64_t ring[K][WINC - 1];
            // element t of a row held as pairs: the low half of pair t, or for the last element
            // the high half of the last pair
            auto pair_elem = [&](const uint64_t (&row)[WINC - 1], int t) {
                float lo, hi;
                dw_unpack(row[t < WINC - 1 ? t : WINC - 2], lo, hi);
                return t < WINC - 1 ? lo : hi;
            };
            auto load_pairs = [&](int iy, uint64_t (&dst)[WINC - 1]) {
                float f[WINC];
                load_row(iy, f);
#pragma unroll
                for (int t = 0; t < WINC - 1; ++t) dst[t] = dw_pack(f[t], f[t + 1]);
            };
#pragma unroll
            for (int r = 0; r < K - 1; ++r) load_pairs(r - PAD, ring[r]);
#pragma unroll
            for (int oy = 0; oy < HO; ++oy) {
                load_pairs(oy - PAD + K - 1, ring[(oy + K - 1) % K]);
                float acc[WOL];
                constexpr int NP = WOL / 2;
                {
                    uint64_t a2[NP > 0 ? NP : 1];
#pragma unroll
                    for (int q = 0; q < NP; ++q) a2[q] = dw_pack(0.0f, 0.0f);
                    float last = 0.0f;
#pragma unroll
                    for (int ky = 0; ky < K; ++ky)
#pragma unroll
                        for (int kx = 0; kx < K; ++kx) {
#pragma unroll
                            for (int q = 0; q < NP; ++q)
                                a2[q] = dw_tap2<MODE>(a2[q], w2[ky * K + kx], ring[(oy + ky) % K][2 * q + kx]);
                            if constexpr (WOL % 2 == 1)
                                last = dw_tap<MODE>(last, wr[ky * K + kx], pair_elem(ring[(oy + ky) % K], WOL - 1 + kx));
                        }
#pragma unroll
                    for (int q = 0; q < NP; ++q) dw_unpack(a2[q], acc[2 * q], acc[2 * q + 1]);
                    if constexpr (WOL % 2 == 1) acc[WOL - 1] = last;
                }
#pragma unroll
                for (int v = 0; v < WOL; ++v) acc[v] = dw_finish<MODE, HAS_BIAS>(acc[v], bv);
                store_row(oy, acc);
            }
        } else {
            float ring[K][WINC];
#pragma unroll
            for (int r = 0; r < K - S; ++r) load_row(r - PAD, ring[(r + K) % K]);
#pragma unroll
            for (int oy = 0; oy < HO; ++oy) {
                // window rows oy*S - PAD + ky; ring slot of input row iy: (iy + PAD) % K
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const int iy = oy * S - PAD + K - S + s;
                    load_row(iy, ring[(iy + PAD + K) % K]);
                }
                float acc[WOL];
#pragma unroll
                for (int v = 0; v < WOL; ++v) {
                    float a = 0.0f;
#pragma unroll
                    for (int ky = 0; ky < K; ++ky)
#pragma unroll
                        for (int kx = 0; kx < K; ++kx)
                            a = dw_tap<MODE>(a, wr[ky * K + kx], ring[(oy * S + ky) % K][v * S + kx]);
                    acc[v] = dw_finish<MODE, HAS_BIAS>(a, bv);
                }
                store_row(oy, acc);
            }
        }
        // input buffer b is free: stage the job NB ahead while this one's outputs leave
        __syncwarp();
        if (job + NB * GW < p.num_jobs) issue(job + NB * GW, b);
        const int nplanes = min(PPJ, p.num_planes - plane0);
        const int total = nplanes * (HO * WO);
        float *gdst = y + static_cast<long long>(plane0) * (HO * WO);
        if (!in_bounds(static_cast<long long>(plane0) * (HO * WO), total, 1LL * p.num_planes * (HO * WO), kSiteDwPlaneY,
                       status)) {
            // skipped (bounds-checked debug build)
        } else if (p.vec_y && ((plane0 * (HO * WO)) & 3) == 0) {
            const int n4 = total >> 2;
            for (int e = lane; e < n4; e += 32)
                reinterpret_cast<float4 *>(gdst)[e] = reinterpret_cast<const float4 *>(sout)[e];
            for (int e = (n4 << 2) + lane; e < total; e += 32) gdst[e] = sout[e];
        } else {
            for (int e = lane; e < total; e += 32) gdst[e] = sout[e];
        }
        __syncwarp();
    }
    if (!ok) {
        if (lane == 0) atomicOr(status, kStatusTimeout);
        // the copies in flight (jobs k .. k + NB - 1) land before the warp exits (bounded waits)
        for (int kk = k; kk < k + NB; ++kk)
            if (gw + kk * GW < p.num_jobs) mbar_wait_warp(bar(kk % NB), (kk / NB) & 1);
    }
}

}  // namespace convb200
