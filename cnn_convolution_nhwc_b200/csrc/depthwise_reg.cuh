// Depthwise forward convolution on NCHW float32 planes with the input window held in
// registers: no shared memory.
//
// Same contract as depthwise.cuh (the OneModel "Depthwise convolution" page, section "What
// each output is": acc = +0; ky outer, kx inner; padding a real zero that is multiplied;
// exact mode __fmul_rn then __fadd_rn with NaN rewritten as 0x7FC00000; fast mode one
// __fmaf_rn per tap; the bias one rounded addition afterwards). This kernel serves the
// compile-time shapes K x K, stride S, padding PAD, dilation 1.
//
// Work layout. Lanes are neighbouring output columns (the page's layout), 4 per lane: lane g
// of a plane owns output columns 4g .. 4g+3 and input columns 4gS .. 4gS+4S-1, which it reads
// with coalesced (128-bit where aligned) loads. The other input columns its filter windows
// need -- PAD to the left, the rest to the right -- are the neighbouring lanes' columns and
// arrive by warp shuffles; outside the image they are real zeros. A warp walks down a band
// of output rows keeping the K input rows in registers (a rolling window), so every input row
// is loaded once per band; the weights of the plane stay in registers. Narrow planes put
// several planes in one warp (32 / lanes-per-plane of them). Every output is computed
// independently in the one tap order, so results are bit-identical to the shared-memory
// kernel.
#pragma once
#include <cstdint>

#include "depthwise.cuh"

namespace convb200 {

struct DwRegParams {
    int Cin, mult, Cout, H, W, Ho, Wo;
    int lpp;          // lanes per plane: ceil(Wo / 4)
    int ppw;          // planes per warp: 32 / lpp
    int band;         // output rows per warp job
    int nbands;       // ceil(Ho / band)
    int num_planes;   // N * Cout
    int num_jobs;     // ceil(num_planes / ppw) * nbands
    int vec_in;       // 1: 128-bit input loads (W % 4 == 0 and x 16-byte aligned)
    int vec_out;      // 1: 128-bit output stores (Wo % 4 == 0 and y 16-byte aligned)
    FastDiv div_cout, div_mult, div_nbands, div_lpp;
};

template <int MODE, bool HAS_BIAS, int K, int S, int PAD>
__global__ void __launch_bounds__(256)
depthwise_reg_kernel(const float *__restrict__ x, const float *__restrict__ w,
                     const float *__restrict__ bias, float *__restrict__ y, const DwRegParams p,
                     unsigned int *status) {
    grid_dependents_launch();   // programmatic dependent launch (see ptx.cuh)
    grid_dependency_wait();
    constexpr int VX = 4;                    // outputs per lane along the row
    constexpr int OWN = VX * S;              // input columns a lane loads per row
    constexpr int WIN = (VX - 1) * S + K;    // input columns one lane's outputs read per row
    static_assert(PAD <= OWN && WIN - PAD <= 2 * OWN, "window must come from this lane and its neighbours");
    const int lane = threadIdx.x & 31;
    const int job = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (job >= p.num_jobs) return;   // whole warp leaves together; no block-wide barrier below

    const int pg = fdiv(job, p.div_nbands);
    const int band_idx = job - pg * p.nbands;
    const int ps = fdiv(lane, p.div_lpp);          // plane slot of this lane
    const int cg = lane - ps * p.lpp;              // column group within the plane
    const int plane = pg * p.ppw + ps;
    const bool active = ps < p.ppw && plane < p.num_planes;
    const int n = active ? fdiv(plane, p.div_cout) : 0;
    const int oc = active ? plane - n * p.Cout : 0;
    const int ic = fdiv(oc, p.div_mult);
    const float *xp = x + (static_cast<long long>(n) * p.Cin + ic) * p.H * static_cast<long long>(p.W);
    float *yp = y + static_cast<long long>(active ? plane : 0) * p.Ho * static_cast<long long>(p.Wo);

    float wr[K * K];
#pragma unroll
    for (int t = 0; t < K * K; ++t) wr[t] = active ? __ldg(w + static_cast<long long>(oc) * (K * K) + t) : 0.0f;
    const float b = (HAS_BIAS && active) ? __ldg(bias + oc) : 0.0f;

    const int c0 = cg * OWN;                       // first input column this lane owns
    const int oy0 = band_idx * p.band;
    const int nrows = min(p.band, p.Ho - oy0);
    const bool lane_has_cols = active && c0 < p.W;

    // tensor extents for the bounds-checked debug build
    const long long x_elems = 1LL * (p.num_planes / p.Cout) * p.Cin * p.H * p.W;
    const long long y_elems = 1LL * p.num_planes * p.Ho * p.Wo;
    // loads this lane's OWN columns of input row r (zeros outside the image)
    auto load_own = [&](int r, float (&own)[OWN]) {
        bool row_ok = lane_has_cols && r >= 0 && r < p.H;
        const float *src = xp + static_cast<long long>(row_ok ? r : 0) * p.W + c0;
        if (row_ok)
            row_ok = in_bounds(src - x, min(OWN, p.W - c0), x_elems, kSiteDwRegX, status);
        if (p.vec_in && row_ok && c0 + OWN <= p.W) {
#pragma unroll
            for (int q = 0; q < OWN / 4; ++q) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(src) + q);
                own[4 * q] = v.x; own[4 * q + 1] = v.y; own[4 * q + 2] = v.z; own[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < OWN; ++i) own[i] = (row_ok && c0 + i < p.W) ? __ldg(src + i) : 0.0f;
        }
    };
    // window column t is input column c0 - PAD + t: from the left neighbour, this lane, or
    // the right neighbour (zero when that lane belongs to another plane or is past the edge)
    auto assemble = [&](const float (&own)[OWN], float (&win)[WIN]) {
#pragma unroll
        for (int t = 0; t < WIN; ++t) {
            const int src = t - PAD;
            const int dl = src < 0 ? -1 : (src >= OWN ? 1 : 0);
            const int idx = src - dl * OWN;
            if (dl == 0) {
                win[t] = own[idx];
            } else {
                const float v = __shfl_sync(0xffffffffu, own[idx], (lane + dl) & 31);
                const int ncg = cg + dl;
                win[t] = (ncg >= 0 && ncg < p.lpp && lane + dl >= 0 && lane + dl < 32) ? v : 0.0f;
            }
        }
    };

    float rows[K][WIN];
    {
        float own[OWN];
#pragma unroll
        for (int ky = 0; ky < K; ++ky) {
            load_own(oy0 * S - PAD + ky, own);
            assemble(own, rows[ky]);
        }
    }
    // L2 prefetch of the input rows AHEAD output rows ahead: more bytes in flight per warp
    // without holding them in registers (one prefetch per lane per row; lanes of a 128-byte
    // line repeat it, which is cheaper than computing a leader)
    constexpr int AHEAD = S == 1 ? 4 : 2;
    auto prefetch_row = [&](int r) {
        if (lane_has_cols && r >= 0 && r < p.H)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(xp + static_cast<long long>(r) * p.W + c0));
    };
#pragma unroll
    for (int a = 1; a <= AHEAD; ++a)
#pragma unroll
        for (int s = 0; s < S; ++s) prefetch_row((oy0 + 1 + a) * S - PAD + (K - S) + s);
    float nxt[S][OWN];
#pragma unroll
    for (int s = 0; s < S; ++s) load_own((oy0 + 1) * S - PAD + (K - S) + s, nxt[s]);

    for (int i = 0; i < nrows; ++i) {
        const int oy = oy0 + i;
        float acc[VX];
#pragma unroll
        for (int v = 0; v < VX; ++v) {
            float a = 0.0f;
#pragma unroll
            for (int ky = 0; ky < K; ++ky)
#pragma unroll
                for (int kx = 0; kx < K; ++kx) a = dw_tap<MODE>(a, wr[ky * K + kx], rows[ky][v * S + kx]);
            acc[v] = dw_finish<MODE, HAS_BIAS>(a, b);
        }
        const int ox = cg * VX;
        if (active && ox < p.Wo) {
            float *dst = yp + static_cast<long long>(oy) * p.Wo + ox;
            if (!in_bounds(dst - y, min(VX, p.Wo - ox), y_elems, kSiteDwRegY, status)) {
                // skipped (bounds-checked debug build)
            } else if (p.vec_out && ox + VX <= p.Wo) {
                *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            } else {
#pragma unroll
                for (int v = 0; v < VX; ++v)
                    if (ox + v < p.Wo) dst[v] = acc[v];
            }
        }
        // advance the window by S input rows; the next loads are already in flight
#pragma unroll
        for (int ky = 0; ky < K - S; ++ky)
#pragma unroll
            for (int t = 0; t < WIN; ++t) rows[ky][t] = rows[ky + S][t];
#pragma unroll
        for (int s = 0; s < S; ++s) assemble(nxt[s], rows[K - S + s]);
        if (i + 1 < nrows) {
#pragma unroll
            for (int s = 0; s < S; ++s) load_own((oy + 2) * S - PAD + (K - S) + s, nxt[s]);
            if (i + 2 + AHEAD <= nrows) {
#pragma unroll
                for (int s = 0; s < S; ++s) prefetch_row((oy + 2 + AHEAD) * S - PAD + (K - S) + s);
            }
        }
    }
}

}  // namespace convb200
