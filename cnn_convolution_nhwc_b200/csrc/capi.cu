// C ABI of the library: argument checks, path choice, TMA tensor maps, launches.
//
// Every entry point validates its arguments before touching CUDA, so a rejected call has
// no device-side effect. Validation mirrors the teaching implementation of the CMU DLSys
// Lecture 14 notes, section 5 (positive dimensions, square filter no larger than the
// image, matching shapes) and the output-size rule of "Convolution Is Wx+b Moving Across a
// Signal" (section "Build an image-gradient map, one number at a time") for depthwise.
#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "../../include/conv_b200.h"
#include "dense_direct.cuh"
#include "dense_tc.cuh"
#include "dense_halo.cuh"
#include "dense_fold.cuh"
#include "dense_stream.cuh"
#include "dense_halo_pad.cuh"
#include "im2col_gemm.cuh"
#include "depthwise.cuh"
#include "depthwise_reg.cuh"
#include "depthwise_tma.cuh"
#include "depthwise_plane.cuh"
#include "dwpw.cuh"
#include "dwpw_gemm.cuh"
#include "ptx.cuh"

namespace convb200 {

// One status word per device; kernels set bits in it with atomicOr.
__device__ unsigned int g_conv_status;

// Scratch of conv2d_nhwc_fwd_im2col_noalloc (its patch matrix), reserved once in every device
// that loads the library. In host code the name is only a host-side stand-in for the array:
// the device address comes from cudaGetSymbolAddress, taken once per device with that device
// current (DeviceState::im2col_scratch). Device code never names it; the kernels get the
// address as an argument like any caller buffer.
static __device__ __align__(256) unsigned char g_im2col_scratch[CONV_IM2COL_STATIC_BYTES];

// One CTA waiting on a barrier that nothing completes: exercises the bounded wait.
__global__ void selftest_wait_kernel(unsigned int *status) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(b, 0)) atomicOr(status, kStatusTimeout);
}

// One thread that checks an element range lying past its (notional) tensor and touches no
// memory either way: in the bounds-checked build the check fails and is recorded.
__global__ void selftest_bounds_kernel(unsigned int *status) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        volatile bool ok = in_bounds(1000, 1, 1000, kSiteSelftest, status);
        (void)ok;
    }
}

namespace {

// family name of the kernel the last successful launch on this host thread used
thread_local const char *t_last_kernel = "";

int launched(cudaError_t e, const char *name) {
    if (e != cudaSuccess) return CONV_ERR_CUDA;
    t_last_kernel = name;
    return CONV_OK;
}

constexpr int kMaxDevices = 64;
constexpr long long kInt32Max = 2147483647LL;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using EncodeIm2colFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const int *, const int *,
                                    cuuint32_t, cuuint32_t, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    unsigned int *status = nullptr;   // device address of g_conv_status on this device
    std::atomic<unsigned long long> attr_done[2] = {{0}, {0}};   // bit per kernel whose shared-memory limit is raised
    cublasHandle_t blas = nullptr;    // for the explicit-im2col comparison path, made on first use
    void *im2col_scratch = nullptr;   // device address of g_im2col_scratch on this device
    // clusters of a kernel that fit on the device at once, per (kernel bit, cluster size, shared
    // memory), asked once (outside any stream capture: the first call of a shape runs eagerly)
    struct ClusterFit {
        unsigned bit;
        int S, smem, active;
    };
    ClusterFit cluster_fit[64];
    int n_cluster_fit = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
EncodeTiledFn g_encode_tiled = nullptr;
EncodeIm2colFn g_encode_im2col = nullptr;

// Per-device set-up, done once with that device current.
int device_state(DeviceState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CONV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return CONV_ERR_CUDA;
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_conv_status) != cudaSuccess) return CONV_ERR_CUDA;
        d.status = static_cast<unsigned int *>(addr);
        d.ready = true;
    }
    if (!g_encode_tiled || !g_encode_im2col) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
            return CONV_ERR_CUDA;
        g_encode_tiled = reinterpret_cast<EncodeTiledFn>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeIm2col", &fn, 12000, cudaEnableDefault, &q) !=
                cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
            return CONV_ERR_CUDA;
        g_encode_im2col = reinterpret_cast<EncodeIm2colFn>(fn);
    }
    *out = &d;
    return CONV_OK;
}

template <typename Kern>
int ensure_smem_attr(DeviceState *d, unsigned bit, Kern kern, int bytes) {
    const unsigned long long mask = 1ull << (bit & 63);
    if (d->attr_done[bit >> 6].load(std::memory_order_acquire) & mask) return CONV_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return CONV_ERR_CUDA;
    d->attr_done[bit >> 6].fetch_or(mask, std::memory_order_release);
    return CONV_OK;
}

// Clusters of S CTAs (`threads` threads, `smem` dynamic bytes) of kernel `kern` that the device
// holds at once, asked once per (kernel bit, S, shared memory) and cached: a persistent grid of
// clusters larger than that would run its last clusters after the others. 0 on failure.
template <typename Kern>
int cluster_fit(DeviceState *d, unsigned bit, Kern kern, int S, int smem, int threads) {
    {
        std::lock_guard<std::mutex> lock(g_mu);
        for (int i = 0; i < d->n_cluster_fit; ++i) {
            const DeviceState::ClusterFit &f = d->cluster_fit[i];
            if (f.bit == bit && f.S == S && f.smem == smem) return f.active;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(S));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess) active = 0;
    std::lock_guard<std::mutex> lock(g_mu);
    if (d->n_cluster_fit < 64) d->cluster_fit[d->n_cluster_fit++] = DeviceState::ClusterFit{bit, S, smem, active};
    return active;
}

// Every tensor of a call must be device memory of the current device (or managed memory): the
// kernels launch on the current device, and a buffer of another GPU, or host memory, would be
// read through the wrong mapping. Null pointers (absent biases) are skipped. While `stream` is
// being captured into a CUDA graph the check is skipped (the capture records launches only;
// the same call made eagerly beforehand is checked).
int check_device_ptrs(cudaStream_t stream, std::initializer_list<const void *> ptrs) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return CONV_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return CONV_OK;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CONV_ERR_CUDA;
    for (const void *p : ptrs) {
        if (!p) continue;
        cudaPointerAttributes a{};
        if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
            cudaGetLastError();   // clear the (non-sticky) error this query left behind
            return CONV_ERR_INVALID_ARG;
        }
        if (a.type == cudaMemoryTypeManaged) continue;
        if (a.type != cudaMemoryTypeDevice || a.device != dev) return CONV_ERR_INVALID_ARG;
    }
    return CONV_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlaps(const void *a, long long abytes, const void *b, long long bbytes) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

const char *env(const char *name) {
    const char *v = std::getenv(name);
    return (v && *v) ? v : nullptr;
}

// An integer setting from the environment, clamped to [lo, hi]; `def` when unset.
int env_int(const char *name, int def, int lo, int hi) {
    const char *v = env(name);
    int r = v ? std::atoi(v) : def;
    if (r < lo) r = lo;
    if (r > hi) r = hi;
    return r;
}

// Every kernel launch allows programmatic dependent launch: the next kernel on the stream may be
// scheduled while this one drains, because each kernel waits for its predecessors before its
// first global-memory access (grid_dependency_wait). CONV_B200_PDL=0 launches without it
// (measurements).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(cudaLaunchConfig_t cfg, void (*kern)(KArgs...), Args... args) {
    cudaLaunchAttribute attrs[4];
    unsigned n = 0;
    for (unsigned i = 0; i < cfg.numAttrs && n < 3; ++i) attrs[n++] = cfg.attrs[i];
    if (env_int("CONV_B200_PDL", 1, 0, 1) == 1) {
        attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}


// ---------------------------------------------------------------------------------------
// Dense
// ---------------------------------------------------------------------------------------
int check_dense(const void *X, const void *F, const void *Y, int N, int H, int W, int Cin, int Cout,
                int K, int elem) {
    if (!X || !F || !Y) return CONV_ERR_INVALID_ARG;
    if (N < 1 || H < 1 || W < 1 || Cin < 1 || Cout < 1 || K < 1) return CONV_ERR_INVALID_ARG;
    if (K > H || K > W) return CONV_ERR_INVALID_ARG;
    const long long Ho = H - K + 1, Wo = W - K + 1;
    const long long nx = 1LL * N * H * W * Cin, nf = 1LL * K * K * Cin * Cout, ny = 1LL * N * Ho * Wo * Cout;
    if (nx > kInt32Max || nf > kInt32Max || ny > kInt32Max || 1LL * N * Ho * Wo > kInt32Max)
        return CONV_ERR_UNSUPPORTED;
    if (!aligned(X, elem) || !aligned(F, elem) || !aligned(Y, elem)) return CONV_ERR_MISALIGNED;
    if (overlaps(Y, ny * elem, X, nx * elem) || overlaps(Y, ny * elem, F, nf * elem))
        return CONV_ERR_INVALID_ARG;
    return CONV_OK;
}

// Geometry of a dense convolution: a KH x KW filter, stride, zero padding and dilation per
// axis, channel groups and an optional bias. The plain operation is a square K with stride 1,
// no padding, dilation 1, one group and no bias.
struct DenseGeom {
    int KH = 1, KW = 1;
    int sh = 1, sw = 1, ph = 0, pw = 0, dh = 1, dw = 1;
    int ph_end = 0, pw_end = 0;   // zeros after the last row / column (ph, pw: before the first)
    int groups = 1;
    const float *bias = nullptr;
    static DenseGeom square(int K, int stride = 1, int pad = 0, int dil = 1, const float *bias = nullptr) {
        DenseGeom g;
        g.KH = g.KW = K;
        g.sh = g.sw = stride;
        g.ph = g.pw = g.ph_end = g.pw_end = pad;
        g.dh = g.dw = dil;
        g.bias = bias;
        return g;
    }
    // output extents; the caller has checked that the dilated filter fits the padded input
    long long ho(int H) const { return (1LL * H + ph + ph_end - (1LL * dh * (KH - 1) + 1)) / sh + 1; }
    long long wo(int W) const { return (1LL * W + pw + pw_end - (1LL * dw * (KW - 1) + 1)) / sw + 1; }
    bool plain() const {
        return KH == KW && sh == 1 && sw == 1 && ph == 0 && pw == 0 && ph_end == 0 && pw_end == 0 && dh == 1 &&
               dw == 1 && groups == 1 && bias == nullptr;
    }
};

template <typename T>
int launch_dense_direct(const T *X, const T *F, T *Y, int N, int H, int W, int Cin, int Cout, const DenseGeom &g,
                        cudaStream_t stream, DeviceState *d) {
    DenseDirectParams p;
    p.H = H; p.W = W; p.Cin = Cin; p.Cout = Cout; p.KH = g.KH; p.KW = g.KW;
    p.Ho = static_cast<int>(g.ho(H)); p.Wo = static_cast<int>(g.wo(W));
    p.Cin_g = Cin / g.groups; p.Cout_g = Cout / g.groups;
    p.sh = g.sh; p.sw = g.sw; p.ph = g.ph; p.pw = g.pw; p.dh = g.dh; p.dw = g.dw; p.bias = g.bias;
    p.total = 1LL * N * p.Ho * p.Wo * Cout;
    p.x_elems = 1LL * N * H * W * Cin;
    long long blocks = (p.total + 255) / 256;
    const long long cap = 1LL * d->num_sms * 16;
    if (blocks > cap) blocks = cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    return launched(launch_k(cfg, dense_direct_kernel<T>, X, F, Y, p, d->status), "dense_direct_kernel");
}

// The im2col tensor-core kernel over groups g0 .. g0 + NG - 1 per launch (one launch when
// there is one group). Per group: X channels g*Cin_g .. +Cin_g, filter and Y columns
// g*Cout_g .. +Cout_g; the caller guarantees Cin_g and Cout_g multiples of 8 (16-byte map
// bases) and window corners and tap reaches inside the 4-D im2col ranges.
template <class Cfg, int NG, bool PAIR = false>
int launch_dense_tc(const void *X, const void *F, void *Y, int N, int H, int W, int Cin, int Cout,
                    const DenseGeom &g, cudaStream_t stream, DeviceState *d, unsigned attr_bit) {
    const int Ho = static_cast<int>(g.ho(H)), Wo = static_cast<int>(g.wo(W));
    const int Cin_g = Cin / g.groups, Cout_g = Cout / g.groups;
    const long long M = 1LL * N * Ho * Wo;
    DenseTcParams p;
    p.M = static_cast<int>(M);
    p.Wo = Wo;
    p.HoWo = Ho * Wo;
    p.KW = g.KW;
    p.ncols = Cout_g;
    p.num_cblk = (Cin_g + 63) / 64;
    p.num_kblk = g.KH * g.KW * p.num_cblk;
    p.num_ntiles = (Cout_g + Cfg::BN - 1) / Cfg::BN;
    p.sh = g.sh; p.sw = g.sw; p.ph = g.ph; p.pw = g.pw; p.dh = g.dh; p.dw = g.dw;
    constexpr int TILE_ROWS = PAIR ? 2 * Cfg::BM : Cfg::BM;   // a CTA pair computes 256 rows per tile
    constexpr int SMEM = PAIR ? Cfg::SMEM_BYTES_PAIR : Cfg::SMEM_BYTES;
    const long long per_group = ((M + TILE_ROWS - 1) / TILE_ROWS) * p.num_ntiles;
    if (per_group * NG > kInt32Max) return CONV_ERR_UNSUPPORTED;
    p.tiles_per_group = static_cast<int>(per_group);
    auto kern = dense_tc_kernel<Cfg, NG, PAIR>;
    if (int rc = ensure_smem_attr(d, attr_bit, kern, SMEM)) return rc;
    const auto *xb = static_cast<const __nv_bfloat16 *>(X);
    const auto *fb = static_cast<const __nv_bfloat16 *>(F);
    auto *yb = static_cast<__nv_bfloat16 *>(Y);
    for (int g0 = 0; g0 < g.groups; g0 += NG) {
        const int ng = g.groups - g0 < NG ? g.groups - g0 : NG;
        DenseTcMaps<NG> maps;
        for (int gl = 0; gl < NG; ++gl) {
            // unused slots repeat the first group's maps (never dereferenced)
            const int gg = g0 + (gl < ng ? gl : 0);
            {   // X: 4-D {Cin_g, W, H, N} im2col at channel gg*Cin_g. The bounding box of window
                // origins runs from -pad_before to (size - 1) + pad_after - dil*(taps - 1) on each
                // spatial axis, walked with that axis's stride as element stride, so its pixels
                // are exactly the output positions; origins, taps and channels outside read zeros.
                const cuuint64_t dims[4] = {(cuuint64_t)Cin_g, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)N};
                const cuuint64_t strides[3] = {(cuuint64_t)Cin * 2, (cuuint64_t)W * Cin * 2,
                                               (cuuint64_t)H * W * Cin * 2};
                const int lower[2] = {-g.pw, -g.ph};
                const int upper[2] = {g.pw_end - g.dw * (g.KW - 1), g.ph_end - g.dh * (g.KH - 1)};
                const cuuint32_t estr[4] = {1, (cuuint32_t)g.sw, (cuuint32_t)g.sh, 1};
                if (g_encode_im2col(&maps.x[gl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                                    const_cast<__nv_bfloat16 *>(xb + 1LL * gg * Cin_g), dims, strides, lower, upper,
                                    64, Cfg::BM, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                    return CONV_ERR_CUDA;
            }
            {   // F: 3-D {Cout_g, Cin_g, KH*KW} at column gg*Cout_g; a box is 64 reduction rows
                // (channels) x 64 output channels
                const cuuint64_t dims[3] = {(cuuint64_t)Cout_g, (cuuint64_t)Cin_g, (cuuint64_t)g.KH * g.KW};
                const cuuint64_t strides[2] = {(cuuint64_t)Cout * 2, (cuuint64_t)Cin_g * Cout * 2};
                const cuuint32_t box[3] = {64, 64, 1};
                const cuuint32_t estr[3] = {1, 1, 1};
                if (g_encode_tiled(&maps.f[gl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                                   const_cast<__nv_bfloat16 *>(fb + 1LL * gg * Cout_g), dims, strides, box, estr,
                                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                    return CONV_ERR_CUDA;
            }
            {   // Y: 2-D {Cout_g, M} at column gg*Cout_g; a box is 32 rows x 64 channels
                const cuuint64_t dims[2] = {(cuuint64_t)Cout_g, (cuuint64_t)M};
                const cuuint64_t strides[1] = {(cuuint64_t)Cout * 2};
                const cuuint32_t box[2] = {64, 32};
                const cuuint32_t estr[2] = {1, 1};
                if (g_encode_tiled(&maps.y[gl], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, yb + 1LL * gg * Cout_g, dims,
                                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                    return CONV_ERR_CUDA;
            }
        }
        p.groups = ng;
        p.num_tiles = ng * p.tiles_per_group;
        p.bias = g.bias ? g.bias + 1LL * g0 * Cout_g : nullptr;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(p.num_tiles < d->num_sms ? p.num_tiles : d->num_sms));
        cfg.blockDim = dim3(192);
        cfg.dynamicSmemBytes = SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        if (PAIR) {
            // 2-CTA clusters, no more than the device holds at once (the grid is persistent)
            const int fit = cluster_fit(d, attr_bit, kern, 2, SMEM, 192);
            if (fit < 1) return CONV_ERR_CUDA;
            const int pairs = p.num_tiles < fit ? p.num_tiles : fit;
            cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
        }
        if (int rc = launched(launch_k(cfg, kern, maps, p, d->status), "dense_tc_kernel")) return rc;
    }
    return CONV_OK;
}

// ---- halo kernel ------------------------------------------------------------------------
constexpr int kSmemLimit = 232448;   // 227 KB of dynamic shared memory per CTA

struct HaloPlan {
    bool ok = false;
    int bn = 0;
    bool bres = false;
    DenseHaloParams p{};
    int smem = 0;
    int grid = 0;
};

template <int BN, bool BRES>
int halo_fixed_bytes() { return DenseHaloCfg<BN, BRES>::FIXED_BYTES; }

// Picks tile width, filter residency and ring depths so that everything fits in shared
// memory; returns !ok when even one halo slot does not fit (the im2col kernel then runs).
HaloPlan plan_halo(int N, int H, int W, int Cin, int Cout, int K, int num_sms, int force_bn) {
    HaloPlan pl;
    const long long rows = 1LL * N * H * W;
    if (rows + 1024 > kInt32Max) return pl;
    const int need = 128 + (K - 1) * W + (K - 1);
    if (need > 4096) return pl;
    const int n_boxes = (need + 255) / 256;
    const int box_rows = (((need + n_boxes - 1) / n_boxes) + 7) & ~7;
    const int halo_rows = n_boxes * box_rows;
    const int halo_bytes = halo_rows * 128;
    const int num_cblk = (Cin + 63) / 64;
    const int num_kblk = K * K * num_cblk;
    int bn = Cout <= 64 ? 64 : (Cout <= 128 ? 128 : 256);
    if (force_bn) bn = force_bn;
    const int b_bytes = 64 * bn * 2;
    const int fixed = bn == 64 ? halo_fixed_bytes<64, true>() : (bn == 128 ? halo_fixed_bytes<128, true>()
                                                                            : halo_fixed_bytes<256, true>());
    const int num_mtiles = static_cast<int>((rows + 127) / 128);
    const int num_ntiles = (Cout + bn - 1) / bn;
    DenseHaloParams &p = pl.p;
    // resident filter: the CTA's whole N-tile slice, loaded once
    const long long b_res = 1LL * num_kblk * b_bytes;
    if (b_res <= 128 * 1024 && num_ntiles <= num_sms && fixed + b_res + 2LL * halo_bytes <= kSmemLimit) {
        pl.bres = true;
        p.b_region = static_cast<int>(b_res);
        p.HS = static_cast<int>((kSmemLimit - fixed - b_res) / halo_bytes);
        p.BS = 1;
    } else {
        pl.bres = false;
        for (int bs : {4, 3, 2}) {
            const long long avail = kSmemLimit - fixed - 1LL * bs * b_bytes;
            if (avail >= 2LL * halo_bytes || (bs == 2 && avail >= halo_bytes)) {
                p.BS = bs;
                p.b_region = bs * b_bytes;
                p.HS = static_cast<int>(avail / halo_bytes);
                break;
            }
        }
        if (p.BS == 0) return pl;
    }
    if (p.HS > DenseHaloCfg<64, true>::MAX_RING) p.HS = DenseHaloCfg<64, true>::MAX_RING;
    if (p.HS < 1) return pl;
    p.rows = static_cast<int>(rows);
    p.H = H; p.W = W; p.Ho = H - K + 1; p.Wo = W - K + 1;
    p.K = K; p.KK = K * K; p.Cout = Cout;
    p.num_cblk = num_cblk;
    p.num_kblk = num_kblk;
    p.halo_rows = halo_rows;
    p.box_rows = box_rows;
    p.n_boxes = n_boxes;
    p.halo_bytes = halo_bytes;
    p.num_mtiles = num_mtiles;
    p.num_ntiles = num_ntiles;
    p.num_tiles = num_mtiles * num_ntiles;
    if (pl.bres && num_ntiles > 1) {
        p.n_fixed = 1;
        int per_n = num_sms / num_ntiles;
        if (per_n > num_mtiles) per_n = num_mtiles;
        pl.grid = per_n * num_ntiles;
    } else {
        p.n_fixed = 0;
        pl.grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    }
    pl.smem = fixed + p.b_region + p.HS * halo_bytes;
    // more than half of the shared memory keeps a second CTA (and its TMEM allocation) off the SM
    if (pl.smem < 116 * 1024) pl.smem = 116 * 1024;
    pl.bn = bn;
    pl.ok = pl.smem <= kSmemLimit && pl.grid >= 1;
    return pl;
}

template <class Cfg>
int launch_dense_halo(const void *X, const void *F, void *Y, int Cin, int Cout, int K, const HaloPlan &pl,
                      cudaStream_t stream, DeviceState *d, unsigned attr_bit) {
    alignas(64) CUtensorMap tmX, tmF;
    {   // X as a 2-D matrix: rows = flattened (n, y, x), Cin channels per row
        const cuuint64_t dims[2] = {(cuuint64_t)Cin, (cuuint64_t)pl.p.rows};
        const cuuint64_t strides[1] = {(cuuint64_t)Cin * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)pl.p.box_rows};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode_tiled(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    {   // F: 3-D {Cout, Cin, K*K}; a box is 64 reduction rows (channels) x 64 output channels
        const cuuint64_t dims[3] = {(cuuint64_t)Cout, (cuuint64_t)Cin, (cuuint64_t)K * K};
        const cuuint64_t strides[2] = {(cuuint64_t)Cout * 2, (cuuint64_t)Cin * Cout * 2};
        const cuuint32_t box[3] = {64, 64, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode_tiled(&tmF, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(F), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    auto kern = dense_halo_kernel<Cfg>;
    if (int rc = ensure_smem_attr(d, attr_bit, kern, kSmemLimit)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    return launched(launch_k(cfg, kern, tmX, tmF, static_cast<__nv_bfloat16 *>(Y), pl.p, d->status),
                    "dense_halo_kernel");
}

int dispatch_halo(const void *X, const void *F, void *Y, int Cin, int Cout, int K, const HaloPlan &pl,
                  cudaStream_t stream, DeviceState *d) {
    // shared-memory attribute bits 3..8
    if (pl.bn == 64) return pl.bres ? launch_dense_halo<DenseHaloCfg<64, true>>(X, F, Y, Cin, Cout, K, pl, stream, d, 3)
                                    : launch_dense_halo<DenseHaloCfg<64, false>>(X, F, Y, Cin, Cout, K, pl, stream, d, 4);
    if (pl.bn == 128) return pl.bres ? launch_dense_halo<DenseHaloCfg<128, true>>(X, F, Y, Cin, Cout, K, pl, stream, d, 5)
                                     : launch_dense_halo<DenseHaloCfg<128, false>>(X, F, Y, Cin, Cout, K, pl, stream, d, 6);
    return pl.bres ? launch_dense_halo<DenseHaloCfg<256, true>>(X, F, Y, Cin, Cout, K, pl, stream, d, 7)
                   : launch_dense_halo<DenseHaloCfg<256, false>>(X, F, Y, Cin, Cout, K, pl, stream, d, 28);
}

// ---- folded-tap kernel (Cout <= 64, K = 2..4) ---------------------------------------------
struct FoldPlan {
    bool ok = false;
    DenseFoldParams p{};
    int smem = 0;
    int grid = 0;
};

template <int KF>
int fold_fixed_bytes() { return DenseFoldCfg<KF>::FIXED_BYTES; }

FoldPlan plan_fold(int N, int H, int W, int Cin, int Cout, int K, int num_sms) {
    FoldPlan pl;
    if (Cout > 64 || K < 2 || K > 4) return pl;
    const long long rows = 1LL * N * H * W;
    if (rows + 1024 > kInt32Max) return pl;
    const int need = 128 + (K - 1) * W;
    if (need > 4096) return pl;
    const int n_boxes = (need + 255) / 256;
    const int box_rows = (((need + n_boxes - 1) / n_boxes) + 7) & ~7;
    const int halo_rows = n_boxes * box_rows;
    const int halo_bytes = halo_rows * 128;
    const int num_cblk = (Cin + 63) / 64;
    const int num_kblk = K * K * num_cblk;
    const int fixed = K == 2 ? fold_fixed_bytes<2>() : (K == 3 ? fold_fixed_bytes<3>() : fold_fixed_bytes<4>());
    const long long b_res = 1LL * num_kblk * DenseFoldCfg<2>::SLOT_BYTES;
    if (fixed + b_res + 2LL * halo_bytes > kSmemLimit) return pl;
    DenseFoldParams &p = pl.p;
    p.HS = static_cast<int>((kSmemLimit - fixed - b_res) / halo_bytes);
    if (p.HS > DenseFoldCfg<2>::MAX_RING) p.HS = DenseFoldCfg<2>::MAX_RING;
    const int TM = 128 - (K - 1);
    p.rows = static_cast<int>(rows);
    p.H = H; p.W = W; p.Ho = H - K + 1; p.Wo = W - K + 1;
    p.K = K; p.KK = K * K; p.Cout = Cout;
    p.num_cblk = num_cblk;
    p.num_kblk = num_kblk;
    p.halo_rows = halo_rows;
    p.box_rows = box_rows;
    p.n_boxes = n_boxes;
    p.halo_bytes = halo_bytes;
    p.b_region = static_cast<int>(b_res);
    p.num_tiles = static_cast<int>((rows + TM - 1) / TM);
    p.div_w = make_fastdiv(static_cast<uint32_t>(W));
    p.div_h = make_fastdiv(static_cast<uint32_t>(H));
    pl.grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    pl.smem = fixed + p.b_region + p.HS * halo_bytes;
    // more than half of the shared memory keeps a second CTA (and its TMEM allocation) off the SM
    if (pl.smem < 116 * 1024) pl.smem = 116 * 1024;
    pl.ok = pl.smem <= kSmemLimit;
    return pl;
}

template <int KF>
int launch_dense_fold(const void *X, const void *F, void *Y, int Cin, int Cout, const FoldPlan &pl,
                      cudaStream_t stream, DeviceState *d, unsigned attr_bit) {
    alignas(64) CUtensorMap tmX, tmF;
    {   // X as a 2-D matrix: rows = flattened (n, y, x), Cin channels per row
        const cuuint64_t dims[2] = {(cuuint64_t)Cin, (cuuint64_t)pl.p.rows};
        const cuuint64_t strides[1] = {(cuuint64_t)Cin * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)pl.p.box_rows};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode_tiled(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    {   // F: 3-D {Cout, Cin, K*K}; a box is 64 channels x 64 output channels of one tap
        const cuuint64_t dims[3] = {(cuuint64_t)Cout, (cuuint64_t)Cin, (cuuint64_t)KF * KF};
        const cuuint64_t strides[2] = {(cuuint64_t)Cout * 2, (cuuint64_t)Cin * Cout * 2};
        const cuuint32_t box[3] = {64, 64, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode_tiled(&tmF, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(F), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    auto kern = dense_fold_kernel<DenseFoldCfg<KF>>;
    if (int rc = ensure_smem_attr(d, attr_bit, kern, kSmemLimit)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(DenseFoldCfg<KF>::THREADS);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    return launched(launch_k(cfg, kern, tmX, tmF, static_cast<__nv_bfloat16 *>(Y), pl.p, d->status),
                    "dense_fold_kernel");
}

int dispatch_fold(const void *X, const void *F, void *Y, int Cin, int Cout, int K, const FoldPlan &pl,
                  cudaStream_t stream, DeviceState *d) {
    // shared-memory attribute bits 29..31
    if (K == 2) return launch_dense_fold<2>(X, F, Y, Cin, Cout, pl, stream, d, 29);
    if (K == 3) return launch_dense_fold<3>(X, F, Y, Cin, Cout, pl, stream, d, 30);
    return launch_dense_fold<4>(X, F, Y, Cin, Cout, pl, stream, d, 31);
}

// ---- streamed-filter kernel (256-row tiles, two accumulators per filter slot) -------------
struct StreamPlan {
    bool ok = false;
    bool pair = false;   // 2-CTA clusters sharing each filter slot (cta_group::2 MMAs)
    int bn = 0;
    DenseStreamParams p{};
    int smem = 0;
    int grid = 0;
};

// Halo slots of 32 channels by rows of the 256-row tile plus its (K-1)*W + K-1 reach, three of
// them when that leaves room for at least 8 filter slots (else two), and as many filter slots as
// fit (at least 4); !ok when the halo is too tall or the ring too shallow.
StreamPlan plan_stream(int N, int H, int W, int Cin, int Cout, int K, int num_sms) {
    StreamPlan pl;
    const long long rows = 1LL * N * H * W;
    if (rows + 2048 > kInt32Max) return pl;
    const long long need = 256 + 1LL * (K - 1) * W + (K - 1);
    if (need > 1024) return pl;
    const int n_boxes = static_cast<int>((need + 255) / 256);
    const int box_rows = ((static_cast<int>((need + n_boxes - 1) / n_boxes)) + 15) & ~15;
    const int halo_rows = n_boxes * box_rows;
    const int halo_bytes = halo_rows * 64;
    const int bn = Cout <= 64 ? 64 : 128;
    // BN = 128 runs as CTA pairs: each CTA stages half of every filter slot and the even CTA's
    // M = 256 MMAs read both halves, halving the filter traffic per tensor-core cycle
    // (CONV_B200_STREAM_PAIR=0 keeps one CTA per tile)
    const bool pair = bn == 128 && num_sms >= 2 && env_int("CONV_B200_STREAM_PAIR", 1, 0, 1) == 1;
    const int b_bytes = 32 * (pair ? 64 : bn) * 2;
    const int fixed = bn == 64 ? DenseStreamCfg<64>::FIXED_BYTES : DenseStreamCfg<128>::FIXED_BYTES;
    int hs = 3;
    long long avail = kSmemLimit - fixed - 3LL * halo_bytes;
    if (avail < 8LL * b_bytes) {
        hs = 2;
        avail = kSmemLimit - fixed - 2LL * halo_bytes;
    }
    long long bs = avail / b_bytes;
    if (bs > DenseStreamCfg<64>::MAX_BS) bs = DenseStreamCfg<64>::MAX_BS;
    if (bs < 4) return pl;
    DenseStreamParams &p = pl.p;
    p.rows = static_cast<int>(rows);
    p.H = H; p.W = W; p.Ho = H - K + 1; p.Wo = W - K + 1;
    p.K = K; p.KK = K * K; p.Cout = Cout;
    p.num_cblk = (Cin + 31) / 32;
    p.halo_rows = halo_rows;
    p.box_rows = box_rows;
    p.n_boxes = n_boxes;
    p.halo_bytes = halo_bytes;
    p.num_mtiles = static_cast<int>((rows + (pair ? 511 : 255)) / (pair ? 512 : 256));
    p.num_ntiles = (Cout + bn - 1) / bn;
    if (1LL * p.num_mtiles * p.num_ntiles > kInt32Max) return pl;
    p.num_tiles = p.num_mtiles * p.num_ntiles;
    p.HS = hs;
    p.BS = static_cast<int>(bs);
    pl.bn = bn;
    pl.pair = pair;
    pl.smem = fixed + p.BS * b_bytes + p.HS * halo_bytes;
    // more than half of the shared memory keeps a second CTA (and its TMEM allocation) off the SM
    if (pl.smem < 116 * 1024) pl.smem = 116 * 1024;
    if (pair) {
        const int pairs = num_sms / 2;
        pl.grid = 2 * (p.num_tiles < pairs ? p.num_tiles : pairs);
    } else {
        pl.grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    }
    pl.ok = pl.smem <= kSmemLimit;
    return pl;
}

template <int BN, bool PAIR>
int launch_dense_stream(const void *X, const void *F, void *Y, int Cin, int Cout, int K, const StreamPlan &pl,
                        cudaStream_t stream, DeviceState *d, unsigned attr_bit) {
    using Cfg = DenseStreamCfg<BN>;
    alignas(64) CUtensorMap tmX, tmF;
    {   // X as a 2-D matrix: rows = flattened (n, y, x), Cin channels per row; a box is 32
        // channels (64 bytes, 64-byte swizzle) x box_rows rows
        const cuuint64_t dims[2] = {(cuuint64_t)Cin, (cuuint64_t)pl.p.rows};
        const cuuint64_t strides[1] = {(cuuint64_t)Cin * 2};
        const cuuint32_t box[2] = {32, (cuuint32_t)pl.p.box_rows};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode_tiled(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    {   // F: 3-D {Cout, Cin, K*K}; a box is 32 reduction rows (channels) x 64 output channels
        const cuuint64_t dims[3] = {(cuuint64_t)Cout, (cuuint64_t)Cin, (cuuint64_t)K * K};
        const cuuint64_t strides[2] = {(cuuint64_t)Cout * 2, (cuuint64_t)Cin * Cout * 2};
        const cuuint32_t box[3] = {64, 32, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode_tiled(&tmF, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(F), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    auto kern = dense_stream_kernel<Cfg, PAIR>;
    if (int rc = ensure_smem_attr(d, attr_bit, kern, kSmemLimit)) return rc;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    if (PAIR) {
        // no more pairs than the device holds at once (the grid is persistent)
        const int fit = cluster_fit(d, attr_bit, kern, 2, pl.smem, Cfg::THREADS);
        if (fit < 1) return CONV_ERR_CUDA;
        if (static_cast<int>(cfg.gridDim.x) > 2 * fit) cfg.gridDim = dim3(static_cast<unsigned>(2 * fit));
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return launched(launch_k(cfg, kern, tmX, tmF, static_cast<__nv_bfloat16 *>(Y), pl.p, d->status),
                    "dense_stream_kernel");
}

using CfgBN64 = DenseTcCfg<64, 6>;
using CfgBN128 = DenseTcCfg<128, 5>;
using CfgBN256 = DenseTcCfg<256, 3>;

// ---------------------------------------------------------------------------------------
// Depthwise
// ---------------------------------------------------------------------------------------
constexpr int kDwSmemLimit = 48 * 1024;

long long dw_out(long long in, int k, int s, int pad, int dil) {
    return (in + 2LL * pad - (1LL * dil * (k - 1) + 1)) / s + 1;
}

// Compile-time specialisations: (KW, stride) with unit dilation, 4 outputs per thread.
enum DwSpec { kDwGeneric = 0, kDwK3S1, kDwK3S2, kDwK5S1, kDwK5S2 };

DwSpec dw_spec(const DwParams &p) {
    if (p.dil != 1) return kDwGeneric;
    if (p.KW == 3 && p.stride == 1) return kDwK3S1;
    if (p.KW == 3 && p.stride == 2) return kDwK3S2;
    if (p.KW == 5 && p.stride == 1) return kDwK5S1;
    if (p.KW == 5 && p.stride == 2) return kDwK5S2;
    return kDwGeneric;
}

int dw_vx(DwSpec s) { return s == kDwGeneric ? 1 : 4; }

long long dw_smem_bytes(const DwParams &p) {
    return 4LL * (dw_smem_head_floats(p.P, p.w_stride) + 1LL * p.P * p.rows_in * p.pitch);
}

// Staged window and shared-memory pitch for the current job shape. The pitch also covers
// the 128-bit window reads of the last strip of a row in the specialised kernels.
void dw_set_window(DwParams &p, DwSpec s) {
    p.rows_in = (p.R - 1) * p.stride + (p.KH - 1) * p.dil + 1;
    p.cols_in = (p.CW - 1) * p.stride + (p.KW - 1) * p.dil + 1;
    int need = p.cols_in;
    if (s != kDwGeneric) {
        const int vx = dw_vx(s);
        const int strips = (p.CW + vx - 1) / vx;
        const int win = (vx - 1) * p.stride + p.KW;
        const int reach = (strips - 1) * vx * p.stride + ((win + 3) / 4) * 4;
        if (reach > need) need = reach;
    }
    p.pitch = (need + 3) & ~3;
    int lg = 0;
    while ((1 << lg) < p.cols_in && lg < 8) ++lg;
    p.tc_log2 = lg;
}

// Job shape: about 2048 outputs per CTA, whole small planes grouped, column bands a
// multiple of the strip width, and a staged window within kDwSmemLimit.
void dw_choose_tiles(DwParams &p, DwSpec s) {
    constexpr int kTarget = 2048;
    const int vx = dw_vx(s);
    p.CW = p.Wo <= 128 ? p.Wo : 128;
    p.R = kTarget / p.CW;
    if (p.R < 1) p.R = 1;
    if (p.R > p.Ho) p.R = p.Ho;
    p.P = 1;
    if (p.R == p.Ho && p.CW == p.Wo) {
        long long P = kTarget / (1LL * p.Ho * p.Wo);
        if (P < 1) P = 1;
        if (P > 64) P = 64;
        if (P > p.num_planes) P = p.num_planes;
        p.P = static_cast<int>(P);
    }
    dw_set_window(p, s);
    while (dw_smem_bytes(p) > kDwSmemLimit) {
        if (p.P > 1) p.P = (p.P + 1) / 2;
        else if (p.R > 1) p.R = (p.R + 1) / 2;
        else if (p.CW > vx) p.CW = ((p.CW / 2 + vx - 1) / vx) * vx;
        else break;
        dw_set_window(p, s);
    }
}

template <int MODE, bool HB, int KW, int S, int VX>
int launch_dw_one(const float *x, const float *w, const float *bias, float *y, const DwParams &p, long long jobs,
                  cudaStream_t stream, DeviceState *d, unsigned bit) {
    auto kern = depthwise_kernel<MODE, HB, KW, S, VX>;
    const int smem = static_cast<int>(dw_smem_bytes(p));
    if (smem > 48 * 1024)
        if (int rc = ensure_smem_attr(d, bit, kern, 227 * 1024)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(jobs));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return launched(launch_k(cfg, kern, x, w, bias, y, p, d->status), "depthwise_kernel");
}

// ---- register-window kernel ---------------------------------------------------------------
template <int MODE, bool HB, int K, int S>
int launch_dw_reg_one(const float *x, const float *w, const float *bias, float *y, const DwRegParams &rp,
                      cudaStream_t stream, DeviceState *d) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((rp.num_jobs + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    return launched(launch_k(cfg, depthwise_reg_kernel<MODE, HB, K, S, (K - 1) / 2>, x, w, bias, y, rp,
                                       d->status),
                    "depthwise_reg_kernel");
}

template <int MODE, bool HB>
int launch_dw_reg(const float *x, const float *w, const float *bias, float *y, const DwRegParams &rp, int K, int S,
                  cudaStream_t stream, DeviceState *d) {
    if (K == 3 && S == 1) return launch_dw_reg_one<MODE, HB, 3, 1>(x, w, bias, y, rp, stream, d);
    if (K == 3 && S == 2) return launch_dw_reg_one<MODE, HB, 3, 2>(x, w, bias, y, rp, stream, d);
    if (K == 5 && S == 1) return launch_dw_reg_one<MODE, HB, 5, 1>(x, w, bias, y, rp, stream, d);
    return launch_dw_reg_one<MODE, HB, 5, 2>(x, w, bias, y, rp, stream, d);
}

// The register kernel serves square 3x3 / 5x5 filters, stride 1 or 2, "same" padding
// (K-1)/2, no dilation, and output rows of at most 128 columns (one warp per row).
bool dw_reg_eligible(int KH, int KW, int stride, int pad, int dil, long long Wo) {
    return KH == KW && (KH == 3 || KH == 5) && (stride == 1 || stride == 2) && pad == (KH - 1) / 2 && dil == 1 &&
           Wo <= 128;
}

DwRegParams dw_reg_plan(int N, int Cin, int mult, int H, int W, int Ho, int Wo, int num_sms, const float *x,
                        const float *y) {
    DwRegParams rp{};
    rp.Cin = Cin; rp.mult = mult; rp.Cout = Cin * mult; rp.H = H; rp.W = W; rp.Ho = Ho; rp.Wo = Wo;
    rp.lpp = (Wo + 3) / 4;
    rp.ppw = 32 / rp.lpp;
    rp.num_planes = N * rp.Cout;
    const long long groups = (rp.num_planes + rp.ppw - 1) / rp.ppw;
    // bands of output rows: enough warps to fill the machine about twice (64 resident warps
    // per SM), but no band shorter than 8 rows unless the plane is
    const long long want = 2LL * num_sms * 64;
    int nb = static_cast<int>((want + groups - 1) / groups);
    if (nb > (Ho + 7) / 8) nb = (Ho + 7) / 8;
    if (nb < 1) nb = 1;
    rp.band = (Ho + nb - 1) / nb;
    rp.nbands = (Ho + rp.band - 1) / rp.band;
    rp.num_jobs = static_cast<int>(groups * rp.nbands);
    rp.vec_in = (W % 4 == 0 && aligned(x, 16)) ? 1 : 0;
    rp.vec_out = (Wo % 4 == 0 && aligned(y, 16)) ? 1 : 0;
    rp.div_cout = make_fastdiv(static_cast<uint32_t>(rp.Cout));
    rp.div_mult = make_fastdiv(static_cast<uint32_t>(mult));
    rp.div_nbands = make_fastdiv(static_cast<uint32_t>(rp.nbands));
    rp.div_lpp = make_fastdiv(static_cast<uint32_t>(rp.lpp));
    return rp;
}

// ---- TMA-staged kernel ----------------------------------------------------------------------
constexpr int kDwTmaMaxSmem = 220 * 1024;   // per CTA: 4 warps x NB buffers (+ output staging)

struct DwTmaPlan {
    bool ok = false;
    DwTmaParams p{};
    int grid = 0;
    int smem = 0;
};

DwTmaPlan dw_tma_plan(int N, int Cin, int mult, int H, int W, int Ho, int Wo, int K, int S, int num_sms,
                      const float *x, const float *y) {
    DwTmaPlan pl;
    if (mult != 1) return pl;
    DwTmaParams &p = pl.p;
    p.H = H; p.W = W; p.Ho = Ho; p.Wo = Wo; p.C = Cin;
    p.lpp = (Wo + 3) / 4;
    p.ppw = 32 / p.lpp;
    if (p.ppw < 1) return pl;
    p.num_planes = N * Cin;
    p.Wp = p.lpp * 4 * S + 8;                       // 4 zeros, the lanes' columns, the right reach
    p.use_tma = (W % 4 == 0 && aligned(x, 16)) ? 1 : 0;
    // staged bytes per job buffer: whole planes when they fit, else bands of rows of even height;
    // NB buffers per warp (two measured fastest on the sweep layers). CONV_B200_DW_RING (buffers), CONV_B200_DW_BUFKB (KiB per buffer) and
    // CONV_B200_DW_CTAS (CTAs per SM) override the defaults (tuning and tests).
    p.nbuf = env_int("CONV_B200_DW_RING", 2, 2, kDwTmaMaxBuf);
    const long long row_bytes = 4LL * p.Wp * p.ppw;
    const long long kBufBytes = 1024LL * env_int("CONV_B200_DW_BUFKB", 9, 2, 48);
    const int whole_rows = (Ho - 1) * S + K;
    if (whole_rows * row_bytes <= kBufBytes || !p.use_tma) {
        p.Rw = Ho;
        if (!p.use_tma && whole_rows * row_bytes > 2 * kBufBytes) return pl;   // cp.async jobs are whole planes
    } else {
        int Rw = static_cast<int>((kBufBytes / row_bytes - K) / S + 1);
        if (Rw < 4) Rw = 4;
        const int nb = (Ho + Rw - 1) / Rw;   // bands of even height: no short last band
        p.Rw = (Ho + nb - 1) / nb;
    }
    p.rows_in = (p.Rw - 1) * S + K;
    // With several planes per warp, a plane stride rows_in * Wp = 4 * lpp * S (mod 32 floats)
    // makes the next plane's lanes continue this plane's shared-memory bank pattern, so the
    // 128-bit loads of a warp do not collide. Reach it with the cheapest of a slightly shorter
    // band, a wider pitch, or extra staged rows (zeros or input rows nobody reads); keep the
    // plain layout if nothing is within 25 % more staged bytes per output row or the larger
    // buffers would fit fewer CTAs per SM.
    if (p.ppw > 1) {
        const int target = (4 * p.lpp * S) % 32;
        const bool whole = p.Rw == Ho;
        double best = 1e30;
        int bRw = p.Rw, bRows = p.rows_in, bWp = p.Wp;
        for (int dr = 0; dr < 8; ++dr) {
            const int Rw = whole ? p.Rw : p.Rw - dr;
            if (Rw < 1) break;
            const int rows0 = (Rw - 1) * S + K;
            for (int extra = 0; extra < 8; ++extra) {
                if (!whole && extra > 0) break;
                for (int t = 0; t < 8; ++t) {
                    const int rows = rows0 + extra, wp = p.Wp + 4 * t;
                    if ((rows * wp) % 32 != target) continue;
                    const double cost = static_cast<double>(rows) * wp / Rw;
                    if (cost < best) { best = cost; bRw = Rw; bRows = rows; bWp = wp; }
                }
            }
        }
        const double plain = static_cast<double>(p.rows_in) * p.Wp / p.Rw;
        auto ctas = [&](int rows, int wp) {   // CTAs per SM the buffers allow
            const long long buf = ((1LL * p.ppw * rows * wp + 31) & ~31LL) * 4;
            return (227 * 1024) / (kDwWarpsPerCta * p.nbuf * buf + 128 + 1024);
        };
        if (best <= 1.25 * plain && ctas(bRows, bWp) >= ctas(p.rows_in, p.Wp)) {
            p.Rw = bRw; p.rows_in = bRows; p.Wp = bWp;
        }
    }
    if (p.use_tma && (p.Wp > 256 || p.rows_in > 256)) return pl;
    p.box_floats = p.ppw * p.rows_in * p.Wp;
    p.buf_floats = (p.box_floats + 31) & ~31;
    p.nbands = (Ho + p.Rw - 1) / p.Rw;
    const long long groups = (p.num_planes + p.ppw - 1) / p.ppw;
    if (groups * p.nbands > kInt32Max) return pl;
    p.num_jobs = static_cast<int>(groups * p.nbands);
    p.vec_out = (Wo % 4 == 0 && aligned(y, 16)) ? 1 : 0;
    p.div_nbands = make_fastdiv(static_cast<uint32_t>(p.nbands));
    p.div_lpp = make_fastdiv(static_cast<uint32_t>(p.lpp));
    p.div_c = make_fastdiv(static_cast<uint32_t>(p.C));
    p.div_w = make_fastdiv(static_cast<uint32_t>(W));
    // whole-plane jobs whose rows cannot be stored 16 bytes at a time collect the outputs in
    // shared memory and store the job's contiguous range coalesced, when that costs no CTA per SM
    p.stage_out = 0;
    p.out_floats = 0;
    p.vec_out_staged = aligned(y, 16) ? 1 : 0;
    p.warp_floats = p.nbuf * p.buf_floats;
    if (p.Rw == Ho && !p.vec_out) {
        const int out_floats = (p.ppw * Ho * Wo + 31) & ~31;
        const int smem_plain = kDwWarpsPerCta * 4 * p.warp_floats + 128;
        const int smem_staged = kDwWarpsPerCta * 4 * (p.warp_floats + out_floats) + 128;
        if (smem_staged <= kDwTmaMaxSmem &&
            (227 * 1024) / (smem_staged + 1024) >= (227 * 1024) / (smem_plain + 1024)) {
            p.stage_out = 1;
            p.out_floats = out_floats;
            p.warp_floats += out_floats;
        }
    }
    pl.smem = kDwWarpsPerCta * 4 * p.warp_floats + 128;   // + alignment slack
    if (pl.smem > kDwTmaMaxSmem) return pl;
    int per_sm = (227 * 1024) / (pl.smem + 1024);
    if (per_sm > 16) per_sm = 16;
    per_sm = env_int("CONV_B200_DW_CTAS", per_sm, 1, per_sm);
    if (per_sm < 1) return pl;
    const long long warps_needed = p.num_jobs;
    long long g = 1LL * num_sms * per_sm;
    const long long g_jobs = (warps_needed + kDwWarpsPerCta - 1) / kDwWarpsPerCta;
    if (g > g_jobs) g = g_jobs;
    pl.grid = static_cast<int>(g);
    // staggered first copies (same-box A/B, 200 launches each: C16 3x3 at 112x112 5 % faster,
    // C64 3x3 stride 2 2 % faster, the 5x5 layers unchanged); CONV_B200_DW_STAGGER=0 turns it
    // off (tests)
    p.stagger = env_int("CONV_B200_DW_STAGGER", 1, 0, 1);
    pl.ok = true;
    return pl;
}

template <int MODE, bool HB, int K, int S>
int launch_dw_tma_one(const float *x, const float *w, const float *bias, float *y, const DwTmaPlan &pl, int Cin, int N,
                      cudaStream_t stream, DeviceState *d, unsigned bit) {
    const DwTmaParams &p = pl.p;
    alignas(64) CUtensorMap tm;
    std::memset(&tm, 0, sizeof tm);
    if (p.use_tma) {
        const cuuint64_t dims[3] = {(cuuint64_t)p.W, (cuuint64_t)p.H, (cuuint64_t)N * Cin};
        const cuuint64_t strides[2] = {(cuuint64_t)p.W * 4, (cuuint64_t)p.H * p.W * 4};
        const cuuint32_t box[3] = {(cuuint32_t)p.Wp, (cuuint32_t)p.rows_in, (cuuint32_t)p.ppw};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode_tiled(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    auto kern = depthwise_tma_kernel<MODE, HB, K, S>;
    if (pl.smem > 48 * 1024)
        if (int rc = ensure_smem_attr(d, bit, kern, kDwTmaMaxSmem)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(32 * kDwWarpsPerCta);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    return launched(launch_k(cfg, kern, tm, x, w, bias, y, p, d->status), "depthwise_tma_kernel");
}

template <int MODE, bool HB>
int launch_dw_tma(const float *x, const float *w, const float *bias, float *y, const DwTmaPlan &pl, int K, int S,
                  int Cin, int N, cudaStream_t stream, DeviceState *d) {
    // shared-memory attribute bits 32..47
    const unsigned base = 32u + 4u * (2u * MODE + (HB ? 1u : 0u));
    if (K == 3 && S == 1) return launch_dw_tma_one<MODE, HB, 3, 1>(x, w, bias, y, pl, Cin, N, stream, d, base + 0);
    if (K == 3 && S == 2) return launch_dw_tma_one<MODE, HB, 3, 2>(x, w, bias, y, pl, Cin, N, stream, d, base + 1);
    if (K == 5 && S == 1) return launch_dw_tma_one<MODE, HB, 5, 1>(x, w, bias, y, pl, Cin, N, stream, d, base + 2);
    return launch_dw_tma_one<MODE, HB, 5, 2>(x, w, bias, y, pl, Cin, N, stream, d, base + 3);
}

// ---- lane-per-plane kernel (7x7 and 14x14 planes) --------------------------------------------
struct DwPlanePlan {
    bool ok = false;
    DwPlaneParams p{};
    int grid = 0;
    int smem = 0;
};

DwPlanePlan dw_plane_plan(int N, int Cin, int mult, int H, int W, int K, int S, int num_sms, const float *x,
                          const float *y) {
    DwPlanePlan pl;
    if (mult != 1 || H != W || (H != 7 && H != 14) || !aligned(x, 16)) return pl;
    const int HW = H, PAD = (K - 1) / 2;
    const int HO = (HW + 2 * PAD - K) / S + 1;
    const int LPP = HW <= 8 ? 1 : 2, PPJ = 32 / LPP;
    DwPlaneParams &p = pl.p;
    p.C = Cin;
    p.num_planes = N * Cin;
    p.num_jobs = (p.num_planes + PPJ - 1) / PPJ;
    p.in_floats = (PPJ * HW * HW + 31) & ~31;
    p.out_floats = (PPJ * HO * HO + 31) & ~31;
    p.vec_y = aligned(y, 16) ? 1 : 0;
    p.div_c = make_fastdiv(static_cast<uint32_t>(Cin));
    // a ring of input buffers per warp (jobs staged ahead; one buffer measured fastest on the
    // sweep layers, as it leaves the most CTAs per SM); CONV_B200_DW_RING and CONV_B200_DW_CTAS
    // (CTAs per SM) override the defaults (tuning and tests)
    p.nbuf = env_int("CONV_B200_DW_RING", 1, 1, kDwPlaneMaxBuf);
    pl.smem = kDwPlaneWarps * (p.nbuf * p.in_floats + p.out_floats) * 4;
    if (pl.smem > 200 * 1024) return pl;
    int per_sm = (227 * 1024) / (pl.smem + 1024);
    if (per_sm > 8) per_sm = 8;
    per_sm = env_int("CONV_B200_DW_CTAS", per_sm, 1, per_sm);
    if (per_sm < 1) return pl;
    const long long g_jobs = (p.num_jobs + kDwPlaneWarps - 1) / kDwPlaneWarps;
    const long long g = 1LL * num_sms * per_sm;
    pl.grid = static_cast<int>(g < g_jobs ? g : g_jobs);
    pl.ok = true;
    return pl;
}

template <int MODE, bool HB, int K, int S, int HW>
int launch_dw_plane_one(const float *x, const float *w, const float *bias, float *y, const DwPlanePlan &pl,
                        cudaStream_t stream, DeviceState *d, unsigned bit) {
    auto kern = depthwise_plane_kernel<MODE, HB, K, S, HW>;
    if (pl.smem > 48 * 1024)
        if (int rc = ensure_smem_attr(d, bit, kern, 200 * 1024)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(32 * kDwPlaneWarps);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    return launched(launch_k(cfg, kern, x, w, bias, y, pl.p, d->status), "depthwise_plane_kernel");
}

template <int MODE, bool HB>
int launch_dw_plane(const float *x, const float *w, const float *bias, float *y, const DwPlanePlan &pl, int K, int S,
                    int HW, cudaStream_t stream, DeviceState *d) {
    // shared-memory attribute bits 64..95: (MODE, HB) x (K, S, HW)
    const unsigned b = 64u + 8u * (2u * MODE + (HB ? 1u : 0u));
    if (K == 3 && S == 1 && HW == 7) return launch_dw_plane_one<MODE, HB, 3, 1, 7>(x, w, bias, y, pl, stream, d, b + 0);
    if (K == 3 && S == 2 && HW == 7) return launch_dw_plane_one<MODE, HB, 3, 2, 7>(x, w, bias, y, pl, stream, d, b + 1);
    if (K == 5 && S == 1 && HW == 7) return launch_dw_plane_one<MODE, HB, 5, 1, 7>(x, w, bias, y, pl, stream, d, b + 2);
    if (K == 5 && S == 2 && HW == 7) return launch_dw_plane_one<MODE, HB, 5, 2, 7>(x, w, bias, y, pl, stream, d, b + 3);
    if (K == 3 && S == 1) return launch_dw_plane_one<MODE, HB, 3, 1, 14>(x, w, bias, y, pl, stream, d, b + 4);
    if (K == 3 && S == 2) return launch_dw_plane_one<MODE, HB, 3, 2, 14>(x, w, bias, y, pl, stream, d, b + 5);
    if (K == 5 && S == 1) return launch_dw_plane_one<MODE, HB, 5, 1, 14>(x, w, bias, y, pl, stream, d, b + 6);
    return launch_dw_plane_one<MODE, HB, 5, 2, 14>(x, w, bias, y, pl, stream, d, b + 7);
}

template <int MODE, bool HB>
int launch_dw(const float *x, const float *w, const float *bias, float *y, const DwParams &p, DwSpec s,
              long long jobs, cudaStream_t stream, DeviceState *d) {
    // attribute bits 8..27: one per instantiation
    const unsigned base = 8u + 5u * (2u * MODE + (HB ? 1u : 0u));
    switch (s) {
        case kDwK3S1: return launch_dw_one<MODE, HB, 3, 1, 4>(x, w, bias, y, p, jobs, stream, d, base + 1);
        case kDwK3S2: return launch_dw_one<MODE, HB, 3, 2, 4>(x, w, bias, y, p, jobs, stream, d, base + 2);
        case kDwK5S1: return launch_dw_one<MODE, HB, 5, 1, 4>(x, w, bias, y, p, jobs, stream, d, base + 3);
        case kDwK5S2: return launch_dw_one<MODE, HB, 5, 2, 4>(x, w, bias, y, p, jobs, stream, d, base + 4);
        default: return launch_dw_one<MODE, HB, 0, 0, 1>(x, w, bias, y, p, jobs, stream, d, base);
    }
}

// ---- fused depthwise -> pointwise -------------------------------------------------------
// shared-memory attribute bits 51..56: MODE x (K 3, K 5, other K)
// Channel split S of the fused kernels: a cluster of S CTAs shares each tile (S = 1: one CTA per
// tile). S * owned 16-column chunks of 8 KB must fit the receive area (the stages they reuse),
// and every rank needs a channel block.
bool dwpw_split_ok(const DwPwParams &p, int S, int recv_bytes) {
    const int nch = p.n_mma / 16;
    return S >= 1 && S <= 4 && S <= p.num_kblk && S * ((nch + S - 1) / S) * kDwPwChunkBytes <= recv_bytes;
}

// Picks the split (or takes the forced one), sets p.S / p.owned and fills the launch geometry
// of `cfg` (whose cluster attribute lives in `attr`). The caller launches with the updated p.
template <typename Kern>
int dwpw_split_config(Kern kern, unsigned bit, int smem, int recv_bytes, DwPwParams &p, int force_split,
                      cudaStream_t stream, DeviceState *d, cudaLaunchConfig_t &cfg, cudaLaunchAttribute *attr) {
    if (int rc = ensure_smem_attr(d, bit, kern, kDwPwMaxSmem)) return rc;
    cfg = cudaLaunchConfig_t{};
    cfg.blockDim = dim3(kDwPwThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // clusters of S CTAs that can run at once (one CTA per SM)
    auto active_clusters = [&](int S) {
        if (S == 1) return d->num_sms;
        {
            std::lock_guard<std::mutex> lock(g_mu);
            for (int i = 0; i < d->n_cluster_fit; ++i) {
                const DeviceState::ClusterFit &f = d->cluster_fit[i];
                if (f.bit == bit && f.S == S && f.smem == smem) return f.active;
            }
        }
        attr[0].val.clusterDim.x = static_cast<unsigned>(S);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(static_cast<unsigned>(S));
        int active = 0;
        if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess) active = 0;
        std::lock_guard<std::mutex> lock(g_mu);
        if (d->n_cluster_fit < 64) d->cluster_fit[d->n_cluster_fit++] = DeviceState::ClusterFit{bit, S, smem, active};
        return active;
    };
    // The split that finishes first: rounds of tiles (ceil(tiles / clusters at once)) times the
    // 1/S share of a tile each CTA computes; a split pays a small reduction cost.
    int S = 1, clusters = d->num_sms;
    if (force_split) {
        if (!dwpw_split_ok(p, force_split, recv_bytes)) return CONV_ERR_UNSUPPORTED;
        S = force_split;
        clusters = active_clusters(S);
        if (clusters < 1) return CONV_ERR_CUDA;
    } else {
        double best = 1e30;
        for (int cand = 1; cand <= 4; ++cand) {
            if (!dwpw_split_ok(p, cand, recv_bytes)) continue;
            const int act = active_clusters(cand);
            if (act < 1) continue;
            const double cost = static_cast<double>((p.num_tiles + act - 1) / act) / cand + (cand > 1 ? 0.05 : 0.0);
            if (cost < best) { best = cost; S = cand; clusters = act; }
        }
    }
    p.S = S;
    p.owned = (p.n_mma / 16 + S - 1) / S;
    if (clusters > p.num_tiles) clusters = p.num_tiles;
    if (S > 1) {
        attr[0].val.clusterDim.x = static_cast<unsigned>(S);
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    } else {
        cfg.attrs = nullptr;
        cfg.numAttrs = 0;
    }
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * S));
    return CONV_OK;
}

template <int MODE, int KC>
int launch_dwpw(const float *x, const float *w, const CUtensorMap &tmF, float *y, DwPwParams p, int force_split,
                cudaStream_t stream, DeviceState *d, unsigned bit) {
    auto kern = dwpw_kernel<MODE, KC>;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    if (int rc = dwpw_split_config(kern, bit, kDwPwFixed + 4 * p.w_floats, kDwPwStages, p, force_split, stream, d,
                                   cfg, attr))
        return rc;
    return launched(launch_k(cfg, kern, x, w, tmF, y, p, d->status), "dwpw_kernel");
}

// The staged kernel's tiles for this shape (ok = false: it does not apply).
struct DwPwStagePlan {
    bool ok = false;
    DwPwStage st{};
    int num_tiles = 0;
};

DwPwStagePlan plan_dwpw_staged(const DwPwParams &p, int N) {
    DwPwStagePlan pl;
    if (p.K != 3 && p.K != 5) return pl;
    DwPwStage &st = pl.st;
    st.N = N;
    if (p.HoWo <= 128) {   // whole images per tile
        st.G = 128 / p.HoWo;
        if (st.G > N) st.G = N;
        st.RB = p.Ho;
        st.nbands = 1;
        pl.num_tiles = (N + st.G - 1) / st.G;
    } else if (p.Wo <= 128) {   // bands of output rows, as even as possible
        const int max_rows = 128 / p.Wo;
        st.nbands = (p.Ho + max_rows - 1) / max_rows;
        st.RB = (p.Ho + st.nbands - 1) / st.nbands;
        st.G = 1;
        pl.num_tiles = N * st.nbands;
    } else {
        return pl;
    }
    st.R_in = (st.RB - 1) * p.stride + (p.K - 1) * p.dil + 1;
    st.Wp = (p.Wo - 1) * p.stride + (p.K - 1) * p.dil + 1;
    st.wcols = p.W < st.Wp - p.pad ? p.W : st.Wp - p.pad;
    if (st.wcols < 1) return pl;
    st.div_wcols = make_fastdiv(static_cast<uint32_t>(st.wcols));
    const long long xf = 64LL * st.G * st.R_in * st.Wp;
    if (xf > (1 << 20)) return pl;
    st.x_floats = static_cast<int>((xf + 3) & ~3LL);
    st.w_floats = 64 * dwpw_kkp(p.K);
    st.b_bytes = p.n_boxes * kDwPwBox;
    pl.ok = dwpw_staged_smem(st) <= kDwPwMaxSmem;
    return pl;
}

template <int MODE, int KC>
int launch_dwpw_staged(const float *x, const float *w, const CUtensorMap &tmF, float *y, DwPwParams p,
                       const DwPwStagePlan &pl, int force_split, cudaStream_t stream, DeviceState *d, unsigned bit) {
    p.num_tiles = pl.num_tiles;
    p.w_floats = 0;
    auto kern = dwpw_staged_kernel<MODE, KC>;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    if (int rc = dwpw_split_config(kern, bit, dwpw_staged_smem(pl.st), dwpw_staged_body(pl.st), p, force_split,
                                   stream, d, cfg, attr))
        return rc;
    return launched(launch_k(cfg, kern, x, w, tmF, y, p, pl.st, d->status), "dwpw_staged_kernel");
}

// Whether the im2col kernel runs as CTA pairs: by default for 256-column tiles whose reduction
// is at least 16 blocks of 64 channels; CONV_B200_TC_PAIR=1 / 0 forces it on / off (tile
// widths of 128 and 256).
bool tc_pair_choice(int bn, int num_kblk, int num_sms) {
    if (bn < 128 || num_sms < 2) return false;
    const int forced = env_int("CONV_B200_TC_PAIR", -1, -1, 1);
    if (forced >= 0) return forced == 1;
    return bn == 256 && num_kblk >= 16;
}

// Output-channel tile width of the im2col kernel: 64 for narrow groups; 256 for groups of at
// least 256 output channels while the tiles still cover every SM (measured on B200: the wider
// tile halves the A-operand traffic per MMA, e.g. a 3-tap 512 -> 512 Conv1D over 48000
// positions, 94 -> 74 us); else 128.
int im2col_bn(long long M, int cout_g, int groups, int num_sms) {
    if (cout_g <= 64) return 64;
    if (cout_g >= 256 && ((M + 127) / 128) * ((cout_g + 255) / 256) * groups >= num_sms) return 256;
    return 128;
}

// Kernel choice and launch of the plain dense convolution (arguments already validated, the
// device state taken).
int dense_plain(const void *X, const void *F, void *Y, int N, int H, int W, int Cin, int Cout, int K,
                cudaStream_t stream, DeviceState *d) {
    const char *force = env("CONV_B200_DENSE");
    // Tensor-core paths need 16-byte rows (Cin, Cout multiples of 8) and 16-byte aligned
    // tensors. The im2col tensor map is used only for inputs of at least 128 KiB.
    const bool tc_shape = (Cin % 8 == 0) && (Cout % 8 == 0) && aligned(X, 16) && aligned(F, 16) && aligned(Y, 16);
    const bool im2col_ok = tc_shape && K <= 128 && 2LL * N * H * W * Cin >= 128 * 1024;
    const DenseGeom sq = DenseGeom::square(K);
    if ((force && std::strcmp(force, "direct") == 0) || !tc_shape)
        return launch_dense_direct(static_cast<const __nv_bfloat16 *>(X), static_cast<const __nv_bfloat16 *>(F),
                                   static_cast<__nv_bfloat16 *>(Y), N, H, W, Cin, Cout, sq, stream, d);
    // Default: the halo kernel; the im2col kernel when a halo does not fit in shared memory
    // (very wide images) or when forced. CONV_B200_DENSE (tests): "direct", "halo",
    // "halo64/128/256" (halo kernel with that tile width), "bn64/128/256" (im2col kernel).
    int force_bn = 0;
    bool force_im2col = false, force_halo = false;
    const bool force_fold = force && std::strcmp(force, "fold") == 0;
    const bool force_stream = force && std::strcmp(force, "stream") == 0;
    if (force) {
        if (std::strncmp(force, "halo", 4) == 0) { force_halo = true; force_bn = std::atoi(force + 4); }
        if (std::strncmp(force, "bn", 2) == 0) { force_im2col = true; force_bn = std::atoi(force + 2); }
    }
    if (force_bn != 0 && force_bn != 64 && force_bn != 128 && force_bn != 256) return CONV_ERR_INVALID_ARG;
    // Narrow layers (Cout <= 64, K = 2..4) with a resident filter: the folded-tap kernel
    // ("fold" forces it).
    if (force_fold || (!force_im2col && !force_halo && !force_stream)) {
        const FoldPlan fp = plan_fold(N, H, W, Cin, Cout, K, d->num_sms);
        if (fp.ok) return dispatch_fold(X, F, Y, Cin, Cout, K, fp, stream, d);
        if (force_fold) return CONV_ERR_UNSUPPORTED;
    }
    if (!force_im2col) {
        // By default the halo kernel runs when the filter stays resident in shared memory; with
        // a streamed filter the 256-row streamed-filter kernel ("stream" forces it).
        const HaloPlan pl = plan_halo(N, H, W, Cin, Cout, K, d->num_sms, force_bn);
        if (pl.ok && (pl.bres || force_halo) && !force_stream) return dispatch_halo(X, F, Y, Cin, Cout, K, pl, stream, d);
        if (force_halo) return CONV_ERR_UNSUPPORTED;
        if (!force_bn) {
            // shared-memory attribute bits 61..62, and 104 for the pair form
            const StreamPlan sp = plan_stream(N, H, W, Cin, Cout, K, d->num_sms);
            if (sp.ok) {
                if (sp.pair) return launch_dense_stream<128, true>(X, F, Y, Cin, Cout, K, sp, stream, d, 104);
                return sp.bn == 64 ? launch_dense_stream<64, false>(X, F, Y, Cin, Cout, K, sp, stream, d, 61)
                                   : launch_dense_stream<128, false>(X, F, Y, Cin, Cout, K, sp, stream, d, 62);
            }
            if (force_stream) return CONV_ERR_UNSUPPORTED;
        }
        if (pl.ok && !im2col_ok) return dispatch_halo(X, F, Y, Cin, Cout, K, pl, stream, d);
    }
    if (!im2col_ok) {
        if (force_im2col) return CONV_ERR_UNSUPPORTED;
        return launch_dense_direct(static_cast<const __nv_bfloat16 *>(X), static_cast<const __nv_bfloat16 *>(F),
                                   static_cast<__nv_bfloat16 *>(Y), N, H, W, Cin, Cout, sq, stream, d);
    }
    int bn = force_bn ? force_bn : im2col_bn(1LL * N * sq.ho(H) * sq.wo(W), Cout, 1, d->num_sms);
    if (bn == 64) return launch_dense_tc<CfgBN64, 1>(X, F, Y, N, H, W, Cin, Cout, sq, stream, d, 0);
    // 256-wide tiles with long reductions run as CTA pairs (each CTA stages half of every B slot:
    // measured on B200, a 3-tap 512-channel causal Conv1D 76 -> 70 us; with a 6-block reduction
    // the pair's hand-offs cost more than they save). CONV_B200_TC_PAIR=1 / 0 forces pairs on /
    // off for tiles of at least 128 columns. Shared-memory attribute bits 107..108.
    const bool tc_pair = tc_pair_choice(bn, K * K * ((Cin + 63) / 64), d->num_sms);
    if (bn == 128)
        return tc_pair ? launch_dense_tc<CfgBN128, 1, true>(X, F, Y, N, H, W, Cin, Cout, sq, stream, d, 107)
                       : launch_dense_tc<CfgBN128, 1>(X, F, Y, N, H, W, Cin, Cout, sq, stream, d, 1);
    return tc_pair ? launch_dense_tc<CfgBN256, 1, true>(X, F, Y, N, H, W, Cin, Cout, sq, stream, d, 108)
                   : launch_dense_tc<CfgBN256, 1>(X, F, Y, N, H, W, Cin, Cout, sq, stream, d, 2);
}

// ---- fused depthwise -> pointwise, transposed GEMM (7x7 and 14x14 images) --------------------
// shared-memory attribute bits 96..103: MODE x K (3, 5) x image (7, 14)
bool dwpw_gemm_eligible(int C, int H, int W, int K, int stride, int pad, int dil, int Cout, const float *x,
                        const float *w, const float *y) {
    return H == W && (H == 7 || H == 14) && (K == 3 || K == 5) && stride == 1 && dil == 1 && pad == (K - 1) / 2 &&
           C % 4 == 0 && Cout <= 256 && aligned(x, 16) && aligned(w, 16) && aligned(y, 16);
}

template <int MODE, int KC, class G>
int launch_dwpw_gemm_one(const float *x, const float *w, const float *b_dw, const void *F, const float *b_pw, float *y,
                         int N, int C, int Cout, cudaStream_t stream, DeviceState *d, unsigned bit) {
    DwPwGemmParams p;
    p.C = C;
    p.Cout = Cout;
    p.num_tiles = N;
    p.nblk = (C + G::CB - 1) / G::CB;
    p.MT = (Cout + 127) / 128;
    p.fslot = p.MT * 2 * G::BOX;
    p.idesc = idesc_bf16_f32_amn(128, G::NPAD, /*B MN-major*/ true);
    p.tmem_cols = 32;
    while (p.tmem_cols < static_cast<uint32_t>(p.MT * G::NPAD)) p.tmem_cols <<= 1;
    p.b_dw = b_dw;
    p.b_pw = b_pw;
    // a 2-CTA cluster per image (every other channel block each) when there are two blocks and
    // its receive area fits; CONV_B200_DWPW_SPLIT=1 keeps one CTA per image (tests)
    // (the pixel-split form: two CTAs per image without a cluster, S = 1)
    const int want = G::HALF ? 1 : env_int("CONV_B200_DWPW_SPLIT", 2, 1, 2);
    p.S = (want == 2 && p.nblk >= 2 && dwpw_gemm_smem<G>(p.fslot, p.MT, 2, KC * KC) <= kSmemLimit) ? 2 : 1;
    const int smem = dwpw_gemm_smem<G>(p.fslot, p.MT, p.S, KC * KC);
    if (smem > kSmemLimit || p.tmem_cols > 512) return CONV_ERR_UNSUPPORTED;
    alignas(64) CUtensorMap tmF;
    {   // F: 2-D {Cout, C}; a box is 64 output columns x CB channel rows (columns past Cout and
        // rows past C read zeros)
        const cuuint64_t dims[2] = {(cuuint64_t)Cout, (cuuint64_t)C};
        const cuuint64_t strides[1] = {(cuuint64_t)Cout * 2};
        const cuuint32_t box[2] = {64, (cuuint32_t)G::CB};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode_tiled(&tmF, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(F), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    alignas(64) CUtensorMap tmX = tmF;   // unused by the 7x7 form (contiguous bulk copies)
    if (G::PADX) {   // x as [N*C][P] fp32; a box of XP columns (past P it reads zeros) x CB planes
        const cuuint64_t dims[2] = {(cuuint64_t)G::P, (cuuint64_t)N * C};
        const cuuint64_t strides[1] = {(cuuint64_t)G::P * 4};
        const cuuint32_t box[2] = {(cuuint32_t)G::XP, (cuuint32_t)G::CB};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode_tiled(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    auto kern = dwpw_gemm_kernel<MODE, KC, G>;
    if (int rc = ensure_smem_attr(d, bit, kern, kSmemLimit)) return rc;
    const int per = G::HALF ? 2 : p.S;   // CTAs per image
    int clusters_max = d->num_sms / per;
    if (p.S > 1) clusters_max = cluster_fit(d, bit, kern, p.S, smem, G::THREADS);
    if (clusters_max < 1) return CONV_ERR_CUDA;
    const int clusters = N < clusters_max ? N : clusters_max;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * per));
    cfg.blockDim = dim3(G::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    if (p.S > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(p.S);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return launched(launch_k(cfg, kern, x, w, tmF, tmX, y, p, d->status), "dwpw_gemm_kernel");
}

template <int MODE>
int launch_dwpw_gemm(const float *x, const float *w, const float *b_dw, const void *F, const float *b_pw, float *y,
                     int N, int C, int H, int K, int Cout, cudaStream_t stream, DeviceState *d) {
    const unsigned b = 96u + 4u * MODE;
    using G7 = DwPwGemmGeom<7>;
    using G14 = DwPwGemmGeom<14>;
    using G14H3 = DwPwGemmGeom<14, true, 3>;
    using G14H5 = DwPwGemmGeom<14, true, 5>;
    if (H == 7)
        return K == 3 ? launch_dwpw_gemm_one<MODE, 3, G7>(x, w, b_dw, F, b_pw, y, N, C, Cout, stream, d, b + 0)
                      : launch_dwpw_gemm_one<MODE, 5, G7>(x, w, b_dw, F, b_pw, y, N, C, Cout, stream, d, b + 1);
    // 14x14: the row split (each CTA half of the rows, all channels; shared-memory attribute
    // bits 109..112) unless CONV_B200_DWPW_HALF=0 asks for the channel-split cluster, or its
    // rings do not fit (5x5 taps with more than 128 outputs)
    if (env_int("CONV_B200_DWPW_HALF", 1, 0, 1) == 1) {
        const unsigned bh = 109u + 2u * MODE;
        const int rc = K == 3 ? launch_dwpw_gemm_one<MODE, 3, G14H3>(x, w, b_dw, F, b_pw, y, N, C, Cout, stream, d, bh + 0)
                              : launch_dwpw_gemm_one<MODE, 5, G14H5>(x, w, b_dw, F, b_pw, y, N, C, Cout, stream, d, bh + 1);
        if (rc != CONV_ERR_UNSUPPORTED) return rc;
    }
    return K == 3 ? launch_dwpw_gemm_one<MODE, 3, G14>(x, w, b_dw, F, b_pw, y, N, C, Cout, stream, d, b + 2)
                  : launch_dwpw_gemm_one<MODE, 5, G14>(x, w, b_dw, F, b_pw, y, N, C, Cout, stream, d, b + 3);
}

}  // namespace
}  // namespace convb200

using namespace convb200;

extern "C" {

int conv2d_nhwc_fwd(const void *X, const void *F, void *Y, int N, int H, int W, int Cin, int Cout, int K,
                    cudaStream_t stream) {
    if (int rc = check_dense(X, F, Y, N, H, W, Cin, Cout, K, 2)) return rc;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {X, F, Y})) return rc;
    return dense_plain(X, F, Y, N, H, W, Cin, Cout, K, stream, d);
}

int conv2d_nhwc_fwd_f32(const float *X, const float *F, float *Y, int N, int H, int W, int Cin, int Cout,
                        int K, cudaStream_t stream) {
    if (int rc = check_dense(X, F, Y, N, H, W, Cin, Cout, K, 4)) return rc;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {X, F, Y})) return rc;
    return launch_dense_direct(X, F, Y, N, H, W, Cin, Cout, DenseGeom::square(K), stream, d);
}

}  // extern "C"

namespace convb200 {
namespace {

// Validation, dispatch and launch of the general dense convolution (every geometry field of g
// set; g.plain() operations already routed to the plain entry by the callers).
// ---- padded halo kernel (stride 1, zero padding, dilation, groups; resident filter) ---------
struct HaloPadPlan {
    bool ok = false;
    int bn = 0;
    DenseHaloPadParams p{};
    int smem = 0;
    int grid = 0;
};

// Tiles of Rout output rows x Wt columns whose padded input window (Rin x Wbox pixels) is one
// tensor copy; the window's flattened rows hold the tile's GEMM rows (at most 128 of them) and
// every tap's reach. Eligible: stride 1, whole 64-channel blocks per group (Cin_g % 64 == 0),
// Cout_g % 8 == 0, the group's filter slice and two window slots fit in shared memory.
HaloPadPlan plan_halo_pad(int N, int H, int W, int Cin, int Cout, const DenseGeom &g, int num_sms) {
    HaloPadPlan pl;
    const int Cin_g = Cin / g.groups, Cout_g = Cout / g.groups;
    if (g.sh != 1 || g.sw != 1 || Cin_g % 64 != 0 || Cout_g % 8 != 0) return pl;
    const long long Ho = g.ho(H), Wo = g.wo(W);
    if (Ho < 1 || Wo < 1) return pl;
    const int reach_w = g.dw * (g.KW - 1), reach_h = g.dh * (g.KH - 1);
    if (reach_w > 96 || reach_h > 127) return pl;
    const int Wt = static_cast<int>(Wo < 128 - reach_w ? Wo : 128 - reach_w);
    const int Wbox = Wt + reach_w;
    int Rout = 128 / Wbox;
    if (Rout > Ho) Rout = static_cast<int>(Ho);
    if (Rout < 1) Rout = 1;
    const int Rin = Rout + reach_h;
    if (Wbox > 256 || Rin > 256) return pl;
    const int bn = Cout_g <= 64 ? 64 : 128;
    const long long reach_rows = 1LL * reach_h * Wbox + reach_w + 128;
    long long slot_rows = 1LL * Rin * Wbox > reach_rows ? 1LL * Rin * Wbox : reach_rows;
    slot_rows = (slot_rows + 7) & ~7LL;
    const long long halo_bytes = slot_rows * 128;
    const int num_cblk = Cin_g / 64;
    const int KK = g.KH * g.KW;
    const long long b_res = 1LL * KK * num_cblk * 64 * bn * 2;
    const int fixed = bn == 64 ? DenseHaloPadCfg<64>::FIXED_BYTES : DenseHaloPadCfg<128>::FIXED_BYTES;
    const long long avail = kSmemLimit - fixed - b_res;
    if (avail < 2 * halo_bytes) return pl;
    int HS = static_cast<int>(avail / halo_bytes);
    if (HS > DenseHaloPadCfg<64>::MAX_RING) HS = DenseHaloPadCfg<64>::MAX_RING;
    const long long n_rb = (Ho + Rout - 1) / Rout, n_cb = (Wo + Wt - 1) / Wt;
    const long long num_spatial = 1LL * N * n_rb * n_cb;
    if (num_spatial > kInt32Max) return pl;
    DenseHaloPadParams &p = pl.p;
    p.H = H; p.W = W; p.Ho = static_cast<int>(Ho); p.Wo = static_cast<int>(Wo);
    p.Cout = Cout; p.Cin_g = Cin_g; p.Cout_g = Cout_g;
    p.KH = g.KH; p.KW = g.KW; p.dh = g.dh; p.dw = g.dw; p.ph = g.ph; p.pw = g.pw;
    p.Rout = Rout; p.Wt = Wt; p.Wbox = Wbox; p.Rin = Rin;
    p.n_rb = static_cast<int>(n_rb); p.n_cb = static_cast<int>(n_cb);
    p.num_spatial = static_cast<int>(num_spatial);
    p.num_cblk = num_cblk; p.KK = KK; p.num_kblk = KK * num_cblk;
    p.num_nt = (Cout_g + bn - 1) / bn;
    p.num_gn = g.groups * p.num_nt;
    p.box_bytes = Rin * Wbox * 128;
    p.halo_bytes = static_cast<int>(halo_bytes);
    p.HS = HS;
    p.b_region = static_cast<int>(b_res);
    p.bias = g.bias;
    p.y_elems = 1LL * N * Ho * Wo * Cout;
    int per = num_sms / p.num_gn;
    if (per < 1) per = 1;
    if (per > p.num_spatial) per = p.num_spatial;
    pl.grid = per * p.num_gn;
    pl.smem = fixed + static_cast<int>(b_res) + HS * p.halo_bytes;
    // more than half of the shared memory keeps a second CTA (and its TMEM allocation) off the SM
    if (pl.smem < 116 * 1024) pl.smem = 116 * 1024;
    pl.bn = bn;
    pl.ok = pl.smem <= kSmemLimit;
    return pl;
}

template <class Cfg>
int launch_dense_halo_pad(const void *X, const void *F, void *Y, int N, int Cin, const HaloPadPlan &pl,
                          cudaStream_t stream, DeviceState *d, unsigned attr_bit) {
    const DenseHaloPadParams &p = pl.p;
    alignas(64) CUtensorMap tmX, tmF;
    {   // X 4-D {Cin, W, H, N}; a box is 64 channels (128 bytes, 128-byte swizzle) x Wbox columns
        // x Rin rows of one image; parts outside the image read zeros (the padding)
        const cuuint64_t dims[4] = {(cuuint64_t)Cin, (cuuint64_t)p.W, (cuuint64_t)p.H, (cuuint64_t)N};
        const cuuint64_t strides[3] = {(cuuint64_t)Cin * 2, (cuuint64_t)p.W * Cin * 2, (cuuint64_t)p.H * p.W * Cin * 2};
        const cuuint32_t box[4] = {64, (cuuint32_t)p.Wbox, (cuuint32_t)p.Rin, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        if (g_encode_tiled(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(X), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    {   // F 3-D {Cout, Cin_g, KH*KW}; a box is 64 reduction rows x 64 output channels
        const cuuint64_t dims[3] = {(cuuint64_t)p.Cout, (cuuint64_t)p.Cin_g, (cuuint64_t)p.KK};
        const cuuint64_t strides[2] = {(cuuint64_t)p.Cout * 2, (cuuint64_t)p.Cin_g * p.Cout * 2};
        const cuuint32_t box[3] = {64, 64, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode_tiled(&tmF, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(F), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    auto kern = dense_halo_pad_kernel<Cfg>;
    if (int rc = ensure_smem_attr(d, attr_bit, kern, kSmemLimit)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    return launched(launch_k(cfg, kern, tmX, tmF, static_cast<__nv_bfloat16 *>(Y), p, d->status),
                    "dense_halo_pad_kernel");
}

int dense_general(const void *X, const void *F, void *Y, int N, int H, int W, int Cin, int Cout,
                  const DenseGeom &g, cudaStream_t stream) {
    const long long Ho = g.ho(H), Wo = g.wo(W);
    const long long nx = 1LL * N * H * W * Cin, nf = 1LL * g.KH * g.KW * (Cin / g.groups) * Cout,
                    ny = 1LL * N * Ho * Wo * Cout;
    if (nx > kInt32Max || nf > kInt32Max || ny > kInt32Max || 1LL * N * Ho * Wo > kInt32Max)
        return CONV_ERR_UNSUPPORTED;
    if (!aligned(X, 2) || !aligned(F, 2) || !aligned(Y, 2) || (g.bias && !aligned(g.bias, 4)))
        return CONV_ERR_MISALIGNED;
    if (overlaps(Y, ny * 2, X, nx * 2) || overlaps(Y, ny * 2, F, nf * 2) ||
        (g.bias && overlaps(Y, ny * 2, g.bias, 4LL * Cout)))
        return CONV_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {X, F, Y, g.bias})) return rc;
    const char *force = env("CONV_B200_DENSE");
    // Tensor cores through the TMA im2col unit: 16-byte channel rows per group (group bases
    // 16-byte aligned), 16-byte aligned tensors, and window corners and tap offsets inside the
    // 4-D im2col ranges (|corner| <= 127, offset <= 127).
    const int Cin_g = Cin / g.groups, Cout_g = Cout / g.groups;
    const bool tc_shape = (Cin_g % 8 == 0) && (Cout_g % 8 == 0) && aligned(X, 16) && aligned(F, 16) && aligned(Y, 16);
    auto axis_ok = [](int pad, int pad_end, int dil, int taps) {
        const long long reach = 1LL * dil * (taps - 1);
        return pad <= 127 && reach <= 127 && pad_end - reach >= -127 && pad_end - reach <= 127;
    };
    const bool im2col_ok = tc_shape && axis_ok(g.ph, g.ph_end, g.dh, g.KH) && axis_ok(g.pw, g.pw_end, g.dw, g.KW) &&
                           2LL * N * H * W * Cin >= 128 * 1024;
    const bool force_bn = force && std::strncmp(force, "bn", 2) == 0;
    // Stride 1 with whole 64-channel blocks per group: the padded halo kernel (each input pixel
    // of a tile staged once; shared-memory attribute bits 105..106). CONV_B200_DENSE=halo
    // requires it, bnXX or direct skip it.
    const bool force_halo = force && std::strcmp(force, "halo") == 0;
    if (tc_shape && (!g.bias || aligned(g.bias, 16)) && (!force || force_halo)) {
        const HaloPadPlan hp = plan_halo_pad(N, H, W, Cin, Cout, g, d->num_sms);
        if (hp.ok)
            return hp.bn == 64 ? launch_dense_halo_pad<DenseHaloPadCfg<64>>(X, F, Y, N, Cin, hp, stream, d, 105)
                               : launch_dense_halo_pad<DenseHaloPadCfg<128>>(X, F, Y, N, Cin, hp, stream, d, 106);
    }
    if (force_halo) return CONV_ERR_UNSUPPORTED;
    if ((force && std::strcmp(force, "direct") == 0) || !im2col_ok) {
        if (force_bn) return CONV_ERR_UNSUPPORTED;
        return launch_dense_direct(static_cast<const __nv_bfloat16 *>(X), static_cast<const __nv_bfloat16 *>(F),
                                   static_cast<__nv_bfloat16 *>(Y), N, H, W, Cin, Cout, g, stream, d);
    }
    int bn = im2col_bn(1LL * N * g.ho(H) * g.wo(W), Cout_g, g.groups, d->num_sms);
    if (force_bn) bn = std::atoi(force + 2);
    if (g.groups == 1) {
        if (bn == 64) return launch_dense_tc<CfgBN64, 1>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 0);
        const bool tc_pair = tc_pair_choice(bn, g.KH * g.KW * ((Cin_g + 63) / 64), d->num_sms);
        if (bn == 128)
            return tc_pair ? launch_dense_tc<CfgBN128, 1, true>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 107)
                           : launch_dense_tc<CfgBN128, 1>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 1);
        if (bn == 256)
            return tc_pair ? launch_dense_tc<CfgBN256, 1, true>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 108)
                           : launch_dense_tc<CfgBN256, 1>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 2);
        return CONV_ERR_INVALID_ARG;
    }
    // several groups: up to kTcGroups per launch (shared-memory attribute bits 48..50)
    if (bn == 64) return launch_dense_tc<CfgBN64, kTcGroups>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 48);
    if (bn == 128) return launch_dense_tc<CfgBN128, kTcGroups>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 49);
    if (bn == 256) return launch_dense_tc<CfgBN256, kTcGroups>(X, F, Y, N, H, W, Cin, Cout, g, stream, d, 50);
    return CONV_ERR_INVALID_ARG;
}

}  // namespace
}  // namespace convb200

extern "C" {

int conv2d_nhwc_fwd_ex(const void *X, const void *F, const float *bias, void *Y, int N, int H, int W, int Cin,
                       int Cout, int K, int stride, int pad, int dil, cudaStream_t stream) {
    if (!X || !F || !Y) return CONV_ERR_INVALID_ARG;
    if (N < 1 || H < 1 || W < 1 || Cin < 1 || Cout < 1 || K < 1 || stride < 1 || dil < 1 || pad < 0)
        return CONV_ERR_INVALID_ARG;
    const DenseGeom g = DenseGeom::square(K, stride, pad, dil, bias);
    if (1LL * H + 2LL * pad > kInt32Max / 2 || 1LL * W + 2LL * pad > kInt32Max / 2 ||
        1LL * dil * (K - 1) > kInt32Max / 2)
        return CONV_ERR_UNSUPPORTED;
    if (1LL * H + 2LL * pad < 1LL * dil * (K - 1) + 1 || 1LL * W + 2LL * pad < 1LL * dil * (K - 1) + 1)
        return CONV_ERR_INVALID_ARG;
    if (g.plain()) return conv2d_nhwc_fwd(X, F, Y, N, H, W, Cin, Cout, K, stream);
    return dense_general(X, F, Y, N, H, W, Cin, Cout, g, stream);
}

int conv2d_nhwc_fwd_grouped(const void *X, const void *F, const float *bias, void *Y, int N, int H, int W, int Cin,
                            int Cout, int KH, int KW, int stride_h, int stride_w, int pad_h, int pad_w, int dil_h,
                            int dil_w, int groups, cudaStream_t stream) {
    if (!X || !F || !Y) return CONV_ERR_INVALID_ARG;
    if (N < 1 || H < 1 || W < 1 || Cin < 1 || Cout < 1 || KH < 1 || KW < 1 || stride_h < 1 || stride_w < 1 ||
        dil_h < 1 || dil_w < 1 || pad_h < 0 || pad_w < 0 || groups < 1 || Cin % groups != 0 || Cout % groups != 0)
        return CONV_ERR_INVALID_ARG;
    if (1LL * H + 2LL * pad_h > kInt32Max / 2 || 1LL * W + 2LL * pad_w > kInt32Max / 2 ||
        1LL * dil_h * (KH - 1) > kInt32Max / 2 || 1LL * dil_w * (KW - 1) > kInt32Max / 2)
        return CONV_ERR_UNSUPPORTED;
    if (1LL * H + 2LL * pad_h < 1LL * dil_h * (KH - 1) + 1 || 1LL * W + 2LL * pad_w < 1LL * dil_w * (KW - 1) + 1)
        return CONV_ERR_INVALID_ARG;
    DenseGeom g;
    g.KH = KH; g.KW = KW;
    g.sh = stride_h; g.sw = stride_w; g.ph = pad_h; g.pw = pad_w; g.dh = dil_h; g.dw = dil_w;
    g.ph_end = pad_h; g.pw_end = pad_w;
    g.groups = groups;
    g.bias = bias;
    if (KH == KW && stride_h == stride_w && pad_h == pad_w && dil_h == dil_w && groups == 1)
        return conv2d_nhwc_fwd_ex(X, F, bias, Y, N, H, W, Cin, Cout, KH, stride_h, pad_h, dil_h, stream);
    return dense_general(X, F, Y, N, H, W, Cin, Cout, g, stream);
}

int conv2d_nhwc_fwd_grouped_pads(const void *X, const void *F, const float *bias, void *Y, int N, int H, int W,
                                 int Cin, int Cout, int KH, int KW, int stride_h, int stride_w, int pad_top,
                                 int pad_bottom, int pad_left, int pad_right, int dil_h, int dil_w, int groups,
                                 cudaStream_t stream) {
    if (pad_top == pad_bottom && pad_left == pad_right)
        return conv2d_nhwc_fwd_grouped(X, F, bias, Y, N, H, W, Cin, Cout, KH, KW, stride_h, stride_w, pad_top, pad_left,
                                       dil_h, dil_w, groups, stream);
    if (!X || !F || !Y) return CONV_ERR_INVALID_ARG;
    if (N < 1 || H < 1 || W < 1 || Cin < 1 || Cout < 1 || KH < 1 || KW < 1 || stride_h < 1 || stride_w < 1 ||
        dil_h < 1 || dil_w < 1 || pad_top < 0 || pad_bottom < 0 || pad_left < 0 || pad_right < 0 || groups < 1 ||
        Cin % groups != 0 || Cout % groups != 0)
        return CONV_ERR_INVALID_ARG;
    if (1LL * H + pad_top + pad_bottom > kInt32Max / 2 || 1LL * W + pad_left + pad_right > kInt32Max / 2 ||
        1LL * dil_h * (KH - 1) > kInt32Max / 2 || 1LL * dil_w * (KW - 1) > kInt32Max / 2)
        return CONV_ERR_UNSUPPORTED;
    if (1LL * H + pad_top + pad_bottom < 1LL * dil_h * (KH - 1) + 1 ||
        1LL * W + pad_left + pad_right < 1LL * dil_w * (KW - 1) + 1)
        return CONV_ERR_INVALID_ARG;
    DenseGeom g;
    g.KH = KH; g.KW = KW;
    g.sh = stride_h; g.sw = stride_w; g.dh = dil_h; g.dw = dil_w;
    g.ph = pad_top; g.ph_end = pad_bottom; g.pw = pad_left; g.pw_end = pad_right;
    g.groups = groups;
    g.bias = bias;
    return dense_general(X, F, Y, N, H, W, Cin, Cout, g, stream);
}

size_t conv2d_nhwc_im2col_workspace(int N, int H, int W, int Cin, int K) {
    if (N < 1 || H < 1 || W < 1 || Cin < 1 || K < 1 || K > H || K > W) return 0;
    return static_cast<size_t>(1ULL * N * (H - K + 1) * (W - K + 1) * K * K * Cin * 2);
}

int conv2d_nhwc_fwd_im2col(const void *X, const void *F, void *Y, void *workspace, size_t workspace_bytes, int N,
                           int H, int W, int Cin, int Cout, int K, cudaStream_t stream) {
    if (int rc = check_dense(X, F, Y, N, H, W, Cin, Cout, K, 2)) return rc;
    const size_t need = conv2d_nhwc_im2col_workspace(N, H, W, Cin, K);
    if (!workspace || workspace_bytes < need) return CONV_ERR_INVALID_ARG;
    const long long Ho = H - K + 1, Wo = W - K + 1, M = 1LL * N * Ho * Wo, kd = 1LL * K * K * Cin;
    if (M * kd > kInt32Max * 4LL || M > kInt32Max || kd > kInt32Max) return CONV_ERR_UNSUPPORTED;
    if (!aligned(workspace, 16)) return CONV_ERR_MISALIGNED;
    const long long nx = 1LL * N * H * W * Cin, nf = kd * Cout, ny = M * Cout;
    if (overlaps(workspace, static_cast<long long>(need), X, 2 * nx) ||
        overlaps(workspace, static_cast<long long>(need), F, 2 * nf) ||
        overlaps(workspace, static_cast<long long>(need), Y, 2 * ny))
        return CONV_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {X, F, Y, workspace})) return rc;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!d->blas && cublasCreate(&d->blas) != CUBLAS_STATUS_SUCCESS) return CONV_ERR_CUDA;
    }
    Im2colParams p;
    p.H = H; p.W = W; p.Cin = Cin; p.K = K; p.Ho = static_cast<int>(Ho); p.Wo = static_cast<int>(Wo);
    p.kd = static_cast<int>(kd);
    p.chunk = (Cin % 8 == 0 && aligned(X, 16)) ? 8 : 1;
    p.chunks = M * kd / p.chunk;
    long long blocks = (p.chunks + 255) / 256;
    if (blocks > 1LL * d->num_sms * 8) blocks = 1LL * d->num_sms * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    auto *A = static_cast<__nv_bfloat16 *>(workspace);
    if (launched(launch_k(cfg, im2col_pack_kernel, static_cast<const __nv_bfloat16 *>(X), A, p, d->status),
                 "im2col_pack_kernel") != CONV_OK)
        return CONV_ERR_CUDA;
    // Y (M x Cout, row-major) = A (M x kd) * F (kd x Cout): in cuBLAS's column-major terms
    // Y^T = F^T * A^T with leading dimensions Cout, Cout and kd
    const float alpha = 1.0f, beta = 0.0f;
    if (cublasSetStream(d->blas, stream) != CUBLAS_STATUS_SUCCESS) return CONV_ERR_CUDA;
    if (cublasGemmEx(d->blas, CUBLAS_OP_N, CUBLAS_OP_N, Cout, static_cast<int>(M), static_cast<int>(kd), &alpha, F,
                     CUDA_R_16BF, Cout, A, CUDA_R_16BF, static_cast<int>(kd), &beta, Y, CUDA_R_16BF, Cout,
                     CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
        return CONV_ERR_CUDA;
    t_last_kernel = "im2col_pack_kernel+cublas";
    return CONV_OK;
}

int conv2d_nhwc_fwd_im2col_noalloc(const void *X, const void *F, void *Y, int N, int H, int W, int Cin, int Cout,
                                   int K, cudaStream_t stream) {
    if (int rc = check_dense(X, F, Y, N, H, W, Cin, Cout, K, 2)) return rc;
    const size_t need = conv2d_nhwc_im2col_workspace(N, H, W, Cin, K);
    if (need > CONV_IM2COL_STATIC_BYTES) return CONV_ERR_UNSUPPORTED;
    const long long Ho = H - K + 1, Wo = W - K + 1, M = 1LL * N * Ho * Wo, kd = 1LL * K * K * Cin;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {X, F, Y})) return rc;
    void *scratch = nullptr;
    {   // set-up once per device, this device current: the array's device address
        std::lock_guard<std::mutex> lock(g_mu);
        if (!d->im2col_scratch) {
            void *addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_im2col_scratch) != cudaSuccess) return CONV_ERR_CUDA;
            d->im2col_scratch = addr;
        }
        scratch = d->im2col_scratch;
    }
    // the patch matrix: every one of its M * kd entries is written, so stale contents of an
    // earlier call never reach the product
    Im2colParams p;
    p.H = H; p.W = W; p.Cin = Cin; p.K = K; p.Ho = static_cast<int>(Ho); p.Wo = static_cast<int>(Wo);
    p.kd = static_cast<int>(kd);
    p.chunk = (Cin % 8 == 0 && aligned(X, 16)) ? 8 : 1;
    p.chunks = M * kd / p.chunk;
    long long blocks = (p.chunks + 255) / 256;
    if (blocks > 1LL * d->num_sms * 8) blocks = 1LL * d->num_sms * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    auto *A = static_cast<__nv_bfloat16 *>(scratch);
    if (launched(launch_k(cfg, im2col_pack_kernel, static_cast<const __nv_bfloat16 *>(X), A, p, d->status),
                 "im2col_pack_kernel") != CONV_OK)
        return CONV_ERR_CUDA;
    // Y = A * F as the 1 x 1 convolution of the patch image [N][Ho][Wo][kd] with F viewed as
    // [1][1][kd][Cout]
    return dense_plain(A, F, Y, N, static_cast<int>(Ho), static_cast<int>(Wo), static_cast<int>(kd), Cout, 1, stream,
                       d);
}

int depthwise_fwd(const float *x, const float *w, const float *bias, float *y, int N, int Cin, int mult, int H,
                  int W, int KH, int KW, int stride, int pad, int dil, int mode, cudaStream_t stream) {
    if (!x || !w || !y) return CONV_ERR_INVALID_ARG;
    if (N < 1 || Cin < 1 || mult < 1 || H < 1 || W < 1 || KH < 1 || KW < 1 || stride < 1 || dil < 1 || pad < 0)
        return CONV_ERR_INVALID_ARG;
    if (mode != DW_EXACT && mode != DW_FAST) return CONV_ERR_INVALID_ARG;
    const long long Ho = dw_out(H, KH, stride, pad, dil), Wo = dw_out(W, KW, stride, pad, dil);
    if (1LL * H + 2LL * pad < 1LL * dil * (KH - 1) + 1 || 1LL * W + 2LL * pad < 1LL * dil * (KW - 1) + 1 ||
        Ho < 1 || Wo < 1)
        return CONV_ERR_INVALID_ARG;
    const long long Cout = 1LL * Cin * mult;
    const long long nx = 1LL * N * Cin * H * W, nw = Cout * KH * KW, ny = 1LL * N * Cout * Ho * Wo;
    if (Cout > kInt32Max || nx > kInt32Max || nw > kInt32Max || ny > kInt32Max || 1LL * KH * KW > 4096 ||
        1LL * H + 2LL * pad > kInt32Max / 2 || 1LL * W + 2LL * pad > kInt32Max / 2)
        return CONV_ERR_UNSUPPORTED;
    if (!aligned(x, 4) || !aligned(w, 4) || !aligned(y, 4) || (bias && !aligned(bias, 4)))
        return CONV_ERR_MISALIGNED;
    if (overlaps(y, ny * 4, x, nx * 4) || overlaps(y, ny * 4, w, nw * 4) || (bias && overlaps(y, ny * 4, bias, Cout * 4)))
        return CONV_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {x, w, bias, y})) return rc;

    // Register-window kernel for the common shapes (CONV_B200_DW_KERNEL=smem forces the
    // shared-memory kernel, =reg requires the register kernel; tests).
    const char *kforce = env("CONV_B200_DW_KERNEL");
    const bool force_smem = kforce && std::strcmp(kforce, "smem") == 0;
    const bool force_reg = kforce && std::strcmp(kforce, "reg") == 0;
    const bool reg_ok = dw_reg_eligible(KH, KW, stride, pad, dil, Wo) && 1LL * N * Cout <= kInt32Max;
    if (force_reg && !reg_ok) return CONV_ERR_UNSUPPORTED;
    const bool force_tma = kforce && std::strcmp(kforce, "tma") == 0;
    const bool force_plane = kforce && std::strcmp(kforce, "plane") == 0;
    // 7x7 and 14x14 planes: a lane per plane (CONV_B200_DW_KERNEL=plane forces it)
    if (reg_ok && !force_smem && !force_reg && !force_tma && !env("CONV_B200_DW_TILE")) {
        const DwPlanePlan pp = dw_plane_plan(N, Cin, mult, H, W, KH, stride, d->num_sms, x, y);
        if (pp.ok) {
            const bool hb = bias != nullptr;
            if (mode == DW_EXACT)
                return hb ? launch_dw_plane<0, true>(x, w, bias, y, pp, KH, stride, H, stream, d)
                          : launch_dw_plane<0, false>(x, w, bias, y, pp, KH, stride, H, stream, d);
            return hb ? launch_dw_plane<1, true>(x, w, bias, y, pp, KH, stride, H, stream, d)
                      : launch_dw_plane<1, false>(x, w, bias, y, pp, KH, stride, H, stream, d);
        }
    }
    if (force_plane) return CONV_ERR_UNSUPPORTED;
    if (reg_ok && !force_smem && !force_reg && !env("CONV_B200_DW_TILE")) {
        const DwTmaPlan tp = dw_tma_plan(N, Cin, mult, H, W, static_cast<int>(Ho), static_cast<int>(Wo), KH, stride,
                                         d->num_sms, x, y);
        if (tp.ok) {
            const bool hb = bias != nullptr;
            if (mode == DW_EXACT)
                return hb ? launch_dw_tma<0, true>(x, w, bias, y, tp, KH, stride, Cin, N, stream, d)
                          : launch_dw_tma<0, false>(x, w, bias, y, tp, KH, stride, Cin, N, stream, d);
            return hb ? launch_dw_tma<1, true>(x, w, bias, y, tp, KH, stride, Cin, N, stream, d)
                      : launch_dw_tma<1, false>(x, w, bias, y, tp, KH, stride, Cin, N, stream, d);
        }
    }
    if (force_tma) return CONV_ERR_UNSUPPORTED;
    if (reg_ok && !force_smem && !env("CONV_B200_DW_TILE")) {
        const DwRegParams rp = dw_reg_plan(N, Cin, mult, H, W, static_cast<int>(Ho), static_cast<int>(Wo), d->num_sms, x, y);
        const bool hb = bias != nullptr;
        if (mode == DW_EXACT)
            return hb ? launch_dw_reg<0, true>(x, w, bias, y, rp, KH, stride, stream, d)
                      : launch_dw_reg<0, false>(x, w, bias, y, rp, KH, stride, stream, d);
        return hb ? launch_dw_reg<1, true>(x, w, bias, y, rp, KH, stride, stream, d)
                  : launch_dw_reg<1, false>(x, w, bias, y, rp, KH, stride, stream, d);
    }

    DwParams p;
    p.Cin = Cin; p.mult = mult; p.Cout = static_cast<int>(Cout); p.H = H; p.W = W; p.KH = KH; p.KW = KW;
    p.stride = stride; p.pad = pad; p.dil = dil; p.Ho = static_cast<int>(Ho); p.Wo = static_cast<int>(Wo);
    p.num_planes = static_cast<int>(1LL * N * Cout);
    p.w_stride = (KH * KW + 3) & ~3;
    DwSpec spec = dw_spec(p);
    if (const char *g = env("CONV_B200_DW_GENERIC"))   // force the runtime-shape kernel (tests)
        if (g[0] == '1') spec = kDwGeneric;
    dw_choose_tiles(p, spec);
    if (const char *t = env("CONV_B200_DW_TILE")) {   // "P,R,CW": a forced job shape (tests)
        int P = 0, R = 0, CW = 0;
        if (std::sscanf(t, "%d,%d,%d", &P, &R, &CW) == 3 && P >= 1 && R >= 1 && CW >= 1) {
            const int vx = dw_vx(spec);
            p.R = R < p.Ho ? R : p.Ho;
            p.CW = CW < p.Wo ? ((CW + vx - 1) / vx) * vx : p.Wo;
            if (p.CW > p.Wo) p.CW = p.Wo;
            p.P = (p.R == p.Ho && p.CW == p.Wo) ? (P < p.num_planes ? P : p.num_planes) : 1;
            dw_set_window(p, spec);
        }
    }
    if (dw_smem_bytes(p) > 227 * 1024) return CONV_ERR_UNSUPPORTED;
    p.n_rbands = (p.Ho + p.R - 1) / p.R;
    p.n_cbands = (p.Wo + p.CW - 1) / p.CW;
    const long long groups = (p.num_planes + p.P - 1) / p.P;
    const long long jobs = groups * p.n_rbands * p.n_cbands;
    if (jobs > kInt32Max) return CONV_ERR_UNSUPPORTED;
    p.vec_store = (p.Wo % 4 == 0 && aligned(y, 16)) ? 1 : 0;
    p.div_cout = make_fastdiv(static_cast<uint32_t>(p.Cout));
    p.div_mult = make_fastdiv(static_cast<uint32_t>(p.mult));
    p.div_taps = make_fastdiv(static_cast<uint32_t>(KH * KW));
    p.div_cbands = make_fastdiv(static_cast<uint32_t>(p.n_cbands));
    p.div_rbands = make_fastdiv(static_cast<uint32_t>(p.n_rbands));
    const bool hb = bias != nullptr;
    if (mode == DW_EXACT)
        return hb ? launch_dw<0, true>(x, w, bias, y, p, spec, jobs, stream, d)
                  : launch_dw<0, false>(x, w, bias, y, p, spec, jobs, stream, d);
    return hb ? launch_dw<1, true>(x, w, bias, y, p, spec, jobs, stream, d)
              : launch_dw<1, false>(x, w, bias, y, p, spec, jobs, stream, d);
}

const char *conv_status_string(int status) {
    switch (status) {
        case CONV_OK: return "ok";
        case CONV_ERR_INVALID_ARG: return "invalid argument";
        case CONV_ERR_UNSUPPORTED: return "unsupported shape or size";
        case CONV_ERR_MISALIGNED: return "misaligned pointer";
        case CONV_ERR_CUDA: return "CUDA call failed";
        case CONV_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case CONV_ERR_DEVICE_BOUNDS: return "device-side bounds check failed (access skipped)";
        default: return "unknown status";
    }
}

const char *conv_last_kernel(void) { return t_last_kernel; }

int conv_selftest_wait_timeout(cudaStream_t stream) {
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(32);
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, selftest_wait_kernel, d->status) == cudaSuccess ? CONV_OK : CONV_ERR_CUDA;
}

int conv_device_status(cudaStream_t stream, int reset) {
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return CONV_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, d->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return CONV_ERR_CUDA;
    if (reset) {
        const unsigned int zero = 0;
        if (cudaMemcpy(d->status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return CONV_ERR_CUDA;
    }
    if (v & kStatusTimeout) return CONV_ERR_DEVICE_TIMEOUT;
    return (v & kStatusBounds) ? CONV_ERR_DEVICE_BOUNDS : CONV_OK;
}

int conv_debug_bounds_build(void) { return kDebugBounds ? 1 : 0; }

int conv_selftest_bounds(cudaStream_t stream) {
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(32);
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, selftest_bounds_kernel, d->status) == cudaSuccess ? CONV_OK : CONV_ERR_CUDA;
}

int conv_debug_bounds_info(long long *info, int reset) {
    if (!info) return CONV_ERR_INVALID_ARG;
    info[0] = info[1] = info[2] = -1;
#ifdef CONV_DEBUG_BOUNDS
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (cudaDeviceSynchronize() != cudaSuccess) return CONV_ERR_CUDA;
    long long rec[4] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbol(rec, g_bounds_first, sizeof rec) != cudaSuccess) return CONV_ERR_CUDA;
    if (rec[0]) {
        info[0] = rec[1];
        info[1] = rec[2];
        info[2] = rec[3];
    }
    if (reset) {
        const long long zero[4] = {0, 0, 0, 0};
        if (cudaMemcpyToSymbol(g_bounds_first, zero, sizeof zero) != cudaSuccess) return CONV_ERR_CUDA;
    }
#else
    (void)reset;
#endif
    return CONV_OK;
}

int dwpw_fwd(const float *x, const float *w_dw, const float *b_dw, const void *F, const float *b_pw, float *y, int N,
             int C, int H, int W, int K, int stride, int pad, int dil, int Cout, int mode, cudaStream_t stream) {
    if (!x || !w_dw || !F || !y) return CONV_ERR_INVALID_ARG;
    if (N < 1 || C < 1 || H < 1 || W < 1 || K < 1 || stride < 1 || dil < 1 || pad < 0 || Cout < 1)
        return CONV_ERR_INVALID_ARG;
    if (mode != DW_EXACT && mode != DW_FAST) return CONV_ERR_INVALID_ARG;
    if (1LL * H + 2LL * pad > kInt32Max / 2 || 1LL * W + 2LL * pad > kInt32Max / 2 ||
        1LL * dil * (K - 1) > kInt32Max / 2)
        return CONV_ERR_UNSUPPORTED;
    if (1LL * H + 2LL * pad < 1LL * dil * (K - 1) + 1 || 1LL * W + 2LL * pad < 1LL * dil * (K - 1) + 1)
        return CONV_ERR_INVALID_ARG;
    const long long Ho = dw_out(H, K, stride, pad, dil), Wo = dw_out(W, K, stride, pad, dil);
    const long long nx = 1LL * N * C * H * W, nw = 1LL * C * K * K, nf = 1LL * C * Cout, ny = 1LL * N * Cout * Ho * Wo;
    if (nx > kInt32Max || nw > kInt32Max || nf > kInt32Max || ny > kInt32Max || 1LL * N * Ho * Wo > kInt32Max - 128 ||
        1LL * K * K > 4096)
        return CONV_ERR_UNSUPPORTED;
    // the pointwise stage runs on the tensor cores: whole 16-byte filter rows, one MMA width
    if (Cout % 8 != 0 || Cout > 256) return CONV_ERR_UNSUPPORTED;
    if (!aligned(F, 16) || !aligned(x, 4) || !aligned(w_dw, 4) || !aligned(y, 4) || (b_dw && !aligned(b_dw, 4)) ||
        (b_pw && !aligned(b_pw, 4)))
        return CONV_ERR_MISALIGNED;
    if (overlaps(y, ny * 4, x, nx * 4) || overlaps(y, ny * 4, w_dw, nw * 4) || overlaps(y, ny * 4, F, nf * 2) ||
        (b_dw && overlaps(y, ny * 4, b_dw, 4LL * C)) || (b_pw && overlaps(y, ny * 4, b_pw, 4LL * Cout)))
        return CONV_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    if (int rc = device_state(&d)) return rc;
    if (int rc = check_device_ptrs(stream, {x, w_dw, b_dw, F, b_pw, y})) return rc;
    alignas(64) CUtensorMap tmF;
    {   // F: 3-D {Cout, C, 1}; a box is 64 channel rows x 64 outputs (rows past C and columns
        // past Cout read zeros)
        const cuuint64_t dims[3] = {(cuuint64_t)Cout, (cuuint64_t)C, 1};
        const cuuint64_t strides[2] = {(cuuint64_t)Cout * 2, (cuuint64_t)C * Cout * 2};
        const cuuint32_t box[3] = {64, 64, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode_tiled(&tmF, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(F), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONV_ERR_CUDA;
    }
    DwPwParams p;
    p.C = C; p.H = H; p.W = W; p.Ho = static_cast<int>(Ho); p.Wo = static_cast<int>(Wo); p.HoWo = p.Ho * p.Wo;
    p.K = K; p.stride = stride; p.pad = pad; p.dil = dil;
    p.Cout = Cout;
    p.n_mma = (Cout + 15) / 16 * 16;
    p.n_boxes = (Cout + 63) / 64;
    p.num_kblk = (C + 63) / 64;
    p.M = static_cast<int>(1LL * N * Ho * Wo);
    p.num_tiles = (p.M + 127) / 128;
    p.idesc = idesc_bf16_f32(128, p.n_mma, /*B MN-major*/ true);
    p.tmem_cols = 32;
    while (p.tmem_cols < static_cast<uint32_t>(p.n_mma)) p.tmem_cols <<= 1;
    p.b_dw = b_dw;
    p.b_pw = b_pw;
    p.div_howo = make_fastdiv(static_cast<uint32_t>(p.HoWo));
    p.div_wo = make_fastdiv(static_cast<uint32_t>(p.Wo));
    // CONV_B200_DWPW_SPLIT (tests) forces the channel split S = 1..4; otherwise the launcher
    // picks the split that fills the GPU best
    int force_split = 0;
    if (const char *f = env("CONV_B200_DWPW_SPLIT")) {
        force_split = std::atoi(f);
        if (force_split < 1 || force_split > 4) return CONV_ERR_UNSUPPORTED;
    }
    p.S = 1;
    p.owned = p.n_mma / 16;
    // 7x7 and 14x14 images with 3x3 or 5x5 "same" filters: the transposed-GEMM kernel; other 3x3
    // and 5x5 shapes whose tiles fit: the kernel that stages input windows in shared memory
    // (CONV_B200_DWPW_KERNEL=gemm / staged / flat forces one; tests)
    const char *kforce = env("CONV_B200_DWPW_KERNEL");
    const bool force_flat = kforce && std::strcmp(kforce, "flat") == 0;
    const bool force_staged = kforce && std::strcmp(kforce, "staged") == 0;
    const bool force_gemm = kforce && std::strcmp(kforce, "gemm") == 0;
    if (!force_flat && !force_staged && force_split <= 2) {
        if (dwpw_gemm_eligible(C, H, W, K, stride, pad, dil, Cout, x, w_dw, y))
            return mode == DW_EXACT ? launch_dwpw_gemm<0>(x, w_dw, b_dw, F, b_pw, y, N, C, H, K, Cout, stream, d)
                                    : launch_dwpw_gemm<1>(x, w_dw, b_dw, F, b_pw, y, N, C, H, K, Cout, stream, d);
    }
    if (force_gemm) return CONV_ERR_UNSUPPORTED;
    if (!force_flat) {
        const DwPwStagePlan pl = plan_dwpw_staged(p, N);
        if (pl.ok) {
            if (mode == DW_EXACT)
                return K == 3 ? launch_dwpw_staged<0, 3>(x, w_dw, tmF, y, p, pl, force_split, stream, d, 57)
                              : launch_dwpw_staged<0, 5>(x, w_dw, tmF, y, p, pl, force_split, stream, d, 58);
            return K == 3 ? launch_dwpw_staged<1, 3>(x, w_dw, tmF, y, p, pl, force_split, stream, d, 59)
                          : launch_dwpw_staged<1, 5>(x, w_dw, tmF, y, p, pl, force_split, stream, d, 60);
        }
        if (kforce && std::strcmp(kforce, "staged") == 0) return CONV_ERR_UNSUPPORTED;
    }
    // The flat kernel: for K = 3 and K = 5 it keeps the depthwise weights in shared memory when
    // they fit; other filter sizes (or very many channels) read them from global memory.
    const bool w_in_smem = (K == 3 || K == 5) && 4LL * C * dwpw_kkp(K) <= kDwPwMaxSmem - kDwPwFixed;
    p.w_floats = w_in_smem ? C * dwpw_kkp(K) : 0;
    if (mode == DW_EXACT) {
        if (w_in_smem && K == 3) return launch_dwpw<0, 3>(x, w_dw, tmF, y, p, force_split, stream, d, 51);
        if (w_in_smem && K == 5) return launch_dwpw<0, 5>(x, w_dw, tmF, y, p, force_split, stream, d, 52);
        return launch_dwpw<0, 0>(x, w_dw, tmF, y, p, force_split, stream, d, 53);
    }
    if (w_in_smem && K == 3) return launch_dwpw<1, 3>(x, w_dw, tmF, y, p, force_split, stream, d, 54);
    if (w_in_smem && K == 5) return launch_dwpw<1, 5>(x, w_dw, tmF, y, p, force_split, stream, d, 55);
    return launch_dwpw<1, 0>(x, w_dw, tmF, y, p, force_split, stream, d, 56);
}

}  // extern "C"
