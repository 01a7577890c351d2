/*
 * conv_b200 -- forward 2-D convolution for NVIDIA B200 (sm_100a), C ABI.
 *
 * Two operations, both in the neural-network cross-correlation convention (the filter is
 * not reversed):
 *
 *  1. Dense NHWC convolution with a square K x K filter, unit stride, no padding, no
 *     dilation, no groups and no bias. Defined in the CMU DLSys Lecture 14 notes, "The hidden
 *     copy behind convolution as matrix multiplication", section 1 "Fix the index contract
 *     before optimizing it":
 *         Ho = H - K + 1,  Wo = W - K + 1,
 *         Y[n,y,x,o] = sum_{i<K} sum_{j<K} sum_{c<Cin} X[n,y+i,x+j,c] * F[i,j,c,o].
 *     Section 5 of the same notes gives the matrix form the kernel evaluates without ever
 *     storing the patch matrix: rows are the N*Ho*Wo output pixels, the reduction runs over
 *     (i, j, c) and the columns are the Cout filters.
 *
 *  2. Depthwise convolution (groups == Cin, Cout = Cin * mult) on NCHW planes with stride,
 *     zero padding, dilation and an optional bias. Defined in the OneModel docs, "Depthwise
 *     convolution", section "What each output is": output channel oc reads input channel
 *     oc / mult; acc starts at +0; taps run ky outer, kx inner; padding is a real zero that
 *     is multiplied (so an infinite or NaN weight meeting padding gives NaN); the bias is a
 *     separate pass of one rounded addition. Output size per axis from "Convolution Is Wx+b
 *     Moving Across a Signal", section "Build an image-gradient map, one number at a time":
 *         out = floor((in + 2*pad - (dil*(k-1) + 1)) / stride) + 1.
 *
 * Around them: the dense operation with stride, padding, dilation and bias (conv2d_nhwc_fwd_ex),
 * with channel groups, KH x KW filters and per-axis geometry, Conv1D included
 * (conv2d_nhwc_fwd_grouped), a depthwise pass fused with the pointwise pass after it (dwpw_fwd),
 * and an explicit-im2col comparison path (conv2d_nhwc_fwd_im2col).
 *
 * Common rules for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller (for example allocated by
 *    PyTorch). Tensors are dense and contiguous in the stated layout. The library keeps no
 *    reference to them after the call returns and allocates no device memory per call.
 *  - Kernels run on the CURRENT device (cudaGetDevice). Every tensor must be memory of that
 *    device (or managed memory); a tensor of another GPU, or host memory, returns
 *    CONV_ERR_INVALID_ARG. The check is made on every call except while `stream` is being
 *    captured into a CUDA graph.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream) and never synchronise.
 *    Outputs are fully overwritten. Inputs are read only. Outputs must not overlap inputs.
 *  - The return value is a conv_status; no exception or abort crosses the ABI. Argument
 *    checks happen before any CUDA call, so a rejected call has no effect on the device.
 *  - A device-side wait that exceeds its time limit (about one second) makes the kernel
 *    stop, record CONV_ERR_DEVICE_TIMEOUT in a per-process device status word and return;
 *    read it with conv_device_status().
 *  - The first call of a kernel (and, for dwpw_fwd, of a shape) on a device raises that
 *    kernel's shared-memory limit and asks the runtime how many thread-block clusters fit;
 *    make that first call outside CUDA-graph stream capture. Later calls only launch.
 */
#ifndef CONV_B200_H
#define CONV_B200_H

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CONV_OK = 0,
    CONV_ERR_INVALID_ARG = -1,    /* null tensor pointer, non-positive size, K > min(H, W), ... */
    CONV_ERR_UNSUPPORTED = -2,    /* valid arguments outside what this library implements */
    CONV_ERR_MISALIGNED = -3,     /* a pointer not aligned to its element size */
    CONV_ERR_CUDA = -4,           /* a CUDA runtime or driver call failed (launch, tensor map) */
    CONV_ERR_DEVICE_TIMEOUT = -5, /* a bounded device-side wait ran out (see conv_device_status) */
    CONV_ERR_DEVICE_BOUNDS = -6   /* bounds-checked build only: a kernel skipped an access outside
                                     its tensor (see conv_debug_bounds_info) */
} conv_status;

typedef enum {
    DW_EXACT = 0, /* product rounded, then sum rounded; NaN results become 0x7FC00000 */
    DW_FAST = 1   /* one fused multiply-add per tap */
} dw_mode;

/*
 * Dense NHWC forward convolution, bfloat16 in and out, float32 accumulation.
 *   X : bfloat16 [N][H][W][Cin]          (NHWC, channels contiguous)
 *   F : bfloat16 [K][K][Cin][Cout]       (KKIO: row (i, j, c) of the K*K*Cin x Cout matrix)
 *   Y : bfloat16 [N][H-K+1][W-K+1][Cout] (NHWC), each output rounded to nearest even once
 * Requirements: N, H, W, Cin, Cout, K >= 1; K <= min(H, W); all pointers non-null and
 * 2-byte aligned; N*H*W*Cin, N*Ho*Wo*Cout and K*K*Cin*Cout below 2^31.
 * The tensor-core path needs Cin and Cout multiples of 8, 16-byte aligned pointers and
 * K <= 128; other valid shapes take a CUDA-core path with the same contract.
 */
int conv2d_nhwc_fwd(const void *X, const void *F, void *Y,
                    int N, int H, int W, int Cin, int Cout, int K, cudaStream_t stream);

/*
 * The same operation with float32 tensors (same layouts and requirements; 4-byte aligned
 * pointers). Products and sums are float32 fused multiply-adds in (i, j, c) order, so any
 * input whose partial sums are integers below 2^24 in magnitude gives the exact result.
 */
int conv2d_nhwc_fwd_f32(const float *X, const float *F, float *Y,
                        int N, int H, int W, int Cin, int Cout, int K, cudaStream_t stream);

/*
 * Dense NHWC forward convolution with stride, symmetric zero padding, dilation and an optional
 * bias: the variants of "Convolution Is Wx+b Moving Across a Signal" (section "Build an
 * image-gradient map, one number at a time" for the output size; section "Find the same sum in
 * CKE's C kernels" for the window indexing out*stride + tap - padding):
 *     Ho = floor((H + 2*pad - (dil*(K-1) + 1)) / stride) + 1   (Wo likewise),
 *     Y[n,y,x,o] = bias[o] + sum_{i,j,c} X[n, y*stride + i*dil - pad, x*stride + j*dil - pad, c]
 *                                         * F[i,j,c,o],
 * with X read as zero outside the image.
 *   X, F, Y : bfloat16, layouts as conv2d_nhwc_fwd (Y is [N][Ho][Wo][Cout])
 *   bias    : float32 [Cout] or NULL; added in float32 to the float32 sum before the single
 *             rounding to bfloat16
 * Requirements: N, H, W, Cin, Cout, K, stride, dil >= 1; pad >= 0; Ho, Wo >= 1; X, F, Y non-null
 * and 2-byte aligned, bias 4-byte aligned; element counts below 2^31. With stride 1, pad 0,
 * dil 1 and no bias this is exactly conv2d_nhwc_fwd. Otherwise the tensor-core path needs Cin and
 * Cout multiples of 8, 16-byte aligned tensors, pad <= 127, dil*(K-1) <= 127 and
 * |pad - dil*(K-1)| <= 127; other valid shapes take a CUDA-core path with the same contract.
 */
int conv2d_nhwc_fwd_ex(const void *X, const void *F, const float *bias, void *Y,
                       int N, int H, int W, int Cin, int Cout, int K,
                       int stride, int pad, int dil, cudaStream_t stream);

/*
 * Grouped dense NHWC forward convolution with a KH x KW filter and separate height and width
 * geometry; a Conv1D over a sequence of W frames is the H = KH = 1 case. The grouping is the
 * one "Convolution Is Wx+b Moving Across a Signal" describes in section "Find the same sum in
 * CKE's C kernels" (an output channel sums only the input channels and taps of its own group,
 * frame index out*stride + tap - padding, taps outside the input skipped), extended to two
 * axes as that section's 2-D grouped kernel does:
 *     Cin_g = Cin / groups, Cout_g = Cout / groups, g(o) = o / Cout_g,
 *     Ho = floor((H + 2*pad_h - (dil_h*(KH-1) + 1)) / stride_h) + 1   (Wo likewise with _w),
 *     Y[n,y,x,o] = bias[o] + sum_{i<KH, j<KW, c<Cin_g}
 *                  X[n, y*stride_h + i*dil_h - pad_h, x*stride_w + j*dil_w - pad_w, g(o)*Cin_g + c]
 *                  * F[i,j,c,o],
 * with X read as zero outside the image.
 *   X    : bfloat16 [N][H][W][Cin]
 *   F    : bfloat16 [KH][KW][Cin_g][Cout] (row (i, j, c) of group g(o)'s filter matrix, column o)
 *   bias : float32 [Cout] or NULL; added in float32 to the float32 sum before the single
 *          rounding to bfloat16 (the order of the dense entries; the page's scalar Conv1D starts
 *          its float32 accumulator at the bias instead, which only reorders the rounding)
 *   Y    : bfloat16 [N][Ho][Wo][Cout]
 * Requirements: N, H, W, Cin, Cout, KH, KW, strides, dilations, groups >= 1; pads >= 0; groups
 * divides Cin and Cout; Ho, Wo >= 1; X, F, Y non-null and 2-byte aligned, bias 4-byte aligned;
 * element counts below 2^31. With KH = KW, equal per-axis values and one group this is exactly
 * conv2d_nhwc_fwd_ex. The tensor-core path needs Cin_g and Cout_g multiples of 8, 16-byte aligned
 * tensors and, per axis, pad <= 127, dil*(taps-1) <= 127 and |pad - dil*(taps-1)| <= 127; other
 * valid shapes take a CUDA-core path with the same contract. Several groups run as independent
 * implicit GEMMs inside one persistent launch per 8 groups.
 */
int conv2d_nhwc_fwd_grouped(const void *X, const void *F, const float *bias, void *Y,
                            int N, int H, int W, int Cin, int Cout, int KH, int KW,
                            int stride_h, int stride_w, int pad_h, int pad_w, int dil_h, int dil_w,
                            int groups, cudaStream_t stream);

/*
 * conv2d_nhwc_fwd_grouped with separate zero padding before and after each axis: pad_top rows
 * above the image and pad_bottom below it, pad_left columns before and pad_right after. An
 * output's window starts at (y*stride_h - pad_top, x*stride_w - pad_left) and
 *     Ho = floor((H + pad_top + pad_bottom - (dil_h*(KH-1) + 1)) / stride_h) + 1   (Wo likewise).
 * The causal Conv1D of "Convolution Is Wx+b Moving Across a Signal", section "Find the same sum
 * in CKE's C kernels" -- a frame's output reads no later frame -- is H = KH = 1 with
 * pad_left = dil_w*(KW-1) and pad_right = 0 (Wo = W for stride 1).
 * Layouts, bias rule and requirements as conv2d_nhwc_fwd_grouped (every pad >= 0); with equal
 * padding before and after both axes this is exactly conv2d_nhwc_fwd_grouped. The tensor-core
 * path needs, per axis, pad_before <= 127, dil*(taps-1) <= 127 and |pad_after - dil*(taps-1)|
 * <= 127 besides its channel and alignment rules; other valid shapes take the CUDA-core path.
 */
int conv2d_nhwc_fwd_grouped_pads(const void *X, const void *F, const float *bias, void *Y,
                                 int N, int H, int W, int Cin, int Cout, int KH, int KW,
                                 int stride_h, int stride_w, int pad_top, int pad_bottom, int pad_left,
                                 int pad_right, int dil_h, int dil_w, int groups, cudaStream_t stream);

/*
 * Comparison path: the same operation as conv2d_nhwc_fwd computed the way the CMU DLSys Lecture
 * 14 notes build it in section 5 "Generalize the patch matrix to channels and batches" -- an
 * explicit patch matrix A[(n,y,x), (i,j,c)] = X[n,y+i,x+j,c] of N*Ho*Wo rows by K*K*Cin columns,
 * written to `workspace`, then one library GEMM Y = A * F (cuBLAS: bf16 operands, float32
 * accumulation, bf16 output). It exists to measure the storage bill of section 6 against the
 * implicit kernels; the pages have no separate definition for it.
 *   workspace       : DEVICE memory owned by the caller, at least conv2d_nhwc_im2col_workspace()
 *                     bytes, 16-byte aligned, not overlapping X, F or Y; overwritten
 * Requirements as conv2d_nhwc_fwd. The first call on a device creates a cuBLAS handle (which
 * allocates cuBLAS's own workspace); later calls allocate nothing.
 */
size_t conv2d_nhwc_im2col_workspace(int N, int H, int W, int Cin, int K);   /* 0 if invalid */
int conv2d_nhwc_fwd_im2col(const void *X, const void *F, void *Y, void *workspace, size_t workspace_bytes,
                           int N, int H, int W, int Cin, int Cout, int K, cudaStream_t stream);

/*
 * conv2d_nhwc_fwd_im2col without the caller's workspace and without any device allocation:
 * the patch matrix goes to scratch memory the library reserves statically. This entry has no
 * counterpart on the pages; it exists for callers that cannot allocate device memory -- code
 * running under a framework that owns every byte of the device through its own pool, a plugin
 * inside a host application that forbids allocation, or a real-time path that must not risk
 * cudaMalloc's implicit synchronisation or an out-of-memory failure after start-up.
 *   X, F, Y : as conv2d_nhwc_fwd (bfloat16 NHWC input, KKIO filter, NHWC output), caller-owned
 * The result is Y = A * F with the patch matrix A of conv2d_nhwc_fwd_im2col (same rows, columns
 * and (i, j, c) order); the product runs on this library's own tensor-core kernels as the
 * 1 x 1 convolution of A, viewed as an N x Ho x Wo image of K*K*Cin channels, with F viewed as
 * [1][1][K*K*Cin][Cout] (float32 accumulation, one rounding to bfloat16), so it matches the
 * workspace entry within the dense tolerance rather than bit for bit.
 * Scratch: one array of CONV_IM2COL_STATIC_BYTES in device memory per GPU that loads the library,
 * held until the process exits. A patch matrix larger than that (N*Ho*Wo*K*K*Cin*2 bytes)
 * returns CONV_ERR_UNSUPPORTED before any CUDA call. Every call overwrites the whole patch
 * matrix it reads, so nothing needs clearing between calls, but all calls on a device share
 * the one array: calls whose kernels overlap in time on the GPU (different streams without an
 * ordering between them) race on it and give wrong results. Order them on one stream.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and raises kernel shared-memory limits; make that first call before
 * any stream capture. The function calls no cudaMalloc, cudaFree or allocating library routine.
 * Other requirements and status codes as conv2d_nhwc_fwd; conv_last_kernel() afterwards names
 * the kernel that ran the product.
 */
#define CONV_IM2COL_STATIC_BYTES (32u * 1024u * 1024u)
int conv2d_nhwc_fwd_im2col_noalloc(const void *X, const void *F, void *Y,
                                   int N, int H, int W, int Cin, int Cout, int K, cudaStream_t stream);

/*
 * Depthwise forward convolution, float32.
 *   x    : [N][Cin][H][W]
 *   w    : [Cin*mult][KH][KW]   (plane oc belongs to input channel oc / mult)
 *   bias : [Cin*mult] or NULL
 *   y    : [N][Cin*mult][Ho][Wo]
 * stride, pad and dil apply to both axes; padding is symmetric. mode is DW_EXACT or DW_FAST.
 * Requirements: N, Cin, mult, H, W, KH, KW, stride, dil >= 1; pad >= 0; Ho, Wo >= 1;
 * pointers non-null (bias may be NULL) and 4-byte aligned; element counts below 2^31.
 * Exact mode is bit-for-bit the page's definition; fast mode uses a correctly rounded
 * fused multiply-add per tap in the same order.
 */
int depthwise_fwd(const float *x, const float *w, const float *bias, float *y,
                  int N, int Cin, int mult, int H, int W, int KH, int KW,
                  int stride, int pad, int dil, int mode, cudaStream_t stream);

/*
 * A depthwise K x K pass followed by a pointwise 1 x 1 pass, fused in one kernel: the block of
 * "Convolution Is Wx+b Moving Across a Signal", section "Why variants matter" (a depthwise filter
 * per channel, then a channel-mixing 1 x 1 layer). The intermediate never goes to memory.
 *     d[n,c,oy,ox] = depthwise_fwd's output for multiplier 1 (same order, mode and bias rule),
 *     y[n,o,oy,ox] = b_pw[o] + sum_c bf16(d[n,c,oy,ox]) * F[c,o],
 * with bf16() rounding to nearest even (the tensor cores' operand type), the sum accumulated in
 * float32 and b_pw added once in float32.
 *   x    : float32 [N][C][H][W]
 *   w_dw : float32 [C][K][K];  b_dw : float32 [C] or NULL
 *   F    : bfloat16 [C][Cout], 16-byte aligned;  b_pw : float32 [Cout] or NULL
 *   y    : float32 [N][Cout][Ho][Wo], Ho/Wo as depthwise_fwd (stride, pad, dil on both axes)
 * Requirements: N, C, H, W, K, stride, dil, Cout >= 1; pad >= 0; Ho, Wo >= 1; mode DW_EXACT or
 * DW_FAST; x, w_dw, y, biases 4-byte aligned; element counts below 2^31. Cout must be a multiple
 * of 8 and at most 256 (one tensor-core tile width); other Cout return CONV_ERR_UNSUPPORTED.
 */
int dwpw_fwd(const float *x, const float *w_dw, const float *b_dw, const void *F, const float *b_pw, float *y,
             int N, int C, int H, int W, int K, int stride, int pad, int dil, int Cout, int mode,
             cudaStream_t stream);

/* Static English text for a conv_status value (never NULL). */
const char *conv_status_string(int status);

/*
 * Synchronises `stream`, then reads the device status word of the current device:
 * CONV_OK, CONV_ERR_DEVICE_TIMEOUT, CONV_ERR_DEVICE_BOUNDS (bounds-checked build only; a timeout
 * takes precedence), or CONV_ERR_CUDA if the synchronisation itself failed. With reset != 0
 * the word is cleared afterwards.
 */
int conv_device_status(cudaStream_t stream, int reset);

/*
 * The bounds-checked build. The library's sources compiled with -DCONV_DEBUG_BOUNDS (the file
 * libconv_b200_debug.so beside libconv_b200.so; the Python binding loads it when
 * CONV_B200_DEBUG_BOUNDS=1 at import) check every global-memory element range a kernel computes
 * before touching it -- plain loads and stores, and 1-D bulk copies, which no tensor map bounds
 * -- against the extent of the tensor it belongs to. A failed check sets CONV_ERR_DEVICE_BOUNDS
 * in the device status word, records the first failure, and skips the access (a skipped bulk
 * copy still completes its barrier's byte count, so no wait is left hanging); no assertion or
 * trap is raised and the context stays usable. Tensor-map copies are bounded by the hardware
 * and are not checked. These are a debugging aid of this library; the pages describe no such
 * mode.
 *
 * conv_debug_bounds_build: 1 in the bounds-checked build, 0 in the normal one (no device access).
 * conv_debug_bounds_info: synchronises the current device and writes to info[0..2] the first
 * failed check since the last reset -- the site (an internal identifier of the access), the
 * element index and the tensor's element count -- or -1, -1, -1 if none (always so in the
 * normal build); reset != 0 clears the record. Returns CONV_OK, CONV_ERR_INVALID_ARG for a null
 * info, or CONV_ERR_CUDA.
 */
int conv_debug_bounds_build(void);
int conv_debug_bounds_info(long long *info, int reset);

/*
 * Diagnostic for the bounds checks: one kernel thread checks the element range [1000, 1001) of
 * a notional 1000-element tensor and touches no memory whatever the outcome. In the
 * bounds-checked build the check fails: the status word gets CONV_ERR_DEVICE_BOUNDS and
 * conv_debug_bounds_info reports site 255, index 1000, limit 1000. In the normal build nothing
 * is recorded. Returns the launch status.
 */
int conv_selftest_bounds(cudaStream_t stream);

/*
 * Name of the kernel family the last successful conv2d_nhwc_fwd, conv2d_nhwc_fwd_f32 or
 * depthwise_fwd call on the calling host thread launched ("dense_halo_kernel",
 * "dense_tc_kernel", "dense_direct_kernel", "depthwise_tma_kernel", "depthwise_reg_kernel",
 * "depthwise_kernel"); "" before the first one. Static storage, never NULL. Host only: it
 * reports the dispatcher's choice, it does not wait for the kernel.
 */
const char *conv_last_kernel(void);

/*
 * Diagnostic for the bounded device waits: launches one CTA that waits, with the same bounded
 * wait every kernel of the library uses, on a shared-memory barrier that nothing completes.
 * After about one second of SM clock cycles the wait gives up, the kernel records
 * CONV_ERR_DEVICE_TIMEOUT in the device status word and returns normally; the CUDA context
 * stays usable. Returns the launch status; read the outcome with conv_device_status().
 */
int conv_selftest_wait_timeout(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CONV_B200_H */
