/*
 * Oracle for the forward convolutions: plain, slow and written to be read against the
 * pages it follows. This is TEST INFRASTRUCTURE. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the library's CUDA path never calls it and
 * shares no code with it.
 *
 * Dense NHWC convolution -- CMU DLSys Lecture 14 notes, "The hidden copy behind convolution
 * as matrix multiplication", section 1 "Fix the index contract before optimizing it":
 *   X is N x H x W x Cin, F is K x K x Cin x Cout (KKIO), Ho = H-K+1, Wo = W-K+1, and
 *   Y[n,y,x,o] = sum_{i<K} sum_{j<K} sum_{c<Cin} X[n,y+i,x+j,c] * F[i,j,c,o]
 *   with the filter not reversed (cross-correlation). The same section calls the direct
 *   seven-loop form the small correctness oracle; that is what oracle_conv2d_nhwc is.
 *   Arithmetic is float64. For bfloat16 or small-integer float32 operands every product
 *   is exact in float64, so the result is the exact sum up to float64 summation error.
 *
 * Depthwise convolution -- OneModel docs, "Depthwise convolution", section "What each
 * output is": output channel oc reads input channel oc / mult; acc starts at +0; taps go
 * ky outer, kx inner; padding is a real zero that is multiplied; exact mode rounds the
 * product and then the sum (no fused operation) and rewrites a NaN result as 0x7FC00000;
 * fast mode uses one fused multiply-add per tap; a bias is a separate pass of one rounded
 * addition per output. Output size per axis follows "Convolution Is Wx+b Moving Across a
 * Signal", section "Build an image-gradient map, one number at a time":
 *   out = floor((in + 2*pad - (dil*(k-1)+1)) / stride) + 1.
 * Padding is read as symmetric (pad zeros before and after each axis). The file must be
 * built with -ffp-contract=off and without fast-math so that every float operation below
 * is one IEEE binary32 operation, rounded to nearest even, with denormals kept.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DW_EXACT 0
#define DW_FAST 1

/* ---------------------------------------------------------------------------------- */
/* Dense                                                                               */
/* ---------------------------------------------------------------------------------- */

/* One output Y[n,y,x,o] and its absolute sum sum|X||F| over the same terms. */
static void dense_one(const float *X, const float *F, int H, int W, int Cin, int Cout, int K,
                      long n, long y, long x, long o, double *out, double *abs_out)
{
    double s = 0.0, a = 0.0;
    for (int i = 0; i < K; ++i)
        for (int j = 0; j < K; ++j)
            for (int c = 0; c < Cin; ++c) {
                double xv = X[((n * H + (y + i)) * W + (x + j)) * Cin + c];
                double fv = F[(((long)i * K + j) * Cin + c) * Cout + o];
                s += xv * fv;
                a += fabs(xv) * fabs(fv);
            }
    *out = s;
    *abs_out = a;
}

/* Full output. Loops n, y, x | i, j, c | o: the output channel o is the innermost loop so
 * that the F row is read contiguously; every output is still summed in (i, j, c) order,
 * exactly as dense_one does. abssum may be NULL. */
void oracle_conv2d_nhwc(const float *X, const float *F, double *Y, double *abssum,
                        int N, int H, int W, int Cin, int Cout, int K)
{
    const int Ho = H - K + 1, Wo = W - K + 1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int n = 0; n < N; ++n)
        for (int y = 0; y < Ho; ++y) {
            double acc[Cout], aacc[Cout];
            for (int x = 0; x < Wo; ++x) {
                for (int o = 0; o < Cout; ++o) { acc[o] = 0.0; aacc[o] = 0.0; }
                for (int i = 0; i < K; ++i)
                    for (int j = 0; j < K; ++j)
                        for (int c = 0; c < Cin; ++c) {
                            double xv = X[(((long)n * H + (y + i)) * W + (x + j)) * Cin + c];
                            const float *frow = F + (((long)i * K + j) * Cin + c) * Cout;
                            for (int o = 0; o < Cout; ++o) {
                                acc[o] += xv * (double)frow[o];
                                aacc[o] += fabs(xv) * fabs((double)frow[o]);
                            }
                        }
                long base = (((long)n * Ho + y) * Wo + x) * Cout;
                for (int o = 0; o < Cout; ++o) {
                    Y[base + o] = acc[o];
                    if (abssum) abssum[base + o] = aacc[o];
                }
            }
        }
}

/* Selected outputs, given as flat indices into Y[N][Ho][Wo][Cout]. */
void oracle_conv2d_nhwc_points(const float *X, const float *F, const int64_t *idx, int64_t npts,
                               double *y, double *abssum,
                               int N, int H, int W, int Cin, int Cout, int K)
{
    const long Ho = H - K + 1, Wo = W - K + 1;
    (void)N;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t p = 0; p < npts; ++p) {
        long t = idx[p];
        long o = t % Cout; t /= Cout;
        long x = t % Wo; t /= Wo;
        long yy = t % Ho; t /= Ho;
        long n = t;
        dense_one(X, F, H, W, Cin, Cout, K, n, yy, x, o, &y[p], &abssum[p]);
    }
}

/* ---------------------------------------------------------------------------------- */
/* Dense with stride, zero padding, dilation and bias                                  */
/* ---------------------------------------------------------------------------------- */
/*
 * The same sum with the variants of "Convolution Is Wx+b Moving Across a Signal": output size
 * per axis from section "Build an image-gradient map, one number at a time",
 *   Ho = floor((H + 2*pad - (dil*(K-1) + 1)) / stride) + 1   (Wo likewise),
 * the window of output (y, x) starting at input row y*stride - pad and column x*stride - pad,
 * filter tap (i, j) reading dil*i rows and dil*j columns further on (the pseudocode of section
 * "Find the same sum in CKE's C kernels" indexes out*stride + tap - padding), positions outside
 * the image reading zero, and a per-output-channel bias added to the sum. Float64; abssum is
 * sum|x||f| + |b| over the same terms.
 */
static long dense_out_size(long in, int k, int stride, int pad, int dil)
{
    long eff = (long)dil * (k - 1) + 1;
    return (in + 2L * pad - eff) / stride + 1;
}

static void dense_ex_one(const float *X, const float *F, const float *bias, int H, int W, int Cin,
                         int Cout, int K, int stride, int pad, int dil, long n, long y, long x, long o,
                         double *out, double *abs_out)
{
    double s = 0.0, a = 0.0;
    for (int i = 0; i < K; ++i)
        for (int j = 0; j < K; ++j) {
            long r = y * stride + (long)i * dil - pad;
            long q = x * stride + (long)j * dil - pad;
            if (r < 0 || r >= H || q < 0 || q >= W) continue;   /* zero padding */
            for (int c = 0; c < Cin; ++c) {
                double xv = X[((n * H + r) * W + q) * Cin + c];
                double fv = F[(((long)i * K + j) * Cin + c) * Cout + o];
                s += xv * fv;
                a += fabs(xv) * fabs(fv);
            }
        }
    if (bias) {
        s += (double)bias[o];
        a += fabs((double)bias[o]);
    }
    *out = s;
    *abs_out = a;
}

/* Full output Y[N][Ho][Wo][Cout]. Returns 0, or -1 when the output would be empty. */
int oracle_conv2d_nhwc_ex(const float *X, const float *F, const float *bias, double *Y, double *abssum,
                          int N, int H, int W, int Cin, int Cout, int K, int stride, int pad, int dil)
{
    const long Ho = dense_out_size(H, K, stride, pad, dil), Wo = dense_out_size(W, K, stride, pad, dil);
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (long n = 0; n < N; ++n)
        for (long y = 0; y < Ho; ++y)
            for (long x = 0; x < Wo; ++x)
                for (long o = 0; o < Cout; ++o) {
                    long t = ((n * Ho + y) * Wo + x) * Cout + o;
                    double a;
                    dense_ex_one(X, F, bias, H, W, Cin, Cout, K, stride, pad, dil, n, y, x, o, &Y[t], &a);
                    if (abssum) abssum[t] = a;
                }
    return 0;
}

/* Selected outputs, given as flat indices into Y[N][Ho][Wo][Cout]. */
int oracle_conv2d_nhwc_ex_points(const float *X, const float *F, const float *bias, const int64_t *idx,
                                 int64_t npts, double *y, double *abssum, int N, int H, int W, int Cin,
                                 int Cout, int K, int stride, int pad, int dil)
{
    const long Ho = dense_out_size(H, K, stride, pad, dil), Wo = dense_out_size(W, K, stride, pad, dil);
    (void)N;
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t p = 0; p < npts; ++p) {
        long t = idx[p];
        long o = t % Cout; t /= Cout;
        long x = t % Wo; t /= Wo;
        long yy = t % Ho; t /= Ho;
        dense_ex_one(X, F, bias, H, W, Cin, Cout, K, stride, pad, dil, t, yy, x, o, &y[p], &abssum[p]);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------- */
/* Grouped, per-axis geometry, non-square kernels (Conv1D is H = KH = 1)                */
/* ---------------------------------------------------------------------------------- */
/*
 * The same sum with the channels split into `groups` independent groups: output channel o
 * belongs to group g = o / (Cout/groups) and reads only input channels g*Cg .. g*Cg + Cg - 1
 * (Cg = Cin/groups) through filter F[i][j][c][o], c < Cg ("Convolution Is Wx+b Moving Across a
 * Signal", section "Find the same sum in CKE's C kernels": grouped Conv1D with a bias). Window
 * and output size per axis as in oracle_conv2d_nhwc_ex, with separate stride, padding and
 * dilation for rows (h) and columns (w); a kernel of KH x KW taps. Float64; abssum as before.
 */
static void grouped_one(const float *X, const float *F, const float *bias, int H, int W, int Cin, int Cout,
                        int KH, int KW, int sh, int sw, int ph, int pw, int dh, int dw, int groups,
                        long n, long y, long x, long o, double *out, double *abs_out)
{
    const int Cg = Cin / groups, Og = Cout / groups;
    const long g = o / Og;
    double s = 0.0, a = 0.0;
    for (int i = 0; i < KH; ++i)
        for (int j = 0; j < KW; ++j) {
            long r = y * sh + (long)i * dh - ph;
            long q = x * sw + (long)j * dw - pw;
            if (r < 0 || r >= H || q < 0 || q >= W) continue;   /* zero padding */
            for (int c = 0; c < Cg; ++c) {
                double xv = X[((n * H + r) * W + q) * Cin + g * Cg + c];
                double fv = F[(((long)i * KW + j) * Cg + c) * Cout + o];
                s += xv * fv;
                a += fabs(xv) * fabs(fv);
            }
        }
    if (bias) {
        s += (double)bias[o];
        a += fabs((double)bias[o]);
    }
    *out = s;
    *abs_out = a;
}

/* Full output Y[N][Ho][Wo][Cout]. Returns 0, or -1 for an empty output or bad groups. */
int oracle_conv2d_grouped(const float *X, const float *F, const float *bias, double *Y, double *abssum,
                          int N, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw, int ph, int pw,
                          int dh, int dw, int groups)
{
    if (groups < 1 || Cin % groups || Cout % groups) return -1;
    const long Ho = dense_out_size(H, KH, sh, ph, dh), Wo = dense_out_size(W, KW, sw, pw, dw);
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (long n = 0; n < N; ++n)
        for (long y = 0; y < Ho; ++y)
            for (long x = 0; x < Wo; ++x)
                for (long o = 0; o < Cout; ++o) {
                    long t = ((n * Ho + y) * Wo + x) * Cout + o;
                    double a;
                    grouped_one(X, F, bias, H, W, Cin, Cout, KH, KW, sh, sw, ph, pw, dh, dw, groups, n, y, x, o,
                                &Y[t], &a);
                    if (abssum) abssum[t] = a;
                }
    return 0;
}

/* Selected outputs of oracle_conv2d_grouped, by flat index into [N][Ho][Wo][Cout]. */
int oracle_conv2d_grouped_points(const float *X, const float *F, const float *bias, const int64_t *idx,
                                 int64_t npts, double *y, double *abssum, int H, int W, int Cin, int Cout, int KH,
                                 int KW, int sh, int sw, int ph, int pw, int dh, int dw, int groups)
{
    if (groups < 1 || Cin % groups || Cout % groups) return -1;
    const long Ho = dense_out_size(H, KH, sh, ph, dh), Wo = dense_out_size(W, KW, sw, pw, dw);
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t p = 0; p < npts; ++p) {
        long t = idx[p];
        long o = t % Cout; t /= Cout;
        long x = t % Wo; t /= Wo;
        long yy = t % Ho; t /= Ho;
        grouped_one(X, F, bias, H, W, Cin, Cout, KH, KW, sh, sw, ph, pw, dh, dw, groups, t, yy, x, o, &y[p],
                    &abssum[p]);
    }
    return 0;
}

/*
 * The grouped sum with separate padding before and after each axis: pad_top / pad_left zeros
 * before the first row / column, pad_bottom / pad_right after the last, so an output's window
 * starts at (y*sh - pad_top, x*sw - pad_left) and Ho = floor((H + pad_top + pad_bottom -
 * (dh*(KH-1) + 1)) / sh) + 1 (Wo likewise). The causal Conv1D of the CKE section of "Convolution
 * Is Wx+b Moving Across a Signal" -- a frame's output reads no later frame -- is H = KH = 1 with
 * pad_left = dw*(KW-1) and pad_right = 0. Per output the sum is grouped_one's, unchanged.
 */
static long out_size_pads(long in, int k, int stride, int pad_begin, int pad_end, int dil)
{
    long eff = (long)dil * (k - 1) + 1;
    return (in + (long)pad_begin + (long)pad_end - eff) / stride + 1;
}

int oracle_conv2d_grouped_pads(const float *X, const float *F, const float *bias, double *Y, double *abssum,
                               int N, int H, int W, int Cin, int Cout, int KH, int KW, int sh, int sw, int pad_top,
                               int pad_bottom, int pad_left, int pad_right, int dh, int dw, int groups)
{
    if (groups < 1 || Cin % groups || Cout % groups) return -1;
    const long Ho = out_size_pads(H, KH, sh, pad_top, pad_bottom, dh);
    const long Wo = out_size_pads(W, KW, sw, pad_left, pad_right, dw);
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (long n = 0; n < N; ++n)
        for (long y = 0; y < Ho; ++y)
            for (long x = 0; x < Wo; ++x)
                for (long o = 0; o < Cout; ++o) {
                    long t = ((n * Ho + y) * Wo + x) * Cout + o;
                    double a;
                    grouped_one(X, F, bias, H, W, Cin, Cout, KH, KW, sh, sw, pad_top, pad_left, dh, dw, groups, n, y,
                                x, o, &Y[t], &a);
                    if (abssum) abssum[t] = a;
                }
    return 0;
}

/* Selected outputs of oracle_conv2d_grouped_pads, by flat index into [N][Ho][Wo][Cout]. */
int oracle_conv2d_grouped_pads_points(const float *X, const float *F, const float *bias, const int64_t *idx,
                                      int64_t npts, double *y, double *abssum, int H, int W, int Cin, int Cout,
                                      int KH, int KW, int sh, int sw, int pad_top, int pad_bottom, int pad_left,
                                      int pad_right, int dh, int dw, int groups)
{
    if (groups < 1 || Cin % groups || Cout % groups) return -1;
    const long Ho = out_size_pads(H, KH, sh, pad_top, pad_bottom, dh);
    const long Wo = out_size_pads(W, KW, sw, pad_left, pad_right, dw);
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t p = 0; p < npts; ++p) {
        long t = idx[p];
        long o = t % Cout; t /= Cout;
        long x = t % Wo; t /= Wo;
        long yy = t % Ho; t /= Ho;
        grouped_one(X, F, bias, H, W, Cin, Cout, KH, KW, sh, sw, pad_top, pad_left, dh, dw, groups, t, yy, x, o,
                    &y[p], &abssum[p]);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------- */
/* Depthwise                                                                           */
/* ---------------------------------------------------------------------------------- */

static float canonical_nan(void)
{
    uint32_t bits = 0x7FC00000u;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

static long dw_out_size(long in, int k, int stride, int pad, int dil)
{
    long eff = (long)dil * (k - 1) + 1;
    return (in + 2L * pad - eff) / stride + 1;
}

/* One output plane position, in the page's order. */
static float dw_one(const float *x, const float *w, const float *bias,
                    int Cin, int mult, int H, int W, int KH, int KW,
                    int stride, int pad, int dil, int mode,
                    long n, long oc, long oy, long ox)
{
    const long ic = oc / mult;
    const float *plane = x + ((n * Cin) + ic) * (long)H * W;
    const float *wp = w + oc * (long)KH * KW;
    float acc = +0.0f;
    for (int ky = 0; ky < KH; ++ky)
        for (int kx = 0; kx < KW; ++kx) {
            long r = oy * stride + (long)ky * dil - pad;
            long q = ox * stride + (long)kx * dil - pad;
            float xv = (r >= 0 && r < H && q >= 0 && q < W) ? plane[r * W + q] : 0.0f;
            float wv = wp[ky * KW + kx];
            if (mode == DW_EXACT) {
                float p = wv * xv;   /* rounded product */
                acc = acc + p;       /* rounded sum */
            } else {
                acc = fmaf(wv, xv, acc);
            }
        }
    if (mode == DW_EXACT && isnan(acc)) acc = canonical_nan();
    if (bias) {
        acc = acc + bias[oc];
        if (mode == DW_EXACT && isnan(acc)) acc = canonical_nan();
    }
    return acc;
}

/* Full output y[N][Cin*mult][Ho][Wo]. Returns 0, or -1 when the output would be empty. */
int oracle_depthwise(const float *x, const float *w, const float *bias, float *y,
                     int N, int Cin, int mult, int H, int W, int KH, int KW,
                     int stride, int pad, int dil, int mode)
{
    const long Ho = dw_out_size(H, KH, stride, pad, dil);
    const long Wo = dw_out_size(W, KW, stride, pad, dil);
    const long Cout = (long)Cin * mult;
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (long n = 0; n < N; ++n)
        for (long oc = 0; oc < Cout; ++oc)
            for (long oy = 0; oy < Ho; ++oy)
                for (long ox = 0; ox < Wo; ++ox)
                    y[((n * Cout + oc) * Ho + oy) * Wo + ox] =
                        dw_one(x, w, bias, Cin, mult, H, W, KH, KW, stride, pad, dil, mode,
                               n, oc, oy, ox);
    return 0;
}

/* Selected outputs, given as flat indices into y[N][Cin*mult][Ho][Wo]. */
int oracle_depthwise_points(const float *x, const float *w, const float *bias,
                            const int64_t *idx, int64_t npts, float *out,
                            int N, int Cin, int mult, int H, int W, int KH, int KW,
                            int stride, int pad, int dil, int mode)
{
    const long Ho = dw_out_size(H, KH, stride, pad, dil);
    const long Wo = dw_out_size(W, KW, stride, pad, dil);
    const long Cout = (long)Cin * mult;
    (void)N;
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t p = 0; p < npts; ++p) {
        long t = idx[p];
        long ox = t % Wo; t /= Wo;
        long oy = t % Ho; t /= Ho;
        long oc = t % Cout; t /= Cout;
        out[p] = dw_one(x, w, bias, Cin, mult, H, W, KH, KW, stride, pad, dil, mode, t, oc, oy, ox);
    }
    return 0;
}

/* Magnitude scale of each output for tolerance checks: sum over taps of |w * x| plus |bias|,
 * in float64, same indexing as dw_one. */
int oracle_depthwise_absbound(const float *x, const float *w, const float *bias, double *out,
                              int N, int Cin, int mult, int H, int W, int KH, int KW,
                              int stride, int pad, int dil)
{
    const long Ho = dw_out_size(H, KH, stride, pad, dil);
    const long Wo = dw_out_size(W, KW, stride, pad, dil);
    const long Cout = (long)Cin * mult;
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (long n = 0; n < N; ++n)
        for (long oc = 0; oc < Cout; ++oc) {
            const float *plane = x + ((n * Cin) + oc / mult) * (long)H * W;
            const float *wp = w + oc * (long)KH * KW;
            for (long oy = 0; oy < Ho; ++oy)
                for (long ox = 0; ox < Wo; ++ox) {
                    double s = bias ? fabs((double)bias[oc]) : 0.0;
                    for (int ky = 0; ky < KH; ++ky)
                        for (int kx = 0; kx < KW; ++kx) {
                            long r = oy * stride + (long)ky * dil - pad;
                            long q = ox * stride + (long)kx * dil - pad;
                            double xv = (r >= 0 && r < H && q >= 0 && q < W) ? plane[r * W + q] : 0.0;
                            s += fabs((double)wp[ky * KW + kx] * xv);
                        }
                    out[((n * Cout + oc) * Ho + oy) * Wo + ox] = s;
                }
        }
    return 0;
}

/* Threads the OpenMP runtime will use (for reporting the CPU baseline's core count). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
int oracle_num_threads(void) { return 1; }
#endif

/* ---------------------------------------------------------------------------------- */
/* Depthwise followed by pointwise (one block)                                         */
/* ---------------------------------------------------------------------------------- */
/*
 * "Convolution Is Wx+b Moving Across a Signal", section "Why variants matter": a depthwise
 * K x K pass followed by a pointwise 1 x 1 channel-mixing pass. Stage 1 is the depthwise
 * output above (OneModel page, multiplier 1, float32 in the page's order, exact or fast mode,
 * with its own bias). Stage 2 feeds it to the tensor cores, so the intermediate is rounded
 * to bfloat16 (nearest, ties to even; a NaN stays a NaN), and the pointwise sum over the
 * channels, y[n][o][oy][ox] = bias_pw[o] + sum_c bf16(d[n][c][oy][ox]) * F[c][o], is taken in
 * float64 with the same absolute sum as the dense oracle.
 */
static float round_bf16(float v)
{
    uint32_t u;
    memcpy(&u, &v, sizeof u);
    if (isnan(v)) {
        u = (u | 0x00400000u) & 0xFFFF0000u;   /* quiet, upper half kept */
    } else {
        /* nearest, ties to even, on the 16 bits that are dropped */
        uint32_t low = u & 0xFFFFu, keep = u & 0xFFFF0000u;
        if (low > 0x8000u || (low == 0x8000u && (keep & 0x10000u))) keep += 0x10000u;
        u = keep;
    }
    float r;
    memcpy(&r, &u, sizeof r);
    return r;
}

/* All Cout outputs of one output pixel; a[] is scratch of C floats. */
static void dwpw_pixel(const float *x, const float *w, const float *bias_dw, const float *F, const float *bias_pw,
                       int C, int H, int W, int K, int stride, int pad, int dil, int mode, int Cout, long n,
                       long oy, long ox, float *a, double *out, double *abs_out, long out_stride)
{
    for (long c = 0; c < C; ++c)
        a[c] = round_bf16(dw_one(x, w, bias_dw, C, 1, H, W, K, K, stride, pad, dil, mode, n, c, oy, ox));
    for (long o = 0; o < Cout; ++o) {
        double s = 0.0, t = 0.0;
        for (long c = 0; c < C; ++c) {
            double av = a[c], fv = F[c * Cout + o];
            s += av * fv;
            t += fabs(av) * fabs(fv);
        }
        if (bias_pw) {
            s += (double)bias_pw[o];
            t += fabs((double)bias_pw[o]);
        }
        out[o * out_stride] = s;
        if (abs_out) abs_out[o * out_stride] = t;
    }
}

/* Full output y[N][Cout][Ho][Wo] (float64) and its absolute sums. */
int oracle_dwpw(const float *x, const float *w, const float *bias_dw, const float *F, const float *bias_pw, double *y,
                double *abssum, int N, int C, int H, int W, int K, int stride, int pad, int dil, int mode, int Cout)
{
    const long Ho = dw_out_size(H, K, stride, pad, dil), Wo = dw_out_size(W, K, stride, pad, dil);
    if (Ho < 1 || Wo < 1) return -1;
    const long plane = Ho * Wo;
#pragma omp parallel
    {
        float *a = (float *)malloc(sizeof(float) * (size_t)C);
#pragma omp for collapse(2) schedule(dynamic)
        for (long n = 0; n < N; ++n)
            for (long oy = 0; oy < Ho; ++oy)
                for (long ox = 0; ox < Wo; ++ox) {
                    long t = n * Cout * plane + oy * Wo + ox;
                    dwpw_pixel(x, w, bias_dw, F, bias_pw, C, H, W, K, stride, pad, dil, mode, Cout, n, oy, ox, a,
                               &y[t], abssum ? &abssum[t] : NULL, plane);
                }
        free(a);
    }
    return 0;
}

/* Selected outputs, by flat index into [N][Cout][Ho][Wo]. */
int oracle_dwpw_points(const float *x, const float *w, const float *bias_dw, const float *F, const float *bias_pw,
                       const int64_t *idx, int64_t npts, double *y, double *abssum, int C, int H, int W, int K,
                       int stride, int pad, int dil, int mode, int Cout)
{
    const long Ho = dw_out_size(H, K, stride, pad, dil), Wo = dw_out_size(W, K, stride, pad, dil);
    if (Ho < 1 || Wo < 1) return -1;
#pragma omp parallel
    {
        float *a = (float *)malloc(sizeof(float) * (size_t)C);
        double *col = (double *)malloc(sizeof(double) * (size_t)Cout * 2);
#pragma omp for schedule(dynamic, 16)
        for (int64_t p = 0; p < npts; ++p) {
            long t = idx[p];
            long ox = t % Wo; t /= Wo;
            long oy = t % Ho; t /= Ho;
            long o = t % Cout;
            long n = t / Cout;
            dwpw_pixel(x, w, bias_dw, F, bias_pw, C, H, W, K, stride, pad, dil, mode, Cout, n, oy, ox, a, col,
                       col + Cout, 1);
            y[p] = col[o];
            abssum[p] = col[Cout + o];
        }
        free(a);
        free(col);
    }
    return 0;
}
