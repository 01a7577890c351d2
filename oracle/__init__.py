"""CPU oracle for the forward convolutions (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The library's CUDA path never imports it, and the two share no code;
both only consume the seeded inputs of the ``workloads`` module.

The arithmetic lives in ``conv_oracle.c`` (plain C, OpenMP over independent outputs):

* ``conv2d_nhwc`` -- the seven-loop definition of the dense NHWC convolution of the CMU
  DLSys Lecture 14 notes ("The hidden copy behind convolution as matrix multiplication",
  section 1), accumulated in float64, with the per-output absolute sum sum|x||f| that the
  dense tolerance is scaled by.
* ``conv2d_nhwc_ex`` -- the same sum with the stride, zero-padding, dilation and bias variants
  of "Convolution Is Wx+b Moving Across a Signal" (output-size rule of section "Build an
  image-gradient map, one number at a time"), float64.
* ``conv2d_grouped`` -- the same sum split into channel groups, with per-axis geometry and a
  KH x KW kernel (Conv1D is H = KH = 1), after the grouped Conv1D of the Wx+b page's CKE
  section, float64.
* ``depthwise`` -- the per-output loop of the OneModel "Depthwise convolution" page
  (section "What each output is"), in IEEE float32 in the page's order, exact or fast mode.
* ``dwpw`` -- a depthwise pass followed by a pointwise 1 x 1 pass (Wx+b page, section "Why
  variants matter"): the depthwise output above, rounded to bfloat16 (nearest even), then the
  channel-mixing sum with a bias in float64.

Parity status: every function here is pinned by tests that do not call it to compute
their expectation (worked examples printed on the pages, library routines for special
cases, closed forms and invariants); see tests/test_oracle.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "conv_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")

DW_EXACT = 0
DW_FAST = 1

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fno-unsafe-math-optimizations", "-frounding-math", "-fsignaling-nans"]


def build(force: bool = False) -> str:
    """Compile conv_oracle.c into _liboracle.so with gcc (no CUDA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_int64
        lib.oracle_conv2d_nhwc.argtypes = [P, P, P, P] + [I] * 6
        lib.oracle_conv2d_nhwc.restype = None
        lib.oracle_conv2d_nhwc_points.argtypes = [P, P, P, L, P, P] + [I] * 6
        lib.oracle_conv2d_nhwc_points.restype = None
        lib.oracle_conv2d_nhwc_ex.argtypes = [P, P, P, P, P] + [I] * 9
        lib.oracle_conv2d_nhwc_ex.restype = I
        lib.oracle_conv2d_nhwc_ex_points.argtypes = [P, P, P, P, L, P, P] + [I] * 9
        lib.oracle_conv2d_nhwc_ex_points.restype = I
        lib.oracle_conv2d_grouped.argtypes = [P, P, P, P, P] + [I] * 14
        lib.oracle_conv2d_grouped.restype = I
        lib.oracle_conv2d_grouped_points.argtypes = [P, P, P, P, L, P, P] + [I] * 13
        lib.oracle_conv2d_grouped_points.restype = I
        lib.oracle_conv2d_grouped_pads.argtypes = [P, P, P, P, P] + [I] * 16
        lib.oracle_conv2d_grouped_pads.restype = I
        lib.oracle_conv2d_grouped_pads_points.argtypes = [P, P, P, P, L, P, P] + [I] * 15
        lib.oracle_conv2d_grouped_pads_points.restype = I
        lib.oracle_dwpw.argtypes = [P] * 7 + [I] * 10
        lib.oracle_dwpw.restype = I
        lib.oracle_dwpw_points.argtypes = [P] * 6 + [L, P, P] + [I] * 9
        lib.oracle_dwpw_points.restype = I
        lib.oracle_depthwise.argtypes = [P, P, P, P] + [I] * 11
        lib.oracle_depthwise.restype = I
        lib.oracle_depthwise_points.argtypes = [P, P, P, P, L, P] + [I] * 11
        lib.oracle_depthwise_points.restype = I
        lib.oracle_depthwise_absbound.argtypes = [P, P, P, P] + [I] * 10
        lib.oracle_depthwise_absbound.restype = I
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def num_threads() -> int:
    return _load().oracle_num_threads()


def conv2d_nhwc(X, F):
    """Dense NHWC forward convolution in float64.

    X: [N, H, W, Cin], F: [K, K, Cin, Cout] (float32 values; bfloat16 data is widened by the
    caller). Returns (Y, abssum), both float64 [N, Ho, Wo, Cout].
    """
    X, F = _f32(X), _f32(F)
    N, H, W, Cin = X.shape
    K, K2, Cin2, Cout = F.shape
    if K != K2 or Cin != Cin2 or K > min(H, W) or min(N, H, W, Cin, K, Cout) <= 0:
        raise ValueError("incompatible input and square filter")
    Ho, Wo = H - K + 1, W - K + 1
    Y = np.empty((N, Ho, Wo, Cout), dtype=np.float64)
    A = np.empty_like(Y)
    _load().oracle_conv2d_nhwc(_ptr(X), _ptr(F), _ptr(Y), _ptr(A), N, H, W, Cin, Cout, K)
    return Y, A


def conv2d_nhwc_points(X, F, flat_idx):
    """Selected outputs of conv2d_nhwc, by flat index into [N, Ho, Wo, Cout]."""
    X, F = _f32(X), _f32(F)
    N, H, W, Cin = X.shape
    K, _, _, Cout = F.shape
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    y = np.empty(idx.size, dtype=np.float64)
    a = np.empty(idx.size, dtype=np.float64)
    _load().oracle_conv2d_nhwc_points(_ptr(X), _ptr(F), _ptr(idx), idx.size, _ptr(y), _ptr(a),
                                      N, H, W, Cin, Cout, K)
    return y, a


def _dense_ex_shape(X, F, bias, stride, pad, dil):
    N, H, W, Cin = X.shape
    K, K2, Cin2, Cout = F.shape
    if K != K2 or Cin != Cin2 or min(N, H, W, Cin, K, Cout, stride, dil) <= 0 or pad < 0:
        raise ValueError("incompatible input and square filter")
    if bias is not None and bias.shape != (Cout,):
        raise ValueError("bias must have Cout entries")
    Ho = (H + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    Wo = (W + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    return N, H, W, Cin, Cout, K, Ho, Wo


def conv2d_nhwc_ex(X, F, bias=None, stride=1, pad=0, dil=1):
    """Dense NHWC forward convolution with stride, symmetric zero padding, dilation and a
    per-output-channel bias, in float64 (the variants of "Convolution Is Wx+b Moving Across a
    Signal": output size per axis floor((in + 2*pad - (dil*(K-1)+1)) / stride) + 1, window of
    output (y, x) starting at (y*stride - pad, x*stride - pad), tap (i, j) dil*i rows and dil*j
    columns on, zeros outside the image, bias added to the sum).

    Returns (Y, abssum), float64 [N, Ho, Wo, Cout]; abssum = sum|x||f| + |b|.
    """
    X, F = _f32(X), _f32(F)
    b = None if bias is None else _f32(bias)
    N, H, W, Cin, Cout, K, Ho, Wo = _dense_ex_shape(X, F, b, stride, pad, dil)
    Y = np.empty((N, Ho, Wo, Cout), dtype=np.float64)
    A = np.empty_like(Y)
    _load().oracle_conv2d_nhwc_ex(_ptr(X), _ptr(F), _ptr(b), _ptr(Y), _ptr(A), N, H, W, Cin, Cout, K,
                                  stride, pad, dil)
    return Y, A


def conv2d_nhwc_ex_points(X, F, flat_idx, bias=None, stride=1, pad=0, dil=1):
    """Selected outputs of conv2d_nhwc_ex, by flat index into [N, Ho, Wo, Cout]."""
    X, F = _f32(X), _f32(F)
    b = None if bias is None else _f32(bias)
    N, H, W, Cin, Cout, K, Ho, Wo = _dense_ex_shape(X, F, b, stride, pad, dil)
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    y = np.empty(idx.size, dtype=np.float64)
    a = np.empty(idx.size, dtype=np.float64)
    _load().oracle_conv2d_nhwc_ex_points(_ptr(X), _ptr(F), _ptr(b), _ptr(idx), idx.size, _ptr(y), _ptr(a),
                                         N, H, W, Cin, Cout, K, stride, pad, dil)
    return y, a


def _pair(v):
    return (v, v) if isinstance(v, int) else (int(v[0]), int(v[1]))


def _pads(pad):
    """(top, bottom, left, right) from one int, an (h, w) pair, or ((top, bottom), (left, right))."""
    if isinstance(pad, int):
        return pad, pad, pad, pad
    ph, pw = pad
    (pt, pb) = (ph, ph) if isinstance(ph, int) else (int(ph[0]), int(ph[1]))
    (pl, pr) = (pw, pw) if isinstance(pw, int) else (int(pw[0]), int(pw[1]))
    return int(pt), int(pb), int(pl), int(pr)


def _grouped_shape(X, F, bias, stride, pad, dil, groups):
    N, H, W, Cin = X.shape
    KH, KW, Cg, Cout = F.shape
    (sh, sw), (dh, dw) = _pair(stride), _pair(dil)
    pt, pb, pl, pr = _pads(pad)
    if groups < 1 or Cin % groups or Cout % groups or Cg * groups != Cin:
        raise ValueError("channels must split into the groups")
    if bias is not None and bias.shape != (Cout,):
        raise ValueError("bias must have Cout entries")
    Ho = (H + pt + pb - (dh * (KH - 1) + 1)) // sh + 1
    Wo = (W + pl + pr - (dw * (KW - 1) + 1)) // sw + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    return (N, H, W, Cin, KH, KW, Cout), (sh, sw, pt, pb, pl, pr, dh, dw), (Ho, Wo)


def conv2d_grouped(X, F, bias=None, stride=1, pad=0, dil=1, groups=1):
    """Grouped NHWC convolution with per-axis stride / padding / dilation and a KH x KW kernel,
    float64. stride, dil: (h, w) pairs or one int for both; pad: one int, an (h, w) pair, or
    ((top, bottom), (left, right)) for different padding before and after an axis (a causal
    Conv1D pads only the left). X: [N, H, W, Cin]; F: [KH, KW, Cin/groups, Cout] (output channel
    o uses input channels of group o // (Cout/groups)); bias: [Cout] or None. Conv1D is H = KH = 1.
    Returns (Y, abssum), float64 [N, Ho, Wo, Cout]."""
    X, F = _f32(X), _f32(F)
    b = None if bias is None else _f32(bias)
    (N, H, W, Cin, KH, KW, Cout), (sh, sw, pt, pb, pl, pr, dh, dw), (Ho, Wo) = \
        _grouped_shape(X, F, b, stride, pad, dil, groups)
    Y = np.empty((N, Ho, Wo, Cout), dtype=np.float64)
    A = np.empty_like(Y)
    if pt == pb and pl == pr:
        rc = _load().oracle_conv2d_grouped(_ptr(X), _ptr(F), _ptr(b), _ptr(Y), _ptr(A), N, H, W, Cin, Cout, KH, KW,
                                           sh, sw, pt, pl, dh, dw, groups)
    else:
        rc = _load().oracle_conv2d_grouped_pads(_ptr(X), _ptr(F), _ptr(b), _ptr(Y), _ptr(A), N, H, W, Cin, Cout, KH,
                                                KW, sh, sw, pt, pb, pl, pr, dh, dw, groups)
    if rc != 0:
        raise ValueError("bad shape")
    return Y, A


def conv2d_grouped_points(X, F, flat_idx, bias=None, stride=1, pad=0, dil=1, groups=1):
    """Selected outputs of conv2d_grouped, by flat index into [N, Ho, Wo, Cout]."""
    X, F = _f32(X), _f32(F)
    b = None if bias is None else _f32(bias)
    (N, H, W, Cin, KH, KW, Cout), (sh, sw, pt, pb, pl, pr, dh, dw), (Ho, Wo) = \
        _grouped_shape(X, F, b, stride, pad, dil, groups)
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    if idx.size and (idx.min() < 0 or idx.max() >= N * Ho * Wo * Cout):
        raise ValueError("bad index")
    y = np.empty(idx.size, dtype=np.float64)
    a = np.empty(idx.size, dtype=np.float64)
    if pt == pb and pl == pr:
        _load().oracle_conv2d_grouped_points(_ptr(X), _ptr(F), _ptr(b), _ptr(idx), idx.size, _ptr(y), _ptr(a), H, W,
                                             Cin, Cout, KH, KW, sh, sw, pt, pl, dh, dw, groups)
    else:
        _load().oracle_conv2d_grouped_pads_points(_ptr(X), _ptr(F), _ptr(b), _ptr(idx), idx.size, _ptr(y), _ptr(a),
                                                  H, W, Cin, Cout, KH, KW, sh, sw, pt, pb, pl, pr, dh, dw, groups)
    return y, a


def _dw_shape(x, w, mult, stride, pad, dil):
    N, Cin, H, W = x.shape
    Cout, KH, KW = w.shape
    if Cout != Cin * mult:
        raise ValueError("w must have Cin*mult planes")
    Ho = (H + 2 * pad - (dil * (KH - 1) + 1)) // stride + 1
    Wo = (W + 2 * pad - (dil * (KW - 1) + 1)) // stride + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    return N, Cin, H, W, Cout, KH, KW, Ho, Wo


def depthwise(x, w, bias, mult=1, stride=1, pad=0, dil=1, mode=DW_EXACT):
    """Depthwise forward convolution in float32, the page's order.

    x: [N, Cin, H, W]; w: [Cin*mult, KH, KW]; bias: [Cin*mult] or None.
    Returns y: float32 [N, Cin*mult, Ho, Wo].
    """
    x, w = _f32(x), _f32(w)
    b = None if bias is None else _f32(bias)
    N, Cin, H, W, Cout, KH, KW, Ho, Wo = _dw_shape(x, w, mult, stride, pad, dil)
    y = np.empty((N, Cout, Ho, Wo), dtype=np.float32)
    rc = _load().oracle_depthwise(_ptr(x), _ptr(w), _ptr(b), _ptr(y), N, Cin, mult, H, W, KH, KW,
                                  stride, pad, dil, mode)
    if rc != 0:
        raise ValueError("empty output")
    return y


def depthwise_points(x, w, bias, flat_idx, mult=1, stride=1, pad=0, dil=1, mode=DW_EXACT):
    """Selected outputs of depthwise, by flat index into [N, Cin*mult, Ho, Wo]."""
    x, w = _f32(x), _f32(w)
    b = None if bias is None else _f32(bias)
    N, Cin, H, W, Cout, KH, KW, Ho, Wo = _dw_shape(x, w, mult, stride, pad, dil)
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np.float32)
    _load().oracle_depthwise_points(_ptr(x), _ptr(w), _ptr(b), _ptr(idx), idx.size, _ptr(out),
                                    N, Cin, mult, H, W, KH, KW, stride, pad, dil, mode)
    return out


def depthwise_absbound(x, w, bias, mult=1, stride=1, pad=0, dil=1):
    """sum over taps of |w*x| plus |bias| per output, float64 [N, Cin*mult, Ho, Wo]."""
    x, w = _f32(x), _f32(w)
    b = None if bias is None else _f32(bias)
    N, Cin, H, W, Cout, KH, KW, Ho, Wo = _dw_shape(x, w, mult, stride, pad, dil)
    out = np.empty((N, Cout, Ho, Wo), dtype=np.float64)
    _load().oracle_depthwise_absbound(_ptr(x), _ptr(w), _ptr(b), _ptr(out), N, Cin, mult, H, W, KH,
                                      KW, stride, pad, dil)
    return out


def _dwpw_shape(x, w, F, b_dw, b_pw, stride, pad, dil):
    N, C, H, W = x.shape
    if w.ndim != 3 or w.shape[0] != C or w.shape[1] != w.shape[2]:
        raise ValueError("w must be [C, K, K]")
    K = w.shape[1]
    if F.ndim != 2 or F.shape[0] != C:
        raise ValueError("F must be [C, Cout]")
    Cout = F.shape[1]
    if b_dw is not None and b_dw.shape != (C,):
        raise ValueError("depthwise bias must have C entries")
    if b_pw is not None and b_pw.shape != (Cout,):
        raise ValueError("pointwise bias must have Cout entries")
    Ho = (H + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    Wo = (W + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    return N, C, H, W, K, Cout, Ho, Wo


def dwpw(x, w, b_dw, F, b_pw, stride=1, pad=0, dil=1, mode=DW_EXACT):
    """Depthwise (x [N,C,H,W] float32, w [C,K,K], b_dw [C] or None; the page's order and
    mode) then pointwise (F [C,Cout], the float32 values of bf16 weights; b_pw [Cout] or
    None) over the bfloat16-rounded intermediate. Returns (y, abssum), float64
    [N, Cout, Ho, Wo]."""
    x, w, F = _f32(x), _f32(w), _f32(F)
    bd = None if b_dw is None else _f32(b_dw)
    bp = None if b_pw is None else _f32(b_pw)
    N, C, H, W, K, Cout, Ho, Wo = _dwpw_shape(x, w, F, bd, bp, stride, pad, dil)
    y = np.empty((N, Cout, Ho, Wo), dtype=np.float64)
    a = np.empty_like(y)
    if _load().oracle_dwpw(_ptr(x), _ptr(w), _ptr(bd), _ptr(F), _ptr(bp), _ptr(y), _ptr(a), N, C, H, W, K, stride,
                           pad, dil, mode, Cout) != 0:
        raise ValueError("bad shape")
    return y, a


def dwpw_points(x, w, b_dw, F, b_pw, flat_idx, stride=1, pad=0, dil=1, mode=DW_EXACT):
    """Selected outputs of dwpw, by flat index into [N, Cout, Ho, Wo]."""
    x, w, F = _f32(x), _f32(w), _f32(F)
    bd = None if b_dw is None else _f32(b_dw)
    bp = None if b_pw is None else _f32(b_pw)
    N, C, H, W, K, Cout, Ho, Wo = _dwpw_shape(x, w, F, bd, bp, stride, pad, dil)
    idx = np.ascontiguousarray(flat_idx, dtype=np.int64)
    if idx.size and (idx.min() < 0 or idx.max() >= N * Cout * Ho * Wo):
        raise ValueError("index out of range")
    y = np.empty(idx.size, dtype=np.float64)
    a = np.empty(idx.size, dtype=np.float64)
    _load().oracle_dwpw_points(_ptr(x), _ptr(w), _ptr(bd), _ptr(F), _ptr(bp), _ptr(idx), idx.size, _ptr(y), _ptr(a),
                               C, H, W, K, stride, pad, dil, mode, Cout)
    return y, a
