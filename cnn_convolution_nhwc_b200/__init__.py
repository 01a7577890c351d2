"""Forward 2-D convolution on B200 (sm_100a): thin Python binding of the C ABI.

The functions here only marshal arguments -- shape and dtype checks, output allocation
through PyTorch, the current CUDA stream -- and call the C entry points of
libconv_b200.so with the same names (declared in include/conv_b200.h). Every step of the
computation runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
importing this package fails if the library cannot be loaded.

    conv2d_nhwc_fwd(X, F)        dense NHWC conv, bf16 [N,H,W,Cin] x [K,K,Cin,Cout] -> bf16
    conv2d_nhwc_fwd_f32(X, F)    the same with float32 tensors
    conv2d_nhwc_fwd_ex(X, F, b)  bf16 with stride, zero padding, dilation and a float32 bias
    depthwise_fwd(x, w, bias)    depthwise conv, float32 NCHW, exact or fast mode
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

CONV_OK = 0
CONV_ERR_INVALID_ARG = -1
CONV_ERR_UNSUPPORTED = -2
CONV_ERR_MISALIGNED = -3
CONV_ERR_CUDA = -4
CONV_ERR_DEVICE_TIMEOUT = -5
CONV_ERR_DEVICE_BOUNDS = -6
DW_EXACT = 0
DW_FAST = 1

# CONV_B200_DEBUG_BOUNDS=1 at import loads the bounds-checked build of the same library (every
# computed global access checked; a failure sets CONV_ERR_DEVICE_BOUNDS and skips the access)
DEBUG_BOUNDS = os.environ.get("CONV_B200_DEBUG_BOUNDS", "0") == "1"
LIB_PATH = _build.build(debug_bounds=DEBUG_BOUNDS)
lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
lib.conv2d_nhwc_fwd.argtypes = [_P, _P, _P] + [_I] * 6 + [_P]
lib.conv2d_nhwc_fwd.restype = _I
lib.conv2d_nhwc_fwd_f32.argtypes = [_P, _P, _P] + [_I] * 6 + [_P]
lib.conv2d_nhwc_fwd_f32.restype = _I
lib.conv2d_nhwc_fwd_ex.argtypes = [_P, _P, _P, _P] + [_I] * 9 + [_P]
lib.conv2d_nhwc_fwd_ex.restype = _I
lib.conv2d_nhwc_fwd_grouped.argtypes = [_P, _P, _P, _P] + [_I] * 14 + [_P]
lib.conv2d_nhwc_fwd_grouped.restype = _I
lib.conv2d_nhwc_fwd_grouped_pads.argtypes = [_P, _P, _P, _P] + [_I] * 16 + [_P]
lib.conv2d_nhwc_fwd_grouped_pads.restype = _I
lib.conv2d_nhwc_im2col_workspace.argtypes = [_I] * 5
lib.conv2d_nhwc_im2col_workspace.restype = ctypes.c_size_t
lib.conv2d_nhwc_fwd_im2col.argtypes = [_P, _P, _P, _P, ctypes.c_size_t] + [_I] * 6 + [_P]
lib.conv2d_nhwc_fwd_im2col.restype = _I
lib.conv2d_nhwc_fwd_im2col_noalloc.argtypes = [_P, _P, _P] + [_I] * 6 + [_P]
lib.conv2d_nhwc_fwd_im2col_noalloc.restype = _I
lib.dwpw_fwd.argtypes = [_P] * 6 + [_I] * 10 + [_P]
lib.dwpw_fwd.restype = _I
lib.depthwise_fwd.argtypes = [_P, _P, _P, _P] + [_I] * 11 + [_P]
lib.depthwise_fwd.restype = _I
lib.conv_status_string.argtypes = [_I]
lib.conv_status_string.restype = ctypes.c_char_p
lib.conv_device_status.argtypes = [_P, _I]
lib.conv_device_status.restype = _I
lib.conv_last_kernel.argtypes = []
lib.conv_last_kernel.restype = ctypes.c_char_p
lib.conv_selftest_wait_timeout.argtypes = [_P]
lib.conv_selftest_wait_timeout.restype = _I
lib.conv_debug_bounds_build.argtypes = []
lib.conv_debug_bounds_build.restype = _I
lib.conv_debug_bounds_info.argtypes = [ctypes.POINTER(ctypes.c_longlong), _I]
lib.conv_debug_bounds_info.restype = _I
lib.conv_selftest_bounds.argtypes = [_P]
lib.conv_selftest_bounds.restype = _I

EXPORTS = ("conv2d_nhwc_fwd", "conv2d_nhwc_fwd_f32", "conv2d_nhwc_fwd_ex", "conv2d_nhwc_fwd_grouped",
           "conv2d_nhwc_fwd_grouped_pads",
           "conv2d_nhwc_im2col_workspace", "conv2d_nhwc_fwd_im2col", "conv2d_nhwc_fwd_im2col_noalloc", "dwpw_fwd",
           "depthwise_fwd", "conv_status_string", "conv_device_status", "conv_last_kernel",
           "conv_selftest_wait_timeout", "conv_debug_bounds_build", "conv_debug_bounds_info",
           "conv_selftest_bounds")
CONV_IM2COL_STATIC_BYTES = 32 * 1024 * 1024   # the scratch of conv2d_nhwc_fwd_im2col_noalloc


class ConvError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {conv_status_string(code)} ({code})")
        self.code = code


def conv_status_string(code: int) -> str:
    return lib.conv_status_string(int(code)).decode()


def _check(code: int, what: str) -> None:
    if code != CONV_OK:
        raise ConvError(code, what)


def _stream(stream, device):
    """The stream handle for a call on `device` (its current stream when None)."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream) and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _device(*tensors):
    """The one CUDA device every given tensor (None skipped) lives on."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"all tensors must be on one CUDA device, got {sorted(map(str, devs))}")
    return devs.pop()


def _call(fn, what, tensors, stream, *args):
    """Runs one C entry point with the tensors' device current (the library launches on the
    current device) and its stream as the last argument."""
    import torch
    dev = _device(*tensors)
    with torch.cuda.device(dev):
        _check(fn(*args, _stream(stream, dev)), what)


def _tensor(t, dtype, ndim, name):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (the C ABI takes dense row-major tensors); "
                         "call .contiguous() first")
    return ctypes.c_void_p(t.data_ptr())


def _dense(X, F, Y, stream, dtype, fn, what):
    import torch
    px = _tensor(X, dtype, 4, "X")
    pf = _tensor(F, dtype, 4, "F")
    N, H, W, Cin = X.shape
    K, K2, Cin2, Cout = F.shape
    if K != K2 or Cin2 != Cin:
        raise ValueError("F must be [K, K, Cin, Cout] matching X")
    if K > min(H, W):
        raise ValueError("K must not exceed min(H, W)")
    if Y is None:
        Y = torch.empty((N, H - K + 1, W - K + 1, Cout), dtype=dtype, device=X.device)
    elif tuple(Y.shape) != (N, H - K + 1, W - K + 1, Cout):
        raise ValueError("Y has the wrong shape")
    py = _tensor(Y, dtype, 4, "Y")
    _call(fn, what, (X, F, Y), stream, px, pf, py, N, H, W, Cin, Cout, K)
    return Y


def conv2d_nhwc_fwd(X, F, Y=None, stream=None):
    """Dense NHWC convolution, bfloat16: X [N,H,W,Cin], F [K,K,Cin,Cout] -> Y [N,Ho,Wo,Cout]."""
    import torch
    return _dense(X, F, Y, stream, torch.bfloat16, lib.conv2d_nhwc_fwd, "conv2d_nhwc_fwd")


def conv2d_nhwc_fwd_f32(X, F, Y=None, stream=None):
    """Dense NHWC convolution, float32 tensors."""
    import torch
    return _dense(X, F, Y, stream, torch.float32, lib.conv2d_nhwc_fwd_f32, "conv2d_nhwc_fwd_f32")


def conv2d_nhwc_fwd_ex(X, F, bias=None, Y=None, stride=1, pad=0, dil=1, stream=None):
    """Dense NHWC convolution, bfloat16, with stride, zero padding, dilation and an optional
    float32 bias [Cout]: X [N,H,W,Cin], F [K,K,Cin,Cout] -> Y [N,Ho,Wo,Cout]."""
    import torch
    px = _tensor(X, torch.bfloat16, 4, "X")
    pf = _tensor(F, torch.bfloat16, 4, "F")
    N, H, W, Cin = X.shape
    K, K2, Cin2, Cout = F.shape
    if K != K2 or Cin2 != Cin:
        raise ValueError("F must be [K, K, Cin, Cout] matching X")
    pb = ctypes.c_void_p(None)
    if bias is not None:
        pb = _tensor(bias, torch.float32, 1, "bias")
        if bias.shape[0] != Cout:
            raise ValueError("bias must have Cout entries")
    Ho = (H + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    Wo = (W + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    if Y is None:
        Y = torch.empty((N, Ho, Wo, Cout), dtype=torch.bfloat16, device=X.device)
    elif tuple(Y.shape) != (N, Ho, Wo, Cout):
        raise ValueError("Y has the wrong shape")
    py = _tensor(Y, torch.bfloat16, 4, "Y")
    _call(lib.conv2d_nhwc_fwd_ex, "conv2d_nhwc_fwd_ex", (X, F, bias, Y), stream,
          px, pf, pb, py, N, H, W, Cin, Cout, K, stride, pad, dil)
    return Y


def _pair(v, name):
    if isinstance(v, (tuple, list)):
        if len(v) != 2:
            raise ValueError(f"{name} must be an int or a pair")
        return int(v[0]), int(v[1])
    return int(v), int(v)


def _pads(pad):
    """(top, bottom, left, right) from one int, an (h, w) pair, or ((top, bottom), (left, right))."""
    if isinstance(pad, (tuple, list)):
        if len(pad) != 2:
            raise ValueError("pad must be an int, an (h, w) pair or ((top, bottom), (left, right))")
        out = []
        for v in pad:
            if isinstance(v, (tuple, list)):
                if len(v) != 2:
                    raise ValueError("a per-axis pad must be an int or a (before, after) pair")
                out += [int(v[0]), int(v[1])]
            else:
                out += [int(v), int(v)]
        return tuple(out)
    return (int(pad),) * 4


def conv2d_nhwc_fwd_grouped(X, F, bias=None, Y=None, stride=1, pad=0, dil=1, groups=1, stream=None):
    """Grouped dense NHWC convolution, bfloat16, with a KH x KW filter, per-axis stride and
    dilation (ints or (h, w) pairs), zero padding (an int, an (h, w) pair, or ((top, bottom),
    (left, right)) for different padding before and after an axis -- a causal Conv1D is
    pad=(0, (KW-1, 0))) and an optional float32 bias [Cout]:
    X [N,H,W,Cin], F [KH,KW,Cin/groups,Cout] -> Y [N,Ho,Wo,Cout]. A Conv1D is H = KH = 1."""
    import torch
    px = _tensor(X, torch.bfloat16, 4, "X")
    pf = _tensor(F, torch.bfloat16, 4, "F")
    N, H, W, Cin = X.shape
    KH, KW, Cg, Cout = F.shape
    groups = int(groups)
    if groups < 1 or Cin % groups or Cout % groups or Cg != Cin // groups:
        raise ValueError("F must be [KH, KW, Cin/groups, Cout] with groups dividing Cin and Cout")
    (sh, sw), (dh, dw) = _pair(stride, "stride"), _pair(dil, "dil")
    pt, pb, pl, pr = _pads(pad)
    pbias = ctypes.c_void_p(None)
    if bias is not None:
        pbias = _tensor(bias, torch.float32, 1, "bias")
        if bias.shape[0] != Cout:
            raise ValueError("bias must have Cout entries")
    Ho = (H + pt + pb - (dh * (KH - 1) + 1)) // sh + 1
    Wo = (W + pl + pr - (dw * (KW - 1) + 1)) // sw + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    if Y is None:
        Y = torch.empty((N, Ho, Wo, Cout), dtype=torch.bfloat16, device=X.device)
    elif tuple(Y.shape) != (N, Ho, Wo, Cout):
        raise ValueError("Y has the wrong shape")
    py = _tensor(Y, torch.bfloat16, 4, "Y")
    if pt == pb and pl == pr:
        _call(lib.conv2d_nhwc_fwd_grouped, "conv2d_nhwc_fwd_grouped", (X, F, bias, Y), stream,
              px, pf, pbias, py, N, H, W, Cin, Cout, KH, KW, sh, sw, pt, pl, dh, dw, groups)
    else:
        _call(lib.conv2d_nhwc_fwd_grouped_pads, "conv2d_nhwc_fwd_grouped_pads", (X, F, bias, Y), stream,
              px, pf, pbias, py, N, H, W, Cin, Cout, KH, KW, sh, sw, pt, pb, pl, pr, dh, dw, groups)
    return Y


def conv2d_nhwc_fwd_im2col(X, F, Y=None, workspace=None, stream=None):
    """Comparison path: explicit patch matrix in `workspace` (allocated here if None, as a uint8
    CUDA tensor of conv2d_nhwc_im2col_workspace bytes), then one cuBLAS GEMM."""
    import torch
    px = _tensor(X, torch.bfloat16, 4, "X")
    pf = _tensor(F, torch.bfloat16, 4, "F")
    N, H, W, Cin = X.shape
    K, K2, Cin2, Cout = F.shape
    if K != K2 or Cin2 != Cin:
        raise ValueError("F must be [K, K, Cin, Cout] matching X")
    need = lib.conv2d_nhwc_im2col_workspace(N, H, W, Cin, K)
    if need == 0:
        raise ValueError("invalid shape")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    if not (workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    if Y is None:
        Y = torch.empty((N, H - K + 1, W - K + 1, Cout), dtype=torch.bfloat16, device=X.device)
    py = _tensor(Y, torch.bfloat16, 4, "Y")
    _call(lib.conv2d_nhwc_fwd_im2col, "conv2d_nhwc_fwd_im2col", (X, F, Y, workspace), stream,
          px, pf, py, ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size(),
          N, H, W, Cin, Cout, K)
    return Y


def conv2d_nhwc_fwd_im2col_noalloc(X, F, Y, stream=None):
    """The explicit-im2col comparison path with its patch matrix in the library's static scratch
    (CONV_IM2COL_STATIC_BYTES per device) instead of a workspace, for callers that cannot
    allocate device memory. Y must be passed: this binding allocates nothing either."""
    import torch
    px = _tensor(X, torch.bfloat16, 4, "X")
    pf = _tensor(F, torch.bfloat16, 4, "F")
    N, H, W, Cin = X.shape
    K, K2, Cin2, Cout = F.shape
    if K != K2 or Cin2 != Cin:
        raise ValueError("F must be [K, K, Cin, Cout] matching X")
    if K > min(H, W):
        raise ValueError("K must not exceed min(H, W)")
    if tuple(Y.shape) != (N, H - K + 1, W - K + 1, Cout):
        raise ValueError("Y has the wrong shape")
    py = _tensor(Y, torch.bfloat16, 4, "Y")
    _call(lib.conv2d_nhwc_fwd_im2col_noalloc, "conv2d_nhwc_fwd_im2col_noalloc", (X, F, Y), stream,
          px, pf, py, N, H, W, Cin, Cout, K)
    return Y


def depthwise_fwd(x, w, bias=None, y=None, stride=1, pad=0, dil=1, mode=DW_EXACT, stream=None):
    """Depthwise convolution, float32: x [N,Cin,H,W], w [Cin*mult,KH,KW], bias [Cin*mult] or None."""
    import torch
    px = _tensor(x, torch.float32, 4, "x")
    pw = _tensor(w, torch.float32, 3, "w")
    N, Cin, H, W = x.shape
    Cout, KH, KW = w.shape
    if Cout % Cin != 0:
        raise ValueError("w must have Cin * mult planes")
    mult = Cout // Cin
    pb = ctypes.c_void_p(None)
    if bias is not None:
        pb = _tensor(bias, torch.float32, 1, "bias")
        if bias.shape[0] != Cout:
            raise ValueError("bias must have Cin * mult entries")
    Ho = (H + 2 * pad - (dil * (KH - 1) + 1)) // stride + 1
    Wo = (W + 2 * pad - (dil * (KW - 1) + 1)) // stride + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    if y is None:
        y = torch.empty((N, Cout, Ho, Wo), dtype=torch.float32, device=x.device)
    elif tuple(y.shape) != (N, Cout, Ho, Wo):
        raise ValueError("y has the wrong shape")
    py = _tensor(y, torch.float32, 4, "y")
    _call(lib.depthwise_fwd, "depthwise_fwd", (x, w, bias, y), stream,
          px, pw, pb, py, N, Cin, mult, H, W, KH, KW, stride, pad, dil, int(mode))
    return y


def dwpw_fwd(x, w_dw, b_dw, F, b_pw=None, y=None, stride=1, pad=0, dil=1, mode=DW_EXACT, stream=None):
    """Depthwise then pointwise, fused: x float32 [N,C,H,W], w_dw float32 [C,K,K], b_dw float32
    [C] or None, F bfloat16 [C,Cout], b_pw float32 [Cout] or None -> y float32 [N,Cout,Ho,Wo]."""
    import torch
    px = _tensor(x, torch.float32, 4, "x")
    pw = _tensor(w_dw, torch.float32, 3, "w_dw")
    pf = _tensor(F, torch.bfloat16, 2, "F")
    N, C, H, W = x.shape
    C2, K, K2 = w_dw.shape
    if C2 != C or K != K2:
        raise ValueError("w_dw must be [C, K, K]")
    C3, Cout = F.shape
    if C3 != C:
        raise ValueError("F must be [C, Cout]")
    pbd = ctypes.c_void_p(None)
    if b_dw is not None:
        pbd = _tensor(b_dw, torch.float32, 1, "b_dw")
        if b_dw.shape[0] != C:
            raise ValueError("b_dw must have C entries")
    pbp = ctypes.c_void_p(None)
    if b_pw is not None:
        pbp = _tensor(b_pw, torch.float32, 1, "b_pw")
        if b_pw.shape[0] != Cout:
            raise ValueError("b_pw must have Cout entries")
    Ho = (H + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    Wo = (W + 2 * pad - (dil * (K - 1) + 1)) // stride + 1
    if Ho < 1 or Wo < 1:
        raise ValueError("empty output")
    if y is None:
        y = torch.empty((N, Cout, Ho, Wo), dtype=torch.float32, device=x.device)
    elif tuple(y.shape) != (N, Cout, Ho, Wo):
        raise ValueError("y has the wrong shape")
    py = _tensor(y, torch.float32, 4, "y")
    _call(lib.dwpw_fwd, "dwpw_fwd", (x, w_dw, b_dw, F, b_pw, y), stream,
          px, pw, pbd, pf, pbp, py, N, C, H, W, K, stride, pad, dil, Cout, int(mode))
    return y


def conv_last_kernel() -> str:
    """Kernel family the last successful call on this thread launched (the dispatcher's choice)."""
    return lib.conv_last_kernel().decode()


def _current():
    import torch
    return torch.device("cuda", torch.cuda.current_device())


def conv_selftest_wait_timeout(stream=None) -> int:
    """Runs the bounded-wait diagnostic (about one second) on the current device; returns the
    launch status."""
    return lib.conv_selftest_wait_timeout(_stream(stream, _current()))


def conv_selftest_bounds(stream=None) -> int:
    """Runs the bounds-check diagnostic (a failing check that touches no memory) on the current
    device; returns the launch status."""
    return lib.conv_selftest_bounds(_stream(stream, _current()))


def conv_debug_bounds_build() -> bool:
    """True when the loaded library is the bounds-checked build."""
    return lib.conv_debug_bounds_build() == 1


def conv_debug_bounds_info(reset=False):
    """First failed bounds check on the current device since the last reset, as (site, index,
    limit), or None; always None in the normal build."""
    info = (ctypes.c_longlong * 3)()
    rc = lib.conv_debug_bounds_info(info, 1 if reset else 0)
    if rc != CONV_OK:
        raise ConvError(rc, "conv_debug_bounds_info")
    return None if info[0] < 0 else (info[0], info[1], info[2])


def conv_device_status(stream=None, reset=False) -> int:
    """Synchronises the stream and returns the current device's status word as a conv_status
    code."""
    return lib.conv_device_status(_stream(stream, _current()), 1 if reset else 0)
