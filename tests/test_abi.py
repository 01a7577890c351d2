"""The C ABI without a GPU: the library loads, exports every symbol the header declares, and
rejects bad arguments with the documented status codes before it makes any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import cnn_convolution_nhwc_b200 as cb
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "conv_b200.h")
V = ctypes.c_void_p


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", src, flags=re.M))


def test_header_declares_the_entry_points():
    assert _declared() == set(cb.EXPORTS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", cb.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in syms, name
        assert getattr(cb.lib, name) is not None


def test_bounds_checked_build_exports_the_same_symbols():
    # the -DCONV_DEBUG_BOUNDS variant of the same sources: every declared entry point, and a
    # build flag that says which variant is loaded (no device access)
    from cnn_convolution_nhwc_b200 import build as b
    path = b.build(debug_bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in syms, name
    dbg = ctypes.CDLL(path)
    assert dbg.conv_debug_bounds_build() == 1
    assert cb.lib.conv_debug_bounds_build() == (1 if cb.DEBUG_BOUNDS else 0)


def test_bounds_info_rejects_null():
    assert cb.lib.conv_debug_bounds_info(None, 0) == cb.CONV_ERR_INVALID_ARG


def test_status_strings():
    for code in (cb.CONV_OK, cb.CONV_ERR_INVALID_ARG, cb.CONV_ERR_UNSUPPORTED, cb.CONV_ERR_MISALIGNED,
                 cb.CONV_ERR_CUDA, cb.CONV_ERR_DEVICE_TIMEOUT, cb.CONV_ERR_DEVICE_BOUNDS):
        s = cb.conv_status_string(code)
        assert s and s != "unknown status"
    assert cb.conv_status_string(12345) == "unknown status"


# Fake device addresses: validation only looks at their values, never dereferences them.
X, F, Y = V(1 << 20), V(1 << 24), V(1 << 28)


@pytest.mark.parametrize("args,code", [
    ((None, F, Y, 1, 5, 5, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),
    ((X, None, Y, 1, 5, 5, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),
    ((X, F, None, 1, 5, 5, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),
    ((X, F, Y, 0, 5, 5, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),
    ((X, F, Y, 1, 5, 5, 0, 8, 3), cb.CONV_ERR_INVALID_ARG),
    ((X, F, Y, 1, 5, 5, 8, -2, 3), cb.CONV_ERR_INVALID_ARG),
    ((X, F, Y, 1, 5, 5, 8, 8, 0), cb.CONV_ERR_INVALID_ARG),
    ((X, F, Y, 1, 5, 2, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),        # K > W
    ((X, F, Y, 1, 2, 5, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),        # K > H
    ((V((1 << 20) + 1), F, Y, 1, 5, 5, 8, 8, 3), cb.CONV_ERR_MISALIGNED),
    ((X, F, V(1 << 20), 1, 5, 5, 8, 8, 3), cb.CONV_ERR_INVALID_ARG),  # Y aliases X
    ((X, F, Y, 4096, 4096, 4096, 64, 8, 3), cb.CONV_ERR_UNSUPPORTED),
])
def test_dense_rejects(args, code):
    assert cb.lib.conv2d_nhwc_fwd(*args, None) == code
    if code != cb.CONV_ERR_MISALIGNED:
        assert cb.lib.conv2d_nhwc_fwd_f32(*args, None) == code


def test_dense_f32_needs_4_byte_alignment():
    assert cb.lib.conv2d_nhwc_fwd_f32(V((1 << 20) + 2), F, Y, 1, 5, 5, 8, 8, 3, None) == cb.CONV_ERR_MISALIGNED


B = V(1 << 30)


@pytest.mark.parametrize("args,code", [
    ((None, F, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),
    ((X, None, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, None, 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, Y, 1, 2, 0, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),   # mult 0
    ((X, F, B, Y, 1, 2, 1, 5, 5, 3, 3, 0, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),   # stride 0
    ((X, F, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, -1, 1, 0), cb.CONV_ERR_INVALID_ARG),  # pad < 0
    ((X, F, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, 1, 0, 0), cb.CONV_ERR_INVALID_ARG),   # dil 0
    ((X, F, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 2), cb.CONV_ERR_INVALID_ARG),   # bad mode
    ((X, F, B, Y, 1, 2, 1, 2, 2, 5, 5, 1, 0, 1, 0), cb.CONV_ERR_INVALID_ARG),   # empty output
    ((X, F, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, 0, 3, 0), cb.CONV_ERR_INVALID_ARG),   # dilated kernel too big
    ((V((1 << 20) + 2), F, B, Y, 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_MISALIGNED),
    ((X, F, V((1 << 30) + 1), Y, 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_MISALIGNED),
    ((X, F, B, V((1 << 20) + 64), 1, 2, 1, 5, 5, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),  # y overlaps x
    ((X, F, B, Y, 65536, 65536, 1, 8, 8, 3, 3, 1, 1, 1, 0), cb.CONV_ERR_UNSUPPORTED),
])
def test_depthwise_rejects(args, code):
    assert cb.lib.depthwise_fwd(*args, None) == code


@pytest.mark.parametrize("args,code", [
    # X, F, bias, Y, N, H, W, Cin, Cout, K, stride, pad, dil
    ((None, F, B, Y, 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_INVALID_ARG),
    ((X, None, B, Y, 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, None, 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, Y, 0, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 0, 1, 1), cb.CONV_ERR_INVALID_ARG),      # stride 0
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 2, -1, 1), cb.CONV_ERR_INVALID_ARG),     # pad < 0
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 2, 1, 0), cb.CONV_ERR_INVALID_ARG),      # dil 0
    ((X, F, B, Y, 1, 2, 2, 8, 8, 5, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),      # dilated window > padded image
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 1, 0, 5), cb.CONV_ERR_INVALID_ARG),      # dilation 5: reach 11 > 9
    ((V((1 << 20) + 1), F, B, Y, 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_MISALIGNED),
    ((X, F, V((1 << 30) + 2), Y, 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_MISALIGNED),   # bias not 4-byte aligned
    ((X, F, B, V(1 << 20), 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_INVALID_ARG),       # Y aliases X
    ((X, F, V((1 << 28) + 8), Y, 1, 9, 9, 8, 8, 3, 2, 1, 1), cb.CONV_ERR_INVALID_ARG),  # bias inside Y
    ((X, F, B, Y, 4096, 4096, 4096, 64, 8, 3, 2, 1, 1), cb.CONV_ERR_UNSUPPORTED),
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 1, 2 ** 30, 1), cb.CONV_ERR_UNSUPPORTED),          # padding beyond int range
])
def test_dense_ex_rejects(args, code):
    assert cb.lib.conv2d_nhwc_fwd_ex(*args, None) == code


def test_dense_ex_plain_geometry_validates_like_the_plain_entry():
    # stride 1, pad 0, dil 1, no bias is conv2d_nhwc_fwd: the same argument checks apply
    assert cb.lib.conv2d_nhwc_fwd_ex(X, F, None, Y, 1, 5, 2, 8, 8, 3, 1, 0, 1, None) == cb.CONV_ERR_INVALID_ARG
    assert cb.lib.conv2d_nhwc_fwd_ex(V((1 << 20) + 1), F, None, Y, 1, 5, 5, 8, 8, 3, 1, 0, 1, None) == \
        cb.CONV_ERR_MISALIGNED


@pytest.mark.parametrize("args,code", [
    # X, F, bias, Y, N, H, W, Cin, Cout, KH, KW, sh, sw, ph, pw, dh, dw, groups
    ((None, F, B, Y, 1, 9, 9, 8, 8, 3, 3, 1, 1, 0, 0, 1, 1, 2), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 3, 1, 1, 0, 0, 1, 1, 0), cb.CONV_ERR_INVALID_ARG),     # no groups
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 3, 1, 1, 0, 0, 1, 1, 3), cb.CONV_ERR_INVALID_ARG),     # 3 does not divide 8
    ((X, F, B, Y, 1, 9, 9, 12, 8, 3, 3, 1, 1, 0, 0, 1, 1, 3), cb.CONV_ERR_INVALID_ARG),    # ... nor Cout
    ((X, F, B, Y, 1, 9, 9, 8, 8, 0, 3, 1, 1, 0, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),     # KH 0
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 3, 1, 0, 0, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),     # stride_w 0
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 3, 1, 1, 0, -1, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),    # pad_w < 0
    ((X, F, B, Y, 1, 9, 9, 8, 8, 3, 3, 1, 1, 0, 0, 0, 1, 1), cb.CONV_ERR_INVALID_ARG),     # dil_h 0
    ((X, F, B, Y, 1, 1, 9, 8, 8, 3, 1, 1, 1, 0, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),     # KH 3 on one row
    ((X, F, B, Y, 1, 9, 4, 8, 8, 1, 3, 1, 1, 0, 0, 1, 2, 1), cb.CONV_ERR_INVALID_ARG),     # dilated KW > W
    ((V((1 << 20) + 1), F, B, Y, 1, 9, 9, 8, 8, 3, 1, 2, 1, 1, 0, 1, 1, 2), cb.CONV_ERR_MISALIGNED),
    ((X, F, B, V(1 << 20), 1, 9, 9, 8, 8, 1, 3, 1, 2, 0, 1, 1, 1, 2), cb.CONV_ERR_INVALID_ARG),   # Y aliases X
    ((X, F, B, Y, 4096, 4096, 4096, 64, 8, 3, 1, 1, 2, 1, 1, 1, 1, 8), cb.CONV_ERR_UNSUPPORTED),
])
def test_dense_grouped_rejects(args, code):
    assert cb.lib.conv2d_nhwc_fwd_grouped(*args, None) == code


def test_dense_grouped_square_one_group_validates_like_ex():
    # KH = KW, equal axes and one group is conv2d_nhwc_fwd_ex: the same checks apply
    args = (X, F, B, Y, 1, 2, 2, 8, 8, 5, 5, 1, 1, 1, 1, 1, 1, 1)
    assert cb.lib.conv2d_nhwc_fwd_grouped(*args, None) == cb.CONV_ERR_INVALID_ARG
    assert cb.lib.conv2d_nhwc_fwd_ex(X, F, B, Y, 1, 2, 2, 8, 8, 5, 1, 1, 1, None) == cb.CONV_ERR_INVALID_ARG


def test_python_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        cb.conv2d_nhwc_fwd(torch.zeros(1, 5, 5, 8, dtype=torch.bfloat16), torch.zeros(3, 3, 8, 8, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        cb.depthwise_fwd(torch.zeros(1, 2, 5, 5), torch.zeros(2, 3, 3))


def test_last_kernel_is_empty_before_any_launch():
    # rejected calls launch nothing, so the dispatcher's record stays empty on a CPU-only host
    assert cb.lib.conv2d_nhwc_fwd(None, F, Y, 1, 5, 5, 8, 8, 3, None) == cb.CONV_ERR_INVALID_ARG
    assert cb.conv_last_kernel() == ""


def test_im2col_workspace_size():
    # N*Ho*Wo rows of K*K*Cin bf16 values (the DLSys notes' patch matrix)
    assert cb.lib.conv2d_nhwc_im2col_workspace(32, 56, 56, 64, 3) == 32 * 54 * 54 * 9 * 64 * 2
    assert cb.lib.conv2d_nhwc_im2col_workspace(1, 6, 6, 1, 3) == 16 * 9 * 2
    assert cb.lib.conv2d_nhwc_im2col_workspace(1, 2, 6, 1, 3) == 0     # K > H
    assert cb.lib.conv2d_nhwc_im2col_workspace(0, 6, 6, 1, 3) == 0


WS = V(1 << 32)


@pytest.mark.parametrize("ws,nbytes,code", [
    (None, 1 << 20, cb.CONV_ERR_INVALID_ARG),
    (WS, 100, cb.CONV_ERR_INVALID_ARG),                     # smaller than the patch matrix
    (V((1 << 32) + 8), 1 << 20, cb.CONV_ERR_MISALIGNED),     # not 16-byte aligned
    (V((1 << 20) - 64), 1 << 20, cb.CONV_ERR_INVALID_ARG),   # overlaps X
])
def test_im2col_path_rejects(ws, nbytes, code):
    assert cb.lib.conv2d_nhwc_fwd_im2col(X, F, Y, ws, nbytes, 1, 5, 5, 8, 8, 3, None) == code


@pytest.mark.parametrize("args,code", [
    # x, w_dw, b_dw, F, b_pw, y, N, C, H, W, K, stride, pad, dil, Cout, mode
    ((None, B, None, F, None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 16, 0), cb.CONV_ERR_INVALID_ARG),
    ((X, B, None, None, None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 16, 0), cb.CONV_ERR_INVALID_ARG),
    ((X, B, None, F, None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 16, 2), cb.CONV_ERR_INVALID_ARG),       # mode 2
    ((X, B, None, F, None, Y, 1, 8, 9, 9, 3, 0, 1, 1, 16, 0), cb.CONV_ERR_INVALID_ARG),       # stride 0
    ((X, B, None, F, None, Y, 1, 8, 2, 2, 5, 1, 1, 1, 16, 0), cb.CONV_ERR_INVALID_ARG),       # window > image
    ((X, B, None, F, None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 12, 0), cb.CONV_ERR_UNSUPPORTED),       # Cout % 8
    ((X, B, None, F, None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 264, 0), cb.CONV_ERR_UNSUPPORTED),      # Cout > 256
    ((X, B, None, V((1 << 22) + 8), None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 16, 0), cb.CONV_ERR_MISALIGNED),  # F
    ((V((1 << 20) + 2), B, None, F, None, Y, 1, 8, 9, 9, 3, 1, 1, 1, 16, 0), cb.CONV_ERR_MISALIGNED),
    ((X, B, None, F, None, V(1 << 20), 1, 8, 9, 9, 3, 1, 1, 1, 16, 0), cb.CONV_ERR_INVALID_ARG),       # y on x
    ((X, B, None, F, None, Y, 4096, 64, 4096, 4096, 3, 1, 1, 1, 16, 0), cb.CONV_ERR_UNSUPPORTED),
])
def test_dwpw_rejects(args, code):
    assert cb.lib.dwpw_fwd(*args, None) == code


def test_binding_requires_one_device():
    # the binding makes the tensors' device current for the call and refuses a mix of devices
    # (the kernels launch on the current device and would read another GPU's buffer through the
    # wrong mapping)
    import torch
    with pytest.raises(ValueError, match="one CUDA device"):
        cb._device(torch.empty(1), torch.empty(1, device="meta"))
    assert cb._device(torch.empty(1), None, torch.empty(2)) == torch.device("cpu")


@pytest.mark.parametrize("args,code", [
    # X, F, bias, Y, N, H, W, Cin, Cout, KH, KW, sh, sw, pad_top, pad_bottom, pad_left, pad_right, dh, dw, groups
    ((None, F, B, Y, 1, 1, 20, 8, 8, 1, 3, 1, 1, 0, 0, 2, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),
    ((X, F, B, Y, 1, 1, 20, 8, 8, 1, 3, 1, 1, 0, 0, -1, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),   # pad_left < 0
    ((X, F, B, Y, 1, 1, 20, 8, 8, 1, 3, 1, 1, 0, 0, 2, -3, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),   # pad_right < 0
    ((X, F, B, Y, 1, 1, 20, 8, 8, 1, 3, 1, 1, 0, -1, 2, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),   # pad_bottom < 0
    ((X, F, B, Y, 1, 1, 2, 8, 8, 1, 5, 1, 1, 0, 0, 1, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),     # window > padded row
    ((X, F, B, Y, 1, 1, 20, 8, 8, 1, 3, 1, 1, 0, 0, 2, 0, 1, 1, 3), cb.CONV_ERR_INVALID_ARG),    # 3 does not divide 8
    ((X, F, B, V(1 << 20), 1, 1, 20, 8, 8, 1, 3, 1, 1, 0, 0, 2, 0, 1, 1, 1), cb.CONV_ERR_INVALID_ARG),  # Y aliases X
])
def test_dense_grouped_pads_rejects(args, code):
    # padding that differs before and after an axis (a causal Conv1D pads only the left)
    assert cb.lib.conv2d_nhwc_fwd_grouped_pads(*args, None) == code
