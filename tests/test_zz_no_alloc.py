"""The allocation-free entry point conv2d_nhwc_fwd_im2col_noalloc, called through the C ABI.

Some callers cannot allocate device memory at all: code running under a framework whose pool
owns the whole device, a plugin inside a host application that forbids allocation, or a
real-time path that must not pay cudaMalloc's implicit synchronisation or risk running out of
memory after start-up. For them the explicit-im2col comparison path has a variant whose patch
matrix lives in scratch the library reserves statically, one array per device, instead of a
workspace the caller allocates.

The test checks it against the workspace entry point, conv2d_nhwc_fwd_im2col, on the same
seeded inputs and within the dense tolerance |y - y_ref| <= 4e-3 * sum|x||w| per output, for
calls in a row on different shapes (the scratch keeps the previous call's contents, which must
not leak into the next result), one of them close to the scratch's size limit. It runs last
(this file's name sorts after the others) and passes alone in a fresh process as well as after
the rest of the suite: the entry point's first call on a device does its own set-up.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

V = ctypes.c_void_p


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _host(Y):
    return workloads.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


# (N, H, W, Cin, Cout, K): a patch matrix of 28.9 MB (near the 32 MiB limit), a small ragged one
# with channel counts that are not multiples of 64, then the first shape again
SHAPES = [(8, 58, 58, 64, 64, 3), (2, 13, 11, 16, 24, 3), (8, 58, 58, 64, 64, 3)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry(cuda):
    import cnn_convolution_nhwc_b200 as cb
    lib = cb.lib
    stream = V(torch.cuda.current_stream().cuda_stream)
    for call, (N, H, W, Cin, Cout, K) in enumerate(SHAPES):
        case = workloads.DenseCase("noalloc", N, H, W, Cin, Cout, K, "bf16", "normal", 100 + call)
        Xb, Fb = workloads.dense_inputs(case)
        X, F = _dev(Xb), _dev(Fb)
        Ho, Wo = H - K + 1, W - K + 1
        need = lib.conv2d_nhwc_im2col_workspace(N, H, W, Cin, K)
        assert 0 < need <= cb.CONV_IM2COL_STATIC_BYTES
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        Y_ws = torch.empty((N, Ho, Wo, Cout), dtype=torch.bfloat16, device="cuda")
        Y_na = torch.full((N, Ho, Wo, Cout), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = lib.conv2d_nhwc_fwd_im2col(V(X.data_ptr()), V(F.data_ptr()), V(Y_ws.data_ptr()), V(ws.data_ptr()),
                                        need, N, H, W, Cin, Cout, K, stream)
        assert rc == cb.CONV_OK, cb.conv_status_string(rc)
        rc = lib.conv2d_nhwc_fwd_im2col_noalloc(V(X.data_ptr()), V(F.data_ptr()), V(Y_na.data_ptr()), N, H, W, Cin,
                                                Cout, K, stream)
        assert rc == cb.CONV_OK, cb.conv_status_string(rc)
        torch.cuda.synchronize()
        assert cb.conv_device_status() == cb.CONV_OK
        y_ws, y_na = _host(Y_ws), _host(Y_na)
        ref, absum = oracle.conv2d_nhwc(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb))
        assert np.isfinite(y_na).all()
        assert np.all(np.abs(y_na - y_ws) <= 4e-3 * absum), f"call {call}: differs from the workspace entry"
        assert np.all(np.abs(y_na - ref) <= 4e-3 * absum), f"call {call}: differs from the oracle"


def test_noalloc_rejects_a_patch_matrix_beyond_the_scratch():
    # 9 x 58 x 58 pixels x 576 columns x 2 bytes = 34.9 MB > 32 MiB: refused before any CUDA call
    # (the fake device addresses below are never touched)
    import cnn_convolution_nhwc_b200 as cb
    assert cb.lib.conv2d_nhwc_im2col_workspace(9, 60, 60, 64, 3) > cb.CONV_IM2COL_STATIC_BYTES
    rc = cb.lib.conv2d_nhwc_fwd_im2col_noalloc(V(1 << 20), V(1 << 34), V(1 << 36), 9, 60, 60, 64, 64, 3, None)
    assert rc == cb.CONV_ERR_UNSUPPORTED
    assert cb.lib.conv2d_nhwc_im2col_workspace(8, 60, 60, 64, 3) <= cb.CONV_IM2COL_STATIC_BYTES
