"""GPU parity of the explicit-im2col comparison path (patch matrix + one cuBLAS GEMM)."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cb(cuda):
    import cnn_convolution_nhwc_b200 as cb
    return cb


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("shape", [(2, 10, 12, 16, 24, 3), (1, 6, 6, 8, 8, 3), (3, 9, 7, 3, 5, 2), (2, 8, 8, 64, 64, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_patch_matrix_and_gemm(cb, shape):
    N, H, W, Cin, Cout, K = shape
    case = workloads.DenseCase("t", N, H, W, Cin, Cout, K, "bf16", "normal", sum(shape))
    Xb, Fb = workloads.dense_inputs(case)
    ws = torch.empty(cb.lib.conv2d_nhwc_im2col_workspace(N, H, W, Cin, K), dtype=torch.uint8, device="cuda")
    Y = cb.conv2d_nhwc_fwd_im2col(_dev(Xb), _dev(Fb), workspace=ws)
    assert cb.conv_last_kernel() == "im2col_pack_kernel+cublas"
    assert cb.conv_device_status() == cb.CONV_OK
    # the workspace holds the patch matrix: rows (n, y, x), columns (i, j, c), a pure copy of X
    Ho, Wo = H - K + 1, W - K + 1
    A = ws.cpu().numpy().view(np.uint16).reshape(N * Ho * Wo, K * K * Cin)
    win = np.lib.stride_tricks.sliding_window_view(Xb, (K, K), axis=(1, 2))        # N,Ho,Wo,C,K,K
    ref_A = np.transpose(win, (0, 1, 2, 4, 5, 3)).reshape(-1, K * K * Cin)
    assert np.array_equal(A, ref_A)
    y = workloads.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    ref, absum = oracle.conv2d_nhwc(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb))
    assert np.all(np.abs(y - ref) <= 4e-3 * absum)


def test_full_size_headline_sampled(cb):
    c = workloads.DENSE_3X3
    Xb, Fb = workloads.dense_inputs(c)
    Y = cb.conv2d_nhwc_fwd_im2col(_dev(Xb), _dev(Fb))
    y = workloads.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64).reshape(-1)
    idx = (workloads.splitmix64(9, 20000) % np.uint64(y.size)).astype(np.int64)
    ref, absum = oracle.conv2d_nhwc_points(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), idx)
    assert np.all(np.abs(y[idx] - ref) <= 4e-3 * absum)


def test_rejects_small_workspace(cb):
    X = torch.zeros((1, 6, 6, 8), dtype=torch.bfloat16, device="cuda")
    F = torch.zeros((3, 3, 8, 8), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(cb.ConvError) as e:
        cb.conv2d_nhwc_fwd_im2col(X, F, workspace=ws)
    assert e.value.code == cb.CONV_ERR_INVALID_ARG
