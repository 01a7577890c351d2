"""GPU parity of conv2d_nhwc_fwd_ex (stride, zero padding, dilation, bias) against the oracle.

Every case goes through the C ABI; the expectation is the float64 oracle of the same bf16
operands, and the bar is the dense tolerance |y - y_ref| <= 4e-3 * (sum|x||w| + |b|) per output.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = 4e-3


@pytest.fixture(scope="module")
def cb(cuda):
    import cnn_convolution_nhwc_b200 as cb
    return cb


def _inputs(N, H, W, Cin, Cout, K, stride, pad, dil, bias, seed):
    case = workloads.DenseCase("t", N, H, W, Cin, Cout, K, "bf16", "normal", seed, stride, pad, dil, bias)
    Xb, Fb = workloads.dense_inputs(case)
    return Xb, Fb, workloads.dense_bias(case)


def _run(cb, Xb, Fb, b, stride, pad, dil, env=None):
    old = os.environ.get("CONV_B200_DENSE")
    if env is not None:
        os.environ["CONV_B200_DENSE"] = env
    try:
        X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
        F = torch.from_numpy(Fb.view(np.int16)).view(torch.bfloat16).cuda()
        bt = None if b is None else torch.from_numpy(np.ascontiguousarray(b, np.float32)).cuda()
        Y = cb.conv2d_nhwc_fwd_ex(X, F, bt, stride=stride, pad=pad, dil=dil)
        kernel = cb.conv_last_kernel()
        y = workloads.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    finally:
        if env is not None:
            if old is None:
                del os.environ["CONV_B200_DENSE"]
            else:
                os.environ["CONV_B200_DENSE"] = old
    assert cb.conv_device_status() == cb.CONV_OK
    return y, kernel


def _check(y, Xb, Fb, b, stride, pad, dil):
    ref, absum = oracle.conv2d_nhwc_ex(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), b, stride, pad, dil)
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    bad = np.abs(y - ref) > TOL * absum
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance"


# (N, H, W, Cin, Cout, K, stride, pad, dil, bias, kernel expected by default)
CASES = [
    (4, 56, 56, 64, 128, 3, 2, 1, 1, True, "dense_tc_kernel"),     # stage transition 56 -> 28
    (2, 30, 30, 64, 64, 3, 1, 1, 1, True, "dense_halo_pad_kernel"),   # "same" padding with a bias
    (2, 40, 36, 32, 64, 3, 1, 2, 2, False, "dense_tc_kernel"),     # dilation 2
    (4, 32, 32, 64, 64, 1, 2, 0, 1, True, "dense_tc_kernel"),      # 1x1 stride-2 projection
    (2, 64, 64, 8, 64, 4, 4, 0, 1, True, "dense_tc_kernel"),       # patch projection, K = stride
    (4, 20, 20, 64, 40, 5, 1, 4, 2, True, "dense_tc_kernel"),      # wide padding, ragged Cout
    (3, 33, 17, 128, 136, 3, 3, 1, 1, True, "dense_tc_kernel"),    # stride 3, ragged rows and N tile
    (2, 9, 11, 3, 5, 3, 2, 1, 2, True, "dense_direct_kernel"),     # Cin not a multiple of 8
    (1, 7, 7, 16, 16, 3, 3, 2, 1, False, "dense_direct_kernel"),   # input below 128 KiB
    (1, 6, 5, 8, 8, 3, 1, 0, 1, True, "dense_direct_kernel"),      # a bias alone, tiny input
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:9])) + ("b" if c[9] else ""))
def test_general_geometry(cb, case):
    N, H, W, Cin, Cout, K, s, p, d, bias, expected = case
    Xb, Fb, b = _inputs(N, H, W, Cin, Cout, K, s, p, d, bias, seed=sum(case[:9]))
    y, kernel = _run(cb, Xb, Fb, b, s, p, d)
    _check(y, Xb, Fb, b, s, p, d)
    assert kernel == expected


@pytest.mark.parametrize("case", [c for c in CASES if c[10] == "dense_tc_kernel"][:4],
                         ids=lambda c: "x".join(map(str, c[:9])))
def test_tensor_core_and_direct_paths_agree(cb, case):
    N, H, W, Cin, Cout, K, s, p, d, bias, _ = case
    Xb, Fb, b = _inputs(N, H, W, Cin, Cout, K, s, p, d, bias, seed=7)
    y_tc, k_tc = _run(cb, Xb, Fb, b, s, p, d)
    y_cc, k_cc = _run(cb, Xb, Fb, b, s, p, d, env="direct")
    assert (k_tc, k_cc) == ("dense_tc_kernel", "dense_direct_kernel")
    _check(y_tc, Xb, Fb, b, s, p, d)
    _check(y_cc, Xb, Fb, b, s, p, d)


@pytest.mark.parametrize("bn", ["bn64", "bn128", "bn256"])
def test_tile_widths(cb, bn):
    Xb, Fb, b = _inputs(2, 28, 28, 64, 192, 3, 2, 1, 1, True, seed=9)
    y, kernel = _run(cb, Xb, Fb, b, 2, 1, 1, env=bn)
    assert kernel == "dense_tc_kernel"
    _check(y, Xb, Fb, b, 2, 1, 1)


def test_plain_geometry_is_the_plain_entry(cb):
    # stride 1, pad 0, dil 1 and no bias take conv2d_nhwc_fwd's path: identical bits
    Xb, Fb, _ = _inputs(2, 20, 20, 64, 64, 3, 1, 0, 1, False, seed=11)
    y, kernel = _run(cb, Xb, Fb, None, 1, 0, 1)
    X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
    F = torch.from_numpy(Fb.view(np.int16)).view(torch.bfloat16).cuda()
    y0 = workloads.bf16_to_f32(cb.conv2d_nhwc_fwd(X, F).view(torch.int16).cpu().numpy().view(np.uint16))
    assert kernel == cb.conv_last_kernel()
    assert np.array_equal(y, y0.astype(np.float64))
    _check(y, Xb, Fb, None, 1, 0, 1)


def test_page_bias_examples(cb):
    # "One window is still a weighted sum" and "The matrix connection": x = 1..5, filters
    # (2, 0, -1) and (1, 1, 1), biases 1 and 0 -> (0, 1, 2) and (6, 9, 12); embedded as row 0 of
    # a 3 x 5 image, 8 channels (channel 0 carries the signal), 8 filters (0 and 1 used)
    X = np.zeros((1, 3, 5, 8), np.float32)
    X[0, 0, :, 0] = [1, 2, 3, 4, 5]
    F = np.zeros((3, 3, 8, 8), np.float32)
    F[0, :, 0, 0] = [2, 0, -1]
    F[0, :, 0, 1] = [1, 1, 1]
    b = np.zeros(8, np.float32)
    b[0] = 1
    for env in (None, "direct"):
        y, _ = _run(cb, workloads.bf16_bits(X), workloads.bf16_bits(F), b, 1, 0, 1, env=env)
        assert np.array_equal(y[0, 0, :, 0], [0, 1, 2]) and np.array_equal(y[0, 0, :, 1], [6, 9, 12])


def test_full_size_stride2_workload_sampled(cb):
    c = workloads.DENSE_S2
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y, kernel = _run(cb, Xb, Fb, b, c.stride, c.pad, c.dil)
    assert kernel == "dense_tc_kernel"
    idx = (workloads.splitmix64(5, 20000) % np.uint64(y.size)).astype(np.int64)
    ref, absum = oracle.conv2d_nhwc_ex_points(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), idx, b, c.stride,
                                              c.pad, c.dil)
    got = y.reshape(-1)[idx]
    assert np.all(np.abs(got - ref) <= TOL * absum)
