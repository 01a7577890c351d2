"""Pins for the CPU oracle. None of these computes its expectation by calling the oracle:

* worked examples printed on the pages (tests/golden, each file citing its page and section);
* library routines for cases that reduce to them (numpy matmul, numpy sliding windows,
  torch's CPU conv2d in float64);
* closed forms derived by hand from IEEE-754 binary32 round-to-nearest-even;
* invariants the pages state (translation equivariance, K=1 is a matmul, the filter that
  spans the whole image is a dot product).
"""
import json
import math
import os
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def _ints(seed, shape, lo=-3, hi=3):
    return workloads.int_uniform(seed, int(np.prod(shape)), lo, hi).reshape(shape)


def _torch_conv_nhwc(X, F):
    """torch CPU conv2d in float64, with the NHWC/KKIO <-> NCHW/OIHW axis changes the DLSys
    notes describe for comparing against PyTorch (section 1)."""
    x = torch.from_numpy(np.asarray(X, dtype=np.float64)).permute(0, 3, 1, 2)
    f = torch.from_numpy(np.asarray(F, dtype=np.float64)).permute(3, 2, 0, 1)
    return torch.nn.functional.conv2d(x, f).permute(0, 2, 3, 1).numpy()


# ------------------------------------------------------------------------------------------
# Dense: worked examples
# ------------------------------------------------------------------------------------------


def test_dense_6x6_arange_example():
    g = _golden("dlsys14_patch_example.json")
    X = np.arange(36, dtype=np.float32).reshape(1, 6, 6, 1)
    F = np.arange(9, dtype=np.float32).reshape(3, 3, 1, 1)
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y[0, :, :, 0], np.array(g["output"], dtype=np.float64))
    # the two flattened windows the page spells out give the first two outputs
    a = np.arange(36).reshape(6, 6)
    assert list(a[0:3, 0:3].ravel()) == g["first_window_flat"]
    assert list(a[0:3, 1:4].ravel()) == g["second_window_flat"]


def test_dense_tiny_2d_example():
    g = _golden("wxb_2d_examples.json")["tiny_2d"]
    X = np.array(g["image"], dtype=np.float32).reshape(1, 3, 3, 1)
    F = np.array(g["filter"], dtype=np.float32).reshape(2, 2, 1, 1)
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y[0, :, :, 0], np.array(g["output"], dtype=np.float64))


def test_dense_sobel_example_two_output_channels():
    g = _golden("wxb_2d_examples.json")["sobel"]
    X = np.array(g["image"], dtype=np.float32).reshape(1, 6, 6, 1)
    F = np.stack([np.array(g["gx"]), np.array(g["gy"])], axis=-1).astype(np.float32).reshape(3, 3, 1, 2)
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y[0, :, :, 0], np.array(g["gx_output"], dtype=np.float64))
    assert np.array_equal(Y[0, :, :, 1], np.array(g["gy_output"], dtype=np.float64))
    assert Y[0, 0, 1, 0] == g["patch_row0_col1_dot_gx"]
    assert Y[0, 0, 1, 1] == g["patch_row0_col1_dot_gy"]


def _embed_1d(x, ks):
    """A 1-D signal as row 0 of a K x L image and 1-D filters as row 0 of K x K filters
    (other rows zero), so that the valid 2-D output is the single 1-D response row."""
    K = len(ks[0])
    L = len(x)
    X = np.zeros((1, K, L, 1), dtype=np.float32)
    X[0, 0, :, 0] = x
    F = np.zeros((K, K, 1, len(ks)), dtype=np.float32)
    for o, k in enumerate(ks):
        F[0, :, 0, o] = k
    return X, F


def test_dense_1d_examples_embedded():
    g = _golden("wxb_1d_examples.json")
    e = g["weighted_sum_with_bias"]
    X, F = _embed_1d(e["x"], [e["k"]])
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert Y[0, 0, 0, 0] == e["first_window_without_bias"]
    assert np.array_equal(Y[0, 0, :, 0] + e["bias"], np.array(e["output"], dtype=np.float64))
    for name in ("step_difference", "motif"):
        e = g[name]
        X, F = _embed_1d(e["x"], [e["k"]])
        Y, _ = oracle.conv2d_nhwc(X, F)
        assert np.array_equal(Y[0, 0, :, 0], np.array(e["output"], dtype=np.float64)), name
    e = g["spike_average"]
    X, F = _embed_1d(e["x"], [[1.0 / 3.0] * 3])
    Y, _ = oracle.conv2d_nhwc(X, F)
    # float32(1/3) * 3 is 1 + 2**-25 * ... in float64: within one float32 ulp of the page's 1
    assert np.allclose(Y[0, 0, :, 0], e["output"], rtol=0, atol=2.0 ** -23)


def test_dense_two_filters_example():
    e = _golden("wxb_1d_examples.json")["two_filters_with_bias"]
    X, F = _embed_1d(e["x"], e["filters"])
    Y, _ = oracle.conv2d_nhwc(X, F)
    for o in range(2):
        assert np.array_equal(Y[0, 0, :, o] + e["bias"][o], np.array(e["output_per_filter"][o], dtype=np.float64))


# ------------------------------------------------------------------------------------------
# Dense: library routines and invariants
# ------------------------------------------------------------------------------------------


def test_dense_k1_is_matmul():
    X = _ints(11, (3, 5, 7, 6))
    F = _ints(12, (1, 1, 6, 5))
    Y, _ = oracle.conv2d_nhwc(X, F)
    ref = (X.reshape(-1, 6).astype(np.float64) @ F[0, 0].astype(np.float64)).reshape(3, 5, 7, 5)
    assert np.array_equal(Y, ref)


def test_dense_shifted_slice_sum_equals_definition():
    # K*K channel matmuls over shifted input slices, accumulated (DLSys notes, section 2)
    N, H, W, C, O, K = 2, 7, 9, 3, 4, 3
    X = _ints(21, (N, H, W, C)).astype(np.float64)
    F = _ints(22, (K, K, C, O)).astype(np.float64)
    Ho, Wo = H - K + 1, W - K + 1
    acc = np.zeros((N, Ho, Wo, O))
    for i in range(K):
        for j in range(K):
            acc = acc + np.matmul(X[:, i:i + Ho, j:j + Wo, :], F[i, j])
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y, acc)


def test_dense_im2col_gemm_equals_definition():
    # patch rows flattened in (i, j, c) order times the filter flattened the same way
    # (DLSys notes, section 5)
    N, H, W, C, O, K = 2, 6, 8, 5, 3, 4
    X = _ints(31, (N, H, W, C)).astype(np.float64)
    F = _ints(32, (K, K, C, O)).astype(np.float64)
    win = np.lib.stride_tricks.sliding_window_view(X, (K, K), axis=(1, 2))   # N,Ho,Wo,C,K,K
    rows = np.transpose(win, (0, 1, 2, 4, 5, 3)).reshape(-1, K * K * C)
    ref = (rows @ F.reshape(K * K * C, O)).reshape(N, H - K + 1, W - K + 1, O)
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y, ref)


@pytest.mark.parametrize("shape", [(2, 9, 5, 3, 7, 3), (1, 6, 11, 8, 2, 2), (3, 4, 4, 2, 5, 4),
                                   (1, 13, 10, 16, 9, 5)])
def test_dense_matches_torch_conv2d_f64(shape):
    N, H, W, C, O, K = shape
    X = workloads.normal(41, N * H * W * C, 1.0).reshape(N, H, W, C)
    F = workloads.normal(42, K * K * C * O, 0.3).reshape(K, K, C, O)
    Y, A = oracle.conv2d_nhwc(X, F)
    ref = _torch_conv_nhwc(X, F)
    assert Y.shape == ref.shape
    assert np.all(np.abs(Y - ref) <= 1e-13 * A)


def test_dense_full_image_filter_is_dot_product():
    N, S, C, O = 3, 5, 4, 3
    X = _ints(51, (N, S, S, C))
    F = _ints(52, (S, S, C, O))
    Y, _ = oracle.conv2d_nhwc(X, F)
    assert Y.shape == (N, 1, 1, O)
    for n in range(N):
        for o in range(O):
            assert Y[n, 0, 0, o] == np.dot(X[n].ravel().astype(np.float64), F[:, :, :, o].ravel().astype(np.float64))


def test_dense_translation_equivariance():
    N, H, W, C, O, K = 1, 8, 10, 3, 2, 3
    X = _ints(61, (N, H, W, C))
    F = _ints(62, (K, K, C, O))
    Xs = np.zeros_like(X)
    Xs[:, :, 1:, :] = X[:, :, :-1, :]       # shift right by one column
    Y, _ = oracle.conv2d_nhwc(X, F)
    Ys, _ = oracle.conv2d_nhwc(Xs, F)
    assert np.array_equal(Ys[:, :, 1:, :], Y[:, :, :-1, :])


def test_dense_abssum_is_conv_of_magnitudes():
    X = workloads.normal(71, 2 * 6 * 7 * 3, 1.0).reshape(2, 6, 7, 3)
    F = workloads.normal(72, 3 * 3 * 3 * 4, 1.0).reshape(3, 3, 3, 4)
    _, A = oracle.conv2d_nhwc(X, F)
    Yabs, _ = oracle.conv2d_nhwc(np.abs(X), np.abs(F))
    assert np.array_equal(A, Yabs)
    ref = _torch_conv_nhwc(np.abs(X), np.abs(F))
    assert np.allclose(A, ref, rtol=1e-13, atol=0)


def test_dense_points_match_full():
    X = workloads.normal(81, 2 * 9 * 8 * 5, 1.0).reshape(2, 9, 8, 5)
    F = workloads.normal(82, 3 * 3 * 5 * 6, 1.0).reshape(3, 3, 5, 6)
    Y, A = oracle.conv2d_nhwc(X, F)
    idx = np.array([0, 1, 17, 100, Y.size - 1], dtype=np.int64)
    y, a = oracle.conv2d_nhwc_points(X, F, idx)
    assert np.array_equal(y, Y.ravel()[idx]) and np.array_equal(a, A.ravel()[idx])


# ------------------------------------------------------------------------------------------
# Dense with stride, zero padding, dilation and bias ("Convolution Is Wx+b Moving Across a
# Signal"): each variant pinned to the plain definition composed with a numpy reshaping that
# has its own textbook meaning (zero-padded input, subsampled output, zero-inserted filter)
# ------------------------------------------------------------------------------------------


def _dilate_filter(F, d):
    K = F.shape[0]
    Kd = d * (K - 1) + 1
    out = np.zeros((Kd, Kd) + F.shape[2:], dtype=F.dtype)
    out[::d, ::d] = F
    return out


def test_dense_ex_defaults_are_the_plain_definition():
    X = _ints(61, (2, 7, 9, 3))
    F = _ints(62, (3, 3, 3, 4))
    Y, A = oracle.conv2d_nhwc_ex(X, F)
    Y0, A0 = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y, Y0) and np.array_equal(A, A0)


@pytest.mark.parametrize("pad", [1, 2, 4])
def test_dense_ex_padding_is_a_zero_padded_input(pad):
    X = _ints(63, (2, 6, 5, 3))
    F = _ints(64, (3, 3, 3, 2))
    Y, _ = oracle.conv2d_nhwc_ex(X, F, pad=pad)
    Xp = np.pad(X, ((0, 0), (pad, pad), (pad, pad), (0, 0)))
    ref, _ = oracle.conv2d_nhwc(Xp, F)
    assert np.array_equal(Y, ref)


@pytest.mark.parametrize("stride", [2, 3])
def test_dense_ex_stride_subsamples_the_output(stride):
    X = _ints(65, (2, 11, 10, 3))
    F = _ints(66, (3, 3, 3, 2))
    Y, _ = oracle.conv2d_nhwc_ex(X, F, stride=stride)
    ref, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y, ref[:, ::stride, ::stride, :])


@pytest.mark.parametrize("dil", [2, 3])
def test_dense_ex_dilation_is_a_zero_inserted_filter(dil):
    X = _ints(67, (1, 12, 13, 2))
    F = _ints(68, (3, 3, 2, 3))
    Y, _ = oracle.conv2d_nhwc_ex(X, F, dil=dil)
    ref, _ = oracle.conv2d_nhwc(X, _dilate_filter(F, dil))
    assert np.array_equal(Y, ref)


def test_dense_ex_bias_is_added_per_output_channel():
    X = _ints(69, (2, 6, 6, 3))
    F = _ints(70, (3, 3, 3, 4))
    b = np.array([1.0, -2.0, 0.5, 3.0], dtype=np.float32)
    Y, A = oracle.conv2d_nhwc_ex(X, F, bias=b)
    Y0, A0 = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y, Y0 + b) and np.array_equal(A, A0 + np.abs(b))


@pytest.mark.parametrize("stride,pad,dil", [(2, 1, 1), (2, 2, 2), (3, 1, 2), (1, 3, 3)])
def test_dense_ex_all_variants_compose(stride, pad, dil):
    X = _ints(71, (2, 13, 11, 3))
    F = _ints(72, (3, 3, 3, 2))
    b = np.array([0.25, -1.0], dtype=np.float32)
    Y, _ = oracle.conv2d_nhwc_ex(X, F, bias=b, stride=stride, pad=pad, dil=dil)
    Xp = np.pad(X, ((0, 0), (pad, pad), (pad, pad), (0, 0)))
    ref, _ = oracle.conv2d_nhwc(Xp, _dilate_filter(F, dil))
    ref = ref[:, ::stride, ::stride, :] + b
    assert np.array_equal(Y, ref)


def test_dense_ex_matches_torch_conv2d_f64():
    X = workloads.normal(73, 2 * 15 * 14 * 5, 1.0).reshape(2, 15, 14, 5)
    F = workloads.normal(74, 3 * 3 * 5 * 6, 0.3).reshape(3, 3, 5, 6)
    b = workloads.normal(75, 6, 0.5)
    Y, A = oracle.conv2d_nhwc_ex(X, F, bias=b, stride=2, pad=1, dil=2)
    x = torch.from_numpy(np.asarray(X, dtype=np.float64)).permute(0, 3, 1, 2)
    f = torch.from_numpy(np.asarray(F, dtype=np.float64)).permute(3, 2, 0, 1)
    ref = torch.nn.functional.conv2d(x, f, torch.from_numpy(np.asarray(b, dtype=np.float64)), stride=2, padding=1,
                                     dilation=2).permute(0, 2, 3, 1).numpy()
    assert Y.shape == ref.shape
    assert np.all(np.abs(Y - ref) <= 1e-13 * A)


def test_dense_ex_output_size_rule():
    # "Build an image-gradient map, one number at a time": five inputs, a width-three filter,
    # no padding, stride and dilation one give 5 - 3 + 1 = 3 positions; the general rule is
    # floor((in + 2*pad - (dil*(k-1) + 1)) / stride) + 1 per axis
    X = np.zeros((1, 3, 5, 1), np.float32)
    F = np.zeros((3, 3, 1, 1), np.float32)
    assert oracle.conv2d_nhwc_ex(X, F)[0].shape == (1, 1, 3, 1)
    X = np.zeros((1, 17, 23, 1), np.float32)
    for stride in (1, 2, 3):
        for pad in (0, 1, 2):
            for dil in (1, 2):
                Y, _ = oracle.conv2d_nhwc_ex(X, F, stride=stride, pad=pad, dil=dil)
                eff = dil * 2 + 1
                assert Y.shape[1:3] == ((17 + 2 * pad - eff) // stride + 1, (23 + 2 * pad - eff) // stride + 1)


def test_dense_ex_weighted_sum_with_bias_example():
    # the page's first window with bias: x = 1..5, k = (2, 0, -1), b = 1 -> (0, 1, 2)
    e = _golden("wxb_1d_examples.json")["weighted_sum_with_bias"]
    X, F = _embed_1d(e["x"], [e["k"]])
    Y, _ = oracle.conv2d_nhwc_ex(X, F, bias=np.array([e["bias"]], np.float32))
    assert np.array_equal(Y[0, 0, :, 0], np.array(e["output"], dtype=np.float64))
    e = _golden("wxb_1d_examples.json")["two_filters_with_bias"]
    X, F = _embed_1d(e["x"], e["filters"])
    Y, _ = oracle.conv2d_nhwc_ex(X, F, bias=np.array(e["bias"], np.float32))
    for o in range(2):
        assert np.array_equal(Y[0, 0, :, o], np.array(e["output_per_filter"][o], dtype=np.float64))


def test_dense_ex_patch_projection_is_flattened_patches_times_weights():
    # "Why variants matter": kernel = stride = P turns each non-overlapping P x P patch into one
    # output; with corresponding weights and bias it equals flattened patches times a
    # [P*P*Cin, D] matrix plus the bias
    N, P, G, C, D = 2, 4, 3, 3, 5
    X = _ints(76, (N, G * P, G * P, C)).astype(np.float64)
    F = _ints(77, (P, P, C, D)).astype(np.float64)
    b = np.array([1.0, 2.0, -1.0, 0.5, 0.0])
    Y, _ = oracle.conv2d_nhwc_ex(X, F, bias=b, stride=P)
    patches = X.reshape(N, G, P, G, P, C).transpose(0, 1, 3, 2, 4, 5).reshape(N * G * G, P * P * C)
    ref = (patches @ F.reshape(P * P * C, D) + b).reshape(N, G, G, D)
    assert np.array_equal(Y, ref)


def test_dense_ex_points_match_full():
    X = _ints(78, (2, 9, 8, 3))
    F = _ints(79, (3, 3, 3, 4))
    b = np.array([1, 2, 3, 4], np.float32)
    Y, A = oracle.conv2d_nhwc_ex(X, F, bias=b, stride=2, pad=1, dil=2)
    idx = np.arange(Y.size, dtype=np.int64)[::7]
    y, a = oracle.conv2d_nhwc_ex_points(X, F, idx, bias=b, stride=2, pad=1, dil=2)
    assert np.array_equal(y, Y.reshape(-1)[idx]) and np.array_equal(a, A.reshape(-1)[idx])


# ------------------------------------------------------------------------------------------
# Grouped convolution, per-axis geometry, KH x KW kernels, Conv1D (the Wx+b page's CKE
# section: grouped Conv1D with a bias)
# ------------------------------------------------------------------------------------------


def test_grouped_one_group_square_is_the_ex_definition():
    X = _ints(81, (2, 9, 8, 6))
    F = _ints(82, (3, 3, 6, 4))
    b = np.array([1, -1, 2, 0.5], np.float32)
    Y, A = oracle.conv2d_grouped(X, F, bias=b, stride=2, pad=1, dil=2)
    Y0, A0 = oracle.conv2d_nhwc_ex(X, F, bias=b, stride=2, pad=1, dil=2)
    assert np.array_equal(Y, Y0) and np.array_equal(A, A0)


@pytest.mark.parametrize("groups", [2, 3, 6])
def test_grouped_is_independent_convolutions_of_the_channel_slices(groups):
    Cin, Cout = 12, 6 * groups
    Cg, Og = Cin // groups, Cout // groups
    X = _ints(83, (2, 8, 7, Cin))
    F = _ints(84, (3, 3, Cg, Cout))
    b = _ints(85, (Cout,)).astype(np.float32)
    Y, _ = oracle.conv2d_grouped(X, F, bias=b, stride=(2, 1), pad=(1, 2), groups=groups)
    for g in range(groups):
        ref, _ = oracle.conv2d_grouped(X[..., g * Cg:(g + 1) * Cg], F[..., g * Og:(g + 1) * Og], bias=b[g * Og:(g + 1) * Og],
                                       stride=(2, 1), pad=(1, 2))
        assert np.array_equal(Y[..., g * Og:(g + 1) * Og], ref)


@pytest.mark.parametrize("case", [((2, 1), (1, 0), (1, 1), (3, 2)), ((1, 3), (0, 2), (2, 1), (2, 5)),
                                  ((2, 2), (1, 1), (1, 2), (1, 3))])
def test_grouped_per_axis_and_non_square_match_torch(case):
    (sh, sw), (ph, pw), (dh, dw), (KH, KW) = case
    groups = 2
    X = workloads.normal(86, 2 * 13 * 11 * 8, 1.0).reshape(2, 13, 11, 8)
    F = workloads.normal(87, KH * KW * 4 * 6, 0.3).reshape(KH, KW, 4, 6)
    b = workloads.normal(88, 6, 0.5)
    Y, A = oracle.conv2d_grouped(X, F, bias=b, stride=(sh, sw), pad=(ph, pw), dil=(dh, dw), groups=groups)
    x = torch.from_numpy(np.asarray(X, dtype=np.float64)).permute(0, 3, 1, 2)
    f = torch.from_numpy(np.asarray(F, dtype=np.float64)).permute(3, 2, 0, 1)
    ref = torch.nn.functional.conv2d(x, f, torch.from_numpy(np.asarray(b, dtype=np.float64)), stride=(sh, sw),
                                     padding=(ph, pw), dilation=(dh, dw), groups=groups).permute(0, 2, 3, 1).numpy()
    assert Y.shape == ref.shape
    assert np.all(np.abs(Y - ref) <= 1e-13 * A)


def test_conv1d_is_the_one_dimensional_correlation():
    # H = KH = 1: every output is numpy's valid 1-D correlation of one input channel with one
    # filter row, summed over the group's channels
    L, Cin, Cout, K = 20, 4, 6, 5
    X = _ints(89, (3, 1, L, Cin))
    F = _ints(90, (1, K, Cin, Cout))
    Y, _ = oracle.conv2d_grouped(X, F)
    for n in range(3):
        for o in range(Cout):
            ref = sum(np.correlate(X[n, 0, :, c].astype(np.float64), F[0, :, c, o].astype(np.float64), "valid")
                      for c in range(Cin))
            assert np.array_equal(Y[n, 0, :, o], ref)


def test_conv1d_page_example_two_filters_with_bias():
    # "The matrix connection": x = 1..5, filters (2, 0, -1) and (1, 1, 1), biases (1, 0)
    e = _golden("wxb_1d_examples.json")["two_filters_with_bias"]
    X = np.array(e["x"], np.float32).reshape(1, 1, 5, 1)
    F = np.array(e["filters"], np.float32).T.reshape(1, 3, 1, 2)
    Y, _ = oracle.conv2d_grouped(X, F, bias=np.array(e["bias"], np.float32))
    for o in range(2):
        assert np.array_equal(Y[0, 0, :, o], np.array(e["output_per_filter"][o], dtype=np.float64))


def test_grouped_points_are_the_full_output():
    X = workloads.normal(91, 2 * 9 * 10 * 12, 1.0).reshape(2, 9, 10, 12)
    F = workloads.normal(92, 3 * 2 * 4 * 6, 0.3).reshape(3, 2, 4, 6)
    b = workloads.normal(93, 6, 0.5)
    kw = dict(stride=(2, 1), pad=(1, 0), dil=(1, 2), groups=3)
    Y, A = oracle.conv2d_grouped(X, F, b, **kw)
    idx = (workloads.splitmix64(94, 300) % np.uint64(Y.size)).astype(np.int64)
    y, a = oracle.conv2d_grouped_points(X, F, idx, b, **kw)
    assert np.array_equal(y, Y.reshape(-1)[idx]) and np.array_equal(a, A.reshape(-1)[idx])


def test_grouped_rejects_bad_groups():
    with pytest.raises(ValueError):
        oracle.conv2d_grouped(np.zeros((1, 5, 5, 6), np.float32), np.zeros((3, 3, 2, 4), np.float32), groups=4)


def test_dense_rejects_incompatible_shapes():
    with pytest.raises(ValueError):
        oracle.conv2d_nhwc(np.zeros((1, 3, 3, 2), np.float32), np.zeros((4, 4, 2, 1), np.float32))
    with pytest.raises(ValueError):
        oracle.conv2d_nhwc(np.zeros((1, 5, 5, 2), np.float32), np.zeros((3, 3, 3, 1), np.float32))


# ------------------------------------------------------------------------------------------
# Depthwise: worked examples (both modes)
# ------------------------------------------------------------------------------------------

MODES = [oracle.DW_EXACT, oracle.DW_FAST]


def _dw1d(x, ks, bias=None, mode=oracle.DW_EXACT):
    """1-D signal as a 1 x L plane, each filter a 1 x k kernel; mult = number of filters."""
    x = np.array(x, dtype=np.float32).reshape(1, 1, 1, -1)
    w = np.array(ks, dtype=np.float32).reshape(len(ks), 1, -1)
    b = None if bias is None else np.array(bias, dtype=np.float32)
    return oracle.depthwise(x, w, b, mult=len(ks), mode=mode)


@pytest.mark.parametrize("mode", MODES)
def test_depthwise_1d_examples(mode):
    g = _golden("wxb_1d_examples.json")
    e = g["weighted_sum_with_bias"]
    assert _dw1d(e["x"], [e["k"]], [e["bias"]], mode).ravel().tolist() == e["output"]
    e = g["spike_average"]
    third = np.float32(1.0) / np.float32(3.0)
    # one nonzero tap per window: fl(3 * fl(1/3)) = 1 in binary32
    assert _dw1d(e["x"], [[third] * 3], None, mode).ravel().tolist() == e["output"]
    for name in ("step_difference", "motif"):
        e = g[name]
        assert _dw1d(e["x"], [e["k"]], None, mode).ravel().tolist() == e["output"], name
    e = g["two_filters_with_bias"]
    y = _dw1d(e["x"], e["filters"], e["bias"], mode)
    assert y[0, :, 0, :].tolist() == e["output_per_filter"]


@pytest.mark.parametrize("mode", MODES)
def test_depthwise_2d_examples(mode):
    g = _golden("wxb_2d_examples.json")
    t = g["tiny_2d"]
    y = oracle.depthwise(np.array(t["image"], np.float32).reshape(1, 1, 3, 3),
                         np.array(t["filter"], np.float32).reshape(1, 2, 2), None, mode=mode)
    assert y[0, 0].tolist() == t["output"]
    s = g["sobel"]
    w = np.stack([np.array(s["gx"]), np.array(s["gy"])]).astype(np.float32)
    y = oracle.depthwise(np.array(s["image"], np.float32).reshape(1, 1, 6, 6), w, None, mult=2, mode=mode)
    assert y[0, 0].tolist() == s["gx_output"] and y[0, 1].tolist() == s["gy_output"]


# ------------------------------------------------------------------------------------------
# Depthwise: closed forms from IEEE binary32 rounding
# ------------------------------------------------------------------------------------------


@pytest.mark.parametrize("mode", MODES)
def test_depthwise_tap_order_row_major(mode):
    # Products 1e8, -1e8 (row 0) then 1, 0 (row 1). Row-major: 1e8, 0, 1, 1 -> 1.
    # Column-major would give 1e8, 1e8 (1e8+1 rounds back: ulp is 8), 0, 0 -> 0.
    x = np.array([[1e8, -1e8], [1.0, 0.0]], np.float32).reshape(1, 1, 2, 2)
    w = np.ones((1, 2, 2), np.float32)
    assert oracle.depthwise(x, w, None, mode=mode)[0, 0, 0, 0] == 1.0
    # 1-D: 1e8, -1e8, 1 in kx order gives 1; the reverse order would give 0.
    assert _dw1d([1e8, -1e8, 1.0], [[1, 1, 1]], None, mode).ravel().tolist() == [1.0]


def test_depthwise_exact_rounds_product_fast_fuses():
    # tap 0: -1 * (1 + 2**-11) = -(1 + 2**-11) exactly.
    # tap 1: (1 + 2**-12)**2 = 1 + 2**-11 + 2**-24, a tie between 1 + 2**-11 (even) and the
    # next float; exact mode rounds it to 1 + 2**-11 and the sum is +0. Fast mode keeps the
    # product unrounded inside the fused operation and returns 2**-24.
    a = np.float32(1 + 2.0 ** -12)
    x = np.array([1 + 2.0 ** -11, a], np.float32).reshape(1, 1, 1, 2)
    w = np.array([-1.0, a], np.float32).reshape(1, 1, 2)
    ye = oracle.depthwise(x, w, None, mode=oracle.DW_EXACT)
    yf = oracle.depthwise(x, w, None, mode=oracle.DW_FAST)
    assert _bits(ye).ravel().tolist() == [0]
    assert yf.ravel().tolist() == [2.0 ** -24]


@pytest.mark.parametrize("mode", MODES)
def test_depthwise_accumulator_starts_at_plus_zero(mode):
    # every product is -0; +0 + -0 = +0 in round-to-nearest, so outputs are +0, not -0
    x = np.zeros((1, 1, 4, 4), np.float32)
    w = -np.ones((1, 3, 3), np.float32)
    y = oracle.depthwise(x, w, None, pad=1, mode=mode)
    assert np.all(_bits(y) == 0)


def test_depthwise_padding_times_infinite_weight_is_canonical_nan():
    # pad=1, tap (0,0) weight +inf, all x = 2: windows whose tap (0,0) lands in the padding
    # (output row 0 or column 0) meet inf * 0 = NaN, rewritten as 0x7FC00000 in exact mode;
    # every other output is +inf. A bias does not change either.
    H = W = 5
    x = np.full((1, 1, H, W), 2.0, np.float32)
    w = np.ones((1, 3, 3), np.float32)
    w[0, 0, 0] = np.inf
    for bias in (None, np.array([0.5], np.float32)):
        y = oracle.depthwise(x, w, bias, pad=1, mode=oracle.DW_EXACT)[0, 0]
        b = _bits(y)
        for oy in range(H):
            for ox in range(W):
                if oy == 0 or ox == 0:
                    assert b[oy, ox] == 0x7FC00000
                else:
                    assert y[oy, ox] == np.inf
        yf = oracle.depthwise(x, w, bias, pad=1, mode=oracle.DW_FAST)[0, 0]
        assert np.isnan(yf[0, 0]) and np.isnan(yf[2, 0]) and yf[2, 2] == np.inf


def test_depthwise_nan_input_canonical_in_exact_mode():
    x = np.ones((1, 1, 3, 3), np.float32)
    x[0, 0, 1, 1] = struct.unpack("<f", struct.pack("<I", 0xFFC00001))[0]   # a NaN with payload
    w = np.ones((1, 1, 1), np.float32)
    y = oracle.depthwise(x, w, np.array([1.0], np.float32), mode=oracle.DW_EXACT)
    b = _bits(y)[0, 0]
    assert b[1, 1] == 0x7FC00000
    assert np.all(np.delete(y[0, 0].ravel(), 4) == 2.0)


def test_depthwise_denormals_kept():
    # 2**-70 * 2**-70 = 2**-140, a subnormal binary32 value (not flushed to zero)
    x = np.full((1, 1, 1, 1), 2.0 ** -70, np.float32)
    w = np.full((1, 1, 1), 2.0 ** -70, np.float32)
    for mode in MODES:
        y = oracle.depthwise(x, w, None, mode=mode)
        assert y.ravel()[0] == np.float32(2.0 ** -140) and y.ravel()[0] != 0


def test_depthwise_single_tap_is_rounded_product():
    # KH=KW=1, stride 1, no padding: y = fl(+0 + fl(w*x)) = fl(w*x) for nonzero products,
    # i.e. numpy's binary32 multiply; weight plane oc goes with input plane oc // mult.
    N, C, m, H, W = 2, 3, 2, 4, 5
    x = workloads.uniform(91, N * C * H * W, -1, 1).reshape(N, C, H, W)
    w = workloads.normal(92, C * m, 1.0).reshape(C * m, 1, 1)
    y = oracle.depthwise(x, w, None, mult=m, mode=oracle.DW_EXACT)
    for oc in range(C * m):
        ref = (w[oc, 0, 0] * x[:, oc // m]).astype(np.float32)
        assert np.array_equal(_bits(y[:, oc]), _bits(ref))


# ------------------------------------------------------------------------------------------
# Depthwise: brute-force grouped convolution (torch CPU, float64, groups = Cin)
# ------------------------------------------------------------------------------------------


def _tiny_cases(count, seed):
    rng_vals = workloads.splitmix64(seed, count * 9)
    cases = []
    for t in range(count):
        v = [int(z) for z in rng_vals[9 * t: 9 * t + 9]]
        N = 1 + v[0] % 2
        C = 1 + v[1] % 3
        m = 1 + v[2] % 3
        KH, KW = 1 + v[3] % 4, 1 + (v[3] >> 8) % 4
        s = 1 + v[4] % 3
        p = v[5] % 3
        d = 1 + v[6] % 2
        H = max(1, 1 + v[7] % 7)
        W = max(1, 1 + (v[7] >> 8) % 7)
        if (H + 2 * p - (d * (KH - 1) + 1)) < 0 or (W + 2 * p - (d * (KW - 1) + 1)) < 0:
            continue
        cases.append((N, C, m, H, W, KH, KW, s, p, d, v[8]))
    return cases


@pytest.mark.parametrize("case", _tiny_cases(60, 2024))
def test_depthwise_matches_torch_grouped_conv(case):
    N, C, m, H, W, KH, KW, s, p, d, seed = case
    x = workloads.uniform(seed, N * C * H * W, -1, 1).reshape(N, C, H, W)
    w = workloads.normal(seed + 1, C * m * KH * KW, 1.0).reshape(C * m, KH, KW)
    b = workloads.normal(seed + 2, C * m, 0.3)
    ref = torch.nn.functional.conv2d(torch.from_numpy(x.astype(np.float64)),
                                     torch.from_numpy(w.astype(np.float64)).reshape(C * m, 1, KH, KW),
                                     torch.from_numpy(b.astype(np.float64)), stride=s, padding=p,
                                     dilation=d, groups=C).numpy()
    bound = oracle.depthwise_absbound(x, w, b, mult=m, stride=s, pad=p, dil=d)
    for mode in MODES:
        y = oracle.depthwise(x, w, b, mult=m, stride=s, pad=p, dil=d, mode=mode)
        assert y.shape == ref.shape
        # float32 evaluation of at most 17 terms: well inside 2**-20 of the magnitude sum
        assert np.all(np.abs(y - ref) <= 2.0 ** -20 * bound), mode
    # integer inputs: every partial sum is an exact small integer, so the match is exact
    xi = _ints(seed + 3, (N, C, H, W))
    wi = _ints(seed + 4, (C * m, KH, KW))
    refi = torch.nn.functional.conv2d(torch.from_numpy(xi.astype(np.float64)),
                                      torch.from_numpy(wi.astype(np.float64)).reshape(C * m, 1, KH, KW),
                                      stride=s, padding=p, dilation=d, groups=C).numpy()
    for mode in MODES:
        assert np.array_equal(oracle.depthwise(xi, wi, None, mult=m, stride=s, pad=p, dil=d, mode=mode), refi)


def test_depthwise_output_size_matches_torch():
    for H in (1, 5, 7, 14, 28):
        for K in (1, 3, 5):
            for s in (1, 2, 3):
                for p in (0, 1, 2):
                    for d in (1, 2):
                        if H + 2 * p - (d * (K - 1) + 1) < 0:
                            continue
                        x = np.zeros((1, 1, H, H), np.float32)
                        w = np.zeros((1, K, K), np.float32)
                        y = oracle.depthwise(x, w, None, stride=s, pad=p, dil=d)
                        r = torch.nn.functional.conv2d(torch.zeros(1, 1, H, H), torch.zeros(1, 1, K, K),
                                                       stride=s, padding=p, dilation=d)
                        assert y.shape == tuple(r.shape)


def test_depthwise_many_taps_and_wide_stride():
    # more than 64 taps and a column stride above 8 still follow the one per-output order;
    # integer data makes the float64 library result exact
    for (K, s) in ((9, 1), (3, 9), (11, 2)):
        x = _ints(101 + K, (1, 2, 23, 25))
        w = _ints(201 + s, (2, K, K))
        ref = torch.nn.functional.conv2d(torch.from_numpy(x.astype(np.float64)),
                                         torch.from_numpy(w.astype(np.float64)).reshape(2, 1, K, K),
                                         stride=s, padding=K // 2, groups=2).numpy()
        for mode in MODES:
            assert np.array_equal(oracle.depthwise(x, w, None, stride=s, pad=K // 2, mode=mode), ref)


def test_depthwise_points_and_absbound():
    x = workloads.uniform(301, 2 * 3 * 9 * 8, -1, 1).reshape(2, 3, 9, 8)
    w = workloads.normal(302, 6 * 3 * 3, 1.0).reshape(6, 3, 3)
    b = workloads.normal(303, 6, 1.0)
    y = oracle.depthwise(x, w, b, mult=2, stride=2, pad=1)
    idx = np.array([0, 5, 33, y.size - 1])
    assert np.array_equal(_bits(oracle.depthwise_points(x, w, b, idx, mult=2, stride=2, pad=1)),
                          _bits(y.ravel()[idx]))
    bound = oracle.depthwise_absbound(x, w, b, mult=2, stride=2, pad=1)
    yabs = oracle.depthwise(np.abs(x), np.abs(w), np.abs(b), mult=2, stride=2, pad=1)
    assert np.allclose(bound, yabs, rtol=1e-6, atol=0)


# ------------------------------------------------------------------------------------------
# Storage bill of explicit im2col (DLSys notes, section 6): the arithmetic of the table
# ------------------------------------------------------------------------------------------


def test_storage_bill_table():
    g = _golden("dlsys14_storage_bill.json")
    s = g["shape"]
    Ho, Wo = s["H"] - s["K"] + 1, s["W"] - s["K"] + 1
    rows, cols = s["N"] * Ho * Wo, s["K"] * s["K"] * s["Cin"]
    assert (rows, cols) == (g["patch_matrix_rows"], g["patch_matrix_cols"])
    assert Ho * Wo * s["K"] ** 2 / (s["H"] * s["W"]) == g["rho"]
    assert rows * cols == g["values"]["patches"]
    assert math.isclose(rows * cols * 4 / 1e6, g["megabytes_f32"]["patches"])
    e = g["small_example"]
    assert ((e["H"] - e["K"] + 1) * (e["W"] - e["K"] + 1) * e["K"] ** 2) / (e["H"] * e["W"]) == e["ratio"]


# ------------------------------------------------------------------------------------------
# Depthwise followed by pointwise (the Wx+b page's section "Why variants matter")
# ------------------------------------------------------------------------------------------


@pytest.mark.parametrize("geom", [(3, 1, 1, 1), (3, 2, 1, 1), (5, 1, 2, 1), (3, 1, 2, 2), (1, 1, 0, 1)])
def test_dwpw_is_depthwise_then_channel_mixing_on_integers(geom):
    # small integers keep every stage exact (|d| <= 25*3*2 fits bf16's 8-bit significand), so
    # the block must equal torch's grouped depthwise conv followed by a 1x1 mixing, in float64
    K, s, p, d = geom
    N, C, H, W, Cout = 2, 6, 9, 8, 5
    x = workloads.int_uniform(101, N * C * H * W, -3, 3).reshape(N, C, H, W)
    w = workloads.int_uniform(102, C * K * K, -2, 2).reshape(C, K, K)
    F = workloads.int_uniform(103, C * Cout, -3, 3).reshape(C, Cout)
    bd = workloads.int_uniform(104, C, -4, 4)
    bp = workloads.int_uniform(105, Cout, -4, 4)
    for mode in (oracle.DW_EXACT, oracle.DW_FAST):
        y, a = oracle.dwpw(x, w, bd, F, bp, s, p, d, mode)
        t = torch.nn.functional.conv2d(torch.from_numpy(x.astype(np.float64)), torch.from_numpy(w.astype(np.float64))[:, None],
                                       torch.from_numpy(bd.astype(np.float64)), stride=s, padding=p, dilation=d, groups=C)
        ref = torch.einsum("nchw,co->nohw", t, torch.from_numpy(F.astype(np.float64))) + \
            torch.from_numpy(bp.astype(np.float64))[None, :, None, None]
        assert np.array_equal(y, ref.numpy())
        refa = torch.einsum("nchw,co->nohw", t.abs(), torch.from_numpy(np.abs(F).astype(np.float64))) + \
            torch.from_numpy(np.abs(bp).astype(np.float64))[None, :, None, None]
        assert np.array_equal(a, refa.numpy())


def test_dwpw_rounds_the_intermediate_to_bf16_nearest_even():
    # K = 1, w = 1, F = 1: y is the bf16 rounding of x itself
    vals = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -7 + 2 ** -9, -(1 + 2 ** -8), 65535.0, 2 ** -130],
                    np.float32)
    expect = [1.0, 1.015625, 1.0078125, -1.0, 65536.0, 2 ** -130]   # ties go to the even significand
    x = vals.reshape(1, 1, 1, -1)
    y, _ = oracle.dwpw(x, np.ones((1, 1, 1), np.float32), None, np.ones((1, 1), np.float32), None)
    assert y.reshape(-1).tolist() == expect


def test_dwpw_nan_intermediate_stays_nan():
    x = np.array([np.nan, 1.0], np.float32).reshape(1, 1, 1, 2)
    y, _ = oracle.dwpw(x, np.ones((1, 1, 1), np.float32), None, np.full((1, 2), 2.0, np.float32), None)
    assert np.isnan(y[0, :, 0, 0]).all() and (y[0, :, 0, 1] == 2.0).all()


@pytest.mark.parametrize("mode", [oracle.DW_EXACT, oracle.DW_FAST])
def test_dwpw_identity_mixing_gives_the_rounded_depthwise_output(mode):
    # F = I: the block returns the depthwise output of the page (its own, pinned oracle)
    # rounded to bf16, here by the input module's independent rounding routine
    N, C, H, W, K = 2, 4, 10, 9, 3
    x = workloads.uniform(106, N * C * H * W, -1, 1).reshape(N, C, H, W)
    w = workloads.normal(107, C * K * K, 1 / 3).reshape(C, K, K)
    b = workloads.normal(108, C, 0.3)
    y, _ = oracle.dwpw(x, w, b, np.eye(C, dtype=np.float32), None, 2, 1, 1, mode)
    dref = oracle.depthwise(x, w, b, mult=1, stride=2, pad=1, dil=1, mode=mode)
    assert np.array_equal(y, workloads.bf16_to_f32(workloads.bf16_bits(dref)).astype(np.float64))


def test_dwpw_points_are_the_full_output():
    N, C, H, W, K, Cout = 2, 5, 7, 6, 3, 7
    x = workloads.uniform(109, N * C * H * W, -1, 1).reshape(N, C, H, W)
    w = workloads.normal(110, C * K * K, 1 / 3).reshape(C, K, K)
    F = workloads.normal(111, C * Cout, 0.4).reshape(C, Cout)
    bp = workloads.normal(112, Cout, 0.3)
    y, a = oracle.dwpw(x, w, None, F, bp, 1, 1, 1)
    idx = (workloads.splitmix64(113, 200) % np.uint64(y.size)).astype(np.int64)
    yp, ap = oracle.dwpw_points(x, w, None, F, bp, idx, 1, 1, 1)
    assert np.array_equal(yp, y.reshape(-1)[idx]) and np.array_equal(ap, a.reshape(-1)[idx])


def test_dwpw_weight_counts_of_the_page():
    # "Why variants matter": 64 -> 64 channels, 3x3: dense 36,864 weights, depthwise plus
    # pointwise 4,672, about 7.9x fewer
    dense, factored = 64 * 64 * 3 * 3, 64 * 3 * 3 + 64 * 64
    assert (dense, factored) == (36864, 4672) and round(dense / factored, 1) == 7.9


# ------------------------------------------------------------------------------------------
# Padding that differs before and after an axis; the causal Conv1D ("Convolution Is Wx+b
# Moving Across a Signal", section "Find the same sum in CKE's C kernels": a frame's output may
# not read later frames, so the sequence is padded on the left only)
# ------------------------------------------------------------------------------------------


def test_causal_conv1d_is_numpy_correlation_of_the_left_padded_sequence():
    # every output is numpy's valid 1-D correlation of the sequence with dil*(K-1) zeros in
    # front, summed over the group's channels (dilation 1 and 2; a bias)
    for dil in (1, 2):
        L, Cin, Cout, K, groups = 17, 6, 4, 3, 2
        Cg, Og = Cin // groups, Cout // groups
        X = _ints(95 + dil, (2, 1, L, Cin))
        F = _ints(97 + dil, (1, K, Cg, Cout))
        b = np.array([1, -2, 3, 0], np.float32)
        P = dil * (K - 1)
        Y, _ = oracle.conv2d_grouped(X, F, b, dil=(1, dil), pad=((0, 0), (P, 0)), groups=groups)
        assert Y.shape == (2, 1, L, Cout)
        for n in range(2):
            for o in range(Cout):
                g = o // Og
                taps = np.zeros(P + 1)
                ref = np.full(L, float(b[o]))
                for c in range(Cg):
                    taps[::dil] = F[0, :, c, o]
                    xp = np.concatenate([np.zeros(P), X[n, 0, :, g * Cg + c].astype(np.float64)])
                    ref = ref + np.correlate(xp, taps, "valid")
                assert np.array_equal(Y[n, 0, :, o], ref)


def test_causal_conv1d_page_example():
    # the page's x = 1..5 with k = (2, 0, -1) and bias 1: the causal form adds two outputs in
    # front of the page's three (0, 1, 2), which read the zeros before the sequence
    e = _golden("wxb_1d_examples.json")["weighted_sum_with_bias"]
    X = np.array(e["x"], np.float32).reshape(1, 1, -1, 1)
    F = np.array(e["k"], np.float32).reshape(1, 3, 1, 1)
    Y, _ = oracle.conv2d_grouped(X, F, np.array([e["bias"]], np.float32), pad=((0, 0), (2, 0)))
    assert Y.ravel().tolist()[2:] == e["output"]
    assert Y.ravel().tolist()[:2] == [1 + (-1) * 1, 1 + (-1) * 2]


def test_causal_output_ignores_later_frames():
    # changing frames after t leaves outputs 0..t unchanged
    X = workloads.normal(99, 1 * 1 * 24 * 8, 1.0).reshape(1, 1, 24, 8)
    F = workloads.normal(100, 1 * 4 * 8 * 5, 0.3).reshape(1, 4, 8, 5)
    Y, _ = oracle.conv2d_grouped(X, F, pad=((0, 0), (3, 0)))
    for t in (0, 7, 22):
        X2 = X.copy()
        X2[:, :, t + 1:, :] = workloads.normal(101 + t, X2[:, :, t + 1:, :].size, 5.0).reshape(X2[:, :, t + 1:, :].shape)
        Y2, _ = oracle.conv2d_grouped(X2, F, pad=((0, 0), (3, 0)))
        assert np.array_equal(Y2[:, :, :t + 1], Y[:, :, :t + 1])
        assert not np.array_equal(Y2[:, :, t + 1:], Y[:, :, t + 1:])


@pytest.mark.parametrize("pads", [((1, 0), (0, 2)), ((0, 2), (3, 1)), ((2, 1), (0, 0))])
def test_asymmetric_padding_matches_torch_pad_then_convolve(pads):
    # explicit zero padding (torch.nn.functional.pad) followed by an unpadded convolution
    (pt, pb), (pl, pr) = pads
    X = workloads.normal(102, 2 * 9 * 11 * 6, 1.0).reshape(2, 9, 11, 6)
    F = workloads.normal(103, 3 * 2 * 3 * 4, 0.3).reshape(3, 2, 3, 4)
    b = workloads.normal(104, 4, 0.5)
    Y, A = oracle.conv2d_grouped(X, F, b, stride=(2, 1), pad=pads, dil=(1, 2), groups=2)
    x = torch.from_numpy(np.asarray(X, dtype=np.float64)).permute(0, 3, 1, 2)
    x = torch.nn.functional.pad(x, (pl, pr, pt, pb))
    f = torch.from_numpy(np.asarray(F, dtype=np.float64)).permute(3, 2, 0, 1)
    ref = torch.nn.functional.conv2d(x, f, torch.from_numpy(np.asarray(b, dtype=np.float64)), stride=(2, 1),
                                     dilation=(1, 2), groups=2).permute(0, 2, 3, 1).numpy()
    assert Y.shape == ref.shape
    assert np.all(np.abs(Y - ref) <= 1e-13 * A)
    idx = (workloads.splitmix64(105, 200) % np.uint64(Y.size)).astype(np.int64)
    y, a = oracle.conv2d_grouped_points(X, F, idx, b, stride=(2, 1), pad=pads, dil=(1, 2), groups=2)
    assert np.array_equal(y, Y.reshape(-1)[idx]) and np.array_equal(a, A.reshape(-1)[idx])
