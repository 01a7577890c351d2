"""Depthwise convolution on the GPU against the CPU oracle, through the C ABI.

Exact mode must be bit-identical to the oracle. Fast mode must satisfy
|y - y_ref| <= 1e-6 * (sum over taps |w*x| + |bias|) per output (the relative bound, scaled
by the magnitude of the terms so outputs near zero are not judged by a meaningless ratio);
both sides use a correctly rounded fused multiply-add in the same order, so the tests also
expect bit identity there. NaN outputs compare as NaN on both sides in fast mode.
"""
import json
import os
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.conftest import GOLDEN

pytestmark = pytest.mark.gpu

MODES = [oracle.DW_EXACT, oracle.DW_FAST]


@pytest.fixture(scope="module")
def cb(cuda):
    import cnn_convolution_nhwc_b200 as cb
    return cb


def _bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def _gpu(cb, x, w, b, stride=1, pad=0, dil=1, mode=0, tile=None):
    old = os.environ.get("CONV_B200_DW_TILE")
    if tile is not None:
        os.environ["CONV_B200_DW_TILE"] = tile
    try:
        y = cb.depthwise_fwd(torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda(),
                             torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda(),
                             None if b is None else torch.from_numpy(np.ascontiguousarray(b, np.float32)).cuda(),
                             stride=stride, pad=pad, dil=dil, mode=mode)
        out = y.cpu().numpy()
    finally:
        if tile is not None:
            if old is None:
                del os.environ["CONV_B200_DW_TILE"]
            else:
                os.environ["CONV_B200_DW_TILE"] = old
    assert cb.conv_device_status() == cb.CONV_OK
    return out


def _compare(y, x, w, b, mult, stride, pad, dil, mode):
    ref = oracle.depthwise(x, w, b, mult=mult, stride=stride, pad=pad, dil=dil, mode=mode)
    assert y.shape == ref.shape
    if mode == oracle.DW_EXACT:
        same = _bits(y) == _bits(ref)
        assert same.all(), f"{(~same).sum()} of {y.size} outputs differ in exact mode"
    else:
        bound = oracle.depthwise_absbound(x, w, b, mult=mult, stride=stride, pad=pad, dil=dil)
        both_nan = np.isnan(y) & np.isnan(ref)
        # equal values pass as such (infinities of the same sign have no finite difference)
        ok = both_nan | (y == ref) | (np.abs(y.astype(np.float64) - ref) <= 1e-6 * bound)
        assert ok.all(), f"{(~ok).sum()} fast-mode outputs out of tolerance"
        same = (_bits(y) == _bits(ref)) | both_nan
        assert same.all(), f"fast mode: {(~same).sum()} outputs not bit-identical"


@pytest.mark.parametrize("mode", MODES, ids=["exact", "fast"])
@pytest.mark.parametrize("case", workloads.DW_SWEEP, ids=lambda c: c.name)
def test_sweep_full_output(cb, case, mode):
    x, w, b = workloads.depthwise_inputs(case)
    y = _gpu(cb, x, w, b, case.stride, case.pad, case.dil, mode)
    _compare(y, x, w, b, case.mult, case.stride, case.pad, case.dil, mode)


@pytest.mark.parametrize("mode", MODES, ids=["exact", "fast"])
def test_page_examples(cb, mode):
    g = json.load(open(os.path.join(GOLDEN, "wxb_1d_examples.json")))
    e = g["weighted_sum_with_bias"]
    y = _gpu(cb, np.array(e["x"]).reshape(1, 1, 1, -1), np.array(e["k"]).reshape(1, 1, -1), [e["bias"]], mode=mode)
    assert y.ravel().tolist() == e["output"]
    third = np.float32(1) / np.float32(3)
    y = _gpu(cb, np.array(g["spike_average"]["x"]).reshape(1, 1, 1, -1), np.full((1, 1, 3), third), None, mode=mode)
    assert y.ravel().tolist() == g["spike_average"]["output"]
    for name in ("step_difference", "motif"):
        e = g[name]
        y = _gpu(cb, np.array(e["x"]).reshape(1, 1, 1, -1), np.array(e["k"]).reshape(1, 1, -1), None, mode=mode)
        assert y.ravel().tolist() == e["output"], name
    e = g["two_filters_with_bias"]
    y = _gpu(cb, np.array(e["x"]).reshape(1, 1, 1, -1), np.array(e["filters"]).reshape(2, 1, 3), e["bias"], mode=mode)
    assert y[0, :, 0, :].tolist() == e["output_per_filter"]
    s = json.load(open(os.path.join(GOLDEN, "wxb_2d_examples.json")))
    t = s["tiny_2d"]
    y = _gpu(cb, np.array(t["image"]).reshape(1, 1, 3, 3), np.array(t["filter"]).reshape(1, 2, 2), None, mode=mode)
    assert y[0, 0].tolist() == t["output"]
    so = s["sobel"]
    y = _gpu(cb, np.array(so["image"]).reshape(1, 1, 6, 6), np.stack([so["gx"], so["gy"]]), None, mode=mode)
    assert y[0, 0].tolist() == so["gx_output"] and y[0, 1].tolist() == so["gy_output"]


def test_ieee_closed_forms(cb):
    # row-major tap order: products 1e8, -1e8, 1, 0 give 1 (column-major would give 0)
    x = np.array([[1e8, -1e8], [1.0, 0.0]], np.float32).reshape(1, 1, 2, 2)
    for mode in MODES:
        assert _gpu(cb, x, np.ones((1, 2, 2)), None, mode=mode).ravel().tolist() == [1.0]
    # exact rounds the product (tie to even) and cancels to +0; fast keeps 2**-24
    a = np.float32(1 + 2.0 ** -12)
    x = np.array([1 + 2.0 ** -11, a], np.float32).reshape(1, 1, 1, 2)
    w = np.array([-1.0, a], np.float32).reshape(1, 1, 2)
    assert _bits(_gpu(cb, x, w, None, mode=0)).ravel().tolist() == [0]
    assert _gpu(cb, x, w, None, mode=1).ravel().tolist() == [2.0 ** -24]
    # accumulator starts at +0: all products -0 give +0
    for mode in MODES:
        y = _gpu(cb, np.zeros((1, 1, 4, 4)), -np.ones((1, 3, 3)), None, pad=1, mode=mode)
        assert np.all(_bits(y) == 0)
    # denormal products are kept
    for mode in MODES:
        y = _gpu(cb, np.full((1, 1, 1, 1), 2.0 ** -70), np.full((1, 1, 1), 2.0 ** -70), None, mode=mode)
        assert y.ravel()[0] == np.float32(2.0 ** -140)


def test_padding_nan_rule(cb):
    H = W = 5
    x = np.full((1, 1, H, W), 2.0, np.float32)
    w = np.ones((1, 3, 3), np.float32)
    w[0, 0, 0] = np.inf
    for bias in (None, np.array([0.5], np.float32)):
        y = _gpu(cb, x, w, bias, pad=1, mode=0)[0, 0]
        b = _bits(y)
        for oy in range(H):
            for ox in range(W):
                if oy == 0 or ox == 0:
                    assert b[oy, ox] == 0x7FC00000
                else:
                    assert y[oy, ox] == np.inf
        yf = _gpu(cb, x, w, bias, pad=1, mode=1)[0, 0]
        assert np.isnan(yf[0, 0]) and np.isnan(yf[3, 0]) and yf[2, 2] == np.inf
    nan = struct.unpack("<f", struct.pack("<I", 0xFFC00001))[0]
    x = np.ones((2, 3, 6, 7), np.float32)
    x[1, 2, 3, 4] = nan
    w = workloads.normal(5, 3 * 9, 1.0).reshape(3, 3, 3)
    for mode in MODES:
        y = _gpu(cb, x, w, np.zeros(3, np.float32), pad=1, mode=mode)
        _compare(y, x, w, np.zeros(3, np.float32), 1, 1, 1, 1, mode)


def _tiny(count, seed):
    v = workloads.splitmix64(seed, count * 9)
    out = []
    for t in range(count):
        z = [int(q) for q in v[9 * t: 9 * t + 9]]
        N, C, m = 1 + z[0] % 3, 1 + z[1] % 5, 1 + z[2] % 3
        KH, KW = 1 + z[3] % 5, 1 + (z[3] >> 8) % 5
        s, p, d = 1 + z[4] % 3, z[5] % 3, 1 + z[6] % 2
        H, W = 1 + z[7] % 23, 1 + (z[7] >> 8) % 23
        if H + 2 * p < d * (KH - 1) + 1 or W + 2 * p < d * (KW - 1) + 1:
            continue
        out.append((N, C, m, H, W, KH, KW, s, p, d, z[8]))
    return out


@pytest.mark.parametrize("case", _tiny(40, 7), ids=lambda c: "_".join(map(str, c[:10])))
def test_random_small_shapes(cb, case):
    N, C, m, H, W, KH, KW, s, p, d, seed = case
    x = workloads.uniform(seed, N * C * H * W, -1, 1).reshape(N, C, H, W)
    w = workloads.normal(seed + 1, C * m * KH * KW, 1.0).reshape(C * m, KH, KW)
    b = workloads.normal(seed + 2, C * m, 0.3) if seed % 2 else None
    for mode in MODES:
        _compare(_gpu(cb, x, w, b, s, p, d, mode), x, w, b, m, s, p, d, mode)


@pytest.mark.parametrize("K,s,d,m", [(9, 1, 1, 1), (3, 9, 1, 2), (11, 2, 1, 1), (3, 3, 2, 3), (5, 1, 3, 2)])
def test_many_taps_wide_stride_dilation(cb, K, s, d, m):
    N, C, H, W = 2, 6, 37, 45
    x = workloads.uniform(K * 100 + s, N * C * H * W, -1, 1).reshape(N, C, H, W)
    w = workloads.normal(K + s, C * m * K * K, 1.0 / K).reshape(C * m, K, K)
    b = workloads.normal(K, C * m, 0.3)
    pad = (d * (K - 1)) // 2
    for mode in MODES:
        _compare(_gpu(cb, x, w, b, s, pad, d, mode), x, w, b, m, s, pad, d, mode)


@pytest.mark.parametrize("tile", ["1,1,1", "1,3,7", "3,100,100", "64,1000,1000", "2,5,1000", "7,2,16"])
def test_results_independent_of_tiling(cb, tile):
    # the page's determinism property: each output has one order, so any job shape gives
    # the same bits
    case = workloads.DepthwiseCase("t", 3, 5, 2, 19, 23, 3, 5, 2, 2, 1, True, 3)
    x, w, b = workloads.depthwise_inputs(case)
    for mode in MODES:
        base = _gpu(cb, x, w, b, case.stride, case.pad, case.dil, mode)
        y = _gpu(cb, x, w, b, case.stride, case.pad, case.dil, mode, tile=tile)
        assert np.array_equal(_bits(y), _bits(base))
        _compare(y, x, w, b, case.mult, case.stride, case.pad, case.dil, mode)


def _with_env(name, value, fn):
    old = os.environ.get(name)
    os.environ[name] = value
    try:
        return fn()
    finally:
        if old is None:
            del os.environ[name]
        else:
            os.environ[name] = old


@pytest.mark.parametrize("case", workloads.DW_SWEEP, ids=lambda c: c.name)
def test_register_and_shared_kernels_identical(cb, case):
    # the register-window kernel (the default for these shapes) and the shared-memory kernel
    # compute every output in the same order: identical bits, both equal to the oracle
    small = workloads.DepthwiseCase(case.name, 2, case.C, 2 if case.C <= 72 else 1, case.H, case.W, case.KH,
                                    case.KW, case.stride, case.pad, case.dil, True, 11)
    x, w, b = workloads.depthwise_inputs(small)
    for mode in MODES:
        yr = _with_env("CONV_B200_DW_KERNEL", "reg",
                       lambda: _gpu(cb, x, w, b, small.stride, small.pad, small.dil, mode))
        ys = _with_env("CONV_B200_DW_KERNEL", "smem",
                       lambda: _gpu(cb, x, w, b, small.stride, small.pad, small.dil, mode))
        assert np.array_equal(_bits(yr), _bits(ys))
        _compare(yr, x, w, b, small.mult, small.stride, small.pad, small.dil, mode)


def test_register_kernel_refuses_other_shapes(cb):
    x = np.ones((1, 2, 9, 9), np.float32)
    w = np.ones((2, 3, 3), np.float32)
    with pytest.raises(cb.ConvError) as e:
        _with_env("CONV_B200_DW_KERNEL", "reg", lambda: _gpu(cb, x, w, None, 1, 0, 1, 0))   # pad 0
    assert e.value.code == cb.CONV_ERR_UNSUPPORTED


@pytest.mark.parametrize("case", workloads.DW_SWEEP, ids=lambda c: c.name)
def test_tma_staged_and_shared_kernels_identical(cb, case):
    # the TMA-staged kernel (the default for multiplier 1) against the shared-memory kernel:
    # identical bits, both equal to the oracle; batch 3 leaves a ragged last job
    small = workloads.DepthwiseCase(case.name, 3, case.C, 1, case.H, case.W, case.KH, case.KW, case.stride,
                                    case.pad, case.dil, True, 12)
    x, w, b = workloads.depthwise_inputs(small)
    for mode in MODES:
        yt = _with_env("CONV_B200_DW_KERNEL", "tma",
                       lambda: _gpu(cb, x, w, b, small.stride, small.pad, small.dil, mode))
        ys = _with_env("CONV_B200_DW_KERNEL", "smem",
                       lambda: _gpu(cb, x, w, b, small.stride, small.pad, small.dil, mode))
        assert np.array_equal(_bits(yt), _bits(ys))
        _compare(yt, x, w, b, 1, small.stride, small.pad, small.dil, mode)


# (N, C, H, W, K, S): TMA bands with a ragged last band; TMA bands with fewer planes than a
# warp's group (the box's missing planes arrive as zeros); a small plane split in two bands;
# whole planes through cp.async (rows not 16-byte multiples), with a partial last group
TMA_SHAPES = [(2, 5, 36, 20, 3, 1), (1, 7, 13, 12, 5, 2), (3, 10, 8, 8, 3, 1), (2, 6, 10, 10, 3, 2),
              (1, 3, 7, 7, 5, 1), (2, 3, 14, 14, 3, 1), (1, 2, 40, 24, 5, 2)]


@pytest.mark.parametrize("shape", TMA_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_tma_staged_job_modes(cb, shape):
    N, C, H, W, K, S = shape
    case = workloads.DepthwiseCase("tma", N, C, 1, H, W, K, K, S, (K - 1) // 2, 1, True, 13)
    x, w, b = workloads.depthwise_inputs(case)
    for mode in MODES:
        yt = _with_env("CONV_B200_DW_KERNEL", "tma", lambda: _gpu(cb, x, w, b, S, case.pad, 1, mode))
        assert cb.conv_last_kernel() == "depthwise_tma_kernel"
        ys = _with_env("CONV_B200_DW_KERNEL", "smem", lambda: _gpu(cb, x, w, b, S, case.pad, 1, mode))
        assert cb.conv_last_kernel() == "depthwise_kernel"
        assert np.array_equal(_bits(yt), _bits(ys))
        _compare(yt, x, w, b, 1, S, case.pad, 1, mode)


def test_dispatcher_choices(cb):
    x, w, b = workloads.depthwise_inputs(
        workloads.DepthwiseCase("d", 1, 8, 1, 16, 16, 3, 3, 1, 1, 1, True, 14))
    _gpu(cb, x, w, b, 1, 1, 1, 0)
    assert cb.conv_last_kernel() == "depthwise_tma_kernel"     # multiplier 1, K 3, 'same' padding
    x2, w2, b2 = workloads.depthwise_inputs(
        workloads.DepthwiseCase("d", 1, 8, 2, 16, 16, 3, 3, 1, 1, 1, True, 14))
    _gpu(cb, x2, w2, b2, 1, 1, 1, 0)
    assert cb.conv_last_kernel() == "depthwise_reg_kernel"     # multiplier 2
    _gpu(cb, x, w, b, 1, 0, 1, 0)
    assert cb.conv_last_kernel() == "depthwise_kernel"         # no padding


def test_forced_tma_refuses_unaligned_planes(cb):
    # rows of 66 floats are not 16-byte multiples, and a 64 x 66 plane is too large to stage
    # whole, so the staged kernel is not eligible
    x = np.ones((1, 2, 64, 66), np.float32)
    w = np.ones((2, 3, 3), np.float32)
    with pytest.raises(cb.ConvError) as e:
        _with_env("CONV_B200_DW_KERNEL", "tma", lambda: _gpu(cb, x, w, None, 1, 1, 1, 0))
    assert e.value.code == cb.CONV_ERR_UNSUPPORTED


# (N, C, HW, K, S): 7x7 and 14x14 planes, a lane per plane; plane counts that leave a partial
# last job, and (7x7, 33 planes) a last job whose size is not a 16-byte multiple
PLANE_SHAPES = [(1, 33, 7, 5, 1), (2, 21, 7, 3, 1), (3, 5, 7, 3, 2), (1, 40, 7, 5, 2), (2, 9, 14, 3, 1),
                (1, 17, 14, 5, 1), (2, 12, 14, 3, 2), (1, 7, 14, 5, 2)]


@pytest.mark.parametrize("shape", PLANE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_plane_kernel(cb, shape):
    N, C, HW, K, S = shape
    case = workloads.DepthwiseCase("plane", N, C, 1, HW, HW, K, K, S, (K - 1) // 2, 1, True, 17)
    x, w, b = workloads.depthwise_inputs(case)
    for mode in MODES:
        yp = _gpu(cb, x, w, b, S, case.pad, 1, mode)
        assert cb.conv_last_kernel() == "depthwise_plane_kernel"
        ys = _with_env("CONV_B200_DW_KERNEL", "smem", lambda: _gpu(cb, x, w, b, S, case.pad, 1, mode))
        assert np.array_equal(_bits(yp), _bits(ys))
        _compare(yp, x, w, b, 1, S, case.pad, 1, mode)
        yn = _gpu(cb, x, w, None, S, case.pad, 1, mode)          # no bias
        _compare(yn, x, w, None, 1, S, case.pad, 1, mode)


# (N, C, H, K, S, kernel): the production kernels -- planes of 7x7 and 14x14 (a lane per
# plane), rows that are 16-byte multiples (one TMA box with the padding zeros written by the
# copy engine) and rows that are not (whole planes by cp.async into pre-zeroed buffers)
NAN_RULE_SHAPES = [(2, 9, 7, 3, 1, "plane"), (1, 21, 7, 5, 1, "plane"), (2, 6, 14, 3, 2, "plane"),
                   (1, 5, 14, 5, 1, "plane"), (2, 3, 16, 3, 1, "tma"), (1, 4, 28, 5, 1, "tma"),
                   (2, 3, 20, 5, 2, "tma"), (1, 3, 14, 3, 1, "tma")]


@pytest.mark.parametrize("shape", NAN_RULE_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + "-" + s[5])
def test_padding_nan_rule_production_kernels(cb, shape):
    # OneModel "Depthwise convolution", "What each output is": padding is a real zero that is
    # multiplied, so an infinite weight meeting padding gives NaN, and exact mode rewrites every
    # NaN result as 0x7FC00000; an input NaN with another payload must come out canonical too
    N, C, H, K, S, kernel = shape
    case = workloads.DepthwiseCase("nan", N, C, 1, H, H, K, K, S, (K - 1) // 2, 1, True, 19)
    x, w, b = workloads.depthwise_inputs(case)
    w = w.copy()
    w[0, 0, 0] = np.inf                 # plane 0: top-left tap meets the top row and left column of padding
    w[C - 1, K - 1, K - 1] = -np.inf    # last plane: bottom-right tap
    x = x.copy()
    x.reshape(-1)[H * H + 2 * H + 3] = np.frombuffer(struct.pack("<I", 0xFFC00001), np.float32)[0]   # plane 1
    for mode in MODES:
        y = _with_env("CONV_B200_DW_KERNEL", kernel, lambda: _gpu(cb, x, w, b, S, case.pad, 1, mode))
        assert cb.conv_last_kernel() == f"depthwise_{kernel}_kernel"
        _compare(y, x, w, b, 1, S, case.pad, 1, mode)
        ref = oracle.depthwise(x, w, b, mult=1, stride=S, pad=case.pad, dil=1, mode=mode)
        assert np.isnan(ref).any() and np.isinf(ref).any()    # the planted values reach the outputs
        if mode == oracle.DW_EXACT:
            assert set(_bits(y)[np.isnan(y)].tolist()) == {0x7FC00000}


# (N, C, H, K, S, kernel): the packed-pair production kernels
ROUNDING_SHAPES = [(1, 8, 7, 3, 1, "plane"), (1, 8, 14, 3, 1, "plane"), (1, 8, 7, 5, 1, "plane"),
                   (1, 8, 16, 3, 1, "tma"), (1, 8, 28, 5, 1, "tma")]


def rounding_case(C, H, K):
    """Channel 3, output (3, 3): two products, -(1 + 2^-11) and a^2 with a = 1 + 2^-12. Rounded
    separately they cancel to +0; fused (one rounding) they leave 2^-24. Channel 0: zero input
    and negative taps, every product -0, every output +0. Returns x, w, the output position."""
    pad = (K - 1) // 2
    a = np.float32(1 + 2.0 ** -12)
    x = np.zeros((1, C, H, H), np.float32)
    w = workloads.normal(31, C * K * K, 0.5).reshape(C, K, K).astype(np.float32)
    w[0] = -1.0
    w[3] = 0.0
    w[3, 0, 0], w[3, 0, 1] = -1.0, a
    oy = ox = 3
    x[0, 3, oy - pad, ox - pad] = np.float32(1 + 2.0 ** -11)
    x[0, 3, oy - pad, ox - pad + 1] = a
    return x, w, (oy, ox)


@pytest.mark.parametrize("shape", ROUNDING_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + "-" + s[5])
def test_exact_mode_rounds_each_product_production_kernels(cb, shape):
    # OneModel "Depthwise convolution", "What each output is": exact mode rounds every product
    # and every sum; the accumulator starts at +0. Pinned on the kernels that compute two
    # outputs per packed instruction, where a fused product would go unnoticed on random data
    N, C, H, K, S, kernel = shape
    x, w, (oy, ox) = rounding_case(C, H, K)
    pad = (K - 1) // 2
    for mode in MODES:
        y = _with_env("CONV_B200_DW_KERNEL", kernel, lambda: _gpu(cb, x, w, None, S, pad, 1, mode))
        assert cb.conv_last_kernel() == f"depthwise_{kernel}_kernel"
        _compare(y, x, w, None, 1, S, pad, 1, mode)
        assert np.all(_bits(y[0, 0]) == 0)          # all products -0: +0
        if mode == oracle.DW_EXACT:
            assert _bits(y[0, 3, oy, ox]) == 0      # rounded separately: exact cancellation
        else:
            assert y[0, 3, oy, ox] == np.float32(2.0 ** -24)   # one rounding


@pytest.mark.parametrize("ring", ["2", "3"])
@pytest.mark.parametrize("shape", [(2, 16, 56, 3, 2), (1, 8, 28, 5, 1), (2, 4, 112, 3, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_tma_staggered_first_copies(cb, shape, ring):
    # the TMA kernel's first copies with and without the stagger (a warp's first job alone,
    # the rest of its ring after it), over rings of 2 and 3 buffers: the same bits, the oracle's
    N, C, H, K, S = shape
    case = workloads.DepthwiseCase("stagger", N, C, 1, H, H, K, K, S, (K - 1) // 2, 1, True, 23)
    x, w, b = workloads.depthwise_inputs(case)
    old = {k: os.environ.get(k) for k in ("CONV_B200_DW_KERNEL", "CONV_B200_DW_RING", "CONV_B200_DW_STAGGER")}
    try:
        os.environ["CONV_B200_DW_KERNEL"] = "tma"
        os.environ["CONV_B200_DW_RING"] = ring
        for mode in MODES:
            ys = []
            for st in ("0", "1"):
                os.environ["CONV_B200_DW_STAGGER"] = st
                ys.append(_gpu(cb, x, w, b, S, case.pad, 1, mode))
                assert cb.conv_last_kernel() == "depthwise_tma_kernel"
            assert np.array_equal(_bits(ys[0]), _bits(ys[1]))
            _compare(ys[1], x, w, b, 1, S, case.pad, 1, mode)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
