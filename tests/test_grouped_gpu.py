"""GPU parity of conv2d_nhwc_fwd_grouped (channel groups, KH x KW filters, per-axis stride,
padding and dilation, Conv1D as H = 1) against the float64 grouped oracle.

Every case goes through the C ABI with seeded bf16 operands; the bar is the dense tolerance
|y - y_ref| <= 4e-3 * (sum|x||w| + |b|) per output.
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


def _case(N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias, seed=0, pad_w_end=-1):
    return workloads.DenseCase("t", N, H, W, Cin, Cout, KH, "bf16", "normal", seed, stride=s[0], pad=p[0], dil=d[0],
                               bias=bias, groups=groups, KW=KW, stride_w=s[1], pad_w=p[1], dil_w=d[1],
                               pad_w_end=pad_w_end)


def _geom(c):
    return (c.stride, c.sw), c.pads, (c.dil, c.dw)


def _run(cb, c, Xb, Fb, b, env=None):
    old = os.environ.get("CONV_B200_DENSE")
    if env is not None:
        os.environ["CONV_B200_DENSE"] = env
    try:
        X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
        F = torch.from_numpy(Fb.view(np.int16)).view(torch.bfloat16).cuda()
        bt = None if b is None else torch.from_numpy(np.ascontiguousarray(b, np.float32)).cuda()
        s, p, d = _geom(c)
        Y = cb.conv2d_nhwc_fwd_grouped(X, F, bt, stride=s, pad=p, dil=d, groups=c.groups)
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


def _check(c, y, Xb, Fb, b):
    s, p, d = _geom(c)
    ref, absum = oracle.conv2d_grouped(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), b, s, p, d, c.groups)
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    bad = np.abs(y - ref) > TOL * absum
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance"


# (N, H, W, Cin, Cout, KH, KW, stride, pad, dil, groups, bias, kernel expected by default)
CASES = [
    (4, 28, 28, 128, 128, 3, 3, (1, 1), (1, 1), (1, 1), 2, True, "dense_halo_pad_kernel"),  # two 64-wide groups
    (2, 28, 28, 256, 256, 3, 3, (2, 2), (1, 1), (1, 1), 4, True, "dense_tc_kernel"),       # RegNet-style, stride 2
    (2, 16, 16, 256, 256, 3, 3, (1, 1), (1, 1), (1, 1), 16, False, "dense_tc_kernel"),     # 16 groups: two launches
    (1, 20, 20, 256, 256, 3, 3, (1, 1), (1, 1), (1, 1), 32, True, "dense_tc_kernel"),      # 8-channel groups
    (2, 24, 20, 96, 192, 3, 3, (1, 1), (2, 2), (2, 1), 3, True, "dense_tc_kernel"),        # dilation per axis, ragged N tile
    (4, 17, 17, 64, 64, 1, 7, (1, 1), (0, 3), (1, 1), 1, True, "dense_halo_pad_kernel"),   # 1x7, one group
    (4, 17, 17, 64, 96, 7, 1, (1, 1), (3, 0), (1, 1), 1, False, "dense_halo_pad_kernel"),  # 7x1
    (4, 30, 30, 64, 64, 3, 1, (2, 1), (1, 0), (1, 1), 1, True, "dense_tc_kernel"),         # stride per axis
    (2, 1, 3000, 80, 512, 1, 3, (1, 1), (0, 1), (1, 1), 1, True, "dense_tc_kernel"),      # Conv1D, 80 channels
    (2, 1, 3000, 256, 256, 1, 3, (1, 2), (0, 1), (1, 1), 1, True, "dense_tc_kernel"),     # Conv1D, stride 2
    (2, 1, 1000, 128, 128, 1, 5, (1, 1), (0, 4), (1, 2), 4, True, "dense_tc_kernel"),     # grouped dilated Conv1D
    (2, 9, 11, 12, 24, 3, 2, (1, 2), (1, 0), (1, 1), 3, True, "dense_direct_kernel"),     # 4-channel groups
    (2, 1, 50, 8, 8, 1, 3, (1, 1), (0, 1), (1, 1), 2, False, "dense_direct_kernel"),      # tiny Conv1D
]


def _ids(c):
    return "N{}H{}W{}C{}-{}k{}x{}s{}p{}d{}g{}".format(*c[:7], *["".join(map(str, t)) for t in c[7:10]], c[10]) + \
        ("b" if c[11] else "")


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_grouped_geometry(cb, case):
    N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias, expected = case
    c = _case(N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias, seed=abs(hash(case[:11])) % 1000)
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y, kernel = _run(cb, c, Xb, Fb, b)
    _check(c, y, Xb, Fb, b)
    assert kernel == expected


@pytest.mark.parametrize("case", [CASES[1], CASES[4], CASES[8]], ids=_ids)
def test_tensor_core_and_direct_paths_agree(cb, case):
    N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias, _ = case
    c = _case(N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias, seed=5)
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y_tc, k_tc = _run(cb, c, Xb, Fb, b)
    y_cc, k_cc = _run(cb, c, Xb, Fb, b, env="direct")
    assert (k_tc, k_cc) == ("dense_tc_kernel", "dense_direct_kernel")
    _check(c, y_tc, Xb, Fb, b)
    _check(c, y_cc, Xb, Fb, b)


# Stride 1 with whole 64-channel blocks per group: the padded halo kernel by default (one 4-D
# tensor copy of a zero-padded window per tile), the im2col kernel when forced; both against the
# oracle. Two 64-wide groups with a bias; one group with "same" padding; dilation 2; an image
# wider than one window (three column bands); 40-wide groups (a partial bias chunk, a partial
# column tile); 128-wide groups (two 64-column boxes per filter slot); a 1 x 5 Conv1D
PAD_HALO = [   # inputs of at least 128 KiB, so that the im2col kernel can be forced for comparison
    (2, 20, 20, 128, 128, 3, 3, (1, 1), (1, 1), (1, 1), 2, True),
    (2, 30, 30, 64, 64, 3, 3, (1, 1), (1, 1), (1, 1), 1, True),
    (3, 24, 20, 64, 64, 3, 3, (1, 1), (2, 2), (2, 2), 1, False),
    (1, 4, 300, 64, 64, 3, 3, (1, 1), (1, 1), (1, 1), 1, True),
    (4, 14, 14, 128, 80, 3, 3, (1, 1), (1, 1), (1, 1), 2, True),
    (4, 12, 12, 128, 256, 3, 3, (1, 1), (1, 1), (1, 1), 2, True),
    (2, 1, 700, 64, 64, 1, 5, (1, 1), (0, 2), (1, 1), 1, True),
]


@pytest.mark.parametrize("case", PAD_HALO, ids=_ids)
def test_padded_halo_kernel(cb, case):
    N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias = case
    c = _case(N, H, W, Cin, Cout, KH, KW, s, p, d, groups, bias, seed=sum(case[:7]) + 13)
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y, kernel = _run(cb, c, Xb, Fb, b)
    assert kernel == "dense_halo_pad_kernel"
    _check(c, y, Xb, Fb, b)
    y2, kernel2 = _run(cb, c, Xb, Fb, b, env="bn128")
    assert kernel2 == "dense_tc_kernel"
    _check(c, y2, Xb, Fb, b)
    y3, kernel3 = _run(cb, c, Xb, Fb, b, env="halo")
    assert kernel3 == "dense_halo_pad_kernel" and np.array_equal(y3, y)


# The im2col kernel at tile widths 128 and 256 can run as CTA pairs (each CTA stages half of
# every filter slot; M = 256 MMAs across both; forced here): the same MMA sequence per output as
# one CTA per tile, so identical bits. Stride 2 with 128-wide tiles; a causal Conv1D with 256-wide tiles and a
# ragged last pair (the odd CTA's rows past the end); a dilated 5x5
TC_PAIR = [
    ((2, 28, 28, 64, 128, 3, 3, (2, 2), (1, 1), (1, 1), 1, True), "bn128"),
    ((2, 1, 999, 256, 512, 1, 3, (1, 1), (0, 2), (1, 1), 1, True), "bn256"),
    ((2, 24, 24, 96, 256, 5, 5, (1, 1), (4, 4), (2, 2), 1, False), "bn256"),
]


@pytest.mark.parametrize("case", TC_PAIR, ids=lambda c: _ids(c[0]) + c[1])
def test_im2col_pairs_match_single_ctas(cb, case, monkeypatch):
    geom, bn = case
    N, H, W, Cin, Cout, KH, KW, s_, p_, d_, groups, bias = geom
    # the Conv1D case (KH = 1) is causal: padding before the sequence only
    c = _case(N, H, W, Cin, Cout, KH, KW, s_, p_, d_, groups, bias, seed=sum(geom[:7]) + 29,
              **({} if KH > 1 else {"pad_w_end": 0}))
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    monkeypatch.setenv("CONV_B200_TC_PAIR", "1")
    y_pair, k1 = _run(cb, c, Xb, Fb, b, env=bn)
    monkeypatch.setenv("CONV_B200_TC_PAIR", "0")
    y_one, k2 = _run(cb, c, Xb, Fb, b, env=bn)
    assert k1 == k2 == "dense_tc_kernel"
    _check(c, y_pair, Xb, Fb, b)
    assert np.array_equal(y_pair, y_one)


def test_padded_halo_refuses_what_it_cannot_do(cb):
    # forced onto a shape it does not take (32-channel groups): CONV_ERR_UNSUPPORTED
    c = _case(2, 16, 16, 64, 64, 3, 3, (1, 1), (1, 1), (1, 1), 2, False, seed=1)
    Xb, Fb = workloads.dense_inputs(c)
    with pytest.raises(cb.ConvError) as e:
        _run(cb, c, Xb, Fb, None, env="halo")
    assert e.value.code == cb.CONV_ERR_UNSUPPORTED


@pytest.mark.parametrize("bn", ["bn64", "bn128", "bn256"])
def test_grouped_tile_widths(cb, bn):
    c = _case(2, 20, 20, 384, 384, 3, 3, (1, 1), (1, 1), (1, 1), 2, True, seed=8)   # 192-wide groups
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y, kernel = _run(cb, c, Xb, Fb, b, env=bn)
    assert kernel == "dense_tc_kernel"
    _check(c, y, Xb, Fb, b)


def test_one_group_square_is_the_ex_entry(cb):
    c = _case(4, 30, 30, 64, 64, 3, 3, (2, 2), (1, 1), (1, 1), 1, True, seed=3)
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y, _ = _run(cb, c, Xb, Fb, b)
    X = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).cuda()
    F = torch.from_numpy(Fb.view(np.int16)).view(torch.bfloat16).cuda()
    y0 = cb.conv2d_nhwc_fwd_ex(X, F, torch.from_numpy(b).cuda(), stride=2, pad=1, dil=1)
    y0 = workloads.bf16_to_f32(y0.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    assert np.array_equal(y, y0)


def test_groups_do_not_mix(cb):
    # a NaN planted in one group's input channels stays out of the other groups' outputs
    c = _case(2, 20, 20, 128, 128, 3, 3, (1, 1), (1, 1), (1, 1), 2, False, seed=4)
    Xb, Fb = workloads.dense_inputs(c)
    Xb = Xb.copy()
    Xb[..., 64:] = np.uint16(0x7FC0)   # bf16 quiet NaN
    ref, absum = oracle.conv2d_grouped(workloads.bf16_to_f32(Xb[..., :64]), workloads.bf16_to_f32(Fb[..., :64]), None,
                                       1, 1, 1, 1)
    # the padded halo kernel (default here) and the im2col kernel (forced)
    for env, name in ((None, "dense_halo_pad_kernel"), ("bn64", "dense_tc_kernel")):
        y, kernel = _run(cb, c, Xb, Fb, None, env=env)
        assert kernel == name
        assert np.all(np.isnan(y[..., 64:]))
        assert np.all(np.abs(y[..., :64] - ref) <= TOL * absum)


def test_page_two_filters_with_bias_as_conv1d(cb):
    # "The matrix connection": x = 1..5, filters (2, 0, -1) and (1, 1, 1), biases 1 and 0 give
    # (0, 1, 2) and (6, 9, 12); a one-row sequence of 8 channels (channel 0 carries the signal),
    # 8 filters of which 0 and 1 are used
    X = np.zeros((1, 1, 5, 8), np.float32)
    X[0, 0, :, 0] = [1, 2, 3, 4, 5]
    F = np.zeros((1, 3, 8, 8), np.float32)
    F[0, :, 0, 0] = [2, 0, -1]
    F[0, :, 0, 1] = [1, 1, 1]
    b = np.zeros(8, np.float32)
    b[0] = 1
    c = _case(1, 1, 5, 8, 8, 1, 3, (1, 1), (0, 0), (1, 1), 1, True)
    y, _ = _run(cb, c, workloads.bf16_bits(X), workloads.bf16_bits(F), b)
    assert np.array_equal(y[0, 0, :, 0], [0, 1, 2]) and np.array_equal(y[0, 0, :, 1], [6, 9, 12])


# the benchmark's workloads and the kernel the dispatcher gives each (the grouped 3x3 runs the
# padded halo kernel; the Conv1D layers have 80 channels, a stride or a filter too large to stay
# resident, and run the im2col kernel)
FULL_SIZE = [(workloads.DENSE_GROUPED, "dense_halo_pad_kernel"), (workloads.CONV1D_STEM1, "dense_tc_kernel"),
             (workloads.CONV1D_STEM2, "dense_tc_kernel"), (workloads.CONV1D_CAUSAL, "dense_tc_kernel")]


@pytest.mark.parametrize("case", FULL_SIZE, ids=["grouped", "conv1d-stem1", "conv1d-stem2", "conv1d-causal"])
def test_full_size_workloads(cb, case):
    # the benchmark's workloads at full size, every output compared with the oracle
    case, expected = case
    Xb, Fb = workloads.dense_inputs(case)
    b = workloads.dense_bias(case)
    y, kernel = _run(cb, case, Xb, Fb, b)
    _check(case, y, Xb, Fb, b)
    assert kernel == expected


# Causal Conv1D ("Convolution Is Wx+b Moving Across a Signal", section "Find the same sum in CKE's
# C kernels": a frame's output reads no later frame): zero padding of dil*(K-1) frames before the
# sequence and none after it.
# (N, L, Cin, Cout, K, dil, groups, bias, kernel expected)
CAUSAL = [(2, 1000, 64, 128, 3, 1, 1, True, "dense_halo_pad_kernel"),
          (2, 777, 128, 64, 5, 2, 4, True, "dense_tc_kernel"),     # dilated, grouped, ragged length
          (3, 50, 12, 8, 3, 1, 1, False, "dense_direct_kernel")]   # channel counts for the CUDA cores


@pytest.mark.parametrize("case", CAUSAL, ids=lambda c: "N{}L{}C{}-{}k{}d{}g{}".format(*c[:7]))
def test_causal_conv1d(cb, case):
    N, L, Cin, Cout, K, d, groups, bias, expected = case
    c = _case(N, 1, L, Cin, Cout, 1, K, (1, 1), (0, d * (K - 1)), (1, d), groups, bias, seed=L + K, pad_w_end=0)
    Xb, Fb = workloads.dense_inputs(c)
    b = workloads.dense_bias(c)
    y, kernel = _run(cb, c, Xb, Fb, b)
    assert kernel == expected
    assert y.shape == (N, 1, L, Cout)
    _check(c, y, Xb, Fb, b)
    # the same outputs as the symmetric padding's first L frames, on the CUDA-core kernel too
    sym = _case(N, 1, L, Cin, Cout, 1, K, (1, 1), (0, d * (K - 1)), (1, d), groups, bias, seed=L + K)
    y_sym, _ = _run(cb, sym, Xb, Fb, b)
    ref, absum = oracle.conv2d_grouped(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), b, 1, c.pads, (1, d),
                                       groups)
    assert np.all(np.abs(y_sym[:, :, :L] - ref) <= TOL * absum)
    y_cc, k_cc = _run(cb, c, Xb, Fb, b, env="direct")
    assert k_cc == "dense_direct_kernel"
    _check(c, y_cc, Xb, Fb, b)
