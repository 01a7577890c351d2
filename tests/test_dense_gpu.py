"""Dense NHWC convolution on the GPU against the CPU oracle, through the C ABI.

Tolerance for bfloat16 output: |y - y_ref| <= 4e-3 * sum|x||w| per output, where y_ref is the
oracle's float64 sum of the same bfloat16 operands. The budget is one round-to-nearest of the
output to bfloat16 (at most 2**-9 relative, below 1.96e-3 of the magnitude sum) plus float32
accumulation error (below 2**-24 * (terms + 1) of the magnitude sum, well inside the rest).
The float32 entry point on small-integer inputs must be exact.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.conftest import GOLDEN

pytestmark = pytest.mark.gpu

TOL = 4e-3


@pytest.fixture(scope="module")
def cb(cuda):
    import cnn_convolution_nhwc_b200 as cb
    return cb


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _host_bf16(t):
    return workloads.bf16_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _run_bf16(cb, Xb, Fb, env=None):
    old = os.environ.get("CONV_B200_DENSE")
    if env is not None:
        os.environ["CONV_B200_DENSE"] = env
    try:
        Y = cb.conv2d_nhwc_fwd(_dev_bf16(Xb), _dev_bf16(Fb))
        torch.cuda.synchronize()
    finally:
        if env is not None:
            if old is None:
                del os.environ["CONV_B200_DENSE"]
            else:
                os.environ["CONV_B200_DENSE"] = old
    assert cb.conv_device_status() == cb.CONV_OK
    return _host_bf16(Y)


def _check_bf16(y, Xb, Fb):
    ref, absum = oracle.conv2d_nhwc(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb))
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    err = np.abs(y.astype(np.float64) - ref)
    bad = err > TOL * absum
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance; worst {np.max(err / np.maximum(absum, 1e-30))}"
    return ref


_LARGE = {}


def _large_inputs():
    if not _LARGE:
        _LARGE["v"] = workloads.dense_inputs(workloads.DENSE_LARGE)
    return _LARGE["v"]


def _case_inputs(N, H, W, Cin, Cout, K, seed):
    c = workloads.DenseCase("t", N, H, W, Cin, Cout, K, "bf16", "normal", seed)
    return workloads.dense_inputs(c)


# ------------------------------------------------------------------------------------------
# Worked examples from the pages, through both paths
# ------------------------------------------------------------------------------------------


def test_pins_direct_path(cb):
    g = json.load(open(os.path.join(GOLDEN, "dlsys14_patch_example.json")))
    X = np.arange(36, dtype=np.float32).reshape(1, 6, 6, 1)
    F = np.arange(9, dtype=np.float32).reshape(3, 3, 1, 1)
    Y = cb.conv2d_nhwc_fwd_f32(torch.from_numpy(X).cuda(), torch.from_numpy(F).cuda()).cpu().numpy()
    assert np.array_equal(Y[0, :, :, 0], np.array(g["output"], np.float32))
    # bfloat16 entry: inputs are exact, outputs above 256 round (1122 -> 1120)
    y = _run_bf16(cb, workloads.bf16_bits(X), workloads.bf16_bits(F))
    assert np.array_equal(y[0, :, :, 0], workloads.bf16_to_f32(workloads.bf16_bits(np.array(g["output"], np.float32))))
    s = json.load(open(os.path.join(GOLDEN, "wxb_2d_examples.json")))
    t = s["tiny_2d"]
    Y = cb.conv2d_nhwc_fwd_f32(torch.tensor(t["image"], dtype=torch.float32).reshape(1, 3, 3, 1).cuda(),
                               torch.tensor(t["filter"], dtype=torch.float32).reshape(2, 2, 1, 1).cuda())
    assert Y[0, :, :, 0].cpu().tolist() == t["output"]
    so = s["sobel"]
    Fs = torch.stack([torch.tensor(so["gx"]), torch.tensor(so["gy"])], -1).float().reshape(3, 3, 1, 2)
    Y = cb.conv2d_nhwc_fwd_f32(torch.tensor(so["image"], dtype=torch.float32).reshape(1, 6, 6, 1).cuda(), Fs.cuda())
    assert Y[0, :, :, 0].cpu().tolist() == so["gx_output"] and Y[0, :, :, 1].cpu().tolist() == so["gy_output"]


def test_pins_tensor_core_path(cb):
    # The 6x6 example and the Sobel pair, replicated over 256 images and placed in channel 0
    # of 8 input channels and output channels 0 and 1 of 8, so the tensor-core path takes it.
    g = json.load(open(os.path.join(GOLDEN, "dlsys14_patch_example.json")))
    so = json.load(open(os.path.join(GOLDEN, "wxb_2d_examples.json")))["sobel"]
    N = 256
    X = np.zeros((N, 6, 6, 8), np.float32)
    X[:, :, :, 0] = np.arange(36, dtype=np.float32).reshape(6, 6)
    X[:, :, :, 3] = np.array(so["image"], np.float32)
    F = np.zeros((3, 3, 8, 8), np.float32)
    F[:, :, 0, 0] = np.arange(9, dtype=np.float32).reshape(3, 3)
    F[:, :, 3, 1] = np.array(so["gx"], np.float32)
    F[:, :, 3, 2] = np.array(so["gy"], np.float32)
    exp0 = workloads.bf16_to_f32(workloads.bf16_bits(np.array(g["output"], np.float32)))
    for path in ("fold", "halo64", "bn64"):   # folded-tap, halo and im2col kernels
        y = _run_bf16(cb, workloads.bf16_bits(X), workloads.bf16_bits(F), env=path)
        for n in (0, 1, 100, N - 1):
            assert np.array_equal(y[n, :, :, 0], exp0), path
            assert np.array_equal(y[n, :, :, 1], np.array(so["gx_output"], np.float32)), path
            assert np.array_equal(y[n, :, :, 2], np.array(so["gy_output"], np.float32)), path
            assert not y[n, :, :, 3:].any(), path


# ------------------------------------------------------------------------------------------
# The workloads
# ------------------------------------------------------------------------------------------


def test_tiny_fp32_config_exact(cb):
    c = workloads.DENSE_TINY
    X, F = workloads.dense_inputs(c)
    Y = cb.conv2d_nhwc_fwd_f32(torch.from_numpy(X).cuda(), torch.from_numpy(F).cuda()).cpu().numpy()
    ref, _ = oracle.conv2d_nhwc(X, F)
    assert np.array_equal(Y.astype(np.float64), ref)


@pytest.mark.parametrize("case", [workloads.DENSE_3X3, workloads.DENSE_1X1], ids=lambda c: c.name)
def test_workload_full_output(cb, case):
    Xb, Fb = workloads.dense_inputs(case)
    y = _run_bf16(cb, Xb, Fb)
    _check_bf16(y, Xb, Fb)


def test_pointwise_is_matmul(cb):
    # K = 1: Y = X @ F[0,0] (DLSys notes section 2), checked against a float64 matmul
    case = workloads.DENSE_1X1
    Xb, Fb = workloads.dense_inputs(case)
    y = _run_bf16(cb, Xb, Fb)
    Xf = workloads.bf16_to_f32(Xb).reshape(-1, case.Cin).astype(np.float64)
    Ff = workloads.bf16_to_f32(Fb)[0, 0].astype(np.float64)
    ref = Xf @ Ff
    bound = np.abs(Xf) @ np.abs(Ff)
    assert np.all(np.abs(y.reshape(ref.shape) - ref) <= TOL * bound)


@pytest.mark.parametrize("path", [None, "halo"], ids=["default", "halo"])
def test_large_workload_sampled(cb, path):
    # N=64, 112x112, 128->128, K=5: compare 20000 sampled outputs (including the first and
    # last pixels of every image corner region and the last M tile) with the oracle; the
    # default path and the halo kernel with its streamed filter.
    case = workloads.DENSE_LARGE
    Xb, Fb = _large_inputs()
    y = _run_bf16(cb, Xb, Fb, env=path)
    Ho, Wo, Co = case.Ho, case.Wo, case.Cout
    total = case.N * Ho * Wo * Co
    r = workloads.splitmix64(77, 20000)
    idx = (r % np.uint64(total)).astype(np.int64)
    corners = []
    for n in (0, case.N // 2, case.N - 1):
        for (yy, xx) in ((0, 0), (0, Wo - 1), (Ho - 1, 0), (Ho - 1, Wo - 1)):
            for o in (0, Co - 1):
                corners.append(((n * Ho + yy) * Wo + xx) * Co + o)
    idx = np.concatenate([idx, np.array(corners, np.int64), np.arange(total - 128 * Co, total, 97)])
    ref, absum = oracle.conv2d_nhwc_points(workloads.bf16_to_f32(Xb), workloads.bf16_to_f32(Fb), idx)
    got = y.reshape(-1)[idx].astype(np.float64)
    assert np.all(np.abs(got - ref) <= TOL * absum)
    assert np.all(np.isfinite(y))


# ------------------------------------------------------------------------------------------
# Edge shapes: ragged M and N tiles, partial channel blocks, small / odd channel counts,
# full-image filters, K = 7, non-square images
# ------------------------------------------------------------------------------------------

EDGE = [
    (3, 20, 23, 72, 24, 3),     # ragged M tile, Cin = 64 + 8, Cout < 64
    (64, 16, 16, 8, 16, 3),     # Cin = 8
    (8, 30, 17, 24, 40, 2),     # Cin = 24, even K, non-square
    (32, 8, 8, 64, 64, 8),      # K = H = W: Ho = Wo = 1, each output a dot product
    (4, 19, 27, 64, 136, 7),    # K = 7, Cout = 128 + 8
    (2, 40, 40, 128, 256, 1),   # pointwise with two 128-wide N tiles
    (5, 33, 9, 40, 200, 4),     # Cout = 200
]


@pytest.mark.parametrize("path", [None, "bn64"], ids=["halo", "im2col"])
@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "x".join(map(str, s)))
def test_edge_shapes(cb, shape, path):
    N, H, W, Cin, Cout, K = shape
    Xb, Fb = _case_inputs(N, H, W, Cin, Cout, K, seed=sum(shape))
    if path == "bn64" and Xb.nbytes < 128 * 1024:
        # the im2col kernel serves inputs of at least 128 KiB; forcing it below is refused
        os.environ["CONV_B200_DENSE"] = path
        try:
            with pytest.raises(cb.ConvError) as e:
                cb.conv2d_nhwc_fwd(_dev_bf16(Xb), _dev_bf16(Fb))
            assert e.value.code == cb.CONV_ERR_UNSUPPORTED
        finally:
            del os.environ["CONV_B200_DENSE"]
        return
    y = _run_bf16(cb, Xb, Fb, env=path)
    _check_bf16(y, Xb, Fb)


def test_wide_image_falls_back_to_im2col(cb):
    # a 2100-pixel-wide image: the halo (128 + 2*2100 rows) does not fit in shared memory,
    # so the im2col kernel runs; forcing the halo kernel is reported as unsupported
    Xb, Fb = _case_inputs(2, 3, 2100, 64, 64, 3, seed=21)
    _check_bf16(_run_bf16(cb, Xb, Fb), Xb, Fb)
    os.environ["CONV_B200_DENSE"] = "halo"
    try:
        with pytest.raises(cb.ConvError) as e:
            cb.conv2d_nhwc_fwd(_dev_bf16(Xb), _dev_bf16(Fb))
        assert e.value.code == cb.CONV_ERR_UNSUPPORTED
    finally:
        del os.environ["CONV_B200_DENSE"]


@pytest.mark.parametrize("shape", [(2, 7, 9, 3, 5, 3), (1, 5, 5, 1, 1, 5), (3, 6, 11, 12, 10, 2)],
                         ids=lambda s: "x".join(map(str, s)))
def test_unaligned_channels_direct_path(cb, shape):
    N, H, W, Cin, Cout, K = shape
    Xb, Fb = _case_inputs(N, H, W, Cin, Cout, K, seed=sum(shape) + 1)
    y = _run_bf16(cb, Xb, Fb)
    _check_bf16(y, Xb, Fb)


def test_kernel_and_tile_width_choices_agree(cb):
    # Cin = 64 is one channel block, so every kernel and tile width walks the same MMA sequence
    # per output (taps in (i, j) order, 16 channels per step). At widths 64 and 128 the halo and
    # im2col kernels alternate those steps between two partial accumulators and add the two in
    # the epilogue; at width 256 one accumulator takes them all. Within each of the two orders:
    # identical bits; across them: the oracle's bound.
    Xb, Fb = _case_inputs(4, 24, 24, 64, 256, 3, seed=5)
    ys = {v: _run_bf16(cb, Xb, Fb, env=v) for v in ("halo64", "halo128", "halo256", "bn64", "bn128", "bn256")}
    for v, y in ys.items():
        _check_bf16(y, Xb, Fb)
    for v in ("halo128", "bn64", "bn128"):
        assert np.array_equal(ys[v], ys["halo64"]), v
    assert np.array_equal(ys["bn256"], ys["halo256"])
    yd = _run_bf16(cb, Xb, Fb, env="direct")
    _check_bf16(yd, Xb, Fb)


def test_streamed_filter_multi_block(cb):
    # Cin = 192 (three channel blocks) and a filter too large to keep resident: the halo
    # kernel streams the filter per tap; the im2col kernel agrees within tolerance
    Xb, Fb = _case_inputs(2, 30, 26, 192, 320, 5, seed=8)
    _check_bf16(_run_bf16(cb, Xb, Fb, env="halo"), Xb, Fb)
    _check_bf16(_run_bf16(cb, Xb, Fb), Xb, Fb)
    _check_bf16(_run_bf16(cb, Xb, Fb, env="bn128"), Xb, Fb)


def test_repeatable(cb):
    Xb, Fb = workloads.dense_inputs(workloads.DENSE_3X3)
    a = _run_bf16(cb, Xb, Fb)
    b = _run_bf16(cb, Xb, Fb)
    assert np.array_equal(a, b)


def test_translation_equivariance(cb):
    # shifting the input one column right shifts the output one column (stride 1, interior)
    Xb, Fb = _case_inputs(8, 20, 30, 64, 64, 3, seed=9)
    Xs = np.zeros_like(Xb)
    Xs[:, :, 1:, :] = Xb[:, :, :-1, :]
    y = _run_bf16(cb, Xb, Fb)
    ys = _run_bf16(cb, Xs, Fb)
    assert np.array_equal(ys[:, :, 1:, :], y[:, :, :-1, :])


def test_noncontiguous_rejected_and_contiguous_copy_works(cb):
    Xb, Fb = _case_inputs(4, 16, 16, 64, 64, 3, seed=3)
    X = _dev_bf16(Xb)
    Xt = X.permute(0, 2, 1, 3)   # a transposed view: not contiguous
    with pytest.raises(ValueError):
        cb.conv2d_nhwc_fwd(Xt, _dev_bf16(Fb))
    y = _host_bf16(cb.conv2d_nhwc_fwd(Xt.contiguous(), _dev_bf16(Fb)))
    torch.cuda.synchronize()
    _check_bf16(y, np.ascontiguousarray(Xb.transpose(0, 2, 1, 3)), Fb)


def test_dispatcher_choices(cb):
    # Cout <= 64 with K = 3 -> folded-tap kernel; wider Cout with a resident filter (at most
    # 128 KiB in 64 x 128 slots) -> halo kernel; a larger filter -> streamed-filter kernel; channels not multiples
    # of 8 -> CUDA-core kernel; a forced im2col tile width -> im2col kernel
    Xb, Fb = _case_inputs(2, 20, 20, 64, 64, 3, seed=21)
    _run_bf16(cb, Xb, Fb)
    assert cb.conv_last_kernel() == "dense_fold_kernel"
    Xb, Fb = _case_inputs(2, 20, 20, 64, 128, 2, seed=24)      # 4 taps x 16 KiB of filter
    _run_bf16(cb, Xb, Fb)
    assert cb.conv_last_kernel() == "dense_halo_kernel"
    Xb, Fb = _case_inputs(2, 20, 20, 64, 128, 3, seed=24)      # 144 KiB of filter
    _run_bf16(cb, Xb, Fb)
    assert cb.conv_last_kernel() == "dense_stream_kernel"
    Xb2, Fb2 = _case_inputs(1, 7, 9, 3, 5, 3, seed=22)
    _run_bf16(cb, Xb2, Fb2)
    assert cb.conv_last_kernel() == "dense_direct_kernel"
    Xb3, Fb3 = _case_inputs(4, 40, 40, 64, 128, 3, seed=23)     # input above 128 KiB
    _run_bf16(cb, Xb3, Fb3, env="bn128")
    assert cb.conv_last_kernel() == "dense_tc_kernel"


# (N, H, W, Cin, Cout, K): the folded-tap kernel (Cout <= 64, K = 2..4, resident filter):
# ragged last tile, Cout below one 64-column group, several channel blocks, a halo spanning
# several TMA boxes (128 + (K-1)*W > 256 rows), one image smaller than a tile
FOLD_SHAPES = [(2, 20, 20, 64, 64, 3), (3, 9, 13, 16, 8, 2), (2, 17, 11, 128, 40, 2), (1, 30, 70, 32, 64, 3),
               (2, 12, 12, 8, 64, 4), (1, 4, 4, 64, 24, 4), (4, 40, 40, 64, 64, 3)]


@pytest.mark.parametrize("shape", FOLD_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_folded_taps(cb, shape):
    N, H, W, Cin, Cout, K = shape
    Xb, Fb = _case_inputs(N, H, W, Cin, Cout, K, seed=sum(shape) + 7)
    y = _run_bf16(cb, Xb, Fb, env="fold")
    assert cb.conv_last_kernel() == "dense_fold_kernel"
    _check_bf16(y, Xb, Fb)


@pytest.mark.parametrize("shape", [(1, 9, 9, 64, 64, 1), (1, 9, 9, 64, 64, 5), (1, 9, 9, 64, 72, 3)],
                         ids=["K1", "K5", "Cout72"])
def test_folded_taps_refuses_other_shapes(cb, shape):
    N, H, W, Cin, Cout, K = shape
    Xb, Fb = _case_inputs(N, H, W, Cin, Cout, K, seed=3)
    with pytest.raises(cb.ConvError) as e:
        _run_bf16(cb, Xb, Fb, env="fold")
    assert e.value.code == cb.CONV_ERR_UNSUPPORTED


# (N, H, W, Cin, Cout, K): the streamed-filter kernel (256-row tiles, 32-channel halo blocks,
# two accumulators per filter slot): a ragged last tile; several N tiles with a partial last
# one; a partial 32-channel block and Cout = 64 (64-column accumulators); K = 7 with Cout below
# the tile width on a wide image (halo of 562 rows in three boxes); K = 1 with an 8-column
# last N tile; K = H = W (one output per image)
STREAM_SHAPES = [(3, 21, 19, 64, 128, 5), (2, 30, 26, 192, 320, 5), (4, 16, 16, 40, 64, 3), (2, 12, 50, 96, 96, 7),
                 (5, 9, 9, 128, 136, 1), (4, 8, 8, 64, 64, 8)]


@pytest.mark.parametrize("shape", STREAM_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_streamed_filter_kernel(cb, shape):
    N, H, W, Cin, Cout, K = shape
    Xb, Fb = _case_inputs(N, H, W, Cin, Cout, K, seed=sum(shape) + 11)
    y = _run_bf16(cb, Xb, Fb, env="stream")
    assert cb.conv_last_kernel() == "dense_stream_kernel"
    _check_bf16(y, Xb, Fb)


# CTA pairs (BN = 128: each CTA of a 2-CTA cluster stages half of every filter slot, and the even
# CTA's M = 256 MMAs span both): a pair whose second CTA has no valid rows (ragged end), several
# N tiles, and more pair tiles than pairs on the device (clusters loop over tiles)
PAIR_SHAPES = [(3, 21, 19, 64, 128, 5), (2, 30, 26, 192, 320, 5), (16, 50, 50, 32, 128, 3)]


@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_streamed_filter_pairs_match_single_ctas(cb, shape):
    # the same MMA sequence per output with or without pairs: identical bits
    N, H, W, Cin, Cout, K = shape
    Xb, Fb = _case_inputs(N, H, W, Cin, Cout, K, seed=sum(shape) + 17)
    os.environ["CONV_B200_STREAM_PAIR"] = "0"
    try:
        y_single = _run_bf16(cb, Xb, Fb, env="stream")
    finally:
        del os.environ["CONV_B200_STREAM_PAIR"]
    y_pair = _run_bf16(cb, Xb, Fb, env="stream")
    assert cb.conv_last_kernel() == "dense_stream_kernel"
    _check_bf16(y_pair, Xb, Fb)
    assert np.array_equal(y_pair, y_single)


def test_streamed_filter_is_the_default_for_large_filters(cb):
    # 5x5x128x128 bf16 is 800 KiB of filter: it cannot stay in shared memory
    Xb, Fb = _case_inputs(2, 20, 20, 128, 128, 5, seed=31)
    _check_bf16(_run_bf16(cb, Xb, Fb), Xb, Fb)
    assert cb.conv_last_kernel() == "dense_stream_kernel"
