"""GPU parity of dwpw_fwd (depthwise then pointwise, fused) against the oracle.

The depthwise stage is the page's bit-exact contract, so both sides round the same float32
intermediate to bf16 and differ only in how the pointwise sum is accumulated: every product
a*F of two bf16 values is exact in float32, and a float32 sum of C + 1 terms in any order, with
any rounding mode, is within (C + 2) * 2^-23 of the absolute sum. That is the bar per output.
Where the mixing matrix is the identity, the block must reproduce the rounded depthwise output
bit for bit.
"""
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


def _dev(a, bf16=False):
    if a is None:
        return None
    if bf16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def _run(cb, case, x, w, bd, F, bp, mode):
    y = cb.dwpw_fwd(_dev(x), _dev(w), _dev(bd), _dev(F, bf16=True), _dev(bp), stride=case.stride, pad=case.pad,
                    dil=case.dil, mode=mode)
    kernel = cb.conv_last_kernel()
    out = y.cpu().numpy().astype(np.float64)
    assert cb.conv_device_status() == cb.CONV_OK
    return out, kernel


KERNELS = ("dwpw_kernel", "dwpw_staged_kernel", "dwpw_gemm_kernel")


def _tol(C):
    return (C + 2) * 2.0 ** -23


# (N, C, H, K, stride, pad, dil, Cout, mode, biases)
CASES = [
    (2, 64, 14, 3, 1, 1, 1, 64, 0, True),       # one channel block
    (4, 72, 28, 5, 2, 2, 1, 40, 0, True),       # ragged channel block, N = 48 MMA
    (2, 120, 28, 5, 1, 2, 1, 40, 1, False),     # fast mode, no biases
    (8, 672, 14, 3, 1, 1, 1, 112, 0, True),     # 10.5 channel blocks, tiles across images
    (4, 960, 7, 5, 1, 2, 1, 160, 1, True),      # three filter boxes, 49-pixel images
    (2, 16, 30, 3, 1, 1, 1, 16, 0, True),       # 16 channels into 16 outputs
    (1, 8, 9, 7, 1, 3, 1, 256, 0, True),        # 7x7 (runtime filter size), 256 outputs
    (3, 24, 11, 3, 2, 1, 2, 24, 1, True),       # stride 2 with dilation 2, N = 32 MMA
    (2, 40, 12, 3, 1, 0, 1, 8, 0, True),        # no padding, 8 outputs
    (3, 32, 5, 1, 1, 0, 1, 32, 0, True),        # 1x1 depthwise (a per-channel scale and bias)
    (5, 24, 1, 3, 1, 1, 1, 16, 0, True),        # 1x1 images: every tap but the centre is padding
    (1, 200, 3, 3, 2, 1, 1, 200, 1, True),      # 2x2 output, one partial tile, ragged Cout chunk
    (2, 64, 12, 3, 2, 0, 1, 64, 0, True),       # stride 2, no padding: the last input column unused
]


def _ids(c):
    return "N{}C{}H{}K{}s{}p{}d{}-O{}-{}".format(*c[:8], "exact" if c[8] == 0 else "fast") + ("b" if c[9] else "")


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_block_matches_oracle(cb, c):
    N, C, H, K, s, p, d, Cout, mode, bias = c
    case = workloads.DwPwCase("t", N, C, H, H, K, s, p, d, Cout, bias, seed=C + K + Cout)
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    y, kernel = _run(cb, case, x, w, bd, F, bp, mode)
    assert kernel in KERNELS
    ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, s, p, d, mode)
    assert y.shape == ref.shape
    assert np.all(np.isfinite(y))
    bad = np.abs(y - ref) > _tol(C) * absum
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance"


@pytest.mark.parametrize("mode", [0, 1])
def test_identity_mixing_is_the_rounded_depthwise_output(cb, mode):
    # F = I: every output is one exact product plus zeros, so the block must equal the
    # depthwise output rounded to bf16, bit for bit
    case = workloads.DwPwCase("t", 3, 64, 20, 20, 3, 2, 1, 1, 64, True, seed=3)
    x, w, bd, _, _ = workloads.dwpw_inputs(case)
    F = workloads.bf16_bits(np.eye(64, dtype=np.float32))
    y, _ = _run(cb, case, x, w, bd, F, None, mode)
    dref = oracle.depthwise(x, w, bd, mult=1, stride=2, pad=1, dil=1, mode=mode)
    assert np.array_equal(y, workloads.bf16_to_f32(workloads.bf16_bits(dref)).astype(np.float64))


def test_unsupported_output_width_is_refused(cb):
    case = workloads.DwPwCase("t", 1, 8, 9, 9, 3, 1, 1, 1, 12, False)
    x, w, _, F, _ = workloads.dwpw_inputs(case)
    with pytest.raises(cb.ConvError) as e:
        _run(cb, case, x, w, None, F, None, 0)
    assert e.value.code == cb.CONV_ERR_UNSUPPORTED


@pytest.mark.parametrize("case", workloads.DWPW_BLOCKS, ids=lambda c: c.name.replace(" ", "-"))
def test_full_size_blocks(cb, case):
    # the benchmark's blocks at full size, every output compared with the oracle
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    for mode in (0, 1):
        y, kernel = _run(cb, case, x, w, bd, F, bp, mode)
        assert kernel == "dwpw_gemm_kernel" and np.all(np.isfinite(y))
        ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, case.stride, case.pad, case.dil, mode)
        assert np.all(np.abs(y - ref) <= _tol(case.C) * absum)


# (N, C, H, K, Cout, mode, biases): the transposed-GEMM kernel (7x7 and 14x14 images, stride 1,
# "same" padding): partial last channel block (C = 72 over blocks of 32; C = 100 over 64),
# 8 outputs, two 128-row M tiles (136, 256 outputs), no biases, more images than CTAs
GEMM_CASES = [(2, 72, 14, 3, 112, 0, True), (3, 100, 7, 5, 160, 1, True), (2, 64, 14, 5, 8, 0, False),
              (2, 32, 7, 3, 136, 0, True), (1, 128, 14, 3, 256, 1, True), (160, 8, 14, 3, 16, 0, True),
              (200, 4, 7, 5, 24, 1, True),
              (2, 48, 14, 5, 144, 1, True)]   # 5x5 with more than 128 outputs: the row split's rings do not fit


# the forms of the transposed-GEMM kernel: one CTA per image; a 2-CTA cluster that splits the
# channel blocks and adds the two partial sums through distributed shared memory; and (14x14
# images) two CTAs per image that each take half of the output rows and every channel
GEMM_FORMS = {"one-cta": {"CONV_B200_DWPW_SPLIT": "1", "CONV_B200_DWPW_HALF": "0"},
              "cluster": {"CONV_B200_DWPW_SPLIT": "2", "CONV_B200_DWPW_HALF": "0"},
              "half-rows": {"CONV_B200_DWPW_HALF": "1"}}


def _form(monkeypatch, form):
    monkeypatch.setenv("CONV_B200_DWPW_KERNEL", "gemm")
    for k in ("CONV_B200_DWPW_SPLIT", "CONV_B200_DWPW_HALF"):
        monkeypatch.delenv(k, raising=False)
    for k, v in GEMM_FORMS[form].items():
        monkeypatch.setenv(k, v)


@pytest.mark.parametrize("form", list(GEMM_FORMS))
@pytest.mark.parametrize("c", GEMM_CASES, ids=lambda c: "N{}C{}H{}K{}-O{}-{}".format(*c[:5], "exact" if c[5] == 0 else "fast"))
def test_transposed_gemm_kernel(cb, c, form, monkeypatch):
    _form(monkeypatch, form)
    N, C, H, K, Cout, mode, bias = c
    case = workloads.DwPwCase("t", N, C, H, H, K, 1, (K - 1) // 2, 1, Cout, bias, seed=C + K + Cout + N)
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    y, kernel = _run(cb, case, x, w, bd, F, bp, mode)
    assert kernel == "dwpw_gemm_kernel"
    ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, 1, (K - 1) // 2, 1, mode)
    assert np.all(np.isfinite(y))
    bad = np.abs(y - ref) > _tol(C) * absum
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance"
    y2, _ = _run(cb, case, x, w, bd, F, bp, mode)
    assert np.array_equal(y, y2)   # a given split repeats its bits


@pytest.mark.parametrize("K,mode", [(3, 0), (3, 1), (5, 0)])
def test_half_rows_form_is_live(cb, K, mode, monkeypatch):
    # the row halves accumulate every channel of an output in one chain, in channel order, as
    # one CTA per image does: the same bits. The channel-split cluster adds two partial sums:
    # over 700k outputs its bits differ somewhere, so equality with the one-CTA form shows that
    # the half-rows form really ran (all three within the bar)
    case = workloads.DwPwCase("t", 8, 672, 14, 14, K, 1, (K - 1) // 2, 1, 112, True, seed=15 + K)
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    ys = {}
    for form in GEMM_FORMS:
        _form(monkeypatch, form)
        ys[form], kernel = _run(cb, case, x, w, bd, F, bp, mode)
        assert kernel == "dwpw_gemm_kernel"
    ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, 1, (K - 1) // 2, 1, mode)
    for y in ys.values():
        assert np.all(np.abs(y - ref) <= _tol(case.C) * absum)
    assert np.array_equal(ys["half-rows"], ys["one-cta"])
    assert not np.array_equal(ys["cluster"], ys["one-cta"])


@pytest.mark.parametrize("form", list(GEMM_FORMS))
@pytest.mark.parametrize("hw,K", [(14, 3), (14, 5), (7, 5)])
@pytest.mark.parametrize("mode", [0, 1])
def test_transposed_gemm_identity_mixing_is_exact(cb, hw, K, mode, form, monkeypatch):
    # F = I: every output is one exact product plus zeros (also each of the two partial sums of
    # a split), so the block must equal the depthwise output rounded to bf16, bit for bit (the
    # depthwise stage of this kernel is the page's order)
    _form(monkeypatch, form)
    case = workloads.DwPwCase("t", 3, 96, hw, hw, K, 1, (K - 1) // 2, 1, 96, True, seed=hw + K)
    x, w, bd, _, _ = workloads.dwpw_inputs(case)
    F = workloads.bf16_bits(np.eye(96, dtype=np.float32))
    y, kernel = _run(cb, case, x, w, bd, F, None, mode)
    assert kernel == "dwpw_gemm_kernel"
    dref = oracle.depthwise(x, w, bd, mult=1, stride=1, pad=(K - 1) // 2, dil=1, mode=mode)
    assert np.array_equal(y, workloads.bf16_to_f32(workloads.bf16_bits(dref)).astype(np.float64))


def test_transposed_gemm_refuses_other_shapes(cb, monkeypatch):
    monkeypatch.setenv("CONV_B200_DWPW_KERNEL", "gemm")
    case = workloads.DwPwCase("t", 1, 8, 12, 12, 3, 1, 1, 1, 16, False)   # 12x12 images
    x, w, _, F, _ = workloads.dwpw_inputs(case)
    with pytest.raises(cb.ConvError) as e:
        _run(cb, case, x, w, None, F, None, 0)
    assert e.value.code == cb.CONV_ERR_UNSUPPORTED


@pytest.mark.parametrize("split", ["1", "2", "3", "4"])
def test_channel_split_across_a_cluster(cb, split, monkeypatch):
    # 13 pixel tiles and 11 channel blocks: by default a 4-CTA cluster splits the channels; every
    # split must meet the same bar, and a given split must repeat its bits exactly
    monkeypatch.setenv("CONV_B200_DWPW_SPLIT", split)
    case = workloads.DwPwCase("t", 8, 672, 14, 14, 3, 1, 1, 1, 112, True, seed=11)
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    y, kernel = _run(cb, case, x, w, bd, F, bp, 0)
    y2, _ = _run(cb, case, x, w, bd, F, bp, 0)
    assert kernel in KERNELS and np.array_equal(y, y2)
    ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, 1, 1, 1, 0)
    assert np.all(np.abs(y - ref) <= _tol(case.C) * absum)


def test_split_identity_mixing_is_exact(cb, monkeypatch):
    # with F = I every partial but one is zero, so the cluster's reduction is exact too
    monkeypatch.setenv("CONV_B200_DWPW_SPLIT", "3")
    case = workloads.DwPwCase("t", 2, 192, 10, 10, 5, 1, 2, 1, 192, True, seed=12)
    x, w, bd, _, _ = workloads.dwpw_inputs(case)
    F = workloads.bf16_bits(np.eye(192, dtype=np.float32))
    y, _ = _run(cb, case, x, w, bd, F, None, 1)
    dref = oracle.depthwise(x, w, bd, mult=1, stride=1, pad=2, dil=1, mode=1)
    assert np.array_equal(y, workloads.bf16_to_f32(workloads.bf16_bits(dref)).astype(np.float64))


@pytest.mark.parametrize("c", [CASES[0], CASES[2], CASES[3], CASES[4], CASES[10]], ids=_ids)
def test_staged_and_flat_kernels_agree(cb, c, monkeypatch):
    # shapes the staged kernel takes by default, run on both kernels: each meets the bar
    N, C, H, K, s, p, d, Cout, mode, bias = c
    case = workloads.DwPwCase("t", N, C, H, H, K, s, p, d, Cout, bias, seed=C + 2 * K)
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, s, p, d, mode)
    for kern, name in (("staged", "dwpw_staged_kernel"), ("flat", "dwpw_kernel")):
        monkeypatch.setenv("CONV_B200_DWPW_KERNEL", kern)
        y, kernel = _run(cb, case, x, w, bd, F, bp, mode)
        assert kernel == name
        assert np.all(np.abs(y - ref) <= _tol(C) * absum)


@pytest.mark.parametrize("kern", ["staged", "flat"])
@pytest.mark.parametrize("split", ["1", "4"])
def test_identity_mixing_exact_on_both_kernels(cb, kern, split, monkeypatch):
    monkeypatch.setenv("CONV_B200_DWPW_KERNEL", kern)
    monkeypatch.setenv("CONV_B200_DWPW_SPLIT", split)
    # F = the first 128 columns of I: output o < 128 is depthwise channel o, exactly
    case = workloads.DwPwCase("t", 6, 256, 7, 7, 5, 1, 2, 1, 128, True, seed=13)
    x, w, bd, _, _ = workloads.dwpw_inputs(case)
    F = workloads.bf16_bits(np.eye(256, 128, dtype=np.float32))
    y, kernel = _run(cb, case, x, w, bd, F, None, 0)
    assert kernel == ("dwpw_staged_kernel" if kern == "staged" else "dwpw_kernel")
    dref = oracle.depthwise(x, w, bd, mult=1, stride=1, pad=2, dil=1, mode=0)[:, :128]
    assert np.array_equal(y, workloads.bf16_to_f32(workloads.bf16_bits(dref)).astype(np.float64))


@pytest.mark.parametrize("kern", ["staged", "flat"])
def test_split_is_live(cb, kern, monkeypatch):
    # a 4-way split adds four partial sums where one CTA accumulates all blocks in order: over a
    # million outputs the two orders must differ somewhere (both within the bar), which shows
    # the split really ran
    monkeypatch.setenv("CONV_B200_DWPW_KERNEL", kern)
    case = workloads.DwPwCase("t", 8, 672, 14, 14, 3, 1, 1, 1, 112, True, seed=14)
    x, w, bd, F, bp = workloads.dwpw_inputs(case)
    ys = {}
    for split in ("1", "4"):
        monkeypatch.setenv("CONV_B200_DWPW_SPLIT", split)
        ys[split], _ = _run(cb, case, x, w, bd, F, bp, 0)
    ref, absum = oracle.dwpw(x, w, bd, workloads.bf16_to_f32(F), bp, 1, 1, 1, 0)
    for y in ys.values():
        assert np.all(np.abs(y - ref) <= _tol(case.C) * absum)
    assert not np.array_equal(ys["1"], ys["4"])


@pytest.mark.parametrize("form", list(GEMM_FORMS))
@pytest.mark.parametrize("hw,K", [(14, 3), (7, 5)])
def test_transposed_gemm_exact_mode_rounds_each_product(cb, hw, K, form, monkeypatch):
    # the depthwise stage's exact mode rounds every product and every sum (OneModel "Depthwise
    # convolution", "What each output is"): with F = I the block returns the bf16 depthwise
    # output, and two products that cancel only when rounded separately must give +0 (fast
    # mode: 2^-24, a bf16 value); zero inputs under negative taps give zeros
    from tests.test_depthwise_gpu import rounding_case
    _form(monkeypatch, form)
    C = 16
    x, w, (oy, ox) = rounding_case(C, hw, K)
    F = workloads.bf16_bits(np.eye(C, dtype=np.float32))
    case = workloads.DwPwCase("t", 1, C, hw, hw, K, 1, (K - 1) // 2, 1, C, False, seed=5)
    for mode in (0, 1):
        y, kernel = _run(cb, case, x, w, None, F, None, mode)
        assert kernel == "dwpw_gemm_kernel"
        dref = oracle.depthwise(x, w, None, mult=1, stride=1, pad=(K - 1) // 2, dil=1, mode=mode)
        assert np.array_equal(y, workloads.bf16_to_f32(workloads.bf16_bits(dref)).astype(np.float64))
        assert np.all(y[0, 0] == 0)
        assert y[0, 3, oy, ox] == (0.0 if mode == 0 else 2.0 ** -24)   # (the mixing sum's zero signs are the tensor cores')
