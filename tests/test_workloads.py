"""The seeded input generators: published reference values and library cross-checks."""
import numpy as np
import torch

import workloads


def test_splitmix64_reference_stream():
    # SplitMix64 with state 0: the first outputs of the published generator
    z = workloads.splitmix64(0, 3)
    assert [hex(int(v)) for v in z] == ["0xe220a8397b1dcdaf", "0x6e789e6aa1b965f4", "0x6c45d188009454f"]


def test_splitmix64_is_counter_based():
    a = workloads.splitmix64(1234, 100)
    b = workloads.splitmix64(1234, 40, offset=60)
    assert np.array_equal(a[60:], b)


def test_bf16_rounding_matches_torch():
    x = workloads.normal(5, 1 << 16, 3.0)
    # add exact ties: low 16 bits 0x8000 with even and odd kept parts
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40490FDB], np.uint32).view(np.float32)
    x = np.concatenate([x, ties])
    ours = workloads.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(workloads.bf16_to_f32(ours), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_normal_and_uniform_moments():
    z = workloads.normal(9, 1 << 20, 2.0).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 2.0) < 0.01
    u = workloads.uniform(9, 1 << 20, -1, 1).astype(np.float64)
    assert u.min() >= -1 and u.max() < 1 and abs(u.mean()) < 0.01
    k = workloads.int_uniform(9, 1 << 16, -3, 3)
    assert set(np.unique(k).tolist()) == set(range(-3, 4))


def test_workload_shapes():
    c = workloads.DENSE_3X3
    assert (c.Ho, c.Wo) == (54, 54) and c.flops == 2 * 32 * 54 * 54 * 64 * 9 * 64
    assert [d.Ho for d in workloads.DW_SWEEP] == [112, 56, 28, 28, 14, 7]
    X, F = workloads.dense_inputs(workloads.DENSE_TINY)
    assert X.shape == (2, 8, 8, 4) and F.shape == (3, 3, 4, 8) and X.dtype == np.float32
    assert set(np.unique(X).tolist()) <= set(range(-3, 4))
    x, w, b = workloads.depthwise_inputs(workloads.DW_SWEEP[0])
    assert x.shape == (64, 16, 112, 112) and w.shape == (16, 3, 3) and b.shape == (16,)


def test_grouped_and_conv1d_case_shapes():
    c = workloads.DENSE_GROUPED
    assert c.f_shape == (3, 3, 64, 256) and (c.Ho, c.Wo) == (28, 28) and not c.square
    assert c.flops == 2 * 32 * 28 * 28 * 256 * 9 * 64
    s1, s2 = workloads.CONV1D_STEM1, workloads.CONV1D_STEM2
    assert s1.f_shape == (1, 3, 80, 512) and (s1.Ho, s1.Wo) == (1, 3000)
    assert s2.f_shape == (1, 3, 512, 512) and (s2.Ho, s2.Wo) == (1, 1500)
    assert workloads.DENSE_S2.square and workloads.DENSE_S2.f_shape == (3, 3, 64, 128)


def test_depthwise_pointwise_blocks():
    # algorithmic bytes: x, y (float32), depthwise weights and both biases (float32), pointwise
    # weights (bf16); the intermediate is not counted
    c = workloads.DWPW_BLOCKS[0]
    assert (c.Ho, c.Wo) == (14, 14)
    assert c.bytes == 4 * (64 * 672 * 196 + 672 * 9 + 64 * 112 * 196) + 2 * 672 * 112 + 4 * (672 + 112)
    assert c.flops == 2 * 64 * 196 * 672 * 9 + 2 * 64 * 196 * 672 * 112
    x, w, bd, F, bp = workloads.dwpw_inputs(workloads.DwPwCase("t", 2, 8, 5, 5, 3, 1, 1, 1, 16, True, seed=3))
    assert x.shape == (2, 8, 5, 5) and w.shape == (8, 3, 3) and F.shape == (8, 16) and F.dtype.name == "uint16"
    assert bd.shape == (8,) and bp.shape == (16,)
    assert float(np.abs(x).max()) <= 1.0
    x2, *_ = workloads.dwpw_inputs(workloads.DwPwCase("t", 2, 8, 5, 5, 3, 1, 1, 1, 16, True, seed=3))
    assert np.array_equal(x, x2)   # seeded: the same bits every time
