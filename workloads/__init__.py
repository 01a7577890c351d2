"""Seeded synthetic inputs shared by the CUDA path's tests and benchmark and by the oracle.

This module holds no convolution arithmetic. It only draws numbers and stores them in
the layouts the two sides consume, so that both read identical bits:

* SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014) as a counter-based stream: value i of a stream with seed s is
  mix(s + (i + 1) * GAMMA).
* Uniform doubles in [0, 1) from the top 53 bits of each 64-bit value.
* Normals by the Box-Muller transform (Box and Muller, 1958), one pair per two uniforms.
* Round-to-nearest-even narrowing of float32 to bfloat16 bit patterns.

The workload table below describes the shapes and value distributions of the
configurations the library is tested and measured on. The dense shapes follow the
NHWC / KKIO contract of the CMU DLSys Lecture 14 notes ("The hidden copy behind
convolution as matrix multiplication", section 1); the depthwise sweep is the set of
MobileNetV3-large depthwise layers measured in the OneModel "Depthwise convolution"
page (section "Measured"), with batch 64 standing in for the unspecified batch.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Values offset .. offset+n-1 of the SplitMix64 stream with the given seed (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        return _mix(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * GAMMA)


def stream_seed(seed: int, tensor_id: int) -> int:
    """Seed of the independent stream used for one tensor of one workload."""
    with np.errstate(over="ignore"):
        z = _mix(np.array([(seed * 0x100000001B3 + tensor_id + 1) & 0xFFFFFFFFFFFFFFFF],
                          dtype=np.uint64))
    return int(z[0])


def uniform01(seed: int, n: int) -> np.ndarray:
    """n doubles in [0, 1): (value >> 11) * 2**-53."""
    out = np.empty(n, dtype=np.float64)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        out[s:s + m] = (splitmix64(seed, m, s) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return out


def uniform(seed: int, n: int, lo: float, hi: float) -> np.ndarray:
    """float32 samples of U(lo, hi)."""
    u = uniform01(seed, n)
    return (lo + (hi - lo) * u).astype(np.float32)


def normal(seed: int, n: int, std: float) -> np.ndarray:
    """float32 samples of N(0, std**2) by Box-Muller on consecutive uniform pairs."""
    out = np.empty(n, dtype=np.float32)
    pairs = (n + 1) // 2
    for s in range(0, pairs, _CHUNK):
        m = min(_CHUNK, pairs - s)
        u = (splitmix64(seed, 2 * m, 2 * s) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))
        t = 2.0 * math.pi * u2
        z = np.empty(2 * m, dtype=np.float64)
        z[0::2] = r * np.cos(t)
        z[1::2] = r * np.sin(t)
        lo = 2 * s
        hi = min(n, lo + 2 * m)
        out[lo:hi] = (std * z[: hi - lo]).astype(np.float32)
    return out


def int_uniform(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """float32 holding integers drawn uniformly from lo..hi inclusive."""
    u = uniform01(seed, n)
    k = np.floor(u * (hi - lo + 1)).astype(np.int64) + lo
    return k.astype(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest-even; returns the uint16 bit patterns (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------------------
# Workload table
# ----------------------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class DenseCase:
    """Dense NHWC forward convolution: X[N,H,W,Cin], F[K,K,Cin,Cout] (KKIO), Y[N,Ho,Wo,Cout]."""
    name: str
    N: int
    H: int
    W: int
    Cin: int
    Cout: int
    K: int
    dtype: str          # "bf16" or "f32": storage type of X, F and Y
    dist: str           # "normal" (X~N(0,1), F~N(0,1/(K*K*Cin))) or "int3" (integers in [-3,3])
    seed: int = 0
    stride: int = 1
    pad: int = 0
    dil: int = 1
    bias: bool = False  # a float32 bias[Cout] ~ N(0, 0.1)
    groups: int = 1     # channel groups: F is [KH, KW, Cin/groups, Cout]
    KW: int = 0         # filter width when it differs from K (K is then the height)
    stride_w: int = 0   # width-axis stride, padding, dilation when they differ (0 / -1: as the
    pad_w: int = -1     # height axis)
    dil_w: int = 0
    pad_w_end: int = -1 # width-axis padding after the last column when it differs (-1: pad_w)

    @property
    def kh(self) -> int:
        return self.K

    @property
    def kw(self) -> int:
        return self.KW or self.K

    @property
    def sw(self) -> int:
        return self.stride_w or self.stride

    @property
    def pw(self) -> int:
        return self.pad if self.pad_w < 0 else self.pad_w

    @property
    def pwe(self) -> int:
        return self.pw if self.pad_w_end < 0 else self.pad_w_end

    @property
    def dw(self) -> int:
        return self.dil_w or self.dil

    @property
    def pads(self):
        """((top, bottom), (left, right)) zero padding."""
        return (self.pad, self.pad), (self.pw, self.pwe)

    @property
    def cin_g(self) -> int:
        return self.Cin // self.groups

    @property
    def square(self) -> bool:
        """One K, one stride, padding and dilation for both axes, one group."""
        return self.kw == self.K and self.sw == self.stride and self.pw == self.pad and self.pwe == self.pw and \
            self.dw == self.dil and self.groups == 1

    @property
    def f_shape(self):
        return (self.kh, self.kw, self.cin_g, self.Cout)

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - (self.dil * (self.kh - 1) + 1)) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + self.pw + self.pwe - (self.dw * (self.kw - 1) + 1)) // self.sw + 1

    @property
    def flops(self) -> int:
        return 2 * self.N * self.Ho * self.Wo * self.Cout * self.kh * self.kw * self.cin_g

    @property
    def bytes(self) -> int:
        e = 2 if self.dtype == "bf16" else 4
        return e * (self.N * self.H * self.W * self.Cin + self.kh * self.kw * self.cin_g * self.Cout
                    + self.N * self.Ho * self.Wo * self.Cout) + (4 * self.Cout if self.bias else 0)


@dataclasses.dataclass(frozen=True)
class DepthwiseCase:
    """Depthwise forward convolution on NCHW float32 planes, Cout = Cin * mult."""
    name: str
    N: int
    C: int
    mult: int
    H: int
    W: int
    KH: int
    KW: int
    stride: int
    pad: int
    dil: int
    bias: bool = True
    seed: int = 0

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - (self.dil * (self.KH - 1) + 1)) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad - (self.dil * (self.KW - 1) + 1)) // self.stride + 1

    @property
    def flops(self) -> int:
        return 2 * self.KH * self.KW * self.N * self.C * self.mult * self.Ho * self.Wo

    @property
    def bytes(self) -> int:
        co = self.C * self.mult
        return 4 * (self.N * self.C * self.H * self.W + co * self.KH * self.KW
                    + (co if self.bias else 0) + self.N * co * self.Ho * self.Wo)


@dataclasses.dataclass(frozen=True)
class DwPwCase:
    """Depthwise K x K (multiplier 1) on NCHW float32 planes, then pointwise C -> Cout with
    bfloat16 weights F[C][Cout]; y float32 NCHW [N][Cout][Ho][Wo]."""
    name: str
    N: int
    C: int
    H: int
    W: int
    K: int
    stride: int
    pad: int
    dil: int
    Cout: int
    bias: bool = True   # both biases present
    seed: int = 0

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - (self.dil * (self.K - 1) + 1)) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad - (self.dil * (self.K - 1) + 1)) // self.stride + 1

    @property
    def flops(self) -> int:
        pix = self.N * self.Ho * self.Wo
        return 2 * pix * self.C * self.K * self.K + 2 * pix * self.C * self.Cout

    @property
    def bytes(self) -> int:
        b = 4 * (self.N * self.C * self.H * self.W + self.C * self.K * self.K + self.N * self.Cout * self.Ho * self.Wo)
        b += 2 * self.C * self.Cout
        if self.bias:
            b += 4 * (self.C + self.Cout)
        return b


def dwpw_inputs(case: DwPwCase):
    """Seeded x ~ U(-1, 1), w ~ N(0, 1/K^2), F ~ N(0, 1/C) as bf16 bits, biases ~ N(0, 0.1)."""
    s = [stream_seed(case.seed, i) for i in range(5)]
    x = uniform(s[0], case.N * case.C * case.H * case.W, -1.0, 1.0).reshape(case.N, case.C, case.H, case.W)
    w = normal(s[1], case.C * case.K * case.K, 1.0 / case.K).reshape(case.C, case.K, case.K)
    F = bf16_bits(normal(s[2], case.C * case.Cout, 1.0 / math.sqrt(case.C)).reshape(case.C, case.Cout))
    bd = normal(s[3], case.C, math.sqrt(0.1)) if case.bias else None
    bp = normal(s[4], case.Cout, math.sqrt(0.1)) if case.bias else None
    return x, w, bd, F, bp


DENSE_TINY = DenseCase("tiny dense fp32 N2 H8 W8 Cin4 Cout8 K3", 2, 8, 8, 4, 8, 3, "f32", "int3", 0)
DENSE_3X3 = DenseCase("dense bf16 N32 H56 W56 Cin64 Cout64 K3", 32, 56, 56, 64, 64, 3, "bf16", "normal", 0)
DENSE_1X1 = DenseCase("pointwise bf16 N32 H28 W28 Cin256 Cout512 K1", 32, 28, 28, 256, 512, 1, "bf16",
                      "normal", 0)
DENSE_LARGE = DenseCase("large dense bf16 N64 H112 W112 Cin128 Cout128 K5", 64, 112, 112, 128, 128, 5,
                        "bf16", "normal", 0)

# stride-2 3x3 layer with "same" padding and a bias (a ResNet stage transition, 56 -> 28)
DENSE_S2 = DenseCase("dense bf16 N32 H56 W56 Cin64 Cout128 K3 s2 p1 bias", 32, 56, 56, 64, 128, 3, "bf16", "normal", 0,
                     stride=2, pad=1, bias=True)
# grouped 3x3 layer, 4 groups of 64 channels (a RegNet-style group width) with a bias
DENSE_GROUPED = DenseCase("grouped bf16 N32 H28 W28 Cin256 Cout256 K3 p1 g4 bias", 32, 28, 28, 256, 256, 3, "bf16",
                          "normal", 0, pad=1, bias=True, groups=4)
# Conv1D audio stem over 3000 log-mel frames (30 s at 10 ms), batch 16, width 512: the first
# layer mixes nearby frames (80 -> 512, K 3, pad 1), the second halves the frame rate
# (512 -> 512, K 3, stride 2, pad 1); both with a bias. A sequence is one image row (H = 1).
CONV1D_STEM1 = DenseCase("conv1d bf16 N16 L3000 Cin80 Cout512 K3 p1 bias", 16, 1, 3000, 80, 512, 1, "bf16", "normal",
                         0, bias=True, KW=3, pad_w=1)
CONV1D_STEM2 = DenseCase("conv1d bf16 N16 L3000 Cin512 Cout512 K3 s2 p1 bias", 16, 1, 3000, 512, 512, 1, "bf16",
                         "normal", 0, bias=True, KW=3, stride_w=2, pad_w=1)
# the causal form of the second layer's channel mixing: 512 -> 512, K 3, stride 1, padded only
# before the sequence (2 frames), so a frame's output reads no later frame; with a bias
CONV1D_CAUSAL = DenseCase("conv1d bf16 N16 L3000 Cin512 Cout512 K3 causal bias", 16, 1, 3000, 512, 512, 1, "bf16",
                          "normal", 0, bias=True, KW=3, pad_w=2, pad_w_end=0)
# depthwise then pointwise blocks (MobileNetV3-large shapes): 672 channels at 14x14, 3x3, into
# 112 outputs; 960 channels at 7x7, 5x5, into 160 outputs; batch 64, both biases
DWPW_BLOCKS = [DwPwCase("dwpw C672 K3 s1 H14 Cout112", 64, 672, 14, 14, 3, 1, 1, 1, 112),
               DwPwCase("dwpw C960 K5 s1 H7 Cout160", 64, 960, 7, 7, 5, 1, 2, 1, 160)]
# MobileNetV3-large depthwise layers (C, K, stride, input H=W), batch 64, multiplier 1,
# pad (K-1)/2, dilation 1.
DW_LAYERS = [(16, 3, 1, 112), (64, 3, 2, 112), (72, 5, 2, 56), (120, 5, 1, 28), (672, 3, 1, 14),
             (960, 5, 1, 7)]
DW_SWEEP = [DepthwiseCase(f"depthwise C{c} K{k} s{s} H{h}", 64, c, 1, h, h, k, k, s, (k - 1) // 2, 1,
                          True, 0) for (c, k, s, h) in DW_LAYERS]


def dense_bias(case: DenseCase):
    """Seeded float32 bias[Cout] ~ N(0, 0.1) of a case with a bias (None otherwise)."""
    if not case.bias:
        return None
    return normal(stream_seed(case.seed, 2), case.Cout, math.sqrt(0.1))


def dense_inputs(case: DenseCase):
    """Seeded X (NHWC) and F (KKIO; [KH, KW, Cin/groups, Cout] for a grouped case).

    Returns (X, F) as uint16 bf16 bit patterns for bf16 cases, float32 arrays otherwise.
    """
    nx = case.N * case.H * case.W * case.Cin
    nf = case.kh * case.kw * case.cin_g * case.Cout
    sx, sf = stream_seed(case.seed, 0), stream_seed(case.seed, 1)
    if case.dist == "int3":
        X = int_uniform(sx, nx, -3, 3)
        F = int_uniform(sf, nf, -3, 3)
    elif case.dist == "normal":
        X = normal(sx, nx, 1.0)
        F = normal(sf, nf, 1.0 / math.sqrt(case.kh * case.kw * case.cin_g))
    else:
        raise ValueError(case.dist)
    X = X.reshape(case.N, case.H, case.W, case.Cin)
    F = F.reshape(case.f_shape)
    if case.dtype == "bf16":
        return bf16_bits(X), bf16_bits(F)
    return X, F


def depthwise_inputs(case: DepthwiseCase):
    """Seeded x (NCHW), w ([C*mult][KH][KW]) and bias ([C*mult] or None), float32.

    x ~ U(-1, 1), w ~ N(0, 1/(KH*KW)), bias ~ N(0, 0.1) with 0.1 read as the variance.
    """
    co = case.C * case.mult
    x = uniform(stream_seed(case.seed, 0), case.N * case.C * case.H * case.W, -1.0, 1.0)
    w = normal(stream_seed(case.seed, 1), co * case.KH * case.KW, 1.0 / math.sqrt(case.KH * case.KW))
    b = normal(stream_seed(case.seed, 2), co, math.sqrt(0.1)) if case.bias else None
    return (x.reshape(case.N, case.C, case.H, case.W), w.reshape(co, case.KH, case.KW), b)
