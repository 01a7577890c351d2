"""The bounds-checked build (CONV_B200_DEBUG_BOUNDS=1): on valid inputs every kernel family gives
bit-identical results to the normal build and records no failed check; its failure path (a
check that fails without touching memory) sets CONV_ERR_DEVICE_BOUNDS and reports the site.

The cases run twice, in this process (normal library) and in a child process that imports the
package with CONV_B200_DEBUG_BOUNDS=1 (the bounds-checked library); the child saves its outputs
and the parent compares them element by element."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cb(cuda):
    import cnn_convolution_nhwc_b200 as m
    return m

# (name, environment for the call, call description)
CASES = [
    ("dense-direct", {"CONV_B200_DENSE": "direct"}, ("dense", (2, 11, 9, 12, 20, 3))),
    ("dense-fold", {}, ("dense", (2, 20, 18, 64, 64, 3))),
    ("dense-halo", {"CONV_B200_DENSE": "halo"}, ("dense", (2, 16, 16, 64, 128, 1))),
    ("dense-stream-pair", {"CONV_B200_DENSE": "stream"}, ("dense", (3, 21, 19, 64, 128, 5))),
    ("dense-stream-single", {"CONV_B200_DENSE": "stream", "CONV_B200_STREAM_PAIR": "0"},
     ("dense", (2, 16, 16, 64, 64, 3))),
    ("dense-im2col-tc", {"CONV_B200_DENSE": "bn128"}, ("dense", (4, 20, 20, 64, 136, 3))),   # X >= 128 KiB
    ("dense-grouped-bias", {}, ("grouped", (2, 16, 16, 128, 128, 3, 2))),
    ("dense-f32", {}, ("dense_f32", (2, 9, 9, 8, 12, 3))),
    ("dw-generic", {"CONV_B200_DW_GENERIC": "1"}, ("dw", (2, 8, 20, 18, 3, 1, 1, 2))),
    ("dw-reg", {"CONV_B200_DW_KERNEL": "reg"}, ("dw", (2, 8, 40, 40, 3, 1, 1, 1))),
    ("dw-tma", {"CONV_B200_DW_KERNEL": "tma"}, ("dw", (2, 8, 112, 112, 3, 2, 1, 1))),
    ("dw-plane", {}, ("dw", (4, 64, 14, 14, 3, 1, 1, 1))),
    ("dwpw-gemm", {}, ("dwpw", (4, 64, 14, 14, 3, 32))),
    ("dwpw-gemm-half-k5", {}, ("dwpw", (3, 136, 14, 14, 5, 48))),
    ("dwpw-gemm-cluster", {"CONV_B200_DWPW_HALF": "0"}, ("dwpw", (4, 128, 14, 14, 3, 32))),
    ("dwpw-gemm-7", {}, ("dwpw", (4, 96, 7, 7, 5, 160))),
    ("dwpw-staged", {"CONV_B200_DWPW_KERNEL": "staged"}, ("dwpw", (2, 64, 28, 28, 3, 32))),
    ("dwpw-flat", {"CONV_B200_DWPW_KERNEL": "flat"}, ("dwpw", (2, 64, 28, 28, 3, 32))),
    ("im2col-explicit", {}, ("im2col", (2, 12, 12, 16, 24, 3))),
]

CHILD = r'''
import json, os, sys
import numpy as np
import torch
sys.path.insert(0, os.environ["CONV_TEST_ROOT"])
import cnn_convolution_nhwc_b200 as cb
from tests.test_debug_bounds_gpu import CASES, run_case
assert cb.conv_debug_bounds_build(), "the bounds-checked library was not loaded"
out = {}
for name, env, call in CASES:
    out[name] = run_case(cb, torch, env, call)
    assert cb.conv_device_status() == cb.CONV_OK, name
    assert cb.conv_debug_bounds_info() is None, name
# the failure path: a check that fails and touches no memory
assert cb.conv_selftest_bounds() == cb.CONV_OK
assert cb.conv_device_status(reset=True) == cb.CONV_ERR_DEVICE_BOUNDS
info = cb.conv_debug_bounds_info(reset=True)
assert cb.conv_device_status() == cb.CONV_OK
np.savez(os.environ["CONV_TEST_OUT"], **out)
print(json.dumps({"selftest": list(info)}))
'''


def _rng(seed):
    return np.random.default_rng(seed)


def run_case(cb, torch, env, call):
    """One call of the library with `env` set for its duration; returns the output as numpy."""
    old = {k: os.environ.get(k) for k in env}
    os.environ.update(env)
    try:
        kind, a = call
        r = _rng(sum(kind.encode()) + sum(a))   # the same inputs in both processes
        dev = "cuda"
        if kind in ("dense", "dense_f32", "grouped", "im2col"):
            if kind == "grouped":
                N, H, W, Cin, Cout, K, g = a
                F = torch.tensor(r.standard_normal((K, K, Cin // g, Cout)), dtype=torch.float32)
            else:
                N, H, W, Cin, Cout, K = a
                F = torch.tensor(r.standard_normal((K, K, Cin, Cout)), dtype=torch.float32)
            X = torch.tensor(r.standard_normal((N, H, W, Cin)), dtype=torch.float32)
            if kind == "dense_f32":
                Y = cb.conv2d_nhwc_fwd_f32(X.to(dev), F.to(dev))
            elif kind == "grouped":
                b = torch.tensor(r.standard_normal(Cout), dtype=torch.float32).to(dev)
                Y = cb.conv2d_nhwc_fwd_grouped(X.to(dev, torch.bfloat16), F.to(dev, torch.bfloat16), b, pad=1,
                                               groups=g)
            elif kind == "im2col":
                Y = cb.conv2d_nhwc_fwd_im2col(X.to(dev, torch.bfloat16), F.to(dev, torch.bfloat16))
            else:
                Y = cb.conv2d_nhwc_fwd(X.to(dev, torch.bfloat16), F.to(dev, torch.bfloat16))
        elif kind == "dw":
            N, C, H, W, K, stride, pad, dil = a
            x = torch.tensor(r.standard_normal((N, C, H, W)), dtype=torch.float32).to(dev)
            w = torch.tensor(r.standard_normal((C, K, K)), dtype=torch.float32).to(dev)
            b = torch.tensor(r.standard_normal(C), dtype=torch.float32).to(dev)
            Y = cb.depthwise_fwd(x, w, b, stride=stride, pad=pad, dil=dil, mode=cb.DW_EXACT)
        else:
            N, C, H, W, K, Cout = a
            x = torch.tensor(r.standard_normal((N, C, H, W)), dtype=torch.float32).to(dev)
            w = torch.tensor(r.standard_normal((C, K, K)), dtype=torch.float32).to(dev)
            bd = torch.tensor(r.standard_normal(C), dtype=torch.float32).to(dev)
            F = torch.tensor(r.standard_normal((C, Cout)) / C ** 0.5, dtype=torch.float32).to(dev, torch.bfloat16)
            bp = torch.tensor(r.standard_normal(Cout), dtype=torch.float32).to(dev)
            Y = cb.dwpw_fwd(x, w, bd, F, bp, pad=(K - 1) // 2, mode=cb.DW_EXACT)
        torch.cuda.synchronize()
        return Y.float().cpu().numpy()
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def test_bounds_checked_build_matches_and_records_nothing(cb, tmp_path):
    import torch
    out = tmp_path / "debug_outputs.npz"
    env = dict(os.environ, CONV_B200_DEBUG_BOUNDS="1", CONV_TEST_ROOT=ROOT, CONV_TEST_OUT=str(out))
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    selftest = json.loads(r.stdout.strip().splitlines()[-1])["selftest"]
    assert selftest == [255, 1000, 1000]
    dbg = np.load(out)
    assert not cb.conv_debug_bounds_build()
    for name, env_c, call in CASES:
        y = run_case(cb, torch, env_c, call)
        assert np.array_equal(y, dbg[name], equal_nan=True), name


def test_normal_build_selftest_records_nothing(cb):
    # the same diagnostic in the normal build: the check is compiled out, nothing is recorded
    assert cb.conv_selftest_bounds() == cb.CONV_OK
    assert cb.conv_device_status() == cb.CONV_OK
    assert cb.conv_debug_bounds_info() is None
