"""Dependent calls back to back on one stream. Every kernel is launched with programmatic
dependent launch allowed and waits for its predecessors before touching global memory, so a
chain of convolutions -- each reading the previous one's output -- must give exactly the bits of
the same calls with a synchronisation between them, eagerly and inside a CUDA graph, and also
with the feature switched off (CONV_B200_PDL=0)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cb(cuda):
    import cnn_convolution_nhwc_b200 as m
    return m


def _dense_chain(cb, torch, X, Fs, sync):
    y = X
    for F in Fs:
        y = cb.conv2d_nhwc_fwd(y, F)
        if sync:
            torch.cuda.synchronize()
    return y


def _dw_chain(cb, torch, x, ws, F, sync):
    y = x
    for w in ws:
        y = cb.depthwise_fwd(y, w, None, pad=1, mode=cb.DW_EXACT)
        if sync:
            torch.cuda.synchronize()
    y = cb.dwpw_fwd(y, ws[0], None, F, None, pad=1, mode=cb.DW_EXACT)
    if sync:
        torch.cuda.synchronize()
    return y


def test_dependent_dense_calls_keep_stream_order(cb, monkeypatch):
    import torch
    g = torch.Generator(device="cuda").manual_seed(3)
    # 3x3 64->64 (folded-tap kernel), 1x1 64->128 (halo kernel), 5x5 128->128 (streamed filter,
    # CTA pairs), 3x3 128->64: each reads the previous output
    X = torch.randn((4, 40, 40, 64), device="cuda", generator=g).to(torch.bfloat16)
    shapes = [(3, 64, 64), (1, 64, 128), (5, 128, 128), (3, 128, 64)]
    Fs = [(torch.randn((k, k, ci, co), device="cuda", generator=g) / (k * k * ci) ** 0.5).to(torch.bfloat16)
          for k, ci, co in shapes]
    ref = _dense_chain(cb, torch, X, Fs, sync=True).float().cpu().numpy()
    eager = _dense_chain(cb, torch, X, Fs, sync=False)
    torch.cuda.synchronize()
    assert np.array_equal(eager.float().cpu().numpy(), ref)
    # the same chain captured in a graph and replayed
    _dense_chain(cb, torch, X, Fs, sync=False)   # first calls eagerly (one-time set-up)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        out = _dense_chain(cb, torch, X, Fs, sync=False)
    graph.replay()
    torch.cuda.synchronize()
    assert np.array_equal(out.float().cpu().numpy(), ref)
    monkeypatch.setenv("CONV_B200_PDL", "0")
    plain = _dense_chain(cb, torch, X, Fs, sync=False)
    torch.cuda.synchronize()
    assert np.array_equal(plain.float().cpu().numpy(), ref)
    assert cb.conv_device_status() == cb.CONV_OK


def test_dependent_depthwise_calls_keep_stream_order(cb):
    import torch
    g = torch.Generator(device="cuda").manual_seed(4)
    # 14x14 planes (plane kernel) twice, then the fused block on the result
    x = torch.rand((8, 64, 14, 14), device="cuda", generator=g) * 2 - 1
    ws = [torch.randn((64, 3, 3), device="cuda", generator=g) / 3 for _ in range(2)]
    F = (torch.randn((64, 32), device="cuda", generator=g) / 8).to(torch.bfloat16)
    ref = _dw_chain(cb, torch, x, ws, F, sync=True).cpu().numpy()
    eager = _dw_chain(cb, torch, x, ws, F, sync=False)
    torch.cuda.synchronize()
    assert np.array_equal(eager.cpu().numpy(), ref)
    assert cb.conv_device_status() == cb.CONV_OK
