"""The allocation-free weight-gradient entry point.

Some callers cannot allocate device memory at all (their device memory is
owned by a fixed pool they may not grow, or they have no allocator to ask for
a workspace).  mqv_conv_wgrad_noalloc serves them: its split-K partial sums go
to a fixed 32 MiB array inside the library instead of a caller workspace.
These tests call it through the C ABI and check it against mqv_conv_wgrad
(the allocating entry point) within the parity tolerance, twice in a row,
since the array keeps the previous call's contents.  This file is collected
last so that a failure here cannot hide the results of the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
import workloads
from oracle import mqv_oracle as O

pytestmark = pytest.mark.gpu


def _layer_case(layer: workloads.Layer):
    s = O.ConvShape(layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.K, layer.K,
                    layer.stride, layer.pad)
    X, Wt, G = workloads.make_layer_inputs(layer)
    seed = workloads.sr_seed(layer)
    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), layer.fmt, mqv.RNE)
    qg = mqv.quantize(G.cuda().view(-1), *s.gy_view(), layer.fmt, mqv.SR, seed)
    # tolerance bound S = T_g·T_x·sum |g·x| from the oracle's own quantization
    f = O.FP4 if layer.fmt == "nvfp4" else O.FP6
    ox = O.quantize(X.numpy().reshape(s.x_view()), f, O.RNE)
    og = O.quantize(G.numpy().reshape(s.gy_view()), f, O.SR, seed)
    _, S = O.conv_wgrad(O.code_values(og).reshape(G.shape), O.code_values(ox).reshape(X.shape), s)
    S = S * np.float64(ox.T) * np.float64(og.T)
    return d, qx, qg, S


def _call_noalloc(d, qg, qx, gw):
    gc, xc = qg.c(), qx.c()
    return mqv.lib().mqv_conv_wgrad_noalloc(ctypes.byref(d), ctypes.byref(gc), ctypes.byref(xc),
                                            gw.data_ptr(), torch.cuda.current_stream().cuda_stream)


LAYERS = [workloads.tiny_layer(),
          workloads.Layer("mid_3x3_c64_n16", 16, 64, 64, 14, 14, 3, 1, 1, "nvfp6", "relu", 1e-4, 3),
          workloads.resnet18_layer2()]


@pytest.mark.parametrize("layer", LAYERS, ids=[l.name for l in LAYERS])
def test_noalloc_wgrad_matches_allocating_entry_point(layer):
    d, qx, qg, S = _layer_case(layer)
    ref = mqv.conv_wgrad(d, qg, qx).cpu().numpy().astype(np.float64).reshape(S.shape)
    assert mqv.conv_workspace_bytes(d, mqv.OP_WGRAD) <= 32 << 20
    lim = 1e-5 * S + 1e-7
    for call in range(2):                       # the scratch keeps the last call's data
        gw = torch.full((d.Cout, d.Kh, d.Kw, d.Cin), float("nan"), device="cuda")
        st = _call_noalloc(d, qg, qx, gw)
        assert st == 0, mqv.lib().mqv_last_error()
        torch.cuda.synchronize()
        got = gw.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= lim), f"call {call}: max err/S {np.max(np.abs(got - ref) / (S + 1e-30))}"
    assert mqv.device_errors() == 0


def test_noalloc_wgrad_after_other_layer_reuses_scratch():
    """A small call after a big one must not read the big call's partials."""
    big = _layer_case(LAYERS[2])
    small = _layer_case(LAYERS[1])
    gw_big = torch.empty((big[0].Cout, big[0].Kh, big[0].Kw, big[0].Cin), device="cuda")
    assert _call_noalloc(big[0], big[2], big[1], gw_big) == 0
    d, qx, qg, S = small
    gw = torch.empty((d.Cout, d.Kh, d.Kw, d.Cin), device="cuda")
    assert _call_noalloc(d, qg, qx, gw) == 0
    ref = mqv.conv_wgrad(d, qg, qx).cpu().numpy().astype(np.float64).reshape(S.shape)
    got = gw.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-5 * S + 1e-7)
