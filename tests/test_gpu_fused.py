"""GPU parity of the fused producer epilogues: the forward pass with optional
ReLU and max|y| folded into its epilogue, and the input-gradient pass with
max|g_x|.  The stored outputs must equal the plain passes' outputs bit for bit
(after ReLU where asked), the fused maximum must equal max|.| of what was
stored, and quantizing with it must give the codes of the two-pass
quantizer; the outputs themselves are checked against the oracle within the
parity tolerance."""
import zlib

import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
import workloads
from oracle import mqv_oracle as O
from tests.parity_utils import FMT, assert_close
from tests.test_gpu_conv import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny_3x3_s1_p0", O.ConvShape(4, 16, 16, 8, 8, 3, 3, 1, 0), "nvfp4"),       # generic kernel
    ("ragged_3x3_s2_p1", O.ConvShape(8, 24, 40, 9, 9, 3, 3, 2, 1), "nvfp4"),     # strided
    ("cin4_3x3_s2_fp6", O.ConvShape(4, 4, 16, 12, 12, 3, 3, 2, 1), "nvfp6"),
    ("halo_n64_ragged_row", O.ConvShape(64, 64, 64, 6, 10, 3, 3, 1, 1), "nvfp4"),  # halo kernel
    ("halo_n32_two_m_tiles", O.ConvShape(32, 128, 192, 5, 9, 3, 3, 1, 1), "nvfp6"),
]


def _quantized(s, fmt, name):
    X, Wt, G = make_inputs(s, zlib.crc32(name.encode()) % 1000)
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, fmt)
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), fmt, mqv.RNE)
    qw = mqv.quantize(Wt.cuda().view(-1), *s.w_view(), fmt, mqv.RNE)
    qg = mqv.quantize(G.cuda().view(-1), *s.gy_view(), fmt, mqv.SR, 5)
    return (X, Wt, G), d, qx, qw, qg


def _same_codes(t, rows, cols, fmt, rnd, seed, amax):
    a = mqv.quantize(t.view(-1), rows, cols, fmt, rnd, seed)
    b = mqv.quantize_with_amax(t.view(-1), rows, cols, fmt, rnd, seed, amax)
    torch.cuda.synchronize()
    for f in ("codes", "scales", "tscale"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f


@pytest.mark.parametrize("name,s,fmt", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("relu", [False, True])
def test_fused_forward(name, s, fmt, relu):
    (X, Wt, G), d, qx, qw, qg = _quantized(s, fmt, name)
    y_plain = mqv.conv_fwd(d, qw, qx)
    y, amax = mqv.conv_fwd_fused(d, qw, qx, relu=relu)
    torch.cuda.synchronize()
    want = torch.where(y_plain > 0, y_plain, torch.zeros_like(y_plain)) if relu else y_plain
    assert torch.equal(y, want)
    assert amax.item() == y.abs().max().item()
    if relu:
        assert bool((y >= 0).all()) and not bool(torch.signbit(y).any())
    _same_codes(y, s.Ho * s.Wo * s.Cout, s.N, fmt, mqv.RNE, 0, amax)
    # the stored values against the oracle's convolution
    oq = O.quantize_layer(X.numpy(), Wt.numpy(), G.numpy(), s, FMT[fmt], 5)
    yr, S = O.layer_outputs(*oq, s)["y"]
    assert_close(y.cpu().numpy(), np.maximum(yr, 0) if relu else yr, S, f"{name} fused fwd")
    assert mqv.device_errors() == 0


@pytest.mark.parametrize("name,s,fmt", CASES, ids=[c[0] for c in CASES])
def test_fused_input_gradient(name, s, fmt):
    (X, Wt, G), d, qx, qw, qg = _quantized(s, fmt, name)
    gx_plain = mqv.conv_dgrad(d, qw, qg)
    gx, amax = mqv.conv_dgrad_fused(d, qw, qg)
    torch.cuda.synchronize()
    assert torch.equal(gx, gx_plain)
    assert amax.item() == gx.abs().max().item()
    _same_codes(gx, s.H * s.W * s.Cin, s.N, fmt, mqv.SR, 9, amax)
    assert mqv.device_errors() == 0


def test_fused_maximum_is_cleared_by_each_call():
    """A second call with a smaller output does not keep the first call's max."""
    s = O.ConvShape(64, 64, 64, 6, 10, 3, 3, 1, 1)
    (X, Wt, G), d, qx, qw, qg = _quantized(s, "nvfp4", "clear")
    big = mqv.quantize((X * 1000).cuda().view(-1), *s.x_view(), "nvfp4", mqv.RNE)
    amax = torch.full((1,), 123.0, device="cuda")
    y1, _ = mqv.conv_fwd_fused(d, qw, big, y_amax=amax)
    a1 = amax.item()
    y2, _ = mqv.conv_fwd_fused(d, qw, qx, y_amax=amax)
    torch.cuda.synchronize()
    assert a1 == y1.abs().max().item()
    assert amax.item() == y2.abs().max().item() < a1


def test_full_size_layer_fused_forward_and_next_quantization():
    """The benchmarked 28x28, N = 64 layer: fused ReLU + max against the plain
    pass, then the next layer's one-pass quantization of the ReLU output."""
    layer = workloads.resnet18_layer2()
    s = O.ConvShape(layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.K, layer.K, layer.stride, layer.pad)
    X, Wt, G = workloads.make_layer_inputs(layer)
    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), layer.fmt, mqv.RNE)
    qw = mqv.quantize(Wt.cuda().view(-1), *s.w_view(), layer.fmt, mqv.RNE)
    y_plain = mqv.conv_fwd(d, qw, qx)
    y, amax = mqv.conv_fwd_fused(d, qw, qx, relu=True)
    torch.cuda.synchronize()
    assert torch.equal(y, torch.relu(y_plain))
    assert amax.item() == y.max().item()
    _same_codes(y, s.Ho * s.Wo * s.Cout, s.N, layer.fmt, mqv.RNE, 0, amax)


@pytest.mark.parametrize("idx", [1, 3])
def test_full_size_yolo_layers_fused_passes(idx):
    """NVFP6 stride-2 layers of the YOLOv8n-shaped mix (the generic kernel on
    transposed tiles, the input gradient grouped by pixel parity): fused
    forward with ReLU and fused input gradient against the plain passes."""
    layer = workloads.yolov8n_mix()[idx]
    s = O.ConvShape(layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.K, layer.K, layer.stride, layer.pad)
    X, Wt, G = workloads.make_layer_inputs(layer)
    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), layer.fmt, mqv.RNE)
    qw = mqv.quantize(Wt.cuda().view(-1), *s.w_view(), layer.fmt, mqv.RNE)
    qg = mqv.quantize(G.cuda().view(-1), *s.gy_view(), layer.fmt, mqv.SR, workloads.sr_seed(layer))
    y_plain = mqv.conv_fwd(d, qw, qx)
    y, ya = mqv.conv_fwd_fused(d, qw, qx, relu=True)
    gx_plain = mqv.conv_dgrad(d, qw, qg)
    gx, ga = mqv.conv_dgrad_fused(d, qw, qg)
    torch.cuda.synchronize()
    assert torch.equal(y, torch.relu(y_plain)) and ya.item() == y.max().item()
    assert torch.equal(gx, gx_plain) and ga.item() == gx.abs().max().item()
    assert mqv.device_errors() == 0
