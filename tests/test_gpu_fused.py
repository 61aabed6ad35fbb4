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
    ("stem_cin4_n16_s2_fp6", O.ConvShape(16, 4, 16, 12, 12, 3, 3, 2, 1), "nvfp6"),   # CUDA-core dgrad
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


# ----------------------------------------------- quantized producer output

QCASES = [
    ("halo_n64_ragged_row", O.ConvShape(64, 64, 64, 6, 10, 3, 3, 1, 1), "nvfp4"),
    ("halo_n32_two_m_tiles_fp6", O.ConvShape(32, 128, 192, 5, 9, 3, 3, 1, 1), "nvfp6"),
    ("halo_multitile_1x1", O.ConvShape(16, 64, 64, 40, 40, 1, 1, 1, 0), "nvfp4"),
]


def _oracle_codes(q: "mqv.QTensor", fmt):
    return (O.unpack_codes(q.codes.cpu().numpy(), q.rows, q.cols, FMT[fmt]),
            q.scales.cpu().numpy().reshape(q.rows // 4, q.cols // 4), np.float32(q.tscale.item()))


def _assert_quantized(got: "mqv.QTensor", ref: O.QTensor, fmt, what):
    codes, scales, T = _oracle_codes(got, fmt)
    assert T == ref.T, what
    assert np.array_equal(scales, ref.scales), f"{what}: scales"
    assert np.array_equal(codes, ref.codes), f"{what}: {int(np.sum(codes != ref.codes))} codes differ"


@pytest.mark.parametrize("name,s,fmt", QCASES, ids=[c[0] for c in QCASES])
@pytest.mark.parametrize("amax_factor", [1.0, 0.5, 3.0])
def test_forward_writes_next_layer_input_quantized(name, s, fmt, amax_factor):
    """The forward epilogue quantizes ReLU(Y) into the next layer's X with T
    from a given max |x|: codes, scales and T equal the oracle's quantizer on
    the fp32 ReLU(Y) the fused pass stores, given that max (the true max,
    half of it, so that blocks saturate, and three times it); the reported
    max is this output's."""
    (X, Wt, G), d, qx, qw, qg = _quantized(s, fmt, name)
    y, amax = mqv.conv_fwd_fused(d, qw, qx, relu=True)
    t_amax = amax * amax_factor
    y_amax = torch.zeros(1, device="cuda")
    yq = mqv.conv_fwd_quantized(d, qw, qx, t_amax, relu=1, y_amax=y_amax)
    torch.cuda.synchronize()
    assert mqv.device_errors() == 0
    assert y_amax.item() == amax.item()
    ref = O.quantize(y.cpu().numpy().reshape(s.Ho * s.Wo * s.Cout, s.N), FMT[fmt], O.RNE,
                     amax=float(t_amax.item()))
    _assert_quantized(yq, ref, fmt, f"{name} fwd x{amax_factor}")
    if amax_factor == 1.0:      # the true max: the two-pass quantizer's codes
        two = mqv.quantize(y.view(-1), s.Ho * s.Wo * s.Cout, s.N, fmt, mqv.RNE)
        torch.cuda.synchronize()
        for f in ("codes", "scales", "tscale"):
            assert torch.equal(getattr(two, f), getattr(yq, f)), f


@pytest.mark.parametrize("name,s,fmt", QCASES, ids=[c[0] for c in QCASES])
def test_input_gradient_writes_quantized_with_stochastic_rounding(name, s, fmt):
    """The input-gradient epilogue quantizes G_X with stochastic rounding
    (the element's Philox word, the quantizer's numbering) and T from a given
    max: equal to the oracle's quantizer on the fp32 G_X of the plain pass."""
    (X, Wt, G), d, qx, qw, qg = _quantized(s, fmt, name)
    gx = mqv.conv_dgrad(d, qw, qg)
    t_amax = gx.abs().max().reshape(1) * 0.75
    gx_amax = torch.zeros(1, device="cuda")
    gq = mqv.conv_dgrad_quantized(d, qw, qg, t_amax, seed=1234, gx_amax=gx_amax)
    torch.cuda.synchronize()
    assert mqv.device_errors() == 0
    assert gx_amax.item() == gx.abs().max().item()
    ref = O.quantize(gx.cpu().numpy().reshape(s.H * s.W * s.Cin, s.N), FMT[fmt], O.SR, 1234,
                     amax=float(t_amax.item()))
    _assert_quantized(gq, ref, fmt, f"{name} dgrad")


def test_quantized_output_rejects_other_layers():
    s = O.ConvShape(8, 24, 40, 9, 9, 3, 3, 2, 1)          # stride 2: the generic kernel
    (X, Wt, G), d, qx, qw, qg = _quantized(s, "nvfp4", "reject")
    t = torch.ones(1, device="cuda")
    with pytest.raises(mqv.MqvError) as e:
        mqv.conv_fwd_quantized(d, qw, qx, t)
    assert e.value.status == 2
