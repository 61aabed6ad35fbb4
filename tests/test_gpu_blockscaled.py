"""GPU parity of the forward pass on the native block-scaled MMA
(mqv_conv_fwd_blockscaled: E2M1 codes with each 4-element block row padded
to a 16-element UE4M3 scale group) against the oracle, element by element on
small layers (several tiles a CTA, ragged output rows, two channel tiles)
and on sampled outputs of the full-size 28 x 28, N = 64 layer, where it is
also compared with the fp16-product forward pass."""
import zlib

import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
import workloads
from oracle import mqv_oracle as O
from tests.parity_utils import FMT, assert_close
from tests.test_gpu_conv import BandOracle, make_inputs

pytestmark = pytest.mark.gpu

SHAPES = [
    ("bs_n64_3x3_p1", O.ConvShape(64, 64, 64, 6, 10, 3, 3, 1, 1)),
    ("bs_n64_3x3_p0_c128", O.ConvShape(64, 128, 96, 7, 9, 3, 3, 1, 0)),
    ("bs_n128_3x2", O.ConvShape(128, 64, 64, 5, 6, 3, 2, 1, 0)),
    ("bs_n64_two_m_tiles", O.ConvShape(64, 64, 192, 5, 7, 3, 3, 1, 1)),
    ("bs_n128_1x1", O.ConvShape(128, 128, 64, 6, 6, 1, 1, 1, 0)),
    ("bs_n64_3x2_rect", O.ConvShape(64, 64, 64, 7, 6, 3, 2, 1, 1)),
    ("bs_multitile_n64", O.ConvShape(64, 64, 64, 40, 40, 3, 3, 1, 1)),
]


@pytest.mark.parametrize("name,s", SHAPES, ids=[c[0] for c in SHAPES])
def test_blockscaled_forward_matches_oracle(name, s):
    X, Wt, G = make_inputs(s, zlib.crc32(name.encode()) % 1000)
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, "nvfp4")
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), "nvfp4", mqv.RNE)
    qw = mqv.quantize(Wt.cuda().view(-1), *s.w_view(), "nvfp4", mqv.RNE)
    y = mqv.conv_fwd_blockscaled(d, qw, qx)
    y2 = mqv.conv_fwd_blockscaled(d, qw, qx)
    torch.cuda.synchronize()
    assert mqv.device_errors() == 0
    ox = O.quantize(X.numpy().reshape(s.x_view()), O.FP4, O.RNE)
    ow = O.quantize(Wt.numpy().reshape(s.w_view()), O.FP4, O.RNE)
    ref, S = O.conv_fwd(O.code_values(ow).reshape(Wt.shape), O.code_values(ox).reshape(X.shape), s)
    T = np.float64(ox.T) * np.float64(ow.T)
    assert_close(y.cpu().numpy(), ref * T, S * T, f"{name} block-scaled fwd")
    assert torch.equal(y, y2)


def test_blockscaled_forward_full_size_layer():
    """The 28 x 28, N = 64, 128 -> 128 layer: 48 sampled outputs against the
    oracle, and every output within twice the tolerance of the fp16-product
    forward pass."""
    layer = workloads.resnet18_layer2()
    s = O.ConvShape(layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.K, layer.K, layer.stride, layer.pad)
    X, Wt, _ = workloads.make_layer_inputs(layer)
    d = mqv.conv_desc(**layer.dims(), fmt="nvfp4")
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), "nvfp4", mqv.RNE)
    qw = mqv.quantize(Wt.cuda().view(-1), *s.w_view(), "nvfp4", mqv.RNE)
    yb = mqv.conv_fwd_blockscaled(d, qw, qx).cpu().numpy().reshape(s.Ho, s.Wo, s.Cout, s.N)
    yf = mqv.conv_fwd(d, qw, qx).cpu().numpy().reshape(s.Ho, s.Wo, s.Cout, s.N)
    assert mqv.device_errors() == 0
    ow = O.quantize(Wt.numpy().reshape(s.w_view()), O.FP4, O.RNE)
    Wcv = O.code_values(ow).reshape(s.Cout, s.Kh, s.Kw, s.Cin)
    bx = BandOracle(X.numpy(), O.FP4, O.RNE, 0)
    T = np.float64(ow.T) * np.float64(bx.T)
    rng = np.random.default_rng(5)
    got, ref, S, other = [], [], [], []
    for _ in range(48):
        ho, wo, co, n = (int(rng.integers(v)) for v in (s.Ho, s.Wo, s.Cout, s.N))
        acc = sacc = 0.0
        for kh in range(s.Kh):
            for kw in range(s.Kw):
                hi, wi = ho + kh - s.pad, wo + kw - s.pad
                if 0 <= hi < s.H and 0 <= wi < s.W:
                    p = Wcv[co, kh, kw, :] * bx.pix(hi, wi)[:, n]
                    acc += p.sum()
                    sacc += np.abs(p).sum()
        got.append(yb[ho, wo, co, n]); ref.append(acc * T); S.append(sacc * T); other.append(yf[ho, wo, co, n])
    assert_close(np.array(got), np.array(ref), np.array(S), "block-scaled fwd sampled")
    # both forms accumulate exact products in fp32, in different orders:
    # each lies within the tolerance of the exact value
    diff = np.abs(np.array(got, np.float64) - np.array(other, np.float64))
    assert np.all(diff <= 2 * (1e-5 * np.array(S) + 1e-7))
