"""GPU parity of the quantize-after-im2col baseline (section "무엇인가" of the
MicroQonv summary) built from mqv_im2col, the quantizer, 1 x 1 convolutions
and mqv_col2im, against the oracle running the same flow.

The scheme itself ("line" blocks): every GEMM operand quantized with
16-element blocks along that GEMM's contraction, one copy per direction; the
six copies are compared byte for byte with `oracle.naive_layer` and the
outputs within the parity tolerance.  The square-block variant (4 x 4 blocks
over (kh·kw·ci, n) of the expanded tensor, every duplicate of a pixel given
the codes of the original block) is checked under its own name, and for
padded stride-1 layers it matches the quantize-once path."""
import zlib

import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
from microscaling_quantized_convolution_b200 import naive
from oracle import mqv_oracle as O
from tests.parity_utils import FMT, assert_close

pytestmark = pytest.mark.gpu

SHAPES = [
    ("n8_3x3_s1_p1", O.ConvShape(8, 16, 12, 7, 6, 3, 3, 1, 1), "nvfp4"),
    ("n4_3x3_s2_p1", O.ConvShape(4, 8, 16, 9, 9, 3, 3, 2, 1), "nvfp4"),
    ("n16_5x5_s1_p2_fp6", O.ConvShape(16, 8, 8, 6, 6, 5, 5, 1, 2), "nvfp6"),
    ("n64_3x3_s1_p1", O.ConvShape(64, 64, 64, 6, 6, 3, 3, 1, 1), "nvfp4"),
]


def _inputs(s: O.ConvShape, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.relu(torch.randn((s.H, s.W, s.Cin, s.N), generator=g))
    Wt = torch.randn((s.Cout, s.Kh, s.Kw, s.Cin), generator=g) * (2.0 / (s.Cin * s.Kh * s.Kw)) ** 0.5
    G = torch.randn((s.Ho, s.Wo, s.Cout, s.N), generator=g) * 1e-3
    return X, Wt, G


def _cbf(cols: np.ndarray, s: O.ConvShape) -> np.ndarray:
    """(K, (ho, wo, n)) -> [Ho][Wo][K][N]."""
    K = s.Kh * s.Kw * s.Cin
    return cols.reshape(K, s.Ho, s.Wo, s.N).transpose(1, 2, 0, 3)


@pytest.mark.parametrize("name,s,fmt", SHAPES, ids=[c[0] for c in SHAPES])
def test_im2col_and_col2im(name, s, fmt):
    X, _, _ = _inputs(s, zlib.crc32(name.encode()) % 997)
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, fmt)
    xc = mqv.im2col(d, X.cuda()).cpu().numpy()
    ref = _cbf(O.im2col(X.numpy(), s), s)
    assert np.array_equal(xc, ref)                          # a copy: bit-exact
    gc = torch.randn(xc.shape, generator=torch.Generator().manual_seed(3))
    gx = mqv.col2im(d, gc.cuda()).cpu().numpy().astype(np.float64)
    K = s.Kh * s.Kw * s.Cin
    cols = gc.numpy().astype(np.float64).transpose(2, 0, 1, 3).reshape(K, -1)
    gref = O.col2im(cols, s)
    Sref = O.col2im(np.abs(cols), s)
    assert np.all(np.abs(gx - gref) <= 1e-6 * Sref + 1e-12)   # at most Kh·Kw fp32 additions


@pytest.mark.parametrize("name,s,fmt", SHAPES, ids=[c[0] for c in SHAPES])
def test_square_variant_matches_oracle(name, s, fmt):
    X, Wt, G = _inputs(s, zlib.crc32(name.encode()) % 997 + 1)
    seed = 11
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, fmt)
    p = naive.plan(d, blocks="square")
    y = torch.empty((s.Ho, s.Wo, s.Cout, s.N), device="cuda")
    gw = torch.empty((s.Cout, s.Kh, s.Kw, s.Cin), device="cuda")
    gx = torch.empty((s.H, s.W, s.Cin, s.N), device="cuda")
    naive.step(p, X.cuda().contiguous(), Wt.cuda().contiguous(), G.cuda().contiguous(), seed, y, gw, gx)
    assert mqv.device_errors() == 0
    # oracle: the same flow (expanded X quantized with 4 x 4 blocks, a 1 x 1
    # convolution per GEMM, col2im of the expanded input gradient)
    f = FMT[fmt]
    K = s.Kh * s.Kw * s.Cin
    s1 = O.ConvShape(s.N, K, s.Cout, s.Ho, s.Wo, 1, 1, 1, 0)
    xc = _cbf(O.im2col(X.numpy(), s), s)
    qx = O.quantize(xc.reshape(-1, s.N), f, O.RNE)
    qw = O.quantize(Wt.numpy().reshape(s.Cout, K), f, O.RNE)
    qg = O.quantize(G.numpy().reshape(-1, s.N), f, O.SR, seed)
    # the GPU's own copies of each direction are bit-identical to these
    for key, ref in (("x_fwd", qx), ("x_wgrad", qx), ("w_fwd", qw), ("w_dgrad", qw), ("g_wgrad", qg), ("g_dgrad", qg)):
        got = p.q[key]
        assert np.float32(got.tscale.item()) == np.float32(ref.T), key
        assert np.array_equal(got.scales.cpu().numpy(), ref.scales.reshape(-1)), key
    Xv = O.code_values(qx).reshape(s.Ho, s.Wo, K, s.N)
    Wv = O.code_values(qw).reshape(s.Cout, 1, 1, K)
    Gv = O.code_values(qg).reshape(s.Ho, s.Wo, s.Cout, s.N)
    Tx, Tw, Tg = (np.float64(q.T) for q in (qx, qw, qg))
    yr, ys = O.conv_fwd(Wv, Xv, s1)
    assert_close(y.cpu().numpy(), yr * Tw * Tx, ys * Tw * Tx, f"{name} naive fwd")
    gwr, gws = O.conv_wgrad(Gv, Xv, s1)
    assert_close(gw.cpu().numpy().reshape(gwr.shape), gwr * Tg * Tx, gws * Tg * Tx, f"{name} naive wgrad")
    gcr, gcs = O.conv_dgrad(Wv, Gv, s1)                      # [Ho][Wo][K][N]
    to_cols = lambda a: a.transpose(2, 0, 1, 3).reshape(K, -1)
    gxr = O.col2im(to_cols(gcr), s)
    gxs = O.col2im(to_cols(gcs), s)
    assert_close(gx.cpu().numpy(), gxr * Tw * Tg, gxs * Tw * Tg, f"{name} naive dgrad")


def test_square_blocks_make_the_baseline_equal_quantize_once():
    """Stride 1 with padding: the expanded tensor holds every pixel, so its
    amax and every block are those of X; the baseline and the quantize-once
    path agree within the tolerance on all three outputs."""
    s = O.ConvShape(16, 32, 32, 8, 8, 3, 3, 1, 1)
    X, Wt, G = _inputs(s, 5)
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, "nvfp4")
    p = naive.plan(d, blocks="square")
    yb = torch.empty((s.Ho, s.Wo, s.Cout, s.N), device="cuda")
    gwb = torch.empty((s.Cout, s.Kh, s.Kw, s.Cin), device="cuda")
    gxb = torch.empty((s.H, s.W, s.Cin, s.N), device="cuda")
    Xd, Wd, Gd = X.cuda(), Wt.cuda(), G.cuda()
    naive.step(p, Xd, Wd, Gd, 3, yb, gwb, gxb)
    qx = mqv.quantize(Xd.view(-1), *s.x_view(), "nvfp4", mqv.RNE)
    qw = mqv.quantize(Wd.view(-1), *s.w_view(), "nvfp4", mqv.RNE)
    qg = mqv.quantize(Gd.view(-1), *s.gy_view(), "nvfp4", mqv.SR, 3)
    y, gw, gx = mqv.conv_fwd(d, qw, qx), mqv.conv_wgrad(d, qg, qx), mqv.conv_dgrad(d, qw, qg)
    assert np.float32(p.q["x_fwd"].tscale.item()) == np.float32(qx.tscale.item())
    ox = O.quantize(X.numpy().reshape(s.x_view()), O.FP4, O.RNE)
    ow = O.quantize(Wt.numpy().reshape(s.w_view()), O.FP4, O.RNE)
    og = O.quantize(G.numpy().reshape(s.gy_view()), O.FP4, O.SR, 3)
    ref = O.layer_outputs(ox, ow, og, s)
    for got, (v, S), nm in ((yb, ref["y"], "y"), (gwb, ref["gw"], "gw"), (gxb, ref["gx"], "gx")):
        assert_close(got.cpu().numpy().reshape(v.shape), v, S, f"baseline {nm}")
    for a, b, (v, S) in ((yb, y, ref["y"]), (gwb, gw, ref["gw"]), (gxb, gx, ref["gx"])):
        diff = np.abs(a.cpu().numpy().astype(np.float64) - b.cpu().numpy().astype(np.float64)).reshape(v.shape)
        assert np.all(diff <= 2e-5 * S + 2e-7)


# ------------------------------------------------------------ line blocks

LINE_SHAPES = [
    ("n16_3x3_s1_p1", O.ConvShape(16, 64, 64, 6, 5, 3, 3, 1, 1), "nvfp4"),
    ("n32_3x3_s2_p1_fp6", O.ConvShape(32, 64, 64, 9, 9, 3, 3, 2, 1), "nvfp6"),
    ("n64_1x1_c128", O.ConvShape(64, 128, 64, 5, 5, 1, 1, 1, 0), "nvfp4"),
    ("n16_5x5_s1_p2_fp6", O.ConvShape(16, 64, 128, 6, 6, 5, 5, 1, 2), "nvfp6"),
]

QCASES = [  # rows, cols, value recipe
    (48, 64, "relu"), (1040, 96, "gauss"), (4112, 160, "outliers"), (64, 32, "tiny"),
]


def _values(rows, cols, recipe, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((rows, cols), generator=g)
    if recipe == "relu":
        x = torch.relu(x)
    elif recipe == "outliers":
        # a few large values, some all-zero 16-element runs in both directions
        x = x * 1e-2
        idx = torch.randint(0, rows * cols, (rows * cols // 500,), generator=g)
        x.view(-1)[idx] = torch.randn(idx.numel(), generator=g) * 300.0
        x[3, :] = 0.0
        x[:, 5] = 0.0
    elif recipe == "tiny":
        # magnitudes where block divisors fall below the fast-division range
        x = x * 1e-36
    return x.float().contiguous()


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rows,cols,recipe", QCASES, ids=[f"{r}x{c}_{v}" for r, c, v in QCASES])
def test_line_quantizer_matches_oracle(rows, cols, recipe, fmt):
    """Both line shapes with both roundings in one mqv_quantize_many call:
    codes, scales and T bit-exact, and the dequantized values exact."""
    x = _values(rows, cols, recipe, rows + cols)
    xd = x.cuda()
    seed = 0x1234_5678_9ABC
    combos = [(mqv.BLOCKS_1X16, mqv.RNE), (mqv.BLOCKS_16X1, mqv.RNE), (mqv.BLOCKS_1X16, mqv.SR),
              (mqv.BLOCKS_16X1, mqv.SR)]
    outs = [mqv.QTensor.empty(rows, cols, fmt, "cuda", b) for b, _ in combos]
    mqv.quantize_many([(xd.view(-1), rows, cols, fmt, r, seed, o) for (b, r), o in zip(combos, outs)])
    torch.cuda.synchronize()
    f = FMT[fmt]
    for (b, r), o in zip(combos, outs):
        what = f"blocks {b} rounding {r}"
        oq = O.quantize_1d(x.numpy(), f, O.RNE if r == mqv.RNE else O.SR, seed, axis=1 if b == mqv.BLOCKS_1X16 else 0)
        assert np.float32(o.tscale.item()).view(np.uint32) == np.float32(oq.T).view(np.uint32), what
        assert np.array_equal(o.scales.cpu().numpy(), oq.scales.reshape(-1)), what
        assert np.array_equal(o.codes.cpu().numpy(), O.pack_codes(oq.codes, f)), what
        deq = mqv.dequantize(o).cpu().numpy().reshape(rows, cols)
        ref = (O.code_values_1d(oq) * np.float64(oq.T)).astype(np.float32)
        assert np.array_equal(deq.view(np.uint32), ref.view(np.uint32)), what


def test_line_blocks_rejected_outside_the_naive_kernels():
    s = O.ConvShape(16, 64, 64, 6, 6, 3, 3, 1, 1)
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, "nvfp4")
    w = mqv.QTensor.empty(*s.w_view(), "nvfp4", "cuda", mqv.BLOCKS_1X16)
    x = mqv.QTensor.empty(*s.x_view(), "nvfp4", "cuda", mqv.BLOCKS_16X1)
    with pytest.raises(mqv.MqvError) as e:                  # a 3 x 3 layer
        mqv.conv_fwd(d, w, x)
    assert e.value.status == 2
    x = torch.zeros(s.x_view()[0] * s.x_view()[1], device="cuda")
    with pytest.raises(mqv.MqvError) as e:                  # the single-tensor quantizer: squares only
        mqv.quantize(x, *s.x_view(), "nvfp4", out=mqv.QTensor.empty(*s.x_view(), "nvfp4", "cuda", 1))
    assert e.value.status == 2


@pytest.mark.parametrize("name,s,fmt", LINE_SHAPES, ids=[c[0] for c in LINE_SHAPES])
def test_naive_step_matches_oracle(name, s, fmt):
    """The scheme's six copies byte for byte, its outputs within tolerance,
    and each operand's two copies differing where the oracle's do."""
    X, Wt, G = _inputs(s, zlib.crc32(name.encode()) % 997 + 2)
    seed = 23
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, fmt)
    p = naive.plan(d)
    y = torch.empty((s.Ho, s.Wo, s.Cout, s.N), device="cuda")
    gw = torch.empty((s.Cout, s.Kh, s.Kw, s.Cin), device="cuda")
    gx = torch.empty((s.H, s.W, s.Cin, s.N), device="cuda")
    naive.step(p, X.cuda().contiguous(), Wt.cuda().contiguous(), G.cuda().contiguous(), seed, y, gw, gx)
    torch.cuda.synchronize()
    assert mqv.device_errors() == 0
    f = FMT[fmt]
    oq, out = O.naive_layer(X.numpy(), Wt.numpy(), G.numpy(), s, f, seed)
    for key, ref in oq.items():
        got = p.q[key]
        assert got.blocks == naive.LINE_BLOCKS[key]
        assert np.float32(got.tscale.item()) == np.float32(ref.T), key
        assert np.array_equal(got.scales.cpu().numpy(), ref.scales.reshape(-1)), key
        assert np.array_equal(got.codes.cpu().numpy(), O.pack_codes(ref.codes, f)), key
    for a, b in (("x_fwd", "x_wgrad"), ("w_fwd", "w_dgrad"), ("g_wgrad", "g_dgrad")):
        va = mqv.dequantize(p.q[a]).cpu().numpy()
        vb = mqv.dequantize(p.q[b]).cpu().numpy()
        oa = (O.code_values_1d(oq[a]) * np.float64(oq[a].T)).astype(np.float32).reshape(-1)
        ob = (O.code_values_1d(oq[b]) * np.float64(oq[b].T)).astype(np.float32).reshape(-1)
        assert np.array_equal(va != vb, oa != ob), (a, b)
        assert np.any(va != vb), (a, b)
    for got, key in ((y, "y"), (gw, "gw"), (gx, "gx")):
        v, S = out[key]
        assert_close(got.cpu().numpy().reshape(v.shape), v, S, f"{name} naive {key}")


def test_line_scheme_needs_its_block_sides():
    """Layers whose expanded channels or batch do not split into 16-element
    lines on the kernels (here N = 8) are rejected, not silently squared."""
    s = O.ConvShape(8, 16, 12, 7, 6, 3, 3, 1, 1)
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, "nvfp4")
    with pytest.raises(mqv.MqvError):
        p = naive.plan(d)
        X, Wt, G = _inputs(s, 1)
        y = torch.empty((s.Ho, s.Wo, s.Cout, s.N), device="cuda")
        gw = torch.empty((s.Cout, s.Kh, s.Kw, s.Cin), device="cuda")
        gx = torch.empty((s.H, s.W, s.Cin, s.N), device="cuda")
        naive.step(p, X.cuda(), Wt.cuda(), G.cuda(), 1, y, gw, gx)
