"""GPU parity of the three implicit-GEMM conv passes against the oracle.

Small shapes (several tiles, ragged in every GEMM dimension) are compared
element by element; full-size layers of the benchmarked workloads are
compared on sampled outputs that the oracle computes one by one.  Both sides
quantize the same seeded fp32 inputs themselves.  Tolerance per output:
|y - y_ref| <= 1e-5·S + 1e-7 with S = T_a·T_b·sum_k |a_k·b_k|."""
import zlib

import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
import workloads
from oracle import mqv_oracle as O
from tests.parity_utils import FMT, assert_close

pytestmark = pytest.mark.gpu


def run_gpu_layer(X, Wt, G, s: O.ConvShape, fmt, seed):
    d = mqv.conv_desc(s.N, s.Cin, s.Cout, s.H, s.W, s.Kh, s.Kw, s.stride, s.pad, fmt)
    qx = mqv.quantize(X.cuda().view(-1), *s.x_view(), fmt, mqv.RNE)
    qw = mqv.quantize(Wt.cuda().view(-1), *s.w_view(), fmt, mqv.RNE)
    qg = mqv.quantize(G.cuda().view(-1), *s.gy_view(), fmt, mqv.SR, seed)
    y = mqv.conv_fwd(d, qw, qx)
    gw = mqv.conv_wgrad(d, qg, qx)
    gx = mqv.conv_dgrad(d, qw, qg)
    assert mqv.device_errors() == 0
    return (qx, qw, qg), y.cpu().numpy(), gw.cpu().numpy(), gx.cpu().numpy()


def make_inputs(s: O.ConvShape, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.relu(torch.randn((s.H, s.W, s.Cin, s.N), generator=g))
    Wt = torch.randn((s.Cout, s.Kh, s.Kw, s.Cin), generator=g) * (2.0 / (s.Cin * s.Kh * s.Kw)) ** 0.5
    G = torch.randn((s.Ho, s.Wo, s.Cout, s.N), generator=g) * 1e-3
    return X, Wt, G


SMALL = [
    ("tiny_3x3_s1_p0", O.ConvShape(4, 16, 16, 8, 8, 3, 3, 1, 0), "nvfp4"),
    ("ragged_3x3_s1_p1", O.ConvShape(8, 24, 40, 9, 9, 3, 3, 1, 1), "nvfp4"),
    ("ragged_3x3_s2_p1", O.ConvShape(8, 24, 40, 9, 9, 3, 3, 2, 1), "nvfp4"),
    ("pointwise_fp6", O.ConvShape(16, 32, 48, 10, 10, 1, 1, 1, 0), "nvfp6"),
    ("cin4_3x3_s2_fp6", O.ConvShape(4, 4, 16, 12, 12, 3, 3, 2, 1), "nvfp6"),
    ("rect_3x2_p1", O.ConvShape(4, 8, 12, 7, 6, 3, 2, 1, 1), "nvfp4"),
    ("two_m_tiles", O.ConvShape(4, 16, 136, 6, 6, 3, 3, 1, 1), "nvfp4"),
    ("n12_c8", O.ConvShape(12, 8, 8, 5, 5, 3, 3, 1, 1), "nvfp6"),
    ("wide_k_s2_p2", O.ConvShape(4, 72, 68, 11, 11, 5, 5, 2, 2), "nvfp4"),
    # stride 2 with 32+ output channels: input-gradient tiles grouped by
    # pixel parity, some parities reached by no tap at all (1 x 1), a
    # one-row input, two channel tiles
    ("s2_1x1_empty_phases", O.ConvShape(4, 8, 32, 7, 7, 1, 1, 2, 0), "nvfp4"),
    ("s2_one_row", O.ConvShape(4, 8, 36, 1, 7, 3, 3, 2, 1), "nvfp6"),
    ("s2_m160_two_m_tiles", O.ConvShape(8, 160, 64, 9, 8, 3, 3, 2, 1), "nvfp4"),
    ("deep_cin", O.ConvShape(8, 256, 32, 4, 4, 3, 3, 1, 1), "nvfp4"),
    # 4-input-channel stems with N % 16 == 0: the input gradient runs on CUDA
    # cores (conv_narrow_dgrad_kernel), stride 2 and 1, both formats
    ("stem_cin4_n16_s2_fp6", O.ConvShape(16, 4, 16, 12, 12, 3, 3, 2, 1), "nvfp6"),
    ("stem_cin4_n32_s2", O.ConvShape(32, 4, 32, 9, 10, 3, 3, 2, 1), "nvfp4"),
    ("stem_cin4_n16_5x5_s1", O.ConvShape(16, 4, 8, 7, 7, 5, 5, 1, 2), "nvfp4"),
    # stride-1 shapes of the kernel-row halo path (N | 256, N % 8 == 0, 64-channel chunks)
    ("halo_n64_ragged_row", O.ConvShape(64, 64, 64, 6, 10, 3, 3, 1, 1), "nvfp4"),
    ("halo_n32_two_m_tiles", O.ConvShape(32, 128, 192, 5, 9, 3, 3, 1, 1), "nvfp4"),
    ("halo_n16_pad0", O.ConvShape(16, 64, 64, 7, 7, 3, 3, 1, 0), "nvfp4"),
    ("halo_n8_5x5", O.ConvShape(8, 64, 128, 9, 9, 5, 5, 1, 2), "nvfp4"),
    ("halo_1x1_n64", O.ConvShape(64, 128, 64, 5, 5, 1, 1, 1, 0), "nvfp4"),
    # the same path on NVFP6 codes (6-byte runs of 8 batch items)
    ("halo_fp6_n64_ragged_row", O.ConvShape(64, 64, 64, 6, 10, 3, 3, 1, 1), "nvfp6"),
    ("halo_fp6_n16_1x1", O.ConvShape(16, 128, 64, 7, 7, 1, 1, 1, 0), "nvfp6"),
    ("halo_fp6_n8_5x5", O.ConvShape(8, 64, 128, 9, 9, 5, 5, 1, 2), "nvfp6"),
    # more than two tiles per persistent CTA, so the weight loaders and the
    # producers finish well before the MMAs (a 1 x 1 layer has one stage a
    # tile) and share the epilogue of the CTA's last tile
    ("halo_multitile_1x1_fp6", O.ConvShape(16, 64, 64, 64, 64, 1, 1, 1, 0), "nvfp6"),
    ("halo_multitile_3x3_n32", O.ConvShape(32, 64, 64, 48, 48, 3, 3, 1, 1), "nvfp4"),
    # stride-1 weight-gradient shapes whose kernel-row taps share operands
    # (N % 16 == 0): ragged rows and channels, split ranges that end inside a
    # row, several channel tiles, a 2 x 2 kernel
    ("wgk_n16_ragged_c", O.ConvShape(16, 24, 40, 9, 7, 3, 3, 1, 1), "nvfp4"),
    ("wgk_n32_fp6_two_tiles", O.ConvShape(32, 200, 136, 6, 5, 3, 3, 1, 0), "nvfp6"),
    ("wgk_n48_2x2", O.ConvShape(48, 16, 20, 8, 8, 2, 2, 1, 0), "nvfp4"),
    ("wgk_rows_split", O.ConvShape(16, 256, 512, 10, 10, 3, 3, 1, 1), "nvfp4"),
    # batch 64: the taps of a kernel row share one run of B rows (paired MMAs)
    ("wgk_n64_pair_2x2", O.ConvShape(64, 200, 72, 6, 7, 2, 2, 1, 0), "nvfp4"),
    ("wgk_n64_pair_fp6", O.ConvShape(64, 136, 40, 5, 6, 3, 3, 1, 1), "nvfp6"),
]


@pytest.mark.parametrize("name,s,fmt", SMALL, ids=[c[0] for c in SMALL])
def test_small_layers_elementwise(name, s, fmt):
    X, Wt, G = make_inputs(s, zlib.crc32(name.encode()) % 1000)
    seed = 77
    _, y, gw, gx = run_gpu_layer(X, Wt, G, s, fmt, seed)
    qx, qw, qg = O.quantize_layer(X.numpy(), Wt.numpy(), G.numpy(), s, FMT[fmt], seed)
    ref = O.layer_outputs(qx, qw, qg, s)
    assert_close(y, *ref["y"], f"{name} fwd")
    assert_close(gw, *ref["gw"], f"{name} wgrad")
    assert_close(gx, *ref["gx"], f"{name} dgrad")


def test_outputs_not_trivially_zero():
    s = SMALL[1][1]
    X, Wt, G = make_inputs(s, 1)
    _, y, gw, gx = run_gpu_layer(X, Wt, G, s, "nvfp4", 5)
    assert np.count_nonzero(y) > 0.9 * y.size and np.count_nonzero(gx) > 0.5 * gx.size
    assert np.count_nonzero(gw) > 0.9 * gw.size


def test_repeat_calls_are_deterministic():
    s = O.ConvShape(16, 64, 64, 14, 14, 3, 3, 1, 1)
    X, Wt, G = make_inputs(s, 2)
    a = run_gpu_layer(X, Wt, G, s, "nvfp4", 3)
    b = run_gpu_layer(X, Wt, G, s, "nvfp4", 3)
    for u, v in zip(a[1:], b[1:]):
        assert np.array_equal(u, v)


# ------------------------------------------------------- full-size sampling

class BandOracle:
    """Oracle code values of single pixels of a big [H][W][C][N] tensor,
    quantized band by band with the tensor's global amax and global SR
    counter (so each band equals the same rows of a full quantization)."""

    def __init__(self, t: np.ndarray, fmt, rnd, seed):
        self.t, self.fmt, self.rnd, self.seed = t, fmt, rnd, seed
        self.H, self.W, self.C, self.N = t.shape
        self.amax = float(np.max(np.abs(t)))
        self.T = np.float32(np.float32(self.amax) / np.float32(O.E4M3_MAX * O.element_max(fmt)))
        self.cache = {}

    def pix(self, h, w):
        key = (h, w)
        if key not in self.cache:
            band = self.t[h, w].reshape(self.C, self.N)
            q = O.quantize(band, self.fmt, self.rnd, self.seed, amax=self.amax,
                           row_offset=(h * self.W + w) * self.C)
            self.cache[key] = O.code_values(q)
        return self.cache[key]


def sampled_check(layer: workloads.Layer, nsamp=96, full_wgrad=False):
    s = O.ConvShape(layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.K, layer.K,
                    layer.stride, layer.pad)
    fmt = layer.fmt
    seed = workloads.sr_seed(layer)
    X, Wt, G = workloads.make_layer_inputs(layer)
    (qx, qw, qg), y, gw, gx = run_gpu_layer(X, Wt, G, s, fmt, seed)
    of = FMT[fmt]
    oq_w = O.quantize(Wt.numpy().reshape(s.w_view()), of, O.RNE)
    Wcv = O.code_values(oq_w).reshape(s.Cout, s.Kh, s.Kw, s.Cin)
    bx = BandOracle(X.numpy(), of, O.RNE, 0)
    bg = BandOracle(G.numpy(), of, O.SR, seed)
    Tw, Tx, Tg = np.float64(oq_w.T), np.float64(bx.T), np.float64(bg.T)
    assert np.float32(qx.tscale.item()) == bx.T and np.float32(qg.tscale.item()) == bg.T
    rng = np.random.default_rng(layer.seed)
    y = y.reshape(s.Ho, s.Wo, s.Cout, s.N)
    gx = gx.reshape(s.H, s.W, s.Cin, s.N)
    got, ref, S = [], [], []
    for _ in range(nsamp):                                  # forward samples
        ho, wo, co, n = (int(rng.integers(d)) for d in (s.Ho, s.Wo, s.Cout, s.N))
        acc = sacc = 0.0
        for kh in range(s.Kh):
            for kw in range(s.Kw):
                hi, wi = ho * s.stride + kh - s.pad, wo * s.stride + kw - s.pad
                if 0 <= hi < s.H and 0 <= wi < s.W:
                    p = Wcv[co, kh, kw, :] * bx.pix(hi, wi)[:, n]
                    acc += p.sum()
                    sacc += np.abs(p).sum()
        got.append(y[ho, wo, co, n]); ref.append(acc * Tw * Tx); S.append(sacc * Tw * Tx)
    assert_close(np.array(got), np.array(ref), np.array(S), f"{layer.name} fwd sampled")
    got, ref, S = [], [], []
    for _ in range(nsamp):                                  # input-gradient samples
        hi, wi, ci, n = (int(rng.integers(d)) for d in (s.H, s.W, s.Cin, s.N))
        acc = sacc = 0.0
        for kh in range(s.Kh):
            th = hi + s.pad - kh
            if th < 0 or th % s.stride or th // s.stride >= s.Ho:
                continue
            for kw in range(s.Kw):
                tw = wi + s.pad - kw
                if tw < 0 or tw % s.stride or tw // s.stride >= s.Wo:
                    continue
                p = Wcv[:, kh, kw, ci] * bg.pix(th // s.stride, tw // s.stride)[:, n]
                acc += p.sum()
                sacc += np.abs(p).sum()
        got.append(gx[hi, wi, ci, n]); ref.append(acc * Tw * Tg); S.append(sacc * Tw * Tg)
    assert_close(np.array(got), np.array(ref), np.array(S), f"{layer.name} dgrad sampled")
    if full_wgrad:                                          # weight-gradient samples
        oqx = O.quantize(X.numpy().reshape(s.x_view()), of, O.RNE)
        oqg = O.quantize(G.numpy().reshape(s.gy_view()), of, O.SR, seed)
        # the whole quantized X and G_Y, byte for byte, at full size
        for what, q, oq in (("X", qx, oqx), ("G_Y", qg, oqg)):
            assert np.float32(q.tscale.item()) == np.float32(oq.T), what
            assert np.array_equal(q.scales.cpu().numpy(), oq.scales.reshape(-1)), f"{layer.name} {what} scales"
            assert np.array_equal(q.codes.cpu().numpy(), O.pack_codes(oq.codes, of)), f"{layer.name} {what} codes"
        Xcv = O.code_values(oqx).reshape(X.shape)
        Gcv = O.code_values(oqg).reshape(G.shape)
        gw = gw.reshape(s.Cout, s.Kh, s.Kw, s.Cin)
        got, ref, S = [], [], []
        for _ in range(max(32, nsamp // 2)):
            co, kh, kw, ci = (int(rng.integers(d)) for d in (s.Cout, s.Kh, s.Kw, s.Cin))
            v, sa = O.wgrad_at(Gcv, Xcv, s, co, kh, kw, ci)
            got.append(gw[co, kh, kw, ci]); ref.append(v * Tg * Tx); S.append(sa * Tg * Tx)
        assert_close(np.array(got), np.array(ref), np.array(S), f"{layer.name} wgrad sampled")


def test_resnet18_layer2_full_size_sampled():
    sampled_check(workloads.resnet18_layer2(), nsamp=128, full_wgrad=True)


BODY = workloads.resnet18_body()


@pytest.mark.parametrize("layer", BODY, ids=[l.name for l in BODY])
def test_resnet18_body_full_size_sampled(layer):
    # the weight gradient and the whole quantized operands on every layer
    sampled_check(layer, nsamp=48, full_wgrad=True)


YOLO = workloads.yolov8n_mix()


@pytest.mark.parametrize("layer", YOLO, ids=[l.name for l in YOLO])
def test_yolov8n_full_size_sampled(layer):
    # NVFP6 at 640²: the weight gradient and the whole quantized operands on
    # the stem, the narrow early layers and one layer per later stage
    sampled_check(layer, nsamp=48, full_wgrad=layer.seed in (0, 1, 3, 7, 17))


def test_concurrent_passes_match_serial():
    """fwd, wgrad and dgrad on three streams (as the bench runs them), with
    G_Y quantized on a fourth beside X and W, give bit-identical outputs to
    the same calls on one stream."""
    layer = workloads.resnet18_layer2()
    s = O.ConvShape(layer.N, layer.Cin, layer.Cout, layer.H, layer.W, layer.K, layer.K, layer.stride, layer.pad)
    X, Wt, G = (t.cuda().contiguous() for t in workloads.make_layer_inputs(layer))
    d = mqv.conv_desc(**layer.dims(), fmt=layer.fmt)
    fmt, seed = layer.fmt, workloads.sr_seed(layer)

    def run(concurrent):
        qx = mqv.QTensor.empty(*s.x_view(), fmt)
        qw = mqv.QTensor.empty(*s.w_view(), fmt)
        qg = mqv.QTensor.empty(*s.gy_view(), fmt)
        cur = torch.cuda.current_stream()
        streams = [torch.cuda.Stream() for _ in range(4)] if concurrent else [cur] * 4
        start = torch.cuda.Event()
        start.record(cur)
        for st in streams:
            st.wait_event(start)
        with torch.cuda.stream(streams[3]):
            mqv.quantize_many([(G.view(-1), *s.gy_view(), fmt, mqv.SR, seed, qg)])
            g_done = torch.cuda.Event()
            g_done.record(streams[3])
        mqv.quantize_many([(X.view(-1), *s.x_view(), fmt, mqv.RNE, 0, qx),
                           (Wt.view(-1), *s.w_view(), fmt, mqv.RNE, 0, qw)])
        xw_done = torch.cuda.Event()
        xw_done.record(cur)
        outs = {}
        for i, (name, fn) in enumerate((("y", lambda: mqv.conv_fwd(d, qw, qx)),
                                        ("gw", lambda: mqv.conv_wgrad(d, qg, qx)),
                                        ("gx", lambda: mqv.conv_dgrad(d, qw, qg)))):
            st = streams[i]
            st.wait_event(xw_done)
            if name != "y":
                st.wait_event(g_done)
            with torch.cuda.stream(st):
                outs[name] = fn()
        torch.cuda.synchronize()
        return {k: v.cpu().numpy() for k, v in outs.items()}

    a, b = run(False), run(True)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    assert mqv.device_errors() == 0
