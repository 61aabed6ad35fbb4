"""GPU parity of the quantize-once kernels against the oracle: packed codes,
E4M3 scales and the tensor scale must match bit for bit."""
import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
import workloads
from oracle import mqv_oracle as O
from tests.parity_utils import FMT, assert_quant_equal, gpu_quantize

pytestmark = pytest.mark.gpu


def _rand(shape, seed, signed=True, scale=1.0, outliers=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * scale
    if not signed:
        x = x.abs()
    if outliers:
        k = max(1, x.numel() // 1000)
        idx = torch.randint(0, x.numel(), (k,), generator=g)
        x.view(-1)[idx] *= 100
    return x


SHAPES = [(4, 4), (8, 84), (16, 64), (6 * 6 * 16, 4), (128, 1152), (7 * 7 * 64, 32), (400, 20)]


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rnd", [mqv.RNE, mqv.SR])
@pytest.mark.parametrize("shape", SHAPES)
def test_quantize_bit_exact(fmt, rnd, shape):
    rows, cols = shape
    for i, kw in enumerate([dict(), dict(signed=False), dict(outliers=True), dict(scale=1e-30)]):
        x = _rand(shape, 10 + i, **kw)
        q, c, s, T = gpu_quantize(x, rows, cols, fmt, rnd, seed=1234 + i)
        assert_quant_equal(x.numpy(), rows, cols, fmt, rnd, 1234 + i, (c, s, T))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
def test_layer_tensors_bit_exact(fmt):
    """X, W and G_Y of the tiny layer and the ResNet-18 layer2-shaped layer."""
    for layer in (workloads.tiny_layer(), workloads.resnet18_layer2()):
        X, Wt, G = workloads.make_layer_inputs(layer)
        s = layer
        for t, (r, c), rnd, seed in [(X, (s.H * s.W * s.Cin, s.N), mqv.RNE, 0),
                                     (Wt, (s.Cout, s.K * s.K * s.Cin), mqv.RNE, 0),
                                     (G, (s.Ho * s.Wo * s.Cout, s.N), mqv.SR, workloads.sr_seed(s))]:
            q, cb, sb, T = gpu_quantize(t, r, c, fmt, rnd, seed)
            assert_quant_equal(t.numpy(), r, c, fmt, rnd, seed, (cb, sb, T))


def _tie_tensor(fmt, seed):
    """T = 1 exactly (amax = 448·emax), then blocks whose max is emax·m for
    chosen m (so B = CastE4M3(m)) and elements drawn from every tie point,
    grid point and their fp32 neighbours."""
    rng = np.random.default_rng(seed)
    emax = O.element_max(FMT[fmt])
    grid = O.element_grid(FMT[fmt])
    mids = (grid[:-1] + grid[1:]) / 2
    cand = np.concatenate([grid, mids, np.nextafter(mids.astype(np.float32), 0),
                           np.nextafter(mids.astype(np.float32), 100)]).astype(np.float32)
    e4 = O.E4M3_GRID
    e4mids = ((e4[:-1] + e4[1:]) / 2).astype(np.float32)
    ms = np.concatenate([e4[1:], e4mids, np.nextafter(e4mids, 0), np.nextafter(e4mids, 1000),
                         rng.uniform(0.001, 448, 200)]).astype(np.float32)
    nblocks = len(ms) + 512
    x = np.zeros((4 * nblocks, 4), np.float32)
    x[0, 0] = np.float32(448.0 * emax)
    for b in range(1, nblocks):
        blk = rng.choice(cand, size=16).astype(np.float32) * rng.choice([-1, 1], size=16)
        if b <= len(ms):                       # scale-rounding block: max = emax·m
            blk = (blk / emax * ms[b - 1]).astype(np.float32)
            blk[rng.integers(16)] = np.float32(emax) * ms[b - 1]
        else:                                  # element-rounding block: B = 1
            blk[rng.integers(16)] = np.float32(emax)
        x[4 * b:4 * b + 4] = blk.reshape(4, 4)
    return x


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rnd", [mqv.RNE, mqv.SR])
def test_rounding_ties_bit_exact(fmt, rnd):
    x = _tie_tensor(fmt, 3)
    rows, cols = x.shape
    q, c, s, T = gpu_quantize(torch.from_numpy(x), rows, cols, fmt, rnd, seed=99)
    assert T == 1.0
    assert_quant_equal(x, rows, cols, fmt, rnd, 99, (c, s, T))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rnd", [mqv.RNE, mqv.SR])
@pytest.mark.parametrize("amax", [3.7, 4e-17, 3.7e-18, 3.7e-33, 3.7e-37])
def test_division_near_grid_points_with_arbitrary_scales(fmt, rnd, amax):
    """Elements within a few ulps of RN(m·d) for every grid value and grid
    midpoint m, with block divisors d = B·T that are not powers of two, so
    the quotient x/d must be correctly rounded for the code to match.  The
    tensor maxima put the divisors in the normal range, just above and below
    2^-64, near the bottom of the normal range and among the subnormals."""
    rng = np.random.default_rng(11 if fmt == "nvfp4" else 12)
    f = FMT[fmt]
    emax = np.float32(O.element_max(f))
    grid = O.element_grid(f)
    targets = np.concatenate([(grid[:-1] + grid[1:]) / 2, grid[1:]])
    amax = np.float32(amax)
    T = np.float32(amax / np.float32(448.0 * O.element_max(f)))
    nblocks = 4096
    x = np.zeros((4 * nblocks, 4), np.float32)
    x[0, 0] = amax
    for b in range(1, nblocks):
        bmax = np.float32(rng.uniform(0.05, 1.0) * amax)
        B = np.float32(O.E4M3_GRID[O.cast_e4m3(np.array([bmax / np.float32(T * emax)], np.float32))[0]])
        d = np.float32(B * T)
        ok = targets[targets * float(d) < float(bmax)]
        t = rng.choice(ok, 15)
        v = (t * np.float64(d)).astype(np.float32)
        steps = rng.integers(-3, 4, 15).astype(np.int32)
        v = np.where(v > 0, (v.view(np.int32) + steps).view(np.float32), v)
        v = np.minimum(np.abs(v), bmax)
        blk = np.concatenate([[bmax], v]).astype(np.float32) * rng.choice([-1.0, 1.0], 16).astype(np.float32)
        x[4 * b:4 * b + 4] = blk.reshape(4, 4)
    rows, cols = x.shape
    q, c, sc, Tg = gpu_quantize(torch.from_numpy(x), rows, cols, fmt, rnd, seed=5)
    assert_quant_equal(x, rows, cols, fmt, rnd, 5, (c, sc, Tg))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rnd", [mqv.RNE, mqv.SR])
@pytest.mark.parametrize("scale", [1e-13, 1e-20, 1e-36, 1e-40])
def test_tiny_tensors_bit_exact(fmt, rnd, scale):
    """Tensors of tiny magnitude, down to subnormal elements: block divisors
    below 2^-64 or subnormal, where the quantizer divides exactly."""
    rows, cols = 64, 32
    x = _rand((rows, cols), 21, scale=scale, outliers=True)
    q, c, s, T = gpu_quantize(x, rows, cols, fmt, rnd, seed=17)
    assert_quant_equal(x.numpy(), rows, cols, fmt, rnd, 17, (c, s, T))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rnd", [mqv.RNE, mqv.SR])
def test_zero_scale_blocks_of_a_large_tensor(fmt, rnd):
    """max|x| = 1e6 makes every block whose maximum is below 2^-10·T·emax
    (about 2.2) round its E4M3 scale to 0: those elements, up to 2 in
    magnitude, must get code 0 with their sign, not the code of x itself."""
    rows, cols = 64, 32
    rng = np.random.default_rng(8)
    x = rng.uniform(-2.0, 2.0, (rows, cols)).astype(np.float32)
    x[0, 0] = 1e6
    q, c, s, T = gpu_quantize(torch.from_numpy(x), rows, cols, fmt, rnd, seed=4)
    assert_quant_equal(x, rows, cols, fmt, rnd, 4, (c, s, T))
    oq = O.quantize(x, FMT[fmt], O.RNE)
    assert np.count_nonzero(oq.scales == 0) == oq.scales.size - 1


@pytest.mark.parametrize("fmt,row,sr_bytes,rne_bytes", [
    ("nvfp4", [2688.0, 196.0, 616.0, -2240.0], [0x07, 0xE3], [0x17, 0xE3]),
    ("nvfp6", [3360.0, 49.0, 980.0, -1904.0], [0x1F, 0x10, 0xE1], [0x5F, 0x10, 0xE1])])
def test_hand_derived_codes_of_the_known_answer_row(fmt, row, sr_bytes, rne_bytes):
    """The row whose stochastic rounding is derived by hand from the first
    Philox4x32-10 known-answer vector (seed 0, counter 0; T = 1, B = 448):
    SR codes 7, 0, 3, 0xE (E2M1) and 31, 0, 17, 0x38 (E2M3), RNE codes
    7, 1, 3, 0xE and 31, 1, 17, 0x38, packed by hand; the other rows are 0."""
    x = torch.zeros(4, 4)
    x[0] = torch.tensor(row)
    for rnd, want in ((mqv.SR, sr_bytes), (mqv.RNE, rne_bytes)):
        q, c, s, T = gpu_quantize(x, 4, 4, fmt, rnd, seed=0)
        assert T == 1.0 and int(s[0]) == 0x7E            # E4M3 448
        assert [int(b) for b in c[:len(want)]] == want and not c[len(want):].any()


def test_zero_tensor_and_negative_zero():
    x = torch.zeros(16, 8)
    x[1, 1] = -0.0
    for fmt in ("nvfp4", "nvfp6"):
        q, c, s, T = gpu_quantize(x, 16, 8, fmt, mqv.RNE)
        assert T == 0.0 and not s.any()
        assert_quant_equal(x.numpy(), 16, 8, fmt, mqv.RNE, 0, (c, s, T))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
def test_dequantize_enumerates_every_code_and_scale(fmt):
    """Every (code, E4M3 scale) product decoded on the GPU equals the
    oracle's exact value: code·B (and the fp32 product with T)."""
    nbits = 4 if fmt == "nvfp4" else 6
    ncodes = 1 << nbits
    cols = ncodes                     # one view row holds every code once
    rows = 4 * 127                    # one block row per finite scale code
    codes = np.tile(np.arange(ncodes), (rows, 1))
    scales = np.repeat(np.arange(127, dtype=np.uint8)[:, None], cols // 4, axis=1)
    for T in (1.0, 0.1234567):
        q = mqv.QTensor.empty(rows, cols, fmt)
        q.codes.copy_(torch.from_numpy(O.pack_codes(codes, FMT[fmt])))
        q.scales.copy_(torch.from_numpy(scales.reshape(-1)))
        q.tscale.fill_(T)
        got = mqv.dequantize(q).cpu().numpy().reshape(rows, cols)
        oq = O.QTensor(codes.astype(np.int64), scales, np.float32(T), FMT[fmt])
        ref = (O.code_values(oq) * np.float64(np.float32(T))).astype(np.float32)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_split_amax_path_matches_fused():
    x = _rand((28 * 28 * 32, 64), 5, outliers=True)
    xd = x.cuda().view(-1)
    a = mqv.amax(xd, *x.shape)
    assert a.item() == float(x.abs().max())
    q1 = mqv.quantize(xd, *x.shape, "nvfp4", mqv.SR, 7)
    q2 = mqv.quantize_with_amax(xd, *x.shape, "nvfp4", mqv.SR, 7, a)
    torch.cuda.synchronize()
    for f in ("codes", "scales", "tscale"):
        assert torch.equal(getattr(q1, f), getattr(q2, f))


@pytest.mark.parametrize("C,H,N,signed,outliers,rnd", [
    (256, 7, 84, False, False, mqv.RNE), (512, 7, 256, True, True, mqv.SR),
    (512, 14, 256, False, True, mqv.RNE)])
def test_replay_shapes_full_tensor(C, H, N, signed, outliers, rnd):
    x = workloads.make_replay_input(C, H, N, signed=signed, outliers=outliers, seed=1)
    rows, cols = H * H * C, N
    q, c, s, T = gpu_quantize(x, rows, cols, "nvfp4", rnd, seed=17)
    assert_quant_equal(x.numpy(), rows, cols, "nvfp4", rnd, 17, (c, s, T))


@pytest.mark.parametrize("C,H,N,rnd", [(512, 14, 2560, mqv.SR), (512, 14, 10240, mqv.RNE)])
def test_replay_shapes_large_sampled_bands(C, H, N, rnd):
    """1/4-G-element and 1-G-element replay buffers: every tensor scale bit,
    then code/scale bytes of 6 row bands (checked against the oracle with the
    global amax and the global SR counter), in the launch the bench times."""
    rows, cols = H * H * C, N
    x = workloads.make_replay_input(C, H, N, outliers=True, seed=2, device="cuda").view(-1)
    q = mqv.quantize(x, rows, cols, "nvfp4", rnd, 23)
    torch.cuda.synchronize()
    amax = float(x.abs().max())
    rng = np.random.default_rng(0)
    T = q.tscale.item()
    rb = cols // 2
    for band in [0, rows - 8] + list(4 * rng.integers(0, rows // 4 - 2, 4)):
        band = int(band)
        xb = x[band * cols:(band + 8) * cols].cpu().numpy().reshape(8, cols)
        cb = q.codes[band * rb:(band + 8) * rb].cpu().numpy()
        sb = q.scales[band // 4 * (cols // 4):(band // 4 + 2) * (cols // 4)].cpu().numpy()
        assert_quant_equal(xb, 8, cols, "nvfp4", rnd, 23, (cb, sb, T), amax=amax, row_offset=band)
    del x, q
    torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
def test_batch_shard_quantization_matches_whole_tensor(fmt):
    """A batch shard quantized with the global amax and its SR column window
    (as the data-parallel step does) equals the matching columns of the
    whole tensor's quantization, and the oracle's."""
    rows, N, world = 7 * 7 * 32, 64, 4
    x = _rand((rows, N), 21, outliers=True)
    xd = x.cuda()
    amax = mqv.amax(xd.view(-1), rows, N)
    n = N // world
    for rank in range(world):
        part = xd[:, rank * n:(rank + 1) * n].contiguous().view(-1)
        q = mqv.quantize_with_amax(part, rows, n, fmt, mqv.SR, 41, amax, sr_col0=rank * n, sr_cols=N)
        torch.cuda.synchronize()
        gq = (q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.tscale.item())
        oq = O.quantize(x.numpy()[:, rank * n:(rank + 1) * n], FMT[fmt], O.SR, 41,
                        amax=float(x.abs().max()), col_offset=rank * n, total_cols=N)
        assert np.array_equal(gq[0], O.pack_codes(oq.codes, FMT[fmt]))
        assert np.array_equal(gq[1], oq.scales.reshape(-1)) and np.float32(gq[2]) == oq.T


@pytest.mark.parametrize("layer", [workloads.resnet18_layer2(), workloads.yolov8n_mix()[6],
                                   workloads.tiny_layer()], ids=lambda l: l.name)
def test_quantize_many_equals_one_call_per_tensor(layer):
    """The layer's X, W (RNE) and G_Y (SR) in one two-launch call are bit for
    bit the three single-tensor quantizations (and so the oracle's)."""
    X, Wt, G = workloads.make_layer_inputs(layer)
    s = layer
    views = [(X, s.H * s.W * s.Cin, s.N, mqv.RNE, 0),
             (Wt, s.Cout, s.K * s.K * s.Cin, mqv.RNE, 0),
             (G, s.Ho * s.Wo * s.Cout, s.N, mqv.SR, workloads.sr_seed(s)),
             (_rand((8, 84), 4), 8, 84, mqv.SR, 9)]                     # odd column blocks
    jobs = [(t.cuda().contiguous().view(-1), r, c, s.fmt, rnd, seed) for t, r, c, rnd, seed in views]
    many = mqv.quantize_many(jobs)
    torch.cuda.synchronize()
    for (t, r, c, rnd, seed), q in zip(views, many):
        one = mqv.quantize(t.cuda().contiguous().view(-1), r, c, s.fmt, rnd, seed)
        torch.cuda.synchronize()
        for f in ("codes", "scales", "tscale"):
            assert torch.equal(getattr(q, f), getattr(one, f)), f
    assert_quant_equal(views[3][0].numpy(), 8, 84, s.fmt, mqv.SR, 9,
                       (many[3].codes.cpu().numpy(), many[3].scales.cpu().numpy(), many[3].tscale.item()))
