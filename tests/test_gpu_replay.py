"""GPU parity of the latent-replay form (magnitude-only storage of post-ReLU
tensors, reading R21) against the oracle: packed bytes, the negative-code
count and unpacked codes bit for bit, and values read straight from the
replay form equal to fp32(code·B·T) exactly."""
import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
import workloads
from oracle import mqv_oracle as O
from tests.parity_utils import FMT

pytestmark = pytest.mark.gpu

# rows x cols views: 16 elements (a lone half run), ragged runs, whole runs,
# several CTAs, and the smallest replay-buffer shape (7·7·256 x 84)
SHAPES = [(4, 4), (12, 20), (64, 36), (4 * 148, 512), (7 * 7 * 256, 84)]


def _random_codes(rows, cols, fmt, seed):
    """Every code value, negative ones included (sign bit set)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 1 << O.element_bits(FMT[fmt]), size=(rows, cols))


def _upload(codes, scales, T, rows, cols, fmt):
    return mqv.QTensor(torch.from_numpy(O.pack_codes(codes, FMT[fmt])).cuda(),
                       torch.from_numpy(np.ascontiguousarray(scales, dtype=np.uint8).reshape(-1)).cuda(),
                       torch.tensor([T], dtype=torch.float32, device="cuda"), rows, cols, mqv._fmt(fmt))


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("shape", SHAPES)
def test_pack_and_unpack_match_oracle(fmt, shape):
    rows, cols = shape
    codes = _random_codes(rows, cols, fmt, seed=rows + cols)
    q = _upload(codes, np.zeros((rows // 4, cols // 4)), 1.0, rows, cols, fmt)
    neg = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed = mqv.replay_pack(q, negatives=neg)
    back = mqv.replay_unpack(packed, rows, cols, fmt)
    torch.cuda.synchronize()
    ref, ref_neg = O.pack_unsigned(codes, FMT[fmt])
    got = packed.cpu().numpy()
    assert got.size == ref.size == mqv.replay_bytes(rows, cols, fmt)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} packed bytes differ, first at {bad[:5]}"
    assert int(neg.item()) == ref_neg
    ref_codes = O.pack_codes(O.unpack_unsigned(ref, rows, cols, FMT[fmt]), FMT[fmt])
    assert np.array_equal(back.cpu().numpy(), ref_codes)


def test_pack_without_counter_and_of_sign_free_codes():
    rows, cols = 8, 16
    codes = _random_codes(rows, cols, "nvfp4", 3) & 7          # no sign bits
    q = _upload(codes, np.zeros((2, 4)), 1.0, rows, cols, "nvfp4")
    packed = mqv.replay_pack(q)
    back = mqv.replay_unpack(packed, rows, cols, "nvfp4")
    torch.cuda.synchronize()
    assert np.array_equal(back.cpu().numpy(), q.codes.cpu().numpy())


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("C,H,N,signed", [(16, 3, 8, False), (64, 7, 84, False), (32, 5, 20, True)])
def test_replay_dequantize_matches_oracle(fmt, C, H, N, signed):
    """Oracle-quantized replay activations (|N(0,1)| with outliers, or signed:
    the replay form then holds the ReLU of the values) read back from the
    replay form: exactly fp32 of the oracle's code·B·T, and bit-identical to
    mqv_dequantize of the full codes."""
    rows, cols = H * H * C, N
    x = workloads.make_replay_input(C, H, N, signed=signed, outliers=True, seed=5).numpy().reshape(rows, cols)
    oq = O.quantize(x, FMT[fmt], O.RNE)
    q = _upload(oq.codes, oq.scales, oq.T, rows, cols, fmt)
    packed = mqv.replay_pack(q)
    got = mqv.replay_dequantize(packed, q.scales, q.tscale, rows, cols, fmt)
    full = mqv.dequantize(q)
    torch.cuda.synchronize()
    ref = np.maximum(O.dequantize(oq), 0).astype(np.float32).reshape(-1)
    g = got.cpu().numpy()
    assert np.array_equal(g.view(np.uint32), ref.view(np.uint32)) or np.array_equal(g, ref)
    if not signed:
        assert torch.equal(got, full)


@pytest.mark.parametrize("C,H,N", [(512, 14, 2560), (512, 14, 10240)])
def test_replay_buffer_full_size_sampled(C, H, N):
    """A 1/4-G- and a 1-G-element buffer in the launch the benchmark times:
    the negative count over the whole tensor, then packed bytes, unpacked
    codes and values read back of 6 row bands against the oracle."""
    rows, cols = H * H * C, N
    g = torch.Generator(device="cuda").manual_seed(C + N)
    codes_dev = torch.randint(0, 256, (rows * cols // 2,), dtype=torch.uint8, device="cuda", generator=g)
    scales_dev = torch.randint(0, 0x7F, (rows // 4 * cols // 4,), dtype=torch.uint8, device="cuda", generator=g)
    T = torch.tensor([2.0 ** -7], dtype=torch.float32, device="cuda")
    q = mqv.QTensor(codes_dev, scales_dev, T, rows, cols, mqv.NVFP4)
    neg = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed = mqv.replay_pack(q, negatives=neg)
    back = mqv.replay_unpack(packed, rows, cols, "nvfp4")
    vals = mqv.replay_dequantize(packed, scales_dev, T, rows, cols, "nvfp4")
    torch.cuda.synchronize()
    nib = torch.stack([codes_dev & 0xF, codes_dev >> 4], dim=1)
    assert int(neg.item()) == int(((nib >= 8) & ((nib & 7) != 0)).sum())
    del nib
    rng = np.random.default_rng(1)
    pb, cb = 3 * cols // 8, cols // 2                      # bytes per row: replay form, codes
    for band in [0, rows - 4] + list(4 * rng.integers(0, rows // 4 - 1, 4)):
        band = int(band)
        c = O.unpack_codes(codes_dev[band * cb:(band + 4) * cb].cpu().numpy(), 4, cols, O.FP4)
        ref, _ = O.pack_unsigned(c, O.FP4)
        assert np.array_equal(packed[band * pb:(band + 4) * pb].cpu().numpy(), ref), band
        ref_c = O.pack_codes(O.unpack_unsigned(ref, 4, cols, O.FP4), O.FP4)
        assert np.array_equal(back[band * cb:(band + 4) * cb].cpu().numpy(), ref_c), band
        s = scales_dev[band // 4 * (cols // 4):(band // 4 + 1) * (cols // 4)].cpu().numpy().reshape(1, -1)
        oq = O.QTensor(O.unpack_unsigned(ref, 4, cols, O.FP4), s, np.float32(2.0 ** -7), O.FP4)
        want = O.dequantize(oq).astype(np.float32).reshape(-1)
        assert np.array_equal(vals[band * cols:(band + 4) * cols].cpu().numpy(), want), band
    del codes_dev, packed, back, vals
    torch.cuda.empty_cache()


def test_replay_buffer_e2m3_sampled():
    """A 6.4 M-element NVFP6 buffer (5-bit magnitudes): whole-tensor negative
    count, then packed bytes and values read back of 4 row bands."""
    C, H, N = 512, 7, 256
    rows, cols = H * H * C, N
    g = torch.Generator(device="cuda").manual_seed(77)
    codes_dev = torch.randint(0, 256, (rows * cols * 3 // 4,), dtype=torch.uint8, device="cuda", generator=g)
    scales_dev = torch.randint(0, 0x7F, (rows // 4 * cols // 4,), dtype=torch.uint8, device="cuda", generator=g)
    T = torch.tensor([2.0 ** -9], dtype=torch.float32, device="cuda")
    q = mqv.QTensor(codes_dev, scales_dev, T, rows, cols, mqv.NVFP6)
    neg = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed = mqv.replay_pack(q, negatives=neg)
    vals = mqv.replay_dequantize(packed, scales_dev, T, rows, cols, "nvfp6")
    torch.cuda.synchronize()
    allc = O.unpack_codes(codes_dev.cpu().numpy(), rows, cols, O.FP6)
    assert int(neg.item()) == int(np.count_nonzero((allc >= 32) & ((allc & 31) != 0)))
    rng = np.random.default_rng(4)
    pb, cb = 5 * cols // 8, 3 * cols // 4
    for band in [0, rows - 4] + list(4 * rng.integers(0, rows // 4 - 1, 2)):
        band = int(band)
        c = allc[band:band + 4]
        ref, _ = O.pack_unsigned(c, O.FP6)
        assert np.array_equal(packed[band * pb:(band + 4) * pb].cpu().numpy(), ref), band
        s = scales_dev[band // 4 * (cols // 4):(band // 4 + 1) * (cols // 4)].cpu().numpy().reshape(1, -1)
        oq = O.QTensor(O.unpack_unsigned(ref, 4, cols, O.FP6), s, np.float32(2.0 ** -9), O.FP6)
        assert np.array_equal(vals[band * cols:(band + 4) * cols].cpu().numpy(),
                              O.dequantize(oq).astype(np.float32).reshape(-1)), band
