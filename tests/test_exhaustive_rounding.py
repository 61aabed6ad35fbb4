"""Every fp32 element value of magnitude at most emax through the quantizer:
a view whose max|x| is 448·emax (so T = 1) and whose other 4x4 blocks each
hold emax in their first slot (so B = 1) makes each element's quotient
x / (B·T) the element itself, so the element codes are the element rounding
of x alone: round to nearest even, or stochastic with each element's own
Philox word.  The GPU sweep covers all 2·(bits(emax) + 1) patterns (about
2.2e9 per format) in slices of 15·2^20 values and takes minutes of host
time for the oracle side: opt in with MQV_EXHAUSTIVE=1.  The CPU test checks
the construction itself on one small slice against the oracle's quantizer."""
import os

import numpy as np
import pytest
import torch

from oracle import mqv_oracle as O
from tests.parity_utils import FMT

COLS = 16                 # four 4x4 blocks across a block row
SEED = 77


def _pattern_count(fmt) -> int:
    top = int(np.float32(O.element_max(FMT[fmt])).view(np.uint32))
    return 2 * (top + 1)


def _patterns(fmt, start, count) -> np.ndarray:
    """fp32 values of patterns start .. start+count-1 of the sweep: the
    non-negative patterns 0 .. bits(emax), then the same with the sign set."""
    top = int(np.float32(O.element_max(FMT[fmt])).view(np.uint32))
    k = np.arange(start, start + count, dtype=np.uint64)
    bits = np.where(k <= top, k, (k - (top + 1)) | np.uint64(0x80000000)).astype(np.uint32)
    return bits.view(np.float32)


def _slice(fmt, values):
    """The view holding `values`: block 0 carries max|x| = 448·emax and no
    test values; every other block has emax in slot 0 and up to 15 values
    (zeros after the last).  Returns (X rows x COLS, blocks, slots) with the
    block and slot (r·4 + c) of every value."""
    emax = np.float32(O.element_max(FMT[fmt]))
    nb = 1 + -(-values.size // 15)
    nb = -(-nb // 4) * 4                                  # whole block rows
    bk = np.zeros((nb, 16), np.float32)
    bk[:, 0] = emax
    bk[0, 0] = np.float32(448.0) * emax
    flat = np.zeros((nb - 1) * 15, np.float32)
    flat[:values.size] = values
    bk[1:, 1:] = flat.reshape(nb - 1, 15)
    X = bk.reshape(nb // 4, 4, 4, 4).transpose(0, 2, 1, 3).reshape(nb, COLS)
    idx = np.arange(values.size)
    return np.ascontiguousarray(X), 1 + idx // 15, 1 + idx % 15


def _positions(blocks, slots):
    """Row-major (row, col) of block slots in the COLS-wide view."""
    br, bc = blocks // 4, blocks % 4
    return br * 4 + slots // 4, bc * 4 + slots % 4


def _expected_codes(fmt, values, rows, cols, rounding):
    """Codes of x itself: grid index of |x| plus the sign bit."""
    a = np.abs(values)
    if rounding == O.RNE:
        mag = O.round_rne(a, FMT[fmt])
    else:
        mag = O.round_sr(a, O.sr_uniforms(SEED, rows.astype(np.uint64) * COLS + cols), FMT[fmt])
    sign = np.signbit(values).astype(np.int64) << (O.element_bits(FMT[fmt]) - 1)
    return mag | sign


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_slice_construction_reduces_quantization_to_element_rounding(fmt, rounding):
    """On CPU: the oracle's quantizer of a slice (patterns around 0, around
    1, around emax and negative ones) gives T = 1, scale 1 for every test
    block and exactly the element-rounding codes the sweep compares with."""
    n = _pattern_count(fmt)
    top = n // 2 - 1
    one = int(np.float32(1.0).view(np.uint32))
    vals = np.concatenate([_patterns(fmt, 0, 3000), _patterns(fmt, one - 1500, 3000),
                           _patterns(fmt, top - 2999, 3000), _patterns(fmt, n - 3000, 3000)])
    X, blocks, slots = _slice(fmt, vals)
    q = O.quantize(X, FMT[fmt], rounding, SEED)
    assert q.T == np.float32(1.0)
    one_code = O.cast_e4m3(np.array([1.0], np.float32))[0]
    assert np.all(q.scales.reshape(-1)[1:] == one_code)
    r, c = _positions(blocks, slots)
    assert np.array_equal(q.codes[r, c], _expected_codes(fmt, vals, r, c, rounding))


@pytest.mark.gpu
@pytest.mark.skipif(os.environ.get("MQV_EXHAUSTIVE") != "1",
                    reason="about 2.2e9 values per format; opt in with MQV_EXHAUSTIVE=1")
@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_every_element_pattern_on_the_gpu(fmt, rounding):
    import microscaling_quantized_convolution_b200 as mqv
    per = 15 << 20
    n = _pattern_count(fmt)
    for start in range(0, n, per):
        vals = _patterns(fmt, start, min(per, n - start))
        X, blocks, slots = _slice(fmt, vals)
        rows = X.shape[0]
        q = mqv.quantize(torch.from_numpy(X).cuda().view(-1), rows, COLS, fmt,
                         mqv.RNE if rounding == O.RNE else mqv.SR, SEED)
        codes = O.unpack_codes(q.codes.cpu().numpy(), rows, COLS, FMT[fmt])
        assert float(q.tscale.item()) == 1.0
        r, c = _positions(blocks, slots)
        want = _expected_codes(fmt, vals, r, c, rounding)
        bad = np.nonzero(codes[r, c] != want)[0]
        assert bad.size == 0, f"patterns from {start}: {bad.size} codes differ, first x = {vals[bad[:4]]}"
