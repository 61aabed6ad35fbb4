"""Slices of the exhaustive element-rounding sweep (imported by
test_exhaustive_rounding.py, and by its worker processes, so it imports
numpy and the oracle only).

A view whose max|x| is 448·emax (so T = 1) and whose other 4x4 blocks each
hold emax in their first slot (so B = 1) makes each element's quotient
x / (B·T) the element itself: its code is the element rounding of x alone
(round to nearest even, or stochastic with the element's own Philox word).
Block 0 carries the maximum and zeros; its quotients x / 448 are emax and
0, whose codes the element rounding of x itself also gives (448·emax
saturates to the top code, 0 stays 0)."""
import numpy as np

from oracle import mqv_oracle as O

COLS = 16                 # four 4x4 blocks across a block row
SEED = 77
FMT = {"nvfp4": O.FP4, "nvfp6": O.FP6}


def pattern_count(fmt) -> int:
    top = int(np.float32(O.element_max(FMT[fmt])).view(np.uint32))
    return 2 * (top + 1)


def patterns(fmt, start, count) -> np.ndarray:
    """fp32 values of patterns start .. start+count-1 of the sweep: the
    non-negative patterns 0 .. bits(emax), then the same with the sign set."""
    top = int(np.float32(O.element_max(FMT[fmt])).view(np.uint32))
    k = np.arange(start, start + count, dtype=np.uint64)
    bits = np.where(k <= top, k, (k - (top + 1)) | np.uint64(0x80000000)).astype(np.uint32)
    return bits.view(np.float32)


def slice_view(fmt, values):
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


def positions(blocks, slots):
    """Row-major (row, col) of block slots in the COLS-wide view."""
    br, bc = blocks // 4, blocks % 4
    return br * 4 + slots // 4, bc * 4 + slots % 4


def element_codes(fmt, values, rows, cols, rounding):
    """Codes of x itself: grid index of |x| plus the sign bit."""
    a = np.abs(values)
    if rounding == O.RNE:
        mag = O.round_rne(a, FMT[fmt])
    else:
        mag = O.round_sr(a, O.sr_uniforms(SEED, rows.astype(np.uint64) * COLS + cols), FMT[fmt])
    sign = np.signbit(values).astype(np.int64) << (O.element_bits(FMT[fmt]) - 1)
    return mag | sign


def slice_job(args):
    """(fmt, rounding, start, count) -> (X, expected packed codes of the
    whole view): the work of one slice on the host."""
    fmt, rounding, start, count = args
    X, _, _ = slice_view(fmt, patterns(fmt, start, count))
    rows = X.shape[0]
    r = np.repeat(np.arange(rows), COLS)
    c = np.tile(np.arange(COLS), rows)
    want = element_codes(fmt, X.reshape(-1), r, c, rounding).reshape(rows, COLS)
    return start, X, O.pack_codes(want, FMT[fmt])
