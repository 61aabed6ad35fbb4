"""Pins of the CPU oracle against what the method description and mathematics
fix, independently of the oracle's own code (no GPU needed).

Each test names the fact it checks.  The method is the MicroQonv summary
(onedev.kr/papers/182); formats follow OCP MX v1.0 / OFP8.
"""
import math

import numpy as np
import pytest
import torch

from oracle import mqv_oracle as O


# ---------------------------------------------------------------- P1 formats

def test_e2m1_table_matches_ocp(golden):
    for code, val in golden("e2m1_values.txt"):
        c = int(code, 16)
        v = O.decode_e2m1(c)
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e2m3_table_matches_ocp(golden):
    for code, val in golden("e2m3_values.txt"):
        c = int(code, 16)
        assert O.decode_e2m3(c) == float(val)
        assert O.decode_e2m3(c | 0x20) == -float(val)


def test_e4m3_points_match_ofp8(golden):
    for code, val in golden("e4m3_points.txt"):
        v = O.decode_e4m3(int(code, 16))
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val)


def test_format_maxima():
    assert O.element_max(O.FP4) == 6.0
    assert O.element_max(O.FP6) == 7.5
    assert O.E4M3_MAX == 448.0
    assert len(O.E4M3_GRID) == 127 and np.all(np.diff(O.E4M3_GRID) > 0)


def test_encode_decode_roundtrip():
    for fmt, n in ((O.FP4, 8), (O.FP6, 32)):
        grid = O.element_grid(fmt)
        assert np.array_equal(O.round_rne(grid.astype(np.float32), fmt), np.arange(n))
        u = np.random.default_rng(0).random(n)
        assert np.array_equal(O.round_sr(grid.astype(np.float32), u, fmt), np.arange(n))
    assert np.array_equal(O.cast_e4m3(O.E4M3_GRID.astype(np.float32)), np.arange(127))


def test_e4m3_cast_matches_torch_float8():
    """Within the finite range, CastE4M3 with RNE is what torch's
    float8_e4m3fn conversion computes (a library routine for the same
    definition)."""
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.uniform(0, 460, 20000), 2.0 ** rng.uniform(-14, 8.8, 20000),
        (O.E4M3_GRID[:-1] + O.E4M3_GRID[1:]) / 2,        # every midpoint
    ]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.cast_e4m3(vals), ref)


# --------------------------------------------------------- P2 rounding ties

def test_hand_derived_rounding_points(golden):
    for fmt, x, code in golden("rounding_ties.txt"):
        a = np.array([float(x)], np.float32)
        if fmt == "e4m3":
            got = int(O.cast_e4m3(a)[0])
        else:
            got = int(O.round_rne(a, O.FP4 if fmt == "e2m1" else O.FP6)[0])
        assert got == int(code), (fmt, x, got, code)


# ------------------------------------------------------------ P11 Philox

def test_philox_known_answers(golden):
    for row in golden("philox4x32_10_kat.txt"):
        w = [int(t, 16) for t in row]
        out = O.philox4x32_10(np.array([w[:4]], np.uint32), (w[4], w[5]))[0]
        assert [int(v) for v in out] == w[6:]


def test_sr_uniforms_use_counter_i_div_4_and_word_i_mod_4():
    seed = 0x123456789
    idx = np.arange(12, dtype=np.uint64)
    u = O.sr_uniforms(seed, idx)
    for g in range(3):
        words = O.philox4x32_10(np.array([[g, 0, 0, 0]], np.uint32),
                                (seed & 0xFFFFFFFF, seed >> 32))[0]
        assert np.array_equal(u[4 * g:4 * g + 4], (words >> 8).astype(np.float64) * 2.0 ** -24)
    assert np.all((u >= 0) & (u < 1))


def test_sr_uniforms_sparse_and_compact_index_sets_agree():
    """The words of an index do not depend on which other indices are asked
    for: a scattered set (one Philox block per element) and each index on
    its own (one block per counter) give the same u; so does a contiguous
    range against its elements taken in reverse order."""
    rng = np.random.default_rng(3)
    idx = rng.choice(1 << 40, 64, replace=False).astype(np.uint64)
    seed = 0xDEADBEEF12
    together = O.sr_uniforms(seed, idx)
    alone = np.array([O.sr_uniforms(seed, idx[i:i + 1])[0] for i in range(idx.size)])
    assert np.array_equal(together, alone)
    rng_idx = np.arange(1000, 1400, dtype=np.uint64)
    assert np.array_equal(O.sr_uniforms(seed, rng_idx)[::-1], O.sr_uniforms(seed, rng_idx[::-1]))


def test_sr_decisions_by_hand_from_the_known_answer_words():
    """Seed 0 is Philox key (0, 0), and the first row of a 4-column view is
    counter (0, 0, 0, 0), whose words the first known-answer vector gives:
    u = (w >> 8)·2^-24 = 0x6627e8, 0xe169c5, 0xbc57ac, 0x9b00db over 2^24
    (0.399, 0.8805, 0.7357, 0.6055).  With max|x| = 2688 (T = 1, B = 448)
    the row 2688, 196, 616, -2240 sits at 6, 0.4375, 1.375, -5 in units of
    B·T: fractional positions 0, 0.875 (step 0.5), 0.75 (step 0.5), 0.5
    (step 2).  Round up iff u < f: 6 stays, 0.4375 goes down to 0, 1.375 up
    to 1.5, -5 down to -4 (codes 7, 0, 3, 0xE).  Round to nearest gives
    7, 1, 3, 0xE."""
    x = np.zeros((4, 4), np.float32)
    x[0] = [2688.0, 196.0, 616.0, -2240.0]
    q = O.quantize(x, O.FP4, O.SR, seed=0)
    assert q.T == np.float32(1.0) and q.scales[0, 0] == O.cast_e4m3(np.array([448.0], np.float32))[0]
    assert [int(c) for c in q.codes[0]] == [7, 0, 3, 0xE]
    r = O.quantize(x, O.FP4, O.RNE)
    assert [int(c) for c in r.codes[0]] == [7, 1, 3, 0xE]
    # E2M3 (max|x| = 3360, T = 1): 7.5, 0.109375 (f 0.875, step 1/8),
    # 2.1875 (f 0.75, step 1/4), -4.25 (f 0.5, step 1/2) -> 31, 0, 17, 0x38;
    # RNE: 31, 1, 17, 0x38 (-4.25 is a tie, to the even code 24)
    x[0] = [3360.0, 49.0, 980.0, -1904.0]
    q = O.quantize(x, O.FP6, O.SR, seed=0)
    assert q.T == np.float32(1.0)
    assert [int(c) for c in q.codes[0]] == [31, 0, 17, 0x38]
    r = O.quantize(x, O.FP6, O.RNE)
    assert [int(c) for c in r.codes[0]] == [31, 1, 17, 0x38]


# ------------------------------------------------ tensor/block scale formula

def test_tensor_scale_formula():
    x = np.zeros((4, 4), np.float32)
    x[1, 2] = -2688.0
    assert O.tensor_scale(x, O.FP4) == np.float32(1.0)
    x[1, 2] = 3360.0
    assert O.tensor_scale(x, O.FP6) == np.float32(1.0)


def test_zero_tensor_and_zero_block():
    z = np.zeros((8, 8), np.float32)
    z[0, 0] = -0.0
    q = O.quantize(z, O.FP4, O.RNE)
    assert q.T == 0 and not q.scales.any()
    assert q.codes[0, 0] == 0x8 and not q.codes.flatten()[1:].any()   # sign kept
    x = np.zeros((8, 8), np.float32)
    x[0, 0] = 1.0
    x[5, 5] = -0.0
    q = O.quantize(x, O.FP4, O.RNE)
    assert q.scales[1, 1] == 0 and q.codes[5, 5] == 0x8 and q.codes[4, 4] == 0


@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_zero_scale_block_of_nonzero_elements(rounding):
    """T = 1 (max|x| = 2688, FP4).  A block whose max is 6·2^-10 has
    bmax/(T·emax) = 2^-10, the E4M3 tie between 0 and 2^-9, which goes to
    the even code 0: its elements, though nonzero, get magnitude 0 and keep
    their sign.  A block max one ulp above rounds the scale up to 2^-9
    (code 1), and that element becomes 3·(1 + 2^-23) in units of B·T, which
    rounds to the grid value 3 (code 5) under RNE and to 3 or 4 under SR."""
    x = np.zeros((8, 8), np.float32)
    x[0, 0] = 2688.0
    m = np.float32(6 * 2.0 ** -10)
    x[4, 4], x[5, 6], x[6, 5] = m, -m / 2, np.float32(0.004)
    x[4, 0] = np.nextafter(m, np.float32(1))
    q = O.quantize(x, O.FP4, rounding, seed=3)
    assert q.T == np.float32(1.0)
    assert q.scales[1, 1] == 0
    assert (q.codes[4, 4], q.codes[5, 6], q.codes[6, 5]) == (0, 0x8, 0)
    assert q.scales[1, 0] == 1
    assert q.codes[4, 0] == 5 if rounding == O.RNE else q.codes[4, 0] in (5, 6)


# ------------------------------------- P3 exactness of representable blocks

@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_representable_blocks_are_recovered_exactly(fmt, rounding):
    """x = c·s·T with T a power of two, s an E4M3 scale and every block
    holding one element of the top code: quantization must return (c, s)."""
    rng = np.random.default_rng(7)
    rows, cols = 16, 24
    mb = O.element_bits(fmt) - 1
    ntop = (1 << mb) - 1
    grid = O.element_grid(fmt)
    T = np.float32(2.0 ** -5)
    s_codes = rng.integers(8, 127, size=(rows // 4, cols // 4))   # normal scales
    s_codes[0, 0] = 126                                           # the 448 block
    mags = rng.integers(0, ntop + 1, size=(rows, cols))
    signs = rng.integers(0, 2, size=(rows, cols))
    for bi in range(rows // 4):
        for bj in range(cols // 4):
            mags[4 * bi + rng.integers(4), 4 * bj + rng.integers(4)] = ntop
    s = np.repeat(np.repeat(O.E4M3_GRID[s_codes], 4, 0), 4, 1)
    x = (np.where(signs == 1, -1.0, 1.0) * grid[mags] * s * float(T)).astype(np.float32)
    assert O.tensor_scale(x, fmt) == T
    q = O.quantize(x, fmt, rounding, seed=3)
    assert np.array_equal(q.scales, s_codes.astype(np.uint8))
    assert np.array_equal(q.codes & ((1 << mb) - 1), mags)
    nz = mags != 0
    assert np.array_equal((q.codes >> mb)[nz], signs[nz])
    assert np.array_equal(O.dequantize(q), x.astype(np.float64))


# ------------------------------------------------------ P4 the global max

@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
def test_global_max_gets_top_scale_and_top_code(fmt):
    rng = np.random.default_rng(11)
    mb = O.element_bits(fmt) - 1
    for trial in range(20):
        x = (rng.standard_normal((32, 48)) * 10.0 ** rng.uniform(-6, 6)).astype(np.float32)
        if trial % 2:
            x.flat[rng.integers(x.size)] *= 100
        q = O.quantize(x, fmt, O.RNE)
        i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
        assert q.scales[i[0] // 4, i[1] // 4] == 126
        assert q.codes[i] & ((1 << mb) - 1) == (1 << mb) - 1
        assert (q.codes[i] >> mb) == int(np.signbit(x[i]))


# --------------------------------------------------- P10 RNE error bound

@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
def test_rne_error_within_half_spacing(fmt):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 64)).astype(np.float32)
    q = O.quantize(x, fmt, O.RNE)
    grid = O.element_grid(fmt)
    d = np.repeat(np.repeat(O.E4M3_GRID[q.scales], 4, 0), 4, 1) * np.float64(q.T)
    v = np.abs(x) / d
    lo = np.clip(np.searchsorted(grid, v, side="right") - 1, 0, len(grid) - 2)
    spacing = grid[lo + 1] - grid[lo]
    err = np.abs(x - O.dequantize(q))
    inside = v <= grid[-1]
    # fp32 rounding of v adds at most a few ulps of v
    assert np.all(err[inside] <= (0.5 * spacing[inside] + 4e-7 * v[inside]) * d[inside])


# --------------------------------------------- P6 stochastic rounding

def test_sr_is_unbiased_and_brackets():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((8, 8)) * 1e-3).astype(np.float32)
    x[0, 0] = 5e-3                                                  # fixes T
    q0 = O.quantize(x, O.FP4, O.RNE)
    lo = O.quantize(x, O.FP4, O.SR, seed=0)
    n = 2000
    acc = np.zeros(x.shape)
    acc2 = np.zeros(x.shape)
    grid = O.element_grid(O.FP4)
    d = np.repeat(np.repeat(O.E4M3_GRID[q0.scales], 4, 0), 4, 1) * np.float64(q0.T)
    v = np.abs(x).astype(np.float64) / d
    below = grid[np.clip(np.searchsorted(grid, v, side="right") - 1, 0, 7)]
    above = grid[np.clip(np.searchsorted(grid, v, side="left"), 0, 7)]
    for seed in range(n):
        q = O.quantize(x, O.FP4, O.SR, seed=seed)
        assert np.array_equal(q.scales, q0.scales) and q.T == q0.T
        mag = grid[q.codes & 7]
        assert np.all((mag == below) | (mag == above))
        xh = O.dequantize(q)
        acc += xh
        acc2 += xh * xh
    mean = acc / n
    var = np.maximum(acc2 / n - mean ** 2, 0)
    tol = 5 * np.sqrt(var / n) + 1e-6 * np.abs(x)   # + fp32 rounding of T
    sat = v > grid[-1]            # block scale rounded down: clamps (reading R5)
    assert np.all(np.abs(mean - x)[~sat] <= tol[~sat])
    assert np.all(np.abs(mean[sat]) == grid[-1] * d[sat])
    assert lo.codes.shape == x.shape


def test_sr_depends_on_seed_only_through_codes():
    x = np.random.default_rng(3).standard_normal((16, 16)).astype(np.float32)
    a = O.quantize(x, O.FP6, O.SR, seed=1)
    b = O.quantize(x, O.FP6, O.SR, seed=2)
    assert np.array_equal(a.scales, b.scales) and a.T == b.T
    assert not np.array_equal(a.codes, b.codes)


# ------------------------------------------------------- packing (R16)

def _outlier_tensor(rows, cols, seed):
    """Signed N(0,1) with 0.1 % of the entries x100 and the largest one
    placed in the first rows, outside every band below."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    idx = rng.choice(x.size, max(1, x.size // 1000), replace=False)
    x.reshape(-1)[idx] *= np.float32(100)
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    x[[0, r]] = x[[r, 0]]
    return x


@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_band_with_global_amax_equals_rows_of_whole_view(fmt, rounding):
    """Section "무엇과 다른가" takes T from max|X| of the whole tensor, and the
    stochastic-rounding counter is the element's index in the whole view
    (reading R8); so a band of rows quantized with the whole view's max|x|
    and its row offset is exactly those rows of the whole-view result: codes,
    scales and T.  The band below holds none of the largest elements."""
    x = _outlier_tensor(64, 24, 11)
    whole = O.quantize(x, fmt, rounding, seed=77)
    amax = float(np.max(np.abs(x)))
    assert np.max(np.abs(x[16:48])) < amax
    for r0, r1 in ((16, 48), (4, 8), (60, 64), (0, 64)):
        band = O.quantize(x[r0:r1], fmt, rounding, seed=77, amax=amax, row_offset=r0)
        assert band.T == whole.T
        assert np.array_equal(band.codes, whole.codes[r0:r1])
        assert np.array_equal(band.scales, whole.scales[r0 // 4:r1 // 4])
    if rounding == O.SR:
        # the offset matters: numbering the band from row 0 draws other words
        wrong = O.quantize(x[16:48], fmt, rounding, seed=77, amax=amax, row_offset=0)
        assert not np.array_equal(wrong.codes, whole.codes[16:48])


@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_column_window_equals_columns_of_whole_view(fmt, rounding):
    """A batch shard: columns [c0, c0 + w) of the [rows][cols] view (batch
    items c0.. of every (pixel, channel) row), quantized with the global
    max|x|, its column offset and the whole view's column count, is exactly
    those columns of the whole-view result (blocks never straddle a shard
    since c0 and w are multiples of 4); a band of rows of a shard likewise."""
    x = _outlier_tensor(32, 48, 12)
    whole = O.quantize(x, fmt, rounding, seed=5)
    amax = float(np.max(np.abs(x)))
    for c0, w in ((0, 16), (16, 16), (32, 16), (8, 4), (44, 4)):
        win = O.quantize(x[:, c0:c0 + w], fmt, rounding, seed=5, amax=amax, col_offset=c0, total_cols=48)
        assert win.T == whole.T
        assert np.array_equal(win.codes, whole.codes[:, c0:c0 + w])
        assert np.array_equal(win.scales, whole.scales[:, c0 // 4:(c0 + w) // 4])
    both = O.quantize(x[8:20, 20:28], fmt, rounding, seed=5, amax=amax, row_offset=8, col_offset=20,
                      total_cols=48)
    assert np.array_equal(both.codes, whole.codes[8:20, 20:28])
    assert np.array_equal(both.scales, whole.scales[2:5, 5:7])


def test_band_amax_sets_the_tensor_scale_formula():
    """With amax given, T = fp32(amax / (448·emax)) exactly as for the whole
    tensor (T depends on the band only through amax)."""
    x = _outlier_tensor(16, 16, 13)
    for fmt, emax in ((O.FP4, 6.0), (O.FP6, 7.5)):
        for amax in (1.0, 3.0, 1234.5, 1e-20):
            q = O.quantize(x[:8], fmt, O.RNE, amax=amax)
            assert q.T == np.float32(np.float32(amax) / np.float32(448.0 * emax))


def test_packing_bit_layout():
    assert list(O.pack_codes(np.array([[1, 2, 15, 0]]), O.FP4)) == [0x21, 0x0F]
    # codes 1, 2, 3, 4 -> 1 | 2<<6 | 3<<12 | 4<<18 = 0x103081, little-endian
    assert list(O.pack_codes(np.array([[1, 2, 3, 4]]), O.FP6)) == [0x81, 0x30, 0x10]
    rng = np.random.default_rng(0)
    for fmt, hi in ((O.FP4, 16), (O.FP6, 64)):
        c = rng.integers(0, hi, size=(8, 12))
        p = O.pack_codes(c, fmt)
        assert p.size == 8 * O.packed_row_bytes(12, fmt)
        assert np.array_equal(O.unpack_codes(p, 8, 12, fmt), c)


# ------------------------------------- replay form of post-ReLU tensors (R21)

def test_unsigned_pack_bit_layout_by_hand():
    # E2M1 magnitudes 1..7, 0 at 3 bits each: 1 | 2<<3 | 3<<6 | 4<<9 | 5<<12
    # | 6<<15 | 7<<18 = 2054353 = 0x1F58D1, little-endian bytes D1 58 1F.
    p, neg = O.pack_unsigned(np.array([[1, 2, 3, 4], [5, 6, 7, 0]]), O.FP4)
    assert list(p) == [0xD1, 0x58, 0x1F] and neg == 0
    # E2M3 magnitudes 31, 1, 0, 17, 2, 3, 4, 5 at 5 bits each:
    # 31 | 1<<5 | 17<<15 | 2<<20 | 3<<25 | 4<<30 | 5<<35 = 176196976703
    # = 0x290628803F, little-endian bytes 3F 80 28 06 29.
    p, neg = O.pack_unsigned(np.array([[31, 1, 0, 17], [2, 3, 4, 5]]), O.FP6)
    assert list(p) == [0x3F, 0x80, 0x28, 0x06, 0x29] and neg == 0


def test_unsigned_pack_drops_only_the_sign_bit():
    rng = np.random.default_rng(1)
    for fmt, hi in ((O.FP4, 8), (O.FP6, 32)):
        c = rng.integers(0, hi, size=(8, 12))
        p, neg = O.pack_unsigned(c, fmt)
        assert neg == 0 and p.size == 8 * 12 * O.magnitude_bits(fmt) // 8
        assert np.array_equal(O.unpack_unsigned(p, 8, 12, fmt), c)
        # one stored element spans bits [i·m, i·m+m): flipping bit k of the
        # stream changes element k // m by 2^(k % m) and nothing else
        m = O.magnitude_bits(fmt)
        for k in (0, m - 1, m, 5 * m + 2, 8 * 12 * m - 1):
            q = p.copy()
            q[k // 8] ^= 1 << (k % 8)
            d = O.unpack_unsigned(q, 8, 12, fmt).reshape(-1) - c.reshape(-1)
            assert np.count_nonzero(d) == 1 and abs(d[k // m]) == 1 << (k % m)


def test_unsigned_pack_counts_negative_codes_and_stores_relu():
    # sign bit set: -0 (mag 0) is fine, -1.5 (E2M1 0b1011) is counted and
    # stored as 0, +6 (0b0111) stays.
    p, neg = O.pack_unsigned(np.array([[0b1000, 0b1011, 0b0111, 0b1111]]), O.FP4)
    assert neg == 2
    assert list(O.unpack_unsigned(p, 1, 4, O.FP4)[0]) == [0, 0, 7, 0]


@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
def test_replay_form_of_relu_activations_dequantizes_to_the_same_values(fmt):
    """Quantizing ReLU(x) yields no negative code, and the replay form reads
    back exactly the values of the full codes; on a signed tensor it reads
    back max(x_hat, 0)."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((16, 32)).astype(np.float32)
    for src, relu in ((np.maximum(x, 0), True), (x, False)):
        q = O.quantize(src, fmt, O.RNE)
        p, neg = O.pack_unsigned(q.codes, fmt)
        back = O.QTensor(O.unpack_unsigned(p, 16, 32, fmt), q.scales, q.T, fmt)
        if relu:
            assert neg == 0
            assert np.array_equal(O.dequantize(back), O.dequantize(q))
        else:
            assert neg == int(np.count_nonzero(O.dequantize(q) < 0))
            assert np.array_equal(O.dequantize(back), np.maximum(O.dequantize(q), 0))


def test_replay_bits_per_element():
    # 3 magnitude bits + one E4M3 byte per 4 x 4 block = 3.5 bits (FP4); the
    # signed form holds 4.5.  The pages' 3.125 would need one byte per 64.
    assert O.unsigned_bits_per_element(O.FP4) == 3.5
    assert O.unsigned_bits_per_element(O.FP6) == 5.5
    assert O.bits_per_element(O.FP4) - O.unsigned_bits_per_element(O.FP4) == 1.0


# --------------------------------- P9 dequantized products fit f16 / bf16

@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
def test_code_times_scale_is_exact_in_half_precision(fmt):
    grid = O.element_grid(fmt)
    prods = np.outer(grid, O.E4M3_GRID).ravel()
    assert np.array_equal(prods.astype(np.float16).astype(np.float64), prods)
    t = torch.from_numpy(prods)
    assert torch.equal(t.to(torch.bfloat16).double(), t)


# ------------------------- P7 im2col GEMM == direct conv == library conv

SHAPES = [O.ConvShape(2, 4, 8, 5, 6, 3, 3, 1, 0), O.ConvShape(2, 8, 4, 7, 7, 3, 3, 2, 1),
          O.ConvShape(1, 4, 4, 4, 5, 1, 1, 1, 0), O.ConvShape(3, 4, 8, 6, 5, 3, 2, 2, 2)]


def _dyadic(rng, shape):
    return rng.integers(-8, 9, size=shape).astype(np.float64) / 8.0


@pytest.mark.parametrize("s", SHAPES)
def test_im2col_gemm_equals_seven_loop_conv(s):
    rng = np.random.default_rng(0)
    X = _dyadic(rng, (s.H, s.W, s.Cin, s.N))
    Wt = _dyadic(rng, (s.Cout, s.Kh, s.Kw, s.Cin))
    Y, _ = O.conv_fwd(Wt, X, s)
    assert np.array_equal(Y, O.direct_conv_fwd(Wt, X, s))


@pytest.mark.parametrize("s", SHAPES)
def test_three_gemms_match_torch_conv_fp64(s):
    rng = np.random.default_rng(1)
    X = rng.standard_normal((s.H, s.W, s.Cin, s.N))
    Wt = rng.standard_normal((s.Cout, s.Kh, s.Kw, s.Cin))
    G = rng.standard_normal((s.Ho, s.Wo, s.Cout, s.N))
    Xt = torch.from_numpy(X).permute(3, 2, 0, 1)          # NCHW
    Wtt = torch.from_numpy(Wt).permute(0, 3, 1, 2)        # OIHW
    Gt = torch.from_numpy(G).permute(3, 2, 0, 1)
    Y, _ = O.conv_fwd(Wt, X, s)
    ref = torch.nn.functional.conv2d(Xt, Wtt, stride=s.stride, padding=s.pad)
    assert np.allclose(Y, ref.permute(2, 3, 1, 0).numpy(), rtol=1e-12, atol=1e-12)
    GW, _ = O.conv_wgrad(G, X, s)
    ref = torch.nn.grad.conv2d_weight(Xt, Wtt.shape, Gt, stride=s.stride, padding=s.pad)
    assert np.allclose(GW, ref.permute(0, 2, 3, 1).numpy(), rtol=1e-12, atol=1e-12)
    GX, _ = O.conv_dgrad(Wt, G, s)
    ref = torch.nn.grad.conv2d_input(Xt.shape, Wtt, Gt, stride=s.stride, padding=s.pad)
    assert np.allclose(GX, ref.permute(2, 3, 1, 0).numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("s", SHAPES)
def test_single_output_functions_match_full_passes(s):
    rng = np.random.default_rng(2)
    X = rng.standard_normal((s.H, s.W, s.Cin, s.N))
    Wt = rng.standard_normal((s.Cout, s.Kh, s.Kw, s.Cin))
    G = rng.standard_normal((s.Ho, s.Wo, s.Cout, s.N))
    Y, SY = O.conv_fwd(Wt, X, s)
    GW, SW = O.conv_wgrad(G, X, s)
    GX, SX = O.conv_dgrad(Wt, G, s)
    for _ in range(20):
        i = tuple(int(rng.integers(d)) for d in Y.shape)
        v, S = O.fwd_at(Wt, X, s, *i)
        assert np.isclose(v, Y[i], rtol=1e-12, atol=1e-12) and np.isclose(S, SY[i])
        i = tuple(int(rng.integers(d)) for d in GW.shape)
        v, S = O.wgrad_at(G, X, s, *i)
        assert np.isclose(v, GW[i], rtol=1e-12, atol=1e-12) and np.isclose(S, SW[i])
        i = tuple(int(rng.integers(d)) for d in GX.shape)
        v, S = O.dgrad_at(Wt, G, s, *i)
        assert np.isclose(v, GX[i], rtol=1e-12, atol=1e-12) and np.isclose(S, SX[i])


# ------------------------------------------------------ P8 adjoint identity

@pytest.mark.parametrize("s", SHAPES)
def test_adjoint_identity_ties_the_three_gemms(s):
    """<conv(X, W), G> = <X, dgrad(G, W)> = <W, wgrad(G, X)>."""
    rng = np.random.default_rng(3)
    X = rng.standard_normal((s.H, s.W, s.Cin, s.N))
    Wt = rng.standard_normal((s.Cout, s.Kh, s.Kw, s.Cin))
    G = rng.standard_normal((s.Ho, s.Wo, s.Cout, s.N))
    a = np.sum(O.conv_fwd(Wt, X, s)[0] * G)
    b = np.sum(X * O.conv_dgrad(Wt, G, s)[0])
    c = np.sum(Wt * O.conv_wgrad(G, X, s)[0])
    assert np.isclose(a, b, rtol=1e-12) and np.isclose(a, c, rtol=1e-12)


# ----------------------------------- P5 one quantized value per pixel

def _values_per_pixel(mat, pix):
    groups = {}
    for k in range(pix.shape[0]):
        for p in range(pix.shape[1]):
            groups.setdefault(pix[k, p], set()).add(mat[k, p])
    return groups


@pytest.mark.parametrize("cin,along", [(16, "p"), (4, "k"), (8, "k")])
def test_quantize_once_gives_one_value_per_pixel_naive_does_not(cin, along):
    """Section "무엇인가": quantizing after im2col groups one pixel with
    different neighbours in different blocks, so its copies get different
    values; quantizing before im2col (the method) gives every copy one value."""
    s = O.ConvShape(4, cin, 16, 6, 6, 3, 3, 1, 0)
    rng = np.random.default_rng(4)
    X = rng.standard_normal((s.H, s.W, s.Cin, s.N)).astype(np.float32)
    X[rng.random(X.shape) < 0.05] *= 30
    pix = O.im2col(np.arange(X.size, dtype=np.float64).reshape(X.shape), s)
    xq = O.dequantize(O.quantize(X.reshape(s.x_view()), O.FP4, O.RNE)).reshape(X.shape)
    ours = _values_per_pixel(O.im2col(xq, s), pix)
    assert all(len(v) == 1 for v in ours.values())
    naive = _values_per_pixel(O.naive_quantize_after_im2col(X, s, O.FP4, along), pix)
    assert sum(len(v) > 1 for v in naive.values()) > 0


# ------------------------------------------ 16-element blocks (the naive scheme)

def test_1d_blocks_are_the_naive_im2col_quantization():
    """quantize_1d on the explicit im2col matrix (K rows x P columns) with
    blocks down its columns (along K) or along its rows (along P) dequantizes
    to the values of naive_quantize_after_im2col, the scheme of section
    "무엇인가" pinned above (P5): the same codes and scales, the values equal
    up to the fp32 rounding of B·T that function multiplies by (relative
    2^-24; a different code or scale would differ by 1/8 or more)."""
    s = O.ConvShape(4, 16, 8, 6, 6, 3, 3, 1, 1)
    rng = np.random.default_rng(21)
    X = rng.standard_normal((s.H, s.W, s.Cin, s.N)).astype(np.float32)
    Xc = O.im2col(X, s).astype(np.float32)                  # (Kh·Kw·Cin) x (Ho·Wo·N)
    for axis, along in ((0, "k"), (1, "p")):
        q = O.quantize_1d(Xc, O.FP4, O.RNE, axis=axis)
        got = O.code_values_1d(q) * np.float64(q.T)
        ref = O.naive_quantize_after_im2col(X, s, O.FP4, along)
        assert np.all(np.abs(got - ref) <= 2.0 ** -23 * np.abs(ref))
        assert np.count_nonzero(got) > 0.5 * got.size


@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
@pytest.mark.parametrize("axis", [0, 1])
def test_1d_representable_blocks_are_recovered_exactly(fmt, rounding, axis):
    """x = c·s·T with T a power of two and s an E4M3 value whose block
    holds the code emax: every step of the formula is exact, so the codes
    and scales come back unchanged (stochastic rounding leaves grid values
    where they are)."""
    rng = np.random.default_rng(22 + axis)
    grid = O.element_grid(fmt)
    nb, emax = 6, grid[-1]
    T = np.float32(2.0 ** -3)
    amax_block = 0
    s_codes = rng.integers(0x18, 0x60, nb).astype(np.uint8)
    s_codes[0] = 0x7E                                          # 448: the tensor max
    c = rng.integers(0, len(grid), (nb, 16))
    c[:, 0] = len(grid) - 1                                    # emax in every block
    sign = rng.integers(0, 2, (nb, 16))
    vals = np.where(sign == 1, -grid[c], grid[c]) * O.E4M3_GRID[s_codes][:, None] * np.float64(T)
    x = vals.astype(np.float32)                                # one block per row
    if axis == 0:
        x = x.T.copy()                                         # one block per column
    q = O.quantize_1d(x, fmt, rounding, seed=9, axis=axis)
    assert q.T == T
    want_codes = c | (sign << (O.element_bits(fmt) - 1))
    got_codes = q.codes if axis == 1 else q.codes.T
    got_scales = q.scales.reshape(-1)
    assert np.array_equal(got_scales, s_codes)
    assert np.array_equal(got_codes, want_codes)


@pytest.mark.parametrize("fmt", [O.FP4, O.FP6])
def test_1d_transposed_view_and_global_max(fmt):
    """Blocks down the columns of X are blocks along the rows of X^T (round
    to nearest: same codes and scales, transposed), and the element of
    largest magnitude gets scale 448 and the top code."""
    rng = np.random.default_rng(23)
    x = (rng.standard_normal((32, 48)) * np.exp(rng.standard_normal((32, 48)))).astype(np.float32)
    a = O.quantize_1d(x, fmt, O.RNE, axis=0)
    b = O.quantize_1d(np.ascontiguousarray(x.T), fmt, O.RNE, axis=1)
    assert a.T == b.T
    assert np.array_equal(a.codes, b.codes.T) and np.array_equal(a.scales, b.scales.T)
    r, cidx = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    top = len(O.element_grid(fmt)) - 1
    assert a.scales[r // 16, cidx] == O.cast_e4m3(np.array([448.0], np.float32))[0]
    assert a.codes[r, cidx] & top == top


def test_1d_stochastic_rounding_brackets_and_keeps_grid_values():
    """SR codes are always one of the two grid neighbours of x/(B·T), and
    values already on the grid never move (any seed)."""
    rng = np.random.default_rng(24)
    x = rng.standard_normal((16, 64)).astype(np.float32)
    rn = O.quantize_1d(x, O.FP4, O.RNE, axis=1)
    grid = O.element_grid(O.FP4)
    d = np.repeat(O.E4M3_GRID[rn.scales], 16, axis=1) * np.float64(rn.T)
    v = np.abs(x) / d
    for seed in (1, 2, 3):
        q = O.quantize_1d(x, O.FP4, O.SR, seed, axis=1)
        assert np.array_equal(q.scales, rn.scales)
        mag = grid[q.codes & 7]
        lo = grid[np.clip(np.searchsorted(grid, v, side="right") - 1, 0, 7)]
        hi = grid[np.clip(np.searchsorted(grid, v, side="left"), 0, 7)]
        assert np.all((mag == lo) | (mag == hi))
        on_grid = np.isin(v, grid)
        assert np.array_equal(mag[on_grid], v[on_grid])


def test_expanded_view_by_brute_force():
    """The naive scheme's expanded X' in the channel-batch-first layout of a
    1 x 1 convolution: row (ho, wo, kh, kw, ci), column n, value
    X[ho·s + kh - p][wo·s + kw - p][ci][n] or 0 outside (stride 2, pad 1)."""
    s = O.ConvShape(4, 3, 2, 5, 6, 3, 2, 2, 1)
    X = np.random.default_rng(25).standard_normal((s.H, s.W, s.Cin, s.N)).astype(np.float32)
    v = O.expanded_view(X, s).reshape(s.Ho, s.Wo, s.Kh, s.Kw, s.Cin, s.N)
    for ho in range(s.Ho):
        for wo in range(s.Wo):
            for kh in range(s.Kh):
                for kw in range(s.Kw):
                    hi, wi = ho * s.stride + kh - s.pad, wo * s.stride + kw - s.pad
                    want = X[hi, wi] if 0 <= hi < s.H and 0 <= wi < s.W else 0 * X[0, 0]
                    assert np.array_equal(v[ho, wo, kh, kw], want)


def test_naive_layer_gemms_against_torch():
    """The naive step's three GEMMs on its own quantized copies equal torch's
    fp64 contractions of the dequantized copies (einsum for Y and G_W, and
    conv2d_input for G_X = col2im(W^T·G_Y)), and each copy is the 1-D block
    quantization of its operand along the stated direction."""
    s = O.ConvShape(16, 16, 16, 5, 5, 3, 3, 1, 1)
    rng = np.random.default_rng(26)
    X = np.maximum(rng.standard_normal((s.H, s.W, s.Cin, s.N)), 0).astype(np.float32)
    Wt = (rng.standard_normal((s.Cout, s.Kh, s.Kw, s.Cin)) * 0.1).astype(np.float32)
    G = (rng.standard_normal((s.Ho, s.Wo, s.Cout, s.N)) * 1e-3).astype(np.float32)
    q, out = O.naive_layer(X, Wt, G, s, O.FP4, seed=3)
    K = s.Kh * s.Kw * s.Cin
    assert q["x_fwd"].axis == 0 and q["x_wgrad"].axis == 1 and q["w_fwd"].axis == 1
    assert q["w_dgrad"].axis == 0 and q["g_wgrad"].axis == 1 and q["g_dgrad"].axis == 0
    deq = {k: torch.from_numpy(O.code_values_1d(v) * np.float64(v.T)) for k, v in q.items()}
    xf = deq["x_fwd"].reshape(s.Ho * s.Wo, K, s.N)
    xw = deq["x_wgrad"].reshape(s.Ho * s.Wo, K, s.N)
    y = torch.einsum("ck,pkn->pcn", deq["w_fwd"], xf)
    gw = torch.einsum("pcn,pkn->ck", deq["g_wgrad"].reshape(s.Ho * s.Wo, s.Cout, s.N), xw)
    wd = deq["w_dgrad"].reshape(s.Cout, s.Kh, s.Kw, s.Cin).permute(0, 3, 1, 2)
    gd = deq["g_dgrad"].reshape(s.Ho, s.Wo, s.Cout, s.N).permute(3, 2, 0, 1)
    gx = torch.nn.grad.conv2d_input((s.N, s.Cin, s.H, s.W), wd, gd, stride=s.stride, padding=s.pad)
    np.testing.assert_allclose(out["y"][0].reshape(-1), y.numpy().reshape(-1), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(out["gw"][0].reshape(-1), gw.numpy().reshape(-1), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(out["gx"][0], gx.permute(2, 3, 1, 0).numpy(), rtol=1e-12, atol=1e-18)
    # the two directions give different copies of the same operand
    for a, b in (("x_fwd", "x_wgrad"), ("w_fwd", "w_dgrad"), ("g_wgrad", "g_dgrad")):
        assert not np.array_equal(O.code_values_1d(q[a]), O.code_values_1d(q[b]))


def test_naive_needs_two_copies():
    """The two GEMM directions quantize the same X' differently."""
    s = O.ConvShape(4, 16, 16, 6, 6, 3, 3, 1, 0)
    X = np.random.default_rng(5).standard_normal((s.H, s.W, s.Cin, s.N)).astype(np.float32)
    a = O.naive_quantize_after_im2col(X, s, O.FP4, "k")
    b = O.naive_quantize_after_im2col(X, s, O.FP4, "p")
    assert a.shape == b.shape and not np.array_equal(a, b)


def test_quantize_work_ratio_naive_vs_once():
    """Quantization work in elements: the naive scheme quantizes the
    Kh·Kw-inflated activation matrix (and W, G twice, once per GEMM
    direction); quantizing once touches each element once."""
    s = O.ConvShape(64, 128, 128, 28, 28, 3, 3, 1, 1)
    x_once = s.H * s.W * s.Cin * s.N
    x_naive = s.Kh * s.Kw * s.Cin * s.Ho * s.Wo * s.N
    assert x_naive / x_once == 9.0
    assert O.bits_per_element(O.FP4) == 4.5 and O.bits_per_element(O.FP6) == 6.5


# ------------------------ layer-level: T factors and rounding roles

def test_layer_outputs_apply_tensor_scales_and_roles():
    s = O.ConvShape(4, 8, 8, 5, 5, 3, 3, 1, 1)
    rng = np.random.default_rng(9)
    X = rng.standard_normal((s.H, s.W, s.Cin, s.N)).astype(np.float32)
    Wt = rng.standard_normal((s.Cout, s.Kh, s.Kw, s.Cin)).astype(np.float32)
    G = (rng.standard_normal((s.Ho, s.Wo, s.Cout, s.N)) * 1e-3).astype(np.float32)
    qx, qw, qg = O.quantize_layer(X, Wt, G, s, O.FP4, seed=5)
    out = O.layer_outputs(qx, qw, qg, s)
    Xh = O.dequantize(qx).reshape(X.shape)
    Wh = O.dequantize(qw).reshape(Wt.shape)
    Gh = O.dequantize(qg).reshape(G.shape)
    assert np.allclose(out["y"][0], O.conv_fwd(Wh, Xh, s)[0], rtol=1e-12, atol=0)
    assert np.allclose(out["gw"][0], O.conv_wgrad(Gh, Xh, s)[0], rtol=1e-12, atol=0)
    assert np.allclose(out["gx"][0], O.conv_dgrad(Wh, Gh, s)[0], rtol=1e-12, atol=0)
    # G_Y is stochastically rounded: another seed changes some codes
    qg2 = O.quantize(G.reshape(s.gy_view()), O.FP4, O.SR, seed=6)
    assert not np.array_equal(qg.codes, qg2.codes)
    assert np.array_equal(qx.codes, O.quantize(X.reshape(s.x_view()), O.FP4, O.RNE).codes)


# ----------------------------------- depthwise layers in BF16 (reading R22)

def test_bf16_rounding_by_hand_and_against_torch():
    """bfloat16 keeps 7 fraction bits.  By hand: 1 + 2^-8 lies halfway
    between 1 and 1 + 2^-7 and goes to the even 1; 1 + 3·2^-8 lies halfway
    between 1 + 2^-7 and 1 + 2^-6 and goes to the even 1 + 2^-6; one ulp
    above a halfway point rounds up.  Then torch's own conversion on random,
    tiny, subnormal and large values."""
    half = np.float32(1 + 2.0 ** -8)
    assert O.to_bf16(np.array([half]))[0] == 1.0
    assert O.to_bf16(np.array([np.float32(1 + 3 * 2.0 ** -8)]))[0] == np.float32(1 + 2.0 ** -6)
    assert O.to_bf16(np.array([np.nextafter(half, np.float32(2))]))[0] == np.float32(1 + 2.0 ** -7)
    assert O.to_bf16(np.array([np.float32(-1 - 2.0 ** -8)]))[0] == -1.0
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.standard_normal(100000), rng.standard_normal(1000) * 1e-39,
                        rng.standard_normal(1000) * 1e37, [0.0, -0.0, 3.0e38]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(O.to_bf16(x).view(np.uint32), ref.view(np.uint32))


DW_SHAPES = [O.ConvShape(4, 8, 8, 7, 9, 3, 3, 1, 1), O.ConvShape(4, 8, 8, 9, 7, 3, 3, 2, 1),
             O.ConvShape(8, 4, 4, 10, 10, 5, 5, 2, 2), O.ConvShape(4, 12, 12, 6, 6, 3, 1, 1, 0)]


@pytest.mark.parametrize("s", DW_SHAPES)
def test_depthwise_passes_match_torch_grouped_conv_fp64(s):
    """Depthwise fwd, weight and input gradients against torch's grouped
    convolution (groups = C) in float64, stride and padding included."""
    rng = np.random.default_rng(2)
    C = s.Cin
    X = rng.standard_normal((s.H, s.W, C, s.N))
    Wd = rng.standard_normal((C, s.Kh, s.Kw))
    G = rng.standard_normal((s.Ho, s.Wo, C, s.N))
    Xt = torch.from_numpy(X).permute(3, 2, 0, 1)          # NCHW
    Wt = torch.from_numpy(Wd).unsqueeze(1)               # C x 1 x Kh x Kw
    Gt = torch.from_numpy(G).permute(3, 2, 0, 1)
    Y, S = O.depthwise_fwd(Wd, X, s)
    ref = torch.nn.functional.conv2d(Xt, Wt, stride=s.stride, padding=s.pad, groups=C)
    assert np.allclose(Y, ref.permute(2, 3, 1, 0).numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(S >= np.abs(Y) - 1e-12)
    GW, _ = O.depthwise_wgrad(G, X, s)
    ref = torch.nn.grad.conv2d_weight(Xt, Wt.shape, Gt, stride=s.stride, padding=s.pad, groups=C)
    assert np.allclose(GW, ref[:, 0].numpy(), rtol=1e-12, atol=1e-12)
    GX, _ = O.depthwise_dgrad(Wd, G, s)
    ref = torch.nn.grad.conv2d_input(Xt.shape, Wt, Gt, stride=s.stride, padding=s.pad, groups=C)
    assert np.allclose(GX, ref.permute(2, 3, 1, 0).numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("s", DW_SHAPES)
def test_depthwise_adjoint_identity_and_bf16_operands(s):
    """<Y, G> = <X, G_X> = <W, G_W> for the three depthwise passes, and the
    layer function rounds every operand to bfloat16 before the exact sums
    (its outputs equal the passes on pre-rounded operands)."""
    rng = np.random.default_rng(3)
    C = s.Cin
    X = rng.standard_normal((s.H, s.W, C, s.N)).astype(np.float32)
    Wd = rng.standard_normal((C, s.Kh, s.Kw)).astype(np.float32)
    G = rng.standard_normal((s.Ho, s.Wo, C, s.N)).astype(np.float32)
    out = O.depthwise_layer_outputs(X, Wd, G, s)
    Xb, Wb, Gb = (O.to_bf16(t).astype(np.float64) for t in (X, Wd, G))
    a = np.sum(out["y"][0] * Gb)
    assert math.isclose(a, np.sum(Xb * out["gx"][0]), rel_tol=1e-12, abs_tol=1e-9)
    assert math.isclose(a, np.sum(Wb * out["gw"][0]), rel_tol=1e-12, abs_tol=1e-9)
    assert np.array_equal(out["y"][0], O.depthwise_fwd(Wb, Xb, s)[0])
    assert not np.array_equal(Xb, X.astype(np.float64))     # the rounding did something
