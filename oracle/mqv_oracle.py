"""Plain, slow CPU oracle of the MicroQonv hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline
leg and ``--impl reference`` arm) may call it.  It shares no code, table or
constant with the CUDA path: every definition below is written from the
method's description and from the OCP element-format definitions.

Sources (cited by page title and section):

* "MicroQonv" summary, onedev.kr/papers/182 (Korean), sections
  - "어떻게 동작하나" (how it works): quantize activations once, before the
    im2col expansion, and store them channel-batch-first, X_{Cin,N} in
    R^{Cin·(Hin·Win·N)}: for every pixel (h, w) all channels and all batch
    items are one contiguous block.
  - "무엇과 다른가" (how it differs): W_f reshaped to Cout·(Kh·Kw·Cin),
    G_Yf reshaped to Cout·(Hout·Wout·N); the three GEMMs Y = W·X',
    G_W = G_Y·X'^T, G_X' = W^T·G_Y; square blocks of B = 16 whose side covers
    sqrt(B) = 4 elements along both dimensions; NVFP4 two-level scaling
    T_scale = max|X| / (max B_sf × max B_ef),
    B_scale = CastE4M3(max|X_i| / (T_scale × max B_ef)),
    X_i^q = Round(X_i / (B_scale × T_scale)) to FP4 E2M1; round-to-nearest
    for activations and weights, stochastic rounding for gradients.
  - "어떻게 쓰나" (how it is used): the NVFP6 variant, FP6 E2M3 elements.
  - "무엇인가" (what it is): the naive scheme quantizes after im2col, so one
    pixel lands in several blocks with different quantized values.
* Element/scale bit layouts (the pages only name the formats): OCP
  Microscaling Formats (MX) v1.0, section 5.3 (E2M1, E2M3) and the OFP8 E4M3
  definition (bias 7, S.1111.111 = NaN, max 448, no infinity).
* Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
  Easy as 1, 2, 3", SC'11, section 3.2 (Philox S-box and key schedule).

Readings where the pages are silent (each also listed in the design notes):
  R1 formats: OCP MX v1.0 bit layouts.
  R2 precision: T, T·emax, m = bmax/(T·emax), d = B·T and v = x/d are each one
     IEEE fp32 operation, evaluated left to right as printed, no reciprocals.
  R3 "Round" for X and W is round-to-nearest, ties to the even code.
  R4 CastE4M3: round to nearest, ties to even code, saturate at 448.
  R5 |v| above the element maximum saturates to the maximum.
  R6 T == 0 or B == 0: all magnitudes in that tensor/block are 0.
  R7 the code's sign bit is the fp32 sign bit of x (so -0.1 may give -0).
  R8 SR: bracket |v| by grid neighbours lo <= |v| <= hi, f = (|v|-lo)/(hi-lo),
     round up iff u < f with u = (w >> 8)·2^-24; w is Philox4x32-10 word
     (i & 3) of counter (lo32(i>>2), hi32(i>>2), 0, 0) and key
     (lo32(seed), hi32(seed)), i the row-major index in the 2D view.
  R9 NVFP6 uses the same rounding roles as NVFP4.
  R10 W's K order is (kh, kw, cin), cin fastest.
  R11 channel-batch-first storage is [H][W][C][N], n fastest; a square block
      is 4 channels x 4 batch items at one pixel.
  R14 G_X = col2im(G_X'), the adjoint of im2col.
  R15 stride/padding follow the usual conv2d meaning (zero padding, floor).
  R16 packing: FP4 two codes per byte, even column in the low nibble; FP6
      four 6-bit codes per 3 bytes, code j at bits [6j, 6j+6) little-endian.
  R21 replay form of a post-ReLU tensor: magnitudes only (3 or 5 bits),
      element i at bits [i·m, i·m + m) of a little-endian bit stream; the
      E4M3 block scales and T are kept as they are.
  R22 depthwise layers, which the pages keep in BF16 outside the quantized
      path (section "전제와 한계"): one Kh x Kw filter per channel (groups
      = C, channel multiplier 1), weights [C][Kh][Kw], activations and
      gradients in the same [H][W][C][N] layout; every operand rounded to
      bfloat16 (round to nearest, ties to even), products summed exactly
      (fp64 here), outputs fp32.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

FP4 = "nvfp4"   # E2M1 elements
FP6 = "nvfp6"   # E2M3 elements
RNE = "rne"
SR = "sr"

# ---------------------------------------------------------------------------
# Element and scale formats (OCP MX v1.0 definitions)
# ---------------------------------------------------------------------------


def _decode_minifloat(code: int, ebits: int, mbits: int, bias: int) -> float:
    """Value of a sign/exponent/mantissa code with subnormals, no inf/NaN."""
    sign = -1.0 if (code >> (ebits + mbits)) & 1 else 1.0
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    if e == 0:
        return sign * (m / (1 << mbits)) * 2.0 ** (1 - bias)
    return sign * (1.0 + m / (1 << mbits)) * 2.0 ** (e - bias)


def decode_e2m1(code: int) -> float:
    """FP4 E2M1: s.ee.m, exponent bias 1 (OCP MX v1.0 sec. 5.3.3)."""
    return _decode_minifloat(code, 2, 1, 1)


def decode_e2m3(code: int) -> float:
    """FP6 E2M3: s.ee.mmm, exponent bias 1 (OCP MX v1.0 sec. 5.3.2)."""
    return _decode_minifloat(code, 2, 3, 1)


def decode_e4m3(code: int) -> float:
    """FP8 E4M3: s.eeee.mmm, bias 7; S.1111.111 is NaN, there is no infinity."""
    if code & 0x7F == 0x7F:
        return float("nan")
    return _decode_minifloat(code, 4, 3, 7)


def element_bits(fmt: str) -> int:
    return 4 if fmt == FP4 else 6


def element_grid(fmt: str) -> np.ndarray:
    """Non-negative element values in magnitude-code order (code 0 first)."""
    if fmt == FP4:
        return np.array([decode_e2m1(c) for c in range(8)], dtype=np.float64)
    return np.array([decode_e2m3(c) for c in range(32)], dtype=np.float64)


def element_max(fmt: str) -> float:
    """max B_ef of the scale formula: the largest element magnitude."""
    return float(element_grid(fmt)[-1])


E4M3_GRID = np.array([decode_e4m3(c) for c in range(0x7F)], dtype=np.float64)
E4M3_MAX = float(E4M3_GRID[-1])   # max B_sf of the scale formula


def _nearest_even(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to each a (a >= 0, grid ascending),
    ties to the even index, values above the top saturate to the top."""
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(grid, a, side="left")          # grid[hi] >= a
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    dlo = a - grid[lo]
    dhi = grid[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a >= grid[-1], len(grid) - 1, idx)
    idx = np.where(a <= 0, 0, idx)
    return idx.astype(np.int64)


def cast_e4m3(m: np.ndarray) -> np.ndarray:
    """CastE4M3 of non-negative fp32 values: nearest E4M3 value, ties to the
    even code, saturating at 448 (reading R4).  Returns uint8 codes."""
    return _nearest_even(np.asarray(m, dtype=np.float32), E4M3_GRID).astype(np.uint8)


def round_rne(a: np.ndarray, fmt: str) -> np.ndarray:
    """Round non-negative fp32 magnitudes onto the element grid, nearest,
    ties to even code, saturating at the element maximum (readings R3, R5)."""
    return _nearest_even(np.asarray(a, dtype=np.float32), element_grid(fmt))


def round_sr(a: np.ndarray, u: np.ndarray, fmt: str) -> np.ndarray:
    """Stochastic rounding of non-negative fp32 magnitudes (reading R8):
    lo <= a <= hi are the grid neighbours, round up iff u < (a-lo)/(hi-lo).
    Values on the grid stay; values above the top saturate."""
    grid = element_grid(fmt)
    a = np.asarray(a, dtype=np.float32).astype(np.float64)
    lo = np.searchsorted(grid, a, side="right") - 1      # grid[lo] <= a
    lo = np.clip(lo, 0, len(grid) - 1)
    top = lo >= len(grid) - 1
    hi = np.minimum(lo + 1, len(grid) - 1)
    span = np.where(top, 1.0, grid[hi] - grid[lo])
    f = np.where(top, 0.0, (a - grid[lo]) / span)
    up = (~top) & (np.asarray(u, dtype=np.float64) < f)
    return np.where(up, hi, lo).astype(np.int64)


# ---------------------------------------------------------------------------
# Philox4x32-10 (Salmon et al., SC'11, sec. 3.2)
# ---------------------------------------------------------------------------

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9   # golden ratio
PHILOX_W1 = 0xBB67AE85   # sqrt(3) - 1


def philox4x32_10(ctr: np.ndarray, key) -> np.ndarray:
    """ctr: (n, 4) uint32 counters, key: two uint32 words. Returns (n, 4)."""
    c = np.asarray(ctr, dtype=np.uint64).reshape(-1, 4).copy()
    k0 = np.uint64(int(key[0]) & 0xFFFFFFFF)
    k1 = np.uint64(int(key[1]) & 0xFFFFFFFF)
    mask = np.uint64(0xFFFFFFFF)
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & mask
            k1 = (k1 + np.uint64(PHILOX_W1)) & mask
        p0 = np.uint64(PHILOX_M0) * c[:, 0]
        p1 = np.uint64(PHILOX_M1) * c[:, 2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c = np.stack([hi1 ^ c[:, 1] ^ k0, lo1, hi0 ^ c[:, 3] ^ k1, lo0], axis=1)
    return c.astype(np.uint32)


def sr_uniforms(seed: int, index: np.ndarray) -> np.ndarray:
    """u = (w >> 8)·2^-24 for the element indices given (reading R8).

    Element i uses word i & 3 of the Philox block of counter i >> 2.  When
    the indices cover a compact range of counters (a whole view or a band of
    one), each counter's block is computed once and its four words serve the
    four elements that share it; otherwise one block per element."""
    index = np.asarray(index, dtype=np.uint64).reshape(-1)
    if index.size == 0:
        return np.zeros(0, np.float64)
    group = index >> np.uint64(2)
    g0 = int(group.min())
    span = int(group.max()) - g0 + 1
    if span <= index.size:
        counters = np.arange(g0, g0 + span, dtype=np.uint64)
        row = (group - np.uint64(g0)).astype(np.int64)
    else:
        counters, row = group, np.arange(index.size)
    ctr = np.zeros((counters.size, 4), dtype=np.uint64)
    ctr[:, 0] = counters & np.uint64(0xFFFFFFFF)
    ctr[:, 1] = counters >> np.uint64(32)
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    w = words[row, (index & np.uint64(3)).astype(np.int64)]
    return (w >> np.uint32(8)).astype(np.float64) * 2.0 ** -24


# ---------------------------------------------------------------------------
# Two-level square-block quantizer
# ---------------------------------------------------------------------------


@dataclass
class QTensor:
    codes: np.ndarray    # int64 (rows, cols): sign bit | magnitude code
    scales: np.ndarray   # uint8 (rows/4, cols/4): E4M3 block scales
    T: np.float32        # tensor scale
    fmt: str

    @property
    def rows(self) -> int:
        return self.codes.shape[0]

    @property
    def cols(self) -> int:
        return self.codes.shape[1]


def tensor_scale(x: np.ndarray, fmt: str) -> np.float32:
    """T_scale = max|X| / (max B_sf × max B_ef), in fp32 (reading R2)."""
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    return np.float32(amax / np.float32(E4M3_MAX * element_max(fmt)))


def quantize(x2d: np.ndarray, fmt: str, rounding: str, seed: int = 0,
             amax: float | None = None, row_offset: int = 0,
             col_offset: int = 0, total_cols: int | None = None) -> QTensor:
    """Square-block (4 x 4) two-level quantization of a 2D fp32 view.

    Follows the NVFP4 formulas of section "무엇과 다른가": tensor scale,
    then per 4x4 block B = CastE4M3(blockmax / (T × emax)), then every
    element x -> Round(x / (B × T)).  Rounding is RNE or SR (reading R8).

    `amax`/`row_offset` quantize a band of rows of a larger view whose
    max|x| is `amax` and whose first row here is row `row_offset` (used to
    spot-check very large tensors band by band; the SR counter uses the
    element's index in the full view).  `col_offset`/`total_cols` do the same
    for a window of columns (a batch shard of a wider view)."""
    x = np.ascontiguousarray(x2d, dtype=np.float32)
    rows, cols = x.shape
    assert rows % 4 == 0 and cols % 4 == 0 and row_offset % 4 == 0
    emax = np.float32(element_max(fmt))
    if amax is None:
        T = tensor_scale(x, fmt)
    else:
        T = np.float32(np.float32(amax) / np.float32(E4M3_MAX * element_max(fmt)))
    blocks = np.abs(x).reshape(rows // 4, 4, cols // 4, 4)
    bmax = blocks.max(axis=(1, 3)).astype(np.float32)
    mbits = element_bits(fmt) - 1
    sign = np.signbit(x).astype(np.int64) << mbits
    if T == 0:
        return QTensor(sign, np.zeros((rows // 4, cols // 4), np.uint8), T, fmt)
    m = (bmax / np.float32(T * emax)).astype(np.float32)
    scales = cast_e4m3(m)
    B = E4M3_GRID[scales].astype(np.float32)
    d = np.repeat(np.repeat((B * T).astype(np.float32), 4, axis=0), 4, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (np.abs(x) / d).astype(np.float32)     # |x/d| == |x|/d exactly
    v = np.where(d == 0, np.float32(0), v)
    if rounding == RNE:
        mag = round_rne(v, fmt)
    else:
        tc = cols if total_cols is None else total_cols
        r_idx = np.arange(rows, dtype=np.uint64)[:, None] + np.uint64(row_offset)
        c_idx = np.arange(cols, dtype=np.uint64)[None, :] + np.uint64(col_offset)
        u = sr_uniforms(seed, (r_idx * np.uint64(tc) + c_idx).reshape(-1)).reshape(rows, cols)
        mag = round_sr(v, u, fmt)
    mag = np.where(d == 0, 0, mag)
    return QTensor(sign | mag, scales, T, fmt)


def code_values(q: QTensor) -> np.ndarray:
    """Element values code·B without the tensor scale, fp64 (exact)."""
    mbits = element_bits(q.fmt) - 1
    grid = element_grid(q.fmt)
    mag = grid[q.codes & ((1 << mbits) - 1)]
    val = np.where((q.codes >> mbits) & 1, -mag, mag)
    B = np.repeat(np.repeat(E4M3_GRID[q.scales], 4, axis=0), 4, axis=1)
    return val * B


def dequantize(q: QTensor) -> np.ndarray:
    """x_hat = code·B·T in fp64."""
    return code_values(q) * np.float64(q.T)


def pack_codes(codes: np.ndarray, fmt: str) -> np.ndarray:
    """Row-major packed bytes (reading R16)."""
    c = np.asarray(codes, dtype=np.uint32)
    rows, cols = c.shape
    if fmt == FP4:
        pairs = c.reshape(rows, cols // 2, 2)
        return (pairs[:, :, 0] | (pairs[:, :, 1] << 4)).astype(np.uint8).reshape(-1)
    quads = c.reshape(rows, cols // 4, 4)
    word = quads[..., 0] | (quads[..., 1] << 6) | (quads[..., 2] << 12) | (quads[..., 3] << 18)
    out = np.stack([word & 0xFF, (word >> 8) & 0xFF, (word >> 16) & 0xFF], axis=-1)
    return out.astype(np.uint8).reshape(-1)


def unpack_codes(packed: np.ndarray, rows: int, cols: int, fmt: str) -> np.ndarray:
    b = np.asarray(packed, dtype=np.uint32)
    if fmt == FP4:
        b = b.reshape(rows, cols // 2)
        return np.stack([b & 0xF, b >> 4], axis=-1).reshape(rows, cols).astype(np.int64)
    b = b.reshape(rows, cols // 4, 3)
    word = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)
    out = np.stack([(word >> (6 * j)) & 0x3F for j in range(4)], axis=-1)
    return out.reshape(rows, cols).astype(np.int64)


def packed_row_bytes(cols: int, fmt: str) -> int:
    return cols // 2 if fmt == FP4 else cols * 3 // 4


# ---------------------------------------------------------------------------
# Latent-replay storage of post-ReLU tensors (reading R21)
# ---------------------------------------------------------------------------


def magnitude_bits(fmt: str) -> int:
    """Bits of an element code without its sign: 3 (E2M1) or 5 (E2M3)."""
    return element_bits(fmt) - 1


def pack_unsigned(codes: np.ndarray, fmt: str):
    """Sections "어떻게 쓰나" and "전제와 한계": an activation after ReLU is never
    negative, so its E2M1 code needs no sign bit and 3 bits per pixel remain.
    Reading R21: element i of the row-major view (its magnitude bits, least
    significant first) fills bits [i·m, i·m + m) of a bit stream stored
    little-endian, m = magnitude_bits(fmt).  A code with the sign bit and a
    nonzero magnitude cannot be stored; it is stored as 0 (the ReLU of its
    value) and counted.  Returns (bytes, count of such codes)."""
    c = np.asarray(codes, dtype=np.int64).reshape(-1)
    m = magnitude_bits(fmt)
    mag = c & ((1 << m) - 1)
    negative = (((c >> m) & 1) == 1) & (mag != 0)
    mag = np.where(negative, 0, mag)
    bits = (mag[:, None] >> np.arange(m)[None, :]) & 1
    return np.packbits(bits.reshape(-1).astype(np.uint8), bitorder="little"), int(negative.sum())


def unpack_unsigned(packed: np.ndarray, rows: int, cols: int, fmt: str) -> np.ndarray:
    """Codes (sign bit 0) of the view stored by pack_unsigned."""
    m = magnitude_bits(fmt)
    n = rows * cols
    bits = np.unpackbits(np.asarray(packed, dtype=np.uint8), bitorder="little")[:n * m]
    mag = (bits.reshape(n, m).astype(np.int64) << np.arange(m)[None, :]).sum(axis=1)
    return mag.reshape(rows, cols)


def unsigned_bits_per_element(fmt: str) -> float:
    """Stored bits per element of the replay form: magnitude plus one E4M3
    byte per 16 elements (T is one float per tensor and is not counted)."""
    return magnitude_bits(fmt) + 8.0 / 16.0


# ---------------------------------------------------------------------------
# Convolution shapes and the three GEMMs on the dequantized operands
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class ConvShape:
    N: int
    Cin: int
    Cout: int
    H: int
    W: int
    Kh: int
    Kw: int
    stride: int = 1
    pad: int = 0

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - self.Kh) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad - self.Kw) // self.stride + 1

    # 2D views used by the quantizer: (rows, cols)
    def x_view(self):
        return (self.H * self.W * self.Cin, self.N)

    def w_view(self):
        return (self.Cout, self.Kh * self.Kw * self.Cin)

    def gy_view(self):
        return (self.Ho * self.Wo * self.Cout, self.N)

    def flops(self) -> int:
        return 2 * self.Cout * self.Cin * self.Kh * self.Kw * self.Ho * self.Wo * self.N


def im2col(X: np.ndarray, s: ConvShape) -> np.ndarray:
    """X [H][W][Cin][N] -> X' with rows (kh, kw, ci) and columns (ho, wo, n).
    Zero padding; padding zeros are exact zeros (reading R15)."""
    Xp = np.zeros((s.H + 2 * s.pad, s.W + 2 * s.pad, s.Cin, s.N), dtype=X.dtype)
    Xp[s.pad:s.pad + s.H, s.pad:s.pad + s.W] = X
    out = np.empty((s.Kh, s.Kw, s.Cin, s.Ho, s.Wo, s.N), dtype=X.dtype)
    for kh in range(s.Kh):
        for kw in range(s.Kw):
            patch = Xp[kh:kh + s.stride * (s.Ho - 1) + 1:s.stride,
                       kw:kw + s.stride * (s.Wo - 1) + 1:s.stride]
            out[kh, kw] = patch.transpose(2, 0, 1, 3)
    return out.reshape(s.Kh * s.Kw * s.Cin, s.Ho * s.Wo * s.N)


def col2im(cols: np.ndarray, s: ConvShape) -> np.ndarray:
    """Adjoint of im2col: scatter-add the (kh, kw, ci) x (ho, wo, n) matrix
    back to [H][W][Cin][N] (reading R14)."""
    c = cols.reshape(s.Kh, s.Kw, s.Cin, s.Ho, s.Wo, s.N)
    Xp = np.zeros((s.H + 2 * s.pad, s.W + 2 * s.pad, s.Cin, s.N), dtype=cols.dtype)
    for kh in range(s.Kh):
        for kw in range(s.Kw):
            Xp[kh:kh + s.stride * (s.Ho - 1) + 1:s.stride,
               kw:kw + s.stride * (s.Wo - 1) + 1:s.stride] += c[kh, kw].transpose(1, 2, 0, 3)
    return Xp[s.pad:s.pad + s.H, s.pad:s.pad + s.W].copy()


def conv_fwd(Wv: np.ndarray, Xv: np.ndarray, s: ConvShape):
    """Y = W·X' with W as Cout x (Kh·Kw·Cin) and X' = im2col(X).
    Wv [Cout][Kh][Kw][Cin], Xv [H][W][Cin][N], fp64.  Returns
    (Y [Ho][Wo][Cout][N], S) with S = sum_k |W_k·X'_k| per output."""
    W2 = Wv.reshape(s.Cout, -1)
    Xc = im2col(Xv, s)
    Y = W2 @ Xc
    S = np.abs(W2) @ np.abs(Xc)
    shape = (s.Cout, s.Ho, s.Wo, s.N)
    return (Y.reshape(shape).transpose(1, 2, 0, 3).copy(),
            S.reshape(shape).transpose(1, 2, 0, 3).copy())


def _gy_matrix(Gv: np.ndarray, s: ConvShape) -> np.ndarray:
    """G_Y [Ho][Wo][Cout][N] -> Cout x (Ho·Wo·N), the 2D form of the pages."""
    return Gv.transpose(2, 0, 1, 3).reshape(s.Cout, s.Ho * s.Wo * s.N)


def conv_wgrad(Gv: np.ndarray, Xv: np.ndarray, s: ConvShape):
    """G_W = G_Y·X'^T -> ([Cout][Kh][Kw][Cin], S)."""
    G2 = _gy_matrix(Gv, s)
    Xc = im2col(Xv, s)
    GW = G2 @ Xc.T
    S = np.abs(G2) @ np.abs(Xc).T
    shape = (s.Cout, s.Kh, s.Kw, s.Cin)
    return GW.reshape(shape), S.reshape(shape)


def conv_dgrad(Wv: np.ndarray, Gv: np.ndarray, s: ConvShape):
    """G_X' = W^T·G_Y, then G_X = col2im(G_X') -> ([H][W][Cin][N], S)."""
    W2 = Wv.reshape(s.Cout, -1)
    G2 = _gy_matrix(Gv, s)
    GX = col2im(W2.T @ G2, s)
    S = col2im(np.abs(W2).T @ np.abs(G2), s)
    return GX, S


def direct_conv_fwd(Wv: np.ndarray, Xv: np.ndarray, s: ConvShape) -> np.ndarray:
    """The seven-loop definition of a strided, zero-padded convolution."""
    Y = np.zeros((s.Ho, s.Wo, s.Cout, s.N), dtype=np.float64)
    for n in range(s.N):
        for co in range(s.Cout):
            for ho in range(s.Ho):
                for wo in range(s.Wo):
                    acc = 0.0
                    for ci in range(s.Cin):
                        for kh in range(s.Kh):
                            for kw in range(s.Kw):
                                hi = ho * s.stride + kh - s.pad
                                wi = wo * s.stride + kw - s.pad
                                if 0 <= hi < s.H and 0 <= wi < s.W:
                                    acc += Wv[co, kh, kw, ci] * Xv[hi, wi, ci, n]
                    Y[ho, wo, co, n] = acc
    return Y


# --- single outputs, for spot checks at full size ---------------------------


def fwd_at(Wv, Xv, s: ConvShape, ho, wo, co, n):
    """One Y element and its S, straight from the definition."""
    acc = 0.0
    S = 0.0
    for kh in range(s.Kh):
        hi = ho * s.stride + kh - s.pad
        if not 0 <= hi < s.H:
            continue
        for kw in range(s.Kw):
            wi = wo * s.stride + kw - s.pad
            if not 0 <= wi < s.W:
                continue
            p = Wv[co, kh, kw, :] * Xv[hi, wi, :, n]
            acc += float(np.sum(p))
            S += float(np.sum(np.abs(p)))
    return acc, S


def wgrad_at(Gv, Xv, s: ConvShape, co, kh, kw, ci):
    """One G_W element: sum over (ho, wo, n) of G_Y·X'."""
    acc = 0.0
    S = 0.0
    for ho in range(s.Ho):
        hi = ho * s.stride + kh - s.pad
        if not 0 <= hi < s.H:
            continue
        for wo in range(s.Wo):
            wi = wo * s.stride + kw - s.pad
            if not 0 <= wi < s.W:
                continue
            p = Gv[ho, wo, co, :] * Xv[hi, wi, ci, :]
            acc += float(np.sum(p))
            S += float(np.sum(np.abs(p)))
    return acc, S


def dgrad_at(Wv, Gv, s: ConvShape, hi, wi, ci, n):
    """One G_X element: every (kh, kw, ho, wo) with ho·s + kh - pad == hi."""
    acc = 0.0
    S = 0.0
    for kh in range(s.Kh):
        t = hi + s.pad - kh
        if t % s.stride:
            continue
        ho = t // s.stride
        if not 0 <= ho < s.Ho:
            continue
        for kw in range(s.Kw):
            u = wi + s.pad - kw
            if u % s.stride:
                continue
            wo = u // s.stride
            if not 0 <= wo < s.Wo:
                continue
            p = Wv[:, kh, kw, ci] * Gv[ho, wo, :, n]
            acc += float(np.sum(p))
            S += float(np.sum(np.abs(p)))
    return acc, S


# ---------------------------------------------------------------------------
# MicroQonv layer pass and the naive scheme it replaces
# ---------------------------------------------------------------------------


def quantize_layer(X, Wt, GY, s: ConvShape, fmt: str, seed: int = 0):
    """Quantize each operand once in its 2D view: X and W with RNE, G_Y with
    SR (section "무엇과 다른가"; reading R9 for NVFP6)."""
    qx = quantize(X.reshape(s.x_view()), fmt, RNE)
    qw = quantize(Wt.reshape(s.w_view()), fmt, RNE)
    qg = quantize(GY.reshape(s.gy_view()), fmt, SR, seed)
    return qx, qw, qg


def layer_outputs(qx: QTensor, qw: QTensor, qg: QTensor, s: ConvShape):
    """The three GEMM results in fp64, with the two tensor scales applied as
    a scalar factor, plus their |product| sums for the tolerance."""
    Xv = code_values(qx).reshape(s.H, s.W, s.Cin, s.N)
    Wv = code_values(qw).reshape(s.Cout, s.Kh, s.Kw, s.Cin)
    Gv = code_values(qg).reshape(s.Ho, s.Wo, s.Cout, s.N)
    twx = np.float64(qw.T) * np.float64(qx.T)
    tgx = np.float64(qg.T) * np.float64(qx.T)
    twg = np.float64(qw.T) * np.float64(qg.T)
    Y, SY = conv_fwd(Wv, Xv, s)
    GW, SW = conv_wgrad(Gv, Xv, s)
    GX, SX = conv_dgrad(Wv, Gv, s)
    return {"y": (Y * twx, SY * twx), "gw": (GW * tgx, SW * tgx), "gx": (GX * twg, SX * twg)}


def naive_quantize_after_im2col(X: np.ndarray, s: ConvShape, fmt: str, along: str = "k") -> np.ndarray:
    """The scheme of section "무엇인가": expand X with im2col first, then
    quantize the (Kh·Kw·Cin) x (Ho·Wo·N) matrix X' with plain 1 x 16 NVFP4
    blocks along the contraction direction of one GEMM: along K (rows,
    (kh, kw, ci)) for Y = W·X', along P (columns, (ho, wo, n)) for
    G_W = G_Y·X'^T.  Each direction needs its own quantized copy, which is
    the double quantization the method removes.  Returns the dequantized
    expanded matrix, same shape as X'."""
    Xc = im2col(X.astype(np.float32), s).astype(np.float32)
    M = Xc.T if along == "k" else Xc          # blocks run along the last axis
    R, L = M.shape
    Lp = -(-L // 16) * 16
    Mp = np.zeros((R, Lp), np.float32)
    Mp[:, :L] = M
    emax = np.float32(element_max(fmt))
    T = tensor_scale(Mp, fmt)
    bmax = np.abs(Mp.reshape(R, Lp // 16, 16)).max(axis=2).astype(np.float32)
    B = E4M3_GRID[cast_e4m3((bmax / np.float32(T * emax)).astype(np.float32))].astype(np.float32)
    d = np.repeat((B * T).astype(np.float32), 16, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(d == 0, np.float32(0), (np.abs(Mp) / d).astype(np.float32))
    mag = element_grid(fmt)[round_rne(v, fmt)]
    xhat = (np.where(np.signbit(Mp), -mag, mag) * d.astype(np.float64))[:, :L]
    return xhat.T if along == "k" else xhat


@dataclass
class QTensor1D:
    codes: np.ndarray    # int64 (rows, cols): sign bit | magnitude code
    scales: np.ndarray   # uint8: (rows, cols/16) for blocks along a row, (rows/16, cols) down a column
    T: np.float32
    fmt: str
    axis: int            # 1: 1 x 16 blocks along a row; 0: 16 x 1 blocks down a column


def quantize_1d(x2d: np.ndarray, fmt: str, rounding: str, seed: int = 0, axis: int = 1) -> QTensor1D:
    """Two-level quantization with plain 16-element blocks along one axis of
    a 2D view: the NVFP4 formulas of section "무엇과 다른가" (T from max|X|,
    B = CastE4M3(blockmax / (T·emax)), code = Round(x / (B·T))) on the
    blocks the scheme of section "무엇인가" uses, 16 consecutive elements of
    a GEMM operand along its contraction.  axis = 1: 1 x 16 blocks along each
    row (cols a multiple of 16); axis = 0: 16 x 1 blocks down each column
    (rows a multiple of 16).  Rounding as in `quantize` (RNE, or SR with the
    row-major index of the element in the view)."""
    x = np.ascontiguousarray(x2d, dtype=np.float32)
    rows, cols = x.shape
    assert (cols if axis == 1 else rows) % 16 == 0
    emax = np.float32(element_max(fmt))
    T = tensor_scale(x, fmt)
    mbits = element_bits(fmt) - 1
    sign = np.signbit(x).astype(np.int64) << mbits
    shape = (rows, cols // 16) if axis == 1 else (rows // 16, cols)
    if T == 0:
        return QTensor1D(sign, np.zeros(shape, np.uint8), T, fmt, axis)
    a = np.abs(x)
    bmax = (a.reshape(rows, cols // 16, 16).max(axis=2) if axis == 1
            else a.reshape(rows // 16, 16, cols).max(axis=1)).astype(np.float32)
    scales = cast_e4m3((bmax / np.float32(T * emax)).astype(np.float32))
    B = E4M3_GRID[scales].astype(np.float32)
    d = (B * T).astype(np.float32)
    d = np.repeat(d, 16, axis=1) if axis == 1 else np.repeat(d, 16, axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (a / d).astype(np.float32)
    v = np.where(d == 0, np.float32(0), v)
    if rounding == RNE:
        mag = round_rne(v, fmt)
    else:
        idx = np.arange(rows * cols, dtype=np.uint64)
        mag = round_sr(v, sr_uniforms(seed, idx).reshape(rows, cols), fmt)
    mag = np.where(d == 0, 0, mag)
    return QTensor1D(sign | mag, scales, T, fmt, axis)


def code_values_1d(q: QTensor1D) -> np.ndarray:
    """code·B of a 1-D-block quantized view, fp64 (exact)."""
    mbits = element_bits(q.fmt) - 1
    mag = element_grid(q.fmt)[q.codes & ((1 << mbits) - 1)]
    val = np.where((q.codes >> mbits) & 1, -mag, mag)
    B = E4M3_GRID[q.scales]
    return val * (np.repeat(B, 16, axis=1) if q.axis == 1 else np.repeat(B, 16, axis=0))


def expanded_view(X: np.ndarray, s: ConvShape) -> np.ndarray:
    """X' of the naive scheme in the channel-batch-first layout of a 1 x 1
    convolution with Kh·Kw·Cin input channels: rows (ho, wo, kh, kw, ci),
    columns n (the im2col matrix with its column index (ho, wo, n) split)."""
    K = s.Kh * s.Kw * s.Cin
    return np.ascontiguousarray(im2col(X, s).reshape(K, s.Ho * s.Wo, s.N).transpose(1, 0, 2)).reshape(-1, s.N)


def naive_layer(X: np.ndarray, Wt: np.ndarray, GY: np.ndarray, s: ConvShape, fmt: str, seed: int = 0):
    """The layer step of the scheme section "무엇인가" describes: expand X
    with im2col first, then quantize every GEMM operand with plain
    16-element blocks along that GEMM's contraction, one copy per direction:
      X'  along K for Y = W·X' (16 x 1 down the expanded view's rows) and
          along P for G_W = G_Y·X'^T (1 x 16 along its batch columns);
      W   along K for Y (1 x 16 along its rows), along Cout for G_X'
          (16 x 1 down its columns);
      G_Y along P for G_W (1 x 16), along Cout for G_X' (16 x 1);
    RNE for X' and W, stochastic rounding for G_Y (the same element
    numbering and seed for both of its copies).  The GEMMs are 1 x 1
    convolutions over the Kh·Kw·Cin expanded channels, and G_X = col2im(G_X').
    Returns the six copies and the outputs (values, |product| sums), in fp64
    with the tensor scales applied."""
    K = s.Kh * s.Kw * s.Cin
    xv = expanded_view(X.astype(np.float32), s)
    wv = Wt.reshape(s.Cout, K).astype(np.float32)
    gv = GY.reshape(s.Ho * s.Wo * s.Cout, s.N).astype(np.float32)
    q = {"x_fwd": quantize_1d(xv, fmt, RNE, axis=0), "x_wgrad": quantize_1d(xv, fmt, RNE, axis=1),
         "w_fwd": quantize_1d(wv, fmt, RNE, axis=1), "w_dgrad": quantize_1d(wv, fmt, RNE, axis=0),
         "g_wgrad": quantize_1d(gv, fmt, SR, seed, axis=1), "g_dgrad": quantize_1d(gv, fmt, SR, seed, axis=0)}
    s1 = ConvShape(s.N, K, s.Cout, s.Ho, s.Wo, 1, 1, 1, 0)
    val = {k: code_values_1d(v) for k, v in q.items()}
    T = {k: np.float64(v.T) for k, v in q.items()}
    xf = val["x_fwd"].reshape(s.Ho, s.Wo, K, s.N)
    xw = val["x_wgrad"].reshape(s.Ho, s.Wo, K, s.N)
    wf = val["w_fwd"].reshape(s.Cout, 1, 1, K)
    wd = val["w_dgrad"].reshape(s.Cout, 1, 1, K)
    gw_ = val["g_wgrad"].reshape(s.Ho, s.Wo, s.Cout, s.N)
    gd = val["g_dgrad"].reshape(s.Ho, s.Wo, s.Cout, s.N)
    Y, SY = conv_fwd(wf, xf, s1)
    GW, SW = conv_wgrad(gw_, xw, s1)
    GXe, SXe = conv_dgrad(wd, gd, s1)                      # [Ho][Wo][K][N], the expanded gradient
    unexp = lambda t: col2im(t.reshape(s.Ho * s.Wo, K, s.N).transpose(1, 0, 2).reshape(K, -1), s)
    tf, tw, td = T["w_fwd"] * T["x_fwd"], T["g_wgrad"] * T["x_wgrad"], T["w_dgrad"] * T["g_dgrad"]
    out = {"y": (Y * tf, SY * tf), "gw": (GW.reshape(s.Cout, s.Kh, s.Kw, s.Cin) * tw,
                                           SW.reshape(s.Cout, s.Kh, s.Kw, s.Cin) * tw),
           "gx": (unexp(GXe) * td, unexp(SXe) * td)}
    return q, out


def bits_per_element(fmt: str) -> float:
    """Stored bits per element: the element code plus one E4M3 byte per 16."""
    return element_bits(fmt) + 8.0 / 16.0


# ---------------------------------------------------------------------------
# Depthwise layers in BF16 (reading R22).  Not part of quantize-once: the
# pages keep these layers in BF16 (section "전제와 한계"), so their operands
# are rounded to bfloat16 and nothing else.

def to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> the nearest bfloat16 value (ties to even), returned as fp32.
    bfloat16 is the top 16 bits of an fp32 encoding; rounding adds half of
    the dropped field (0x7FFF, plus the kept field's last bit for ties to
    even) before truncating.  Finite inputs only."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32)


def _dw_pad(X: np.ndarray, s: ConvShape) -> np.ndarray:
    Xp = np.zeros((s.H + 2 * s.pad, s.W + 2 * s.pad) + X.shape[2:], dtype=np.float64)
    Xp[s.pad:s.pad + s.H, s.pad:s.pad + s.W] = X
    return Xp


def _dw_window(Xp: np.ndarray, s: ConvShape, kh: int, kw: int) -> np.ndarray:
    """The input pixels tap (kh, kw) meets: [Ho][Wo][C][N]."""
    return Xp[kh:kh + s.stride * (s.Ho - 1) + 1:s.stride, kw:kw + s.stride * (s.Wo - 1) + 1:s.stride]


def depthwise_fwd(Wd: np.ndarray, X: np.ndarray, s: ConvShape):
    """Y[ho,wo,c,n] = sum_{kh,kw} W[c,kh,kw]·X[ho·s+kh-p, wo·s+kw-p, c, n]
    (zero padding), fp64.  Wd [C][Kh][Kw], X [H][W][C][N] (s.Cin = s.Cout
    = C).  Returns (Y [Ho][Wo][C][N], S = sum |W·X|)."""
    Xp = _dw_pad(X, s)
    Y = np.zeros((s.Ho, s.Wo, s.Cin, s.N))
    S = np.zeros_like(Y)
    for kh in range(s.Kh):
        for kw in range(s.Kw):
            w = Wd[:, kh, kw].astype(np.float64)[None, None, :, None]
            x = _dw_window(Xp, s, kh, kw)
            Y += w * x
            S += np.abs(w) * np.abs(x)
    return Y, S


def depthwise_wgrad(G: np.ndarray, X: np.ndarray, s: ConvShape):
    """G_W[c,kh,kw] = sum_{ho,wo,n} G_Y[ho,wo,c,n]·X[ho·s+kh-p, wo·s+kw-p, c, n],
    fp64.  Returns (G_W [C][Kh][Kw], S)."""
    Xp = _dw_pad(X, s)
    G = G.astype(np.float64)
    GW = np.zeros((s.Cin, s.Kh, s.Kw))
    S = np.zeros_like(GW)
    for kh in range(s.Kh):
        for kw in range(s.Kw):
            x = _dw_window(Xp, s, kh, kw)
            GW[:, kh, kw] = (G * x).sum(axis=(0, 1, 3))
            S[:, kh, kw] = (np.abs(G) * np.abs(x)).sum(axis=(0, 1, 3))
    return GW, S


def depthwise_dgrad(Wd: np.ndarray, G: np.ndarray, s: ConvShape):
    """G_X, the adjoint of depthwise_fwd in X: every G_Y[ho,wo,c,n] adds
    W[c,kh,kw]·G_Y to the input pixel tap (kh, kw) read; padding positions
    are dropped.  Returns (G_X [H][W][C][N], S)."""
    Gp = np.zeros((s.H + 2 * s.pad, s.W + 2 * s.pad, s.Cin, s.N))
    Sp = np.zeros_like(Gp)
    G = G.astype(np.float64)
    for kh in range(s.Kh):
        for kw in range(s.Kw):
            w = Wd[:, kh, kw].astype(np.float64)[None, None, :, None]
            _dw_window(Gp, s, kh, kw)[...] += w * G
            _dw_window(Sp, s, kh, kw)[...] += np.abs(w) * np.abs(G)
    return (Gp[s.pad:s.pad + s.H, s.pad:s.pad + s.W].copy(),
            Sp[s.pad:s.pad + s.H, s.pad:s.pad + s.W].copy())


def depthwise_layer_outputs(X: np.ndarray, Wd: np.ndarray, G: np.ndarray, s: ConvShape):
    """The three passes of a BF16 depthwise layer from fp32 operands: each
    operand rounded to bfloat16 first.  Returns {"y": (Y, S), "gw": ...,
    "gx": ...}."""
    Xb, Wb, Gb = to_bf16(X), to_bf16(Wd), to_bf16(G)
    return {"y": depthwise_fwd(Wb, Xb, s), "gw": depthwise_wgrad(Gb, Xb, s),
            "gx": depthwise_dgrad(Wb, Gb, s)}
