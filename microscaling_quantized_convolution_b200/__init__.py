"""Python binding of libmqv.so, the C ABI declared in include/mqv.h.

Argument marshalling only: every step of the quantize-once convolution path
runs in the library's CUDA kernels.  PyTorch supplies device memory and the
current stream.  There is no CPU fallback: if the library or a CUDA device is
missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmqv.so")

NVFP4, NVFP6 = 0, 1
RNE, SR = 0, 1
OP_FWD, OP_WGRAD, OP_DGRAD, OP_FWD_BLOCKSCALED = 1, 2, 3, 4
FORMATS = {"nvfp4": NVFP4, "nvfp6": NVFP6, NVFP4: NVFP4, NVFP6: NVFP6}


def _fmt(f) -> int:
    """Format code; unknown integers pass through for the library to reject."""
    return FORMATS[f] if f in FORMATS else int(f)

MQV_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA", 5: "TIMEOUT"}


class MqvError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"mqv {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class ConvDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("Cin", ctypes.c_int64), ("Cout", ctypes.c_int64),
                ("H", ctypes.c_int64), ("W", ctypes.c_int64), ("Kh", ctypes.c_int64),
                ("Kw", ctypes.c_int64), ("stride", ctypes.c_int64), ("pad", ctypes.c_int64),
                ("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class QTensorC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tscale", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("fmt", ctypes.c_int32), ("blocks", ctypes.c_int32)]


class QuantJobC(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("fmt", ctypes.c_int32), ("rounding", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("out", QTensorC)]


class DwDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("C", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64),
                ("Kh", ctypes.c_int64), ("Kw", ctypes.c_int64), ("stride", ctypes.c_int64),
                ("pad", ctypes.c_int64), ("reserved", ctypes.c_int32), ("reserved2", ctypes.c_int32)]


_lib = None

_SIGS = {
    "mqv_version": (ctypes.c_int32, []),
    "mqv_last_error": (ctypes.c_char_p, []),
    "mqv_qtensor_bytes": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)]),
    "mqv_quantize_workspace_size": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64,
                                                   ctypes.POINTER(ctypes.c_size_t)]),
    "mqv_quantize_cbf": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_uint64, ctypes.POINTER(QTensorC),
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_amax": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_quantize_with_amax": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_int32, ctypes.c_int32, ctypes.c_uint64,
                                              ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.POINTER(QTensorC), ctypes.c_void_p]),
    "mqv_dequantize": (ctypes.c_int, [ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p]),
    "mqv_conv_workspace_size": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.c_int32,
                                               ctypes.POINTER(ctypes.c_size_t)]),
    "mqv_conv_fwd": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                    ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_fwd_blockscaled": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                                ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_fwd_quantized": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                              ctypes.POINTER(QTensorC), ctypes.c_int32, ctypes.c_void_p,
                                              ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_dgrad_quantized": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                                ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_uint64,
                                                ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_wgrad": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                      ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_dgrad": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                      ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_device_errors": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_void_p]),
    "mqv_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int64, ctypes.c_void_p]),
    "mqv_quantize_many_workspace_size": (ctypes.c_int, [ctypes.POINTER(QuantJobC), ctypes.c_int32,
                                                        ctypes.POINTER(ctypes.c_size_t)]),
    "mqv_quantize_many": (ctypes.c_int, [ctypes.POINTER(QuantJobC), ctypes.c_int32, ctypes.c_void_p,
                                         ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_wgrad_noalloc": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                              ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p]),
    "mqv_im2col": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "mqv_col2im": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "mqv_conv_fwd_fused": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                          ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_int32,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_conv_dgrad_fused": (ctypes.c_int, [ctypes.POINTER(ConvDesc), ctypes.POINTER(QTensorC),
                                            ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "mqv_replay_bytes": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.POINTER(ctypes.c_size_t)]),
    "mqv_replay_pack": (ctypes.c_int, [ctypes.POINTER(QTensorC), ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p]),
    "mqv_replay_unpack": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_void_p, ctypes.c_void_p]),
    "mqv_replay_dequantize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "mqv_dw_fwd": (ctypes.c_int, [ctypes.POINTER(DwDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p]),
    "mqv_dw_dgrad": (ctypes.c_int, [ctypes.POINTER(DwDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p]),
    "mqv_dw_wgrad_workspace_size": (ctypes.c_int, [ctypes.POINTER(DwDesc), ctypes.POINTER(ctypes.c_size_t)]),
    "mqv_dw_wgrad": (ctypes.c_int, [ctypes.POINTER(DwDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
}


def lib() -> ctypes.CDLL:
    """Load libmqv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m microscaling_quantized_convolution_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _check(status: int):
    if status != MQV_OK:
        raise MqvError(status, lib().mqv_last_error().decode())


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _require_cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


# ---------------------------------------------------------------- tensors

def qtensor_bytes(rows: int, cols: int, fmt) -> tuple[int, int]:
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().mqv_qtensor_bytes(rows, cols, _fmt(fmt), ctypes.byref(cb), ctypes.byref(sb)))
    return cb.value, sb.value


BLOCKS_4X4, BLOCKS_1X16, BLOCKS_16X1 = 0, 1, 2


@dataclass
class QTensor:
    """A quantized rows x cols view: packed codes, E4M3 scale plane, fp32 T.
    blocks: the scale blocks (mqv_blocks): 4 x 4 squares, or the 16-element
    lines of 1 x 16 along a row / 16 x 1 down a column."""
    codes: torch.Tensor
    scales: torch.Tensor
    tscale: torch.Tensor
    rows: int
    cols: int
    fmt: int
    blocks: int = BLOCKS_4X4

    @classmethod
    def empty(cls, rows: int, cols: int, fmt, device="cuda", blocks: int = BLOCKS_4X4) -> "QTensor":
        fmt = _fmt(fmt)
        cb, sb = qtensor_bytes(rows, cols, fmt)
        return cls(torch.empty(cb, dtype=torch.uint8, device=device),
                   torch.empty(sb, dtype=torch.uint8, device=device),
                   torch.empty(1, dtype=torch.float32, device=device), rows, cols, fmt, blocks)

    def c(self) -> QTensorC:
        return QTensorC(self.codes.data_ptr(), self.scales.data_ptr(), self.tscale.data_ptr(),
                        self.rows, self.cols, self.fmt, self.blocks)


def quantize_workspace_bytes(rows: int, cols: int) -> int:
    b = ctypes.c_size_t()
    _check(lib().mqv_quantize_workspace_size(rows, cols, ctypes.byref(b)))
    return b.value


def quantize(src: torch.Tensor, rows: int, cols: int, fmt, rounding: int = RNE, seed: int = 0,
             out: QTensor | None = None, ws: torch.Tensor | None = None, stream=None) -> QTensor:
    """Quantize the rows x cols fp32 view of `src` (see mqv_quantize_cbf)."""
    _require_cuda(src, "src", torch.float32)
    if src.numel() != rows * cols:
        raise ValueError("src size does not match rows x cols")
    out = out or QTensor.empty(rows, cols, fmt, src.device)
    if ws is None:
        ws = torch.empty(quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device=src.device)
    qc = out.c()
    _check(lib().mqv_quantize_cbf(src.data_ptr(), rows, cols, _fmt(fmt), rounding, seed,
                                  ctypes.byref(qc), ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


def quantize_many(jobs, ws: torch.Tensor | None = None, stream=None) -> list[QTensor]:
    """Quantize several tensors in two launches (see mqv_quantize_many).
    jobs: (src, rows, cols, fmt, rounding, seed[, out QTensor]) tuples; the
    block shape is the out QTensor's (4 x 4 when no out is given)."""
    outs, cjobs = [], []
    for j in jobs:
        src, rows, cols, fmt, rnd, seed = j[:6]
        _require_cuda(src, "src", torch.float32)
        out = j[6] if len(j) > 6 and j[6] is not None else QTensor.empty(rows, cols, fmt, src.device)
        outs.append(out)
        cjobs.append(QuantJobC(src.data_ptr(), rows, cols, _fmt(fmt), rnd, seed, out.c()))
    arr = (QuantJobC * len(cjobs))(*cjobs)
    if ws is None:
        b = ctypes.c_size_t()
        _check(lib().mqv_quantize_many_workspace_size(arr, len(cjobs), ctypes.byref(b)))
        ws = torch.empty(b.value, dtype=torch.uint8, device=jobs[0][0].device)
    _check(lib().mqv_quantize_many(arr, len(cjobs), ws.data_ptr(), ws.numel(), _stream(stream)))
    return outs


def quantize_many_workspace_bytes(jobs) -> int:
    cjobs = [QuantJobC(0, j[1], j[2], _fmt(j[3]), j[4], j[5], QTensorC(16, 16, 16, j[1], j[2], _fmt(j[3]), 0))
             for j in jobs]
    arr = (QuantJobC * len(cjobs))(*cjobs)
    b = ctypes.c_size_t()
    _check(lib().mqv_quantize_many_workspace_size(arr, len(cjobs), ctypes.byref(b)))
    return b.value


def amax(src: torch.Tensor, rows: int, cols: int, out: torch.Tensor | None = None,
         ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Device fp32 max|src| of the view (see mqv_amax)."""
    _require_cuda(src, "src", torch.float32)
    out = out if out is not None else torch.empty(1, dtype=torch.float32, device=src.device)
    if ws is None:
        ws = torch.empty(quantize_workspace_bytes(rows, cols), dtype=torch.uint8, device=src.device)
    _check(lib().mqv_amax(src.data_ptr(), rows, cols, out.data_ptr(), ws.data_ptr(), ws.numel(),
                          _stream(stream)))
    return out


def quantize_with_amax(src: torch.Tensor, rows: int, cols: int, fmt, rounding: int, seed: int,
                       amax_dev: torch.Tensor, out: QTensor | None = None, sr_col0: int = 0,
                       sr_cols: int = 0, stream=None) -> QTensor:
    """Quantize with a given device amax; (sr_col0, sr_cols) place a batch
    shard inside the full view for stochastic rounding."""
    _require_cuda(src, "src", torch.float32)
    _require_cuda(amax_dev, "amax", torch.float32)
    out = out or QTensor.empty(rows, cols, fmt, src.device)
    qc = out.c()
    _check(lib().mqv_quantize_with_amax(src.data_ptr(), rows, cols, _fmt(fmt), rounding, seed,
                                        amax_dev.data_ptr(), sr_col0, sr_cols, ctypes.byref(qc),
                                        _stream(stream)))
    return out


def dequantize(q: QTensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = out if out is not None else torch.empty(q.rows * q.cols, dtype=torch.float32,
                                                  device=q.codes.device)
    qc = q.c()
    _check(lib().mqv_dequantize(ctypes.byref(qc), out.data_ptr(), _stream(stream)))
    return out


# ------------------------------------------------------- latent-replay form

def replay_bytes(rows: int, cols: int, fmt) -> int:
    """Bytes of the magnitude-only replay form of a rows x cols view."""
    b = ctypes.c_size_t()
    _check(lib().mqv_replay_bytes(rows, cols, _fmt(fmt), ctypes.byref(b)))
    return b.value


def replay_pack(q: QTensor, out: torch.Tensor | None = None, negatives: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """Magnitude-only form of a post-ReLU tensor's codes (see
    mqv_replay_pack); `negatives` (int32 device scalar, zeroed by the
    caller) receives the count of negative codes, which are stored as 0."""
    out = out if out is not None else torch.empty(replay_bytes(q.rows, q.cols, q.fmt), dtype=torch.uint8,
                                                  device=q.codes.device)
    _require_cuda(out, "out", torch.uint8)
    if negatives is not None:
        _require_cuda(negatives, "negatives", torch.int32)
    qc = q.c()
    _check(lib().mqv_replay_pack(ctypes.byref(qc), out.data_ptr(), _ptr(negatives), _stream(stream)))
    return out


def replay_unpack(packed: torch.Tensor, rows: int, cols: int, fmt, codes: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """Standard-packing codes (sign bit 0) from the replay form."""
    _require_cuda(packed, "packed", torch.uint8)
    codes = codes if codes is not None else torch.empty(qtensor_bytes(rows, cols, fmt)[0], dtype=torch.uint8,
                                                        device=packed.device)
    _require_cuda(codes, "codes", torch.uint8)
    _check(lib().mqv_replay_unpack(packed.data_ptr(), rows, cols, _fmt(fmt), codes.data_ptr(), _stream(stream)))
    return codes


def replay_dequantize(packed: torch.Tensor, scales: torch.Tensor, tscale: torch.Tensor, rows: int, cols: int,
                      fmt, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 values code·B·T read straight from the replay form."""
    _require_cuda(packed, "packed", torch.uint8)
    _require_cuda(scales, "scales", torch.uint8)
    _require_cuda(tscale, "tscale", torch.float32)
    out = out if out is not None else torch.empty(rows * cols, dtype=torch.float32, device=packed.device)
    _require_cuda(out, "out", torch.float32)
    _check(lib().mqv_replay_dequantize(packed.data_ptr(), scales.data_ptr(), tscale.data_ptr(), rows, cols,
                                       _fmt(fmt), out.data_ptr(), _stream(stream)))
    return out


# ------------------------------------------------------------------ conv

def conv_desc(N, Cin, Cout, H, W, Kh, Kw, stride=1, pad=0, fmt=NVFP4) -> ConvDesc:
    return ConvDesc(N, Cin, Cout, H, W, Kh, Kw, stride, pad, _fmt(fmt), 0)


def out_hw(d: ConvDesc) -> tuple[int, int]:
    return ((d.H + 2 * d.pad - d.Kh) // d.stride + 1, (d.W + 2 * d.pad - d.Kw) // d.stride + 1)


def conv_workspace_bytes(d: ConvDesc, op: int) -> int:
    b = ctypes.c_size_t()
    _check(lib().mqv_conv_workspace_size(ctypes.byref(d), op, ctypes.byref(b)))
    return b.value


def _ws(d, op, ws, device):
    need = conv_workspace_bytes(d, op)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws


def im2col(d: ConvDesc, x: torch.Tensor, xc: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Explicit im2col of fp32 X [H][W][Cin][N] -> [Ho][Wo][Kh·Kw·Cin][N]
    (see mqv_im2col); for the quantize-after-im2col baseline."""
    _require_cuda(x, "x", torch.float32)
    Ho, Wo = out_hw(d)
    xc = xc if xc is not None else torch.empty((Ho, Wo, d.Kh * d.Kw * d.Cin, d.N), dtype=torch.float32,
                                               device=x.device)
    _require_cuda(xc, "xc", torch.float32)
    _check(lib().mqv_im2col(ctypes.byref(d), x.data_ptr(), xc.data_ptr(), _stream(stream)))
    return xc


def col2im(d: ConvDesc, gc: torch.Tensor, gx: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The adjoint of im2col: [Ho][Wo][Kh·Kw·Cin][N] -> G_X [H][W][Cin][N]
    (see mqv_col2im)."""
    _require_cuda(gc, "gc", torch.float32)
    gx = gx if gx is not None else torch.empty((d.H, d.W, d.Cin, d.N), dtype=torch.float32, device=gc.device)
    _require_cuda(gx, "gx", torch.float32)
    _check(lib().mqv_col2im(ctypes.byref(d), gc.data_ptr(), gx.data_ptr(), _stream(stream)))
    return gx


def conv_fwd(d: ConvDesc, w: QTensor, x: QTensor, y: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y [Ho][Wo][Cout][N] fp32 = T_w·T_x·(W·X'), implicit im2col."""
    Ho, Wo = out_hw(d)
    y = y if y is not None else torch.empty((Ho, Wo, d.Cout, d.N), dtype=torch.float32, device=x.codes.device)
    ws = _ws(d, OP_FWD, ws, x.codes.device)
    wc, xc = w.c(), x.c()
    _check(lib().mqv_conv_fwd(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(xc), y.data_ptr(),
                              _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return y


def conv_fwd_blockscaled(d: ConvDesc, w: QTensor, x: QTensor, y: torch.Tensor | None = None,
                         ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y as conv_fwd, on the native block-scaled MMA with each 4-element
    block row padded to a 16-element scale group (see mqv_conv_fwd_blockscaled)."""
    Ho, Wo = out_hw(d)
    y = y if y is not None else torch.empty((Ho, Wo, d.Cout, d.N), dtype=torch.float32, device=x.codes.device)
    ws = _ws(d, OP_FWD_BLOCKSCALED, ws, x.codes.device)
    wc, xc = w.c(), x.c()
    _check(lib().mqv_conv_fwd_blockscaled(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(xc), y.data_ptr(),
                                          _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return y


def conv_fwd_quantized(d: ConvDesc, w: QTensor, x: QTensor, t_amax: torch.Tensor, relu: int = 1,
                       y_q: QTensor | None = None, y_amax: torch.Tensor | None = None,
                       ws: torch.Tensor | None = None, stream=None) -> QTensor:
    """The next layer's X quantized straight from the forward epilogue, T from
    the device max |x| t_amax (see mqv_conv_fwd_quantized)."""
    Ho, Wo = out_hw(d)
    y_q = y_q or QTensor.empty(Ho * Wo * d.Cout, d.N, d.fmt, x.codes.device)
    ws = _ws(d, OP_FWD, ws, x.codes.device)
    wc, xc, yc = w.c(), x.c(), y_q.c()
    _check(lib().mqv_conv_fwd_quantized(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(xc), relu,
                                        t_amax.data_ptr(), ctypes.byref(yc), _ptr(y_amax), _ptr(ws),
                                        0 if ws is None else ws.numel(), _stream(stream)))
    return y_q


def conv_dgrad_quantized(d: ConvDesc, w: QTensor, gy: QTensor, t_amax: torch.Tensor, seed: int,
                         gx_q: QTensor | None = None, gx_amax: torch.Tensor | None = None,
                         ws: torch.Tensor | None = None, stream=None) -> QTensor:
    """G_X quantized (stochastic rounding) straight from the input-gradient
    epilogue, T from t_amax (see mqv_conv_dgrad_quantized)."""
    gx_q = gx_q or QTensor.empty(d.H * d.W * d.Cin, d.N, d.fmt, gy.codes.device)
    ws = _ws(d, OP_DGRAD, ws, gy.codes.device)
    wc, gc, xc = w.c(), gy.c(), gx_q.c()
    _check(lib().mqv_conv_dgrad_quantized(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(gc), t_amax.data_ptr(),
                                          seed, ctypes.byref(xc), _ptr(gx_amax), _ptr(ws),
                                          0 if ws is None else ws.numel(), _stream(stream)))
    return gx_q


def conv_wgrad(d: ConvDesc, gy: QTensor, x: QTensor, gw: torch.Tensor | None = None,
               ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """G_W [Cout][Kh][Kw][Cin] fp32 = T_g·T_x·(G_Y·X'^T)."""
    gw = gw if gw is not None else torch.empty((d.Cout, d.Kh, d.Kw, d.Cin), dtype=torch.float32,
                                               device=x.codes.device)
    ws = _ws(d, OP_WGRAD, ws, x.codes.device)
    gc, xc = gy.c(), x.c()
    _check(lib().mqv_conv_wgrad(ctypes.byref(d), ctypes.byref(gc), ctypes.byref(xc), gw.data_ptr(),
                                _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return gw


def conv_dgrad(d: ConvDesc, w: QTensor, gy: QTensor, gx: torch.Tensor | None = None,
               ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """G_X [H][W][Cin][N] fp32 = T_w·T_g·col2im(W^T·G_Y), implicit."""
    gx = gx if gx is not None else torch.empty((d.H, d.W, d.Cin, d.N), dtype=torch.float32,
                                               device=gy.codes.device)
    ws = _ws(d, OP_DGRAD, ws, gy.codes.device)
    wc, gc = w.c(), gy.c()
    _check(lib().mqv_conv_dgrad(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(gc), gx.data_ptr(),
                                _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return gx


def conv_fwd_fused(d: ConvDesc, w: QTensor, x: QTensor, relu: bool = False, y: torch.Tensor | None = None,
                   y_amax: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                   stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """conv_fwd with optional ReLU and max|y| fused into the epilogue (see
    mqv_conv_fwd_fused); returns (y, y_amax), y_amax a device fp32 scalar."""
    Ho, Wo = out_hw(d)
    dev = x.codes.device
    y = y if y is not None else torch.empty((Ho, Wo, d.Cout, d.N), dtype=torch.float32, device=dev)
    y_amax = y_amax if y_amax is not None else torch.empty(1, dtype=torch.float32, device=dev)
    _require_cuda(y_amax, "y_amax", torch.float32)
    ws = _ws(d, OP_FWD, ws, dev)
    wc, xc = w.c(), x.c()
    _check(lib().mqv_conv_fwd_fused(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(xc), y.data_ptr(),
                                    1 if relu else 0, y_amax.data_ptr(), _ptr(ws),
                                    0 if ws is None else ws.numel(), _stream(stream)))
    return y, y_amax


def conv_dgrad_fused(d: ConvDesc, w: QTensor, gy: QTensor, gx: torch.Tensor | None = None,
                     gx_amax: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                     stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """conv_dgrad with max|gx| fused into the epilogue; returns (gx, gx_amax)."""
    dev = gy.codes.device
    gx = gx if gx is not None else torch.empty((d.H, d.W, d.Cin, d.N), dtype=torch.float32, device=dev)
    gx_amax = gx_amax if gx_amax is not None else torch.empty(1, dtype=torch.float32, device=dev)
    _require_cuda(gx_amax, "gx_amax", torch.float32)
    ws = _ws(d, OP_DGRAD, ws, dev)
    wc, gc = w.c(), gy.c()
    _check(lib().mqv_conv_dgrad_fused(ctypes.byref(d), ctypes.byref(wc), ctypes.byref(gc), gx.data_ptr(),
                                      gx_amax.data_ptr(), _ptr(ws), 0 if ws is None else ws.numel(),
                                      _stream(stream)))
    return gx, gx_amax


def conv_wgrad_noalloc(d: ConvDesc, gy: QTensor, x: QTensor, gw: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """As conv_wgrad, but the library's built-in scratch replaces the
    workspace (for callers that cannot allocate; see mqv_conv_wgrad_noalloc)."""
    gw = gw if gw is not None else torch.empty((d.Cout, d.Kh, d.Kw, d.Cin), dtype=torch.float32,
                                               device=x.codes.device)
    gc, xc = gy.c(), x.c()
    _check(lib().mqv_conv_wgrad_noalloc(ctypes.byref(d), ctypes.byref(gc), ctypes.byref(xc),
                                        gw.data_ptr(), _stream(stream)))
    return gw


def device_errors(stream=None) -> int:
    f = ctypes.c_uint32()
    st = lib().mqv_device_errors(ctypes.byref(f), _stream(stream))
    if st not in (MQV_OK, 5):
        _check(st)
    return f.value


def selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Test hook: a one-CTA kernel whose bounded wait runs out after
    limit_cycles SM cycles and sets bit 8 of the device error word (see
    mqv_selftest_wait_timeout); read it with device_errors()."""
    _check(lib().mqv_selftest_wait_timeout(limit_cycles, _stream(stream)))


# ------------------------------------------- depthwise layers in BF16

def dw_desc(N, C, H, W, Kh, Kw, stride=1, pad=0) -> DwDesc:
    """Descriptor of a BF16 depthwise layer (one filter per channel)."""
    return DwDesc(N, C, H, W, Kh, Kw, stride, pad, 0, 0)


def dw_wgrad_workspace_bytes(d: DwDesc) -> int:
    """Workspace bytes of dw_wgrad; raises MqvError for an invalid descriptor
    (the library's own check, which every dw_* call runs first)."""
    b = ctypes.c_size_t()
    _check(lib().mqv_dw_wgrad_workspace_size(ctypes.byref(d), ctypes.byref(b)))
    return b.value


def dw_out_hw(d: DwDesc) -> tuple[int, int]:
    """Output pixel grid (Ho, Wo) of a validated descriptor."""
    dw_wgrad_workspace_bytes(d)
    return (d.H + 2 * d.pad - d.Kh) // d.stride + 1, (d.W + 2 * d.pad - d.Kw) // d.stride + 1


def _dw_numel(t: torch.Tensor, name: str, n: int):
    # the C ABI takes no tensor sizes: a short tensor would be read or
    # written out of bounds on the device, so the sizes are checked here
    if t.numel() != n:
        raise ValueError(f"{name}: {t.numel()} elements, the descriptor needs {n}")


def dw_fwd(d: DwDesc, w: torch.Tensor, x: torch.Tensor, y: torch.Tensor | None = None, stream=None):
    """Y [Ho][Wo][C][N] fp32 from bfloat16 w [C][Kh][Kw] and x [H][W][C][N]."""
    Ho, Wo = dw_out_hw(d)
    _require_cuda(w, "w", torch.bfloat16)
    _require_cuda(x, "x", torch.bfloat16)
    y = y if y is not None else torch.empty((Ho, Wo, d.C, d.N), dtype=torch.float32, device=x.device)
    _require_cuda(y, "y", torch.float32)
    _dw_numel(w, "w", d.C * d.Kh * d.Kw)
    _dw_numel(x, "x", d.H * d.W * d.C * d.N)
    _dw_numel(y, "y", Ho * Wo * d.C * d.N)
    _check(lib().mqv_dw_fwd(ctypes.byref(d), w.data_ptr(), x.data_ptr(), y.data_ptr(), _stream(stream)))
    return y


def dw_dgrad(d: DwDesc, w: torch.Tensor, gy: torch.Tensor, gx: torch.Tensor | None = None, stream=None):
    """G_X [H][W][C][N] fp32 from bfloat16 w and gy [Ho][Wo][C][N]."""
    Ho, Wo = dw_out_hw(d)
    _require_cuda(w, "w", torch.bfloat16)
    _require_cuda(gy, "gy", torch.bfloat16)
    gx = gx if gx is not None else torch.empty((d.H, d.W, d.C, d.N), dtype=torch.float32, device=gy.device)
    _require_cuda(gx, "gx", torch.float32)
    _dw_numel(w, "w", d.C * d.Kh * d.Kw)
    _dw_numel(gy, "gy", Ho * Wo * d.C * d.N)
    _dw_numel(gx, "gx", d.H * d.W * d.C * d.N)
    _check(lib().mqv_dw_dgrad(ctypes.byref(d), w.data_ptr(), gy.data_ptr(), gx.data_ptr(), _stream(stream)))
    return gx


def dw_wgrad(d: DwDesc, gy: torch.Tensor, x: torch.Tensor, gw: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream=None):
    """G_W [C][Kh][Kw] fp32 from bfloat16 gy and x."""
    Ho, Wo = dw_out_hw(d)
    _require_cuda(gy, "gy", torch.bfloat16)
    _require_cuda(x, "x", torch.bfloat16)
    gw = gw if gw is not None else torch.empty((d.C, d.Kh, d.Kw), dtype=torch.float32, device=x.device)
    _require_cuda(gw, "gw", torch.float32)
    _dw_numel(gy, "gy", Ho * Wo * d.C * d.N)
    _dw_numel(x, "x", d.H * d.W * d.C * d.N)
    _dw_numel(gw, "gw", d.C * d.Kh * d.Kw)
    if ws is None:
        ws = torch.empty(dw_wgrad_workspace_bytes(d), dtype=torch.uint8, device=x.device)
    _check(lib().mqv_dw_wgrad(ctypes.byref(d), gy.data_ptr(), x.data_ptr(), gw.data_ptr(), ws.data_ptr(),
                              ws.numel(), _stream(stream)))
    return gw
