"""The baseline MicroQonv removes, run on the same kernels for measurement.

Section "무엇인가" of the MicroQonv summary (onedev.kr/papers/182) describes
the usual low-precision training flow: expand X with im2col first, then
quantize every GEMM operand with plain 16-element blocks along that GEMM's
contraction, once per direction (W for the forward and the input gradient,
G_Y for the two gradients, the expanded X' for the forward and the weight
gradient).  This module composes that flow from the library's entry points:
`mqv_im2col`; one `mqv_quantize_many` call writing the six copies

    X'  16 x 1 down its (pixel, K) rows for Y = W·X' (contraction K),
        1 x 16 along its batch columns for G_W = G_Y·X'^T (contraction P);
    W   1 x 16 along its K rows for Y, 16 x 1 down its Cout column for G_X';
    G_Y 1 x 16 along its batch columns for G_W, 16 x 1 down its (pixel,
        Cout) rows for G_X' (stochastic rounding, one seed and element
        numbering for both copies);

1 x 1 convolutions over the Kh·Kw·Cin expanded channels as the three GEMMs;
and `mqv_col2im` for the input gradient.  One pixel's duplicates in X' land
in different blocks and take different codes, and each operand's two copies
differ: the numerics of the scheme, not only its memory traffic.

`blocks="square"` keeps a second variant under its own name: the same flow
with 4 x 4 blocks over (kh·kw·ci, n) of the expanded tensor, whose
duplicates all get equal codes (its six copies are three identical pairs);
it isolates the cost of the expansion from the change of numerics.
Every step runs on the GPU; nothing here computes on the host."""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (NVFP4, RNE, SR, BLOCKS_1X16, BLOCKS_16X1, BLOCKS_4X4, ConvDesc, QTensor, col2im, conv_desc,
               conv_dgrad, conv_fwd, conv_wgrad, conv_workspace_bytes, im2col, out_hw, quantize_many,
               quantize_many_workspace_bytes, OP_FWD, OP_WGRAD, OP_DGRAD)

# block shape of each copy: along the contraction of the GEMM it feeds
LINE_BLOCKS = {"x_fwd": BLOCKS_16X1, "x_wgrad": BLOCKS_1X16, "w_fwd": BLOCKS_1X16, "w_dgrad": BLOCKS_16X1,
               "g_wgrad": BLOCKS_1X16, "g_dgrad": BLOCKS_16X1}


@dataclass
class NaivePlan:
    """Buffers of the baseline step for one layer (allocated once)."""
    d: ConvDesc          # the layer
    d1: ConvDesc         # the 1 x 1 convolution over the expanded tensor
    xc: torch.Tensor     # expanded X, fp32 [Ho][Wo][Kh·Kw·Cin][N]
    gxc: torch.Tensor    # expanded input gradient, same shape
    q: dict              # quantized copies, one per GEMM direction
    ws: dict             # workspaces


def plan(d: ConvDesc, device="cuda", blocks: str = "line") -> NaivePlan:
    """blocks: "line" (the scheme's 16-element blocks) or "square"."""
    if blocks not in ("line", "square"):
        raise ValueError(f"blocks must be 'line' or 'square', got {blocks!r}")
    Ho, Wo = out_hw(d)
    K = d.Kh * d.Kw * d.Cin
    d1 = conv_desc(d.N, K, d.Cout, Ho, Wo, 1, 1, 1, 0, d.fmt)
    xc = torch.empty((Ho, Wo, K, d.N), dtype=torch.float32, device=device)
    gxc = torch.empty_like(xc)
    rows_x, rows_g = Ho * Wo * K, Ho * Wo * d.Cout
    shape = {"x_fwd": (rows_x, d.N), "x_wgrad": (rows_x, d.N), "w_fwd": (d.Cout, K), "w_dgrad": (d.Cout, K),
             "g_wgrad": (rows_g, d.N), "g_dgrad": (rows_g, d.N)}
    q = {k: QTensor.empty(r, c, d.fmt, device, LINE_BLOCKS[k] if blocks == "line" else BLOCKS_4X4)
         for k, (r, c) in shape.items()}
    jobs = [(None, rows_x, d.N, d.fmt, RNE, 0), (None, rows_x, d.N, d.fmt, RNE, 0),
            (None, d.Cout, K, d.fmt, RNE, 0), (None, d.Cout, K, d.fmt, RNE, 0),
            (None, rows_g, d.N, d.fmt, SR, 0), (None, rows_g, d.N, d.fmt, SR, 0)]
    ws = {"quant": torch.empty(quantize_many_workspace_bytes(jobs), dtype=torch.uint8, device=device),
          "fwd": torch.empty(max(16, conv_workspace_bytes(d1, OP_FWD)), dtype=torch.uint8, device=device),
          "wgrad": torch.empty(max(16, conv_workspace_bytes(d1, OP_WGRAD)), dtype=torch.uint8, device=device),
          "dgrad": torch.empty(max(16, conv_workspace_bytes(d1, OP_DGRAD)), dtype=torch.uint8, device=device)}
    return NaivePlan(d, d1, xc, gxc, q, ws)


def quantize_all(p: NaivePlan, X: torch.Tensor, W: torch.Tensor, G: torch.Tensor, seed: int):
    """im2col, then every operand once per GEMM direction (six quantized
    tensors in one two-launch call, each in its copy's block shape)."""
    d, d1 = p.d, p.d1
    im2col(d, X, p.xc)
    rows_x = d1.H * d1.W * d1.Cin
    rows_g = d1.H * d1.W * d1.Cout
    K = d1.Cin
    xv, wv, gv = p.xc.view(-1), W.view(-1), G.view(-1)
    quantize_many([(xv, rows_x, d.N, d.fmt, RNE, 0, p.q["x_fwd"]), (xv, rows_x, d.N, d.fmt, RNE, 0, p.q["x_wgrad"]),
                   (wv, d.Cout, K, d.fmt, RNE, 0, p.q["w_fwd"]), (wv, d.Cout, K, d.fmt, RNE, 0, p.q["w_dgrad"]),
                   (gv, rows_g, d.N, d.fmt, SR, seed, p.q["g_wgrad"]), (gv, rows_g, d.N, d.fmt, SR, seed, p.q["g_dgrad"])],
                  ws=p.ws["quant"])


def fwd(p: NaivePlan, y: torch.Tensor):
    conv_fwd(p.d1, p.q["w_fwd"], p.q["x_fwd"], y=y, ws=p.ws["fwd"])


def wgrad(p: NaivePlan, gw: torch.Tensor):
    # G_W over the expanded channels is [Cout][1][1][Kh·Kw·Cin] = [Cout][Kh][Kw][Cin]
    conv_wgrad(p.d1, p.q["g_wgrad"], p.q["x_wgrad"], gw=gw.view(p.d.Cout, 1, 1, -1), ws=p.ws["wgrad"])


def dgrad(p: NaivePlan, gx: torch.Tensor):
    conv_dgrad(p.d1, p.q["w_dgrad"], p.q["g_dgrad"], gx=p.gxc, ws=p.ws["dgrad"])
    col2im(p.d, p.gxc, gx)


def step(p: NaivePlan, X, W, G, seed, y, gw, gx):
    quantize_all(p, X, W, G, seed)
    fwd(p, y)
    wgrad(p, gw)
    dgrad(p, gx)


def layer_bytes(d: ConvDesc) -> dict:
    """Algorithmic HBM bytes of the baseline step, per phase: the quantizer
    reads its fp32 input twice (amax and quantize) and writes 0.5625 B
    (FP4) or 0.8125 B (FP6) per element; im2col reads X and writes X';
    each GEMM reads its two quantized operands once and writes fp32;
    col2im reads the expanded gradient and writes G_X."""
    Ho, Wo = out_hw(d)
    K = d.Kh * d.Kw * d.Cin
    qb = 0.5625 if d.fmt == NVFP4 or d.fmt == 0 else 0.8125
    ex = Ho * Wo * K * d.N            # expanded X elements
    eg = Ho * Wo * d.Cout * d.N
    ew = d.Cout * K
    ex0 = d.H * d.W * d.Cin * d.N
    quant = 2 * (ex * (8 + qb)) + 2 * (ew * (8 + qb)) + 2 * (eg * (8 + qb))
    return {"im2col": 4 * ex0 + 4 * ex, "quantize": quant,
            "fwd": ew * qb + ex * qb + 4 * eg, "wgrad": eg * qb + ex * qb + 4 * ew,
            "dgrad": ew * qb + eg * qb + 4 * ex, "col2im": 4 * ex + 4 * ex0}
