"""Data-parallel step of one quantize-once conv layer, sharded over the batch.

Every 4 x 4 block of X and G_Y is 4 channels x 4 batch items at one pixel,
so a shard of N/world batch items (a multiple of 4) holds whole blocks and
each rank quantizes and convolves its own shard.  Two exchanges make the
sharded step equal to the single-process step on the whole batch:

  * a MAX all-reduce of max|X| and max|G_Y| before quantizing, so every rank
    uses the global tensor scales;
  * a SUM all-reduce of G_W after the weight-gradient pass.

Stochastic rounding of G_Y numbers elements by their column in the whole
batch (sr_col0 = rank·N_local, sr_cols = N), so the shards draw exactly the
words the single-process step draws.  W is replicated and quantized locally.

The kernels (`ops`) and the collectives (`comm`) are passed in, so the same
exchange logic runs over NCCL with the CUDA kernels and over gloo in the
CPU tests.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Any, Callable


@dataclass
class Comm:
    """Collectives on one-element (amax) and G_W-sized tensors, in place."""
    all_reduce_max: Callable[[Any], None]
    all_reduce_sum: Callable[[Any], None]


def torch_comm():
    """torch.distributed collectives (NCCL on GPUs, gloo on CPUs)."""
    import torch.distributed as dist
    return Comm(lambda t: dist.all_reduce(t, op=dist.ReduceOp.MAX),
                lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM))


def shard_columns(n_global: int, rank: int, world: int) -> tuple[int, int]:
    """(first column, column count) of this rank's batch shard."""
    if n_global % world or (n_global // world) % 4:
        raise ValueError(f"batch {n_global} does not split into {world} shards of a multiple of 4")
    n = n_global // world
    return rank * n, n


def data_parallel_step(ops, comm: Comm, X, W, G, dims: dict, fmt, n_global: int, rank: int,
                       world: int, seed: int, mark=None, quantized=None):
    """One layer: quantize X, W (RNE), G_Y (SR), then fwd, wgrad, dgrad.

    X [H][W][Cin][n_local], G [Ho][Wo][Cout][n_local]: this rank's shard.
    dims: N (= n_local), Cin, Cout, H, W, Kh, Kw, stride, pad.
    `ops` provides amax(t, rows, cols) -> 1-element tensor,
    quantize_with_amax(t, rows, cols, fmt, rounding, seed, amax, sr_col0, sr_cols),
    quantize(t, rows, cols, fmt, rounding, seed), fwd(dims, qw, qx), wgrad(dims, qg, qx),
    dgrad(dims, qw, qg), and the rounding constants RNE and SR.
    `mark(name)`, if given, is called at the phase boundaries "start",
    "quantized", "fwd", "wgrad" (after the G_W sum) and "dgrad" (the
    benchmark records timing events there); `quantized`, if a dict, receives
    the quantized operands (qx, qw, qg).
    Returns (Y_local, G_W (summed over ranks), G_X_local)."""
    mark = mark or (lambda name: None)
    col0, n_local = shard_columns(n_global, rank, world)
    assert dims["N"] == n_local
    Ho = (dims["H"] + 2 * dims["pad"] - dims["Kh"]) // dims["stride"] + 1
    Wo = (dims["W"] + 2 * dims["pad"] - dims["Kw"]) // dims["stride"] + 1
    xr = dims["H"] * dims["W"] * dims["Cin"]
    gr = Ho * Wo * dims["Cout"]
    wr, wc = dims["Cout"], dims["Kh"] * dims["Kw"] * dims["Cin"]
    mark("start")
    ax = ops.amax(X, xr, n_local)
    ag = ops.amax(G, gr, n_local)
    comm.all_reduce_max(ax)
    comm.all_reduce_max(ag)
    qx = ops.quantize_with_amax(X, xr, n_local, fmt, ops.RNE, 0, ax, col0, n_global)
    qg = ops.quantize_with_amax(G, gr, n_local, fmt, ops.SR, seed, ag, col0, n_global)
    qw = ops.quantize(W, wr, wc, fmt, ops.RNE, 0)
    if quantized is not None:
        quantized.update(qx=qx, qw=qw, qg=qg)
    mark("quantized")
    y = ops.fwd(dims, qw, qx)
    mark("fwd")
    gw = ops.wgrad(dims, qg, qx)
    comm.all_reduce_sum(gw)
    mark("wgrad")
    gx = ops.dgrad(dims, qw, qg)
    mark("dgrad")
    return y, gw, gx


class CudaOps:
    """The library's CUDA kernels behind the `ops` interface."""
    def __init__(self, fmt):
        from microscaling_quantized_convolution_b200 import (RNE, SR, amax, conv_desc, conv_dgrad,
                                                             conv_fwd, conv_wgrad, quantize,
                                                             quantize_with_amax)
        self.RNE, self.SR = RNE, SR
        self._desc = lambda dims: conv_desc(**dims, fmt=fmt)
        self.amax = lambda t, r, c: amax(t, r, c)
        self.quantize_with_amax = lambda t, r, c, f, rnd, s, a, c0, tc: quantize_with_amax(
            t, r, c, f, rnd, s, a, sr_col0=c0, sr_cols=tc)
        self.quantize = lambda t, r, c, f, rnd, s: quantize(t, r, c, f, rnd, s)
        self.fwd = lambda dims, qw, qx: conv_fwd(self._desc(dims), qw, qx)
        self.wgrad = lambda dims, qg, qx: conv_wgrad(self._desc(dims), qg, qx)
        self.dgrad = lambda dims, qw, qg: conv_dgrad(self._desc(dims), qw, qg)
