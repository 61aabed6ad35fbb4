"""The data-parallel exchange of the layer step on two and four CPU ranks (gloo).

Each rank runs its batch shard through `dp.data_parallel_step` with the
oracle as the kernels: the sharded step must reproduce the single-process
step on the whole batch (codes bit for bit, outputs to fp64 rounding)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from microscaling_quantized_convolution_b200 import dp
from oracle import mqv_oracle as O

DIMS = dict(Cin=8, Cout=12, H=6, W=5, Kh=3, Kw=3, stride=1, pad=1)
N_GLOBAL = 16
SEED = 31


class OracleOps:
    """The oracle behind the ops interface (torch CPU tensors in and out)."""
    RNE, SR = O.RNE, O.SR

    def amax(self, t, rows, cols):
        return torch.tensor([float(t.abs().max())], dtype=torch.float32)

    def quantize_with_amax(self, t, rows, cols, fmt, rnd, seed, amax, col0, total):
        return O.quantize(t.numpy().reshape(rows, cols), fmt, rnd, seed, amax=float(amax[0]),
                          col_offset=col0, total_cols=total)

    def quantize(self, t, rows, cols, fmt, rnd, seed):
        return O.quantize(t.numpy().reshape(rows, cols), fmt, rnd, seed)

    @staticmethod
    def _shape(d):
        return O.ConvShape(d["N"], d["Cin"], d["Cout"], d["H"], d["W"], d["Kh"], d["Kw"],
                           d["stride"], d["pad"])

    def _vals(self, q, shape):
        return O.code_values(q).reshape(shape)

    def fwd(self, d, qw, qx):
        s = self._shape(d)
        Y, _ = O.conv_fwd(self._vals(qw, (s.Cout, s.Kh, s.Kw, s.Cin)),
                          self._vals(qx, (s.H, s.W, s.Cin, s.N)), s)
        return torch.from_numpy(Y * np.float64(qw.T) * np.float64(qx.T))

    def wgrad(self, d, qg, qx):
        s = self._shape(d)
        GW, _ = O.conv_wgrad(self._vals(qg, (s.Ho, s.Wo, s.Cout, s.N)),
                             self._vals(qx, (s.H, s.W, s.Cin, s.N)), s)
        return torch.from_numpy(GW * np.float64(qg.T) * np.float64(qx.T))

    def dgrad(self, d, qw, qg):
        s = self._shape(d)
        GX, _ = O.conv_dgrad(self._vals(qw, (s.Cout, s.Kh, s.Kw, s.Cin)),
                             self._vals(qg, (s.Ho, s.Wo, s.Cout, s.N)), s)
        return torch.from_numpy(GX * np.float64(qw.T) * np.float64(qg.T))


def _inputs():
    g = torch.Generator().manual_seed(5)
    Ho = (DIMS["H"] + 2 * DIMS["pad"] - DIMS["Kh"]) // DIMS["stride"] + 1
    Wo = (DIMS["W"] + 2 * DIMS["pad"] - DIMS["Kw"]) // DIMS["stride"] + 1
    X = torch.randn((DIMS["H"], DIMS["W"], DIMS["Cin"], N_GLOBAL), generator=g)
    X[0, 0, 0, 3] = 40.0                         # the global max lives on rank 0
    W = torch.randn((DIMS["Cout"], DIMS["Kh"], DIMS["Kw"], DIMS["Cin"]), generator=g)
    G = torch.randn((Ho, Wo, DIMS["Cout"], N_GLOBAL), generator=g) * 1e-3
    G[1, 1, 2, 13] = 0.5                         # ... and this one on rank 1
    return X, W, G


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, W, G = _inputs()
        col0, n = dp.shard_columns(N_GLOBAL, rank, world)
        dims = dict(DIMS, N=n)
        y, gw, gx = dp.data_parallel_step(OracleOps(), dp.torch_comm(), X[..., col0:col0 + n].contiguous(),
                                          W, G[..., col0:col0 + n].contiguous(), dims, O.FP4,
                                          N_GLOBAL, rank, world, SEED)
        torch.save({"y": y, "gw": gw, "gx": gx}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_match_single_process(tmp_path, world):
    """Two ranks (8 batch items each) and four (4 each; the maxima of X and
    G_Y then live on ranks 0 and 3)."""
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    X, W, G = _inputs()
    ref = dp.data_parallel_step(OracleOps(), dp.Comm(lambda t: None, lambda t: None), X, W, G,
                                dict(DIMS, N=N_GLOBAL), O.FP4, N_GLOBAL, 0, 1, SEED)
    outs = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    n = N_GLOBAL // world
    for r, o in enumerate(outs):
        sl = slice(r * n, (r + 1) * n)
        assert torch.allclose(o["y"], ref[0][..., sl], rtol=1e-12, atol=1e-15)
        assert torch.allclose(o["gx"], ref[2][..., sl], rtol=1e-12, atol=1e-15)
        assert torch.allclose(o["gw"], ref[1], rtol=1e-12, atol=1e-15)


def test_shard_quantization_equals_whole_batch_codes():
    """Global amax + global SR numbering: each shard's codes are exactly the
    matching columns of the whole-batch quantization (X RNE, G_Y SR)."""
    X, W, G = _inputs()
    ops = OracleOps()
    rows = G.numel() // N_GLOBAL
    whole = O.quantize(G.numpy().reshape(rows, N_GLOBAL), O.FP4, O.SR, SEED)
    amax = ops.amax(G, rows, N_GLOBAL)
    for rank in range(2):
        col0, n = dp.shard_columns(N_GLOBAL, rank, 2)
        part = ops.quantize_with_amax(G[..., col0:col0 + n].contiguous(), rows, n, O.FP4, O.SR,
                                      SEED, amax, col0, N_GLOBAL)
        assert np.array_equal(part.codes, whole.codes[:, col0:col0 + n])
        assert np.array_equal(part.scales, whole.scales[:, col0 // 4:(col0 + n) // 4])


def test_shard_columns_rejects_ragged_batches():
    with pytest.raises(ValueError):
        dp.shard_columns(12, 0, 2)      # 6 per rank is not a multiple of 4
    assert dp.shard_columns(16, 1, 2) == (8, 8)
