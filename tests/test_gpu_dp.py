"""The data-parallel step (dp.data_parallel_step, the exchange the benchmark
runs for several ranks) with the library's CUDA kernels: two ranks share the
one visible GPU, with the collectives on gloo (host-side; no kernel waits on
another rank).  Each rank's quantized shards must be the columns of the
oracle's quantization of the whole batch, bit for bit (global T, Philox words
numbered in the whole batch), and its outputs (Y and G_X of its shard, G_W
summed over the ranks) must match the oracle's single-process step within
the parity tolerance."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import mqv_oracle as O
from tests.parity_utils import FMT, assert_close

pytestmark = pytest.mark.gpu

LAYERS = [("nvfp4", dict(Cin=64, Cout=64, H=6, W=7, Kh=3, Kw=3, stride=1, pad=1), 32),    # kernel-row paths
          ("nvfp6", dict(Cin=24, Cout=40, H=9, W=9, Kh=3, Kw=3, stride=2, pad=1), 16)]   # generic kernels
SEED = 91


def _inputs(dims, n_global):
    g = torch.Generator().manual_seed(5)
    X = torch.relu(torch.randn((dims["H"], dims["W"], dims["Cin"], n_global), generator=g))
    W = torch.randn((dims["Cout"], dims["Kh"], dims["Kw"], dims["Cin"]), generator=g) * 0.1
    Ho = (dims["H"] + 2 * dims["pad"] - dims["Kh"]) // dims["stride"] + 1
    Wo = (dims["W"] + 2 * dims["pad"] - dims["Kw"]) // dims["stride"] + 1
    G = torch.randn((Ho, Wo, dims["Cout"], n_global), generator=g) * 1e-3
    return X, W, G


def _rank(rank, world, port, fmt, dims, n_global, out_dir):
    import microscaling_quantized_convolution_b200 as mqv
    from microscaling_quantized_convolution_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, G = _inputs(dims, n_global)
    c0, n = dp.shard_columns(n_global, rank, world)
    xs, gs = (t[..., c0:c0 + n].contiguous().cuda() for t in (X, G))
    q = {}
    y, gw, gx = dp.data_parallel_step(dp.CudaOps(fmt), dp.torch_comm(), xs.view(-1), W.cuda().view(-1), gs.view(-1),
                                      dict(dims, N=n), fmt, n_global, rank, world, SEED, quantized=q)
    torch.cuda.synchronize()
    res = {"y": y.cpu().numpy(), "gw": gw.cpu().numpy(), "gx": gx.cpu().numpy(), "err": mqv.device_errors()}
    for name in ("qx", "qg"):
        t = q[name]
        res[name + "_codes"] = O.unpack_codes(t.codes.cpu().numpy(), t.rows, t.cols, FMT[fmt])
        res[name + "_scales"] = t.scales.cpu().numpy().reshape(t.rows // 4, t.cols // 4)
        res[name + "_T"] = np.float32(t.tscale.item())
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **res)
    dist.destroy_process_group()


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("fmt,dims,n_global", LAYERS, ids=[l[0] for l in LAYERS])
def test_two_ranks_reproduce_the_single_process_step(fmt, dims, n_global):
    world = 2
    with tempfile.TemporaryDirectory() as tmp:
        mp.spawn(_rank, args=(world, _port(), fmt, dims, n_global, tmp), nprocs=world, join=True)
        ranks = [dict(np.load(os.path.join(tmp, f"rank{r}.npz"))) for r in range(world)]
    s = O.ConvShape(n_global, dims["Cin"], dims["Cout"], dims["H"], dims["W"], dims["Kh"], dims["Kw"],
                    dims["stride"], dims["pad"])
    X, W, G = _inputs(dims, n_global)
    qx, qw, qg = O.quantize_layer(X.numpy(), W.numpy(), G.numpy(), s, FMT[fmt], SEED)
    ref = O.layer_outputs(qx, qw, qg, s)
    n = n_global // world
    gw_sum = None
    for r, res in enumerate(ranks):
        assert int(res["err"]) == 0
        cols = slice(r * n, (r + 1) * n)
        for name, oq in (("qx", qx), ("qg", qg)):
            assert res[name + "_T"] == oq.T, f"rank {r} {name} T"
            assert np.array_equal(res[name + "_codes"], oq.codes[:, cols]), f"rank {r} {name} codes"
            assert np.array_equal(res[name + "_scales"], oq.scales[:, r * n // 4:(r + 1) * n // 4]), f"rank {r} {name}"
        y_ref, y_s = ref["y"]
        gx_ref, gx_s = ref["gx"]
        assert_close(res["y"].reshape(-1), y_ref[..., cols].reshape(-1), y_s[..., cols].reshape(-1), f"rank {r} Y")
        assert_close(res["gx"].reshape(-1), gx_ref[..., cols].reshape(-1), gx_s[..., cols].reshape(-1), f"rank {r} G_X")
        gw_sum = res["gw"] if gw_sum is None else gw_sum
        assert np.array_equal(res["gw"], gw_sum), "G_W differs between the ranks after the sum"
    gw_ref, gw_s = ref["gw"]
    # two fp32 partial sums added once more: the tolerance of the two halves
    assert_close(gw_sum.reshape(-1), gw_ref.reshape(-1), gw_s.reshape(-1), "summed G_W")
