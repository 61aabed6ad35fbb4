"""The BF16 depthwise kernels' per-thread code, built for the host with an
address and undefined-behaviour sanitizer and run over every thread index of
each launch, against the oracle (reading R22): fwd, input and weight
gradients within the parity tolerance, no access outside any buffer.  The
GPU runs the same functions, one thread each."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import mqv_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "microscaling_quantized_convolution_b200", "csrc")

# (N, C, H, W, Kh, Kw, stride, pad): odd sizes, stride 2 with padding,
# rectangular and 5x5 kernels, a 1x1 kernel, one pixel wide inputs
SHAPES = [(4, 3, 7, 9, 3, 3, 1, 1), (8, 5, 9, 7, 3, 3, 2, 1), (4, 6, 10, 10, 5, 5, 2, 2),
          (12, 4, 6, 6, 3, 1, 1, 0), (4, 7, 5, 5, 1, 1, 1, 0), (16, 2, 1, 8, 1, 3, 1, 0),
          (4, 3, 40, 36, 3, 3, 1, 1)]
# larger layers the GPU test adds: a 80x80 and a strided 5x5 one, one whose
# 8x8 output tiles end ragged at stride 2, and one at stride 3
GPU_LARGE = [(16, 64, 80, 80, 3, 3, 1, 1), (16, 32, 40, 40, 5, 5, 2, 2), (16, 64, 83, 77, 3, 3, 2, 1),
             (8, 64, 50, 47, 5, 5, 3, 2)]


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ is not installed")
    exe = str(tmp_path_factory.mktemp("dw") / "dw_host_harness")
    base = [gxx, "-O1", "-std=c++17", "-I", CSRC, os.path.join(ROOT, "tests", "dw_host_harness.cpp"), "-o", exe]
    r = subprocess.run(base[:2] + ["-fsanitize=address,undefined", "-fno-sanitize-recover=all"] + base[2:],
                       capture_output=True, text=True)
    if r.returncode != 0:            # no sanitizer runtime: plain build
        subprocess.run(base, check=True)
    return exe


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """Raw bfloat16 bit patterns of x (torch's round-to-nearest-even)."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy()


def _run(exe, tmp, op, dims, a, b, count):
    pa, pb, po = (os.path.join(tmp, f) for f in ("a.bin", "b.bin", "o.bin"))
    _bf16_bits(a).tofile(pa)
    _bf16_bits(b).tofile(pb)
    subprocess.run([exe, str(op), *map(str, dims), pa, pb, po], check=True, timeout=300)
    out = np.fromfile(po, np.float32)
    assert out.size == count
    return out


def _close(got, ref, S, what):
    err = np.abs(got.astype(np.float64) - ref)
    tol = 1e-5 * S + 1e-7
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, f"{what}: {bad.size} outputs off, worst {err.max():.3g}"


@pytest.mark.parametrize("dims", SHAPES, ids=[f"n{d[0]}c{d[1]}_{d[2]}x{d[3]}_k{d[4]}x{d[5]}s{d[6]}p{d[7]}"
                                              for d in SHAPES])
def test_host_build_of_depthwise_kernels_matches_oracle(harness, tmp_path, dims):
    N, C, H, W, Kh, Kw, st, pad = dims
    s = O.ConvShape(N, C, C, H, W, Kh, Kw, st, pad)
    rng = np.random.default_rng(sum(dims))
    X = rng.standard_normal((H, W, C, N)).astype(np.float32)
    Wd = (rng.standard_normal((C, Kh, Kw)) * 0.3).astype(np.float32)
    G = (rng.standard_normal((s.Ho, s.Wo, C, N)) * 1e-3).astype(np.float32)
    ref = O.depthwise_layer_outputs(X, Wd, G, s)
    y = _run(harness, tmp_path, 0, dims, Wd, X, s.Ho * s.Wo * C * N)
    _close(y, ref["y"][0].reshape(-1), ref["y"][1].reshape(-1), "fwd")
    gx = _run(harness, tmp_path, 1, dims, Wd, G, H * W * C * N)
    _close(gx, ref["gx"][0].reshape(-1), ref["gx"][1].reshape(-1), "dgrad")
    gw = _run(harness, tmp_path, 2, dims, G, X, C * Kh * Kw)
    _close(gw, ref["gw"][0].reshape(-1), ref["gw"][1].reshape(-1), "wgrad")


def test_host_build_of_depthwise_weight_gradient_long_reduction(harness, tmp_path):
    """A 56x56, N = 32 layer: 100,352 terms per weight, split into parts of
    about 512 terms per running sum, still within the tolerance."""
    dims = (32, 2, 56, 56, 3, 3, 1, 1)
    N, C, H, W, Kh, Kw, st, pad = dims
    s = O.ConvShape(N, C, C, H, W, Kh, Kw, st, pad)
    rng = np.random.default_rng(9)
    X = np.maximum(rng.standard_normal((H, W, C, N)), 0).astype(np.float32)
    G = (rng.standard_normal((s.Ho, s.Wo, C, N)) * 1e-3).astype(np.float32)
    GW, S = O.depthwise_wgrad(O.to_bf16(G), O.to_bf16(X), s)
    gw = _run(harness, tmp_path, 2, dims, G, X, C * Kh * Kw)
    _close(gw, GW.reshape(-1), S.reshape(-1), "wgrad")


def test_library_accepts_every_test_shape():
    """The library's own descriptor check passes for every shape the host
    and GPU tests use (run without a GPU: sizing validates the descriptor)."""
    import microscaling_quantized_convolution_b200 as mqv
    for dims in SHAPES + GPU_LARGE:
        assert mqv.dw_wgrad_workspace_bytes(mqv.dw_desc(*dims)) > 0
