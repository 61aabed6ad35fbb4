"""Shared helpers of the GPU parity tests: run the oracle and the CUDA path on
the same seeded fp32 inputs and compare (codes/scales/T bit for bit, conv
outputs within |y - y_ref| <= 1e-5·S + 1e-7, S = sum_k |a_k·b_k|)."""
import numpy as np
import torch

import microscaling_quantized_convolution_b200 as mqv
from oracle import mqv_oracle as O

REL_TOL = 1e-5
ABS_TOL = 1e-7

FMT = {"nvfp4": O.FP4, "nvfp6": O.FP6}
RND = {mqv.RNE: O.RNE, mqv.SR: O.SR}


def gpu_quantize(x: torch.Tensor, rows, cols, fmt, rnd, seed=0):
    """Quantize on the GPU; returns (packed codes, scales, T) as numpy."""
    xd = x.to("cuda").contiguous().view(-1)
    q = mqv.quantize(xd, rows, cols, fmt, rnd, seed)
    torch.cuda.synchronize()
    return q, q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.tscale.cpu().numpy()[0]


def assert_quant_equal(x_np, rows, cols, fmt, rnd, seed, gq, amax=None, row_offset=0):
    """Oracle quantization of x_np (rows x cols) vs GPU bytes (gq = codes,
    scales, T); codes/scales may be the matching band of a larger tensor."""
    oq = O.quantize(x_np.reshape(rows, cols), FMT[fmt], RND[rnd], seed, amax=amax, row_offset=row_offset)
    codes, scales, T = gq
    ocodes = O.pack_codes(oq.codes, FMT[fmt])
    assert np.float32(T).view(np.uint32) == np.float32(oq.T).view(np.uint32), (T, oq.T)
    bad_s = np.nonzero(scales != oq.scales.reshape(-1))[0]
    assert bad_s.size == 0, f"{bad_s.size} scale bytes differ, first at {bad_s[:5]}"
    bad_c = np.nonzero(codes != ocodes)[0]
    assert bad_c.size == 0, f"{bad_c.size} code bytes differ, first at {bad_c[:5]}"
    return oq


def assert_close(got: np.ndarray, ref: np.ndarray, S: np.ndarray, what: str):
    err = np.abs(got.astype(np.float64) - ref)
    lim = REL_TOL * S + ABS_TOL
    bad = np.nonzero(err > lim)
    assert bad[0].size == 0, (f"{what}: {bad[0].size} of {err.size} outside tolerance; "
                              f"worst err/lim {np.max(err / lim):.3g}")
    return float(np.max(err / np.maximum(S, 1e-30)))
