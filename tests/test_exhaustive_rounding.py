"""Every fp32 element value of magnitude at most emax through the quantizer.

The construction (tests/exhaustive_slices.py) makes T = 1 and B = 1, so each
element's code is the element rounding of x alone: round to nearest even,
or stochastic with the element's own Philox word.  The GPU sweep covers all
2·(bits(emax) + 1) patterns (about 2.2e9 per format, 139 slices of 15·2^20
values) and compares every packed code byte with the oracle's element
rounding, which a spawn-started process pool computes slice by slice on the
host cores: opt in with MQV_EXHAUSTIVE=1 (about two minutes per format and
rounding on a 16-core host).  The CPU tests check the construction against
the oracle's quantizer and the pool's packed expectation on small slices."""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

from oracle import mqv_oracle as O
from tests import exhaustive_slices as E

PER = 15 << 20


@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_slice_construction_reduces_quantization_to_element_rounding(fmt, rounding):
    """On CPU: the oracle's quantizer of a slice (patterns around 0, around
    1, around emax and negative ones) gives T = 1, scale 1 for every test
    block and exactly the element-rounding codes the sweep compares with;
    the slice job's packed expectation is the packing of those codes."""
    n = E.pattern_count(fmt)
    top = n // 2 - 1
    one = int(np.float32(1.0).view(np.uint32))
    vals = np.concatenate([E.patterns(fmt, 0, 3000), E.patterns(fmt, one - 1500, 3000),
                           E.patterns(fmt, top - 2999, 3000), E.patterns(fmt, n - 3000, 3000)])
    X, blocks, slots = E.slice_view(fmt, vals)
    q = O.quantize(X, E.FMT[fmt], rounding, E.SEED)
    assert q.T == np.float32(1.0)
    one_code = O.cast_e4m3(np.array([1.0], np.float32))[0]
    assert np.all(q.scales.reshape(-1)[1:] == one_code)
    r, c = E.positions(blocks, slots)
    assert np.array_equal(q.codes[r, c], E.element_codes(fmt, vals, r, c, rounding))
    for start in (0, one - 1500, n - 3000):
        s0, Xj, packed = E.slice_job((fmt, rounding, start, 3000))
        qj = O.quantize(Xj, E.FMT[fmt], rounding, E.SEED)
        assert s0 == start and np.array_equal(packed, O.pack_codes(qj.codes, E.FMT[fmt]))


@pytest.mark.gpu
@pytest.mark.skipif(os.environ.get("MQV_EXHAUSTIVE") != "1",
                    reason="about 2.2e9 values per format; opt in with MQV_EXHAUSTIVE=1")
@pytest.mark.parametrize("fmt", ["nvfp4", "nvfp6"])
@pytest.mark.parametrize("rounding", [O.RNE, O.SR])
def test_every_element_pattern_on_the_gpu(fmt, rounding):
    import microscaling_quantized_convolution_b200 as mqv
    n = E.pattern_count(fmt)
    jobs = [(fmt, rounding, s, min(PER, n - s)) for s in range(0, n, PER)]
    procs = max(1, min(16, (os.cpu_count() or 2) - 1))
    checked = 0
    with mp.get_context("spawn").Pool(procs) as pool:
        for start, X, want in pool.imap(E.slice_job, jobs):
            rows = X.shape[0]
            q = mqv.quantize(torch.from_numpy(X).cuda().view(-1), rows, E.COLS, fmt,
                             mqv.RNE if rounding == O.RNE else mqv.SR, E.SEED)
            got = q.codes.cpu().numpy().reshape(want.shape)
            assert float(q.tscale.item()) == 1.0
            if not np.array_equal(got, want):
                codes = O.unpack_codes(got, rows, E.COLS, E.FMT[fmt])
                ref = O.unpack_codes(want, rows, E.COLS, E.FMT[fmt])
                bad = np.argwhere(codes != ref)[:4]
                raise AssertionError(f"patterns from {start}: {int(np.sum(codes != ref))} codes differ, "
                                     f"first x = {[float(X[r, c]) for r, c in bad]}")
            checked += min(PER, n - start)
    assert checked == n
