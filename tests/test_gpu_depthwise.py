"""GPU parity of the BF16 depthwise passes (reading R22) against the oracle:
fwd, input and weight gradients within the parity tolerance, the same bits
on a second run; the bindings reject bad descriptors and short tensors."""
import numpy as np
import pytest
import torch

import microscaling_quantized_convolution_b200 as mqv
from oracle import mqv_oracle as O
from tests.test_depthwise_host import GPU_LARGE, SHAPES, _close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dims", SHAPES + GPU_LARGE,
                         ids=[f"n{d[0]}c{d[1]}_{d[2]}x{d[3]}_k{d[4]}x{d[5]}s{d[6]}p{d[7]}" for d in SHAPES + GPU_LARGE])
def test_depthwise_passes_match_oracle(dims):
    N, C, H, W, Kh, Kw, st, pad = dims
    s = O.ConvShape(N, C, C, H, W, Kh, Kw, st, pad)
    rng = np.random.default_rng(sum(dims) + 1)
    X = rng.standard_normal((H, W, C, N)).astype(np.float32)
    Wd = (rng.standard_normal((C, Kh, Kw)) * 0.3).astype(np.float32)
    G = (rng.standard_normal((s.Ho, s.Wo, C, N)) * 1e-3).astype(np.float32)
    ref = O.depthwise_layer_outputs(X, Wd, G, s)
    d = mqv.dw_desc(N, C, H, W, Kh, Kw, st, pad)
    xb, wb, gb = (torch.from_numpy(t).to(torch.bfloat16).cuda() for t in (X, Wd, G))
    y = mqv.dw_fwd(d, wb, xb)
    gx = mqv.dw_dgrad(d, wb, gb)
    gw = mqv.dw_wgrad(d, gb, xb)
    y2, gx2, gw2 = mqv.dw_fwd(d, wb, xb), mqv.dw_dgrad(d, wb, gb), mqv.dw_wgrad(d, gb, xb)
    torch.cuda.synchronize()
    _close(y.cpu().numpy().reshape(-1), ref["y"][0].reshape(-1), ref["y"][1].reshape(-1), "fwd")
    _close(gx.cpu().numpy().reshape(-1), ref["gx"][0].reshape(-1), ref["gx"][1].reshape(-1), "dgrad")
    _close(gw.cpu().numpy().reshape(-1), ref["gw"][0].reshape(-1), ref["gw"][1].reshape(-1), "wgrad")
    assert torch.equal(y, y2) and torch.equal(gx, gx2) and torch.equal(gw, gw2)


def test_depthwise_rejects_bad_descriptors():
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(16, dtype=torch.float32, device="cuda")
    for bad in (mqv.dw_desc(6, 2, 4, 4, 3, 3, 1, 1),       # N % 4
                mqv.dw_desc(4, 2, 4, 4, 3, 3, 0, 1),       # stride 0
                mqv.dw_desc(4, 2, 4, 4, 3, 3, 1, 3)):      # pad >= K
        with pytest.raises(mqv.MqvError):
            mqv.dw_fwd(bad, x, x, y)
    assert mqv.device_errors() == 0


def test_depthwise_rejects_short_tensors():
    """The C ABI takes no tensor sizes; the bindings compare every operand's
    element count with the descriptor before anything is launched."""
    d = mqv.dw_desc(4, 8, 6, 6, 3, 3, 1, 1)
    w = torch.zeros(8 * 9, dtype=torch.bfloat16, device="cuda")
    x = torch.zeros(6 * 6 * 8 * 4, dtype=torch.bfloat16, device="cuda")
    short = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        mqv.dw_fwd(d, w, short)
    with pytest.raises(ValueError):
        mqv.dw_fwd(d, short, x)
    with pytest.raises(ValueError):
        mqv.dw_fwd(d, w, x, torch.zeros(16, device="cuda"))
    with pytest.raises(ValueError):
        mqv.dw_dgrad(d, w, short)
    with pytest.raises(ValueError):
        mqv.dw_wgrad(d, short, x)
    with pytest.raises(ValueError):
        mqv.dw_wgrad(d, x, x, torch.zeros(16, device="cuda"))
    assert mqv.device_errors() == 0
