"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/mqv.h declares, sizes workspaces and codes, and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import microscaling_quantized_convolution_b200 as mqv
from microscaling_quantized_convolution_b200 import build as mqv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mqv.h")


@pytest.fixture(scope="module")
def lib():
    mqv_build.build()
    return mqv.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mqv_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ["mqv_quantize_cbf", "mqv_conv_fwd", "mqv_conv_wgrad", "mqv_conv_dgrad",
                 "mqv_last_error", "mqv_qtensor_bytes", "mqv_conv_workspace_size"]:
        assert need in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in mqv._SIGS, f"binding lacks {name}"


def test_version_and_empty_error(lib):
    assert lib.mqv_version() >= 100
    assert isinstance(lib.mqv_last_error(), bytes)


@pytest.mark.parametrize("rows,cols,fmt,codes,scales", [
    (4, 4, mqv.NVFP4, 8, 1), (8, 16, mqv.NVFP4, 64, 8), (4, 4, mqv.NVFP6, 12, 1),
    (28 * 28 * 128, 64, mqv.NVFP4, 28 * 28 * 128 * 32, 28 * 28 * 128 * 4),
    (12, 84, mqv.NVFP6, 12 * 63, 3 * 21)])
def test_qtensor_bytes(lib, rows, cols, fmt, codes, scales):
    assert mqv.qtensor_bytes(rows, cols, fmt) == (codes, scales)


@pytest.mark.parametrize("rows,cols", [(0, 4), (4, 0), (3, 4), (4, 6), (-4, 4)])
def test_bad_views_rejected(lib, rows, cols):
    with pytest.raises(mqv.MqvError) as e:
        mqv.qtensor_bytes(rows, cols, mqv.NVFP4)
    assert e.value.status == 1


def test_bad_format_rejected(lib):
    with pytest.raises(mqv.MqvError):
        mqv.qtensor_bytes(4, 4, 7)


def test_quantize_workspace_is_partial_maxima(lib):
    assert mqv.quantize_workspace_bytes(4, 4) == 256
    big = mqv.quantize_workspace_bytes(512 * 14 * 14, 10240)
    assert big >= 4 * 148 and big % 256 == 0


def _desc(**kw):
    base = dict(N=64, Cin=128, Cout=128, H=28, W=28, Kh=3, Kw=3, stride=1, pad=1, fmt=mqv.NVFP4)
    base.update(kw)
    return mqv.conv_desc(**base)


def test_conv_workspace_sizes(lib):
    d = _desc()
    # fwd/dgrad: one 128 x 64 fp16 tile of the dequantized weight image per
    # (row tile, K tile): 1 x 18 tiles of 16 KB for 128 -> 128 channels, 3x3
    # (row-major tiles for the stride-1 halo kernel, swizzled otherwise)
    assert mqv.conv_workspace_bytes(d, mqv.OP_FWD) == 18 * 16384
    assert mqv.conv_workspace_bytes(d, mqv.OP_DGRAD) == 18 * 16384
    d2 = _desc(stride=2)
    assert mqv.conv_workspace_bytes(d2, mqv.OP_FWD) == 18 * 16384
    assert mqv.conv_workspace_bytes(d2, mqv.OP_DGRAD) == 18 * 16384
    ws = mqv.conv_workspace_bytes(d, mqv.OP_WGRAD)
    assert ws > 0 and ws % (128 * 1152 * 4) == 0          # whole split partial tiles


@pytest.mark.parametrize("kw", [dict(N=6), dict(Cin=3), dict(Cout=10), dict(stride=0),
                                dict(pad=3), dict(H=1, pad=0), dict(fmt=5), dict(Kh=0)])
def test_bad_conv_desc_rejected(lib, kw):
    with pytest.raises(mqv.MqvError) as e:
        mqv.conv_workspace_bytes(_desc(**kw), mqv.OP_FWD)
    assert e.value.status in (1, 2)


def test_conv_rejects_null_and_mismatched_operands(lib):
    d = _desc()
    w = mqv.QTensorC(16, 16, 16, 128, 1152, 0, 0)
    x = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 64, 0, 0)
    bad = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 32, 0, 0)     # wrong N
    st = lib.mqv_conv_fwd(ctypes.byref(d), ctypes.byref(w), ctypes.byref(bad), 16, None, 0, None)
    assert st == 1 and b"x" in lib.mqv_last_error()
    st = lib.mqv_conv_fwd(ctypes.byref(d), None, ctypes.byref(x), 16, None, 0, None)
    assert st == 1
    st = lib.mqv_conv_fwd(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 8, None, 0, None)
    assert st == 1                                              # misaligned output
    gy = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 64, 0, 0)
    st = lib.mqv_conv_wgrad(ctypes.byref(d), ctypes.byref(gy), ctypes.byref(x), 16, None, 0, None)
    assert st == 3                                              # needs split workspace
    wfp6 = mqv.QTensorC(16, 16, 16, 128, 1152, 1, 0)
    st = lib.mqv_conv_dgrad(ctypes.byref(d), ctypes.byref(wfp6), ctypes.byref(gy), 16, None, 0, None)
    assert st == 1                                              # format mismatch


def test_quantize_rejects_bad_arguments(lib):
    q = mqv.QTensorC(16, 16, 16, 8, 8, 0, 0)
    st = lib.mqv_quantize_cbf(None, 8, 8, 0, 0, 0, ctypes.byref(q), 16, 256, None)
    assert st == 1
    st = lib.mqv_quantize_cbf(16, 8, 8, 0, 2, 0, ctypes.byref(q), 16, 256, None)
    assert st == 1                                              # rounding mode
    st = lib.mqv_quantize_cbf(16, 8, 8, 1, 0, 0, ctypes.byref(q), 16, 256, None)
    assert st == 1                                              # out fmt differs
    st = lib.mqv_quantize_cbf(16, 8, 8, 0, 0, 0, ctypes.byref(q), None, 0, None)
    assert st == 3                                              # workspace
    st = lib.mqv_quantize_cbf(4, 8, 8, 0, 0, 0, ctypes.byref(q), 16, 256, None)
    assert st == 1                                              # misaligned src


@pytest.mark.parametrize("rows,cols,fmt,nbytes", [
    (4, 4, mqv.NVFP4, 6), (4, 4, mqv.NVFP6, 10), (8, 16, mqv.NVFP4, 48),
    (7 * 7 * 256, 84, mqv.NVFP4, 7 * 7 * 256 * 84 * 3 // 8)])
def test_replay_bytes_are_magnitude_bits(lib, rows, cols, fmt, nbytes):
    assert mqv.replay_bytes(rows, cols, fmt) == nbytes


def test_replay_entry_points_reject_bad_arguments(lib):
    q = mqv.QTensorC(16, 16, 16, 8, 8, 0, 0)
    assert lib.mqv_replay_pack(ctypes.byref(q), None, None, None) == 1         # null output
    assert lib.mqv_replay_pack(ctypes.byref(q), 8, None, None) == 1            # misaligned output
    assert lib.mqv_replay_pack(ctypes.byref(q), 16, 2, None) == 1              # misaligned counter
    bad = mqv.QTensorC(16, 16, 16, 6, 8, 0, 0)
    assert lib.mqv_replay_pack(ctypes.byref(bad), 16, None, None) == 1         # rows not a multiple of 4
    assert lib.mqv_replay_unpack(16, 8, 8, 2, 16, None) == 1                   # format
    assert lib.mqv_replay_unpack(16, 8, 8, 0, 4, None) == 1                    # misaligned codes
    assert lib.mqv_replay_dequantize(16, 16, None, 8, 8, 0, 16, None) == 1     # null tscale
    assert lib.mqv_replay_dequantize(16, 16, 16, 8, 8, 0, 8, None) == 1        # misaligned dst


def test_fused_passes_reject_bad_epilogue_arguments(lib):
    d = mqv.conv_desc(64, 128, 128, 28, 28, 3, 3, 1, 1, "nvfp4")
    w = mqv.QTensorC(16, 16, 16, 128, 1152, 0, 0)
    x = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 64, 0, 0)
    ws = mqv.conv_workspace_bytes(d, mqv.OP_FWD)
    st = lib.mqv_conv_fwd_fused(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 16, 2, None, 16, ws, None)
    assert st == 1                                              # relu must be 0 or 1
    st = lib.mqv_conv_fwd_fused(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 16, 1, 18, 16, ws, None)
    assert st == 1                                              # misaligned amax
    st = lib.mqv_conv_dgrad_fused(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 16, 18, 16, ws, None)
    assert st == 1                                              # misaligned gx_amax


def test_cuda_path_has_no_cpu_fallback():
    import torch
    x = torch.zeros(16)
    with pytest.raises(ValueError):
        mqv.quantize(x, 4, 4, "nvfp4")


def test_depthwise_entry_points_validate_before_launching(lib):
    """Workspace of the BF16 depthwise weight gradient (parts x C x Kh x Kw
    floats, rounded up to 256 bytes: for 3x3 filters at stride 1 or 2 a part
    per spatial tile, 8 output pixels wide, else a part per range of output
    pixels) and descriptor or pointer errors returned without a launch."""
    d = mqv.dw_desc(16, 32, 20, 20, 3, 3, 1, 1)       # 20x20 output in 8x8 tiles: 3 x 3 parts
    assert mqv.dw_wgrad_workspace_bytes(d) == 10496   # 9 x 32 x 9 x 4 = 10368, rounded up
    d = mqv.dw_desc(32, 2, 56, 56, 3, 3, 1, 1)        # 56x56 in 8x8 tiles: 49 parts
    assert mqv.dw_wgrad_workspace_bytes(d) == 3584    # 49 x 18 x 4 = 3528, rounded up
    d = mqv.dw_desc(16, 32, 40, 40, 5, 5, 2, 2)       # 5x5: 400 output pixels, 64 ranges
    assert mqv.dw_wgrad_workspace_bytes(d) == 64 * 32 * 25 * 4
    for bad in (mqv.dw_desc(6, 2, 4, 4, 3, 3, 1, 1), mqv.dw_desc(4, 2, 4, 4, 3, 3, 0, 1),
                mqv.dw_desc(4, 2, 4, 4, 3, 3, 1, 3), mqv.dw_desc(4, 0, 4, 4, 3, 3, 1, 1),
                mqv.dw_desc(4, 2, 2, 2, 5, 5, 1, 1)):
        with pytest.raises(mqv.MqvError):
            mqv.dw_wgrad_workspace_bytes(bad)
    d = mqv.dw_desc(4, 2, 4, 4, 3, 3, 1, 1)
    invalid = 1                                        # MQV_ERR_INVALID_ARG
    assert lib.mqv_dw_fwd(ctypes.byref(d), None, None, None, None) == invalid
    assert lib.mqv_dw_dgrad(ctypes.byref(d), None, None, None, None) == invalid
    assert lib.mqv_dw_wgrad(ctypes.byref(d), None, None, None, None, 0, None) == invalid
    assert lib.mqv_dw_fwd(None, None, None, None, None) == invalid


def test_depthwise_bindings_validate_before_shape_arithmetic(lib):
    """The Python calls ask the library to check the descriptor before they
    size anything, so a bad descriptor raises MqvError (a stride of 0 must
    not become a Python ZeroDivisionError)."""
    import torch
    x = torch.zeros(16, dtype=torch.bfloat16)
    y = torch.zeros(16, dtype=torch.float32)
    for bad in (mqv.dw_desc(6, 2, 4, 4, 3, 3, 1, 1), mqv.dw_desc(4, 2, 4, 4, 3, 3, 0, 1),
                mqv.dw_desc(4, 2, 4, 4, 3, 3, 1, 3)):
        for call in (lambda: mqv.dw_fwd(bad, x, x, y), lambda: mqv.dw_dgrad(bad, x, x, y),
                     lambda: mqv.dw_wgrad(bad, x, x, y), lambda: mqv.dw_out_hw(bad)):
            with pytest.raises(mqv.MqvError):
                call()


def test_noalloc_scratch_covers_every_planned_layer(lib):
    """The weight gradient's split planner keeps its partial sums under the
    32 MiB array of mqv_conv_wgrad_noalloc for every shape (at most 148
    tiles of 128 x 384 fp32), so no layer of the benchmarked workloads, nor
    any shape of a wide sweep, is rejected by that entry point.  Sizing is a
    host call: no GPU needed."""
    import workloads
    shapes = [l.dims() | {"fmt": l.fmt} for l in
              [workloads.tiny_layer(), workloads.resnet18_layer2()] + workloads.resnet18_body()
              + workloads.yolov8n_mix()]
    for cin in (4, 16, 64, 128, 256, 512, 1024):
        for cout in (16, 64, 128, 384, 512, 2048):
            for k in (1, 3, 5):
                shapes.append(dict(N=32, Cin=cin, Cout=cout, H=14, W=14, Kh=k, Kw=k, stride=1,
                                   pad=k // 2, fmt="nvfp4"))
    worst = max(mqv.conv_workspace_bytes(mqv.conv_desc(**s), mqv.OP_WGRAD) for s in shapes)
    assert 0 < worst <= 148 * 128 * 384 * 4 < 32 << 20


def test_blockscaled_forward_workspace_and_rejections(lib):
    """The block-scaled forward pass: its weight image is 18 KB per (row tile,
    K tile) (16 KB of padded codes and 2 KB of scale atoms); layers outside
    its range (NVFP6, stride 2, N other than 64 or 128, Cin not a multiple
    of 64, Kw > 3) are rejected as unsupported before any launch."""
    d = _desc()
    assert mqv.conv_workspace_bytes(d, mqv.OP_FWD_BLOCKSCALED) == 18 * 18432
    for kw in (dict(fmt=mqv.NVFP6), dict(stride=2), dict(N=16), dict(N=32), dict(N=256), dict(Cin=96),
               dict(Kh=5, Kw=5, pad=2)):
        with pytest.raises(mqv.MqvError) as e:
            mqv.conv_workspace_bytes(_desc(**kw), mqv.OP_FWD_BLOCKSCALED)
        assert e.value.status == 2
    w = mqv.QTensorC(16, 16, 16, 128, 1152, 0, 0)
    x = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 64, 0, 0)
    assert lib.mqv_conv_fwd_blockscaled(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 16, None, 0, None) == 3


def test_block_shapes_are_validated(lib):
    """The 16-element line blocks of the naive scheme: accepted by the
    many-tensor quantizer (not mixed with squares in one call), refused by
    the single-tensor quantizer, by shapes that do not split into lines, and
    by conv passes other than the stride-1 1 x 1 GEMMs in the stated shapes.
    Every refusal comes before any CUDA call."""
    def job(rows, cols, blocks):
        return mqv.QuantJobC(16, rows, cols, 0, 0, 0, mqv.QTensorC(16, 16, 16, rows, cols, 0, blocks))

    def many(*jobs):
        arr = (mqv.QuantJobC * len(jobs))(*jobs)
        return lib.mqv_quantize_many(arr, len(jobs), 16, 1 << 20, None)

    assert many(job(64, 64, 3)) == 1                             # unknown shape
    assert many(job(64, 8, mqv.BLOCKS_1X16)) == 1                # cols not a multiple of 16
    assert many(job(8, 64, mqv.BLOCKS_16X1)) == 1                # rows not a multiple of 16
    assert many(job(64, 64, mqv.BLOCKS_4X4), job(64, 64, mqv.BLOCKS_1X16)) == 2   # mixed in one call
    q = mqv.QTensorC(16, 16, 16, 64, 64, 0, mqv.BLOCKS_1X16)
    assert lib.mqv_quantize_cbf(16, 64, 64, 0, 0, 0, ctypes.byref(q), 16, 256, None) == 2
    # conv passes: a 3 x 3 layer refuses line blocks
    d = _desc()
    w = mqv.QTensorC(16, 16, 16, 128, 1152, 0, mqv.BLOCKS_1X16)
    x = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 64, 0, mqv.BLOCKS_16X1)
    assert lib.mqv_conv_fwd(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 16, 16, 1 << 24, None) == 2
    assert b"line blocks" in lib.mqv_last_error()
    # a 1 x 1 layer: only the stated shape per operand
    d1 = _desc(Cin=1152, Kh=1, Kw=1, pad=0)
    w1 = mqv.QTensorC(16, 16, 16, 128, 1152, 0, mqv.BLOCKS_16X1)          # fwd wants 1 x 16
    x1 = mqv.QTensorC(16, 16, 16, 28 * 28 * 1152, 64, 0, mqv.BLOCKS_16X1)
    assert lib.mqv_conv_fwd(ctypes.byref(d1), ctypes.byref(w1), ctypes.byref(x1), 16, 16, 1 << 24, None) == 2
    gy = mqv.QTensorC(16, 16, 16, 28 * 28 * 128, 64, 0, mqv.BLOCKS_16X1)  # wgrad wants 1 x 16
    xw = mqv.QTensorC(16, 16, 16, 28 * 28 * 1152, 64, 0, mqv.BLOCKS_1X16)
    assert lib.mqv_conv_wgrad(ctypes.byref(d1), ctypes.byref(gy), ctypes.byref(xw), 16, 16, 1 << 28, None) == 2
    # the block-scaled forward pass takes squares only
    assert lib.mqv_conv_fwd_blockscaled(ctypes.byref(d), ctypes.byref(w), ctypes.byref(x), 16, 16, 1 << 24,
                                        None) == 2


def test_selftest_wait_limit_is_validated(lib):
    for bad in (0, -5, (1 << 32) + 1):
        assert lib.mqv_selftest_wait_timeout(bad, None) == 1
    assert b"limit_cycles" in lib.mqv_last_error()
