"""Seeded synthetic inputs for the MicroQonv layer workloads.

This module only draws random numbers and describes shapes; it holds none of
the quantization or convolution arithmetic, so both the CPU oracle tests and
the CUDA path can take their inputs from it.

Tensor layouts (channel-batch-first, n fastest):
  X   [H][W][Cin][N]      fp32
  W   [Cout][Kh][Kw][Cin] fp32
  G_Y [Ho][Wo][Cout][N]   fp32
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Layer:
    name: str
    N: int
    Cin: int
    Cout: int
    H: int
    W: int
    K: int
    stride: int
    pad: int
    fmt: str              # "nvfp4" | "nvfp6"
    x_dist: str           # "normal" | "relu" | "silu"
    gy_std: float
    seed: int
    cin_real: int = 0     # channels carrying data; the rest are zero padding

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - self.K) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad - self.K) // self.stride + 1

    def flops(self) -> int:
        return 2 * self.Cout * self.Cin * self.K * self.K * self.Ho * self.Wo * self.N

    def dims(self):
        return dict(N=self.N, Cin=self.Cin, Cout=self.Cout, H=self.H, W=self.W,
                    Kh=self.K, Kw=self.K, stride=self.stride, pad=self.pad)


def tiny_layer() -> Layer:
    """Single 3x3 conv, stride 1, no padding, N=4, 16 -> 16 channels, 8x8."""
    return Layer("tiny_3x3_c16_n4", 4, 16, 16, 8, 8, 3, 1, 0, "nvfp4", "normal", 1e-3, 0)


def resnet18_layer2() -> Layer:
    """ResNet-18 layer2-shaped 3x3 conv: N=64, 128 -> 128, 28x28, pad 1."""
    return Layer("resnet18_layer2_3x3_c128_n64", 64, 128, 128, 28, 28, 3, 1, 1,
                 "nvfp4", "relu", 1e-4, 0)


def resnet18_body(N: int = 32) -> list[Layer]:
    """The sixteen 3x3 convs of a ResNet-18 body at 224x224 input."""
    spec = [(64, 64, 56, 1)] * 4
    spec += [(64, 128, 56, 2)] + [(128, 128, 28, 1)] * 3
    spec += [(128, 256, 28, 2)] + [(256, 256, 14, 1)] * 3
    spec += [(256, 512, 14, 2)] + [(512, 512, 7, 1)] * 3
    return [Layer(f"resnet18_body_l{i:02d}_{ci}to{co}_{h}px_s{s}", N, ci, co, h, h, 3, s, 1,
                  "nvfp4", "relu", 1e-4, i)
            for i, (ci, co, h, s) in enumerate(spec)]


def yolov8n_mix(N: int = 16) -> list[Layer]:
    """A YOLOv8n-shaped layer mix at 640x640, 20 layers, 8 of them 1x1.

    Stride-2 3x3 stem/downsample convs 3(->4)->16->32->64->128->256, and per
    stage C in {32@160, 64@80, 128@40, 256@20} two 1x1 C->C convs plus 3x3
    stride-1 C/2->C/2 convs (one at 160, two elsewhere).  The 3-channel input
    is zero-padded to 4 channels."""
    layers: list[Layer] = []
    i = 0
    down = [(4, 16, 640), (16, 32, 320), (32, 64, 160), (64, 128, 80), (128, 256, 40)]
    for ci, co, h in down:
        layers.append(Layer(f"yolov8n_l{i:02d}_3x3s2_{ci}to{co}_{h}px", N, ci, co, h, h, 3, 2, 1,
                            "nvfp6", "silu", 1e-4, i, cin_real=3 if i == 0 else 0))
        i += 1
    for C, h, n3 in [(32, 160, 1), (64, 80, 2), (128, 40, 2), (256, 20, 2)]:
        for _ in range(2):
            layers.append(Layer(f"yolov8n_l{i:02d}_1x1_{C}_{h}px", N, C, C, h, h, 1, 1, 0,
                                "nvfp6", "silu", 1e-4, i))
            i += 1
        for _ in range(n3):
            layers.append(Layer(f"yolov8n_l{i:02d}_3x3_{C // 2}_{h}px", N, C // 2, C // 2, h, h,
                                3, 1, 1, "nvfp6", "silu", 1e-4, i))
            i += 1
    return layers


# Quantize-only sweep: (C, H = W, N) of the latent-replay buffer case.
REPLAY_SHAPES = [(256, 7, 84), (512, 7, 256), (256, 14, 256), (512, 14, 256),
                 (512, 14, 2560), (512, 14, 10240)]


# Depthwise 3x3 layers kept in BF16 (the YOLOv26n-style stages at 640 px
# input, batch 16): (C, H = W, stride); stride-2 layers halve the pixels.
DEPTHWISE_SHAPES = [(32, 160, 1), (64, 160, 2), (64, 80, 1), (128, 80, 2), (128, 40, 1),
                    (256, 40, 2), (256, 20, 1)]
DEPTHWISE_N = 16


def make_depthwise_inputs(C: int, H: int, stride: int, N: int = DEPTHWISE_N, seed: int = 0, device="cpu"):
    """(x [H][H][C][N], w [C][3][3], gy [Ho][Ho][C][N]) fp32: x = SiLU(N(0,1)),
    w ~ N(0, 2/9) (one 3x3 filter per channel), gy ~ N(0, 1e-4)."""
    g = _gen(seed, device)
    ho = (H + 2 - 3) // stride + 1
    x = torch.nn.functional.silu(torch.randn((H, H, C, N), generator=g, device=device))
    w = torch.randn((C, 3, 3), generator=g, device=device) * math.sqrt(2.0 / 9.0)
    gy = torch.randn((ho, ho, C, N), generator=g, device=device) * 1e-4
    return x, w, gy


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_layer_inputs(layer: Layer, device="cpu"):
    """(X, W, G_Y) fp32 tensors in the channel-batch-first layouts.

    X: N(0,1) passed through the layer's activation (ReLU: half-normal,
    SiLU), W: Kaiming-normal, std sqrt(2 / (Cin·Kh·Kw)), G_Y: N(0, gy_std)."""
    g = _gen(layer.seed, device)
    cin_real = layer.cin_real or layer.Cin
    X = torch.randn((layer.H, layer.W, cin_real, layer.N), generator=g, device=device)
    if layer.x_dist == "relu":
        X = torch.relu(X)
    elif layer.x_dist == "silu":
        X = torch.nn.functional.silu(X)
    std = math.sqrt(2.0 / (cin_real * layer.K * layer.K))
    Wt = torch.randn((layer.Cout, layer.K, layer.K, cin_real), generator=g, device=device) * std
    GY = torch.randn((layer.Ho, layer.Wo, layer.Cout, layer.N), generator=g, device=device) * layer.gy_std
    if cin_real != layer.Cin:
        pad = layer.Cin - cin_real
        X = torch.cat([X, X.new_zeros((layer.H, layer.W, pad, layer.N))], dim=2)
        Wt = torch.cat([Wt, Wt.new_zeros((layer.Cout, layer.K, layer.K, pad))], dim=3)
    return X.contiguous(), Wt.contiguous(), GY.contiguous()


def make_replay_input(C: int, H: int, N: int, signed: bool = False, outliers: bool = False,
                      seed: int = 0, device="cpu") -> torch.Tensor:
    """Latent-replay activations [H][H][C][N]: |N(0,1)| (post-ReLU latents),
    or signed N(0,1); with outliers, 0.1% of the entries (a seeded random
    choice) are multiplied by 100."""
    g = _gen(seed, device)
    x = torch.randn((H, H, C, N), generator=g, device=device)
    if not signed:
        x = x.abs()
    if outliers:
        n = x.numel()
        k = max(1, n // 1000)
        idx = torch.randint(0, n, (k,), generator=g, device=device)
        x.view(-1)[idx] *= 100.0
    return x


def sr_seed(layer: Layer) -> int:
    """Seed of the stochastic rounding of a layer's G_Y."""
    return 1000 * layer.seed + 7
