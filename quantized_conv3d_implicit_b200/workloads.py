"""Seeded synthetic workloads for the Conv3D implicit GEMM.

This module only draws inputs: shapes, seeds and value distributions.  It
holds none of the method's arithmetic, so both the CUDA path and the CPU
oracle can be fed from it.

The shapes stand in for the Wan2.2 VAE Conv3D layers the Model-Optimizer
"Conv3D Implicit GEMM CUDA kernel" article targets (sections 1 and 10); no
model weights or videos are used.  Recipe per workload:
  x ~ N(0, 1) (cast to the workload dtype), optional outliers (a seeded
  Bernoulli mask of the stated fraction multiplied by the stated factor);
  w ~ N(0, 1/sqrt(K)) with K = Cin*kd*kh*kw; bias ~ N(0, sigma) or none;
  act_amax = max|x| (after outliers) as a float32 scalar.
Random numbers come from torch.Generator seeded per workload, drawn in
float32 on the requested device and then cast.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import torch

Triple = Tuple[int, int, int]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: torch.dtype
    x_shape: Tuple[int, int, int, int, int]     # N, Cin, D, H, W
    cout: int
    kernel: Triple                              # kd, kh, kw
    stride: Triple = (1, 1, 1)
    pad_lo: Triple = (1, 1, 1)
    pad_hi: Triple = (1, 1, 1)
    dil: Triple = (1, 1, 1)
    quant_act: bool = True
    bias_sigma: Optional[float] = None
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    seed: int = 0

    @property
    def k_gemm(self) -> int:
        return self.x_shape[1] * self.kernel[0] * self.kernel[1] * self.kernel[2]

    def out_spatial(self) -> Triple:
        dims = []
        for i in range(3):
            span = self.x_shape[2 + i] + self.pad_lo[i] + self.pad_hi[i] - self.dil[i] * (self.kernel[i] - 1) - 1
            dims.append(span // self.stride[i] + 1 if span >= 0 else 0)
        return tuple(dims)

    @property
    def m_gemm(self) -> int:
        od, oh, ow = self.out_spatial()
        return self.x_shape[0] * od * oh * ow

    @property
    def flops(self) -> int:
        """2*M*Cout*K, the metric's operation count."""
        return 2 * self.m_gemm * self.cout * self.k_gemm

    def out_shape(self):
        return (self.x_shape[0], self.cout) + tuple(self.out_spatial())


_CAUSAL = dict(pad_lo=(2, 1, 1), pad_hi=(0, 1, 1))

WORKLOADS = {
    # small case: fp32, 16 -> 16 channels, 3x3x3, pad 1, seed 0
    "tiny_16x16_fp32": Workload("tiny_16x16_fp32", torch.float32, (1, 16, 4, 16, 16), 16, (3, 3, 3),
                                bias_sigma=0.1, seed=0),
    # Wan-VAE-like mid-resolution block conv, 384 -> 384, causal temporal pad
    "wan_mid_384_bf16": Workload("wan_mid_384_bf16", torch.bfloat16, (1, 384, 5, 60, 104), 384, (3, 3, 3),
                                 bias_sigma=0.02, seed=1, **_CAUSAL),
    # Wan-VAE-like high-resolution decoder conv, 192 -> 192, 0.1% outliers x20
    "wan_hi_192_bf16": Workload("wan_hi_192_bf16", torch.bfloat16, (1, 192, 9, 240, 416), 192, (3, 3, 3),
                                outlier_frac=1e-3, outlier_scale=20.0, seed=2, **_CAUSAL),
    "wan_hi_192_bf16_noquant": Workload("wan_hi_192_bf16_noquant", torch.bfloat16, (1, 192, 9, 240, 416), 192,
                                        (3, 3, 3), quant_act=False, outlier_frac=1e-3, outlier_scale=20.0,
                                        seed=2, **_CAUSAL),
    # strided downsample conv, fp16, stride (1,2,2)
    "down_s122_128to256_fp16": Workload("down_s122_128to256_fp16", torch.float16, (2, 128, 17, 256, 256), 256,
                                        (3, 3, 3), stride=(1, 2, 2), seed=3),
    # pointwise 1x1x1 conv, fp16, 512 -> 1024
    "pointwise_512to1024_fp16": Workload("pointwise_512to1024_fp16", torch.float16, (2, 512, 5, 64, 64), 1024,
                                         (1, 1, 1), pad_lo=(0, 0, 0), pad_hi=(0, 0, 0), seed=4),
    # full-resolution edge conv, 96 -> 96, causal temporal pad
    "edge_full_96_bf16": Workload("edge_full_96_bf16", torch.bfloat16, (1, 96, 17, 480, 832), 96, (3, 3, 3),
                                  seed=5, **_CAUSAL),
    # same with spatial dilation 2 (spatial pad stays 1)
    "edge_full_96_bf16_dil122": Workload("edge_full_96_bf16_dil122", torch.bfloat16, (1, 96, 17, 480, 832), 96,
                                         (3, 3, 3), dil=(1, 2, 2), seed=5, **_CAUSAL),
}

# the five configurations in order (the third and fourth have two entries)
SMALL = "tiny_16x16_fp32"
# the largest single-GPU layer: the benchmark's default workload
HEADLINE = "edge_full_96_bf16"

# Fewer-frame copies of the full-resolution layers: the same spatial extent,
# hence the same tiling plan and per-tile work, with a smaller input, for
# profiler captures that must hold only a few GB on the device.
CROPS = {
    "edge_full_96_bf16_d5": dataclasses.replace(WORKLOADS["edge_full_96_bf16"], name="edge_full_96_bf16_d5",
                                                x_shape=(1, 96, 5, 480, 832)),
}


def get(name: str) -> Workload:
    """A workload or crop by name."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    return CROPS[name]


def make_inputs(wl: Workload | str, device="cpu", with_out: bool = False):
    """Draw the seeded inputs of a workload on `device`.

    Returns dict(x, w, bias, act_amax) (+ out, an uninitialised output tensor
    when with_out).  act_amax is a float32 tensor of shape [1].
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    x = torch.randn(wl.x_shape, generator=gen, device=dev, dtype=torch.float32)
    if wl.outlier_frac > 0:
        mask = torch.rand(wl.x_shape, generator=gen, device=dev, dtype=torch.float32) < wl.outlier_frac
        x = torch.where(mask, x * wl.outlier_scale, x)
        del mask
    x = x.to(wl.dtype)
    cin = wl.x_shape[1]
    w = torch.randn((wl.cout, cin) + tuple(wl.kernel), generator=gen, device=dev, dtype=torch.float32)
    w = (w * (1.0 / math.sqrt(wl.k_gemm))).to(wl.dtype)
    bias = None
    if wl.bias_sigma is not None:
        bias = (torch.randn((wl.cout,), generator=gen, device=dev, dtype=torch.float32) * wl.bias_sigma).to(wl.dtype)
    act_amax = x.abs().max().to(torch.float32).reshape(1)
    d = dict(x=x, w=w, bias=bias, act_amax=act_amax)
    if with_out:
        d["out"] = torch.empty(wl.out_shape(), dtype=wl.dtype, device=dev)
    return d


def random_conv_inputs(seed: int, x_shape, cout: int, kernel, dtype=torch.float32, bias: bool = True,
                       device="cpu", scale: float = 1.0):
    """Generic seeded inputs for parity sweeps over arbitrary shapes."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    x = (torch.randn(tuple(x_shape), generator=gen, device=dev) * scale).to(dtype)
    k = x_shape[1] * kernel[0] * kernel[1] * kernel[2]
    w = (torch.randn((cout, x_shape[1]) + tuple(kernel), generator=gen, device=dev) / math.sqrt(k)).to(dtype)
    b = (torch.randn((cout,), generator=gen, device=dev) * 0.1).to(dtype) if bias else None
    amax = x.abs().max().to(torch.float32).reshape(1)
    return dict(x=x, w=w, bias=b, act_amax=amax)
