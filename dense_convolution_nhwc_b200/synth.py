"""Seeded synthetic inputs and the named workloads.

This module holds no convolution arithmetic: it only draws seeded random
tensors with the distributions and shapes of the workloads below, so the GPU
library, its tests and the CPU oracle all see the same bits.  Inputs are drawn
with ``torch.Generator`` on the requested device (seed for activations,
seed + 1 for weights) and cast to the storage dtype.

Workloads (shapes and distributions of the three MLX pull requests' measured
cases, made concrete):

* ``small_f32``: N=2, 16x16, 32->32, 3x3, stride 1, pad 1 (uniform inputs).
* ``winograd_f32``: N=40, 512x512, 192->96, 3x3, stride 1, pad 1 -- the shape
  of "Bound winograd conv2d working set by tiling the batch" (Testing and the
  reviewer's batch sweep).
* ``resnet50``: the ResNet-50 v1.5 conv layer set at 224x224 -- the model the
  "Use the explicit gemm for wide convs on neural accelerators" page times.
* ``wide_sweep``: 3x3/5x5/7x7 filters, stride 1/2, dilation 1/2,
  C_in 128..1024 (K = C*k*k from 1152 to 9216), C_out 128..4096,
  M = N*OH*OW from 1024 to 65536 -- the axes of that page's C_out table.
* ``conv3d_taps``: 3x3x3 NDHWC bf16 convs 17x64x64 256->256,
  41x60x104 256->256, 41x120x208 512->512 -- the cases of "Decompose small
  kernel-depth 3D convs into 2D convs" (Results).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Conv2dShape:
    n: int
    h: int
    w: int
    c: int
    o: int
    kh: int
    kw: int
    stride: Tuple[int, int] = (1, 1)
    pad: Tuple[int, int] = (0, 0)
    dilation: Tuple[int, int] = (1, 1)

    @property
    def oh(self) -> int:
        return (self.h + 2 * self.pad[0] - self.dilation[0] * (self.kh - 1) - 1) // self.stride[0] + 1

    @property
    def ow(self) -> int:
        return (self.w + 2 * self.pad[1] - self.dilation[1] * (self.kw - 1) - 1) // self.stride[1] + 1

    @property
    def flops(self) -> int:
        """Direct-equivalent FLOPs, 2*N*OH*OW*O*C*KH*KW."""
        return 2 * self.n * self.oh * self.ow * self.o * self.c * self.kh * self.kw

    def name(self) -> str:
        return (f"n{self.n}_{self.h}x{self.w}_{self.c}to{self.o}_k{self.kh}x{self.kw}"
                f"_s{self.stride[0]}{self.stride[1]}_p{self.pad[0]}{self.pad[1]}"
                f"_d{self.dilation[0]}{self.dilation[1]}")


@dataclass(frozen=True)
class Conv3dShape:
    n: int
    d: int
    h: int
    w: int
    c: int
    o: int
    kd: int
    kh: int
    kw: int
    stride: Tuple[int, int, int] = (1, 1, 1)
    pad: Tuple[int, int, int] = (0, 0, 0)
    dilation: Tuple[int, int, int] = (1, 1, 1)

    def _out(self, i, k, s, p, d):
        return (i + 2 * p - d * (k - 1) - 1) // s + 1

    @property
    def od(self) -> int:
        return self._out(self.d, self.kd, self.stride[0], self.pad[0], self.dilation[0])

    @property
    def oh(self) -> int:
        return self._out(self.h, self.kh, self.stride[1], self.pad[1], self.dilation[1])

    @property
    def ow(self) -> int:
        return self._out(self.w, self.kw, self.stride[2], self.pad[2], self.dilation[2])

    @property
    def flops(self) -> int:
        return 2 * self.n * self.od * self.oh * self.ow * self.o * self.c * self.kd * self.kh * self.kw

    def name(self) -> str:
        return (f"n{self.n}_{self.d}x{self.h}x{self.w}_{self.c}to{self.o}_k{self.kd}{self.kh}{self.kw}"
                f"_s{''.join(map(str, self.stride))}_p{''.join(map(str, self.pad))}"
                f"_d{''.join(map(str, self.dilation))}")


# ---------------------------------------------------------------------------
# Named workloads
# ---------------------------------------------------------------------------

SMALL_F32 = Conv2dShape(2, 16, 16, 32, 32, 3, 3, (1, 1), (1, 1), (1, 1))
WINOGRAD_F32 = Conv2dShape(40, 512, 512, 192, 96, 3, 3, (1, 1), (1, 1), (1, 1))
# The tiny shape of the same page: 1-element Winograd tiles lose to implicit GEMM.
TINY_WINOGRAD = Conv2dShape(256, 4, 4, 64, 192, 3, 3, (1, 1), (1, 1), (1, 1))


def resnet50_layers(batch: int) -> List[Tuple[str, Conv2dShape, int]]:
    """ResNet-50 v1.5 conv layers at 224x224: (name, shape, repeat count).

    Bottleneck blocks 3/4/6/3 with widths 64/128/256/512 and outputs
    256/512/1024/2048; the stride sits on the 3x3 of each stage's first block,
    whose 1x1 projection has the same stride.
    """
    L: List[Tuple[str, Conv2dShape, int]] = []

    def add(name, h, c, o, k, s, p, count):
        L.append((name, Conv2dShape(batch, h, h, c, o, k, k, (s, s), (p, p), (1, 1)), count))

    add("stem", 224, 3, 64, 7, 2, 3, 1)
    # layer1 at 56x56 (after the stem and max-pool)
    add("l1.a1x1.first", 56, 64, 64, 1, 1, 0, 1)
    add("l1.a1x1", 56, 256, 64, 1, 1, 0, 2)
    add("l1.b3x3", 56, 64, 64, 3, 1, 1, 3)
    add("l1.c1x1", 56, 64, 256, 1, 1, 0, 3)
    add("l1.proj", 56, 64, 256, 1, 1, 0, 1)
    # layer2
    add("l2.a1x1.first", 56, 256, 128, 1, 1, 0, 1)
    add("l2.b3x3.s2", 56, 128, 128, 3, 2, 1, 1)
    add("l2.proj.s2", 56, 256, 512, 1, 2, 0, 1)
    add("l2.a1x1", 28, 512, 128, 1, 1, 0, 3)
    add("l2.b3x3", 28, 128, 128, 3, 1, 1, 3)
    add("l2.c1x1", 28, 128, 512, 1, 1, 0, 4)
    # layer3
    add("l3.a1x1.first", 28, 512, 256, 1, 1, 0, 1)
    add("l3.b3x3.s2", 28, 256, 256, 3, 2, 1, 1)
    add("l3.proj.s2", 28, 512, 1024, 1, 2, 0, 1)
    add("l3.a1x1", 14, 1024, 256, 1, 1, 0, 5)
    add("l3.b3x3", 14, 256, 256, 3, 1, 1, 5)
    add("l3.c1x1", 14, 256, 1024, 1, 1, 0, 6)
    # layer4
    add("l4.a1x1.first", 14, 1024, 512, 1, 1, 0, 1)
    add("l4.b3x3.s2", 14, 512, 512, 3, 2, 1, 1)
    add("l4.proj.s2", 14, 1024, 2048, 1, 2, 0, 1)
    add("l4.a1x1", 7, 2048, 512, 1, 1, 0, 2)
    add("l4.b3x3", 7, 512, 512, 3, 1, 1, 2)
    add("l4.c1x1", 7, 512, 2048, 1, 1, 0, 3)
    return L


def wide_sweep(aligned: bool = True) -> List[Conv2dShape]:
    """The wide-channel implicit-GEMM grid: (k, C) with K = C*k*k in [1152, 9216],
    stride {1,2} x dilation {1,2} with "same" padding, C_out in 128..4096 and
    M = N*OH*OW in {1024, 4096, 16384, 65536}; or the unaligned subset."""
    out: List[Conv2dShape] = []
    m_cases = [(1, 32), (4, 32), (4, 64), (16, 64)]
    if aligned:
        kc = [(3, 128), (3, 256), (3, 512), (3, 1024), (5, 128), (5, 256), (7, 128)]
        couts = [128, 256, 512, 1024, 2048, 4096]
    else:
        kc = None
        m_cases = [(1, 32), (4, 64)]
    for s in (1, 2):
        for d in (1, 2):
            for (nb, ohw) in m_cases:
                if aligned:
                    for (k, c) in kc:
                        for o in couts:
                            p = d * (k - 1) // 2
                            h = s * ohw
                            out.append(Conv2dShape(nb, h, h, c, o, k, k, (s, s), (p, p), (d, d)))
                else:
                    for (c, o) in [(136, 520), (130, 1030), (256, 129)]:
                        for k in (3, 5):
                            p = d * (k - 1) // 2
                            h = s * ohw
                            out.append(Conv2dShape(nb, h, h, c, o, k, k, (s, s), (p, p), (d, d)))
    return out


CONV3D_TAPS = [
    Conv3dShape(1, 17, 64, 64, 256, 256, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
    Conv3dShape(1, 41, 60, 104, 256, 256, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
    Conv3dShape(1, 41, 120, 208, 512, 512, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
]


# ---------------------------------------------------------------------------
# Seeded tensors
# ---------------------------------------------------------------------------

def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_inputs(x_shape, w_shape, dtype: str, dist: str, seed: int = 0, device="cpu"):
    """Seeded activations and weights.

    dist:
      "uniform"  -- x ~ U[-1,1], w ~ U[-1,1] / sqrt(fan_in)
      "normal"   -- x ~ N(0,1), w ~ N(0, 1/fan_in)
      "he"       -- x ~ N(0,1), w ~ N(0, 2/fan_in)
      "int"      -- small integers in [-4, 4] for both (exact in every dtype)
    fan_in is the product of w_shape[1:] (KH*KW*C, or KD*KH*KW*C).
    """
    device = torch.device(device)
    fan_in = int(math.prod(w_shape[1:]))
    gx, gw = _gen(device, seed), _gen(device, seed + 1)
    t = TORCH_DTYPES[dtype]
    if dist == "uniform":
        x = torch.rand(x_shape, generator=gx, device=device, dtype=torch.float32).mul_(2).sub_(1)
        w = torch.rand(w_shape, generator=gw, device=device, dtype=torch.float32).mul_(2).sub_(1)
        w.div_(math.sqrt(fan_in))
    elif dist in ("normal", "he"):
        x = torch.randn(x_shape, generator=gx, device=device, dtype=torch.float32)
        w = torch.randn(w_shape, generator=gw, device=device, dtype=torch.float32)
        w.mul_(math.sqrt((2.0 if dist == "he" else 1.0) / fan_in))
    elif dist == "int":
        x = torch.randint(-4, 5, x_shape, generator=gx, device=device).to(torch.float32)
        w = torch.randint(-4, 5, w_shape, generator=gw, device=device).to(torch.float32)
    else:
        raise ValueError(dist)
    return x.to(t).contiguous(), w.to(t).contiguous()


def conv2d_inputs(s: Conv2dShape, dtype: str, dist: str, seed: int = 0, device="cpu"):
    return make_inputs((s.n, s.h, s.w, s.c), (s.o, s.kh, s.kw, s.c), dtype, dist, seed, device)


def conv3d_inputs(s: Conv3dShape, dtype: str, dist: str, seed: int = 0, device="cpu"):
    return make_inputs((s.n, s.d, s.h, s.w, s.c), (s.o, s.kd, s.kh, s.kw, s.c), dtype, dist, seed, device)


def sample_pixels(n: int, oh: int, ow: int, count: int = 4096, seed: int = 0, od: Optional[int] = None):
    """Seeded output-pixel sample: uniform without replacement, plus the four
    corners and one full edge row and column of the first and last image.

    Returns an int32 tensor [P,3] of (n, oh, ow), or [P,4] of (n, od, oh, ow)
    when od is given (edges then taken on the first and last frame).
    """
    frames = 1 if od is None else od
    total = n * frames * oh * ow
    g = torch.Generator().manual_seed(seed)
    want = min(count, total)
    idx = torch.randperm(total, generator=g)[:want] if total > want else torch.arange(total)
    extra = []
    for nn in sorted({0, n - 1}):
        for ff in sorted({0, frames - 1}):
            base = (nn * frames + ff) * oh * ow
            for y in range(oh):
                extra.append(base + y * ow + 0)
                extra.append(base + y * ow + ow - 1)
            for x in range(ow):
                extra.append(base + 0 * ow + x)
                extra.append(base + (oh - 1) * ow + x)
    idx = torch.unique(torch.cat([idx, torch.tensor(extra, dtype=torch.int64)]))
    x_ = idx % ow
    r = idx // ow
    y_ = r % oh
    r = r // oh
    f_ = r % frames
    n_ = r // frames
    if od is None:
        return torch.stack([n_, y_, x_], 1).to(torch.int32)
    return torch.stack([n_, f_, y_, x_], 1).to(torch.int32)
