"""GPU parity: the library (through the C ABI) against the CPU oracle.

Grid in the spirit of the cross-check of "Use the explicit gemm for wide
convs on neural accelerators" (Verified: filter 1/3/5/7, stride 1/2, padding
0/1/2, dilation 1/2, aligned and unaligned channels, two batch shapes), every
dtype, every algorithm and engine, plus shapes that span several GEMM tiles
with ragged tails, and the named workloads (sampled where the oracle cannot
do the full tensor).  Output buffers are NaN-poisoned so an unwritten element
fails.
"""
import itertools

import pytest
import torch

from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import check_conv2d

pytestmark = pytest.mark.gpu

GRID = []
for k, s, p, d in itertools.product([1, 3, 5, 7], [1, 2], [0, 1, 2], [1, 2]):
    for (c, o) in [(16, 24), (13, 21)]:
        for n, hw in [(1, 11), (3, 9)]:
            if hw + 2 * p - d * (k - 1) - 1 < 0:
                continue
            GRID.append(synth.Conv2dShape(n, hw, hw + 1, c, o, k, k, (s, s), (p, p), (d, d)))


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_grid_auto(dtype):
    worst = 0.0
    for shape in GRID:
        worst = max(worst, check_conv2d(shape, dtype))
    print(f"{dtype}: worst rel err over {len(GRID)} shapes = {worst:.3e}")


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("algo", ["implicit", "direct"])
def test_grid_forced(dtype, algo):
    for shape in GRID[::5]:
        check_conv2d(shape, dtype, options=B.make_options(algo))


MULTI_TILE = [
    # several 128-row tiles with a ragged tail; O spanning 256-wide tiles with a tail
    synth.Conv2dShape(3, 23, 23, 72, 300, 3, 3, (1, 1), (1, 1), (1, 1)),
    synth.Conv2dShape(2, 31, 17, 136, 129, 3, 3, (2, 1), (1, 1), (1, 2)),
    # asymmetric kernel / stride / pad / dilation
    synth.Conv2dShape(2, 19, 27, 64, 96, 3, 5, (1, 2), (1, 2), (2, 1)),
    synth.Conv2dShape(1, 40, 33, 48, 64, 5, 3, (2, 1), (0, 2), (1, 3)),
    # 1x1 stride-2 projection and a C = 3 stem (channel pad pre-pass)
    synth.Conv2dShape(2, 28, 28, 256, 512, 1, 1, (2, 2), (0, 0), (1, 1)),
    synth.Conv2dShape(2, 64, 64, 3, 64, 7, 7, (2, 2), (3, 3), (1, 1)),
    # wide K, small M
    synth.Conv2dShape(1, 7, 7, 512, 512, 3, 3, (1, 1), (1, 1), (1, 1)),
    # unaligned channel counts of the sweep
    synth.Conv2dShape(1, 16, 16, 130, 1030, 3, 3, (1, 1), (1, 1), (1, 1)),
    synth.Conv2dShape(1, 16, 16, 256, 129, 5, 5, (1, 1), (2, 2), (1, 1)),
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", MULTI_TILE, ids=lambda s: s.name())
def test_multi_tile(shape, dtype):
    check_conv2d(shape, dtype)


# Few-channel inputs with every tap folded into channels (KH*KW*C <= 192): the
# conv runs as a 1x1 conv over the packed channels.  Strides, padding,
# dilation, rectangular windows and C from 1 to 7.
FULLPACK = [
    synth.Conv2dShape(2, 30, 31, 3, 64, 7, 7, (2, 2), (3, 3), (1, 1)),
    synth.Conv2dShape(1, 17, 19, 1, 40, 3, 3, (1, 1), (1, 1), (2, 2)),
    synth.Conv2dShape(2, 20, 20, 5, 24, 5, 5, (2, 2), (2, 2), (1, 1)),
    synth.Conv2dShape(1, 9, 33, 2, 8, 3, 5, (1, 2), (1, 2), (2, 1)),
    synth.Conv2dShape(3, 12, 12, 7, 16, 1, 3, (1, 1), (0, 1), (1, 1)),
    # packing staged in 128-pixel row segments: 300 output columns end in a ragged 44
    synth.Conv2dShape(1, 5, 300, 3, 16, 3, 3, (1, 1), (1, 1), (1, 1)),
    # 32 staged input rows of (127*8 + 128 + 1) values overflow 48 KB: 64-pixel segments
    synth.Conv2dShape(1, 40, 921, 1, 16, 32, 2, (1, 8), (0, 0), (1, 128)),
    # 96 rows of 257 values exceed 48 KB even for one pixel: the unstaged packing kernel
    synth.Conv2dShape(1, 100, 20, 1, 8, 96, 2, (1, 1), (0, 128), (1, 256)),
]


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("shape", FULLPACK, ids=lambda s: s.name())
def test_full_tap_packing(shape, dtype):
    d = B.make_desc2d(shape.n, shape.h, shape.w, shape.c, shape.o, shape.kh, shape.kw, shape.stride, shape.pad,
                      shape.dilation)
    assert B.plan2d(d, dtype, 0, None)["packed_taps"] == 2
    check_conv2d(shape, dtype)


WINO = [
    synth.Conv2dShape(2, 20, 20, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1)),     # ragged 6x6 tiles
    synth.Conv2dShape(3, 13, 29, 32, 64, 3, 3, (1, 1), (0, 0), (1, 1)),     # no padding
    synth.Conv2dShape(1, 9, 9, 24, 40, 3, 3, (1, 1), (2, 1), (1, 1)),       # C % 8 == 0, odd pads
    synth.Conv2dShape(2, 12, 12, 13, 17, 3, 3, (1, 1), (1, 1), (1, 1)),     # C % 8 != 0
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("shape", WINO, ids=lambda s: s.name())
def test_winograd_forced(shape, dtype):
    check_conv2d(shape, dtype, options=B.make_options("winograd"))


def test_small_f32_workload():
    """N=2, 16x16, 32->32, 3x3, pad 1, uniform inputs: the full tensor."""
    check_conv2d(synth.SMALL_F32, "f32", dist="uniform")


def test_tf32_is_never_used():
    """A 1x1 conv with C = 1 and x = w = 1 + 2^-11: the exact product
    1 + 2^-10 + 2^-22 is representable in fp32 but not after TF32's 10-bit
    mantissa truncation of the operands (which would give 1 + 2^-10)."""
    v = 1.0 + 2.0 ** -11
    x = torch.full((1, 4, 4, 1), v, dtype=torch.float32, device="cuda")
    w = torch.full((1, 1, 1, 1), v, dtype=torch.float32, device="cuda")
    for algo in ("auto", "implicit", "direct"):
        out = B.conv2d(x, w, options=B.make_options(algo))
        assert torch.all(out == torch.tensor(v * v, dtype=torch.float32)).item(), algo


@pytest.mark.parametrize("batch", [1, 8])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_resnet50_layers(batch, dtype):
    worst = 0.0
    for name, shape, _ in synth.resnet50_layers(batch):
        worst = max(worst, check_conv2d(shape, dtype, dist="he", sample=4096))
    print(f"resnet50 b{batch} {dtype}: worst {worst:.3e}")


# Config-4 coverage: every (filter, C_in) x C_out x (stride, dilation)
# combination of the wide-channel sweep once per dtype, at the sweep's largest
# M (N = 16, 64x64 outputs), on >= 4096 seeded output pixels; and the whole
# unaligned subset.  Grouped by (k, C_in) so a failure names its group.
SWEEP_M_MAX = [s for s in synth.wide_sweep(True) if s.n == 16]
SWEEP_GROUPS = sorted({(s.kh, s.c) for s in SWEEP_M_MAX})


def test_sweep_coverage_is_complete():
    combos = {(s.kh, s.c, s.o, s.stride, s.dilation) for s in SWEEP_M_MAX}
    assert len(combos) == len(SWEEP_M_MAX) == 7 * 6 * 4
    assert all(s.n * s.oh * s.ow == 65536 for s in SWEEP_M_MAX)
    assert len(synth.wide_sweep(False)) == 48


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("group", SWEEP_GROUPS, ids=lambda g: f"k{g[0]}_c{g[1]}")
def test_wide_sweep_every_combination(group, dtype):
    worst = 0.0
    for shape in SWEEP_M_MAX:
        if (shape.kh, shape.c) == group:
            worst = max(worst, check_conv2d(shape, dtype, sample=4096))
    print(f"k{group[0]} C={group[1]} {dtype}: worst {worst:.3e}")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_wide_sweep_unaligned(dtype):
    for shape in synth.wide_sweep(False):
        check_conv2d(shape, dtype, sample=4096)


CONV1D = [
    # Whisper-encoder-style pair (the implicit-GEMM page's conv1d follow-up): 80 -> 384, then stride 2
    (1, 3000, 80, 384, 3, 1, 1, 1),
    (1, 3000, 384, 384, 3, 2, 1, 1),
    (3, 97, 13, 21, 5, 2, 2, 2),      # ragged, unaligned channels, dilation
]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("case", CONV1D, ids=str)
def test_conv1d_through_the_2d_path(case, dtype):
    import numpy as np
    import oracle
    from tests.gpu_util import as_f64, assert_close
    n, l, c, o, k, s, p, d = case
    x, w = synth.make_inputs((n, l, c), (o, k, c), dtype, "normal", 11, device="cuda")
    out = B.conv1d(x, w, s, p, d)
    torch.cuda.synchronize()
    ref = oracle.conv2d(x.cpu().reshape(n, 1, l, c), w.cpu().reshape(o, 1, k, c), dtype, (1, s), (0, p), (1, d))
    assert_close(as_f64(out), ref.reshape(out.shape), dtype, f"conv1d {case}")
