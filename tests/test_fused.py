"""The persistent fp32 Winograd kernel against the three-launch path and the oracle.

The Winograd path ("Bound winograd conv2d working set by tiling the batch",
Problem and Fix: input transform, batched GEMM, output transform) can run as
one persistent kernel whose CTAs each take blocks of 128 tiles and overlap the
input transform of the next block and the output transform of the previous one
with the GEMM of the current one.  Every tile is transformed on its own and
every GEMM output reduces over the channels in one fixed order, so the result
must equal the three-launch path bit for bit whatever the grid, and match the
oracle.

B200CONV_WINOGRAD_FUSED=0/1 (read on every call) turns the persistent kernel
off/on; B200CONV_WINOGRAD_FUSED_GRID runs it on fewer CTAs, so that each CTA
takes many blocks and reuses its two V and two M buffers (every mbarrier phase
of the hand-over between its warpgroups).
"""
import os

import pytest
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import as_f64, assert_close, run_conv2d

pytestmark = pytest.mark.gpu


class env:
    def __init__(self, **kv):
        self.kv = {k: str(v) for k, v in kv.items()}

    def __enter__(self):
        self.old = {k: os.environ.get(k) for k in self.kv}
        os.environ.update(self.kv)

    def __exit__(self, *a):
        for k, v in self.old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def _bits(t):
    return t.view(torch.int32)


def _plan(s, opts):
    d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
    return B.plan2d(d, "f32", 0, opts)


def _tiles(s):
    return s.n * ((s.oh + 5) // 6) * ((s.ow + 5) // 6)


CASES = [
    # 7 x 6 tiles per image: 126 tiles, one ragged block
    synth.Conv2dShape(3, 40, 36, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1)),
    # no padding, ragged edge tiles, O = 160: two 128-wide column blocks, the second ragged
    synth.Conv2dShape(2, 47, 29, 32, 160, 3, 3, (1, 1), (0, 0), (1, 1)),
    # 1088 tiles = 9 blocks (the last of 64 tiles); C = 48 leaves a ragged 16-wide k slice
    synth.Conv2dShape(4, 96, 100, 48, 64, 3, 3, (1, 1), (1, 1), (1, 1)),
    # C % 64 != 0 (32-channel transform blocks), O = 40 (a partial 32-channel output group)
    synth.Conv2dShape(2, 64, 64, 36, 40, 3, 3, (1, 1), (1, 1), (1, 1)),
    # O % 4 != 0: M rows written element by element
    synth.Conv2dShape(1, 30, 30, 32, 42, 3, 3, (1, 1), (1, 1), (1, 1)),
    # asymmetric padding
    synth.Conv2dShape(2, 50, 44, 64, 96, 3, 3, (1, 1), (2, 0), (1, 1)),
]


@pytest.mark.parametrize("shape", CASES, ids=lambda s: s.name())
def test_fused_equals_three_launches_bit_for_bit(shape):
    opts = B.make_options("winograd")
    x, w = synth.conv2d_inputs(shape, "f32", "normal", 31, device="cuda")
    with env(B200CONV_WINOGRAD_FUSED=0):
        p0 = _plan(shape, opts)
        assert p0["algo"] == "winograd" and p0["winograd_fused"] == 0
        ref = run_conv2d(x, w, shape, opts)
    want = oracle.conv2d(x.cpu(), w.cpu(), "f32", shape.stride, shape.pad, shape.dilation)
    assert_close(as_f64(ref), want, "f32", shape.name())
    blocks = -(-_tiles(shape) // 128)
    for grid in sorted({1, 2, 3, max(1, blocks // 2), 148}):
        with env(B200CONV_WINOGRAD_FUSED=1, B200CONV_WINOGRAD_FUSED_GRID=grid):
            p = _plan(shape, opts)
            assert p["winograd_fused"] == 1 and p["num_batch_tiles"] == 1
            got = run_conv2d(x, w, shape, opts)
        assert torch.equal(_bits(got), _bits(ref)), f"grid {grid}"


def test_fused_many_blocks_per_cta_against_oracle():
    """Eight images of 128 x 128 (3872 tiles, 31 blocks) on 2 CTAs: 15 and 16
    blocks each, both buffers reused seven times."""
    s = synth.Conv2dShape(8, 128, 128, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1))
    opts = B.make_options("winograd")
    x, w = synth.conv2d_inputs(s, "f32", "normal", 32, device="cuda")
    with env(B200CONV_WINOGRAD_FUSED=0):
        ref = run_conv2d(x, w, s, opts)
    with env(B200CONV_WINOGRAD_FUSED=1, B200CONV_WINOGRAD_FUSED_GRID=2):
        got = run_conv2d(x, w, s, opts)
    assert torch.equal(_bits(got), _bits(ref))
    want = oracle.conv2d(x[:2].cpu(), w.cpu(), "f32", s.stride, s.pad, s.dilation)
    assert_close(as_f64(got[:2]), want, "f32", s.name())


def test_fused_depth_taps_accumulate():
    """KD = 2 forced Winograd in fp32: the second depth tap adds into out in the
    persistent kernel's output stage, bit for bit as in the three-launch path."""
    s = synth.Conv3dShape(1, 7, 10, 12, 64, 96, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    opt = B.make_options("winograd")
    x, w = synth.conv3d_inputs(s, "f32", "normal", 33, device="cuda")
    with env(B200CONV_WINOGRAD_FUSED=0):
        ref = B.conv3d(x, w, s.stride, s.pad, s.dilation, options=opt)
    with env(B200CONV_WINOGRAD_FUSED=1, B200CONV_WINOGRAD_FUSED_GRID=1):
        got = B.conv3d(x, w, s.stride, s.pad, s.dilation, options=opt)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(_bits(got), _bits(ref))
    want = oracle.conv3d(x.cpu(), w.cpu(), "f32", s.stride, s.pad, s.dilation)
    assert_close(as_f64(got), want, "f32", s.name())


def test_fused_headline_shape():
    """40 x 512 x 512, 192 -> 96 on the persistent kernel (one CTA per SM, 2,312
    blocks): the whole output equals the three-launch path bit for bit."""
    s = synth.WINOGRAD_F32
    x, w = synth.conv2d_inputs(s, "f32", "uniform", 34, device="cuda")
    with env(B200CONV_WINOGRAD_FUSED=1):
        assert _plan(s, B.make_options())["winograd_fused"] == 1
        got = B.conv2d(x, w, s.stride, s.pad, s.dilation)
    ref = B.conv2d(x, w, s.stride, s.pad, s.dilation)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(_bits(got), _bits(ref))


def test_fused_unaligned_input_reads_without_tma():
    """An input 4 bytes off a 16-byte boundary cannot be a TMA source: the
    transform warpgroup then reads it with per-thread loads, same bits."""
    s = synth.Conv2dShape(2, 64, 64, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1))
    x0, w = synth.conv2d_inputs(s, "f32", "normal", 35, device="cuda")
    buf = torch.empty(x0.numel() + 1, dtype=torch.float32, device="cuda")
    x = buf[1:].view(x0.shape)
    x.copy_(x0)
    assert x.data_ptr() % 16 != 0
    with env(B200CONV_WINOGRAD_FUSED=0):
        ref = B.conv2d(x0, w, s.stride, s.pad, s.dilation)
    with env(B200CONV_WINOGRAD_FUSED=1, B200CONV_WINOGRAD_FUSED_GRID=3):
        got = B.conv2d(x, w, s.stride, s.pad, s.dilation)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(_bits(got), _bits(ref))
