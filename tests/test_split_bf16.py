"""The fp32 Winograd GEMM on the tensor cores over split-bf16 operands.

The fp32 Winograd path ("Bound winograd conv2d working set by tiling the
batch", Problem and Fix: input transform, batched GEMM, output transform) can
run its batched GEMM on tcgen05: every fp32 value of V and U is the exact sum
of three bf16 parts, and the six products a_i b_j with i + j <= 2 are
accumulated in fp32 in one K = 6C reduction.  The transforms stay fp32.  The
result must stay inside the fp32 tolerance against the oracle (the dropped
products are below 2^-24 of the result), and batch tiling must stay
bit-identical.

B200CONV_WINOGRAD_SPLIT_BF16=1 (read on every call) turns the route on.
"""
import os

import pytest
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import as_f64, assert_close, rel_err, run_conv2d

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


def _plan(s, opts):
    d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
    return B.plan2d(d, "f32", 0, opts)


SHAPES = [
    # 4 x 4 tiles of F(6,3) per image, O = 96 (one 128-wide column tile, 96 valid)
    synth.Conv2dShape(2, 20, 20, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1)),
    # no padding, ragged edge tiles
    synth.Conv2dShape(3, 13, 29, 64, 64, 3, 3, (1, 1), (0, 0), (1, 1)),
    # C = 128 (two 64-wide blocks per part), O = 40
    synth.Conv2dShape(1, 30, 30, 128, 40, 3, 3, (1, 1), (1, 1), (1, 1)),
    # C = 192, many GEMM row tiles
    synth.Conv2dShape(2, 64, 60, 192, 96, 3, 3, (1, 1), (1, 1), (1, 1)),
    # O = 200: 256-wide column tiles, partly empty
    synth.Conv2dShape(2, 24, 24, 64, 200, 3, 3, (1, 1), (1, 1), (1, 1)),
    # asymmetric padding
    synth.Conv2dShape(2, 26, 22, 64, 128, 3, 3, (1, 1), (2, 0), (1, 1)),
]


@pytest.mark.parametrize("dist", ["normal", "uniform"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name())
def test_split_bf16_against_oracle(shape, dist):
    opts = B.make_options("winograd")
    x, w = synth.conv2d_inputs(shape, "f32", dist, 41, device="cuda")
    want = oracle.conv2d(x.cpu(), w.cpu(), "f32", shape.stride, shape.pad, shape.dilation)
    ffma = run_conv2d(x, w, shape, opts)
    with env(B200CONV_WINOGRAD_SPLIT_BF16=1):
        p = _plan(shape, opts)
        assert p["algo"] == "winograd" and p["engine"] == "tcgen05" and p["winograd_m"] == 6, p
        got = run_conv2d(x, w, shape, opts)
    e_split = assert_close(as_f64(got), want, "f32", shape.name())
    e_ffma = rel_err(as_f64(ffma), want)
    # fp32-accurate: within a small factor of the FFMA GEMM's own error
    assert e_split <= max(4 * e_ffma, 1e-6), (e_split, e_ffma)


def test_split_bf16_batch_tiling_is_bit_identical():
    s = synth.Conv2dShape(5, 40, 36, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1))
    x, w = synth.conv2d_inputs(s, "f32", "normal", 42, device="cuda")
    with env(B200CONV_WINOGRAD_SPLIT_BF16=1):
        outs = [run_conv2d(x, w, s, B.make_options("winograd", winograd_tile_batch=tb)) for tb in (0, 1, 2)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int32), outs[0].view(torch.int32))


def test_split_bf16_depth_taps_accumulate():
    """KD = 2 forced Winograd in fp32: the second tap adds into out."""
    s = synth.Conv3dShape(1, 7, 10, 12, 64, 96, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    opt = B.make_options("winograd")
    x, w = synth.conv3d_inputs(s, "f32", "normal", 43, device="cuda")
    with env(B200CONV_WINOGRAD_SPLIT_BF16=1):
        got = B.conv3d(x, w, s.stride, s.pad, s.dilation, options=opt)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    want = oracle.conv3d(x.cpu(), w.cpu(), "f32", s.stride, s.pad, s.dilation)
    assert_close(as_f64(got), want, "f32", s.name())


def test_split_bf16_headline_shape_sampled():
    """40 x 512 x 512, 192 -> 96: 4096 sampled pixels against the oracle."""
    s = synth.WINOGRAD_F32
    x, w = synth.conv2d_inputs(s, "f32", "uniform", 44, device="cuda")
    with env(B200CONV_WINOGRAD_SPLIT_BF16=1):
        p = _plan(s, B.make_options())
        assert p["engine"] == "tcgen05" and p["algo"] == "winograd", p
        got = B.conv2d(x, w, s.stride, s.pad, s.dilation)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    pix = synth.sample_pixels(s.n, s.oh, s.ow, 4096, 7)
    want = oracle.conv2d(x.cpu(), w.cpu(), "f32", s.stride, s.pad, s.dilation, pixels=pix.numpy())
    p = pix.long()
    assert_close(as_f64(got[p[:, 0], p[:, 1], p[:, 2]]), want, "f32", s.name())
