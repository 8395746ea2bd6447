"""CTA pairs on the tensor cores: a 256-row tile computed by two SMs
(tcgen05 cta_group::2), each holding 128 rows of the input tile and half of
the weight tile, so the weight tile crosses L2 once per pair instead of once
per SM -- the wide-C_out regime of "Use the explicit gemm for wide convs on
neural accelerators" (description).  Used for 256-wide column tiles with a K
loop of at least 8 steps of 64 when there are enough 256-row tiles;
B200CONV_TC_PAIR=0 (a test hook read on every call) keeps 128-row tiles.

Checked against the oracle and against the 128-row kernel, on the implicit
GEMM (aligned, ragged M with a pair whose second half is past the end,
stride and dilation, the depth-tap accumulate mode), the native 3D implicit
GEMM and the 16-bit Winograd GEMM.
"""
import os

import pytest
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import TOL, as_f64, assert_close, check_conv2d, rel_err, run_conv2d

pytestmark = pytest.mark.gpu


class env:
    def __init__(self, **kv):
        self.kv = kv

    def __enter__(self):
        self.old = {k: os.environ.get(k) for k in self.kv}
        os.environ.update({k: str(v) for k, v in self.kv.items()})

    def __exit__(self, *a):
        for k, v in self.old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def plan(s, dt, opts=None):
    d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
    return B.plan2d(d, dt, 0, opts)


SHAPES = [
    synth.Conv2dShape(16, 64, 64, 256, 1024, 3, 3, (1, 1), (1, 1), (1, 1)),     # M = 65536, 256 x 4 tiles
    synth.Conv2dShape(5, 45, 47, 128, 2048, 3, 3, (1, 1), (1, 1), (1, 1)),      # ragged M, last pair half empty
    synth.Conv2dShape(4, 128, 128, 128, 512, 5, 5, (2, 2), (4, 4), (2, 2)),     # stride and dilation
    synth.Conv2dShape(8, 40, 40, 1024, 520, 1, 1, (1, 1), (0, 0), (1, 1)),      # 1x1, O past the last full tile
]


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name())
def test_pair_tiles_match_oracle_and_single_cta(shape, dtype):
    p = plan(shape, dtype)
    assert p["engine"] == "tcgen05" and p["tile_n"] == 256 and p["tile_m"] == 256, p
    with env(B200CONV_TC_PAIR=0):
        assert plan(shape, dtype)["tile_m"] == 128
    x, w = synth.conv2d_inputs(shape, dtype, "normal", 41, device="cuda")
    got = run_conv2d(x, w, shape)
    with env(B200CONV_TC_PAIR=0):
        single = run_conv2d(x, w, shape)
    # the same MMAs in the same K order per output element: same values
    e = rel_err(as_f64(got), as_f64(single))
    assert e <= 1e-6, e
    pix = synth.sample_pixels(shape.n, shape.oh, shape.ow, 4096, 41)
    want = oracle.conv2d(x.cpu(), w.cpu(), dtype, shape.stride, shape.pad, shape.dilation, pixels=pix.numpy())
    p_ = pix.long()
    assert_close(as_f64(got[p_[:, 0], p_[:, 1], p_[:, 2]]), want, dtype, shape.name())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_pair_tiles_winograd_gemm(dtype):
    """The 16-bit Winograd GEMM with C = 1024 (16 K steps) runs in pairs; with
    C = 256 (4 K steps) it keeps 128-row tiles."""
    short = synth.Conv2dShape(8, 48, 48, 256, 512, 3, 3, (1, 1), (1, 1), (1, 1))
    assert plan(short, dtype, B.make_options("winograd"))["tile_m"] == 128
    s = synth.Conv2dShape(4, 48, 48, 1024, 512, 3, 3, (1, 1), (1, 1), (1, 1))
    opts = B.make_options("winograd")
    p = plan(s, dtype, opts)
    assert p["algo"] == "winograd" and p["engine"] == "tcgen05" and p["tile_m"] == 256, p
    check_conv2d(s, dtype, options=opts)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_pair_tiles_native_conv3d_and_depth_taps(dtype):
    s = synth.Conv3dShape(2, 10, 24, 24, 128, 512, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1))   # native 3D
    d = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    p = B.plan3d(d, dtype, 0, None)
    assert p["taps"] == 1 and p["tile_m"] == 256, p
    x, w = synth.conv3d_inputs(s, dtype, "normal", 42, device="cuda")
    got = B.conv3d(x, w, s.stride, s.pad, s.dilation)
    torch.cuda.synchronize()
    pix = synth.sample_pixels(s.n, s.oh, s.ow, 4096, 42, od=s.od)
    want = oracle.conv3d(x.cpu(), w.cpu(), dtype, s.stride, s.pad, s.dilation, pixels=pix.numpy())
    p_ = pix.long()
    assert_close(as_f64(got[p_[:, 0], p_[:, 1], p_[:, 2], p_[:, 3]]), want, dtype, "native3d pairs")
    # depth taps (N = 1, no depth padding): 2D pair tiles that add into out
    t = synth.Conv3dShape(1, 8, 48, 48, 256, 512, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    dt_ = B.make_desc3d(t.n, t.d, t.h, t.w, t.c, t.o, t.kd, t.kh, t.kw, t.stride, t.pad, t.dilation)
    pt = B.plan3d(dt_, dtype, 0, None)
    assert pt["taps"] == 3 and pt["tile_m"] == 256, pt
    x, w = synth.conv3d_inputs(t, dtype, "normal", 43, device="cuda")
    got = B.conv3d(x, w, t.stride, t.pad, t.dilation)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    pix = synth.sample_pixels(t.n, t.oh, t.ow, 4096, 43, od=t.od)
    want = oracle.conv3d(x.cpu(), w.cpu(), dtype, t.stride, t.pad, t.dilation, pixels=pix.numpy())
    p_ = pix.long()
    assert_close(as_f64(got[p_[:, 0], p_[:, 1], p_[:, 2], p_[:, 3]]), want, dtype, "depth taps pairs")
