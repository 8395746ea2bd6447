"""Split-K on the tensor cores: the K range of a small-M, long-K implicit GEMM
is split over several CTAs per output tile ("Use the explicit gemm for wide
convs on neural accelerators", ResNet-50 follow-up: the small late-stage
layers).  Two routes give the same bits:

* the default: every split writes its fp32 partial to the workspace and a
  reduce kernel sums the splits in split order;
* the cluster route (B200CONV_SPLITK_CLUSTER=1, a test hook read on every
  call): the splits of a tile run as one thread-block cluster, each leaving its
  partial in its own shared memory, and every CTA of the cluster sums a slice
  of the tile's rows over the splits in split order and writes those rows,
  with no reduce launch (taken when a launch's clusters all fit at once);
* the serial route (B200CONV_SPLITK_SERIAL=1): every split writes its partial
  and counts its arrival per (tile, epilogue warp); the split that arrives last
  sums the partials in split order and writes the output, no reduce launch.

Checked: both routes agree bit for bit, match the oracle, repeat bit for bit,
the cluster route launches no reduce kernel when its clusters fit in one wave,
and the depth-tap accumulate mode (conv3d) works through the cluster epilogue.
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


# (shape, whether the in-kernel cluster route must be taken on a B200).  A
# cluster of ks CTAs needs ks SMs of one GPC; when a launch's clusters do not
# all fit at once the kernel writes partials for the reduce kernel instead
# (same sums, same order), so the 26 clusters of 5 may take either route.
SHAPES = [
    # 1 row tile x 4 column tiles, 72 K steps: 16 splits (four 16-CTA clusters)
    (synth.Conv2dShape(1, 7, 7, 512, 512, 3, 3, (1, 1), (1, 1), (1, 1)), True),
    # 13 x 2 tiles, 36 K steps: 5 splits
    (synth.Conv2dShape(8, 14, 14, 256, 256, 3, 3, (1, 1), (1, 1), (1, 1)), None),
    # a 1x1 with a long K and a ragged M: 8 tiles, 8 splits
    (synth.Conv2dShape(3, 7, 7, 2048, 512, 1, 1, (1, 1), (0, 0), (1, 1)), None),
    # stride 2, O not a multiple of the column tile: 2 tiles, 16 splits
    (synth.Conv2dShape(2, 14, 14, 512, 200, 3, 3, (2, 2), (1, 1), (1, 1)), True),
]


def _plan(s, dt):
    d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
    return B.plan2d(d, dt, 0, None)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("case", SHAPES, ids=lambda c: c[0].name())
def test_cluster_split_k_matches_reduce_route_and_oracle(case, dtype):
    shape, must_cluster = case
    p = _plan(shape, dtype)
    assert p["engine"] == "tcgen05" and p["k_split"] > 1, p
    x, w = synth.conv2d_inputs(shape, dtype, "he", 31, device="cuda")
    with env(B200CONV_SPLITK_CLUSTER=1):
        B.conv_profile_begin()
        got = run_conv2d(x, w, shape)
        again = run_conv2d(x, w, shape)
        prof = B.profile_end()
    if must_cluster:
        assert "splitk_reduce" not in prof, prof      # summed inside the conv kernel
    B.conv_profile_begin()
    ref = run_conv2d(x, w, shape)                     # the default: partials and the reduce kernel
    prof2 = B.profile_end()
    assert "splitk_reduce" in prof2, prof2
    assert torch.equal(got.view(torch.int16), again.view(torch.int16))
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    want = oracle.conv2d(x.cpu(), w.cpu(), dtype, shape.stride, shape.pad, shape.dilation)
    assert_close(as_f64(got), want, dtype, shape.name())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_cluster_split_k_accumulates_depth_taps(dtype):
    """conv3d depth taps whose 2D convs are split-K: taps after the first add
    into out in the cluster's epilogue; equal to the reduce route bit for bit."""
    s = synth.Conv3dShape(1, 5, 7, 7, 512, 512, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    d = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    p = B.plan3d(d, dtype, 0, None)
    assert p["taps"] == 3 and p["k_split"] > 1 and p["engine"] == "tcgen05", p
    x, w = synth.conv3d_inputs(s, dtype, "normal", 32, device="cuda")
    with env(B200CONV_SPLITK_CLUSTER=1):
        got = B.conv3d(x, w, s.stride, s.pad, s.dilation)
        torch.cuda.synchronize()
    ref = B.conv3d(x, w, s.stride, s.pad, s.dilation)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    want = oracle.conv3d(x.cpu(), w.cpu(), dtype, s.stride, s.pad, s.dilation)
    assert_close(as_f64(got), want, dtype, s.name())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("case", SHAPES, ids=lambda c: c[0].name())
def test_serial_split_k_matches_reduce_route_and_oracle(case, dtype):
    """The last-arriving split reduces: no reduce launch, the same bits as the
    reduce kernel, repeatable (the counters reset themselves), and the oracle."""
    shape, _ = case
    p = _plan(shape, dtype)
    assert p["engine"] == "tcgen05" and p["k_split"] > 1, p
    x, w = synth.conv2d_inputs(shape, dtype, "he", 33, device="cuda")
    with env(B200CONV_SPLITK_SERIAL=1):
        B.conv_profile_begin()
        got = run_conv2d(x, w, shape)
        again = run_conv2d(x, w, shape)
        prof = B.profile_end()
    assert "splitk_reduce" not in prof, prof
    ref = run_conv2d(x, w, shape)
    assert torch.equal(got.view(torch.int16), again.view(torch.int16))
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    want = oracle.conv2d(x.cpu(), w.cpu(), dtype, shape.stride, shape.pad, shape.dilation)
    assert_close(as_f64(got), want, dtype, shape.name())


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_serial_split_k_accumulates_depth_taps(dtype):
    """conv3d depth taps whose 2D convs are split-K on the serial route: the
    last split adds into out; equal to the reduce route bit for bit."""
    s = synth.Conv3dShape(1, 5, 7, 7, 512, 512, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    x, w = synth.conv3d_inputs(s, dtype, "normal", 34, device="cuda")
    with env(B200CONV_SPLITK_SERIAL=1):
        got = B.conv3d(x, w, s.stride, s.pad, s.dilation)
        torch.cuda.synchronize()
    ref = B.conv3d(x, w, s.stride, s.pad, s.dilation)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
