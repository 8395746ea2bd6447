"""The allocation-free Winograd entry point, conv2d_forward_winograd_static.

It exists for callers that cannot allocate device memory or pass a workspace
(code inside another runtime's hooks, services that must not allocate once
running, callers with only borrowed pointers): its scratch is a fixed 64 MiB
device array inside the library.  These tests call it through the C ABI and
compare it with the existing conv2d_forward entry point, on two calls in a
row (the array keeps the previous call's contents, which must not matter):
bit for bit against conv2d_forward forced to Winograd at the same batch tile,
and within the parity tolerance against the CPU oracle and the auto path.  A
conv too large for the array is refused before any launch.

This file is named to be collected last, and it sets up nothing that depends
on the other test files, so it passes alone in a fresh process too.
"""
import numpy as np
import pytest
import torch

from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import TOL, as_f64, rel_err

pytestmark = pytest.mark.gpu

CASES = [
    # 128x128, 128 -> 128 fp32: one image's transform buffers (32 MB) plus the
    # filter fill most of the array, so the batch runs as three 1-image tiles
    (synth.Conv2dShape(3, 128, 128, 128, 128, 3, 3, (1, 1), (1, 1), (1, 1)), "f32"),
    (synth.Conv2dShape(5, 40, 36, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1)), "f32"),
    (synth.Conv2dShape(4, 30, 30, 64, 64, 3, 3, (1, 1), (0, 0), (1, 1)), "bf16"),
    (synth.Conv2dShape(2, 33, 17, 32, 48, 3, 3, (1, 1), (2, 1), (1, 1)), "f16"),
]


def _desc(s):
    return B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)


STATIC_BYTES = 64 << 20


def _static_tile(shape, dtype):
    """The batch tile the static entry point settles on: the largest tile whose
    transformed filter plus transform buffers fit the 64 MiB array (the same
    search, done here through conv2d_plan)."""
    desc = _desc(shape)
    tile = shape.n
    while True:
        p = B.plan2d(desc, dtype, 0, B.make_options("winograd", STATIC_BYTES, tile))
        if p["workspace_bytes"] <= STATIC_BYTES:
            return p
        assert p["batch_tile"] > 1, "not even one image fits"
        tile = p["batch_tile"] - 1


@pytest.mark.parametrize("shape,dtype", CASES, ids=lambda v: v.name() if hasattr(v, "name") else v)
def test_static_scratch_matches_conv2d_forward(shape, dtype):
    import oracle
    x, w = synth.conv2d_inputs(shape, dtype, "normal", 3, device="cuda")
    plan = _static_tile(shape, dtype)
    assert plan["algo"] == "winograd"
    if shape == CASES[0][0]:
        assert plan["num_batch_tiles"] > 1, plan      # the first case really runs batch-tiled
    # the existing entry point, forced to Winograd at the static entry's tile size
    ref_win = B.conv2d(x, w, shape.stride, shape.pad, shape.dilation,
                       options=B.make_options("winograd", winograd_tile_batch=plan["batch_tile"]))
    ref_auto = B.conv2d(x, w, shape.stride, shape.pad, shape.dilation)
    want = oracle.conv2d(x.cpu(), w.cpu(), dtype, shape.stride, shape.pad, shape.dilation)
    stream = torch.cuda.current_stream().cuda_stream
    desc = _desc(shape)
    for call in range(2):
        out = torch.full((shape.n, shape.oh, shape.ow, shape.o), float("nan"), dtype=x.dtype, device="cuda")
        st = B.conv2d_forward_winograd_static(x.data_ptr(), w.data_ptr(), out.data_ptr(), desc,
                                              B.DTYPE[dtype], stream)
        assert st == 0, B.conv_status_string(st)
        torch.cuda.synchronize()
        assert B.conv_check(stream) == 0
        got = as_f64(out)
        assert np.isfinite(got).all(), f"call {call}: unwritten output"
        # bit for bit what conv2d_forward's Winograd path gives at the same tile size
        assert torch.equal(out.view(torch.int32 if dtype == "f32" else torch.int16),
                           ref_win.view(torch.int32 if dtype == "f32" else torch.int16)), f"call {call}"
        e = rel_err(got, want)
        assert e <= TOL[dtype], f"call {call} vs the oracle: {e:.3e}"
        e2 = rel_err(got, as_f64(ref_auto))
        assert e2 <= TOL[dtype], f"call {call} vs conv2d_forward (auto): {e2:.3e}"


def test_static_scratch_refuses_what_does_not_fit():
    """512x512, 192 -> 96 fp32 needs 545 MB of transform buffers per image:
    refused with CONV_ERR_WORKSPACE before any launch (null pointers prove it
    never reaches a kernel: a launch attempt would report CONV_ERR_INVALID)."""
    st = B.conv2d_forward_winograd_static(0, 0, 0, _desc(synth.WINOGRAD_F32), B.DTYPE["f32"], 0)
    assert st == 4, B.conv_status_string(st)


def test_static_scratch_refuses_non_winograd_shapes():
    s = synth.Conv2dShape(1, 16, 16, 32, 32, 5, 5, (1, 1), (2, 2), (1, 1))
    st = B.conv2d_forward_winograd_static(0, 0, 0, _desc(s), B.DTYPE["f32"], 0)
    assert st == 2, B.conv_status_string(st)
