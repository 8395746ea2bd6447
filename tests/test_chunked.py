"""The chunked fp32 Winograd pipeline against the unchunked path and the oracle.

Within a batch tile the fp32-store Winograd path ("Bound winograd conv2d
working set by tiling the batch", Fix) runs its transforms and GEMM over
chunks of tiles sized so that V and M stay in L2, with the output transform of
one chunk and the input transform of the next in one launch.  Every tile is
transformed on its own and every GEMM output reduces over the channels in one
fixed order, so any chunk size -- ragged, one tile, chunks that cross images
and batch tiles -- must give the unchunked result bit for bit (the page's
"bit-identical" tiling claim, Testing), and match the oracle.

B200CONV_WINOGRAD_CHUNK_TILES (read on every call) sets the chunk; 0 turns
chunking off.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import as_f64, assert_close, run_conv2d

pytestmark = pytest.mark.gpu


class chunk_env:
    def __init__(self, tiles):
        self.tiles = tiles

    def __enter__(self):
        self.old = os.environ.get("B200CONV_WINOGRAD_CHUNK_TILES")
        os.environ["B200CONV_WINOGRAD_CHUNK_TILES"] = str(self.tiles)

    def __exit__(self, *a):
        if self.old is None:
            os.environ.pop("B200CONV_WINOGRAD_CHUNK_TILES", None)
        else:
            os.environ["B200CONV_WINOGRAD_CHUNK_TILES"] = self.old


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def _plan(s, dtype, opts):
    d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
    return B.plan2d(d, dtype, 0, opts)


CASES = [
    # 7x6 = 42 tiles per image of F(6,3), O not a multiple of the GEMM tile
    (synth.Conv2dShape(3, 40, 36, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1)), "f32"),
    # ragged tiles at the bottom/right edge, no padding, wider O
    (synth.Conv2dShape(2, 47, 29, 32, 160, 3, 3, (1, 1), (0, 0), (1, 1)), "f32"),
    # 16-bit input on the FFMA engine (C % 8 != 0, C % 4 == 0): F(2,3) with fp32 V and M
    (synth.Conv2dShape(2, 21, 19, 20, 36, 3, 3, (1, 1), (1, 1), (1, 1)), "bf16"),
]


@pytest.mark.parametrize("shape,dtype", CASES, ids=lambda v: v.name() if hasattr(v, "name") else v)
def test_chunked_equals_unchunked_bit_for_bit(shape, dtype):
    opts = B.make_options("winograd")
    x, w = synth.conv2d_inputs(shape, dtype, "normal", 21, device="cuda")
    with chunk_env(0):
        p0 = _plan(shape, dtype, opts)
        assert p0["algo"] == "winograd" and p0["engine"] == "simt"
        ref = run_conv2d(x, w, shape, opts)
    want = oracle.conv2d(x.cpu(), w.cpu(), dtype, shape.stride, shape.pad, shape.dilation)
    assert_close(as_f64(ref), want, dtype, shape.name())
    tiles = shape.n * ((shape.oh + (6 if dtype == "f32" else 2) - 1) // (6 if dtype == "f32" else 2)) * \
        ((shape.ow + (6 if dtype == "f32" else 2) - 1) // (6 if dtype == "f32" else 2))
    for chunk in (1, 5, 37, 128, tiles - 1, tiles, 4 * tiles):
        with chunk_env(chunk):
            p = _plan(shape, dtype, opts)
            assert p["workspace_bytes"] <= p0["workspace_bytes"] + 2 * 64 * chunk * shape.c * 4 + 256
            got = run_conv2d(x, w, shape, opts)
        assert torch.equal(_bits(got), _bits(ref)), f"chunk {chunk}"


def test_chunks_inside_forced_batch_tiles():
    """Chunks run inside each batch tile (a forced tile of 1 and of 2 images),
    and the result is the untiled, unchunked one bit for bit."""
    s = CASES[0][0]
    x, w = synth.conv2d_inputs(s, "f32", "uniform", 22, device="cuda")
    with chunk_env(0):
        ref = run_conv2d(x, w, s, B.make_options("winograd"))
    for tile in (1, 2):
        for chunk in (11, 42, 50):
            opts = B.make_options("winograd", winograd_tile_batch=tile)
            with chunk_env(chunk):
                p = _plan(s, "f32", opts)
                assert p["batch_tile"] == tile and p["num_batch_tiles"] == (s.n + tile - 1) // tile
                got = run_conv2d(x, w, s, opts)
            assert torch.equal(_bits(got), _bits(ref)), (tile, chunk)


def test_chunked_depth_taps_accumulate():
    """conv3d depth taps on the fp32 Winograd path: each tap's output stage adds
    into out inside the pass kernel; chunked equals unchunked bit for bit."""
    s = synth.Conv3dShape(1, 6, 20, 22, 64, 96, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))   # KD = 2: depth taps
    opts = B.make_options("winograd")
    x, w = synth.conv3d_inputs(s, "f32", "normal", 23, device="cuda")
    d = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    outs = []
    for chunk in (0, 7, 64):
        with chunk_env(chunk):
            p = B.plan3d(d, "f32", 0, opts)
            assert p["taps"] == 2 and p["algo"] == "winograd" and p["engine"] == "simt"
            out = B.conv3d(x, w, s.stride, s.pad, s.dilation, options=opts)
            torch.cuda.synchronize()
            outs.append(out)
    assert torch.equal(_bits(outs[0]), _bits(outs[1])) and torch.equal(_bits(outs[0]), _bits(outs[2]))
    want = oracle.conv3d(x.cpu(), w.cpu(), "f32", s.stride, s.pad, s.dilation)
    assert_close(as_f64(outs[0]), want, "f32", s.name())
