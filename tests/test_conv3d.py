"""conv3d as depth-tap 2D convs ("Decompose small kernel-depth 3D convs into 2D
convs", Change, Tests) and as the native K-fused 3D implicit GEMM.

* the fast path against the oracle over shapes with Cout != Cin,
  KD in {1, 2, 3, 5} and a 1x1-spatial case;
* the cases the page sends to its fallback -- depth stride > 1, depth padding,
  non-multiple-of-16 channels, N > 1, kernel depth dilation, KD > 7 -- stay
  correct here because the taps are generalised instead;
* the depth-tap result equals a manual loop of conv2d_forward over frame views
  plus conv_accumulate, bit for bit (the page's "numerically identical to"
  per-frame 2D);
* the workload's three shapes on sampled pixels;
* the native tcgen05 3D GEMM (5D TMA im2col) against the oracle, and against
  the depth taps.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import TOL, as_f64, assert_close, guarded_input, guarded_output, guarded_workspace

pytestmark = pytest.mark.gpu


def run3d(x, w, s, options=None):
    """Through the C ABI with the inputs inside NaN bands (a read past either
    end reaches the output as a NaN), a NaN-poisoned output and the plan's exact
    workspace inside canary bands that must stay untouched."""
    desc = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[x.dtype]
    plan = B.plan3d(desc, dt, x.device.index or 0, options)
    g_x, xg = guarded_input(x)
    g_w, wg = guarded_input(w)
    g_out, out = guarded_output((s.n, s.od, s.oh, s.ow, s.o), x.dtype, x.device)
    g_ws = guarded_workspace(plan["workspace_bytes"], x.device)
    out = B.conv3d(xg, wg, s.stride, s.pad, s.dilation, options=options, out=out,
                   workspace=g_ws.inner() if g_ws else None)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    g_out.assert_intact(f"{s.name()} out")
    g_x.assert_intact(f"{s.name()} input")
    g_w.assert_intact(f"{s.name()} weights")
    if g_ws:
        g_ws.assert_intact(f"{s.name()} workspace")
    return out


def check3d(s, dtype, dist="normal", options=None, sample=None):
    x, w = synth.conv3d_inputs(s, dtype, dist, 0, device="cuda")
    out = run3d(x, w, s, options)
    if sample:
        pix = synth.sample_pixels(s.n, s.oh, s.ow, sample, 0, od=s.od)
        ref = oracle.conv3d(x.cpu(), w.cpu(), dtype, s.stride, s.pad, s.dilation, pixels=pix.numpy())
        p = pix.long()
        got = as_f64(out[p[:, 0], p[:, 1], p[:, 2], p[:, 3]])
    else:
        ref = oracle.conv3d(x.cpu(), w.cpu(), dtype, s.stride, s.pad, s.dilation)
        got = as_f64(out)
    return assert_close(got, ref, dtype, s.name())


FAST = [
    synth.Conv3dShape(1, 6, 10, 12, 32, 48, 1, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
    synth.Conv3dShape(1, 7, 9, 9, 48, 32, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
    synth.Conv3dShape(1, 8, 12, 10, 64, 64, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
    synth.Conv3dShape(1, 9, 6, 7, 32, 64, 5, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
    synth.Conv3dShape(1, 6, 1, 1, 64, 32, 3, 1, 1, (1, 1, 1), (0, 0, 0), (1, 1, 1)),   # 1x1 spatial
]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("s", FAST, ids=lambda s: s.name())
def test_depth_taps_against_oracle(s, dtype):
    check3d(s, dtype)


FALLBACK_CASES = [
    synth.Conv3dShape(1, 9, 8, 8, 32, 32, 3, 3, 3, (2, 1, 1), (0, 1, 1), (1, 1, 1)),   # depth stride 2
    synth.Conv3dShape(1, 6, 8, 8, 32, 32, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1)),   # depth pad 1
    synth.Conv3dShape(1, 6, 8, 8, 20, 13, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),   # non-mod-16 channels
    synth.Conv3dShape(3, 5, 7, 6, 32, 16, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),   # N > 1
    synth.Conv3dShape(1, 9, 6, 6, 16, 16, 3, 3, 3, (1, 2, 2), (2, 1, 1), (2, 1, 1)),   # depth dilation, pads
    synth.Conv3dShape(1, 12, 5, 5, 16, 16, 9, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),  # KD > 7
    synth.Conv3dShape(2, 7, 9, 11, 24, 40, 3, 3, 5, (3, 2, 1), (2, 0, 2), (1, 1, 2)),  # everything at once
]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("s", FALLBACK_CASES, ids=lambda s: s.name())
def test_generalised_taps(s, dtype):
    check3d(s, dtype)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_taps_equal_manual_per_frame_loop(dtype):
    """conv3d == for kd: conv2d_forward(frame view kd, w[:, kd]) then an in-place add."""
    s = synth.Conv3dShape(1, 9, 14, 12, 64, 48, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    x, w = synth.conv3d_inputs(s, dtype, "normal", 5, device="cuda")
    got = run3d(x, w, s)
    OD = s.od
    acc = None
    for kd in range(s.kd):
        view = x[0, kd:kd + OD]                     # [OD, H, W, C], contiguous frames
        wk = w[:, kd].contiguous()                  # [O, KH, KW, C]
        tap = B.conv2d(view, wk, s.stride[1:], s.pad[1:], s.dilation[1:])
        if acc is None:
            acc = tap
        else:
            st = B.conv_accumulate(acc.data_ptr(), tap.data_ptr(), acc.numel(), B.DTYPE[dtype],
                                   torch.cuda.current_stream().cuda_stream)
            assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(got[0], acc)


@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
def test_winograd_taps_accumulate_equal_manual_loop(dtype):
    """KD = 2 with forced Winograd: depth taps whose 2D Winograd output stage adds
    into out equal conv2d (forced Winograd) per frame view + conv_accumulate, bit
    for bit, and match the oracle."""
    s = synth.Conv3dShape(1, 7, 10, 12, 64, 96, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    opt = B.make_options("winograd")
    x, w = synth.conv3d_inputs(s, dtype, "normal", 8, device="cuda")
    got = run3d(x, w, s, opt)
    acc = None
    for kd in range(s.kd):
        tap = B.conv2d(x[0, kd:kd + s.od], w[:, kd].contiguous(), s.stride[1:], s.pad[1:], s.dilation[1:], options=opt)
        if acc is None:
            acc = tap
        else:
            assert B.conv_accumulate(acc.data_ptr(), tap.data_ptr(), acc.numel(), B.DTYPE[dtype],
                                     torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert torch.equal(got[0], acc)
    ref = oracle.conv3d(x.cpu(), w.cpu(), dtype, s.stride, s.pad, s.dilation)
    assert_close(as_f64(got), ref, dtype, s.name())


@pytest.mark.parametrize("s", synth.CONV3D_TAPS, ids=lambda s: s.name())
def test_workload_shapes_sampled(s):
    check3d(s, "bf16", sample=4096)


def test_accumulate_rounds_once_per_add():
    """out = round(out + tap) with an fp32 add, every dtype, ragged length."""
    for dt, tt in (("f32", torch.float32), ("f16", torch.float16), ("bf16", torch.bfloat16)):
        n = 1000003
        g = torch.Generator(device="cuda").manual_seed(9)
        a = torch.randn(n, generator=g, device="cuda").to(tt)
        b = torch.randn(n, generator=g, device="cuda").to(tt)
        want = (a.float() + b.float()).to(tt)
        st = B.conv_accumulate(a.data_ptr(), b.data_ptr(), n, B.DTYPE[dt], torch.cuda.current_stream().cuda_stream)
        assert st == 0
        torch.cuda.synchronize()
        assert torch.equal(a, want), dt


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("s", FAST[1:4] + FALLBACK_CASES[:2], ids=lambda s: s.name())
def test_native_3d_gemm_against_oracle(s, dtype):
    """The K-fused tcgen05 3D implicit GEMM (forced) against the oracle."""
    desc = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    assert B.plan3d(desc, dtype, 0, B.make_options("implicit"))["taps"] == 1
    check3d(s, dtype, options=B.make_options("implicit"))


def test_native_and_taps_agree():
    s = synth.Conv3dShape(2, 7, 12, 10, 64, 96, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1))
    x, w = synth.conv3d_inputs(s, "bf16", "normal", 7, device="cuda")
    a = run3d(x, w, s, B.make_options("implicit"))
    b = run3d(x, w, s, B.make_options("direct"))
    ref = oracle.conv3d(x.cpu(), w.cpu(), "bf16", s.stride, s.pad, s.dilation)
    assert_close(as_f64(a), ref, "bf16", "native")
    assert_close(as_f64(b), ref, "bf16", "taps")


# ---------------------------------------------------------------------------
# Native 3D Winograd F(m^3, 3^3): the depth-tap page's open question on a
# native 3D Winograd, built as the 2D method nested along depth.
# ---------------------------------------------------------------------------

WINO3D = [
    synth.Conv3dShape(1, 10, 12, 12, 128, 128, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),   # whole 4^3 tiles
    synth.Conv3dShape(2, 9, 13, 11, 64, 192, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1)),     # ragged in every dim, N = 2
    synth.Conv3dShape(1, 7, 9, 10, 96, 160, 3, 3, 3, (1, 1, 1), (2, 0, 2), (1, 1, 1)),      # pads 2 / 0 / 2
    synth.Conv3dShape(3, 5, 6, 7, 32, 224, 3, 3, 3, (1, 1, 1), (0, 2, 1), (1, 1, 1)),       # small volumes, OD = 3
]


def wino3d_plan(s, dtype, options=None):
    desc = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    return B.plan3d(desc, dtype, 0, options)


@pytest.mark.parametrize("s", WINO3D, ids=lambda s: s.name())
def test_winograd3d_f32_auto_against_oracle(s):
    p = wino3d_plan(s, "f32")
    assert p["algo"] == "winograd" and p["winograd_m"] == 4 and p["taps"] == 1
    check3d(s, "f32")


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("s", WINO3D[1:3], ids=lambda s: s.name())
def test_winograd3d_16bit_forced_against_oracle(s, dtype):
    opt = B.make_options("winograd")
    p = wino3d_plan(s, dtype, opt)
    assert p["algo"] == "winograd" and p["winograd_m"] == 2 and p["engine"] == "tcgen05"
    check3d(s, dtype, options=opt)


def test_winograd3d_large_pads_and_empty_batch():
    """Pads beyond the filter reach (whole tiles of padding) in every dimension,
    and N = 0, which is a no-op that touches nothing."""
    s = synth.Conv3dShape(1, 4, 5, 6, 32, 64, 3, 3, 3, (1, 1, 1), (3, 4, 2), (1, 1, 1))
    opt = B.make_options("winograd")
    assert wino3d_plan(s, "f32", opt)["algo"] == "winograd"
    check3d(s, "f32", options=opt)
    e = synth.Conv3dShape(0, 6, 8, 8, 32, 32, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1))
    d = B.make_desc3d(0, e.d, e.h, e.w, e.c, e.o, 3, 3, 3, e.stride, e.pad, e.dilation)
    st = B.conv3d_forward(0, 0, 0, d, 0, opt, 0, 0, torch.cuda.current_stream().cuda_stream)
    assert st == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_winograd3d_forced_unaligned_channels(dtype):
    """C % 8 != 0 (16-bit operands then go through the FFMA GEMM in fp32) and an
    O that is no multiple of 32 or of a GEMM tile."""
    s = synth.Conv3dShape(2, 6, 7, 9, 36, 20, 3, 3, 3, (1, 1, 1), (1, 1, 0), (1, 1, 1))
    opt = B.make_options("winograd")
    p = wino3d_plan(s, dtype, opt)
    assert p["algo"] == "winograd" and p["taps"] == 1 and p["engine"] == "simt"
    check3d(s, dtype, options=opt)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_winograd3d_unit_tiling_is_bit_identical(dtype):
    """Tiles of 1 and 2 units (the latter straddling images) equal the untiled
    run bit for bit."""
    s = synth.Conv3dShape(2, 11, 10, 9, 64, 192, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))   # OD = 9
    units = 2 * (3 if dtype == "f32" else 5)          # depth tiles of 4 (fp32) or 2 (16-bit) frames
    x, w = synth.conv3d_inputs(s, dtype, "normal", 3, device="cuda")
    outs = []
    for tb in (0, 1, 2):
        opt = B.make_options("winograd", winograd_tile_batch=tb)
        p = wino3d_plan(s, dtype, opt)
        assert p["algo"] == "winograd" and p["batch_tile"] == (units if tb == 0 else tb)
        outs.append(run3d(x, w, s, opt))
    iv = torch.int32 if dtype == "f32" else torch.int16
    assert torch.equal(outs[0].view(iv), outs[1].view(iv))
    assert torch.equal(outs[0].view(iv), outs[2].view(iv))


@pytest.mark.parametrize("s", synth.CONV3D_TAPS, ids=lambda s: s.name())
def test_workload_shapes_f32_sampled(s):
    """The conv3d workload in fp32: the native 3D Winograd on all three shapes
    (the largest in batch tiles of depth units under the 8 GiB workspace cap)."""
    check3d(s, "f32", sample=4096)
