"""Error paths on the GPU.

The failure the Winograd page fixes is a silent one: an out-of-memory during
the conv was dropped and the output came back all zeros ("Bound winograd
conv2d working set by tiling the batch", Problem).  Here every call returns a
status, an undersized workspace is refused before anything runs (the output
keeps its poison), overlapping buffers are refused, misaligned pointers take
the any-alignment path and stay correct, and N = 0 is a no-op.
"""
import numpy as np
import pytest
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth
from tests.gpu_util import TOL, as_f64, assert_close

pytestmark = pytest.mark.gpu

S = synth.Conv2dShape(3, 18, 18, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1))


def desc(s):
    return B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)


def stream():
    return torch.cuda.current_stream().cuda_stream


def test_undersized_workspace_is_refused_and_nothing_runs():
    x, w = synth.conv2d_inputs(S, "f32", "normal", 0, device="cuda")
    opts = B.make_options("winograd")
    need = B.conv2d_workspace_size(desc(S), 0, 0, opts)
    assert need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    out = torch.full((S.n, S.oh, S.ow, S.o), float("nan"), device="cuda")
    st = B.conv2d_forward(x.data_ptr(), w.data_ptr(), out.data_ptr(), desc(S), 0, opts, ws.data_ptr(),
                          ws.numel(), stream())
    assert st == 4       # CONV_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out).all()      # never a partial or zeroed result
    st = B.conv2d_forward(x.data_ptr(), w.data_ptr(), out.data_ptr(), desc(S), 0, opts, 0, 0, stream())
    assert st == 4


def test_misaligned_workspace_is_refused_and_nothing_runs():
    """A workspace base off a 256-byte boundary is CONV_ERR_ALIGNMENT before any
    launch, for conv2d (Winograd and split-K plans) and conv3d (3D Winograd)."""
    x, w = synth.conv2d_inputs(S, "f32", "normal", 0, device="cuda")
    for opts in (B.make_options("winograd"), None):
        shape = S if opts else synth.Conv2dShape(8, 14, 14, 512, 512, 3, 3, (2, 2), (1, 1), (1, 1))   # split-K
        xx, ww = (x, w) if opts else synth.conv2d_inputs(shape, "f32", "normal", 0, device="cuda")
        need = B.conv2d_workspace_size(desc(shape), 0, 0, opts)
        assert need > 0
        ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
        out = torch.full((shape.n, shape.oh, shape.ow, shape.o), float("nan"), device="cuda")
        st = B.conv2d_forward(xx.data_ptr(), ww.data_ptr(), out.data_ptr(), desc(shape), 0, opts, ws.data_ptr() + 16,
                              need, stream())
        assert st == 3       # CONV_ERR_ALIGNMENT
        torch.cuda.synchronize()
        assert torch.isnan(out).all()
    s3 = synth.Conv3dShape(1, 6, 8, 8, 128, 128, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    x3, w3 = synth.conv3d_inputs(s3, "f32", "normal", 0, device="cuda")
    d3 = B.make_desc3d(s3.n, s3.d, s3.h, s3.w, s3.c, s3.o, s3.kd, s3.kh, s3.kw, s3.stride, s3.pad, s3.dilation)
    need = B.conv3d_workspace_size(d3, 0, 0, None)
    assert need > 0
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    out = torch.full((1, s3.od, s3.oh, s3.ow, s3.o), float("nan"), device="cuda")
    st = B.conv3d_forward(x3.data_ptr(), w3.data_ptr(), out.data_ptr(), d3, 0, None, ws.data_ptr() + 128, need,
                          stream())
    assert st == 3
    torch.cuda.synchronize()
    assert torch.isnan(out).all()


def test_fp32_fma_rate_probe():
    """The FMA-chain probe reports a plausible CUDA-core fp32 rate for both forms
    (a B200 at 1.9-2.0 GHz: ~70-80 TFLOP/s scalar), and refuses a null output."""
    import ctypes
    scalar = B.fp32_fma_rate(packed=False)
    packed = B.fp32_fma_rate(packed=True)
    print(f"fp32 FMA rate: scalar {scalar:.1f}, packed {packed:.1f} TFLOP/s")
    assert 20.0 < scalar < 400.0 and 20.0 < packed < 400.0
    assert B._conv_fp32_fma_rate(0, None, None) == 1


def test_overlapping_output_is_refused():
    x, w = synth.conv2d_inputs(S, "f32", "normal", 0, device="cuda")
    st = B.conv2d_forward(x.data_ptr(), w.data_ptr(), x.data_ptr(), desc(S), 0, None, 0, 0, stream())
    assert st == 1
    st = B.conv2d_forward(x.data_ptr(), w.data_ptr(), w.data_ptr(), desc(S), 0, None, 0, 0, stream())
    assert st == 1


def test_null_pointers_are_refused():
    assert B.conv2d_forward(0, 0, 0, desc(S), 0, None, 0, 0, stream()) == 1


def test_empty_batch_is_a_no_op():
    d = desc(synth.Conv2dShape(0, 18, 18, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1)))
    assert B.conv2d_forward(0, 0, 0, d, 0, None, 0, 0, stream()) == 0
    d3 = B.make_desc3d(0, 4, 8, 8, 16, 16, 3, 3, 3, 1, (0, 1, 1), 1)
    assert B.conv3d_forward(0, 0, 0, d3, 2, None, 0, 0, stream()) == 0


def test_invalid_shape_on_device():
    d = desc(synth.Conv2dShape(1, 2, 2, 4, 4, 5, 5))
    assert B.conv2d_forward(1, 1, 1, d, 0, None, 0, 0, stream()) == 1


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_misaligned_pointers_take_the_any_alignment_path(dtype):
    """Inputs that start 2 (16-bit) or 4 (fp32) bytes past a 16-byte boundary:
    no TMA or vector load may touch them; the result is still correct."""
    s = synth.Conv2dShape(2, 13, 11, 24, 40, 3, 3, (1, 1), (1, 1), (1, 1))
    x, w = synth.conv2d_inputs(s, dtype, "normal", 4, device="cuda")
    xb = torch.empty(x.numel() + 8, dtype=x.dtype, device="cuda")
    wb = torch.empty(w.numel() + 8, dtype=w.dtype, device="cuda")
    xm = xb[1:1 + x.numel()].view(x.shape)
    wm = wb[1:1 + w.numel()].view(w.shape)
    xm.copy_(x)
    wm.copy_(w)
    assert xm.data_ptr() % 16 != 0 and wm.data_ptr() % 16 != 0
    out = torch.full((s.n, s.oh, s.ow, s.o), float("nan"), dtype=x.dtype, device="cuda")
    need = B.conv2d_workspace_size(desc(s), B.DTYPE[dtype], 0, None)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    st = B.conv2d_forward(xm.data_ptr(), wm.data_ptr(), out.data_ptr(), desc(s), B.DTYPE[dtype], None,
                          ws.data_ptr(), need, stream())
    assert st == 0
    torch.cuda.synchronize()
    ref = oracle.conv2d(x.cpu(), w.cpu(), dtype, s.stride, s.pad, s.dilation)
    assert_close(as_f64(out), ref, dtype, "misaligned")


def test_forced_winograd_on_other_shapes_is_unsupported():
    s = synth.Conv2dShape(1, 16, 16, 32, 32, 3, 3, (2, 2), (1, 1), (1, 1))
    x, w = synth.conv2d_inputs(s, "f32", "normal", 0, device="cuda")
    with pytest.raises(B.ConvError) as e:
        B.conv2d(x, w, s.stride, s.pad, s.dilation, options=B.make_options("winograd"))
    assert e.value.status == 2


def test_conv_check_is_clean_after_normal_work():
    x, w = synth.conv2d_inputs(S, "bf16", "normal", 0, device="cuda")
    B.conv2d(x, w, S.stride, S.pad, S.dilation)
    assert B.conv_check(stream()) == 0


def test_plan_matches_props_selector():
    p = B.DeviceProps()
    assert B.conv_device_props(0, p) == 0
    assert p.sm_count > 0 and p.total_global_mem > 0
    for shape in (S, synth.WINOGRAD_F32, synth.TINY_WINOGRAD):
        for dt in ("f32", "bf16"):
            a, b = B.ConvPlan(), B.ConvPlan()
            assert B.conv2d_plan(desc(shape), B.DTYPE[dt], 0, None, a) == 0
            assert B.conv2d_plan_for_props(desc(shape), B.DTYPE[dt], p, None, b) == 0
            assert a.as_dict() == b.as_dict()


def test_plan_ignores_current_memory_use():
    """The selector never looks at free memory: allocate a large block and re-plan."""
    before = B.plan2d(desc(synth.WINOGRAD_F32), "f32")
    free, total = torch.cuda.mem_get_info()
    hog = torch.empty(int(min(free * 0.5, 60e9)), dtype=torch.uint8, device="cuda")
    after = B.plan2d(desc(synth.WINOGRAD_F32), "f32")
    del hog
    torch.cuda.empty_cache()
    assert before == after


def test_bounded_wait_reports_timeout_instead_of_hanging():
    """A kernel waits on an mbarrier that nothing completes, with a 2 ms limit:
    it returns, and conv_check reports CONV_ERR_TIMEOUT once, then clears it."""
    s = stream()
    assert B.conv_check(s) == 0
    assert B.conv_selftest_timeout(2_000_000, s) == 0
    assert B.conv_check(s) == 6      # CONV_ERR_TIMEOUT
    assert B.conv_check(s) == 0
    # the context is still usable
    x, w = synth.conv2d_inputs(S, "bf16", "normal", 0, device="cuda")
    B.conv2d(x, w, S.stride, S.pad, S.dilation)
    assert B.conv_check(s) == 0
    assert B.conv_selftest_timeout(10, s) == 1     # limit out of range


def test_bad_out_tensor_is_refused_before_any_launch():
    """The torch conveniences check a caller's out= (shape, dtype, device,
    contiguity) and workspace= (device, size) before a pointer reaches the
    library: each raises ValueError and the poisoned buffers stay untouched
    (no kernel ran)."""
    x, w = synth.conv2d_inputs(S, "f32", "normal", 0, device="cuda")
    good = (S.n, S.oh, S.ow, S.o)
    bad_outs = [
        torch.full((S.n, S.oh, S.ow - 1, S.o), float("nan"), device="cuda"),                # too small
        torch.full((S.n, S.oh, S.ow, S.o + 1), float("nan"), device="cuda"),                # wrong shape
        torch.full(good, float("nan"), dtype=torch.float16, device="cuda"),                 # wrong dtype
        torch.full(good, float("nan")),                                                     # host memory
        torch.full((S.n, S.oh, S.o, S.ow), float("nan"), device="cuda").transpose(2, 3),    # not contiguous
    ]
    for out in bad_outs:
        with pytest.raises(ValueError):
            B.conv2d(x, w, 1, 1, 1, out=out)
    torch.cuda.synchronize()
    for out in bad_outs:
        assert torch.isnan(out.float()).all()
    # conv3d and conv1d take the same checks
    s3 = synth.Conv3dShape(1, 5, 6, 6, 16, 16, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    x3, w3 = synth.conv3d_inputs(s3, "bf16", "normal", 0, device="cuda")
    o3 = torch.full((1, s3.od + 1, s3.oh, s3.ow, s3.o), float("nan"), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        B.conv3d(x3, w3, 1, (0, 1, 1), 1, out=o3)
    x1, w1 = synth.make_inputs((2, 50, 16), (24, 3, 16), "f32", "normal", 0, device="cuda")
    o1 = torch.full((2, 47, 24), float("nan"), device="cuda")
    with pytest.raises(ValueError):
        B.conv1d(x1, w1, 1, 0, 1, out=o1)
    # a workspace smaller than the plan's, or on the host
    opts = B.make_options("winograd")
    need = B.conv2d_workspace_size(desc(S), 0, 0, opts)
    out = torch.full(good, float("nan"), device="cuda")
    for ws in (torch.empty(need - 1, dtype=torch.uint8, device="cuda"), torch.empty(need, dtype=torch.uint8)):
        with pytest.raises(ValueError):
            B.conv2d(x, w, 1, 1, 1, options=opts, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(o3.float()).all() and torch.isnan(o1).all()


def test_plan_log_line(capfd, monkeypatch):
    """B200CONV_LOG=1 (read on every call) prints one stderr line per forward call
    with the shape, the dtype and the plan that runs; unset or 0 prints nothing."""
    s = synth.Conv2dShape(2, 20, 20, 64, 96, 3, 3, (1, 1), (1, 1), (1, 1))
    x, w = synth.conv2d_inputs(s, "bf16", "normal", 0, device="cuda")
    capfd.readouterr()
    monkeypatch.setenv("B200CONV_LOG", "1")
    B.conv2d(x, w, 1, 1, 1)
    B.conv2d(x.float(), w.float(), 1, 1, 1, options=B.make_options("winograd"))
    torch.cuda.synchronize()
    lines = [ln for ln in capfd.readouterr().err.splitlines() if ln.startswith("b200conv: ")]
    assert len(lines) == 2, lines
    assert "conv2d n2 20x20 64->96 k3x3 s1,1 p1,1 d1,1 bf16" in lines[0]
    assert "algo=implicit engine=tcgen05" in lines[0] and "workspace=" in lines[0]
    assert " f32 " in lines[1] and "algo=winograd engine=simt" in lines[1] and "winograd_m=6" in lines[1]
    monkeypatch.setenv("B200CONV_LOG", "0")
    B.conv2d(x, w, 1, 1, 1)
    torch.cuda.synchronize()
    assert "b200conv: " not in capfd.readouterr().err
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
