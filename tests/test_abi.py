"""The C-ABI library without a GPU: it loads, exports every symbol that
include/b200conv.h declares, and its selector behaves as a pure function of
(shape, dtype, constant device properties, options).

The selector follows "Bound winograd conv2d working set by tiling the batch"
(Fix): Winograd batch tiles sized from a budget of 3/4 of device memory minus
the conv's own tensors (capped at 8 GiB here), a fallback to the scratch-free
implicit GEMM when no image fits or tiles carry too few GEMM rows, a forced
tile size capped by the budget, and no dependence on current free memory.
"""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import dense_convolution_nhwc_b200 as dc
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "b200conv.h")

B200 = B.DeviceProps(148, 10, 0, 183359 * 2 ** 20)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"B200CONV_API[^;(]*?\b(conv\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for name in ["conv2d_forward", "conv3d_forward", "conv2d_plan", "conv3d_plan", "conv2d_workspace_size",
                 "conv3d_workspace_size", "conv_status_string", "conv_check", "conv_accumulate",
                 "conv2d_plan_for_props", "conv3d_plan_for_props", "conv_device_props"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(B.library_path)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing, missing


def test_binding_has_the_same_names():
    for s in declared_symbols():
        assert callable(getattr(dc, s)), s


def test_status_strings():
    for code in range(7):
        assert B.conv_status_string(code)
    assert B.conv_status_string(4) == "workspace too small"


def plan2d(shape: synth.Conv2dShape, dtype="f32", **opt):
    desc = B.make_desc2d(shape.n, shape.h, shape.w, shape.c, shape.o, shape.kh, shape.kw,
                         shape.stride, shape.pad, shape.dilation)
    p = B.ConvPlan()
    st = B.conv2d_plan_for_props(desc, B.DTYPE[dtype], B200, B.make_options(**opt) if opt else B.make_options(), p)
    return st, p.as_dict()


def test_winograd_shape_plan(monkeypatch):
    """40 x 512 x 512, 192 -> 96, fp32, in three launches: F(6x6,3x3), per-image
    scratch 64 * 86^2 * (192 + 96) * 4 bytes = 545 MB, so an 8 GiB budget gives
    batch tiles of 15 images (15, 15, 10)."""
    monkeypatch.setenv("B200CONV_WINOGRAD_FUSED", "0")
    st, p = plan2d(synth.WINOGRAD_F32)
    assert st == 0
    assert p["algo"] == "winograd" and p["winograd_m"] == 6 and p["engine"] == "simt"
    assert p["winograd_fused"] == 0
    assert p["batch_tile"] == 15 and p["num_batch_tiles"] == 3
    per_img = 64 * 86 * 86 * (192 + 96) * 4
    assert p["workspace_bytes"] >= 15 * per_img
    assert p["workspace_bytes"] < 15 * per_img + 64 * 192 * 96 * 4 + 4096


def test_winograd_fused_plan(monkeypatch):
    """The same shape on the persistent kernel (B200CONV_WINOGRAD_FUSED=1):
    untiled, one CTA per SM, each holding two V and two M buffers of a 128-tile
    block: 148 * 2 * 64 * 128 * (192 + 96) * 4 bytes after U (64 * 192 * 96 * 4)."""
    assert plan2d(synth.WINOGRAD_F32)[1]["winograd_fused"] == 0      # off by default
    monkeypatch.setenv("B200CONV_WINOGRAD_FUSED", "1")
    st, p = plan2d(synth.WINOGRAD_F32)
    assert st == 0
    assert p["algo"] == "winograd" and p["winograd_m"] == 6 and p["engine"] == "simt"
    assert p["winograd_fused"] == 1 and p["batch_tile"] == 40 and p["num_batch_tiles"] == 1
    u = 64 * 192 * 96 * 4
    scratch = 148 * 2 * 64 * 128 * (192 + 96) * 4
    assert p["workspace_bytes"] == -(-u // 256) * 256 + -(-scratch // 256) * 256


def test_winograd_fused_rules(monkeypatch):
    """Not for 16-bit inputs, a forced batch tile, or a budget below the per-CTA
    scratch; the test hook turns it on and off."""
    big = synth.WINOGRAD_F32
    small = synth.Conv2dShape(2, 40, 40, 64, 64, 3, 3, (1, 1), (1, 1), (1, 1))
    monkeypatch.setenv("B200CONV_WINOGRAD_FUSED", "1")
    assert plan2d(big, "f16")[1]["winograd_fused"] == 0
    assert plan2d(big, winograd_tile_batch=8)[1]["winograd_fused"] == 0
    st, p = plan2d(big, winograd_budget_bytes=2 * 2 ** 30)                    # 2.79 GB of scratch does not fit
    assert st == 0 and p["winograd_fused"] == 0 and p["batch_tile"] == 3
    st, p = plan2d(small, algo="winograd")
    assert st == 0 and p["winograd_fused"] == 1
    assert p["workspace_bytes"] == -(-64 * 64 * 64 * 4 // 256) * 256 + 2 * 64 * 128 * (64 + 64) * 4
    monkeypatch.setenv("B200CONV_WINOGRAD_FUSED", "0")
    assert plan2d(big)[1]["winograd_fused"] == 0


def test_winograd_split_bf16_plan(monkeypatch):
    """The fp32 Winograd GEMM over split-bf16 operands (B200CONV_WINOGRAD_SPLIT_BF16=1,
    off by default): the tcgen05 engine on 96-column tiles for O = 96, and a workspace
    of U [64][O][3C] and V [64][T][3C] in bf16 plus M [64][T][O] in fp32.  The batch
    tile comes from the same 8 GiB budget: 64 * 7396 * (192 * 6 + 96 * 4) bytes per
    image gives 11 images (11, 11, 11, 7)."""
    monkeypatch.delenv("B200CONV_WINOGRAD_FUSED", raising=False)
    assert plan2d(synth.WINOGRAD_F32)[1]["winograd_split_bf16"] == 0
    monkeypatch.setenv("B200CONV_WINOGRAD_SPLIT_BF16", "1")
    st, p = plan2d(synth.WINOGRAD_F32)
    assert st == 0
    assert p["algo"] == "winograd" and p["engine"] == "tcgen05" and p["winograd_m"] == 6
    assert p["winograd_split_bf16"] == 1 and p["winograd_fused"] == 0
    assert p["tile_n"] == 96 and p["tile_m"] == 128
    tiles = 86 * 86
    nb = (8 * 2 ** 30) // (64 * tiles * (192 * 6 + 96 * 4))
    assert nb == 11 and p["batch_tile"] == nb and p["num_batch_tiles"] == 4
    t = nb * tiles

    def al(x):
        return -(-x // 256) * 256

    assert p["workspace_bytes"] == al(64 * 96 * 192 * 6) + al(64 * t * 192 * 6) + al(64 * t * 96 * 4)
    # O > 96: 128-column tiles
    wide = synth.Conv2dShape(2, 64, 64, 64, 128, 3, 3, (1, 1), (1, 1), (1, 1))
    st, p = plan2d(wide, algo="winograd")
    assert st == 0 and p["winograd_split_bf16"] == 1 and p["tile_n"] == 128


def test_winograd_split_bf16_rules(monkeypatch):
    """Only fp32 inputs with C % 64 == 0 and O % 4 == 0 on a compute-capability-10
    device take it, and the persistent fp32 kernel's hook takes precedence."""
    monkeypatch.delenv("B200CONV_WINOGRAD_FUSED", raising=False)
    monkeypatch.setenv("B200CONV_WINOGRAD_SPLIT_BF16", "1")
    big = synth.WINOGRAD_F32
    assert plan2d(big, "f16")[1]["winograd_split_bf16"] == 0
    assert plan2d(big, "bf16")[1]["winograd_split_bf16"] == 0
    for c, o in ((96, 96), (64, 98)):
        s = synth.Conv2dShape(2, 40, 40, c, o, 3, 3, (1, 1), (1, 1), (1, 1))
        st, p = plan2d(s, algo="winograd")
        assert st == 0 and p["algo"] == "winograd" and p["winograd_split_bf16"] == 0 and p["engine"] == "simt"
    desc = B.make_desc2d(big.n, big.h, big.w, big.c, big.o, big.kh, big.kw, big.stride, big.pad, big.dilation)
    p = B.ConvPlan()
    hopper = B.DeviceProps(132, 9, 0, 80 * 2 ** 30)
    assert B.conv2d_plan_for_props(desc, B.DTYPE["f32"], hopper, B.make_options(), p) == 0
    assert p.as_dict()["winograd_split_bf16"] == 0
    monkeypatch.setenv("B200CONV_WINOGRAD_FUSED", "1")
    st, p = plan2d(big)
    assert st == 0 and p["winograd_split_bf16"] == 0 and p["winograd_fused"] == 1


def test_small_shape_takes_implicit_gemm():
    st, p = plan2d(synth.SMALL_F32)       # C + O = 64 < 256
    assert st == 0 and p["algo"] == "implicit" and p["engine"] == "simt"
    assert (p["workspace_bytes"] == 0) == (p["k_split"] == 1)


@pytest.mark.parametrize("budget,expect", [
    (2 * 2 ** 30, ("winograd", 3)),        # 3 images/tile
    (2 ** 30, ("winograd", 1)),            # 1 image/tile = 7396 GEMM rows per point: still Winograd (fp32)
    (2 ** 20, ("implicit", None)),         # not even one image fits
])
def test_budget_injection(budget, expect):
    st, p = plan2d(synth.WINOGRAD_F32, winograd_budget_bytes=budget)
    assert st == 0 and p["algo"] == expect[0]
    if expect[1]:
        assert p["batch_tile"] == expect[1]


@pytest.mark.parametrize("forced,nb,tiles", [(1, 1, 40), (7, 7, 6), (40, 15, 3), (15, 15, 3)])
def test_forced_tile_is_capped_by_budget(forced, nb, tiles):
    st, p = plan2d(synth.WINOGRAD_F32, winograd_tile_batch=forced)
    assert st == 0 and p["algo"] == "winograd"
    assert p["batch_tile"] == nb and p["num_batch_tiles"] == tiles


def test_tiny_spatial_shape_falls_back_with_one_image_tiles():
    """256 x 4 x 4, 64 -> 192: cut into one-image Winograd tiles it is the
    page's ~40x-slower case, so the selector takes the implicit GEMM."""
    per_img = 64 * 1 * (64 + 192) * 4
    st, p = plan2d(synth.TINY_WINOGRAD, winograd_budget_bytes=per_img)
    assert st == 0 and p["algo"] == "implicit"
    st, p = plan2d(synth.TINY_WINOGRAD)   # whole batch fits: untiled Winograd
    assert st == 0 and p["algo"] == "winograd" and p["num_batch_tiles"] == 1


def test_few_channel_tap_packing_choice():
    """A few-channel input folds every tap into channels when KH*KW*C <= 192
    (at most three 64-wide K steps), only the KW taps when KW*C <= 64 and the
    window is larger, else pads the channels to a multiple of 8."""
    cases = [((1, 32, 32, 3, 64, 7, 7), 2, 152), ((1, 32, 32, 3, 16, 3, 3), 2, 32), ((1, 32, 32, 5, 16, 5, 5), 2, 128),
             ((1, 32, 32, 6, 16, 7, 7), 1, 48), ((1, 32, 32, 12, 16, 1, 1), 0, 16)]
    for (n, h, w, c, o, kh, kw), packed, cp in cases:
        s = synth.Conv2dShape(n, h, w, c, o, kh, kw, (1, 1), (kh // 2, kw // 2), (1, 1))
        st, p = plan2d(s, "bf16")
        assert st == 0 and p["engine"] == "tcgen05", s
        assert p["packed_taps"] == packed and p["channel_pad"] == cp, (s, p)


def test_sixteen_bit_takes_tensor_cores():
    for name, shape, _ in synth.resnet50_layers(8):
        for dt in ("f16", "bf16"):
            st, p = plan2d(shape, dt)
            assert st == 0 and p["algo"] == "implicit" and p["engine"] == "tcgen05", name
            if shape.c == 3:      # the stem: 7 x 7 taps x 3 channels folded into 152 channels, a 1x1 conv
                assert p["channel_pad"] == 152 and p["packed_taps"] == 2 and p["workspace_bytes"] > 0
            else:
                assert p["channel_pad"] == 0 and (p["workspace_bytes"] == 0) == (p["k_split"] == 1)


def test_sixteen_bit_auto_winograd_only_for_deep_wide_gemms():
    """16-bit auto takes F(2,3) on the tensor cores where it measured faster
    than the implicit GEMM: C >= 1024 with O >= 1024, or C >= 512 with O >= 2048."""
    for (c, o), want in [((1024, 1024), True), ((1024, 4096), True), ((512, 2048), True), ((1024, 512), False),
                         ((512, 1024), False), ((256, 4096), False), ((2048, 2048), True)]:
        s = synth.Conv2dShape(16, 64, 64, c, o, 3, 3, (1, 1), (1, 1), (1, 1))
        for dt in ("bf16", "f16"):
            st, p = plan2d(s, dt)
            assert st == 0 and (p["algo"] == "winograd") == want, (c, o, dt, p["algo"])
            assert p["engine"] == "tcgen05"
            if want:
                assert p["winograd_m"] == 2
    # stride 2 or a 5x5 filter never takes it
    for s in (synth.Conv2dShape(16, 64, 64, 1024, 1024, 3, 3, (2, 2), (1, 1), (1, 1)),
              synth.Conv2dShape(16, 64, 64, 1024, 1024, 5, 5, (1, 1), (2, 2), (1, 1))):
        st, p = plan2d(s, "bf16")
        assert st == 0 and p["algo"] == "implicit"


def test_sixteen_bit_forced_winograd_uses_f2x2():
    """F(2x2,3x3) on the tensor cores, with U, V and M all in the 16-bit type:
    workspace = 16 * (O*C + T*C + T*O) * 2 bytes (each buffer 256-aligned)."""
    s = synth.Conv2dShape(2, 32, 32, 256, 192, 3, 3, (1, 1), (1, 1), (1, 1))
    for dt in ("bf16", "f16"):
        st, p = plan2d(s, dt, algo="winograd")
        assert st == 0 and p["algo"] == "winograd" and p["winograd_m"] == 2 and p["engine"] == "tcgen05"
        al = lambda x: (x + 255) // 256 * 256
        T = 2 * 16 * 16
        assert p["workspace_bytes"] == al(16 * 192 * 256 * 2) + al(16 * T * 256 * 2) + al(16 * T * 192 * 2)


def test_forced_winograd_rejects_other_shapes():
    st, _ = plan2d(synth.Conv2dShape(1, 16, 16, 32, 32, 5, 5, (1, 1), (2, 2), (1, 1)), algo="winograd")
    assert st == 2   # CONV_ERR_UNSUPPORTED


@pytest.mark.parametrize("shape", [
    synth.Conv2dShape(1, 2, 2, 4, 4, 5, 5),                          # OH <= 0
    synth.Conv2dShape(1, 8, 8, 4, 4, 3, 3, (0, 1)),                  # zero stride
    synth.Conv2dShape(1, 8, 8, 4, 4, 3, 3, (1, 1), (-1, 0)),         # negative pad
    synth.Conv2dShape(1, 8, 8, 0, 4, 3, 3),                          # no channels
    synth.Conv2dShape(1, 8, 8, 4, 4, 3, 3, (1, 1), (0, 0), (0, 1)),  # zero dilation
])
def test_invalid_descriptors(shape):
    st, _ = plan2d(shape)
    assert st == 1   # CONV_ERR_INVALID


def test_plan_is_pure_across_calls_and_processes():
    shapes = [synth.WINOGRAD_F32, synth.SMALL_F32, synth.TINY_WINOGRAD] + [s for _, s, _ in synth.resnet50_layers(1)]
    first = [plan2d(s, dt) for s in shapes for dt in ("f32", "bf16")]
    again = [plan2d(s, dt) for s in shapes for dt in ("f32", "bf16")]
    assert first == again
    code = ("import sys; sys.path.insert(0, %r); from tests import test_abi as t; from dense_convolution_nhwc_b200 import synth; "
            "print(repr([t.plan2d(s, dt) for s in [synth.WINOGRAD_F32, synth.SMALL_F32, synth.TINY_WINOGRAD] + "
            "[s for _, s, _ in synth.resnet50_layers(1)] for dt in ('f32', 'bf16')]))" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, check=True, cwd=ROOT)
    assert out.stdout.strip() == repr(first)


def test_environment_hooks_apply_only_without_options():
    desc = B.make_desc2d(40, 512, 512, 192, 96, 3, 3, 1, 1, 1)
    code = ("import sys; sys.path.insert(0, %r); from dense_convolution_nhwc_b200 import binding as B; "
            "d = B.make_desc2d(40, 512, 512, 192, 96, 3, 3, 1, 1, 1); p = B.ConvPlan(); "
            "B.conv2d_plan_for_props(d, 0, B.DeviceProps(148, 10, 0, 183359 * 2 ** 20), None, p); "
            "print(p.as_dict()['algo'], p.as_dict()['batch_tile'])" % ROOT)
    env = dict(os.environ, B200CONV_WINOGRAD_TILE_BATCH="7")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, check=True, env=env, cwd=ROOT)
    assert out.stdout.split() == ["winograd", "7"]
    env = dict(os.environ, B200CONV_ALGO="direct")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, check=True, env=env, cwd=ROOT)
    assert out.stdout.split()[0] == "direct"
    env = dict(os.environ, B200CONV_WINOGRAD_WORKSPACE_BYTES=str(2 ** 20))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, check=True, env=env, cwd=ROOT)
    assert out.stdout.split()[0] == "implicit"


def test_conv3d_plan_depth_taps():
    for s in synth.CONV3D_TAPS:
        desc = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
        p = B.ConvPlan()
        assert B.conv3d_plan_for_props(desc, B.DTYPE["bf16"], B200, None, p) == 0
        d = p.as_dict()
        assert d["taps"] == 3 and d["engine"] == "tcgen05"
        assert d["workspace_bytes"] == 0       # taps add into out in their own epilogue: no scratch


def test_conv3d_invalid():
    desc = B.make_desc3d(1, 2, 8, 8, 4, 4, 3, 3, 3, 1, (0, 1, 1), 1)     # OD <= 0
    p = B.ConvPlan()
    assert B.conv3d_plan_for_props(desc, 0, B200, None, p) == 1


def plan3d(s, dtype="bf16", **opt):
    desc = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    p = B.ConvPlan()
    st = B.conv3d_plan_for_props(desc, B.DTYPE[dtype], B200, B.make_options(**opt) if opt else B.make_options(), p)
    return st, p.as_dict()


def test_conv3d_guard_selects_depth_taps_or_native_gemm():
    """The depth-tap page's guard keeps the taps; what it sends elsewhere goes to
    the native K-fused 3D GEMM (16-bit) when a 5D im2col map can express it."""
    guarded = synth.Conv3dShape(1, 9, 16, 16, 64, 64, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    st, p = plan3d(guarded)
    assert st == 0 and p["taps"] == 3
    for other in [synth.Conv3dShape(2, 9, 16, 16, 64, 64, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),   # N > 1
                  synth.Conv3dShape(1, 9, 16, 16, 64, 64, 3, 3, 3, (2, 1, 1), (0, 1, 1), (1, 1, 1)),   # depth stride
                  synth.Conv3dShape(1, 9, 16, 16, 64, 64, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1)),   # depth pad
                  synth.Conv3dShape(1, 12, 8, 8, 64, 64, 9, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))]:  # KD > 7
        st, p = plan3d(other)
        assert st == 0 and p["taps"] == 1 and p["engine"] == "tcgen05" and p["workspace_bytes"] == 0, other
        st, p = plan3d(other, "f32")                 # fp32: always depth taps (FFMA)
        assert st == 0 and p["taps"] == other.kd
    # a depth pad beyond the 5D box-corner range stays on depth taps
    st, p = plan3d(synth.Conv3dShape(1, 40, 8, 8, 64, 64, 3, 3, 3, (1, 1, 1), (17, 1, 1), (1, 1, 1)))
    assert st == 0 and p["taps"] == 3
    # forcing the implicit GEMM takes the native kernel even inside the guard
    st, p = plan3d(guarded, algo="implicit")
    assert st == 0 and p["taps"] == 1


def wino3d_ws(s, m, store_bytes, ffma, nu):
    """U + V + M bytes of the 3D Winograd workspace for batch tiles of nu units."""
    al = lambda x: (x + 255) // 256 * 256
    a3 = (m + 2) ** 3
    tiles_hw = -(-s.oh // m) * -(-s.ow // m)
    t = nu * tiles_hw
    o_u = (s.o + 3) // 4 * 4 if ffma else s.o
    return al(a3 * s.c * o_u * store_bytes) + al(a3 * t * s.c * store_bytes) + al(a3 * t * s.o * 4)


def test_conv3d_winograd_plan():
    """fp32 3x3x3 stride-1 convs under the channel rule take the native 3D
    Winograd F(4,3)^3 on the FFMA GEMM; 16-bit keeps the taps / native GEMM
    unless Winograd is forced, which gives F(2,3)^3 on the tensor cores."""
    s = synth.Conv3dShape(2, 17, 32, 32, 128, 128, 3, 3, 3, (1, 1, 1), (1, 1, 1), (1, 1, 1))
    units = 2 * -(-s.od // 4)
    st, p = plan3d(s, "f32")
    assert st == 0 and p["algo"] == "winograd" and p["winograd_m"] == 4 and p["taps"] == 1
    assert p["engine"] == "simt" and p["batch_tile"] == units and p["num_batch_tiles"] == 1
    assert p["workspace_bytes"] == wino3d_ws(s, 4, 4, True, units)
    st, p = plan3d(s, "bf16")
    assert st == 0 and p["algo"] != "winograd"
    for dt in ("bf16", "f16"):
        st, p = plan3d(s, dt, algo="winograd")
        assert st == 0 and p["algo"] == "winograd" and p["winograd_m"] == 2 and p["engine"] == "tcgen05"
        assert p["workspace_bytes"] == wino3d_ws(s, 2, 2, False, p["batch_tile"])
    # channel rule (auto): C + O < 256 stays on depth taps; forcing ignores the rule
    small = synth.Conv3dShape(1, 6, 8, 8, 32, 64, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    st, p = plan3d(small, "f32")
    assert st == 0 and p["taps"] == 3
    st, p = plan3d(small, "f32", algo="winograd")
    assert st == 0 and p["algo"] == "winograd" and p["taps"] == 1 and p["winograd_m"] == 4
    # not 3x3x3 / stride 1 / dilation 1: depth taps (forced Winograd: each tap's 2D Winograd)
    for other in [synth.Conv3dShape(1, 9, 16, 16, 128, 128, 2, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1)),
                  synth.Conv3dShape(1, 9, 16, 16, 128, 128, 3, 3, 3, (2, 1, 1), (0, 1, 1), (1, 1, 1)),
                  synth.Conv3dShape(1, 9, 16, 16, 128, 128, 3, 3, 3, (1, 1, 1), (2, 1, 1), (2, 1, 1))]:
        st, p = plan3d(other, "f32", algo="winograd")
        assert st == 0 and p["taps"] == other.kd and p["winograd_m"] == 6, other
    # C % 4 != 0: no 3D Winograd even when forced
    odd = synth.Conv3dShape(1, 6, 8, 8, 6, 32, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    st, p = plan3d(odd, "f32", algo="winograd")
    assert st == 0 and p["taps"] == 3


def test_conv3d_winograd_budget_tiles_units():
    """The budget bounds V + M per unit (one image's depth tile of m frames); a
    forced tile is capped by it; tiles of fewer than four 128-row GEMM tiles per
    point (all alpha^3 points run in one batched launch), or a budget under one
    unit, fall back to the depth taps."""
    s = synth.Conv3dShape(1, 42, 64, 64, 64, 256, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))   # OD = 40: 10 units
    per_unit = 216 * (16 * 16) * (64 * 4 + 256 * 4)
    st, p = plan3d(s, "f32", winograd_budget_bytes=3 * per_unit + 5, winograd_tile_batch=10)
    assert st == 0 and p["algo"] == "winograd" and p["batch_tile"] == 3 and p["num_batch_tiles"] == 4
    assert p["workspace_bytes"] == wino3d_ws(s, 4, 4, True, 3)
    st, p = plan3d(s, "f32", winograd_budget_bytes=3 * per_unit, winograd_tile_batch=2)
    assert st == 0 and p["batch_tile"] == 2 and p["num_batch_tiles"] == 5
    st, p = plan3d(s, "f32", winograd_budget_bytes=3 * per_unit)      # 3 * 256 = 768 rows per point >= 512
    # 10 units in tiles of at most 3: four tiles, evened out to 3, 3, 3, 1
    assert st == 0 and p["algo"] == "winograd" and p["taps"] == 1 and p["batch_tile"] == 3
    st, p = plan3d(s, "f32", winograd_budget_bytes=6 * per_unit)      # two tiles: 5 + 5, not 6 + 4
    assert st == 0 and p["batch_tile"] == 5 and p["num_batch_tiles"] == 2
    st, p = plan3d(s, "f32", winograd_budget_bytes=per_unit)          # 256 rows per point < 512
    assert st == 0 and p["taps"] == 3 and p["winograd_m"] != 4        # depth taps (each a 2D Winograd)
    st, p = plan3d(s, "f32", winograd_budget_bytes=per_unit - 1, winograd_tile_batch=1)
    assert st == 0 and p["taps"] == 3
    big = synth.Conv3dShape(1, 42, 256, 256, 64, 256, 3, 3, 3, (1, 1, 1), (0, 1, 1), (1, 1, 1))
    per_unit = 216 * (64 * 64) * (64 * 4 + 256 * 4)
    st, p = plan3d(big, "f32", winograd_budget_bytes=4 * per_unit)    # 4 * 4096 rows per point; tiles of 4, 4, 2 units
    assert st == 0 and p["algo"] == "winograd" and p["batch_tile"] == 4 and p["num_batch_tiles"] == 3


def test_split_k_for_small_m_long_k():
    """Under half a wave of tiles with a long K loop: the K range is split and
    the workspace holds the fp32 partials; large grids are never split."""
    small = synth.Conv2dShape(8, 14, 14, 512, 512, 3, 3, (2, 2), (1, 1), (1, 1))     # M = 392, K = 4608
    for dt, tile in (("bf16", 128), ("f32", 128)):
        st, p = plan2d(small, dt)
        assert st == 0 and p["k_split"] >= 2
        M = 8 * 7 * 7
        assert p["workspace_bytes"] >= p["k_split"] * M * 512 * 4
    big = synth.Conv2dShape(16, 64, 64, 512, 512, 3, 3, (1, 1), (1, 1), (1, 1))
    for dt in ("bf16", "f32"):
        st, p = plan2d(big, dt, algo="implicit")
        assert st == 0 and p["k_split"] == 1 and p["workspace_bytes"] == 0
    # Winograd plans never split (bit identity of batch tiling)
    st, p = plan2d(synth.WINOGRAD_F32)
    assert p["algo"] == "winograd" and p["k_split"] == 1


def test_binding_out_checks_need_no_gpu():
    """The out= / workspace= checks of the torch conveniences reject host
    tensors and non-tensors without touching a device."""
    import torch
    x = torch.zeros(2, 3)
    for bad in (None, 3, "out"):
        if bad is None:
            continue
        with pytest.raises(ValueError):
            B._check_out(bad, (2, 3), x)
        with pytest.raises(ValueError):
            B._check_workspace(bad, 16, x)
    with pytest.raises(ValueError):
        B._check_out(torch.zeros(2, 3), (2, 3), x)        # host memory is never a valid out
    with pytest.raises(ValueError):
        B._check_workspace(torch.zeros(64, dtype=torch.uint8), 16, x)
