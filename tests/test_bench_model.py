"""The benchmark's algorithmic-work model, the numerator of every roofline
figure it reports (CPU only).

Each kernel's FLOPs and bytes per call are checked against the closed forms
written out by hand here for the plans the library selects: the default
Winograd workload, a 16-bit implicit GEMM, the 16-bit Winograd (M in the
operand type), the native 3D Winograd and conv3d depth taps.
"""
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from dense_convolution_nhwc_b200 import binding as B  # noqa: E402
from dense_convolution_nhwc_b200 import synth  # noqa: E402

PROPS = B.DeviceProps(148, 10, 0, 183359 * 2 ** 20)


def plan2d(s, dt, algo="auto"):
    desc = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
    p = B.ConvPlan()
    assert B.conv2d_plan_for_props(desc, B.DTYPE[dt], PROPS, B.make_options(algo), p) == 0
    return p.as_dict()


def plan3d(s, dt, algo="auto"):
    desc = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
    p = B.ConvPlan()
    assert B.conv3d_plan_for_props(desc, B.DTYPE[dt], PROPS, B.make_options(algo), p) == 0
    return p.as_dict()


def test_default_workload_winograd_fp32():
    """40 x 512 x 512, 192 -> 96: F(6x6,3x3), T = 40 * 86 * 86 tiles, alpha^2 = 64,
    on the persistent kernel: the GEMM's FLOPs; input, output and the V / M
    round trips through its scratch."""
    s = synth.WINOGRAD_F32
    p = plan2d(s, "f32")
    p["winograd_fused"] = 1
    w = bench.kernel_work(bench.Conv(s, "f32", "uniform"), p)
    T = 40 * 86 * 86
    assert set(w) == {"wino_filter", "wino_fused"}
    assert w["wino_fused"][0] == 2.0 * 64 * T * 192 * 96
    assert w["wino_fused"][1] == (40 * 512 * 512 * (192 + 96) + 2 * 64 * T * (192 + 96)) * 4
    assert bench.kernel_bound("wino_fused") == "alu"


def test_default_workload_winograd_fp32_three_launches():
    """The same shape in three launches (the default plan)."""
    s = synth.WINOGRAD_F32
    p = plan2d(s, "f32")
    assert p["winograd_fused"] == 0
    w = bench.kernel_work(bench.Conv(s, "f32", "uniform"), p)
    T = 40 * 86 * 86
    assert w["wino_gemm_simt"][0] == 2.0 * 64 * T * 192 * 96
    assert w["wino_gemm_simt"][1] == 64 * T * (192 + 96) * 4            # V read + M write
    assert w["wino_input"][1] == 40 * 512 * 512 * 192 * 4 + 64 * T * 192 * 4
    assert w["wino_output"][1] == 64 * T * 96 * 4 + 40 * 512 * 512 * 96 * 4
    # the direct-equivalent FLOPs the metric counts
    assert s.flops == 2 * 40 * 512 * 512 * 96 * 192 * 9


def test_sixteen_bit_implicit_gemm():
    s = synth.Conv2dShape(32, 64, 64, 512, 2048, 3, 3, (1, 1), (1, 1), (1, 1))
    p = plan2d(s, "bf16", "implicit")
    w = bench.kernel_work(bench.Conv(s, "bf16", "normal"), p)
    M, K = 32 * 64 * 64, 512 * 9
    assert w == {"tc_conv": (2.0 * M * 2048 * K, (32 * 64 * 64 * 512 + 2048 * K + M * 2048) * 2)}


def test_sixteen_bit_winograd_m_in_operand_type():
    s = synth.Conv2dShape(16, 64, 64, 1024, 1024, 3, 3, (1, 1), (1, 1), (1, 1))
    p = plan2d(s, "bf16")
    assert p["algo"] == "winograd" and p["winograd_m"] == 2
    w = bench.kernel_work(bench.Conv(s, "bf16", "normal"), p)
    T = 16 * 32 * 32
    assert w["wino_gemm_tc"] == (2.0 * 16 * T * 1024 * 1024, 16 * T * (1024 + 1024) * 2)
    assert w["wino_output"][1] == 16 * T * 1024 * 2 + 16 * 64 * 64 * 1024 * 2


def test_native_3d_winograd():
    s = synth.CONV3D_TAPS[1]          # 41 x 60 x 104, 256 -> 256
    p = plan3d(s, "f32")
    assert p["algo"] == "winograd" and p["winograd_m"] == 4
    w = bench.kernel_work(bench.Conv(s, "f32", "normal"), p)
    T = math.ceil(39 / 4) * math.ceil(60 / 4) * math.ceil(104 / 4)
    assert w["wino3d_gemm_simt"][0] == 2.0 * 216 * T * 256 * 256
    # 8x fewer multiplies than direct, up to the ragged depth tile (40 frames for 39)
    assert w["wino3d_gemm_simt"][0] == pytest.approx(s.flops / 8 * 40 / 39)


def test_conv3d_depth_taps_count_every_tap():
    s = synth.CONV3D_TAPS[0]          # 17 x 64 x 64, 256 -> 256, KD = 3
    p = plan3d(s, "bf16")
    assert p["taps"] == 3 and p["algo"] == "implicit"
    w = bench.kernel_work(bench.Conv(s, "bf16", "normal"), p)
    assert w["tc_conv"][0] == s.flops
    out_b = s.od * s.oh * s.ow * s.o * 2
    tap_b = (s.od * s.h * s.w * s.c + s.o * 9 * s.c + s.od * s.oh * s.ow * s.o) * 2   # frames in, slice, out
    assert w["tc_conv"][1] == 3 * tap_b + 2 * out_b     # taps 2 and 3 also read the output they add into


def test_per_config_block_covers_every_config():
    """The bench's per-config block measures configs 1, 3, 4 and 5 beside the
    config-2 headline, every dtype the configs name, and every workload it
    names resolves (no device needed)."""
    keys = [k for k, *_ in bench.PER_CONFIG]
    for cfg in ("config1_", "config2_", "config3_", "config4_", "config5_"):
        assert any(k.startswith(cfg) for k in keys), cfg
    seen = set()
    for key, wl, algo, _, *env in bench.PER_CONFIG:
        desc, convs, dt = bench.workload(wl)
        assert convs and algo in ("auto", "implicit", "winograd", "direct")
        seen.add((key.split("_")[0], dt))
    assert {("config3", "f16"), ("config3", "bf16"), ("config4", "f16"), ("config4", "bf16"),
            ("config5", "bf16"), ("config1", "f32")} <= seen
    # the wide-channel members: C_out >= 512 and M >= 16384, stride 1, dilation 1
    _, convs, _ = bench.workload("wide_bf16")
    assert all(c.shape.o >= 512 and c.shape.n * c.shape.oh * c.shape.ow >= 16384 for c in convs)
    assert all(c.shape.stride == (1, 1) and c.shape.dilation == (1, 1) for c in convs)


def test_split_bf16_work_counts_the_bf16_products():
    """The split-bf16 GEMM route's roofline counts the tensor cores' six bf16
    products per fp32 product; the conv's own FLOPs (the metric) do not change."""
    s = synth.WINOGRAD_F32
    p = plan2d(s, "f32")
    p["engine"] = "tcgen05"
    p["winograd_split_bf16"] = 1
    w = bench.kernel_work(bench.Conv(s, "f32", "uniform"), p)
    T = 40 * 86 * 86
    assert w["wino_gemm_tc"][0] == 6 * 2.0 * 64 * T * 192 * 96
    assert w["wino_gemm_tc"][1] == 64 * T * (3 * 192 * 2 + 96 * 4)
    assert bench.kernel_bound("wino_gemm_tc") == "tensor"
