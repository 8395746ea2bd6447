"""The bench's roofline arithmetic and clock record without a GPU.

For the dominant kernel of a step the bench reports the kernel's algorithmic
work per launch (its FLOPs or bytes, from the plan the library will run) over
its event-timed duration per launch, the peak it is judged against (the
measured peaks when present, else the fallback figures; the FP32 probe for
FFMA kernels), the sustained and shape-bound fractions of a tensor kernel, and
the ncu DRAM traffic only while the kernel's sources are unchanged since the
capture.  Here the plans come from the selector with constant B200 properties
and the event times are synthetic, so every figure has a closed form.
"""
import pytest

import bench
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth

PROPS = B.DeviceProps(148, 10, 0, 183359 * 2 ** 20)


class PlannedWorkload:
    """A bench workload planned on the CPU: the items the bench's work model reads."""

    work = bench.Bench.work
    per_conv_work = bench.Bench.per_conv_work

    def __init__(self, wl_name, algo="auto"):
        _, convs, _ = bench.workload(wl_name)
        opts = B.make_options(algo)
        self.items = []
        for cv in convs:
            s = cv.shape
            p = B.ConvPlan()
            if cv.is3d:
                d = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
                assert B.conv3d_plan_for_props(d, B.DTYPE[cv.dtype], PROPS, opts, p) == 0
            else:
                d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
                assert B.conv2d_plan_for_props(d, B.DTYPE[cv.dtype], PROPS, opts, p) == 0
            self.items.append((cv, None, None, d, p.as_dict(), None))


def test_ffma_headline_roofline():
    """40 x 512 x 512, 192 -> 96 in three launches: the GEMM's 2 * 64 * T * 192 * 96
    FLOP (T = 40 * 86 * 86) over three launches of 4.32 ms each is 53.86 TFLOP/s,
    judged against the FP32 probe's rate; the shares add up to one."""
    w = PlannedWorkload("winograd_f32")
    steps = 10
    prof = {"wino_gemm_simt": (3 * steps, 12.96 * steps), "wino_input": (3 * steps, 3.68 * steps),
            "wino_output": (3 * steps, 1.79 * steps), "wino_filter": (steps, 0.011 * steps)}
    kernels, roof = bench.kernels_and_roofline(w, prof, steps, {}, (73.5, "probe"), "winograd_f32")
    flops = 2 * 64 * (40 * 86 * 86) * 192 * 96
    assert roof["kernel"] == "wino_gemm_simt" and roof["bound"] == "alu" and roof["unit"] == "TFLOP/s"
    assert roof["algorithmic_per_launch"] == pytest.approx(flops / 3)
    assert roof["achieved"] == pytest.approx(flops / 3 / 4.32e-3 / 1e12)
    assert roof["achieved"] == pytest.approx(53.86, abs=0.01)
    assert roof["peak"] == 73.5 and roof["frac"] == pytest.approx(roof["achieved"] / 73.5)
    assert sum(k["share"] for k in kernels.values()) == pytest.approx(1.0)
    assert kernels["wino_gemm_simt"]["launches_per_step"] == 3
    # the stored ncu traffic counts only while the kernel's sources hash the same
    stored = bench.load_traffic().get("winograd_f32:wino_gemm_simt")
    if stored and stored["source_hash"] == bench.source_hash("wino_gemm_simt"):
        assert roof["traffic"] == stored["bytes_per_launch"]
    else:
        assert roof["traffic"] is None
    # without a workload name no traffic is looked up
    assert bench.kernels_and_roofline(w, prof, steps, {}, (73.5, "probe"))[1]["traffic"] is None


def test_hbm_roofline_and_peak_choice(monkeypatch):
    """The split-bf16 route, input transform dominant: its bytes (the input once,
    V as three bf16 parts: 6 bytes a value) per launch over the launch time,
    against 6650 GB/s without measured peaks and the measured figure with them."""
    monkeypatch.setenv("B200CONV_WINOGRAD_SPLIT_BF16", "1")
    monkeypatch.delenv("B200CONV_WINOGRAD_FUSED", raising=False)
    w = PlannedWorkload("winograd_f32")
    assert w.items[0][4]["winograd_split_bf16"] == 1 and w.items[0][4]["num_batch_tiles"] == 4
    steps = 5
    prof = {"wino_input": (4 * steps, 6.67 * steps), "wino_gemm_tc": (4 * steps, 5.06 * steps),
            "wino_output": (4 * steps, 1.88 * steps), "wino_filter": (steps, 0.01 * steps)}
    nbytes = 40 * 512 * 512 * 192 * 4 + 64 * (40 * 86 * 86) * 192 * 6
    _, roof = bench.kernels_and_roofline(w, prof, steps, {}, (73.5, "probe"))
    assert roof["kernel"] == "wino_input" and roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["algorithmic_per_launch"] == pytest.approx(nbytes / 4)
    assert roof["achieved"] == pytest.approx(nbytes / 4 / (6.67 / 4 * 1e-3) / 1e9)
    assert roof["peak"] == 6650.0 and "fallback" in roof["peak_source"]
    _, roof_m = bench.kernels_and_roofline(w, prof, steps, {"hbm_gbs": 6548.0}, (73.5, "probe"))
    assert roof_m["peak"] == 6548.0 and "measured" in roof_m["peak_source"]
    assert roof_m["frac"] == pytest.approx(roof["achieved"] / 6548.0)


def test_tensor_roofline_sustained_and_shape_bound():
    """The wide-channel set with the implicit GEMM forced: FLOPs per launch over
    the launch time against the bf16 burst peak, plus the sustained fraction and
    the fraction of the per-conv bound max(FLOPs / tensor peak, bytes / HBM peak),
    which can never exceed the tensor peak."""
    w = PlannedWorkload("wide_bf16", "implicit")
    n = len(w.items)
    assert n == 56
    steps = 4
    prof = {"tc_conv": (n * steps, 33.9 * steps)}
    flops = sum(cv.flops for cv, *_ in w.items)
    _, roof = bench.kernels_and_roofline(w, prof, steps, {}, (73.5, "probe"))
    assert roof["kernel"] == "tc_conv" and roof["bound"] == "tensor"
    assert roof["achieved"] == pytest.approx(flops / n / (33.9 / n * 1e-3) / 1e12)
    assert roof["peak"] == 1590.0 and roof["sustained_peak"] == 1400.0
    assert roof["frac_of_sustained"] == pytest.approx(roof["achieved"] / 1400.0)
    ideal = sum(max(f / 1590e12, b / 6650e9) for f, b in w.per_conv_work("tc_conv"))
    assert roof["attainable"] == pytest.approx(flops / ideal / 1e12)
    assert roof["attainable"] <= 1590.0 + 1e-6
    assert roof["frac_of_attainable"] == pytest.approx(roof["achieved"] / roof["attainable"])
    measured = {"bf16_tflops": 1642.0, "bf16_tflops_sustained": 1397.0, "hbm_gbs": 6548.0}
    _, roof_m = bench.kernels_and_roofline(w, prof, steps, measured, (73.5, "probe"))
    assert roof_m["peak"] == 1642.0 and roof_m["sustained_peak"] == 1397.0


def test_conv_flops_are_the_direct_count():
    """The metric's FLOPs are the direct convolution's 2 * N * OH * OW * O * C * KH * KW,
    whatever algorithm runs (Winograd is reported direct-equivalent)."""
    s = synth.WINOGRAD_F32
    cv = bench.Conv(s, "f32", "uniform")
    assert cv.flops == 2 * 40 * 512 * 512 * 96 * 192 * 9


def test_clock_record_from_samples(tmp_path):
    """The clock record of a timed region: the median SM clock under load, the
    maximum, every throttle reason seen active in any sample, the peak power;
    rows that are not full samples are skipped."""
    p = tmp_path / "clocks.csv"
    p.write_text(
        "0, 1965, 1965, 640.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
        "0, 1590, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
        "0, 1800, 1965, 800.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
        "0, [N/A]\n")
    cs = bench.ClockSampler(0)
    cs.path = str(p)
    rec = cs.summary()
    assert rec["sm_mhz"] == 1800.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"] and rec["samples"] == 3 and rec["power_w_max"] == 990.0
    assert not p.exists()                       # the sample file is removed once read
    q = tmp_path / "hot.csv"
    q.write_text("0, 1400, 1965, 700, 0x48, Active, Active, Not Active, Not Active\n")
    cs.path = str(q)
    assert cs.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    cs.path = str(tmp_path / "missing.csv")
    assert cs.summary()["reasons"] == ["nvidia-smi unavailable"]
