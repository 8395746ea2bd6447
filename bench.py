#!/usr/bin/env python
"""Benchmark: convolution TFLOP/s on one B200 (or N replicas).

Metric: direct-equivalent conv TFLOP/s, 2*N*OH*OW*O*C*KH*KW per second (Winograd
counted at direct-equivalent FLOPs), and its fraction of the peak of the
dominant kernel.  Default workload: the fp32 Winograd case of "Bound winograd
conv2d working set by tiling the batch" (Testing): N=40, 512x512, 192->96,
3x3, stride 1, pad 1, seeded uniform inputs, batch-tiled Winograd F(6x6,3x3).
Other workloads (--workload) are measurement aids: the ResNet-50 layer set,
the wide-channel implicit-GEMM sweep, the conv3d depth-tap cases, the small
fp32 case.

One step = one forward pass of the whole path over one batch with inputs
resident in HBM.  Timed with CUDA events on the launching stream, W untimed
warm-ups, K timed steps bracketed by a barrier and a synchronize; for N > 1
each rank runs an independent replica (the forward pass needs no collective)
and the slowest rank's time is reported.  `e2e` repeats the step through the
same C ABI with host buffers: pinned host -> device copy of the inputs, the
conv, device -> host copy of the output, all inside the timed region.

--impl reference times the CPU oracle (the plain fp64 direct convolution) on
host cores on a bounded pixel sample of the same workload.
"""
import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from dense_convolution_nhwc_b200 import synth  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FP32_LANES_PER_SM = 128
PAGES_NUMBER = {
    # direct-equivalent TFLOP/s of the pages' own measurement of the same workload
    # (310 ms on an M2 Max: 2*40*512*512*96*192*9 / 0.310 s); context, another machine
    "winograd_f32": 11.2,
}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

class Conv:
    """One conv2d or conv3d call of a workload."""

    def __init__(self, shape, dtype, dist, algo="auto", name=None):
        self.shape, self.dtype, self.dist, self.algo = shape, dtype, dist, algo
        self.is3d = isinstance(shape, synth.Conv3dShape)
        self.name = name or shape.name()

    @property
    def flops(self):
        return self.shape.flops


def workload(name):
    if name.startswith("conv2d:"):
        # conv2d:<n>,<h>,<w>,<c>,<o>,<k>,<stride>,<pad>,<dilation>:<dtype>  (a single conv, e.g. for ncu)
        _, dims, dt = name.split(":")
        n, h, w, c, o, k, st, pd, dl = (int(v) for v in dims.split(","))
        shape = synth.Conv2dShape(n, h, w, c, o, k, k, (st, st), (pd, pd), (dl, dl))
        return f"conv2d {dt} NHWC {shape.name()}", [Conv(shape, dt, "uniform" if dt == "f32" else "normal")], dt
    if name.startswith("conv3d:"):
        # conv3d:<n>,<d>,<h>,<w>,<c>,<o>,<k>,<stride>,<pad_d>,<pad_hw>:<dtype>  (a single conv, e.g. for ncu)
        _, dims, dt = name.split(":")
        n, d, h, w, c, o, k, st, pdd, phw = (int(v) for v in dims.split(","))
        shape = synth.Conv3dShape(n, d, h, w, c, o, k, k, k, (st, st, st), (pdd, phw, phw), (1, 1, 1))
        return f"conv3d {dt} NDHWC {shape.name()}", [Conv(shape, dt, "normal")], dt
    if name == "winograd_f32":
        return ("conv2d fp32 NHWC N=40 H=W=512 C=192->O=96 3x3 stride 1 pad 1 (Winograd, batch-tiled workspace)",
                [Conv(synth.WINOGRAD_F32, "f32", "uniform")], "f32")
    if name == "small_f32":
        return ("conv2d fp32 NHWC N=2 H=W=16 C=32->O=32 3x3 stride 1 pad 1",
                [Conv(synth.SMALL_F32, "f32", "uniform")], "f32")
    if name.startswith("resnet50_"):
        _, dt, b = name.split("_")
        convs = []
        for lname, shape, count in synth.resnet50_layers(int(b[1:])):
            for i in range(count):
                convs.append(Conv(shape, dt, "he", name=f"{lname}#{i}"))
        return (f"ResNet-50 v1.5 conv layer set (53 convs) {dt} batch {b[1:]} 224x224", convs, dt)
    if name.startswith("conv3d_"):
        dt = name.split("_")[1]
        return (f"conv3d {dt} NDHWC 3x3x3 s1 spatial pad 1 depth pad 0 N=1: 17x64x64 256->256, "
                "41x60x104 256->256, 41x120x208 512->512", [Conv(s, dt, "normal") for s in synth.CONV3D_TAPS], dt)
    if name.startswith("wide_") or name.startswith("wide3_"):
        # wide_<dtype>: C_out >= 512 and M >= 16384 aligned members of the sweep
        dt = name.split("_")[1]
        shapes = [s for s in synth.wide_sweep(True) if s.o >= 512 and s.n * s.oh * s.ow >= 16384]
        if not name.endswith("_all"):
            shapes = [s for s in shapes if s.stride == (1, 1) and s.dilation == (1, 1)]
        if name.startswith("wide3_"):     # the 3x3 members (the ones Winograd can also run)
            shapes = [s for s in shapes if s.kh == 3]
        return (f"wide-channel implicit-GEMM sweep {dt}: C_out>=512, M>=16384, aligned ({len(shapes)} shapes)",
                [Conv(s, dt, "normal") for s in shapes], dt)
    raise SystemExit(f"unknown workload {name}")


# ---------------------------------------------------------------------------
# per-kernel algorithmic work (for the roofline)
# ---------------------------------------------------------------------------

def kernel_work(conv, plan):
    """{kernel name: (flops, bytes)} of algorithmic work for one call, by the
    plan the library will run."""
    s = conv.shape
    esz = 4 if conv.dtype == "f32" else 2
    w = {}

    def add(k, f=0.0, b=0.0):
        f0, b0 = w.get(k, (0.0, 0.0))
        w[k] = (f0 + f, b0 + b)

    if conv.is3d and plan["algo"] == "winograd" and plan["taps"] == 1:
        # native 3D Winograd F(m^3, 3^3)
        m = plan["winograd_m"]
        a3 = (m + 2) ** 3
        T = s.n * math.ceil(s.od / m) * math.ceil(s.oh / m) * math.ceil(s.ow / m)
        st = 4 if plan["engine"] == "simt" else esz
        in_b = s.n * s.d * s.h * s.w * s.c * esz
        out_b = s.n * s.od * s.oh * s.ow * s.o * esz
        add("wino3d_filter", 0.0, s.o * 27 * s.c * esz + a3 * s.o * s.c * st)
        add("wino3d_input", 0.0, in_b + a3 * T * s.c * st)
        gk = "wino3d_gemm_tc" if plan["engine"] == "tcgen05" else "wino3d_gemm_simt"
        add(gk, 2.0 * a3 * T * s.c * s.o, a3 * T * (s.c * st + s.o * 4))
        add("wino3d_output", 0.0, a3 * T * s.o * 4 + out_b)
        return w
    if conv.is3d and plan["taps"] == 1 and plan["engine"] == "tcgen05":
        # native K-fused 3D implicit GEMM: one pass, output written once
        M = s.n * s.od * s.oh * s.ow
        K = s.c * s.kd * s.kh * s.kw
        add("tc_conv3d", 2.0 * M * s.o * K,
            (s.n * s.d * s.h * s.w * s.c + s.o * K + M * s.o) * esz)
        return w
    if conv.is3d:
        frames_out = s.od
        n2 = synth.Conv2dShape(frames_out, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride[1:], s.pad[1:], s.dilation[1:])
        taps = s.kd
        out_bytes = s.n * s.od * s.oh * s.ow * s.o * esz
        for t in range(taps):
            for k, (f, b) in kernel_work(Conv(n2, conv.dtype, conv.dist), plan).items():
                # taps after the first also read the output they add into
                extra = out_bytes if (t > 0 and k in ("tc_conv", "simt_conv", "wino_output")) else 0.0
                add(k, f * s.n, b * s.n + extra)
        return w
    M = s.n * s.oh * s.ow
    K = s.c * s.kh * s.kw
    in_b, w_b, out_b = s.n * s.h * s.w * s.c * esz, s.o * K * esz, M * s.o * esz
    if plan["algo"] == "winograd":
        m = plan["winograd_m"]
        a2 = (m + 2) ** 2
        T = s.n * math.ceil(s.oh / m) * math.ceil(s.ow / m)
        st = 4 if plan["engine"] == "simt" else esz
        add("wino_filter", 0.0, w_b + a2 * s.o * s.c * st)
        if plan.get("winograd_fused"):
            # one persistent kernel: the GEMM's FLOPs; bytes = input + output + the V and M
            # round trips through its per-CTA scratch
            add("wino_fused", 2.0 * a2 * T * s.c * s.o, in_b + out_b + 2 * a2 * T * (s.c + s.o) * 4)
            return w
        # the split-bf16 route writes V as three bf16 parts (6 bytes per value)
        add("wino_input", 0.0, in_b + a2 * T * s.c * (6 if plan.get("winograd_split_bf16") else st))
        gk = "wino_gemm_tc" if plan["engine"] == "tcgen05" else "wino_gemm_simt"
        if plan.get("winograd_split_bf16"):
            # six bf16 products per fp32 product on the tensor cores: 3C bf16 parts of V read,
            # fp32 M written
            add("wino_gemm_tc", 6 * 2.0 * a2 * T * s.c * s.o, a2 * T * (3 * s.c * 2 + s.o * 4))
        else:
            # M is fp32 on the FFMA path and in the 16-bit operand type on the tensor-core path
            add(gk, 2.0 * a2 * T * s.c * s.o, a2 * T * (s.c * st + s.o * st))
        add("wino_output", 0.0, a2 * T * s.o * st + out_b)
    else:
        k = "tc_conv" if plan["engine"] == "tcgen05" else "simt_conv"
        add(k, 2.0 * M * s.o * K, in_b + w_b + out_b)
        if plan["channel_pad"]:
            cp = plan["channel_pad"]
            add("channel_pad", 0.0, in_b + s.n * s.h * s.w * cp * esz + w_b + s.o * s.kh * s.kw * cp * esz)
    return w


def kernel_bound(name):
    if name in ("tc_conv", "tc_conv3d", "wino_gemm_tc", "wino3d_gemm_tc"):
        return "tensor"
    if name in ("simt_conv", "wino_gemm_simt", "wino3d_gemm_simt", "wino_fused"):
        return "alu"
    return "hbm"


KERNEL_SOURCES = {
    "simt_conv": ["simt_conv.cu", "common.cuh"], "wino_gemm_simt": ["wino_gemm_f32.cu"],
    "wino_fused": ["wino_fused_f32.cu", "wino_tile.cuh", "mbar.cuh", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "tc_conv": ["tc_conv.cu", "tc_ptx.cuh", "common.cuh"], "wino_gemm_tc": ["tc_conv.cu", "tc_ptx.cuh", "common.cuh"],
    "tc_conv3d": ["tc_conv.cu", "tc_ptx.cuh", "common.cuh"],
    "wino_input": ["winograd.cu", "wino_tile.cuh", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "wino_output": ["winograd.cu", "wino_tile.cuh", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "wino_filter": ["winograd.cu", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "wino3d_gemm_simt": ["wino_gemm_f32.cu"], "wino3d_gemm_tc": ["tc_conv.cu", "tc_ptx.cuh", "common.cuh"],
    "wino3d_input": ["winograd3d.cu", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "wino3d_output": ["winograd3d.cu", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "wino3d_filter": ["winograd3d.cu", "wino_1d.cuh", "winograd_gen.cuh", "common.cuh"],
    "accumulate": ["elementwise.cu", "common.cuh"], "channel_pad": ["elementwise.cu", "common.cuh"],
}


def source_hash(kernel):
    """Hash of the source files a kernel is built from (ncu traffic is void once it changes)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dense_convolution_nhwc_b200", "csrc")
    for f in KERNEL_SOURCES.get(kernel, []):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def load_traffic():
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    try:
        return json.load(open(p))
    except Exception:
        return {}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if getattr(self, "fh", None):
            self.fh.close()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1])]
        smax = max((num(r[2]) or 0) for r in rows)
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower() == "active":
                    reasons.add(n)
        power = [num(r[3]) for r in rows if num(r[3])]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)
# ---------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def reduce_max(x, world, device):
    """Max over ranks (the slowest replica sets the time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------

# the headline metric, verbatim; TFLOP/s are direct-equivalent (2*N*OH*OW*O*C*KH*KW per second)
METRIC = "conv TFLOP/s per dtype and fraction of tensor (or FP32) peak, 1 B200"


def oracle_sample_rate(conv, x_host, w_host, target_s, seed=0):
    """Time the oracle on a pixel sample sized for about target_s seconds.
    Returns (TFLOP/s, cores, description, seconds of the timed pass)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    s = conv.shape
    per_px = 2.0 * s.o * s.c * s.kh * s.kw * (s.kd if conv.is3d else 1)

    def run(npx):
        import torch
        g = torch.Generator().manual_seed(seed)
        if conv.is3d:
            nimg = x_host.shape[0]
            idx = torch.randint(0, nimg * s.od * s.oh * s.ow, (npx,), generator=g)
            ow_, r = idx % s.ow, idx // s.ow
            oh_, r = r % s.oh, r // s.oh
            od_, n_ = r % s.od, r // s.od
            pix = torch.stack([n_, od_, oh_, ow_], 1).int().numpy()
            t0 = time.perf_counter()
            oracle.conv3d(x_host, w_host, conv.dtype, s.stride, s.pad, s.dilation, pixels=pix, threads=cores)
        else:
            nimg = x_host.shape[0]
            idx = torch.randint(0, nimg * s.oh * s.ow, (npx,), generator=g)
            ow_, r = idx % s.ow, idx // s.ow
            oh_, n_ = r % s.oh, r // s.oh
            pix = torch.stack([n_, oh_, ow_], 1).int().numpy()
            t0 = time.perf_counter()
            oracle.conv2d(x_host, w_host, conv.dtype, s.stride, s.pad, s.dilation, pixels=pix, threads=cores)
        return time.perf_counter() - t0

    npx = 64
    dt = run(npx)
    while dt < 0.5 and npx < 1 << 22:
        npx *= 4
        dt = run(npx)
    npx = max(1, int(npx * target_s / max(dt, 1e-6)))
    dt = run(npx)
    return (per_px * npx / dt / 1e12, cores,
            f"{npx} seeded output pixels (with replacement) x all {s.o} channels of {conv.name}, one pass", dt)


def run_reference(args, wl_name):
    """The CPU oracle as it stands, on the host cores, on a bounded sample."""
    world, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    import torch
    desc, convs, dtype = workload(wl_name)
    conv = max(convs, key=lambda c: c.flops)
    s = conv.shape
    # one image (frame stack) of the workload, seeded, on the host
    if conv.is3d:
        one = synth.Conv3dShape(1, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
        x, w = synth.conv3d_inputs(one, dtype, conv.dist, 0, "cpu")
    else:
        one = synth.Conv2dShape(1, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
        x, w = synth.conv2d_inputs(one, dtype, conv.dist, 0, "cpu")
    per_step_s = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    rates, secs = [], []
    desc_s = ""
    cores = len(os.sched_getaffinity(0))
    for i in range(args.warmup + args.steps):
        r, cores, desc_s, sec = oracle_sample_rate(conv, x, w, per_step_s, seed=i)
        if i >= args.warmup:
            rates.append(r)
            secs.append(sec)
    value = statistics.mean(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(secs) * 1000.0, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {"f32": "f64 (fp32 inputs)", "f16": "f64 (fp16 inputs)",
                                         "bf16": "f64 (bf16 inputs)"}[dtype],
        "data": "synthetic", "config": {"workload": desc, "sample_of": conv.name},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc_s},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

# Per-config entries printed inside the headline's JSON line (same run, same
# GPU): the small fp32 case, the ResNet-50 layer sets (fp16/bf16, batch 1/8),
# the wide-channel implicit-GEMM members (auto and forced implicit GEMM), the
# wide 3x3 members with Winograd forced (the Winograd GEMM core), and the
# conv3d cases.  (key, workload, algo, time as a CUDA graph too)
PER_CONFIG = [
    ("config1_small_f32", "small_f32", "auto", False),
    ("config3_resnet50_f16_b1", "resnet50_f16_b1", "auto", True),
    ("config3_resnet50_bf16_b1", "resnet50_bf16_b1", "auto", True),
    ("config3_resnet50_f16_b8", "resnet50_f16_b8", "auto", True),
    ("config3_resnet50_bf16_b8", "resnet50_bf16_b8", "auto", True),
    ("config4_wide_bf16_auto", "wide_bf16", "auto", False),
    ("config4_wide_f16_auto", "wide_f16", "auto", False),
    ("config4_wide_bf16_implicit", "wide_bf16", "implicit", False),
    ("config4_wide_f16_implicit", "wide_f16", "implicit", False),
    ("config4_wide3_bf16_winograd", "wide3_bf16", "winograd", False),
    ("config4_wide3_f16_winograd", "wide3_f16", "winograd", False),
    ("config5_conv3d_bf16", "conv3d_bf16", "auto", False),
    ("config5_conv3d_f32", "conv3d_f32", "auto", False),
    # config 2 with the fp32 Winograd GEMM on the tensor cores over split-bf16 operands
    # (fp32-accurate emulation, not the default; the headline line keeps FFMA arithmetic)
    ("config2_f32_gemm_split_bf16", "winograd_f32", "auto", False, {"B200CONV_WINOGRAD_SPLIT_BF16": "1"}),
]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return json.load(open(p)) if os.path.exists(p) else {}
    except Exception:
        return {}


class Bench:
    """One workload made resident on the device: inputs, outputs, plans and a
    shared workspace, and the step that runs every conv of it once."""

    def __init__(self, wl_name, algo, dev, stream):
        import torch
        from dense_convolution_nhwc_b200 import binding as B
        self.B, self.torch = B, torch
        self.desc, convs, self.dtype = workload(wl_name)
        self.opts = B.make_options(algo)
        self.dev, self.stream = dev, stream
        self.sptr = stream.cuda_stream
        self.items = []
        ws_max = 0
        local = dev.index or 0
        for i, cv in enumerate(convs):
            s = cv.shape
            if cv.is3d:
                x, w = synth.conv3d_inputs(s, cv.dtype, cv.dist, i, dev)
                d = B.make_desc3d(s.n, s.d, s.h, s.w, s.c, s.o, s.kd, s.kh, s.kw, s.stride, s.pad, s.dilation)
                plan = B.plan3d(d, cv.dtype, local, self.opts)
                out = torch.empty((s.n, s.od, s.oh, s.ow, s.o), dtype=x.dtype, device=dev)
            else:
                x, w = synth.conv2d_inputs(s, cv.dtype, cv.dist, i, dev)
                d = B.make_desc2d(s.n, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
                plan = B.plan2d(d, cv.dtype, local, self.opts)
                out = torch.empty((s.n, s.oh, s.ow, s.o), dtype=x.dtype, device=dev)
            ws_max = max(ws_max, plan["workspace_bytes"])
            self.items.append((cv, x, w, d, plan, out))
        self.ws = torch.empty(max(ws_max, 256), dtype=torch.uint8, device=dev)
        self.dt_code = B.DTYPE[self.dtype]
        self.fwd = B.conv3d_forward if convs[0].is3d else B.conv2d_forward
        self.total_flops = sum(cv.flops for cv, *_ in self.items)
        self.in_bytes = sum(x.numel() * x.element_size() for _, x, _, _, _, _ in self.items)
        self.flush = (torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
                      if self.in_bytes < 2 * L2_BYTES else None)
        self.graph = None

    def step(self, sptr=None):
        sptr = sptr or self.sptr
        for cv, x, w, d, plan, out in self.items:
            st = self.fwd(x.data_ptr(), w.data_ptr(), out.data_ptr(), d, self.dt_code, self.opts,
                          self.ws.data_ptr(), self.ws.numel(), sptr)
            if st != 0:
                raise self.B.ConvError(st, cv.name)

    def capture(self):
        """One step captured as a CUDA graph (removes host launch gaps)."""
        torch = self.torch
        g_stream = torch.cuda.Stream(self.dev)
        g_stream.wait_stream(self.stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(g_stream):
            with torch.cuda.graph(graph, stream=g_stream):
                self.step(g_stream.cuda_stream)
        self.stream.wait_stream(g_stream)
        torch.cuda.synchronize()
        self.graph = graph

    def timed(self, steps, use_graph=False):
        """Device time of `steps` steps, ms each (CUDA events on the launching
        stream; an L2 flush between steps when the inputs fit in L2, outside
        the events).  No profiling hook is active."""
        torch = self.torch
        run = self.graph.replay if use_graph else self.step
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for k in range(steps):
            if self.flush is not None:
                self.flush.zero_()
            ev[k][0].record(self.stream)
            run()
            ev[k][1].record(self.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def kernel_split(self, steps):
        """Per-kernel launches and event time from separate, profiled steps."""
        B = self.B
        B.conv_profile_begin()
        for _ in range(steps):
            if self.flush is not None:
                self.flush.zero_()
            self.step()
        self.torch.cuda.synchronize()
        return B.profile_end()

    def work(self):
        w = {}
        for cv, x, wt, d, plan, out in self.items:
            for k, (f, b) in kernel_work(cv, plan).items():
                f0, b0 = w.get(k, (0.0, 0.0))
                w[k] = (f0 + f, b0 + b)
        return w

    def per_conv_work(self, kernel):
        return [kernel_work(cv, plan).get(kernel, (0.0, 0.0)) for cv, _, _, _, plan, _ in self.items]


def fp32_peak(B, torch, peaks):
    smax = peaks.get("sm_max_mhz", 1965.0)
    derived = 148 * FP32_LANES_PER_SM * 2 * smax * 1e6 / 1e12
    # measured: the library's FMA-chain probe (scalar FFMA and the packed two-lane FMA);
    # the higher of the two is the CUDA cores' fp32 peak
    rates = {}
    for packed in (0, 1):
        v = ctypes.c_double(0.0)
        if B.conv_fp32_fma_rate(packed, v, torch.cuda.current_stream().cuda_stream) == 0:
            rates["packed" if packed else "scalar"] = v.value
    if rates:
        return max(rates.values()), ("measured: fp32 FMA-chain probe in this run (scalar %.1f, packed %.1f TFLOP/s; "
                                     "derived 148 SMs x 128 lanes x 2 x %.0f MHz = %.1f)" %
                                     (rates.get("scalar", 0.0), rates.get("packed", 0.0), smax, derived))
    return derived, f"derived: 148 SMs x 128 FP32 lanes x 2 x {smax:.0f} MHz"


def kernels_and_roofline(bench, prof, steps, peaks, fp32_pk, wl_name=None):
    """Per-kernel shares and the roofline of the dominant kernel."""
    work = bench.work()
    kernels = {}
    tot_all = max(1e-9, sum(t for _, t in prof.values()))
    for name, (launches, tot) in prof.items():
        f, b = work.get(name, (0.0, 0.0))
        kernels[name] = {"launches_per_step": launches / steps, "ms_per_step": tot / steps, "share": tot / tot_all,
                         "flops_per_step": f, "bytes_per_step": b, "per_launch_ms": tot / max(launches, 1)}
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    kd = kernels[dom]
    bound = kernel_bound(dom)
    lps = kd["launches_per_step"]
    hbm = peaks.get("hbm_gbs")
    bf16 = peaks.get("bf16_tflops")
    bf16_sus = peaks.get("bf16_tflops_sustained")
    src_note = "measured (MEASURED_PEAKS.json)" if peaks else "fallback (profiling recipe: 6.65 TB/s, 1.59 PFLOP/s)"
    extra = {}
    if bound == "hbm":
        achieved = kd["bytes_per_step"] / lps / (kd["per_launch_ms"] * 1e-3) / 1e9
        peak, unit, peak_src = hbm or 6650.0, "GB/s", f"HBM copy bandwidth, {src_note}"
    elif bound == "tensor":
        achieved = kd["flops_per_step"] / lps / (kd["per_launch_ms"] * 1e-3) / 1e12
        peak, unit = bf16 or 1590.0, "TFLOP/s"
        peak_src = f"dense bf16 burst, {src_note}; fp16 taken at the same nominal rate"
        sus = bf16_sus or 1400.0
        extra["frac_of_sustained"] = achieved / sus
        extra["sustained_peak"] = sus
        # the shape-bound: per conv, the kernel cannot beat max(flops / tensor peak, bytes / HBM)
        ideal = sum(max(f / (peak * 1e12), b / ((hbm or 6650.0) * 1e9)) for f, b in bench.per_conv_work(dom))
        if ideal > 0:
            attainable = kd["flops_per_step"] / ideal / 1e12
            extra["attainable"] = attainable
            extra["frac_of_attainable"] = achieved / attainable
            extra["attainable_note"] = "sum over convs of max(FLOPs / tensor peak, algorithmic bytes / HBM peak)"
    else:
        achieved = kd["flops_per_step"] / lps / (kd["per_launch_ms"] * 1e-3) / 1e12
        peak, peak_src = fp32_pk
        unit = "TFLOP/s"
    traffic = None
    if wl_name is not None:
        tr = load_traffic().get(f"{wl_name}:{dom}")
        if tr and tr.get("source_hash") == source_hash(dom):
            traffic = tr.get("bytes_per_launch")
    roof = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic, "peak_source": peak_src,
            "algorithmic_per_launch": (kd["bytes_per_step"] if bound == "hbm" else kd["flops_per_step"]) / lps}
    roof.update(extra)
    return kernels, roof


def per_config_entry(key, wl_name, algo, use_graph, dev, stream, world, peaks, fp32_pk, min_steps, env=None):
    old_env = {k: os.environ.get(k) for k in (env or {})}
    os.environ.update(env or {})
    try:
        return _per_config_entry(key, wl_name, algo, use_graph, dev, stream, world, peaks, fp32_pk, min_steps, env)
    finally:
        for k, v in old_env.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def _per_config_entry(key, wl_name, algo, use_graph, dev, stream, world, peaks, fp32_pk, min_steps, env):
    import torch
    bench = Bench(wl_name, algo, dev, stream)
    for _ in range(3):
        bench.step()
    torch.cuda.synchronize()
    one = statistics.median(bench.timed(3))
    # enough steps that the clock record covers the timed region (>= ~0.4 s)
    steps = int(min(2000, max(min_steps, math.ceil(400.0 / max(one, 1e-3)))))
    entry = {"workload": bench.desc, "algo": algo, "dtype": bench.dtype, "convs": len(bench.items),
             "flops_per_step": bench.total_flops}
    if env:
        entry["env"] = dict(env)
    if any(plan.get("winograd_split_bf16") for *_, plan, _ in bench.items):
        entry["arithmetic"] = ("fp32 transforms; the Winograd GEMM on the tensor cores over split-bf16 operands "
                               "(each fp32 value the exact sum of three bf16 parts, six bf16 products per fp32 "
                               "product accumulated in fp32): fp32-accurate emulation, not FFMA arithmetic")
    barrier(world)
    with ClockSampler(dev.index or 0) as clk:
        ms_eager = statistics.median(bench.timed(steps))
    entry["clocks"] = clk.summary()
    ms_eager = reduce_max(ms_eager, world, dev)
    entry["ms_issued"] = ms_eager
    ms = ms_eager
    if use_graph:
        bench.capture()
        for _ in range(3):
            bench.graph.replay()
        ms_graph = reduce_max(statistics.median(bench.timed(steps, use_graph=True)), world, dev)
        entry["ms_graph"] = ms_graph
        ms = ms_graph
        entry["timing"] = "CUDA graph replay of one step (host launch gaps removed); ms_issued is call by call"
    entry["ms"] = ms
    entry["value"] = world * bench.total_flops / (ms * 1e-3) / 1e12
    entry["unit"] = "TFLOP/s"
    entry["steps"] = steps
    prof = bench.kernel_split(min(steps, 20))
    kernels, roof = kernels_and_roofline(bench, prof, min(steps, 20), peaks, fp32_pk)
    entry["kernels"] = {k: {"share": v["share"], "ms_per_step": v["ms_per_step"],
                            "launches_per_step": v["launches_per_step"]} for k, v in kernels.items()}
    entry["roofline"] = roof
    if bench.dtype != "f32":
        entry["frac_of_bf16_peak"] = entry["value"] / (peaks.get("bf16_tflops") or 1590.0)
    plans = {}
    for cv, *_, plan, _ in bench.items:
        k = f'{plan["algo"]}/{plan["engine"]}'
        plans[k] = plans.get(k, 0) + 1
    entry["plans"] = plans
    entry["l2"] = ("L2 flushed between steps (outside the events)" if bench.flush is not None
                   else f"inputs larger than L2 ({bench.in_bytes / 1e9:.2f} GB per step)")
    del bench
    torch.cuda.empty_cache()
    return entry


def run_headline(args, B, torch, dev, stream, world, rank, local, peaks):
    """The headline workload: timed steps, kernel split, e2e and the CPU
    baseline.  Returns the pieces of the JSON line; every device buffer of the
    workload is released when it returns."""
    bench = Bench(args.workload, args.algo, dev, stream)
    desc, dtype, items = bench.desc, bench.dtype, bench.items
    sptr = bench.sptr
    for _ in range(args.warmup):
        bench.step()
    torch.cuda.synchronize()
    assert B.conv_check(sptr) == 0
    if args.graph:
        bench.capture()

    # timed region: no profiling hook, only the events around each step
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        times = bench.timed(args.steps, use_graph=args.graph)
    barrier(world)
    assert B.conv_check(sptr) == 0
    ms = sum(times) / args.steps
    ms = reduce_max(ms, world, dev)
    value = world * bench.total_flops / (ms * 1e-3) / 1e12
    clocks = clk.summary()

    # per-kernel split from separate, profiled steps (outside the timed region)
    prof_steps = min(args.steps, 10)
    prof = bench.kernel_split(prof_steps)
    fp32_pk = fp32_peak(B, torch, peaks)
    kernels, roof = kernels_and_roofline(bench, prof, prof_steps, peaks, fp32_pk, args.workload)
    launches_per_step = sum(l for l, _ in prof.values()) / prof_steps
    gpu_launches = int(round(launches_per_step * args.steps))
    fwd, opts, dt_code, ws = bench.fwd, bench.opts, bench.dt_code, bench.ws
    total_flops = bench.total_flops

    # e2e through the C ABI with host buffers.  Images are independent, so each
    # conv's batch is cut into chunks that flow through three streams: the
    # host->device copy of chunk i+1 and the device->host copy of chunk i-1
    # overlap the conv of chunk i (copy engines and SMs work at the same time).
    e2e = None
    if not args.no_e2e:
        hx = [x.cpu().pin_memory() for _, x, *_ in items]
        hw = [w.cpu().pin_memory() for _, _, w, *_ in items]
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for *_, out in items]
        dx = [torch.empty_like(x) for _, x, *_ in items]
        dw = [torch.empty_like(w) for _, _, w, *_ in items]
        k_e2e = max(1, min(args.steps, 3))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        chunk_descs = []
        for j, (cv, x, w, d, plan, out) in enumerate(items):
            s = cv.shape
            nchunk = min(s.n, 8) if not cv.is3d else 1
            bounds = [round(i * s.n / nchunk) for i in range(nchunk + 1)]
            cds = []
            for c0, c1 in zip(bounds[:-1], bounds[1:]):
                if c1 <= c0:
                    continue
                if cv.is3d:
                    dd = d
                else:
                    dd = B.make_desc2d(c1 - c0, s.h, s.w, s.c, s.o, s.kh, s.kw, s.stride, s.pad, s.dilation)
                cds.append((c0, c1, dd))
            chunk_descs.append(cds)

        def e2e_step():
            for j, (cv, x, w, d, plan, out) in enumerate(items):
                ev_in = []
                with torch.cuda.stream(s_in):
                    dw[j].copy_(hw[j], non_blocking=True)
                    for (c0, c1, dd) in chunk_descs[j]:
                        dx[j][c0:c1].copy_(hx[j][c0:c1], non_blocking=True)
                        e = torch.cuda.Event()
                        e.record(s_in)
                        ev_in.append(e)
                for (c0, c1, dd), e in zip(chunk_descs[j], ev_in):
                    stream.wait_event(e)
                    st = fwd(dx[j][c0:c1].data_ptr(), dw[j].data_ptr(), out[c0:c1].data_ptr(), dd, dt_code, opts,
                             ws.data_ptr(), ws.numel(), sptr)
                    if st != 0:
                        raise B.ConvError(st, cv.name)
                    e2 = torch.cuda.Event()
                    e2.record(stream)
                    s_out.wait_event(e2)
                    with torch.cuda.stream(s_out):
                        hout[j][c0:c1].copy_(out[c0:c1], non_blocking=True)
            done = torch.cuda.Event()
            done.record(s_out)
            stream.wait_event(done)
            s_in.wait_stream(stream)   # the next step's uploads wait for this step's convs

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        ems = reduce_max(a.elapsed_time(b) / k_e2e, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in hx + hw)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        e2e = {"value": world * total_flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": k_e2e,
               "how": "per conv, the batch in up to 8 chunks; H2D of chunk i+1 and D2H of chunk i-1 overlap the "
                      "conv of chunk i on separate streams; pinned host buffers"}
        del hx, hw, hout, dx, dw

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        big = max(items, key=lambda it: it[0].flops)
        cv, x, w = big[0], big[1], big[2]
        xh = x[:1].cpu()
        r, cores, sample, _ = oracle_sample_rate(cv, xh, w.cpu(), 15.0)
        cpu = {"value": r, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample}

    plan0 = items[0][4]
    per_conv_lines = []
    if args.per_conv and rank == 0:
        per_conv_lines = per_conv_report(bench, peaks)
    config = {"workload": desc, "plan": {k: plan0[k] for k in ("algo", "engine", "winograd_m", "batch_tile",
                                                               "num_batch_tiles", "tile_n")},
              "convs_per_step": len(items), "flops_per_step": total_flops,
              "l2": "L2 flushed between steps (outside the events)" if bench.flush is not None
              else f"inputs larger than L2 ({bench.in_bytes / 1e9:.2f} GB per step)",
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
              "cuda_graph": bool(args.graph)}

    return {"value": value, "ms": ms, "dtype": dtype, "desc": desc, "config": config, "roof": roof,
            "kernels": kernels, "clocks": clocks, "gpu_launches": gpu_launches,
            "launches_per_step": launches_per_step, "e2e": e2e, "cpu": cpu, "fp32_pk": fp32_pk,
            "per_conv_lines": per_conv_lines, "sptr": sptr}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="winograd_f32")
    ap.add_argument("--algo", default="auto", choices=["auto", "implicit", "winograd", "direct"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-config block")
    ap.add_argument("--per-config-only", default="", help="comma-separated per-config keys to run (default: all)")
    ap.add_argument("--per-conv", action="store_true", help="also print one line per conv of the workload")
    ap.add_argument("--graph", action="store_true",
                    help="capture one step as a CUDA graph and time its replays (removes host launch gaps)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, args.workload)
        return

    import torch
    from dense_convolution_nhwc_b200 import binding as B

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()

    h = run_headline(args, B, torch, dev, stream, world, rank, local, peaks)
    torch.cuda.empty_cache()
    value, ms, dtype, config, roof, kernels, clocks = (h["value"], h["ms"], h["dtype"], h["config"], h["roof"],
                                                       h["kernels"], h["clocks"])
    gpu_launches, launches_per_step, e2e, cpu, fp32_pk = (h["gpu_launches"], h["launches_per_step"], h["e2e"],
                                                          h["cpu"], h["fp32_pk"])
    per_conv_lines, sptr = h["per_conv_lines"], h["sptr"]

    per_config = None
    if not args.no_per_config:
        only = {k for k in args.per_config_only.split(",") if k}
        per_config = {}
        for key, wl, algo, use_graph, *rest in PER_CONFIG:
            if only and key not in only:
                continue
            try:
                per_config[key] = per_config_entry(key, wl, algo, use_graph, dev, stream, world, peaks, fp32_pk,
                                                   min_steps=10, env=rest[0] if rest else None)
            except Exception as exc:      # report, never hide, a failed entry
                per_config[key] = {"error": f"{type(exc).__name__}: {exc}"}
        assert B.conv_check(sptr) == 0

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": (value / PAGES_NUMBER[args.workload]) if args.workload in PAGES_NUMBER else None,
            "dtype": dtype, "data": "synthetic", "config": config,
            "roofline": roof, "kernels": kernels, "clocks": clocks, "gpu_launches": gpu_launches,
            "gpu_launches_per_step": launches_per_step,
            "e2e": e2e, "cpu_baseline": cpu,
        }
        if args.workload in PAGES_NUMBER:
            line["vs_baseline_note"] = "pages' 310 ms on an M2 Max for the same workload (context, other hardware)"
        if per_config is not None:
            line["per_config"] = per_config
        print(json.dumps(line))
        for l in per_conv_lines:
            print(json.dumps(l))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def per_conv_report(bench, peaks):
    """One line per conv of the workload: its own event time and kernel split."""
    import torch
    B = bench.B
    lines = []
    evs = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for cv, x, w, d, plan, out in bench.items:
        def fwd_one():
            st = bench.fwd(x.data_ptr(), w.data_ptr(), out.data_ptr(), d, bench.dt_code, bench.opts,
                           bench.ws.data_ptr(), bench.ws.numel(), bench.sptr)
            if st != 0:
                raise B.ConvError(st, cv.name)
        for _ in range(3):
            fwd_one()
        reps = 10
        times = []
        for _ in range(reps):
            if bench.flush is not None:
                bench.flush.zero_()
            evs[0].record(bench.stream)
            fwd_one()
            evs[1].record(bench.stream)
            torch.cuda.synchronize()
            times.append(evs[0].elapsed_time(evs[1]))
        t = statistics.median(times)
        B.conv_profile_begin()
        for _ in range(reps):
            fwd_one()
        torch.cuda.synchronize()
        kp = B.profile_end()
        kw = kernel_work(cv, plan)
        ker = {}
        for kn, (nl, tot) in kp.items():
            kms = tot / reps
            f, b = kw.get(kn, (0.0, 0.0))
            ker[kn] = {"ms": kms, "tflops": f / (kms * 1e-3) / 1e12 if f else None,
                       "gbs": b / (kms * 1e-3) / 1e9 if b else None}
        lines.append({"conv": cv.name, "dtype": cv.dtype, "algo": plan["algo"], "engine": plan["engine"],
                      "tile_n": plan["tile_n"], "k_split": plan["k_split"], "ms": t,
                      "tflops": cv.flops / (t * 1e-3) / 1e12,
                      "frac_of_bf16_peak": cv.flops / (t * 1e-3) / 1e12 / (peaks.get("bf16_tflops") or 1590.0),
                      "kernels": ker})
    return lines


if __name__ == "__main__":
    main()
