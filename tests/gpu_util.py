"""Shared helpers for the GPU tests: run the library through the C ABI and
compare with the CPU oracle.

Tolerance (the bound every GPU result must meet): over the checked set of
outputs (the full tensor, or all channels of a seeded pixel sample),
max|gpu - oracle| <= tol * max|oracle| with tol = 1e-4 for fp32 and 1e-2 for
fp16/bf16 (fp32 accumulation in both).  The pages' own CPU cross-checks sit
well inside it: fp16 7.5e-4, bf16 5.5e-3, fp32 9.1e-6 ("Use the explicit gemm
for wide convs on neural accelerators", Verified).
"""
import numpy as np
import torch

import oracle
from dense_convolution_nhwc_b200 import binding as B
from dense_convolution_nhwc_b200 import synth

TOL = {"f32": 1e-4, "f16": 1e-2, "bf16": 1e-2}
FULL_MAC_LIMIT = 5e9


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    return float(err / scale) if scale > 0 else float(err)


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output (unwritten or overflow)"
    e = rel_err(got, ref)
    assert e <= TOL[dtype], f"{what}: max|gpu-oracle|/max|oracle| = {e:.3e} > {TOL[dtype]:.0e}"
    return e


GUARD_BYTES = 4096          # canary band on each side of out and of the workspace
GUARD_VALUE = 0x5B          # a byte pattern no kernel writes by accident (not 0, not a NaN half)


NAN_BYTE = 0xFF             # 0xFFFF... is a NaN in fp32, bf16 and fp16 alike


class Guarded:
    """A device buffer of `nbytes` between two canary bands.  The inner
    region starts 4096 bytes into a fresh allocation (so it keeps the
    allocator's 256-byte alignment) and the upper band starts right at its
    last byte, so any write past either end lands in a band.  Around an input
    the bands hold NaN bytes, so a read past either end turns into a NaN in
    the output."""

    def __init__(self, nbytes: int, device, fill: int = GUARD_VALUE):
        self.nbytes = int(nbytes)
        self.fill = fill
        self.buf = torch.full((GUARD_BYTES + self.nbytes + GUARD_BYTES,), fill, dtype=torch.uint8,
                              device=device)

    def inner(self) -> torch.Tensor:
        return self.buf[GUARD_BYTES:GUARD_BYTES + self.nbytes]

    def tensor(self, shape, dtype) -> torch.Tensor:
        return self.inner().view(dtype).view(shape)

    def assert_intact(self, what: str):
        lo = self.buf[:GUARD_BYTES]
        hi = self.buf[GUARD_BYTES + self.nbytes:]
        bad_lo = int((lo != self.fill).sum())
        bad_hi = int((hi != self.fill).sum())
        assert bad_lo == 0 and bad_hi == 0, \
            f"{what}: write outside the buffer ({bad_lo} bytes below, {bad_hi} bytes above)"


def guarded_output(shape, dtype, device):
    """A NaN-poisoned output tensor inside canary bands."""
    esz = torch.empty((), dtype=dtype).element_size()
    g = Guarded(int(np.prod(shape)) * esz, device)
    out = g.tensor(shape, dtype)
    out.fill_(float("nan"))
    return g, out


def guarded_input(t: torch.Tensor):
    """A copy of t inside NaN bands (see Guarded)."""
    g = Guarded(t.numel() * t.element_size(), t.device, fill=NAN_BYTE)
    x = g.tensor(tuple(t.shape), t.dtype)
    x.copy_(t)
    return g, x


def guarded_workspace(nbytes: int, device):
    """The plan's workspace, exactly its size, inside canary bands (None if the plan needs none)."""
    return Guarded(nbytes, device) if nbytes else None


def run_conv2d(x, w, shape: synth.Conv2dShape, options=None):
    """Run through the C ABI with the input and weights inside NaN bands (a read
    past either end of them reaches the output as a NaN), a NaN-poisoned output
    and the exact workspace the plan asks for inside canary bands; every band is
    checked after the call (no write outside out and the workspace, none into
    the inputs)."""
    desc = B.make_desc2d(shape.n, shape.h, shape.w, shape.c, shape.o, shape.kh, shape.kw, shape.stride, shape.pad,
                         shape.dilation)
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[x.dtype]
    plan = B.plan2d(desc, dt, x.device.index or 0, options)
    g_x, xg = guarded_input(x)
    g_w, wg = guarded_input(w)
    g_out, out = guarded_output((shape.n, shape.oh, shape.ow, shape.o), x.dtype, x.device)
    g_ws = guarded_workspace(plan["workspace_bytes"], x.device)
    out = B.conv2d(xg, wg, shape.stride, shape.pad, shape.dilation, options=options, out=out,
                   workspace=g_ws.inner() if g_ws else None)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
    g_out.assert_intact(f"{shape.name()} out")
    g_x.assert_intact(f"{shape.name()} input")
    g_w.assert_intact(f"{shape.name()} weights")
    if g_ws:
        g_ws.assert_intact(f"{shape.name()} workspace")
    return out


def check_conv2d(shape: synth.Conv2dShape, dtype: str, dist: str = "normal", options=None, seed: int = 0,
                 sample: int = 4096):
    """Run on the GPU and compare with the oracle (full, or sampled pixels)."""
    x, w = synth.conv2d_inputs(shape, dtype, dist, seed, device="cuda")
    out = run_conv2d(x, w, shape, options)
    xh, wh = x.cpu(), w.cpu()
    macs = shape.flops / 2
    if macs <= FULL_MAC_LIMIT:
        ref = oracle.conv2d(xh, wh, dtype, shape.stride, shape.pad, shape.dilation)
        got = as_f64(out)
    else:
        pix = synth.sample_pixels(shape.n, shape.oh, shape.ow, sample, seed)
        ref = oracle.conv2d(xh, wh, dtype, shape.stride, shape.pad, shape.dilation, pixels=pix.numpy())
        p = pix.long()
        got = as_f64(out[p[:, 0], p[:, 1], p[:, 2]])
    return assert_close(got, ref, dtype, shape.name())
