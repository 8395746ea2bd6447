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


def run_conv2d(x, w, shape: synth.Conv2dShape, options=None, poison=True):
    out = torch.full((shape.n, shape.oh, shape.ow, shape.o), float("nan"), dtype=x.dtype, device=x.device) \
        if poison else None
    out = B.conv2d(x, w, shape.stride, shape.pad, shape.dilation, options=options, out=out)
    torch.cuda.synchronize()
    assert B.conv_check(torch.cuda.current_stream().cuda_stream) == 0
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
