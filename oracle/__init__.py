"""CPU oracle for NHWC/NDHWC convolution forward -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
leg may import this package.  The GPU library never calls it, shares no code
with it, and must fail loudly (never fall back here) when its CUDA extension is
missing.

The arithmetic lives in ``oracle_conv.c``: the direct nested-loop sum

    out[n,oh,ow,o] = sum_{kh,kw,c} in[n, oh*sh-ph+kh*dh, ow*sw-pw+kw*dw, c] * w[o,kh,kw,c]

accumulated in float64 after an exact conversion of every input element, the
"CPU reference" that each of the MLX pull requests "Bound winograd conv2d
working set by tiling the batch" (Testing), "Use the explicit gemm for wide
convs on neural accelerators" (Verified) and "Decompose small kernel-depth 3D
convs into 2D convs" (Results) checks its GPU kernels against.  This module
only marshals numpy arrays into it.

Every function here is pinned by ``tests/test_oracle.py`` against brute force,
closed forms, textbook identities and a library convolution.
"""
import ctypes
import os

import numpy as np

from . import build as _build

DTYPE_CODES = {"f32": 0, "f16": 1, "bf16": 2}

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        LL = ctypes.c_longlong
        lib.oracle_conv3d.argtypes = [P, P, I] + [I] * 18 + [P, LL, P, I]
        lib.oracle_conv3d.restype = I
        lib.oracle_conv2d.argtypes = [P, P, I] + [I] * 13 + [P, LL, P, I]
        lib.oracle_conv2d.restype = I
        lib.oracle_decode.argtypes = [I, P, P, LL]
        lib.oracle_decode.restype = I
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = I
        _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def _raw(a, dtype: str) -> np.ndarray:
    """Storage bits as a contiguous numpy array (float32 or uint16)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if dtype == "f32":
                a = a.view(torch.float32).numpy()
            else:
                a = a.view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    want = np.float32 if dtype == "f32" else np.uint16
    if a.dtype == np.float16 and dtype == "f16":
        a = a.view(np.uint16)
    if a.dtype != want:
        raise TypeError(f"oracle: expected {want} storage for {dtype}, got {a.dtype}")
    return a


def out_size(i: int, k: int, s: int, p: int, d: int) -> int:
    return (i + 2 * p - d * (k - 1) - 1) // s + 1


def decode(a, dtype: str) -> np.ndarray:
    """Exact float64 value of every element of a float32/f16/bf16 storage array."""
    raw = _raw(a, dtype)
    out = np.empty(raw.shape, dtype=np.float64)
    rc = _load().oracle_decode(DTYPE_CODES[dtype], raw.ctypes.data, out.ctypes.data, raw.size)
    if rc != 0:
        raise ValueError("oracle_decode failed")
    return out


def conv2d(x, w, dtype: str, stride=(1, 1), pad=(0, 0), dilation=(1, 1), pixels=None, threads: int = 0):
    """Direct conv2d in float64.  x: [N,H,W,C] storage, w: [O,KH,KW,C] storage.

    pixels: None for the full [N,OH,OW,O] output, or an int array [P,3] of
    (n, oh, ow) giving a [P,O] result (all output channels of each pixel).
    """
    xr, wr = _raw(x, dtype), _raw(w, dtype)
    N, H, W, C = xr.shape
    O, KH, KW, C2 = wr.shape
    if C2 != C:
        raise ValueError("channel mismatch")
    OH = out_size(H, KH, stride[0], pad[0], dilation[0])
    OW = out_size(W, KW, stride[1], pad[1], dilation[1])
    if pixels is None:
        out = np.empty((N, OH, OW, O), dtype=np.float64)
        pp, npix = None, 0
    else:
        pix = np.ascontiguousarray(pixels, dtype=np.int32).reshape(-1, 3)
        out = np.empty((pix.shape[0], O), dtype=np.float64)
        pp, npix = pix.ctypes.data, pix.shape[0]
    rc = _load().oracle_conv2d(xr.ctypes.data, wr.ctypes.data, DTYPE_CODES[dtype],
                               N, H, W, C, O, KH, KW, stride[0], stride[1], pad[0], pad[1],
                               dilation[0], dilation[1], pp, npix, out.ctypes.data, threads)
    if rc != 0:
        raise ValueError(f"oracle_conv2d failed ({rc})")
    return out


def conv3d(x, w, dtype: str, stride=(1, 1, 1), pad=(0, 0, 0), dilation=(1, 1, 1), pixels=None,
           threads: int = 0):
    """Direct conv3d in float64.  x: [N,D,H,W,C], w: [O,KD,KH,KW,C].

    pixels: None for the full [N,OD,OH,OW,O] output, or [P,4] of (n, od, oh, ow).
    """
    xr, wr = _raw(x, dtype), _raw(w, dtype)
    N, D, H, W, C = xr.shape
    O, KD, KH, KW, C2 = wr.shape
    if C2 != C:
        raise ValueError("channel mismatch")
    OD = out_size(D, KD, stride[0], pad[0], dilation[0])
    OH = out_size(H, KH, stride[1], pad[1], dilation[1])
    OW = out_size(W, KW, stride[2], pad[2], dilation[2])
    if pixels is None:
        out = np.empty((N, OD, OH, OW, O), dtype=np.float64)
        pp, npix = None, 0
    else:
        pix = np.ascontiguousarray(pixels, dtype=np.int32).reshape(-1, 4)
        out = np.empty((pix.shape[0], O), dtype=np.float64)
        pp, npix = pix.ctypes.data, pix.shape[0]
    rc = _load().oracle_conv3d(xr.ctypes.data, wr.ctypes.data, DTYPE_CODES[dtype],
                               N, D, H, W, C, O, KD, KH, KW,
                               stride[0], stride[1], stride[2], pad[0], pad[1], pad[2],
                               dilation[0], dilation[1], dilation[2], pp, npix, out.ctypes.data, threads)
    if rc != 0:
        raise ValueError(f"oracle_conv3d failed ({rc})")
    return out
