"""ctypes binding of ``libb200conv.so`` (declared in ``include/b200conv.h``).

The functions named like the C entry points take raw device pointers (ints)
and return the integer status, exactly as the C ABI does.  ``conv2d`` /
``conv3d`` are torch conveniences that allocate the output and the workspace
with torch on the input's device and enqueue on torch's current stream; every
step of the convolution runs in the library's kernels.

Importing this module fails loudly if the shared object is missing: there is
no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Union

HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(HERE, "libb200conv.so")

if not os.path.exists(library_path):
    raise ImportError(
        f"dense_convolution_nhwc_b200: {library_path} is missing; build it with "
        "`python -m dense_convolution_nhwc_b200.build` (nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(library_path)

DTYPE = {"f32": 0, "f16": 1, "bf16": 2}
ALGO = {"auto": 0, "implicit": 1, "winograd": 2, "direct": 3}
ENGINE = {0: "none", 1: "tcgen05", 2: "simt"}
STATUS = {0: "CONV_OK", 1: "CONV_ERR_INVALID", 2: "CONV_ERR_UNSUPPORTED", 3: "CONV_ERR_ALIGNMENT",
          4: "CONV_ERR_WORKSPACE", 5: "CONV_ERR_CUDA", 6: "CONV_ERR_TIMEOUT"}


class Conv2dDesc(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int), ("c", ctypes.c_int),
                ("o", ctypes.c_int), ("kh", ctypes.c_int), ("kw", ctypes.c_int),
                ("stride", ctypes.c_int * 2), ("pad", ctypes.c_int * 2), ("dilation", ctypes.c_int * 2)]


class Conv3dDesc(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("d", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int),
                ("c", ctypes.c_int), ("o", ctypes.c_int), ("kd", ctypes.c_int), ("kh", ctypes.c_int),
                ("kw", ctypes.c_int), ("stride", ctypes.c_int * 3), ("pad", ctypes.c_int * 3),
                ("dilation", ctypes.c_int * 3)]


class Conv1dDesc(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("l", ctypes.c_int), ("c", ctypes.c_int), ("o", ctypes.c_int),
                ("k", ctypes.c_int), ("stride", ctypes.c_int), ("pad", ctypes.c_int), ("dilation", ctypes.c_int)]


class DeviceProps(ctypes.Structure):
    _fields_ = [("sm_count", ctypes.c_int), ("cc_major", ctypes.c_int), ("cc_minor", ctypes.c_int),
                ("total_global_mem", ctypes.c_ulonglong)]


class ConvOptions(ctypes.Structure):
    _fields_ = [("algo", ctypes.c_int), ("winograd_budget_bytes", ctypes.c_longlong),
                ("winograd_tile_batch", ctypes.c_int)]


class ConvPlan(ctypes.Structure):
    _fields_ = [("algo", ctypes.c_int), ("engine", ctypes.c_int), ("tile_m", ctypes.c_int),
                ("tile_n", ctypes.c_int), ("winograd_m", ctypes.c_int), ("batch_tile", ctypes.c_int),
                ("num_batch_tiles", ctypes.c_int), ("channel_pad", ctypes.c_int), ("packed_taps", ctypes.c_int),
                ("k_split", ctypes.c_int), ("taps", ctypes.c_int), ("winograd_fused", ctypes.c_int),
                ("winograd_split_bf16", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self) -> dict:
        inv = {v: k for k, v in ALGO.items()}
        return {"algo": inv.get(self.algo, self.algo), "engine": ENGINE.get(self.engine, self.engine),
                "tile_m": self.tile_m, "tile_n": self.tile_n, "winograd_m": self.winograd_m,
                "batch_tile": self.batch_tile, "num_batch_tiles": self.num_batch_tiles,
                "channel_pad": self.channel_pad, "packed_taps": self.packed_taps, "k_split": self.k_split, "taps": self.taps,
                "winograd_fused": self.winograd_fused, "winograd_split_bf16": self.winograd_split_bf16,
                "workspace_bytes": int(self.workspace_bytes)}


_P = ctypes.c_void_p
_I = ctypes.c_int


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_conv_device_props = _sig("conv_device_props", _I, _I, ctypes.POINTER(DeviceProps))
_conv2d_plan = _sig("conv2d_plan", _I, ctypes.POINTER(Conv2dDesc), _I, _I, ctypes.POINTER(ConvOptions),
                    ctypes.POINTER(ConvPlan))
_conv2d_plan_for_props = _sig("conv2d_plan_for_props", _I, ctypes.POINTER(Conv2dDesc), _I,
                              ctypes.POINTER(DeviceProps), ctypes.POINTER(ConvOptions), ctypes.POINTER(ConvPlan))
_conv2d_workspace_size = _sig("conv2d_workspace_size", ctypes.c_size_t, ctypes.POINTER(Conv2dDesc), _I, _I,
                              ctypes.POINTER(ConvOptions))
_conv2d_forward = _sig("conv2d_forward", _I, _P, _P, _P, ctypes.POINTER(Conv2dDesc), _I,
                       ctypes.POINTER(ConvOptions), _P, ctypes.c_size_t, _P)
_conv3d_plan = _sig("conv3d_plan", _I, ctypes.POINTER(Conv3dDesc), _I, _I, ctypes.POINTER(ConvOptions),
                    ctypes.POINTER(ConvPlan))
_conv3d_plan_for_props = _sig("conv3d_plan_for_props", _I, ctypes.POINTER(Conv3dDesc), _I,
                              ctypes.POINTER(DeviceProps), ctypes.POINTER(ConvOptions), ctypes.POINTER(ConvPlan))
_conv3d_workspace_size = _sig("conv3d_workspace_size", ctypes.c_size_t, ctypes.POINTER(Conv3dDesc), _I, _I,
                              ctypes.POINTER(ConvOptions))
_conv3d_forward = _sig("conv3d_forward", _I, _P, _P, _P, ctypes.POINTER(Conv3dDesc), _I,
                       ctypes.POINTER(ConvOptions), _P, ctypes.c_size_t, _P)
_conv1d_plan = _sig("conv1d_plan", _I, ctypes.POINTER(Conv1dDesc), _I, _I, ctypes.POINTER(ConvOptions),
                    ctypes.POINTER(ConvPlan))
_conv1d_workspace_size = _sig("conv1d_workspace_size", ctypes.c_size_t, ctypes.POINTER(Conv1dDesc), _I, _I,
                              ctypes.POINTER(ConvOptions))
_conv1d_forward = _sig("conv1d_forward", _I, _P, _P, _P, ctypes.POINTER(Conv1dDesc), _I,
                       ctypes.POINTER(ConvOptions), _P, ctypes.c_size_t, _P)
_conv_accumulate = _sig("conv_accumulate", _I, _P, _P, ctypes.c_size_t, _I, _P)
_conv2d_forward_winograd_static = _sig("conv2d_forward_winograd_static", _I, _P, _P, _P,
                                       ctypes.POINTER(Conv2dDesc), _I, _P)
_conv_check = _sig("conv_check", _I, _P)
_conv_selftest_timeout = _sig("conv_selftest_timeout", _I, ctypes.c_longlong, _P)
_conv_fp32_fma_rate = _sig("conv_fp32_fma_rate", _I, _I, ctypes.POINTER(ctypes.c_double), _P)
_conv_status_string = _sig("conv_status_string", ctypes.c_char_p, _I)


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


_conv_profile_begin = _sig("conv_profile_begin", _I)
_conv_profile_end = _sig("conv_profile_end", _I, ctypes.POINTER(KernelTime), _I)


class ConvError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({conv_status_string(status)})")


def _opt(opts: Optional[ConvOptions]):
    return ctypes.byref(opts) if opts is not None else None


# ---------------------------------------------------------------------------
# The C entry points, same names, same arguments (ints for pointers)
# ---------------------------------------------------------------------------

def conv_status_string(status: int) -> str:
    return _conv_status_string(status).decode()


def conv_device_props(device: int, props: DeviceProps) -> int:
    return _conv_device_props(device, ctypes.byref(props))


def conv2d_plan(desc: Conv2dDesc, dtype: int, device: int, opts: Optional[ConvOptions], plan: ConvPlan) -> int:
    return _conv2d_plan(ctypes.byref(desc), dtype, device, _opt(opts), ctypes.byref(plan))


def conv2d_plan_for_props(desc: Conv2dDesc, dtype: int, props: DeviceProps, opts: Optional[ConvOptions],
                          plan: ConvPlan) -> int:
    return _conv2d_plan_for_props(ctypes.byref(desc), dtype, ctypes.byref(props), _opt(opts), ctypes.byref(plan))


def conv2d_workspace_size(desc: Conv2dDesc, dtype: int, device: int, opts: Optional[ConvOptions]) -> int:
    return int(_conv2d_workspace_size(ctypes.byref(desc), dtype, device, _opt(opts)))


def conv2d_forward(inp: int, w: int, out: int, desc: Conv2dDesc, dtype: int, opts: Optional[ConvOptions],
                   workspace: int, workspace_bytes: int, stream: int) -> int:
    return _conv2d_forward(inp, w, out, ctypes.byref(desc), dtype, _opt(opts), workspace or None,
                           workspace_bytes, stream or None)


def conv1d_plan(desc: Conv1dDesc, dtype: int, device: int, opts: Optional[ConvOptions], plan: ConvPlan) -> int:
    return _conv1d_plan(ctypes.byref(desc), dtype, device, _opt(opts), ctypes.byref(plan))


def conv1d_workspace_size(desc: Conv1dDesc, dtype: int, device: int, opts: Optional[ConvOptions]) -> int:
    return int(_conv1d_workspace_size(ctypes.byref(desc), dtype, device, _opt(opts)))


def conv1d_forward(inp: int, w: int, out: int, desc: Conv1dDesc, dtype: int, opts: Optional[ConvOptions],
                   workspace: int, workspace_bytes: int, stream: int) -> int:
    return _conv1d_forward(inp, w, out, ctypes.byref(desc), dtype, _opt(opts), workspace or None,
                           workspace_bytes, stream or None)


def conv3d_plan(desc: Conv3dDesc, dtype: int, device: int, opts: Optional[ConvOptions], plan: ConvPlan) -> int:
    return _conv3d_plan(ctypes.byref(desc), dtype, device, _opt(opts), ctypes.byref(plan))


def conv3d_plan_for_props(desc: Conv3dDesc, dtype: int, props: DeviceProps, opts: Optional[ConvOptions],
                          plan: ConvPlan) -> int:
    return _conv3d_plan_for_props(ctypes.byref(desc), dtype, ctypes.byref(props), _opt(opts), ctypes.byref(plan))


def conv3d_workspace_size(desc: Conv3dDesc, dtype: int, device: int, opts: Optional[ConvOptions]) -> int:
    return int(_conv3d_workspace_size(ctypes.byref(desc), dtype, device, _opt(opts)))


def conv3d_forward(inp: int, w: int, out: int, desc: Conv3dDesc, dtype: int, opts: Optional[ConvOptions],
                   workspace: int, workspace_bytes: int, stream: int) -> int:
    return _conv3d_forward(inp, w, out, ctypes.byref(desc), dtype, _opt(opts), workspace or None,
                           workspace_bytes, stream or None)


def conv2d_forward_winograd_static(inp: int, w: int, out: int, desc: Conv2dDesc, dtype: int, stream: int) -> int:
    """Winograd conv2d with the library's fixed 64 MiB device scratch: no workspace, no allocation."""
    return _conv2d_forward_winograd_static(inp, w, out, ctypes.byref(desc), dtype, stream or None)


def conv_accumulate(out: int, tap: int, count: int, dtype: int, stream: int) -> int:
    return _conv_accumulate(out, tap, count, dtype, stream or None)


def conv_check(stream: int) -> int:
    return _conv_check(stream or None)


def conv_selftest_timeout(limit_ns: int, stream: int) -> int:
    return _conv_selftest_timeout(limit_ns, stream or None)


def conv_fp32_fma_rate(packed: int, tflops, stream: int) -> int:
    """tflops: a ctypes.c_double filled with the measured fp32 FMA rate (TFLOP/s)."""
    return _conv_fp32_fma_rate(packed, ctypes.byref(tflops), stream or None)


def fp32_fma_rate(packed: bool = True, stream: int = 0) -> float:
    """The measured CUDA-core fp32 FMA rate of the current device, TFLOP/s."""
    v = ctypes.c_double(0.0)
    st = _conv_fp32_fma_rate(1 if packed else 0, ctypes.byref(v), stream or None)
    if st != 0:
        raise ConvError(st, "conv_fp32_fma_rate")
    return v.value


def conv_profile_begin() -> int:
    return _conv_profile_begin()


def conv_profile_end(out, max_entries: int) -> int:
    return _conv_profile_end(out, max_entries)


def profile_end() -> dict:
    """Stop kernel timing; {kernel name: (launches, total ms)} since conv_profile_begin()."""
    buf = (KernelTime * 32)()
    n = conv_profile_end(buf, 32)
    if n < 0:
        raise ConvError(5, "conv_profile_end")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(n)}


# ---------------------------------------------------------------------------
# Descriptor / option helpers
# ---------------------------------------------------------------------------

def _pair(v, n):
    if isinstance(v, int):
        return (v,) * n
    v = tuple(v)
    if len(v) != n:
        raise ValueError(f"expected {n} values, got {v}")
    return v


def make_desc2d(n, h, w, c, o, kh, kw, stride=1, pad=0, dilation=1) -> Conv2dDesc:
    d = Conv2dDesc(n, h, w, c, o, kh, kw)
    d.stride[:] = list(_pair(stride, 2))
    d.pad[:] = list(_pair(pad, 2))
    d.dilation[:] = list(_pair(dilation, 2))
    return d


def make_desc3d(n, dd, h, w, c, o, kd, kh, kw, stride=1, pad=0, dilation=1) -> Conv3dDesc:
    d = Conv3dDesc(n, dd, h, w, c, o, kd, kh, kw)
    d.stride[:] = list(_pair(stride, 3))
    d.pad[:] = list(_pair(pad, 3))
    d.dilation[:] = list(_pair(dilation, 3))
    return d


def make_options(algo: str = "auto", winograd_budget_bytes: int = -1, winograd_tile_batch: int = 0) -> ConvOptions:
    return ConvOptions(ALGO[algo], winograd_budget_bytes, winograd_tile_batch)


# ---------------------------------------------------------------------------
# torch conveniences (memory and streams only)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    m = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
    if t not in m:
        raise TypeError(f"unsupported dtype {t}")
    return m[t]


def _check(x, name):
    torch = _torch()
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous (NHWC / OHWI)")


def _check_out(out, shape, like):
    """A caller's out= must be exactly the tensor the library will write: the C
    ABI sees only a pointer, so a wrong shape, dtype, device or stride here
    would become an out-of-bounds device write.  Raises before any launch."""
    torch = _torch()
    if not isinstance(out, torch.Tensor):
        raise ValueError(f"out must be a torch tensor, got {type(out).__name__}")
    if not out.is_cuda or out.device != like.device:
        raise ValueError(f"out is on {out.device}, the input on {like.device}")
    if out.dtype != like.dtype:
        raise ValueError(f"out has dtype {out.dtype}, the input {like.dtype}")
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out has shape {tuple(out.shape)}, the conv writes {tuple(shape)}")
    if not out.is_contiguous():
        raise ValueError("out must be contiguous (NHWC)")


def _check_workspace(ws, need, like):
    """A caller's workspace= must sit on the input's device, be contiguous and
    hold at least the bytes the plan asks for.  Raises before any launch."""
    torch = _torch()
    if not isinstance(ws, torch.Tensor):
        raise ValueError(f"workspace must be a torch tensor, got {type(ws).__name__}")
    if not ws.is_cuda or ws.device != like.device:
        raise ValueError(f"workspace is on {ws.device}, the input on {like.device}")
    if not ws.is_contiguous():
        raise ValueError("workspace must be contiguous")
    have = ws.numel() * ws.element_size()
    if have < need:
        raise ValueError(f"workspace holds {have} bytes, the plan needs {need}")


def _check_pair(x, w):
    _check(x, "x")
    _check(w, "w")
    if x.dtype != w.dtype:
        raise TypeError("x and w must share a dtype")
    if x.device != w.device:
        raise ValueError(f"x is on {x.device}, w on {w.device}")


def plan2d(desc: Conv2dDesc, dtype: str, device: int = 0, options: Optional[ConvOptions] = None) -> dict:
    p = ConvPlan()
    st = conv2d_plan(desc, DTYPE[dtype], device, options, p)
    if st != 0:
        raise ConvError(st, "conv2d_plan")
    return p.as_dict()


def plan3d(desc: Conv3dDesc, dtype: str, device: int = 0, options: Optional[ConvOptions] = None) -> dict:
    p = ConvPlan()
    st = conv3d_plan(desc, DTYPE[dtype], device, options, p)
    if st != 0:
        raise ConvError(st, "conv3d_plan")
    return p.as_dict()


def conv2d(x, w, stride=1, padding=0, dilation=1, options: Optional[ConvOptions] = None, out=None,
           workspace=None):
    """NHWC conv2d: x [N,H,W,C], w [O,KH,KW,C] -> [N,OH,OW,O] on x's device."""
    torch = _torch()
    _check_pair(x, w)
    N, H, W, C = x.shape
    O, KH, KW, C2 = w.shape
    if C2 != C:
        raise ValueError("channel mismatch")
    desc = make_desc2d(N, H, W, C, O, KH, KW, stride, padding, dilation)
    dt = _dtype_code(x.dtype)
    dev = x.device.index if x.device.index is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        plan = ConvPlan()
        st = conv2d_plan(desc, dt, dev, options, plan)
        if st != 0:
            raise ConvError(st, "conv2d_plan")
        s, p, d = _pair(stride, 2), _pair(padding, 2), _pair(dilation, 2)
        OH = (H + 2 * p[0] - d[0] * (KH - 1) - 1) // s[0] + 1
        OW = (W + 2 * p[1] - d[1] * (KW - 1) - 1) // s[1] + 1
        if out is None:
            out = torch.empty((N, OH, OW, O), dtype=x.dtype, device=x.device)
        else:
            _check_out(out, (N, OH, OW, O), x)
        ws_bytes = int(plan.workspace_bytes)
        if workspace is None and ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
        elif workspace is not None:
            _check_workspace(workspace, ws_bytes, x)
        ws_ptr = workspace.data_ptr() if workspace is not None else 0
        ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
        stream = torch.cuda.current_stream(x.device).cuda_stream
        st = conv2d_forward(x.data_ptr(), w.data_ptr(), out.data_ptr(), desc, dt, options, ws_ptr, ws_n, stream)
        if st != 0:
            raise ConvError(st, "conv2d_forward")
    return out


def conv1d(x, w, stride=1, padding=0, dilation=1, options: Optional[ConvOptions] = None, out=None,
           workspace=None):
    """NLC conv1d: x [N,L,C], w [O,K,C] -> [N,OL,O] on x's device (through conv1d_forward)."""
    torch = _torch()
    _check_pair(x, w)
    N, L, C = x.shape
    O, K, C2 = w.shape
    if C2 != C:
        raise ValueError("channel mismatch")
    desc = Conv1dDesc(N, L, C, O, K, stride, padding, dilation)
    dt = _dtype_code(x.dtype)
    dev = x.device.index if x.device.index is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        plan = ConvPlan()
        st = conv1d_plan(desc, dt, dev, options, plan)
        if st != 0:
            raise ConvError(st, "conv1d_plan")
        OL = (L + 2 * padding - dilation * (K - 1) - 1) // stride + 1
        if out is None:
            out = torch.empty((N, OL, O), dtype=x.dtype, device=x.device)
        else:
            _check_out(out, (N, OL, O), x)
        ws_bytes = int(plan.workspace_bytes)
        if workspace is None and ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
        elif workspace is not None:
            _check_workspace(workspace, ws_bytes, x)
        ws_ptr = workspace.data_ptr() if workspace is not None else 0
        ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
        stream = torch.cuda.current_stream(x.device).cuda_stream
        st = conv1d_forward(x.data_ptr(), w.data_ptr(), out.data_ptr(), desc, dt, options, ws_ptr, ws_n, stream)
        if st != 0:
            raise ConvError(st, "conv1d_forward")
    return out


def conv3d(x, w, stride=1, padding=0, dilation=1, options: Optional[ConvOptions] = None, out=None,
           workspace=None):
    """NDHWC conv3d: x [N,D,H,W,C], w [O,KD,KH,KW,C] -> [N,OD,OH,OW,O]."""
    torch = _torch()
    _check_pair(x, w)
    N, D, H, W, C = x.shape
    O, KD, KH, KW, C2 = w.shape
    if C2 != C:
        raise ValueError("channel mismatch")
    desc = make_desc3d(N, D, H, W, C, O, KD, KH, KW, stride, padding, dilation)
    dt = _dtype_code(x.dtype)
    dev = x.device.index if x.device.index is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        plan = ConvPlan()
        st = conv3d_plan(desc, dt, dev, options, plan)
        if st != 0:
            raise ConvError(st, "conv3d_plan")
        s, p, d = _pair(stride, 3), _pair(padding, 3), _pair(dilation, 3)
        dims = [(D, KD), (H, KH), (W, KW)]
        OD, OH, OW = [(i + 2 * p[a] - d[a] * (k - 1) - 1) // s[a] + 1 for a, (i, k) in enumerate(dims)]
        if out is None:
            out = torch.empty((N, OD, OH, OW, O), dtype=x.dtype, device=x.device)
        else:
            _check_out(out, (N, OD, OH, OW, O), x)
        ws_bytes = int(plan.workspace_bytes)
        if workspace is None and ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=x.device)
        elif workspace is not None:
            _check_workspace(workspace, ws_bytes, x)
        ws_ptr = workspace.data_ptr() if workspace is not None else 0
        ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
        stream = torch.cuda.current_stream(x.device).cuda_stream
        st = conv3d_forward(x.data_ptr(), w.data_ptr(), out.data_ptr(), desc, dt, options, ws_ptr, ws_n, stream)
        if st != 0:
            raise ConvError(st, "conv3d_forward")
    return out
