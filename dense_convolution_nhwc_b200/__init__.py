"""B200 (sm_100a) NHWC convolution forward.

The library itself is the C-ABI shared object built from ``csrc/`` (declared in
``include/b200conv.h``); ``binding`` marshals arguments into it with ctypes and
nothing else.  The binding is loaded on first use of one of its names, and
loading fails loudly if the shared object has not been built: there is no CPU
fallback.
"""
_BINDING_NAMES = frozenset({
    # C-ABI entry points (same names as include/b200conv.h)
    "conv2d_forward", "conv3d_forward", "conv1d_forward", "conv1d_plan", "conv1d_workspace_size", "conv2d_forward_winograd_static", "conv2d_plan", "conv3d_plan",
    "conv2d_plan_for_props", "conv3d_plan_for_props",
    "conv2d_workspace_size", "conv3d_workspace_size", "conv_check", "conv_selftest_timeout", "conv_fp32_fma_rate",
    "fp32_fma_rate",
    "conv_status_string", "conv_device_props", "conv_accumulate", "conv_profile_begin", "conv_profile_end",
    "profile_end", "KernelTime",
    # types and helpers
    "ConvError", "Conv1dDesc", "Conv2dDesc", "Conv3dDesc", "ConvPlan", "ConvOptions", "DeviceProps",
    "ALGO", "DTYPE", "STATUS", "ENGINE", "library_path", "make_desc2d", "make_desc3d", "make_options",
    # torch conveniences
    "conv1d", "conv2d", "conv3d", "plan2d", "plan3d",
})


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(f"module 'dense_convolution_nhwc_b200' has no attribute {name!r}")
