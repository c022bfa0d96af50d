"""B200-native dynamic short convolutions.

Each token generates its own K-tap depthwise causal filter from its hidden
state (low-rank ``z = h A, w = z B`` or head-wise ``w = h W``) and the layer
returns ``y = u + dynamic causal conv(u)``, forward and backward, in
hand-written sm_100a kernels behind the C ABI of ``include/dynconv.h``.

``ops`` holds the torch-facing helpers (output/workspace allocation and an
autograd Function); ``_lib`` is the raw ctypes binding with the C names.
"""
from ._lib import (  # noqa: F401
    ALGO_AUTO, ALGO_SIMT, ALGO_TC, BF16, F32, HEADWISE, LOWRANK, DynConvError, dynconv_bwd, dynconv_desc,
    dynconv_device_status, dynconv_fwd, dynconv_profile_enable, dynconv_profile_read, dynconv_fwd_varlen, dynconv_last_error, dynconv_version,
    dynconv_workspace_bytes, load, make_desc,
)
from .ops import DynamicShortConv, dynamic_short_conv, DynConvPlan  # noqa: F401
