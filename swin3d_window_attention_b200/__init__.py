"""B200-native (sm_100a) Swin3D shifted-window attention and AdaLN + residual.

The compute lives in CUDA kernels behind a C ABI (``include/swin3d_wa.h``); this
package is the thin ctypes binding over that library.  Importing the package does not
load the shared library; the first call does, and fails loudly if it is missing.
"""
from .api import (  # noqa: F401
    S3WError,
    adaln_residual_fwd,
    library_path,
    load_library,
    poll_device_error,
    set_test_stall,
    set_wait_limit_ns,
    status_string,
    swin3d_window_attn_adaln_fwd,
    swin3d_window_attn_adaln_fwd_static_ws,
    swin3d_window_attn_fwd,
    swin3d_window_attn_fwd_legacy_mma,
    swin3d_qkv_proj_fwd,
    swin3d_qkv_window_attn_fwd,
    window_attn_adaln_workspace_bytes,
)
