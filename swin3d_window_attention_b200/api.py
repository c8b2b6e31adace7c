"""ctypes binding of the C ABI in include/swin3d_wa.h.

Argument marshalling only: every step of the computation runs in the CUDA library.
Tensors are PyTorch CUDA tensors (PyTorch supplies device memory and streams); the
current stream of the tensors' device is passed to the library.  There is no CPU
fallback: if the shared library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libswin3d_wa.so"

S3W_OK, S3W_ERR_INVALID_ARG, S3W_ERR_UNSUPPORTED, S3W_ERR_MISALIGNED, S3W_ERR_CUDA, S3W_ERR_DEVICE_TIMEOUT = range(6)
S3W_BF16, S3W_F32 = 0, 1

_lib = None


class S3WError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def library_path() -> str:
    return os.path.join(HERE, _LIB_NAME)


def load_library():
    """Load the in-tree shared library; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m swin3d_window_attention_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    lib.swin3d_window_attn_fwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, I, LL, LL, F, I, I, P]
    lib.swin3d_window_attn_fwd.restype = I
    lib.swin3d_window_attn_fwd_legacy_mma.argtypes = lib.swin3d_window_attn_fwd.argtypes
    lib.swin3d_window_attn_fwd_legacy_mma.restype = I
    lib.s3w_set_wait_limit_ns.argtypes = [LL]
    lib.s3w_set_wait_limit_ns.restype = LL
    lib.s3w_set_test_stall.argtypes = [ctypes.c_int]
    lib.s3w_set_test_stall.restype = ctypes.c_int
    lib.adaln_residual_fwd.argtypes = [P, I, P, P, P, P, I, I, LL, I, F, P]
    lib.adaln_residual_fwd.restype = I
    lib.s3w_status_string.argtypes = [I]
    lib.s3w_status_string.restype = ctypes.c_char_p
    lib.s3w_poll_device_error.argtypes = [P]
    lib.s3w_poll_device_error.restype = I
    lib.s3w_version.argtypes = []
    lib.s3w_version.restype = I
    lib.swin3d_window_attn_adaln_fwd.argtypes = [P, P, P, LL, P, P, P, P, I, P, P, LL, I, I, I, I, I, I, I, I, I, I,
                                                 I, I, F, F, P]
    lib.swin3d_window_attn_adaln_fwd.restype = I
    lib.swin3d_window_attn_adaln_workspace_bytes.argtypes = [I] * 9
    lib.swin3d_window_attn_adaln_workspace_bytes.restype = LL
    lib.swin3d_window_attn_adaln_fwd_static_ws.argtypes = [P, P, P, LL, P, P, P, P, I, P] + [I] * 12 + [F, F, P]
    lib.swin3d_window_attn_adaln_fwd_static_ws.restype = I
    lib.swin3d_qkv_proj_fwd.argtypes = [P, P, P, P, LL, I, P]
    lib.swin3d_qkv_proj_fwd.restype = I
    lib.swin3d_qkv_window_attn_fwd.argtypes = [P, P, P, P, P, I] + [I] * 12 + [F, P]
    lib.swin3d_qkv_window_attn_fwd.restype = I
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().s3w_status_string(int(status)).decode()


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return S3W_BF16
    if t.dtype == torch.float32:
        return S3W_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_of(t) -> int:
    import torch

    return torch.cuda.current_stream(t.device).cuda_stream


def _token_stride(t, C: int) -> int:
    """Elements between consecutive grid tokens of a [B, T, H, W, >=C] view."""
    if t.dim() != 5:
        raise ValueError("expected a grid-layout tensor [B, T, H, W, channels]")
    if t.stride(4) != 1:
        raise ValueError("channels must be contiguous")
    ts = t.stride(3)
    if t.stride(2) != ts * t.shape[3] or t.stride(1) != t.stride(2) * t.shape[2] or t.stride(0) != t.stride(1) * t.shape[1]:
        raise ValueError("grid tokens must be evenly strided")
    if t.shape[4] < C:
        raise ValueError("fewer channels than heads * head_dim")
    return ts


def swin3d_window_attn_fwd(q, k, v, o, heads: int, head_dim: int, window=(2, 6, 12), shift=(0, 0, 0),
                           scale: float = 0.0, stream=None, check: bool = True) -> int:
    """Shifted-window attention (tcgen05 path).  q, k, v: bf16 CUDA tensors
    [B, T, H, W, >=heads*head_dim] with one token stride; o: bf16 or fp32
    [B, T, H, W, >=heads*head_dim].  Returns the status (raises S3WError on a non-zero
    status when ``check``)."""
    return _attn("swin3d_window_attn_fwd", q, k, v, o, heads, head_dim, window, shift, scale, stream, check)


def swin3d_window_attn_fwd_legacy_mma(q, k, v, o, heads: int, head_dim: int, window=(2, 6, 12), shift=(0, 0, 0),
                                      scale: float = 0.0, stream=None, check: bool = True) -> int:
    """The same call on the legacy mma.sync baseline kernel."""
    return _attn("swin3d_window_attn_fwd_legacy_mma", q, k, v, o, heads, head_dim, window, shift, scale, stream,
                 check)


def _attn(entry, q, k, v, o, heads, head_dim, window, shift, scale, stream, check):
    lib = load_library()
    C = heads * head_dim
    B, T, H, W = q.shape[:4]
    ts = _token_stride(q, C)
    if _token_stride(k, C) != ts or _token_stride(v, C) != ts:
        raise ValueError("q, k and v must share one token stride")
    if tuple(o.shape[:4]) != (B, T, H, W) or tuple(k.shape[:4]) != (B, T, H, W) or tuple(v.shape[:4]) != (B, T, H, W):
        raise ValueError("q, k, v and o must have the same grid shape")
    ots = _token_stride(o, C)
    st = _stream_of(q) if stream is None else stream
    rc = getattr(lib, entry)(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), B, T, H, W,
                                    *window, *shift, heads, head_dim, ts, ots, float(scale),
                                    _dtype_code(q), _dtype_code(o), st)
    if check and rc != S3W_OK:
        raise S3WError(rc, entry)
    return rc


def window_attn_adaln_workspace_bytes(B, T, H, W, heads: int, head_dim: int, window=(2, 6, 12)) -> int:
    """Workspace bytes of the fused attention + AdaLN call on the current device."""
    n = int(load_library().swin3d_window_attn_adaln_workspace_bytes(B, T, H, W, *window, heads, head_dim))
    if n < 0:
        raise S3WError(-n, "swin3d_window_attn_adaln_workspace_bytes")
    return n


def swin3d_window_attn_adaln_fwd(q, k, v, residual, scale, shift, out, heads: int, head_dim: int,
                                 window=(2, 6, 12), shift_=(0, 0, 0), o=None, workspace=None, eps: float = 1e-5,
                                 attn_scale: float = 0.0, stream=None, check: bool = True) -> int:
    """Window attention fused with AdaLN + residual.  q, k, v: bf16 [B, T, H, W, >=C] (one token
    stride); residual: fp32 [B, L, C]; scale, shift: fp32 [B, C]; out: fp32/bf16 [B, L, C] (may
    be ``residual``); o: optional bf16 [B, T, H, W, C] for the attention output.  workspace: a
    CUDA tensor of at least window_attn_adaln_workspace_bytes(...) bytes (allocated here when
    None)."""
    import torch

    lib = load_library()
    C = heads * head_dim
    B, T, H, W = q.shape[:4]
    ts = _token_stride(q, C)
    if _token_stride(k, C) != ts or _token_stride(v, C) != ts:
        raise ValueError("q, k and v must share one token stride")
    for t in (residual, out):
        if not t.is_contiguous() or t.numel() != B * T * H * W * C:
            raise ValueError("residual and out must be contiguous [B, L, C]")
    if o is not None and (not o.is_contiguous() or o.dtype != torch.bfloat16 or tuple(o.shape) != (B, T, H, W, C)):
        raise ValueError("o must be a contiguous bf16 [B, T, H, W, C] tensor")
    need = window_attn_adaln_workspace_bytes(B, T, H, W, heads, head_dim, window)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _stream_of(q) if stream is None else stream
    rc = lib.swin3d_window_attn_adaln_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), ts, residual.data_ptr(),
                                          scale.data_ptr(), shift.data_ptr(), out.data_ptr(), _dtype_code(out),
                                          None if o is None else o.data_ptr(), workspace.data_ptr(), ws_bytes,
                                          B, T, H, W, *window, *shift_, heads, head_dim, float(attn_scale),
                                          float(eps), st)
    if check and rc != S3W_OK:
        raise S3WError(rc, "swin3d_window_attn_adaln_fwd")
    return rc


def swin3d_window_attn_adaln_fwd_static_ws(q, k, v, residual, scale, shift, out, heads: int, head_dim: int,
                                           window=(2, 6, 12), shift_=(0, 0, 0), o=None, eps: float = 1e-5,
                                           attn_scale: float = 0.0, stream=None, check: bool = True) -> int:
    """The fused call on the library's static workspace: allocates nothing, here or in the
    library.  Same arguments and results as :func:`swin3d_window_attn_adaln_fwd` without
    ``workspace``; every call on a device shares the one workspace, so calls must not overlap
    on the GPU."""
    import torch

    lib = load_library()
    C = heads * head_dim
    B, T, H, W = q.shape[:4]
    ts = _token_stride(q, C)
    if _token_stride(k, C) != ts or _token_stride(v, C) != ts:
        raise ValueError("q, k and v must share one token stride")
    for t in (residual, out):
        if not t.is_contiguous() or t.numel() != B * T * H * W * C:
            raise ValueError("residual and out must be contiguous [B, L, C]")
    if o is not None and (not o.is_contiguous() or o.dtype != torch.bfloat16 or tuple(o.shape) != (B, T, H, W, C)):
        raise ValueError("o must be a contiguous bf16 [B, T, H, W, C] tensor")
    st = _stream_of(q) if stream is None else stream
    rc = lib.swin3d_window_attn_adaln_fwd_static_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), ts, residual.data_ptr(),
                                                    scale.data_ptr(), shift.data_ptr(), out.data_ptr(),
                                                    _dtype_code(out), None if o is None else o.data_ptr(),
                                                    B, T, H, W, *window, *shift_, heads, head_dim, float(attn_scale),
                                                    float(eps), st)
    if check and rc != S3W_OK:
        raise S3WError(rc, "swin3d_window_attn_adaln_fwd_static_ws")
    return rc


def swin3d_qkv_proj_fwd(x, w, b, qkv, stream=None, check: bool = True) -> int:
    """QKV projection on the tensor cores.  x: contiguous bf16 [..., C]; w: contiguous bf16
    [3C, C]; b: fp32 [3C] or None; qkv: contiguous bf16 [..., 3C] (the same leading shape)."""
    lib = load_library()
    C = x.shape[-1]
    tokens = x.numel() // C
    for t in (x, w, qkv):
        if not t.is_contiguous():
            raise ValueError("x, w and qkv must be contiguous")
    if tuple(w.shape) != (3 * C, C) or qkv.numel() != tokens * 3 * C or qkv.shape[-1] != 3 * C:
        raise ValueError("w must be [3C, C] and qkv [..., 3C]")
    st = _stream_of(x) if stream is None else stream
    rc = lib.swin3d_qkv_proj_fwd(x.data_ptr(), w.data_ptr(), None if b is None else b.data_ptr(), qkv.data_ptr(),
                                 tokens, C, st)
    if check and rc != S3W_OK:
        raise S3WError(rc, "swin3d_qkv_proj_fwd")
    return rc


def swin3d_qkv_window_attn_fwd(x, w, b, qkv, o, heads: int, head_dim: int, window=(2, 6, 12), shift=(0, 0, 0),
                               scale: float = 0.0, stream=None, check: bool = True) -> int:
    """QKV projection followed by the shifted-window attention on its output.  x: contiguous bf16
    [B, T, H, W, C]; w: bf16 [3C, C]; b: fp32 [3C] or None; qkv: bf16 [B, T, H, W, 3C]
    workspace (holds the projected q, k, v afterwards); o: bf16 or fp32 [B, T, H, W, C]."""
    lib = load_library()
    B, T, H, W, C = x.shape
    if C != heads * head_dim:
        raise ValueError("x must have heads * head_dim channels")
    for t in (x, w, qkv, o):
        if not t.is_contiguous():
            raise ValueError("x, w, qkv and o must be contiguous")
    if tuple(qkv.shape) != (B, T, H, W, 3 * C) or tuple(o.shape) != (B, T, H, W, C) or tuple(w.shape) != (3 * C, C):
        raise ValueError("qkv must be [B, T, H, W, 3C], o [B, T, H, W, C] and w [3C, C]")
    st = _stream_of(x) if stream is None else stream
    rc = lib.swin3d_qkv_window_attn_fwd(x.data_ptr(), w.data_ptr(), None if b is None else b.data_ptr(),
                                        qkv.data_ptr(), o.data_ptr(), _dtype_code(o), B, T, H, W, *window, *shift,
                                        heads, head_dim, float(scale), st)
    if check and rc != S3W_OK:
        raise S3WError(rc, "swin3d_qkv_window_attn_fwd")
    return rc


def adaln_residual_fwd(x, residual, scale, shift, out, eps: float = 1e-5, stream=None, check: bool = True) -> int:
    """AdaLN + residual.  x: bf16/fp32 [B, L, C]; residual: fp32 [B, L, C]; scale, shift:
    fp32 [B, C]; out: fp32/bf16 [B, L, C] (may be ``residual`` itself)."""
    lib = load_library()
    B, L, C = x.shape
    for t in (x, residual, out):
        if not t.is_contiguous():
            raise ValueError("x, residual and out must be contiguous")
    st = _stream_of(x) if stream is None else stream
    rc = lib.adaln_residual_fwd(x.data_ptr(), _dtype_code(x), residual.data_ptr(), scale.data_ptr(),
                                shift.data_ptr(), out.data_ptr(), _dtype_code(out), B, L, C, float(eps), st)
    if check and rc != S3W_OK:
        raise S3WError(rc, "adaln_residual_fwd")
    return rc


def poll_device_error(stream=None) -> int:
    import torch

    st = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return load_library().s3w_poll_device_error(st)


def set_wait_limit_ns(ns: int) -> int:
    """Set the kernels' bounded-wait limit (ns); returns the previous one."""
    return int(load_library().s3w_set_wait_limit_ns(int(ns)))


def set_test_stall(on: bool) -> bool:
    """Failure injection for tests: later attention launches first wait on a barrier that
    nothing signals, so they take the bounded-wait timeout path.  Returns the previous
    setting."""
    return bool(load_library().s3w_set_test_stall(1 if on else 0))
