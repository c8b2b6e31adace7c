"""fp64 CPU oracle for the shifted-window attention path and AdaLN + residual.

TEST INFRASTRUCTURE: only the test suite, the package's smoke check and the
benchmark's CPU-baseline / reference leg may import this module.  The CUDA path
never calls it and shares no code with it.

The arithmetic lives in ``swin3d_oracle.cpp`` (plain C++, double precision, OpenMP
over independent (window, head) jobs).  This wrapper only marshals numpy arrays.

Parity status of each function (what pins it, in ``tests/test_oracle.py``):
  * ``window_attn``       pinned: brute-force dense masked attention built in the
    forward direction, a PyTorch fp64 roll/pad/partition/SDPA route, closed forms
    (Q = 0 gives the mean of V over the region group, group sizes fixed by hand in
    ``tests/golden/``), softmax rows summing to 1, constant V, shift 0 equal to plain
    block attention, exactly-once merge.
  * ``dense_masked_attn`` pinned against the same PyTorch route and the group sizes.
  * ``adaln``             pinned: ``torch.nn.functional.layer_norm`` in fp64, a
    constant row, zero-input closed form.
  * ``qkv_proj``          pinned: a permutation weight returns the permuted channels
    (a transposed weight or swapped q/k/v thirds fails it), a zero input returns the
    bias, additivity in x, and the q/k/v thirds equal three separate projections.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swin3d_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

IN_BF16, IN_F32, IN_F64 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (OpenMP) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path):
    """Open an oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P, I, LL, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.orc_window_attn.argtypes = [P, P, P, I, I, I, I, I, I, I, I, I, I, I, I, I, LL, D, I, LL, P, P, P, P]
    lib.orc_window_attn.restype = I
    lib.orc_dense_masked_attn.argtypes = [P, P, P, I, I, I, I, I, I, I, I, I, I, I, I, I, LL, D, P]
    lib.orc_dense_masked_attn.restype = I
    lib.orc_adaln.argtypes = [P, I, P, P, P, I, LL, I, D, I, P]
    lib.orc_adaln.restype = I
    lib.orc_num_threads.argtypes = []
    lib.orc_num_threads.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(_LIB_PATH)
    return _lib


def num_threads() -> int:
    return _load().orc_num_threads()


def _kind(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return IN_BF16
    if a.dtype == np.float32:
        return IN_F32
    if a.dtype == np.float64:
        return IN_F64
    raise TypeError(f"unsupported oracle input dtype {a.dtype} (bf16 bits as uint16, float32, float64)")


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def padded_dims(T, H, W, window):
    return tuple(-(-d // w) * w for d, w in zip((T, H, W), window))


def windows_per_sample(T, H, W, window):
    P = padded_dims(T, H, W, window)
    return (P[0] // window[0]) * (P[1] // window[1]) * (P[2] // window[2])


def window_attn(q, k, v, heads, head_dim, window=(2, 6, 12), shift=(0, 0, 0), scale=0.0,
                window_ids=None, mask_mode=0, return_probs=False):
    """Shifted-window attention of grid-layout q/k/v ``[B, T, H, W, token_stride]``.

    Returns ``(out, out_tok, probs)``: ``out`` is ``[n, N, heads*head_dim]`` doubles in
    intra-window order, ``out_tok`` is ``[n, N]`` flat grid indices (-1 = padding), and
    ``probs`` is ``[n, heads, N, N]`` or None.
    """
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    assert q.shape == k.shape == v.shape and q.ndim == 5 and q.dtype == k.dtype == v.dtype
    B, T, H, W, ts = q.shape
    N = window[0] * window[1] * window[2]
    if window_ids is None:
        n = B * windows_per_sample(T, H, W, window)
        ids = None
    else:
        ids = np.ascontiguousarray(window_ids, dtype=np.int64)
        n = ids.size
    C = heads * head_dim
    out = np.empty((n, N, C), dtype=np.float64)
    tok = np.empty((n, N), dtype=np.int64)
    probs = np.empty((n, heads, N, N), dtype=np.float64) if return_probs else None
    rc = _load().orc_window_attn(_ptr(q), _ptr(k), _ptr(v), _kind(q), B, T, H, W, *window, *shift,
                                 heads, head_dim, ts, float(scale), int(mask_mode), n, _ptr(ids),
                                 _ptr(out), _ptr(tok), _ptr(probs))
    if rc != 0:
        raise ValueError("oracle rejected the window-attention arguments")
    return out, tok, probs


def merge_to_grid(out, tok, B, T, H, W):
    """Scatter window rows to their grid tokens (rows with tok = -1 are dropped).

    Returns ``(grid, writes)``: the grid ``[B, T, H, W, C]`` (NaN where nothing was written)
    and the per-token write count.
    """
    C = out.shape[-1]
    L = B * T * H * W
    grid = np.full((L, C), np.nan)
    flat_tok = tok.reshape(-1)
    rows = out.reshape(-1, C)
    keep = flat_tok >= 0
    grid[flat_tok[keep]] = rows[keep]
    writes = np.bincount(flat_tok[keep], minlength=L)
    return grid.reshape(B, T, H, W, C), writes.reshape(B, T, H, W)


def window_attn_grid(q, k, v, heads, head_dim, window=(2, 6, 12), shift=(0, 0, 0), scale=0.0, mask_mode=0):
    B, T, H, W, _ = q.shape
    out, tok, _ = window_attn(q, k, v, heads, head_dim, window, shift, scale, None, mask_mode)
    grid, _ = merge_to_grid(out, tok, B, T, H, W)
    return grid


def dense_masked_attn(q, k, v, heads, head_dim, window=(2, 6, 12), shift=(0, 0, 0), scale=0.0):
    q, k, v = (np.ascontiguousarray(a) for a in (q, k, v))
    B, T, H, W, ts = q.shape
    out = np.empty((B, T, H, W, heads * head_dim), dtype=np.float64)
    rc = _load().orc_dense_masked_attn(_ptr(q), _ptr(k), _ptr(v), _kind(q), B, T, H, W, *window, *shift,
                                       heads, head_dim, ts, float(scale), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the dense-attention arguments")
    return out


def adaln(x, residual, scale, shift, eps=1e-5, film_form=0):
    """AdaLN + residual.  x ``[B, L, C]`` (bf16 bits, f32 or f64); residual ``[B, L, C]``
    f32 or None; scale, shift ``[B, C]`` f32.  Returns ``[B, L, C]`` doubles."""
    x = np.ascontiguousarray(x)
    B, L, C = x.shape
    res = None if residual is None else np.ascontiguousarray(residual, dtype=np.float32)
    sc = np.ascontiguousarray(scale, dtype=np.float32)
    sh = np.ascontiguousarray(shift, dtype=np.float32)
    assert sc.shape == (B, C) and sh.shape == (B, C)
    if res is not None:
        assert res.shape == (B, L, C)
    out = np.empty((B, L, C), dtype=np.float64)
    rc = _load().orc_adaln(_ptr(x), _kind(x), _ptr(res), _ptr(sc), _ptr(sh), B, L, C, float(eps),
                           int(film_form), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the AdaLN arguments")
    return out


def _as_f64(a):
    """bf16 bits (uint16) widened exactly, or a float array as doubles."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def qkv_proj(x, w, b=None):
    """QKV projection of grid-layout tokens ("Flash-Aurora: Toward Efficient Inference for
    Geospatial Foundation Models", section "Mixed-precision inference": the BF16 QKV
    projection ahead of the window attention): ``x`` ``[..., C]`` and ``w`` ``[3C, C]``
    (bf16 bits or floats), ``b`` ``[3C]`` or None.  Returns ``x w^T + b`` in doubles,
    ``[..., 3C]``; one fp64 matrix product (a library primitive) and the bias add."""
    xf, wf = _as_f64(x), _as_f64(w)
    assert wf.ndim == 2 and wf.shape[1] == xf.shape[-1] and wf.shape[0] == 3 * wf.shape[1]
    y = xf.reshape(-1, xf.shape[-1]) @ wf.T
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :]
    return y.reshape(*xf.shape[:-1], wf.shape[0])
