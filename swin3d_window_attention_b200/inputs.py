"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds no arithmetic of the attention or AdaLN methods: it only draws
numbers.  The generator is counter based, so element ``i`` of stream ``key`` is a
pure function of ``(key, i)`` and any slice of a tensor can be regenerated on its
own.

Definition (written out so the stream can be re-implemented anywhere):

* ``splitmix64(x)``: ``z = x + 0x9E3779B97F4A7C15``;
  ``z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9``; ``z = (z ^ (z >> 27)) * 0x94D049BB133111EB``;
  ``return z ^ (z >> 31)`` (all mod 2**64).  This is Steele, Lea and Flood's SplitMix64
  finaliser ("Fast splittable pseudorandom number generators", OOPSLA 2014).
* Stream key: ``splitmix64(seed * 0x100000001B3 + tensor_index)``.
* Pair ``n`` of a stream draws ``z = splitmix64(key ^ (n * 0xD1B54A32D192ED03))``;
  ``u1 = ((z >> 40) + 0.5) / 2**24`` and ``u2 = (((z >> 16) & 0xFFFFFF) + 0.5) / 2**24``.
* Box-Muller (Box and Muller, 1958): ``r = sqrt(-2 ln u1)``; element ``2n`` is
  ``r cos(2 pi u2)`` and element ``2n+1`` is ``r sin(2 pi u2)``; both are scaled by ``sigma``
  and rounded to float32.
* bf16 values are the float32 values rounded to nearest, ties to even, on the bit
  pattern (no NaN can occur).

The seed is 42 throughout, as in the Flash-Aurora numerical check.
"""
from __future__ import annotations

import numpy as np

SEED = 42

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_PAIR = np.uint64(0xD1B54A32D192ED03)
_SEEDMUL = np.uint64(0x100000001B3)

_CHUNK = 1 << 22  # pairs per numpy chunk; bounds temporaries to ~100 MB


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on a uint64 array (wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = (x + _GOLDEN).astype(np.uint64)
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_index: int) -> np.uint64:
    with np.errstate(over="ignore"):
        x = np.uint64(seed) * _SEEDMUL + np.uint64(tensor_index)
    return splitmix64(np.array([x], dtype=np.uint64))[0]


def normal_f32(n: int, seed: int = SEED, tensor_index: int = 0, sigma: float = 1.0) -> np.ndarray:
    """``n`` float32 samples of N(0, sigma^2) from stream (seed, tensor_index)."""
    key = stream_key(seed, tensor_index)
    out = np.empty(n, dtype=np.float32)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, _CHUNK):
        p1 = min(npairs, p0 + _CHUNK)
        idx = np.arange(p0, p1, dtype=np.uint64)
        with np.errstate(over="ignore"):
            z = splitmix64(key ^ (idx * _PAIR))
        u1 = ((z >> np.uint64(40)).astype(np.float64) + 0.5) * (1.0 / (1 << 24))
        u2 = (((z >> np.uint64(16)) & np.uint64(0xFFFFFF)).astype(np.float64) + 0.5) * (1.0 / (1 << 24))
        r = np.sqrt(-2.0 * np.log(u1)) * sigma
        ang = 2.0 * np.pi * u2
        pair = np.empty((p1 - p0, 2), dtype=np.float32)
        pair[:, 0] = r * np.cos(ang)
        pair[:, 1] = r * np.sin(ang)
        flat = pair.reshape(-1)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = flat[: hi - lo]
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_bits(shape, seed: int = SEED, tensor_index: int = 0, sigma: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    return f32_to_bf16_bits(normal_f32(n, seed, tensor_index, sigma)).reshape(shape)


def normal_f32_tensor(shape, seed: int = SEED, tensor_index: int = 0, sigma: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    return normal_f32(n, seed, tensor_index, sigma).reshape(shape)


def attention_qkv_bits(B, T, H, W, channels, seed=SEED, base_index=0, token_stride=None):
    """Q, K, V as bf16 bit arrays of shape [B, T, H, W, token_stride].

    Channels beyond ``channels`` (when token_stride > channels) are filled with a
    distinct stream so that a kernel reading them by mistake shows up in parity.
    """
    ts = channels if token_stride is None else token_stride
    shape = (B, T, H, W, ts)
    return tuple(normal_bf16_bits(shape, seed, base_index + i) for i in range(3))


def bits_to_torch_bf16(bits: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def torch_bf16_to_bits(t) -> np.ndarray:
    import torch

    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _to_i64(u: int) -> int:
    """A uint64 constant as the int64 with the same bit pattern."""
    return u - (1 << 64) if u >= (1 << 63) else u


def normal_f32_torch(n: int, device, seed: int = SEED, tensor_index: int = 0, sigma: float = 1.0,
                     chunk_pairs: int = 1 << 25):
    """The same stream as :func:`normal_f32`, evaluated with torch int64 / float64 ops on
    ``device`` (for inputs too large to draw on the host in a test).  int64 arithmetic
    wraps like uint64; right shifts are made logical by masking.  The float64 log, sqrt,
    cos and sin may differ from numpy's in the last bit, so a float32 sample can differ by
    one unit in rare cases: tests that use this hand the same device tensor to both sides."""
    import torch

    def lsr(z, k):
        return (z >> k) & ((1 << (64 - k)) - 1)

    def mix(x):
        z = x + _to_i64(int(_GOLDEN))
        z = (z ^ lsr(z, 30)) * _to_i64(int(_M1))
        z = (z ^ lsr(z, 27)) * _to_i64(int(_M2))
        return z ^ lsr(z, 31)

    key = _to_i64(int(stream_key(seed, tensor_index)))
    out = torch.empty(n, dtype=torch.float32, device=device)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, chunk_pairs):
        p1 = min(npairs, p0 + chunk_pairs)
        idx = torch.arange(p0, p1, dtype=torch.int64, device=device)
        z = mix(key ^ (idx * _to_i64(int(_PAIR))))
        u1 = (lsr(z, 40).to(torch.float64) + 0.5) * (1.0 / (1 << 24))
        u2 = ((lsr(z, 16) & 0xFFFFFF).to(torch.float64) + 0.5) * (1.0 / (1 << 24))
        r = torch.sqrt(-2.0 * torch.log(u1)) * sigma
        ang = 2.0 * np.pi * u2
        pair = torch.stack([(r * torch.cos(ang)).to(torch.float32), (r * torch.sin(ang)).to(torch.float32)], 1)
        lo, hi = 2 * p0, min(n, 2 * p1)
        out[lo:hi] = pair.reshape(-1)[: hi - lo]
    return out


def normal_bf16_torch(shape, device, seed: int = SEED, tensor_index: int = 0, sigma: float = 1.0):
    """bf16 tensor of the stream on ``device`` (float32 rounded to nearest, ties to even)."""
    import torch

    n = int(np.prod(shape))
    return normal_f32_torch(n, device, seed, tensor_index, sigma).to(torch.bfloat16).reshape(shape)
