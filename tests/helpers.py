"""Shared helpers of the parity tests: seeded inputs on host and device, error metrics."""
import numpy as np

import oracle
from swin3d_window_attention_b200 import inputs

# Tolerances of the attention path (bf16 inputs, fp32 accumulation / softmax) and of the
# FP32 AdaLN path, against the fp64 oracle.
ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 3e-3
ADALN_F32_MAX_ABS = 1e-5


def window_geometry(T, H, W, window):
    P = oracle.padded_dims(T, H, W, window)
    n = tuple(P[a] // window[a] for a in range(3))
    return P, n


def edge_window_ids(B, T, H, W, window, extra_random=8, seed=0):
    """Window ids covering every combination of first / last window along each axis in
    every sample, plus a few seeded random ones."""
    _, n = window_geometry(T, H, W, window)
    per = n[0] * n[1] * n[2]
    ids = set()
    for b in range(B):
        for it in {0, n[0] - 1}:
            for ih in {0, n[1] - 1}:
                for iw in {0, n[2] - 1}:
                    ids.add(b * per + (it * n[1] + ih) * n[2] + iw)
    rng = np.random.default_rng(seed)
    for x in rng.integers(0, B * per, size=extra_random):
        ids.add(int(x))
    return sorted(ids)


def attn_errors(got, ref):
    """(max-abs, relative L2) between two float64 arrays of equal shape."""
    d = got.astype(np.float64) - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def make_qkv(B, T, H, W, C, base, token_stride=None, device="cuda"):
    """Seeded bf16 Q, K, V: (host bit arrays, device bf16 tensors)."""
    bits = inputs.attention_qkv_bits(B, T, H, W, C, base_index=base, token_stride=token_stride)
    dev = tuple(inputs.bits_to_torch_bf16(b).to(device) for b in bits)
    return bits, dev
