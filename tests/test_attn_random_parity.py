"""Seeded random sweep of swin3d_window_attn_fwd against the fp64 oracle: window shapes on both
sides of 144 slots (single-tile and streaming kernels), random shifts and grid sizes (so padding
on any axis and pad != shift), 1-3 heads of 32 or 64, bf16 or fp32 output, and the TF32 mode
where it applies.  Every element of every case is compared at the bar of its precision."""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, make_qkv

pytestmark = pytest.mark.gpu

TF32_MAX_ABS, TF32_REL_L2 = 1e-2, 2e-3


def cases(n=72, seed=2026):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        big = len(out) % 3 == 2   # every third case a window of more than 144 slots
        if big:
            wt, wh, ww = int(rng.integers(1, 5)), int(rng.integers(2, 14)), int(rng.integers(4, 33))
            if not 144 < wt * wh * ww <= 600:
                continue
        else:
            wt, wh, ww = int(rng.integers(1, 4)), int(rng.integers(1, 9)), int(rng.integers(1, 17))
            if wt * wh * ww > 144:
                continue
        win = (wt, wh, ww)
        shift = tuple(int(rng.integers(0, a)) for a in win)
        grid = tuple(int(rng.integers(1, int(2.5 * a) + 2)) for a in win)
        B = int(rng.integers(1, 3))
        heads, hd = int(rng.integers(1, 4)), int(rng.choice([32, 64]))
        out_f32 = bool(rng.integers(0, 2))
        tf32 = (not big) and bool(rng.integers(0, 3) == 0)
        out.append((B, grid, win, shift, heads, hd, out_f32, tf32))
    return out


def cid(c):
    B, grid, win, shift, heads, hd, out_f32, tf32 = c
    return (f"B{B}g{'x'.join(map(str, grid))}w{'x'.join(map(str, win))}s{'x'.join(map(str, shift))}"
            f"h{heads}d{hd}{'f32' if out_f32 else 'bf16'}{'_tf32' if tf32 else ''}")


@pytest.mark.parametrize("case", cases(), ids=cid)
def test_random_geometry(cuda_ok, case):
    B, (T, H, W), win, shift, heads, hd, out_f32, tf32 = case
    C = heads * hd
    if tf32:
        host = tuple(inputs.normal_f32_tensor((B, T, H, W, C), tensor_index=8000 + j) for j in range(3))
        q, k, v = (torch.from_numpy(a).cuda() for a in host)
    else:
        host, (q, k, v) = make_qkv(B, T, H, W, C, base=8000)
    o = torch.full((B, T, H, W, C), 8192.0, dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, win, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    got = o.float().cpu().numpy().astype(np.float64)
    assert not np.any(got == 8192.0), "a real token was not written"
    ref = oracle.window_attn_grid(*host, heads, hd, win, shift)
    mx, rl2 = attn_errors(got, ref)
    bar = (TF32_MAX_ABS, TF32_REL_L2) if (tf32 and out_f32) else (ATTN_MAX_ABS, ATTN_REL_L2)
    assert mx <= bar[0] and rl2 <= bar[1], (mx, rl2)
