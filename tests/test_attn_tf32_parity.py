"""GPU parity of the TF32_ACC_FP32 mode of swin3d_window_attn_fwd (fp32 Q/K/V) against the
fp64 oracle, through the C ABI.

Bar (fp32 output): max-abs 1e-2 and relative L2 2e-3.  Every operand the tensor cores read is
TF32: Q, K and V as the MMA reads fp32 (relative error below 2^-10), P rounded to nearest
(2^-11); accumulation is FP32.  A logit is scale * a sum of head_dim products: for N(0,1)
inputs, head_dim 64 and scale 1/8 its error is about 1e-3 rms; the softmax carries it into P
and O at about 1.4 times, so the expected relative L2 error of O is about 1e-3 (measured
1.1e-3), and 2e-3 leaves a factor of two.  With bf16 output the output rounding (2^-9)
dominates and the bar of the BF16 path applies (max-abs 1e-2, relative L2 3e-3).
"""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, edge_window_ids

TF32_MAX_ABS = 1e-2
TF32_REL_L2 = 2e-3


def bar(out_dtype):
    return (TF32_MAX_ABS, TF32_REL_L2) if out_dtype == torch.float32 else (ATTN_MAX_ABS, ATTN_REL_L2)

pytestmark = pytest.mark.gpu

SENTINEL = 8192.0

SMALL = [
    # (B, T, H, W, heads, hd, window, shift)
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (1, 3, 6)),    # tiny workload
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (0, 0, 0)),
    (2, 4, 13, 29, 3, 64, (2, 6, 12), (1, 3, 6)),    # ragged on H and W, pad != shift
    (1, 5, 7, 11, 2, 64, (2, 6, 12), (1, 2, 5)),     # pad on every axis, odd shifts
    (1, 4, 12, 24, 4, 64, (2, 6, 12), (0, 0, 0)),    # exact tiling, unshifted
    (2, 3, 5, 7, 2, 32, (2, 3, 4), (1, 1, 2)),       # N = 24 window
    (1, 2, 3, 3, 1, 64, (1, 1, 1), (0, 0, 0)),       # N = 1
    (1, 4, 6, 12, 1, 64, (4, 6, 6), (3, 5, 5)),      # N = 144 with another window shape
    (1, 4, 36, 72, 8, 64, (2, 6, 12), (1, 3, 6)),    # several tiles per CTA (576 tiles)
]


def case_id(c):
    return f"B{c[0]}T{c[1]}H{c[2]}W{c[3]}h{c[4]}d{c[5]}w{c[6]}s{c[7]}"


def f32_qkv(B, T, H, W, ts, base):
    return tuple(inputs.normal_f32_tensor((B, T, H, W, ts), tensor_index=base + j) for j in range(3))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["o_f32", "o_bf16"])
@pytest.mark.parametrize("case", SMALL, ids=case_id)
def test_tf32_small_grids_full_compare(cuda_ok, case, out_dtype):
    B, T, H, W, heads, hd, window, shift = case
    C = heads * hd
    host = f32_qkv(B, T, H, W, C, 3000)
    q, k, v = (torch.from_numpy(a).cuda() for a in host)
    o = torch.full((B, T, H, W, C + 8), SENTINEL, dtype=out_dtype, device="cuda")
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    got = o.float().cpu().numpy().astype(np.float64)
    assert np.all(got[..., C:] == SENTINEL), "channels beyond heads*head_dim were written"
    got = got[..., :C]
    assert not np.any(got == SENTINEL), "a real token was not written"
    ref = oracle.window_attn_grid(*host, heads, hd, window, shift)
    mx, rl2 = attn_errors(got, ref)
    print(f"tf32 {case_id(case)} {out_dtype}: max-abs {mx:.3e} rel-L2 {rl2:.3e}")
    mab, rlb = bar(out_dtype)
    assert mx <= mab and rl2 <= rlb, (mx, rl2)


def test_tf32_fused_qkv_buffer(cuda_ok):
    """q, k, v as channel slices of one fp32 [tokens][3C] buffer."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 13, 25, 2, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    host = f32_qkv(B, T, H, W, C, 3100)
    fused = torch.from_numpy(np.concatenate(host, axis=-1)).cuda()
    q, k, v = fused[..., :C], fused[..., C:2 * C], fused[..., 2 * C:]
    o = torch.empty((B, T, H, W, C), dtype=torch.float32, device="cuda")
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    ref = oracle.window_attn_grid(*host, heads, hd, window, shift)
    mx, rl2 = attn_errors(o.cpu().numpy(), ref)
    assert mx <= TF32_MAX_ABS and rl2 <= TF32_REL_L2, (mx, rl2)


@pytest.mark.parametrize("shift", [(1, 3, 6), (0, 0, 0)], ids=["shifted", "unshifted"])
def test_tf32_stage1_full_size_sampled(cuda_ok, shift):
    """Stage 1 (B=1, 4x180x360, 8 x 64) in fp32: sampled windows against the oracle, and the
    properties that hold at any size on the whole output."""
    B, T, H, W, heads, hd, window = 1, 4, 180, 360, 8, 64, (2, 6, 12)
    C = heads * hd
    dev = [inputs.normal_f32_torch(B * T * H * W * C, "cuda", tensor_index=3200 + j).reshape(B, T, H, W, C)
           for j in range(3)]
    o = torch.full((B, T, H, W, C), SENTINEL, dtype=torch.float32, device="cuda")
    s3w.swin3d_window_attn_fwd(*dev, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    host = tuple(t.cpu().numpy() for t in dev)
    ids = edge_window_ids(B, T, H, W, window, extra_random=12)
    out, tok, _ = oracle.window_attn(*host, heads, hd, window, shift, window_ids=ids)
    real = tok >= 0
    got = o.view(-1, C)[torch.from_numpy(tok[real]).cuda()].cpu().numpy()
    mx, rl2 = attn_errors(got, out[real])
    print(f"tf32 stage1 {shift}: max-abs {mx:.3e} rel-L2 {rl2:.3e}")
    assert mx <= TF32_MAX_ABS and rl2 <= TF32_REL_L2, (mx, rl2)
    assert not torch.any(o == SENTINEL)
    assert torch.isfinite(o).all()
    vmax = dev[2].abs().amax()
    assert float(o.abs().amax()) <= float(vmax) * (1 + 2 ** -10)


def test_tf32_bounded_wait_timeout(cuda_ok):
    """The TF32 kernel's bounded waits unwind like the BF16 kernel's."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 36, 72, 8, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    host = f32_qkv(B, T, H, W, C, 3300)
    q, k, v = (torch.from_numpy(a).cuda() for a in host)
    o = torch.zeros((B, T, H, W, C), dtype=torch.float32, device="cuda")
    assert s3w.poll_device_error() == 0
    prev = s3w.set_wait_limit_ns(1_000_000)
    prev_stall = s3w.set_test_stall(True)
    try:
        s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
        status = s3w.poll_device_error()
    finally:
        s3w.set_test_stall(prev_stall)
        s3w.set_wait_limit_ns(prev)
    assert status == 5
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    ref = oracle.window_attn_grid(*host, heads, hd, window, shift)
    mx, rl2 = attn_errors(o.cpu().numpy(), ref)
    assert mx <= TF32_MAX_ABS and rl2 <= TF32_REL_L2, (mx, rl2)
