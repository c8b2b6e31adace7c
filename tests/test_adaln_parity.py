"""GPU parity of adaln_residual_fwd against the fp64 oracle, through the C ABI.

FP32 output: max-abs <= 1e-5.  bf16 output: the oracle value rounded to bf16, within one
bf16 rounding step (the kernel's fp32 result and the fp64 result may straddle a rounding
boundary).
"""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs
from tests.helpers import ADALN_F32_MAX_ABS

pytestmark = pytest.mark.gpu


def make_inputs(B, L, C, x_bf16, base, film_sigma=0.1):
    if x_bf16:
        xh = inputs.normal_bf16_bits((B, L, C), tensor_index=base)
        xd = inputs.bits_to_torch_bf16(xh).cuda()
    else:
        xh = inputs.normal_f32_tensor((B, L, C), tensor_index=base)
        xd = torch.from_numpy(xh).cuda()
    res = inputs.normal_f32_tensor((B, L, C), tensor_index=base + 1)
    sc = inputs.normal_f32_tensor((B, C), tensor_index=base + 2, sigma=film_sigma)
    sh = inputs.normal_f32_tensor((B, C), tensor_index=base + 3, sigma=film_sigma)
    dev = (xd, torch.from_numpy(res).cuda(), torch.from_numpy(sc).cuda(), torch.from_numpy(sh).cuda())
    return (xh, res, sc, sh), dev


def check_bf16(got_bf16, ref):
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    # one bf16 step at the value's magnitude, plus the fp32 arithmetic error of the kernel
    # (values near zero have tiny bf16 steps but keep the fp32 rounding of the larger terms)
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= step + 1e-5)


SHAPES = [
    # (B, L, C, x_bf16)
    (1, 1000, 1024, True),     # stage-2 width, bf16 attention output in
    (2, 777, 512, True),       # stage-1 width, ragged row count
    (1, 300, 2048, False),     # stage-3 width, fp32 x
    (3, 17, 96, True),         # C not a multiple of 256 (partial lanes)
    (1, 5, 8, False),          # narrowest row
    (1, 64, 4096, True),       # widest row
]


@pytest.mark.parametrize("case", SHAPES, ids=lambda c: f"B{c[0]}L{c[1]}C{c[2]}{'bf16' if c[3] else 'f32'}")
def test_adaln_f32_out(cuda_ok, case):
    B, L, C, xb = case
    host, dev = make_inputs(B, L, C, xb, base=2000)
    out = torch.empty((B, L, C), dtype=torch.float32, device="cuda")
    s3w.adaln_residual_fwd(dev[0], dev[1], dev[2], dev[3], out, eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.adaln(*host, eps=1e-5)
    assert float(np.abs(out.cpu().numpy() - ref).max()) <= ADALN_F32_MAX_ABS


@pytest.mark.parametrize("case", SHAPES[:3], ids=lambda c: f"B{c[0]}L{c[1]}C{c[2]}")
def test_adaln_bf16_out(cuda_ok, case):
    B, L, C, xb = case
    host, dev = make_inputs(B, L, C, xb, base=2100)
    out = torch.empty((B, L, C), dtype=torch.bfloat16, device="cuda")
    s3w.adaln_residual_fwd(dev[0], dev[1], dev[2], dev[3], out, eps=1e-5)
    torch.cuda.synchronize()
    check_bf16(out, oracle.adaln(*host, eps=1e-5))


def test_adaln_in_place_residual(cuda_ok):
    B, L, C = 2, 500, 512
    host, dev = make_inputs(B, L, C, True, base=2200, film_sigma=1.0)
    res = dev[1]
    s3w.adaln_residual_fwd(dev[0], res, dev[2], dev[3], res, eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.adaln(*host, eps=1e-5)
    assert float(np.abs(res.cpu().numpy() - ref).max()) <= ADALN_F32_MAX_ABS


def test_adaln_stage2_full_size(cuda_ok):
    """Stage-2 AdaLN at full size: 64,800 tokens x 1024, bf16 x, fp32 residual stream."""
    B, L, C = 1, 4 * 90 * 180, 1024
    host, dev = make_inputs(B, L, C, True, base=2300)
    out = torch.empty((B, L, C), dtype=torch.float32, device="cuda")
    s3w.adaln_residual_fwd(dev[0], dev[1], dev[2], dev[3], out, eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.adaln(*host, eps=1e-5)
    assert float(np.abs(out.cpu().numpy() - ref).max()) <= ADALN_F32_MAX_ABS


def test_adaln_zero_tokens(cuda_ok):
    x = torch.empty((1, 0, 64), dtype=torch.bfloat16, device="cuda")
    r = torch.empty((1, 0, 64), dtype=torch.float32, device="cuda")
    sc = torch.zeros((1, 64), device="cuda")
    assert s3w.adaln_residual_fwd(x, r, sc, sc, r) == 0
