"""GPU parity of swin3d_window_attn_adaln_fwd (window attention fused with AdaLN + residual).

Three references:
* the two-call path on the GPU (swin3d_window_attn_fwd, then adaln_residual_fwd): the fused
  call's optional attention output must equal the attention call's output bit for bit (same
  arithmetic), and its AdaLN output must match within 1e-5 (the statistics are merged head by
  head in a different order);
* the oracle's AdaLN fed the fused call's own bf16 attention output and the residual: max-abs
  1e-5, the FP32 AdaLN bar; the attention output itself against the oracle's attention: the
  attention bar (max-abs 1e-2, relative L2 3e-3);
* the oracle's chain (oracle attention -> oracle AdaLN): the attention error passes through
  the normalisation, which divides by the row's standard deviation (about 0.2 here) and
  multiplies by 1 + scale: a 1e-2 error in x moves the output by up to about 0.05, so one
  block is held to max-abs 0.1 and relative L2 3e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs
from tests.helpers import (ADALN_F32_MAX_ABS, ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, edge_window_ids,
                           window_geometry)

pytestmark = pytest.mark.gpu

CHAIN_MAX_ABS = 0.1
CHAIN_REL_L2 = 3e-3


def make(B, T, H, W, heads, hd, base, film_sigma=0.1):
    C = heads * hd
    L = T * H * W
    dev = "cuda"
    q, k, v = (inputs.normal_bf16_torch((B, T, H, W, C), dev, tensor_index=base + j) for j in range(3))
    sc = inputs.normal_f32_torch(B * C, dev, tensor_index=base + 3, sigma=film_sigma).reshape(B, C)
    sh = inputs.normal_f32_torch(B * C, dev, tensor_index=base + 4, sigma=film_sigma).reshape(B, C)
    res = inputs.normal_f32_torch(B * L * C, dev, tensor_index=base + 5).reshape(B, L, C)
    return q, k, v, sc, sh, res


def two_call(q, k, v, sc, sh, res, heads, hd, window, shift, out_dtype=torch.float32):
    B, T, H, W, C = q.shape
    o = torch.empty_like(q)
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    out = torch.empty((B, T * H * W, C), dtype=out_dtype, device="cuda")
    s3w.adaln_residual_fwd(o.view(B, T * H * W, C), res, sc, sh, out, eps=1e-5)
    torch.cuda.synchronize()
    return o, out


def fused(q, k, v, sc, sh, res, heads, hd, window, shift, out_dtype=torch.float32, in_place=False):
    B, T, H, W, C = q.shape
    o = torch.empty_like(q)
    out = res if in_place else torch.empty((B, T * H * W, C), dtype=out_dtype, device="cuda")
    s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, sc, sh, out, heads, hd, window, shift, o=o, eps=1e-5)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    return o, out


SMALL = [
    # (B, T, H, W, heads, hd, window, shift)
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (1, 3, 6)),    # the tiny workload
    (2, 4, 13, 29, 3, 64, (2, 6, 12), (1, 3, 6)),    # ragged grid, pad != shift, C = 192
    (2, 3, 5, 7, 2, 32, (2, 3, 4), (1, 1, 2)),       # N = 24 window
    (1, 4, 36, 72, 8, 64, (2, 6, 12), (1, 3, 6)),    # 72 windows of 8 heads: several windows per CTA
]


def cid(c):
    return f"B{c[0]}T{c[1]}H{c[2]}W{c[3]}h{c[4]}d{c[5]}w{c[6]}s{c[7]}"


@pytest.mark.parametrize("case", SMALL, ids=cid)
def test_fused_matches_two_call_path_and_oracle(cuda_ok, case):
    B, T, H, W, heads, hd, window, shift = case
    C = heads * hd
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=4000)
    o2, out2 = two_call(q, k, v, sc, sh, res, heads, hd, window, shift)
    of, outf = fused(q, k, v, sc, sh, res, heads, hd, window, shift)
    assert torch.equal(of, o2), "fused attention output differs from the attention call's"
    d = float((outf - out2).abs().max())
    assert d <= ADALN_F32_MAX_ABS, d
    # oracle: attention, AdaLN on the GPU's own x, and the chain
    qb, kb, vb = (inputs.torch_bf16_to_bits(t) for t in (q, k, v))
    ref_o = oracle.window_attn_grid(qb, kb, vb, heads, hd, window, shift)
    mx, rl2 = attn_errors(of.float().cpu().numpy(), ref_o)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
    L = T * H * W
    res_h, sc_h, sh_h = res.cpu().numpy(), sc.cpu().numpy(), sh.cpu().numpy()
    want = oracle.adaln(inputs.torch_bf16_to_bits(of).reshape(B, L, C), res_h, sc_h, sh_h)
    assert float(np.abs(outf.cpu().numpy() - want).max()) <= ADALN_F32_MAX_ABS
    chain = oracle.adaln(ref_o.reshape(B, L, C), res_h, sc_h, sh_h)
    mx, rl2 = attn_errors(outf.cpu().numpy(), chain)
    assert mx <= CHAIN_MAX_ABS and rl2 <= CHAIN_REL_L2, (mx, rl2)


def test_fused_in_place_and_bf16_out(cuda_ok):
    B, T, H, W, heads, hd, window, shift = 1, 4, 24, 48, 4, 64, (2, 6, 12), (1, 3, 6)
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=4100, film_sigma=1.0)
    _, out2 = two_call(q, k, v, sc, sh, res, heads, hd, window, shift)
    _, outb = fused(q, k, v, sc, sh, res, heads, hd, window, shift, out_dtype=torch.bfloat16)
    # bf16 out: the fp32 result rounded to nearest even, so within one bf16 step of it
    step = torch.exp2(torch.floor(torch.log2(out2.abs().clamp_min(1e-30))) - 7)
    assert bool(((outb.float() - out2).abs() <= step + 1e-5).all())
    res_copy = res.clone()
    _, outi = fused(q, k, v, sc, sh, res_copy, heads, hd, window, shift, in_place=True)
    assert outi.data_ptr() == res_copy.data_ptr()
    assert float((res_copy - out2).abs().max()) <= ADALN_F32_MAX_ABS


def test_fused_without_attention_output(cuda_ok):
    B, T, H, W, heads, hd, window, shift = 1, 4, 12, 24, 4, 64, (2, 6, 12), (0, 0, 0)
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=4150)
    _, out2 = two_call(q, k, v, sc, sh, res, heads, hd, window, shift)
    out = torch.empty_like(out2)
    s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, sc, sh, out, heads, hd, window, shift, o=None, eps=1e-5)
    torch.cuda.synchronize()
    assert float((out - out2).abs().max()) <= ADALN_F32_MAX_ABS


def test_fused_stage2_full_size(cuda_ok):
    """Stage 2 (B=1, 4x90x180, 16 heads x 64, C=1024, AdaLN on the attention output): the whole
    output against the two-call path, sampled windows against the oracle."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 90, 180, 16, 64, (2, 6, 12), (1, 3, 6)
    C, L = heads * hd, T * H * W
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=4200)
    o2, out2 = two_call(q, k, v, sc, sh, res, heads, hd, window, shift)
    of, outf = fused(q, k, v, sc, sh, res, heads, hd, window, shift)
    assert torch.equal(of, o2)
    assert float((outf - out2).abs().max()) <= ADALN_F32_MAX_ABS
    qb, kb, vb = (inputs.torch_bf16_to_bits(t) for t in (q, k, v))
    ids = edge_window_ids(B, T, H, W, window, extra_random=8)
    ref, tok, _ = oracle.window_attn(qb, kb, vb, heads, hd, window, shift, window_ids=ids)
    real = tok >= 0
    toks = torch.from_numpy(tok[real]).cuda()
    x_gpu = inputs.torch_bf16_to_bits(of.view(-1, C)[toks])
    r = res.view(-1, C)[toks].cpu().numpy()
    want = oracle.adaln(x_gpu[None], r[None], sc.cpu().numpy(), sh.cpu().numpy())[0]
    assert float(np.abs(outf.view(-1, C)[toks].cpu().numpy() - want).max()) <= ADALN_F32_MAX_ABS
    chain = oracle.adaln(ref[real][None], r[None], sc.cpu().numpy(), sh.cpu().numpy())[0]
    mx, rl2 = attn_errors(outf.view(-1, C)[toks].cpu().numpy(), chain)
    assert mx <= CHAIN_MAX_ABS and rl2 <= CHAIN_REL_L2, (mx, rl2)


def test_fused_stack_matches_two_call_stack(cuda_ok):
    """The six-block stage-1 stack at B=4 (alternating shifts, fresh Q/K/V per block, fp32
    residual updated in place, FiLM N(0,1)): the fused call against the two-call path, block by
    block, on the whole residual stream."""
    B, T, H, W, heads, hd, window = 4, 4, 180, 360, 8, 64, (2, 6, 12)
    C, L = heads * hd, T * H * W
    res_a = inputs.normal_f32_torch(B * L * C, "cuda", tensor_index=4300).reshape(B, L, C)
    res_b = res_a.clone()
    o = torch.empty((B, T, H, W, C), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(s3w.window_attn_adaln_workspace_bytes(B, T, H, W, heads, hd, window), dtype=torch.uint8,
                     device="cuda")
    for blk, shift in enumerate([(0, 0, 0), (1, 3, 6)] * 3):
        q, k, v = (inputs.normal_bf16_torch((B, T, H, W, C), "cuda", tensor_index=4310 + 10 * blk + j)
                   for j in range(3))
        sc = inputs.normal_f32_torch(B * C, "cuda", tensor_index=4390 + 2 * blk).reshape(B, C)
        sh = inputs.normal_f32_torch(B * C, "cuda", tensor_index=4391 + 2 * blk).reshape(B, C)
        s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
        s3w.adaln_residual_fwd(o.view(B, L, C), res_a, sc, sh, res_a, eps=1e-5)
        s3w.swin3d_window_attn_adaln_fwd(q, k, v, res_b, sc, sh, res_b, heads, hd, window, shift, workspace=ws,
                                         eps=1e-5)
        torch.cuda.synchronize()
        assert s3w.poll_device_error() == 0
        d = float((res_a - res_b).abs().max())
        # each block adds its own 1e-5-level difference to the residual stream
        assert d <= ADALN_F32_MAX_ABS * (blk + 1), (blk, d)
        del q, k, v


def test_fused_workspace_too_small_is_rejected(cuda_ok):
    B, T, H, W, heads, hd, window = 1, 4, 12, 24, 4, 64, (2, 6, 12)
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=4400)
    need = s3w.window_attn_adaln_workspace_bytes(B, T, H, W, heads, hd, window)
    ws = torch.empty(need - 32, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(res)
    rc = s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, sc, sh, out, heads, hd, window, (0, 0, 0), workspace=ws,
                                          check=False)
    assert rc == 1   # S3W_ERR_INVALID_ARG, nothing launched


def test_fused_bounded_wait_timeout(cuda_ok):
    """The fused kernel unwinds on an expired wait like the attention kernel."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 36, 72, 8, 64, (2, 6, 12), (1, 3, 6)
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=4500)
    out = torch.empty_like(res)
    assert s3w.poll_device_error() == 0
    prev = s3w.set_wait_limit_ns(1_000_000)
    prev_stall = s3w.set_test_stall(True)
    try:
        s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, sc, sh, out, heads, hd, window, shift, eps=1e-5)
        status = s3w.poll_device_error()
    finally:
        s3w.set_test_stall(prev_stall)
        s3w.set_wait_limit_ns(prev)
    assert status == 5
    _, out2 = two_call(q, k, v, sc, sh, res, heads, hd, window, shift)
    _, outf = fused(q, k, v, sc, sh, res, heads, hd, window, shift)
    assert float((outf - out2).abs().max()) <= ADALN_F32_MAX_ABS
