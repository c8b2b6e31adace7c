"""GPU parity of the streaming path of swin3d_window_attn_fwd (windows of more than 144 slots:
K/V blocks of whole (t, h) rows streamed past each query block with online-softmax
rescaling) against the fp64 oracle, through the C ABI.

The bar is the attention bar of the BF16 path (max-abs 1e-2, relative L2 3e-3 over real
tokens): the operands and roundings are the same (bf16 Q/K/V, fp32 logits and softmax, P
rounded to bf16, fp32 accumulation); the online rescaling multiplies the running output and
sum by exp2 of max differences in fp32, a relative error of a few fp32 ulps per block.
"""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, edge_window_ids, make_qkv

pytestmark = pytest.mark.gpu

SENTINEL = 8192.0

SMALL = [
    # (B, T, H, W, heads, hd, window, shift)
    (1, 4, 24, 48, 2, 64, (2, 12, 12), (1, 6, 6)),    # N = 288, shifted: two blocks of 72 per slab
    (1, 4, 24, 48, 2, 64, (2, 12, 12), (0, 0, 0)),
    (2, 5, 13, 29, 2, 32, (3, 7, 11), (1, 3, 5)),     # N = 231, one 77-slot block per slab, pad != shift
    (1, 4, 24, 24, 1, 64, (4, 12, 12), (2, 6, 6)),    # N = 576, eight blocks
    (1, 2, 16, 40, 2, 64, (2, 8, 20), (1, 4, 10)),    # N = 320, 80-slot blocks
    (1, 3, 10, 30, 3, 64, (2, 6, 24), (1, 3, 12)),    # N = 288, padded on T, 72-slot blocks
    (1, 2, 20, 20, 2, 32, (1, 16, 16), (0, 8, 8)),    # N = 256, shift only on H and W
    (1, 2, 3, 256, 1, 64, (1, 2, 128), (0, 1, 64)),   # win_w = 128: one row per block
]


def case_id(c):
    return f"B{c[0]}T{c[1]}H{c[2]}W{c[3]}h{c[4]}d{c[5]}w{'x'.join(map(str, c[6]))}s{'x'.join(map(str, c[7]))}"


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["o_bf16", "o_f32"])
@pytest.mark.parametrize("case", SMALL, ids=case_id)
def test_stream_small_grids_full_compare(cuda_ok, case, out_dtype):
    B, T, H, W, heads, hd, window, shift = case
    C = heads * hd
    bits, (q, k, v) = make_qkv(B, T, H, W, C, base=6000)
    o = torch.full((B, T, H, W, C + 8), SENTINEL, dtype=out_dtype, device="cuda")
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    got = o.float().cpu().numpy().astype(np.float64)
    assert np.all(got[..., C:] == SENTINEL), "channels beyond heads*head_dim were written"
    got = got[..., :C]
    assert not np.any(got == SENTINEL), "a real token was not written"
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    mx, rl2 = attn_errors(got, ref)
    print(f"stream {case_id(case)} {out_dtype}: max-abs {mx:.3e} rel-L2 {rl2:.3e}")
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)


def test_stream_q_k_v_slices_of_fused_buffer(cuda_ok):
    B, T, H, W, heads, hd, window, shift = 1, 4, 24, 48, 2, 64, (2, 12, 12), (1, 6, 6)
    C = heads * hd
    bits, dev = make_qkv(B, T, H, W, C, base=6100)
    fused = torch.empty((B, T, H, W, 3 * C), dtype=torch.bfloat16, device="cuda")
    for j in range(3):
        fused[..., j * C:(j + 1) * C] = dev[j]
    q, k, v = fused[..., :C], fused[..., C:2 * C], fused[..., 2 * C:]
    o = torch.empty((B, T, H, W, C), dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    mx, rl2 = attn_errors(o.float().cpu().numpy(), ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)


def test_stream_stage1_grid_sampled(cuda_ok):
    """The stage-1 grid (B=1, 4x180x360, 8 x 64) with (2,12,12) windows, shift (1,6,6): corner,
    edge and random windows against the oracle; every real token written, finite, bounded."""
    from swin3d_window_attention_b200 import inputs

    B, T, H, W, heads, hd, window, shift = 1, 4, 180, 360, 8, 64, (2, 12, 12), (1, 6, 6)
    C = heads * hd
    dev = [inputs.normal_bf16_torch((B, T, H, W, C), "cuda", tensor_index=6200 + j) for j in range(3)]
    o = torch.full((B, T, H, W, C), SENTINEL, dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_window_attn_fwd(*dev, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    host = tuple(inputs.torch_bf16_to_bits(t) for t in dev)
    ids = edge_window_ids(B, T, H, W, window, extra_random=8)
    out, tok, _ = oracle.window_attn(*host, heads, hd, window, shift, window_ids=ids)
    real = tok >= 0
    got = o.view(-1, C)[torch.from_numpy(tok[real]).cuda()].float().cpu().numpy()
    mx, rl2 = attn_errors(got, out[real])
    print(f"stream stage1 (2,12,12): max-abs {mx:.3e} rel-L2 {rl2:.3e}")
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
    assert not torch.any(o == SENTINEL)
    assert torch.isfinite(o.float()).all()
    assert float(o.float().abs().amax()) <= float(dev[2].float().abs().amax()) * (1 + 2 ** -7)


def test_stream_rejections(cuda_ok):
    """Streaming-only limits: BF16 inputs, win_w <= 128; the fused call and the legacy kernel
    take single-tile windows only."""
    B, T, H, W, heads, hd = 1, 2, 4, 260, 1, 64
    C = heads * hd
    q = torch.zeros((B, T, H, W, C), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    assert s3w.swin3d_window_attn_fwd(q, q, q, o, heads, hd, (1, 2, 130), (0, 0, 0), check=False) == 2
    qf = q.float()
    assert s3w.swin3d_window_attn_fwd(qf, qf, qf, qf.clone(), heads, hd, (2, 2, 64), (0, 0, 0), check=False) == 2
    assert s3w.swin3d_window_attn_fwd_legacy_mma(q, q, q, o, heads, hd, (2, 2, 64), (0, 0, 0), check=False) == 2
    res = torch.zeros((B, T * H * W, C), dtype=torch.float32, device="cuda")
    sc = torch.zeros((B, C), dtype=torch.float32, device="cuda")
    rc = s3w.swin3d_window_attn_adaln_fwd(q, q, q, res, sc, sc, res, heads, hd, (2, 2, 64), (0, 0, 0),
                                          workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"),
                                          check=False)
    assert rc == 2


def test_stream_bounded_wait_timeout(cuda_ok):
    """The streaming kernel's bounded waits unwind like the other kernels'."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 24, 48, 2, 64, (2, 12, 12), (1, 6, 6)
    C = heads * hd
    bits, (q, k, v) = make_qkv(B, T, H, W, C, base=6300)
    o = torch.zeros((B, T, H, W, C), dtype=torch.bfloat16, device="cuda")
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
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    mx, rl2 = attn_errors(o.float().cpu().numpy(), ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
