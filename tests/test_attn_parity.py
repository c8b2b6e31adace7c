"""GPU parity of swin3d_window_attn_fwd against the fp64 oracle, through the C ABI.

Small grids (several windows, ragged padding, every wrap) are compared element by element
over every real token; the full-size workloads are compared on sampled windows (every
first/last-window combination along each axis plus seeded random windows), which the
oracle computes one by one.  Bar: max-abs <= 1e-2 and relative L2 <= 3e-3 (bf16 inputs,
fp32 accumulation).  Every real token must be written exactly where the oracle's merge
puts it; padded slots and channels beyond heads*head_dim must stay untouched.
"""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, edge_window_ids, make_qkv

pytestmark = pytest.mark.gpu

SENTINEL = 8192.0   # exact in bf16; written into o before the call; must survive outside the real channels


IMPLS = {"tcgen05": s3w.swin3d_window_attn_fwd, "legacy_mma": s3w.swin3d_window_attn_fwd_legacy_mma}


def run_gpu(dev_qkv, B, T, H, W, heads, hd, window, shift, out_dtype, o_extra=0, impl="tcgen05"):
    C = heads * hd
    o = torch.full((B, T, H, W, C + o_extra), SENTINEL, dtype=out_dtype, device="cuda")
    q, k, v = dev_qkv
    IMPLS[impl](q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    return o


SMALL = [
    # (B, T, H, W, heads, hd, window, shift)
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (1, 3, 6)),    # tiny workload
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (0, 0, 0)),
    (2, 4, 13, 29, 3, 64, (2, 6, 12), (1, 3, 6)),    # ragged on H and W, pad != shift
    (1, 5, 7, 11, 2, 64, (2, 6, 12), (1, 2, 5)),     # pad on every axis, odd shifts
    (1, 4, 12, 24, 4, 64, (2, 6, 12), (0, 0, 0)),    # exact tiling, unshifted
    (2, 3, 5, 7, 2, 32, (2, 3, 4), (1, 1, 2)),       # N = 24 window
    (1, 2, 3, 3, 1, 64, (1, 1, 1), (0, 0, 0)),       # N = 1: each token attends to itself
    (1, 1, 1, 1, 1, 64, (2, 6, 12), (1, 3, 6)),      # a single real token in one window
    (1, 4, 6, 12, 1, 64, (4, 6, 6), (3, 5, 5)),      # N = 144 with another window shape
]


def case_id(c):
    return f"B{c[0]}T{c[1]}H{c[2]}W{c[3]}h{c[4]}d{c[5]}w{c[6]}s{c[7]}"


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["o_bf16", "o_f32"])
@pytest.mark.parametrize("case", SMALL, ids=case_id)
def test_small_grids_full_compare(cuda_ok, case, out_dtype):
    _small_compare(case, out_dtype, "tcgen05")


@pytest.mark.parametrize("case", [SMALL[0], SMALL[2], SMALL[5]], ids=case_id)
def test_legacy_mma_baseline_small(cuda_ok, case):
    _small_compare(case, torch.bfloat16, "legacy_mma")


def _small_compare(case, out_dtype, impl):
    B, T, H, W, heads, hd, window, shift = case
    C = heads * hd
    bits, dev = make_qkv(B, T, H, W, C, base=10)
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    o = run_gpu(dev, B, T, H, W, heads, hd, window, shift, out_dtype, o_extra=8, impl=impl)
    got = o.float().cpu().numpy().astype(np.float64)
    assert np.all(got[..., C:] == SENTINEL), "channels beyond heads*head_dim were written"
    got = got[..., :C]
    assert not np.any(got == SENTINEL), "a real token was not written"
    mx, rl2 = attn_errors(got, ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)


def test_fused_qkv_buffer_token_stride(cuda_ok):
    """q, k, v as three channel slices of one [tokens][3C] buffer (token stride 3C)."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 13, 25, 2, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    bits, _ = make_qkv(B, T, H, W, C, base=20)
    fused = np.concatenate(bits, axis=-1)
    from swin3d_window_attention_b200 import inputs

    dev = inputs.bits_to_torch_bf16(fused).cuda()
    q, k, v = dev[..., :C], dev[..., C:2 * C], dev[..., 2 * C:]
    o = torch.empty((B, T, H, W, C), dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_window_attn_fwd(q, k, v, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    mx, rl2 = attn_errors(o.float().cpu().numpy(), ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)


def test_f32_output_rows_only_16_byte_aligned(cuda_ok):
    """o token stride C + 4 floats: rows start on 16- but not 32-byte boundaries."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 13, 25, 2, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    bits, dev = make_qkv(B, T, H, W, C, base=25)
    o = run_gpu(dev, B, T, H, W, heads, hd, window, shift, torch.float32, o_extra=4)
    got = o.cpu().numpy().astype(np.float64)
    assert np.all(got[..., C:] == SENTINEL)
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    mx, rl2 = attn_errors(got[..., :C], ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)


def test_explicit_scale(cuda_ok):
    B, T, H, W, heads, hd, window, shift = 1, 2, 12, 24, 2, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    bits, dev = make_qkv(B, T, H, W, C, base=30)
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift, scale=0.3)
    o = torch.empty((B, T, H, W, C), dtype=torch.float32, device="cuda")
    s3w.swin3d_window_attn_fwd(*dev, o, heads, hd, window, shift, scale=0.3)
    torch.cuda.synchronize()
    mx, rl2 = attn_errors(o.cpu().numpy(), ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)


def test_repeat_calls_identical(cuda_ok):
    """The kernel is deterministic: two calls give bit-identical outputs."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 18, 36, 4, 64, (2, 6, 12), (1, 3, 6)
    _, dev = make_qkv(B, T, H, W, heads * hd, base=40)
    o1 = torch.empty((B, T, H, W, heads * hd), dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(o1)
    s3w.swin3d_window_attn_fwd(*dev, o1, heads, hd, window, shift)
    s3w.swin3d_window_attn_fwd(*dev, o2, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


# Full-size workloads of the Aurora 0.25-degree encoder stages (sampled windows).
FULL = [
    ("stage1_shifted", 1, 4, 180, 360, 8, 64, (1, 3, 6)),
    ("stage1_unshifted", 1, 4, 180, 360, 8, 64, (0, 0, 0)),
    ("stage2_shifted", 1, 4, 90, 180, 16, 64, (1, 3, 6)),
    ("stage3_padded", 2, 4, 45, 90, 32, 64, (1, 3, 6)),
]


@pytest.mark.parametrize("case", FULL, ids=lambda c: c[0])
def test_full_size_sampled_windows(cuda_ok, case):
    name, B, T, H, W, heads, hd, shift = case
    window = (2, 6, 12)
    C = heads * hd
    bits, dev = make_qkv(B, T, H, W, C, base=50)
    o = torch.full((B, T, H, W, C), SENTINEL, dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_window_attn_fwd(*dev, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    ids = edge_window_ids(B, T, H, W, window, extra_random=12)
    out, tok, _ = oracle.window_attn(*bits, heads, hd, window, shift, window_ids=ids)
    flat = o.view(-1, C)
    real = tok >= 0
    got = flat[torch.from_numpy(tok[real]).cuda()].float().cpu().numpy()
    mx, rl2 = attn_errors(got, out[real])
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
    # properties that hold at any size: every real token written, values finite and bounded
    # by the extreme V values of the sample (an attention output is a convex combination)
    assert not torch.any(o == SENTINEL)
    assert torch.isfinite(o).all()
    vmax = dev[2].float().abs().amax()
    assert float(o.float().abs().amax()) <= float(vmax) * (1 + 2 ** -7)


def test_bounded_wait_timeout_is_reported_and_context_survives(cuda_ok):
    """With the stall injection on, the kernel's first wait is on a barrier nothing signals
    and expires after the (short) limit: the call must unwind, report
    S3W_ERR_DEVICE_TIMEOUT through the error word, and leave the context usable for a
    normal call right after."""
    B, T, H, W, heads, hd, window, shift = 1, 4, 36, 72, 8, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    bits, dev = make_qkv(B, T, H, W, C, base=60)
    o = torch.zeros((B, T, H, W, C), dtype=torch.bfloat16, device="cuda")
    assert s3w.poll_device_error() == 0
    prev = s3w.set_wait_limit_ns(1_000_000)
    prev_stall = s3w.set_test_stall(True)
    try:
        s3w.swin3d_window_attn_fwd(*dev, o, heads, hd, window, shift)
        status = s3w.poll_device_error()
    finally:
        s3w.set_test_stall(prev_stall)
        s3w.set_wait_limit_ns(prev)
    assert status == 5
    assert s3w.poll_device_error() == 0          # the word was cleared by the poll
    s3w.swin3d_window_attn_fwd(*dev, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    ref = oracle.window_attn_grid(*bits, heads, hd, window, shift)
    mx, rl2 = attn_errors(o.float().cpu().numpy(), ref)
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
