"""GPU parity of the QKV projection (swin3d_qkv_proj_fwd) and of the projection followed by the
window attention on its output (swin3d_qkv_window_attn_fwd), through the C ABI, against the
fp64 oracle.

Projection bar: bf16 output of an fp32-accumulated product; the oracle's value in fp64.  The
output rounding is at most half a bf16 ulp (2^-9 relative) and the fp32 accumulation over
C <= 512 terms of size ~1/sqrt(C) adds well under 1e-5, so |gpu - oracle| <= 2^-8 |oracle| +
1e-5 element-wise.
Chained bar: the attention bar of the BF16 path (max-abs 1e-2, relative L2 3e-3), comparing
the GPU's attention on its own projection with the oracle's attention on the oracle's
projection rounded to bf16 (q, k, v that differ by at most one bf16 ulp in rare elements).
"""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, edge_window_ids

pytestmark = pytest.mark.gpu


def make(shape, C, base, bias=True):
    """x ~ N(0,1), w ~ N(0, 1/C) (a Linear weight's scale), b ~ N(0, 0.1): bf16 / fp32 tensors."""
    x = inputs.normal_bf16_torch(tuple(shape) + (C,), "cuda", tensor_index=base)
    w = inputs.normal_bf16_torch((3 * C, C), "cuda", tensor_index=base + 1, sigma=C ** -0.5)
    b = inputs.normal_f32_torch(3 * C, "cuda", tensor_index=base + 2, sigma=0.1) if bias else None
    return x, w, b


def check_proj(x, w, b, qkv_gpu, rows=None):
    xb = inputs.torch_bf16_to_bits(x.reshape(-1, x.shape[-1]) if rows is None else x.reshape(-1, x.shape[-1])[rows])
    ref = oracle.qkv_proj(xb, inputs.torch_bf16_to_bits(w), None if b is None else b.cpu().numpy())
    got = qkv_gpu.reshape(-1, 3 * x.shape[-1])
    got = (got if rows is None else got[rows]).float().cpu().numpy().astype(np.float64)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) - bound))
    return ref


@pytest.mark.parametrize("tokens,C,bias", [(900, 64, True), (1000, 96, False), (4 * 36 * 72, 512, True),
                                           (129, 1024, True)],
                         ids=["tiny_C64_Ntail", "C96_Ktail_nobias", "C512", "C1024_Mtail"])
def test_qkv_proj_small(cuda_ok, tokens, C, bias):
    x, w, b = make((tokens,), C, 7000, bias)
    qkv = torch.full((tokens, 3 * C), 777.0, dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_qkv_proj_fwd(x, w, b, qkv)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    check_proj(x, w, b, qkv)


def test_qkv_proj_stage1_sampled_rows(cuda_ok):
    """Stage-1 width on the whole grid (259,200 tokens x 512 -> 1536): sampled rows (first,
    last, every tile boundary region and random) against the oracle; the rest finite."""
    shape, C = (1, 4, 180, 360), 512
    x, w, b = make(shape, C, 7100)
    qkv = torch.empty(shape + (3 * C,), dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_qkv_proj_fwd(x, w, b, qkv)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    L = int(np.prod(shape))
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 129, L - 1], rng.integers(0, L, 300)]))
    check_proj(x, w, b, qkv, rows=torch.from_numpy(rows).cuda())
    assert torch.isfinite(qkv.float()).all()


@pytest.mark.parametrize("grid,heads,hd,window,shift", [
    ((1, 2, 15, 30), 2, 32, (2, 6, 12), (1, 3, 6)),     # the tiny workload
    ((2, 4, 13, 29), 3, 64, (2, 6, 12), (1, 3, 6)),     # ragged, pad != shift, C = 192
    ((1, 4, 24, 48), 2, 64, (2, 12, 12), (1, 6, 6)),    # N = 288: the streaming path
], ids=["tiny", "ragged_C192", "stream_N288"])
def test_qkv_window_attn_matches_oracle_chain(cuda_ok, grid, heads, hd, window, shift):
    C = heads * hd
    x, w, b = make(grid, C, 7200)
    qkv = torch.empty(grid + (3 * C,), dtype=torch.bfloat16, device="cuda")
    o = torch.empty(grid + (C,), dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_qkv_window_attn_fwd(x, w, b, qkv, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    ref_qkv = check_proj(x, w, b, qkv).reshape(grid + (3 * C,))
    bits = inputs.f32_to_bf16_bits(ref_qkv.astype(np.float32))
    q, k, v = bits[..., :C], bits[..., C:2 * C], bits[..., 2 * C:]
    ref = oracle.window_attn_grid(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v), heads, hd,
                                  window, shift)
    mx, rl2 = attn_errors(o.float().cpu().numpy(), ref)
    print(f"qkv+attn {grid} {window}: max-abs {mx:.3e} rel-L2 {rl2:.3e}")
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
    # the attention part equals the attention call on the projection's slices
    o2 = torch.empty_like(o)
    s3w.swin3d_window_attn_fwd(qkv[..., :C], qkv[..., C:2 * C], qkv[..., 2 * C:], o2, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)


def test_qkv_window_attn_stage1_sampled(cuda_ok):
    """Stage 1 (B=1, 4x180x360, 8 x 64), shifted: sampled windows of the chain against the oracle
    chain (projection of the windows' tokens only)."""
    grid, heads, hd, window, shift = (1, 4, 180, 360), 8, 64, (2, 6, 12), (1, 3, 6)
    C = heads * hd
    x, w, b = make(grid, C, 7300)
    qkv = torch.empty(grid + (3 * C,), dtype=torch.bfloat16, device="cuda")
    o = torch.empty(grid + (C,), dtype=torch.bfloat16, device="cuda")
    s3w.swin3d_qkv_window_attn_fwd(x, w, b, qkv, o, heads, hd, window, shift)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    # the oracle attention of the sampled windows, on the GPU's projection (pinned above)
    ids = edge_window_ids(*grid, window, extra_random=6)
    qb = inputs.torch_bf16_to_bits(qkv)
    out, tok, _ = oracle.window_attn(np.ascontiguousarray(qb[..., :C]), np.ascontiguousarray(qb[..., C:2 * C]),
                                     np.ascontiguousarray(qb[..., 2 * C:]), heads, hd, window, shift, window_ids=ids)
    real = tok >= 0
    got = o.view(-1, C)[torch.from_numpy(tok[real]).cuda()].float().cpu().numpy()
    mx, rl2 = attn_errors(got, out[real])
    assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (mx, rl2)
    # and the projection at those windows' tokens against the oracle
    check_proj(x, w, b, qkv, rows=torch.from_numpy(np.unique(tok[real])).cuda())


def test_qkv_rejections(cuda_ok):
    C = 48   # not a multiple of 32
    x = torch.zeros((10, C), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((3 * C, C), dtype=torch.bfloat16, device="cuda")
    qkv = torch.zeros((10, 3 * C), dtype=torch.bfloat16, device="cuda")
    assert s3w.swin3d_qkv_proj_fwd(x, w, None, qkv, check=False) == 2
    C = 64
    x = torch.zeros((10, C), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((3 * C, C), dtype=torch.bfloat16, device="cuda")
    big = torch.zeros(10 * 3 * C + 16, dtype=torch.bfloat16, device="cuda")
    lib = s3w.load_library()
    st = torch.cuda.current_stream().cuda_stream
    assert lib.swin3d_qkv_proj_fwd(x.data_ptr(), w.data_ptr(), None, big.data_ptr() + 16, 10, C, st) == 3   # qkv not 32-B aligned
    assert lib.swin3d_qkv_proj_fwd(x.data_ptr(), w.data_ptr(), None, x.data_ptr(), 10, C, st) == 1          # qkv over x


def test_qkv_proj_bounded_wait_timeout(cuda_ok):
    x, w, b = make((2000,), 256, 7400)
    qkv = torch.empty((2000, 768), dtype=torch.bfloat16, device="cuda")
    assert s3w.poll_device_error() == 0
    prev = s3w.set_wait_limit_ns(1_000_000)
    prev_stall = s3w.set_test_stall(True)
    try:
        s3w.swin3d_qkv_proj_fwd(x, w, b, qkv)
        status = s3w.poll_device_error()
    finally:
        s3w.set_test_stall(prev_stall)
        s3w.set_wait_limit_ns(prev)
    assert status == 5
    s3w.swin3d_qkv_proj_fwd(x, w, b, qkv)
    torch.cuda.synchronize()
    assert s3w.poll_device_error() == 0
    check_proj(x, w, b, qkv)
