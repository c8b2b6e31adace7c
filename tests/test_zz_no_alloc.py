"""GPU test of swin3d_window_attn_adaln_fwd_static_ws, the fused attention + AdaLN call on the
library's static workspace (allocates nothing).

Two calls in a row through the C ABI, on different inputs and shifts, each checked against
swin3d_window_attn_adaln_fwd (caller-supplied workspace) on the same inputs: the AdaLN output
within the fused path's tolerance (max-abs 1e-5; the two calls run the same kernel, so the
outputs are in fact identical) and the optional attention output bit for bit.  Collected last
so that it runs both alone in a fresh process and after every other test.
"""
import pytest
import torch

import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs
from swin3d_window_attention_b200.api import S3W_ERR_UNSUPPORTED, load_library
from tests.helpers import ADALN_F32_MAX_ABS

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 48 << 20


def make(B, T, H, W, heads, hd, base):
    C, L = heads * hd, T * H * W
    q, k, v = (inputs.normal_bf16_torch((B, T, H, W, C), "cuda", tensor_index=base + j) for j in range(3))
    sc = inputs.normal_f32_torch(B * C, "cuda", tensor_index=base + 3, sigma=0.1).reshape(B, C)
    sh = inputs.normal_f32_torch(B * C, "cuda", tensor_index=base + 4, sigma=0.1).reshape(B, C)
    res = inputs.normal_f32_torch(B * L * C, "cuda", tensor_index=base + 5).reshape(B, L, C)
    return q, k, v, sc, sh, res


@pytest.mark.parametrize("grid", [(1, 4, 36, 72, 8, 64), (1, 4, 180, 360, 8, 64), (2, 4, 13, 29, 3, 64)],
                         ids=["B1_4x36x72_8x64", "stage1_B1_4x180x360_8x64", "B2_4x13x29_3x64"])
def test_static_workspace_call_matches_fused_call_twice(cuda_ok, grid):
    B, T, H, W, heads, hd = grid
    window = (2, 6, 12)
    need = s3w.window_attn_adaln_workspace_bytes(B, T, H, W, heads, hd, window)
    assert need <= STATIC_WS_BYTES
    for call, shift in enumerate([(0, 0, 0), (1, 3, 6)]):
        q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=5000 + 10 * call)
        o_ref, o_st = torch.empty_like(q), torch.empty_like(q)
        out_ref, out_st = torch.empty_like(res), torch.empty_like(res)
        s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, sc, sh, out_ref, heads, hd, window, shift, o=o_ref, eps=1e-5)
        s3w.swin3d_window_attn_adaln_fwd_static_ws(q, k, v, res, sc, sh, out_st, heads, hd, window, shift, o=o_st,
                                                   eps=1e-5)
        torch.cuda.synchronize()
        assert s3w.poll_device_error() == 0
        assert torch.equal(o_st, o_ref), call
        d = float((out_st - out_ref).abs().max())
        assert d <= ADALN_F32_MAX_ABS, (call, d)


def test_static_workspace_rejects_a_grid_beyond_its_size(cuda_ok):
    """Stage 2 (C = 1024, 450 windows): one CTA per SM needs 2 x 144 x 1024 bf16 each, more
    than 48 MiB on a GPU with more than 85 SMs; the call is refused before any launch."""
    B, T, H, W, heads, hd = 1, 4, 90, 180, 16, 64
    need = s3w.window_attn_adaln_workspace_bytes(B, T, H, W, heads, hd, (2, 6, 12))
    if need <= STATIC_WS_BYTES:
        pytest.skip(f"this GPU's grid needs only {need} bytes")
    q, k, v, sc, sh, res = make(B, T, H, W, heads, hd, base=5100)
    out = torch.full_like(res, 7.0)
    rc = s3w.swin3d_window_attn_adaln_fwd_static_ws(q, k, v, res, sc, sh, out, heads, hd, (2, 6, 12), (1, 3, 6),
                                                    check=False)
    torch.cuda.synchronize()
    assert rc == S3W_ERR_UNSUPPORTED
    assert bool((out == 7.0).all())
    assert "unsupported" in load_library().s3w_status_string(rc).decode()
