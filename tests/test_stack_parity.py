"""The six-block encoder stack at full size: B=4, 4 x 180 x 360, 8 heads x 64; block k runs
attention on fresh seeded Q/K/V with the shift alternating (0,0,0), (1,3,6), ..., then AdaLN
(fp32 out) on its output into the fp32 residual stream, which chains through the six blocks.
Checked on sampled windows: each block's attention against the oracle; each block's AdaLN
at max-abs 1e-5 against the oracle's AdaLN fed the GPU's own bf16 attention output and the
GPU's residual before the block (so the AdaLN bar is the FP32 one, independent of the
attention error); and the residual stream at the sampled tokens against the oracle's own
chain (attention -> AdaLN, six times).

Tolerance of the chained residual: each block adds y (1 + scale) + shift, y the normalised
attention output.  The attention output carries the attention tolerance (max-abs 1e-2 at
most; rel-L2 ~1.3e-3 measured); normalising divides by its standard deviation (~0.2) and
|1 + scale| ~ N(1, 1) multiplies, so one block can move the residual by ~0.05 at the worst
element, six blocks by ~0.15, on a residual whose scale grows to ~3-4: max-abs 0.25 and a
relative L2 of 3e-3 bound it with margin while a wrong step (a dropped term, a wrong shift,
an off-by-one window) is orders of magnitude larger."""
import numpy as np
import pytest
import torch

import oracle
import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import inputs

from .helpers import ADALN_F32_MAX_ABS, ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, edge_window_ids, window_geometry

pytestmark = pytest.mark.gpu

B, T, H, W, HEADS, HD = 4, 4, 180, 360, 8, 64
C = HEADS * HD
L = T * H * W
WINDOW = (2, 6, 12)
SHIFTS = [(0, 0, 0), (1, 3, 6)] * 3
STACK_MAX_ABS = 0.25
STACK_REL_L2 = 3e-3


def windows_of_tokens(toks, shift):
    """Window ids (flat over samples) holding the given flat grid tokens under `shift`:
    the token's coordinate moved by -shift modulo the padded extent, divided by the window."""
    P, n = window_geometry(T, H, W, WINDOW)
    b, rem = np.divmod(toks, L)
    t, rem = np.divmod(rem, H * W)
    h, w = np.divmod(rem, W)
    idx = [((c - s) % p) // wa for c, s, p, wa in zip((t, h, w), shift, P, WINDOW)]
    return np.unique(b * (n[0] * n[1] * n[2]) + (idx[0] * n[1] + idx[1]) * n[2] + idx[2])


def test_encoder_stack_six_blocks_sampled(cuda_ok):
    dev = "cuda"
    res = inputs.normal_f32_torch(B * L * C, dev, tensor_index=600).reshape(B, L, C)
    o = torch.empty((B, T, H, W, C), dtype=torch.bfloat16, device=dev)
    # sampled tokens: those of block 0's edge and random windows
    ids0 = edge_window_ids(B, T, H, W, WINDOW, extra_random=6, seed=5)
    toks = None
    ref_res = None
    for k, shift in enumerate(SHIFTS):
        q, kk, v = (inputs.normal_bf16_torch((B, T, H, W, C), dev, tensor_index=610 + 10 * k + j) for j in range(3))
        scale = inputs.normal_f32_torch(B * C, dev, tensor_index=690 + 2 * k).reshape(B, C)
        shift_v = inputs.normal_f32_torch(B * C, dev, tensor_index=691 + 2 * k).reshape(B, C)
        if k == 0:
            res_host0 = res.cpu().numpy()
        s3w.swin3d_window_attn_fwd(q, kk, v, o, HEADS, HD, WINDOW, shift)
        torch.cuda.synchronize()
        if toks is not None:
            toks_d = torch.from_numpy(toks).to(dev)
            res_before = res.view(B * L, C)[toks_d].cpu().numpy()
            x_gpu = inputs.torch_bf16_to_bits(o.view(B * L, C)[toks_d])
        s3w.adaln_residual_fwd(o.view(B, L, C), res, scale, shift_v, res, eps=1e-5)
        torch.cuda.synchronize()
        assert s3w.poll_device_error() == 0
        qb, kb, vb = (inputs.torch_bf16_to_bits(t) for t in (q, kk, v))
        if toks is None:
            _, tok0, _ = oracle.window_attn(qb, kb, vb, HEADS, HD, WINDOW, shift, window_ids=ids0)
            toks = np.unique(tok0[tok0 >= 0])
            ref_res = res_host0.reshape(B * L, C)[toks].astype(np.float64)
        if k == 0:
            toks_d = torch.from_numpy(toks).to(dev)
            res_before = res_host0.reshape(B * L, C)[toks]
            x_gpu = inputs.torch_bf16_to_bits(o.view(B * L, C)[toks_d])
        # this block's AdaLN on the GPU's own attention output and residual: the FP32 bar
        sc_h, sh_h = scale.cpu().numpy(), shift_v.cpu().numpy()
        samp = toks // L
        res_after = res.view(B * L, C)[toks_d].cpu().numpy()
        for b in np.unique(samp):
            sel = samp == b
            want = oracle.adaln(x_gpu[sel][None], res_before[sel][None], sc_h[b:b + 1], sh_h[b:b + 1])[0]
            err = float(np.abs(res_after[sel] - want).max())
            assert err <= ADALN_F32_MAX_ABS, (k, int(b), err)
        ids = windows_of_tokens(toks, shift)
        out, tok, _ = oracle.window_attn(qb, kb, vb, HEADS, HD, WINDOW, shift, window_ids=ids)
        real = tok >= 0
        # this block's attention at every real token of the windows evaluated
        got = o.view(-1, C)[torch.from_numpy(tok[real]).to(dev)].float().cpu().numpy()
        mx, rl2 = attn_errors(got, out[real])
        assert mx <= ATTN_MAX_ABS and rl2 <= ATTN_REL_L2, (k, mx, rl2)
        # the oracle's chain at the sampled tokens: AdaLN of the oracle's attention output
        att = dict(zip(tok[real].tolist(), out[real]))
        x = np.stack([att[int(t)] for t in toks])
        new = np.empty_like(ref_res)
        for b in np.unique(samp):
            sel = samp == b
            # the residual stream is stored in fp32 on both sides
            new[sel] = oracle.adaln(x[sel][None], ref_res[sel][None].astype(np.float32), sc_h[b:b + 1],
                                    sh_h[b:b + 1])[0]
        ref_res = new
        del q, kk, v
    got_res = res.view(B * L, C)[torch.from_numpy(toks).to(dev)].cpu().numpy()
    mx, rl2 = attn_errors(got_res, ref_res)
    assert mx <= STACK_MAX_ABS and rl2 <= STACK_REL_L2, (mx, rl2)
