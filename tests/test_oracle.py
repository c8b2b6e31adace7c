"""Pins of the fp64 CPU oracle against things other than itself (CPU only).

* a brute-force dense masked attention whose mask is built in the forward direction
  (original coordinate -> shifted window, wrap-strip membership);
* an independent PyTorch fp64 route: pad, roll, partition, Swin slice labels,
  scaled_dot_product_attention, reverse;
* closed forms: hand-derived region-group sizes (tests/golden), constant V, Q = 0;
* invariants: softmax rows sum to 1, exactly-once merge, shift 0 equal to plain
  block attention, the -100 additive bias equal to exclusion;
* AdaLN against torch.nn.functional.layer_norm in fp64 and two closed forms.
"""
import itertools
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from swin3d_window_attention_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "region_group_sizes.txt")


def bf16_grid(B, T, H, W, C, base, ts=None):
    return inputs.attention_qkv_bits(B, T, H, W, C, base_index=base, token_stride=ts)


def torch_route(q, k, v, heads, hd, window, shift, scale, additive=False):
    """Swin-style reference built from PyTorch fp64 ops (pad -> roll -> partition -> SDPA
    -> reverse).  Labels are Swin's three slices per axis on the shifted, padded grid."""
    B, T, H, W, _ = q.shape
    C = heads * hd
    wt, wh, ww = window
    P = oracle.padded_dims(T, H, W, window)
    n = [P[a] // window[a] for a in range(3)]
    N = wt * wh * ww

    def to_windows(x, feat):
        x = F.pad(x, (0, 0, 0, P[2] - W, 0, P[1] - H, 0, P[0] - T))
        x = torch.roll(x, shifts=tuple(-s for s in shift), dims=(1, 2, 3))
        x = x.reshape(B, n[0], wt, n[1], wh, n[2], ww, feat)
        return x.permute(0, 1, 3, 5, 2, 4, 6, 7).reshape(B * n[0] * n[1] * n[2], N, feat)

    def heads_first(x):
        return x.reshape(x.shape[0], N, heads, hd).permute(0, 2, 1, 3)

    qt, kt, vt = (torch.from_numpy(np.asarray(a[..., :C], dtype=np.float64)) for a in (q, k, v))
    qw, kw, vw = (heads_first(to_windows(a, C)) for a in (qt, kt, vt))
    real = to_windows(torch.ones(B, T, H, W, 1, dtype=torch.float64), 1)[..., 0] > 0.5  # [BW, N]

    lab = torch.zeros(P, dtype=torch.long)
    for a in range(3):
        if shift[a] == 0:
            continue
        sl = [slice(0, -window[a]), slice(-window[a], -shift[a]), slice(-shift[a], None)]
        for r, s in enumerate(sl):
            idx = [slice(None)] * 3
            idx[a] = s
            lab[tuple(idx)] += r * (3 ** (2 - a))
    labw = lab.reshape(n[0], wt, n[1], wh, n[2], ww).permute(0, 2, 4, 1, 3, 5).reshape(-1, N)
    labw = labw.repeat(B, 1)
    same = labw[:, :, None] == labw[:, None, :]
    if additive:
        mask = torch.where(same, 0.0, -100.0).to(torch.float64)
        mask = mask.masked_fill(~real[:, None, :], float("-inf"))
    else:
        mask = same & real[:, None, :]
    o = F.scaled_dot_product_attention(qw, kw, vw, attn_mask=mask[:, None], scale=scale)
    o = o.permute(0, 2, 1, 3).reshape(B, n[0], n[1], n[2], wt, wh, ww, C)
    o = o.permute(0, 1, 4, 2, 5, 3, 6, 7).reshape(B, P[0], P[1], P[2], C)
    o = torch.roll(o, shifts=tuple(shift), dims=(1, 2, 3))
    return o[:, :T, :H, :W].numpy()


def widened(bits):
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


CASES = [
    # (B, T, H, W, heads, hd, window, shift)
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (1, 3, 6)),   # tiny workload, shifted
    (1, 2, 15, 30, 2, 32, (2, 6, 12), (0, 0, 0)),   # tiny workload, unshifted
    (2, 3, 5, 7, 2, 8, (2, 3, 4), (1, 1, 2)),       # pad != shift on every axis
    (1, 4, 6, 8, 1, 4, (2, 3, 4), (1, 2, 3)),       # no padding, shift != w/2
    (1, 5, 4, 9, 3, 4, (2, 2, 4), (1, 1, 1)),
    (1, 1, 1, 1, 1, 8, (2, 6, 12), (1, 3, 6)),      # one real token
]


@pytest.mark.parametrize("case", CASES)
def test_window_attn_matches_dense_bruteforce(case):
    B, T, H, W, heads, hd, window, shift = case
    q, k, v = bf16_grid(B, T, H, W, heads * hd, 100)
    got = oracle.window_attn_grid(q, k, v, heads, hd, window, shift)
    ref = oracle.dense_masked_attn(q, k, v, heads, hd, window, shift)
    assert not np.isnan(got).any()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", CASES)
def test_window_attn_matches_torch_route(case):
    B, T, H, W, heads, hd, window, shift = case
    q, k, v = bf16_grid(B, T, H, W, heads * hd, 200)
    scale = 1.0 / np.sqrt(hd)
    got = oracle.window_attn_grid(q, k, v, heads, hd, window, shift)
    ref = torch_route(widened(q), widened(k), widened(v), heads, hd, window, shift, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    dense = oracle.dense_masked_attn(q, k, v, heads, hd, window, shift)
    np.testing.assert_allclose(dense, ref, rtol=0, atol=1e-12)


def test_additive_minus100_equals_exclusion():
    B, T, H, W, heads, hd, window, shift = CASES[0]
    q, k, v = bf16_grid(B, T, H, W, heads * hd, 300)
    scale = 1.0 / np.sqrt(hd)
    hard = oracle.window_attn_grid(q, k, v, heads, hd, window, shift, mask_mode=0)
    soft = oracle.window_attn_grid(q, k, v, heads, hd, window, shift, mask_mode=1)
    ref = torch_route(widened(q), widened(k), widened(v), heads, hd, window, shift, scale, additive=True)
    np.testing.assert_allclose(soft, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(hard, soft, rtol=0, atol=1e-30)


def test_token_stride_and_extra_channels_ignored():
    B, T, H, W, heads, hd, window, shift = CASES[2]
    C = heads * hd
    q, k, v = bf16_grid(B, T, H, W, C, 400, ts=C + 8)
    got = oracle.window_attn_grid(q, k, v, heads, hd, window, shift)
    ref = oracle.window_attn_grid(*(np.ascontiguousarray(a[..., :C]) for a in (q, k, v)), heads, hd, window, shift)
    np.testing.assert_array_equal(got, ref)


def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            name = parts[0]
            T, H, W, st, sh, sw, it, ih, iw = (int(x) for x in parts[1:10])
            expect = {}
            for tok in parts[10:]:
                size, count = tok.split(":")
                expect[int(size)] = int(count)
            rows.append((name, (T, H, W), (st, sh, sw), (it, ih, iw), expect))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: f"{r[0]}-{r[2]}-{r[3]}")
def test_region_group_sizes_golden(row):
    """Q = 0 makes every allowed logit 0, so each real query spreads weight 1/|group|
    uniformly over its group: the group sizes must equal the hand-derived ones."""
    name, (T, H, W), shift, (it, ih, iw), expect = row
    window = (2, 6, 12)
    P = oracle.padded_dims(T, H, W, window)
    n = [P[a] // window[a] for a in range(3)]
    wid = (it * n[1] + ih) * n[2] + iw
    shape = (1, T, H, W, 4)
    q = np.zeros(shape, dtype=np.float64)
    k = inputs.normal_f32_tensor(shape, tensor_index=7).astype(np.float64)
    v = inputs.normal_f32_tensor(shape, tensor_index=8).astype(np.float64)
    out, tok, probs = oracle.window_attn(q, k, v, 1, 4, window, shift, window_ids=[wid], return_probs=True)
    real = tok[0] >= 0
    p = probs[0, 0][real]                      # [n_real, N]
    sizes = (p > 0).sum(axis=1)
    got = {int(s): int(c) for s, c in zip(*np.unique(sizes, return_counts=True))}
    assert got == expect
    # uniform weights 1/|group|, and the output is the plain mean of V over the group
    for i, row_p in enumerate(p):
        nz = row_p[row_p > 0]
        np.testing.assert_allclose(nz, 1.0 / sizes[i], rtol=0, atol=1e-15)
    vt = v.reshape(-1, 4)
    members = [np.nonzero(row_p > 0)[0] for row_p in p]
    for i, m in enumerate(members):
        np.testing.assert_allclose(out[0][real][i], vt[tok[0][m]].mean(axis=0), rtol=0, atol=1e-14)


@pytest.mark.parametrize("case", CASES[:4])
def test_softmax_rows_sum_to_one_and_masked_zero(case):
    B, T, H, W, heads, hd, window, shift = case
    q, k, v = bf16_grid(B, T, H, W, heads * hd, 500)
    out, tok, probs = oracle.window_attn(q, k, v, heads, hd, window, shift, return_probs=True)
    real = tok >= 0
    for w in range(tok.shape[0]):
        pr = probs[w][:, real[w]]                     # [heads, n_real_q, N]
        np.testing.assert_allclose(pr.sum(axis=-1), 1.0, rtol=0, atol=1e-13)
        assert (pr[:, :, ~real[w]] == 0).all()        # padded keys get no weight
        assert (pr >= 0).all()


@pytest.mark.parametrize("case", CASES)
def test_constant_v_returns_v(case):
    B, T, H, W, heads, hd, window, shift = case
    C = heads * hd
    q, k, _ = bf16_grid(B, T, H, W, C, 600)
    const = inputs.normal_f32(C, tensor_index=601).astype(np.float64)
    v = np.broadcast_to(const, (B, T, H, W, C)).copy()
    got = oracle.window_attn_grid(widened(q), widened(k), v, heads, hd, window, shift)
    np.testing.assert_allclose(got, np.broadcast_to(const, got.shape), rtol=0, atol=1e-13)


@pytest.mark.parametrize("case", CASES)
def test_every_real_token_written_once(case):
    B, T, H, W, heads, hd, window, shift = case
    q, k, v = bf16_grid(B, T, H, W, heads * hd, 700)
    out, tok, _ = oracle.window_attn(q, k, v, heads, hd, window, shift)
    grid, writes = oracle.merge_to_grid(out, tok, B, T, H, W)
    assert (writes == 1).all()
    assert np.isnan(out[tok < 0]).all()


def test_shift0_equals_block_attention():
    """No shift and no padding: the method is plain softmax attention inside each block."""
    B, T, H, W, heads, hd = 2, 4, 6, 8, 2, 8
    window = (2, 3, 4)
    q, k, v = (widened(a) for a in bf16_grid(B, T, H, W, heads * hd, 800))
    got = oracle.window_attn_grid(q, k, v, heads, hd, window, (0, 0, 0))
    scale = 1.0 / np.sqrt(hd)
    ref = np.empty_like(got)
    for b, t0, h0, w0 in itertools.product(range(B), range(0, T, 2), range(0, H, 3), range(0, W, 4)):
        sl = (b, slice(t0, t0 + 2), slice(h0, h0 + 3), slice(w0, w0 + 4))
        for h in range(heads):
            cs = slice(h * hd, (h + 1) * hd)
            Q = q[sl][..., cs].reshape(-1, hd)
            K = k[sl][..., cs].reshape(-1, hd)
            V = v[sl][..., cs].reshape(-1, hd)
            S = scale * Q @ K.T
            E = np.exp(S - S.max(axis=1, keepdims=True))
            A = E / E.sum(axis=1, keepdims=True)
            ref[sl + (cs,)] = (A @ V).reshape(2, 3, 4, hd)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_window_subset_matches_full():
    B, T, H, W, heads, hd, window, shift = CASES[2]
    q, k, v = bf16_grid(B, T, H, W, heads * hd, 900)
    full, tok_full, _ = oracle.window_attn(q, k, v, heads, hd, window, shift)
    ids = [5, 0, full.shape[0] - 1]
    sub, tok_sub, _ = oracle.window_attn(q, k, v, heads, hd, window, shift, window_ids=ids)
    np.testing.assert_array_equal(tok_sub, tok_full[ids])
    np.testing.assert_array_equal(np.nan_to_num(sub, nan=7.0), np.nan_to_num(full[ids], nan=7.0))


def test_oracle_rejects_bad_args():
    q = np.zeros((1, 2, 2, 2, 4), dtype=np.float64)
    with pytest.raises(ValueError):
        oracle.window_attn(q, q, q, 1, 4, (2, 2, 2), (2, 0, 0))   # shift == window
    with pytest.raises(ValueError):
        oracle.window_attn(q, q, q, 2, 4, (2, 2, 2), (0, 0, 0))   # heads*hd > token stride


# --------------------------------------------------------------------------- AdaLN
def _adaln_inputs(B, L, C, x_bf16=True, base=1000, sig_film=0.1):
    if x_bf16:
        x = inputs.normal_bf16_bits((B, L, C), tensor_index=base)
    else:
        x = inputs.normal_f32_tensor((B, L, C), tensor_index=base)
    res = inputs.normal_f32_tensor((B, L, C), tensor_index=base + 1)
    sc = inputs.normal_f32_tensor((B, C), tensor_index=base + 2, sigma=sig_film)
    sh = inputs.normal_f32_tensor((B, C), tensor_index=base + 3, sigma=sig_film)
    return x, res, sc, sh


@pytest.mark.parametrize("x_bf16", [True, False])
def test_adaln_matches_torch_layer_norm(x_bf16):
    B, L, C = 2, 37, 96
    x, res, sc, sh = _adaln_inputs(B, L, C, x_bf16)
    got = oracle.adaln(x, res, sc, sh, eps=1e-5)
    xd = torch.from_numpy(widened(x) if x_bf16 else x.astype(np.float64))
    ln = F.layer_norm(xd, (C,), eps=1e-5).numpy()
    ref = res.astype(np.float64) + ln * (1.0 + sc[:, None, :].astype(np.float64)) + sh[:, None, :]
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # the alternative FiLM form multiplies by scale alone
    got1 = oracle.adaln(x, res, sc, sh, eps=1e-5, film_form=1)
    ref1 = res.astype(np.float64) + ln * sc[:, None, :].astype(np.float64) + sh[:, None, :]
    np.testing.assert_allclose(got1, ref1, rtol=0, atol=1e-12)


def test_adaln_constant_row_gives_residual_plus_shift():
    B, L, C = 1, 5, 64
    _, res, sc, sh = _adaln_inputs(B, L, C)
    x = np.full((B, L, C), 3.25, dtype=np.float32)
    got = oracle.adaln(x, res, sc, sh)
    np.testing.assert_allclose(got, res + sh[:, None, :].astype(np.float64), rtol=0, atol=1e-14)


def test_adaln_zero_film_closed_form():
    """scale = shift = residual = 0: each output row has mean 0 and variance var/(var+eps)."""
    B, L, C = 1, 16, 128
    x = inputs.normal_f32_tensor((B, L, C), tensor_index=1100, sigma=0.01).astype(np.float64)
    z = np.zeros((B, C), dtype=np.float32)
    eps = 1e-5
    got = oracle.adaln(x, None, z, z, eps=eps)
    var = x.var(axis=-1)
    np.testing.assert_allclose(got.mean(axis=-1), 0.0, atol=1e-14)
    np.testing.assert_allclose(got.var(axis=-1), var / (var + eps), rtol=1e-12)


# ---------------------------------------------------------------------------- QKV projection
def test_qkv_proj_permutation_weight_returns_permuted_channels():
    """w[n][c] = 1 iff c = perm(n): the output is x at the permuted channels.  A transposed
    weight (x w instead of x w^T) or swapped q/k/v thirds give other channels."""
    rng = np.random.default_rng(1)
    C = 8
    x = rng.standard_normal((5, C))
    perm = rng.integers(0, C, size=3 * C)
    w = np.zeros((3 * C, C))
    w[np.arange(3 * C), perm] = 1.0
    y = oracle.qkv_proj(x, w)
    assert y.shape == (5, 3 * C)
    np.testing.assert_array_equal(y, x[:, perm])


def test_qkv_proj_zero_input_gives_bias_and_is_additive():
    rng = np.random.default_rng(2)
    C = 16
    w = rng.standard_normal((3 * C, C))
    b = rng.standard_normal(3 * C)
    np.testing.assert_array_equal(oracle.qkv_proj(np.zeros((4, C)), w, b), np.broadcast_to(b, (4, 3 * C)))
    x1, x2 = rng.standard_normal((6, C)), rng.standard_normal((6, C))
    lhs = oracle.qkv_proj(x1 + x2, w, b)
    rhs = oracle.qkv_proj(x1, w, b) + oracle.qkv_proj(x2, w, b) - b
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_qkv_proj_thirds_are_the_q_k_v_projections_and_bf16_bits_widen_exactly():
    """The three thirds of the output are the projections by the three row blocks of w (grid
    shape kept), and bf16 bit patterns enter as their exact values."""
    from swin3d_window_attention_b200 import inputs

    C = 32
    xb = inputs.normal_bf16_bits((2, 3, 4, C), tensor_index=91)
    wb = inputs.normal_bf16_bits((3 * C, C), tensor_index=92)
    y = oracle.qkv_proj(xb, wb)
    assert y.shape == (2, 3, 4, 3 * C)
    xf, wf = inputs.bf16_bits_to_f32(xb).astype(np.float64), inputs.bf16_bits_to_f32(wb).astype(np.float64)
    for j in range(3):
        part = oracle.qkv_proj(xf, np.concatenate([wf[j * C:(j + 1) * C]] * 3))[..., :C]
        np.testing.assert_allclose(y[..., j * C:(j + 1) * C], part, rtol=0, atol=1e-12)
