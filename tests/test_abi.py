"""C-ABI checks that need no GPU: the library loads, exports every declared entry point,
and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import swin3d_window_attention_b200 as s3w
from swin3d_window_attention_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # 16-byte aligned dummy address; only used with arguments that are rejected first
FAKE_QKV = 0x40000000   # a second dummy region, far from FAKE


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = s3w.load_library()
    names = declared_functions()
    assert {"swin3d_window_attn_fwd", "adaln_residual_fwd", "s3w_status_string", "s3w_poll_device_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings():
    assert s3w.status_string(0) == "ok"
    for code in range(1, 6):
        assert s3w.status_string(code) not in ("ok", "unknown status")
    assert s3w.status_string(99) == "unknown status"
    assert s3w.load_library().s3w_version() >= 100


def _attn(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, T=4, H=12, W=24, wt=2, wh=6, ww=12, st=1, sh=3, sw=6,
             heads=8, hd=64, qs=512, os_=512, scale=0.0, ind=0, outd=0, stream=None)
    a.update(over)
    return s3w.load_library().swin3d_window_attn_fwd(
        a["q"], a["k"], a["v"], a["o"], a["B"], a["T"], a["H"], a["W"], a["wt"], a["wh"], a["ww"], a["st"],
        a["sh"], a["sw"], a["heads"], a["hd"], a["qs"], a["os_"], a["scale"], a["ind"], a["outd"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(q=None), api.S3W_ERR_INVALID_ARG),
    (dict(o=None), api.S3W_ERR_INVALID_ARG),
    (dict(B=0), api.S3W_ERR_INVALID_ARG),
    (dict(T=-1), api.S3W_ERR_INVALID_ARG),
    (dict(st=2), api.S3W_ERR_INVALID_ARG),          # shift == window
    (dict(sw=-1), api.S3W_ERR_INVALID_ARG),
    (dict(wh=0), api.S3W_ERR_INVALID_ARG),
    (dict(qs=100), api.S3W_ERR_INVALID_ARG),        # token stride < heads * head_dim
    (dict(os_=511), api.S3W_ERR_INVALID_ARG),
    (dict(outd=7), api.S3W_ERR_INVALID_ARG),
    (dict(scale=float("nan")), api.S3W_ERR_INVALID_ARG),
    (dict(ww=130, sw=6), api.S3W_ERR_UNSUPPORTED),  # N > 144 with win_w > 128: no streaming blocks of whole rows
    (dict(wh=300, ww=120, sh=3, sw=6), api.S3W_ERR_UNSUPPORTED),   # N = 72,000 > 65,536
    (dict(wt=70000, st=1), api.S3W_ERR_UNSUPPORTED),                # a window extent above 65,536
    (dict(ww=13, sw=6, ind=1, qs=512, os_=512), api.S3W_ERR_UNSUPPORTED),   # N = 156: streaming is BF16 only
    (dict(hd=48, qs=384, os_=384), api.S3W_ERR_UNSUPPORTED),
    (dict(ind=1, qs=514), api.S3W_ERR_MISALIGNED),  # fp32 token rows not on 16-byte boundaries
    (dict(q=FAKE + 8), api.S3W_ERR_MISALIGNED),
    (dict(o=FAKE + 2), api.S3W_ERR_MISALIGNED),
    (dict(qs=516), api.S3W_ERR_MISALIGNED),         # token rows not on 16-byte boundaries
    # o overlapping q, k, v (1,152 tokens x 512 channels x 2 bytes = 1,179,648 bytes each)
    (dict(), api.S3W_ERR_INVALID_ARG),                                  # o == q == k == v
    (dict(o=FAKE + 1179648 - 1024), api.S3W_ERR_INVALID_ARG),           # o starts inside the last row
    (dict(o=FAKE - 1024), api.S3W_ERR_INVALID_ARG),                     # o ends inside the first rows
    (dict(q=FAKE_QKV, k=FAKE_QKV + 1024, v=FAKE_QKV + 2048, qs=1536, o=FAKE_QKV + 1536 * 2 * 1151 + 2048),
     api.S3W_ERR_INVALID_ARG),                                          # o on the last token row of v
])
def test_attn_rejects_bad_arguments_on_host(over, expect):
    assert _attn(**over) == expect


def test_legacy_baseline_is_bf16_only():
    lib = s3w.load_library()
    rc = lib.swin3d_window_attn_fwd_legacy_mma(FAKE, FAKE, FAKE, FAKE_QKV, 1, 4, 12, 24, 2, 6, 12, 1, 3, 6, 8, 64,
                                               512, 512, 0.0, api.S3W_F32, 0, None)
    assert rc == api.S3W_ERR_UNSUPPORTED


def _adaln(**over):
    a = dict(x=FAKE, xd=0, res=FAKE, sc=FAKE, sh=FAKE, out=FAKE, outd=1, B=1, L=16, C=512, eps=1e-5)
    a.update(over)
    return s3w.load_library().adaln_residual_fwd(a["x"], a["xd"], a["res"], a["sc"], a["sh"], a["out"], a["outd"],
                                                 a["B"], a["L"], a["C"], a["eps"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(x=None), api.S3W_ERR_INVALID_ARG),
    (dict(res=None), api.S3W_ERR_INVALID_ARG),
    (dict(B=0), api.S3W_ERR_INVALID_ARG),
    (dict(L=-1), api.S3W_ERR_INVALID_ARG),
    (dict(eps=-1.0), api.S3W_ERR_INVALID_ARG),
    (dict(xd=5), api.S3W_ERR_INVALID_ARG),
    (dict(C=12), api.S3W_ERR_UNSUPPORTED),
    (dict(C=8192), api.S3W_ERR_UNSUPPORTED),
    (dict(sc=FAKE + 4), api.S3W_ERR_MISALIGNED),
    (dict(out=FAKE + 16 * 512), api.S3W_ERR_INVALID_ARG),   # partial overlap with residual
    (dict(x=FAKE_QKV, sc=FAKE_QKV, sh=FAKE_QKV, res=FAKE_QKV + 8192, out=FAKE_QKV + 8192),
     api.S3W_ERR_INVALID_ARG),                               # out in place on residual, but over x
    (dict(x=FAKE_QKV, sc=FAKE + 4096, sh=FAKE_QKV + 65536, res=FAKE, out=FAKE, xd=1, L=4),
     api.S3W_ERR_INVALID_ARG),                               # out over scale (x, shift elsewhere)
    (dict(L=(2 ** 31 - 1) * 8 + 1), api.S3W_ERR_UNSUPPORTED),   # more row blocks than a grid holds
    (dict(B=4, L=2 ** 62), api.S3W_ERR_UNSUPPORTED),             # B * L * C would overflow int64
])
def test_adaln_rejects_bad_arguments_on_host(over, expect):
    # the overlap case keeps out != residual while the two ranges intersect
    if "out" in over and "res" not in over:
        over = dict(over, res=FAKE + 64)
    assert _adaln(**over) == expect


def test_adaln_zero_tokens_is_a_no_op():
    assert _adaln(L=0) == api.S3W_OK
    assert _adaln(L=0, x=None, res=None, out=None) == api.S3W_OK


def _fused(**over):
    # every default is valid except the workspace size, which is checked last (a call with these
    # defaults returns on the host on every machine)
    a = dict(q=FAKE_QKV, k=FAKE_QKV, v=FAKE_QKV, qs=512, res=FAKE, sc=FAKE, sh=FAKE, out=FAKE, outd=1, o=None,
             ws=FAKE, wsb=0, B=1, T=4, H=12, W=24, wt=2, wh=6, ww=12, st=1, sh_=3, sw=6, heads=8, hd=64, scale=0.0,
             eps=1e-5)
    a.update(over)
    return s3w.load_library().swin3d_window_attn_adaln_fwd(
        a["q"], a["k"], a["v"], a["qs"], a["res"], a["sc"], a["sh"], a["out"], a["outd"], a["o"], a["ws"], a["wsb"],
        a["B"], a["T"], a["H"], a["W"], a["wt"], a["wh"], a["ww"], a["st"], a["sh_"], a["sw"], a["heads"], a["hd"],
        a["scale"], a["eps"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(res=None), api.S3W_ERR_INVALID_ARG),
    (dict(ws=None), api.S3W_ERR_INVALID_ARG),
    (dict(q=None), api.S3W_ERR_INVALID_ARG),
    (dict(eps=-1.0), api.S3W_ERR_INVALID_ARG),
    (dict(outd=5), api.S3W_ERR_INVALID_ARG),
    (dict(st=2), api.S3W_ERR_INVALID_ARG),                  # shift == window
    (dict(hd=48, qs=384), api.S3W_ERR_UNSUPPORTED),
    (dict(heads=80, qs=5120), api.S3W_ERR_UNSUPPORTED),     # C = 5120 > 4096
    (dict(ws=FAKE + 16), api.S3W_ERR_MISALIGNED),           # workspace not 32-byte aligned
    (dict(o=FAKE + 16), api.S3W_ERR_MISALIGNED),            # attention output not 32-byte aligned
    (dict(res=FAKE + 16, out=FAKE + 16), api.S3W_ERR_MISALIGNED),   # residual / out (in place) not 32-byte aligned
    (dict(sc=FAKE + 16), api.S3W_ERR_MISALIGNED),           # FiLM scale not 32-byte aligned
    (dict(sh=FAKE + 48), api.S3W_ERR_MISALIGNED),           # FiLM shift not 32-byte aligned
    (dict(out=FAKE + 16 * 512), api.S3W_ERR_INVALID_ARG),   # partial overlap of out with residual
    (dict(out=FAKE_QKV + 4096, res=FAKE_QKV + 4096), api.S3W_ERR_INVALID_ARG),   # out over q, k, v
    (dict(o=FAKE_QKV + 1024), api.S3W_ERR_INVALID_ARG),     # attention output over q, k, v
])
def test_fused_rejects_bad_arguments_on_host(over, expect):
    if "out" in over and "res" not in over:
        over = dict(over, res=FAKE + 64)
    assert _fused(**over) == expect


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "HERE", str(tmp_path))
    with pytest.raises(RuntimeError, match="missing"):
        api.load_library()


def _qkv(**over):
    # defaults: qkv over x (rejected last), so a call with them returns on the host everywhere
    a = dict(x=FAKE, w=FAKE_QKV, b=None, qkv=FAKE, tokens=1152, C=512)
    a.update(over)
    return s3w.load_library().swin3d_qkv_proj_fwd(a["x"], a["w"], a["b"], a["qkv"], a["tokens"], a["C"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(x=None), api.S3W_ERR_INVALID_ARG),
    (dict(tokens=0), api.S3W_ERR_INVALID_ARG),
    (dict(C=0), api.S3W_ERR_INVALID_ARG),
    (dict(C=48), api.S3W_ERR_UNSUPPORTED),                    # not a multiple of 32
    (dict(C=16416), api.S3W_ERR_UNSUPPORTED),                 # above 16,384
    (dict(tokens=2 ** 31), api.S3W_ERR_UNSUPPORTED),          # TMA row coordinates are 32-bit
    (dict(x=FAKE + 8), api.S3W_ERR_MISALIGNED),
    (dict(qkv=FAKE + 16), api.S3W_ERR_MISALIGNED),            # qkv needs 32-byte alignment
    (dict(), api.S3W_ERR_INVALID_ARG),                        # qkv over x
    (dict(qkv=FAKE_QKV + 3 * 512 * 512 * 2 - 64), api.S3W_ERR_INVALID_ARG),   # qkv over the end of w
])
def test_qkv_proj_rejects_bad_arguments_on_host(over, expect):
    assert _qkv(**over) == expect


def _qkv_attn(**over):
    a = dict(x=FAKE, w=FAKE_QKV, b=None, qkv=2 * FAKE_QKV, o=2 * FAKE_QKV + 4096, outd=0, B=1, T=4, H=12, W=24,
             wt=2, wh=6, ww=12, st=1, sh=3, sw=6, heads=8, hd=64, scale=0.0)
    a.update(over)
    return s3w.load_library().swin3d_qkv_window_attn_fwd(
        a["x"], a["w"], a["b"], a["qkv"], a["o"], a["outd"], a["B"], a["T"], a["H"], a["W"], a["wt"], a["wh"],
        a["ww"], a["st"], a["sh"], a["sw"], a["heads"], a["hd"], a["scale"], None)


@pytest.mark.parametrize("over,expect", [
    (dict(o=None), api.S3W_ERR_INVALID_ARG),
    (dict(heads=0), api.S3W_ERR_INVALID_ARG),
    (dict(heads=300), api.S3W_ERR_UNSUPPORTED),               # C = 19,200 > 16,384
    (dict(hd=48), api.S3W_ERR_UNSUPPORTED),                   # head_dim 32 or 64 only
    (dict(st=2), api.S3W_ERR_INVALID_ARG),                    # shift == window
    (dict(), api.S3W_ERR_INVALID_ARG),                        # o over the projection's output
])
def test_qkv_window_attn_rejects_bad_arguments_on_host(over, expect):
    assert _qkv_attn(**over) == expect
