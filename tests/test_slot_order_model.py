"""Model of the attention kernels' slot order and TMA box plan (csrc/attn_common.cuh):
init_slot_consts' slot_off, which gives every slot of a window its (t, h, w) offset, and the
loader's boxes, which decide which grid token lands in which shared-memory row.  The two are
written independently in the kernel; this checks, on the CPU, for many window shapes, shifts
and padded grids, that every row a box writes holds the token its slot stands for, that the
boxes of a tile write each of its N rows exactly once and nothing else, and that every box
shape the loader uses is one the host encodes."""
import itertools

import pytest


def slot_off(r, a, g):
    per_slab = g["ww"] * g["wh"]
    rt, i = divmod(r, per_slab)
    if a == 0:
        return rt
    if g["sw"] > 0:
        n1 = g["ww"] - g["sw"]
        if i < g["wh"] * n1:
            rh, rw = divmod(i, n1)
        else:
            rh, j = divmod(i - g["wh"] * n1, g["sw"])
            rw = n1 + j
    else:
        rh, rw = divmod(i, g["ww"])
    return rh if a == 1 else rw


def box_shapes(g):
    ww, wh, sw, sh = g["ww"], g["wh"], g["sw"], g["sh"]
    n1, n2, h1, h2 = ww - sw, (sw if sw > 0 else ww), wh - sh, (sh if sh > 0 else wh)
    return {"slab": (ww, wh), "h1": (ww, h1), "h2": (ww, h2), "A": (n1, wh), "B": (n2, wh),
            "A1": (n1, h1), "A2": (n1, h2), "B1": (n2, h1), "B2": (n2, h2)}


def loader_boxes(g, bh, bw):
    """(first row inside the slab, shape name, w0, h0) of every box of one slab."""
    wh, ww, sw, Ph, Pw = g["wh"], g["ww"], g["sw"], g["Ph"], g["Pw"]
    wrap_h = bh + wh > Ph
    n1h = Ph - bh
    n1 = ww - sw
    xb = bw + n1
    if xb >= Pw:
        xb -= Pw
    if sw == 0:
        if not wrap_h:
            return [(0, "slab", bw, bh)]
        return [(0, "h1", bw, bh), (n1h * ww, "h2", bw, 0)]
    b = wh * n1
    if not wrap_h:
        return [(0, "A", bw, bh), (b, "B", xb, bh)]
    return [(0, "A1", bw, bh), (n1h * n1, "A2", bw, 0), (b, "B1", xb, bh), (b + n1h * sw, "B2", xb, 0)]


def geometries():
    for (wt, wh, ww), (T, H, W) in itertools.product(
            [(2, 6, 12), (1, 12, 12), (2, 3, 5), (1, 1, 8), (3, 4, 4), (2, 6, 7)],
            [(4, 12, 24), (5, 13, 29), (2, 6, 12), (3, 7, 9)]):
        if wt * wh * ww > 144:
            continue
        for st, sh, sw in {(0, 0, 0), (wt // 2, wh // 2, ww // 2), (wt - 1, wh - 1, ww - 1), (0, wh // 2, 0),
                           (wt // 2, 0, ww // 2)}:
            Pt, Ph, Pw = (-(-T // wt) * wt, -(-H // wh) * wh, -(-W // ww) * ww)
            yield dict(wt=wt, wh=wh, ww=ww, st=st, sh=sh, sw=sw, T=T, H=H, W=W, Pt=Pt, Ph=Ph, Pw=Pw)


@pytest.mark.parametrize("g", list(geometries()), ids=lambda g: "w{wt}x{wh}x{ww}_s{st}{sh}{sw}_g{T}x{H}x{W}".format(**g))
def test_boxes_write_every_slot_its_token(g):
    N = g["wt"] * g["wh"] * g["ww"]
    shapes = box_shapes(g)
    for itw, ih, iw in itertools.product(range(g["Pt"] // g["wt"]), range(g["Ph"] // g["wh"]), range(g["Pw"] // g["ww"])):
        bt, bh, bw = itw * g["wt"] + g["st"], ih * g["wh"] + g["sh"], iw * g["ww"] + g["sw"]
        rows = {}
        for rt in range(g["wt"]):
            t = (bt + rt) % g["Pt"]
            slab = rt * g["wh"] * g["ww"]
            for first, name, w0, h0 in loader_boxes(g, bh, bw):
                bw_, bh_ = shapes[name]
                assert bw_ >= 1 and bh_ >= 1 and 0 <= w0 < g["Pw"] and 0 <= h0 < g["Ph"]
                for hh in range(bh_):
                    for xx in range(bw_):
                        row = slab + first + hh * bw_ + xx
                        assert row not in rows, "two boxes write one row"
                        rows[row] = (t, h0 + hh, w0 + xx)
        assert sorted(rows) == list(range(N)), "the boxes must write exactly the window's rows"
        for r in range(N):
            rt, rh, rw = (slot_off(r, a, g) for a in range(3))
            want = ((bt + rt) % g["Pt"], (bh + rh) % g["Ph"], (bw + rw) % g["Pw"])
            assert rows[r] == want, (r, rows[r], want)


def test_slot_order_is_a_permutation_of_window_offsets():
    for g in geometries():
        N = g["wt"] * g["wh"] * g["ww"]
        offs = {tuple(slot_off(r, a, g) for a in range(3)) for r in range(N)}
        assert offs == set(itertools.product(range(g["wt"]), range(g["wh"]), range(g["ww"])))
