"""GPU mask/layout builder vs the oracle, bit-exact (integers only)."""
import numpy as np
import pytest

import sa_workloads as W
from oracle import gist as Gi
from oracle import gzip_mask as G

from _cases import gist_layout, gzip_flags_oracle, gzip_flags_product

pytestmark = pytest.mark.gpu


def _np(t, dt=None):
    a = t.cpu().numpy()
    return a.view(dt) if dt is not None else a


def check_gzip_lists(lists, flags, batch, B, b, w, head_class_list=None, full_tiles=True):
    N = B * b
    T = (N + 127) // 128
    region, tregion = B * (B + 1) // 2, T * (T + 1) // 2
    rp = _np(lists.row_ptr).reshape(batch * 3, B + 1)
    cp = _np(lists.col_ptr).reshape(batch * 3, B + 1)
    ci, ri = _np(lists.col_idx), _np(lists.row_idx)
    bits = _np(lists.bits, np.uint32).reshape(batch * 3, B, (B + 31) // 32)
    trp = _np(lists.tile_row_ptr).reshape(batch * 3, T + 1)
    tcp = _np(lists.tile_col_ptr).reshape(batch * 3, T + 1)
    tc, tk = _np(lists.tile_col), _np(lists.tile_kind)
    tr, tkt = _np(lists.tile_row), _np(lists.tile_kind_t)
    for bt in range(batch):
        masks = G.block_masks(flags[bt], w)
        for c in range(3):
            bc = bt * 3 + c
            orp, oci = G.csr(masks[c])
            assert np.array_equal(rp[bc] - bc * region, orp), (bt, c)
            assert np.array_equal(ci[bc * region: bc * region + orp[-1]], oci), (bt, c)
            ocp, ori = G.csc(masks[c])
            assert np.array_equal(cp[bc] - bc * region, ocp), (bt, c)
            assert np.array_equal(ri[bc * region: bc * region + ocp[-1]], ori), (bt, c)
            assert np.array_equal(bits[bc], G.bitmask(masks[c])), (bt, c)
            if full_tiles:
                otrp, otc, otk = G.tile_lists(masks[c], b)
            else:
                # b == 128: the oracle pins tile lists == block lists, diagonal masked
                otrp, otc = orp, oci
                otk = np.array([1 if otc[e] == i else 0 for i in range(B)
                                for e in range(otrp[i], otrp[i + 1])], np.int32)
            assert np.array_equal(trp[bc] - bc * tregion, otrp), (bt, c)
            s = slice(bc * tregion, bc * tregion + otrp[-1])
            assert np.array_equal(tc[s], otc) and np.array_equal(tk[s], otk), (bt, c)
            otcp, otr, otkt = G.transpose_lists(otrp, otc, otk, T)
            assert np.array_equal(tcp[bc] - bc * tregion, otcp), (bt, c)
            s = slice(bc * tregion, bc * tregion + otcp[-1])
            assert np.array_equal(tr[s], otr) and np.array_equal(tkt[s], otkt), (bt, c)


@pytest.mark.parametrize("name", ["gzip_tiny_fp32", "gzip_8k", "gzip_64k_fwdbwd"])
def test_gzip_lists_on_workloads(sa, name):
    w = W.WORKLOADS[name]
    fp, fo = gzip_flags_product(sa, w), gzip_flags_oracle(w)
    assert np.array_equal(fp, fo)
    B = w["seq_len"] // w["block"]
    md = sa.gzip_mask(w["batch"], w["seq_len"], w["block"], w["window"], w["heads"])
    lists = sa.build_block_mask(md, fp)
    check_gzip_lists(lists, fo, w["batch"], B, w["block"], w["window"],
                     full_tiles=w["block"] != 128)


@pytest.mark.parametrize("b,B,w,mode", [
    (16, 24, 0, "rand"), (32, 12, 1, "all"), (64, 19, 2, "none"), (64, 19, 30, "rand"),
    (128, 9, 1, "rand"), (256, 5, 1, "all"), (256, 6, 0, "rand"), (16, 40, 3, "rand")])
def test_gzip_lists_sweep(sa, b, B, w, mode):
    rng = np.random.default_rng(b * 100 + B)
    batch = 2
    if mode == "all":
        flags = np.ones((batch, B), np.uint8)
    elif mode == "none":
        flags = np.zeros((batch, B), np.uint8)
    else:
        flags = (rng.random((batch, B)) < 0.35).astype(np.uint8)
    md = sa.gzip_mask(batch, B * b, b, w, 6)
    lists = sa.build_block_mask(md, flags)
    check_gzip_lists(lists, flags, batch, B, b, w)


def check_gist(sa, lists, N, sinks, ratio, window, tail, flags=None):
    g, perm, _ = gist_layout(N, sinks, ratio, flags)
    assert np.array_equal(_np(lists.perm), perm)
    words = _np(lists.gist_bits, np.uint32)
    bits = ((words[:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(-1)[:N].astype(bool)
    assert np.array_equal(bits, g)
    T = (N + 127) // 128
    vis = lambda rows: Gi.visibility(g, sinks, window, rows=perm[rows])[:, perm]
    otrp, otc, otk = Gi.tile_lists(vis, 128, tail, N=N)
    assert np.array_equal(_np(lists.tile_row_ptr), otrp)
    assert np.array_equal(_np(lists.tile_col)[:otrp[-1]], otc)
    assert np.array_equal(_np(lists.tile_kind)[:otrp[-1]], otk)
    otcp, otr, otkt = G.transpose_lists(otrp, otc, otk, T)
    assert np.array_equal(_np(lists.tile_col_ptr), otcp)
    assert np.array_equal(_np(lists.tile_row)[:otcp[-1]], otr)
    assert np.array_equal(_np(lists.tile_kind_t)[:otcp[-1]], otkt)
    far_idx, far_ptr = Gi.always_visible_keys(g, sinks, perm, 128)
    assert np.array_equal(_np(lists.far_ptr), far_ptr)
    assert np.array_equal(_np(lists.far_idx)[:far_ptr[-1]], far_idx)


@pytest.mark.parametrize("N,sinks,ratio,window,tail", [
    (32768, 128, 4, 128, 32), (1000, 128, 4, 128, 32), (4096 + 77, 5, 2, 16, 64),
    (700, 0, 1, 300, 32), (129, 128, 4, 128, 32)])
def test_gist_layout(sa, N, sinks, ratio, window, tail):
    md = sa.gist_mask(N, 8, sinks, ratio, window, gist_tail=tail)
    lists = sa.build_block_mask(md, None)
    check_gist(sa, lists, N, sinks, ratio, window, tail)


def test_gist_layout_explicit_flags(sa):
    N = 3000
    flags = (np.random.default_rng(5).random(N) < 0.2).astype(np.uint8)
    md = sa.gist_mask(N, 8, 64, 4, 100)
    lists = sa.build_block_mask(md, flags)
    check_gist(sa, lists, N, 64, 4, 100, 32, flags=flags)
