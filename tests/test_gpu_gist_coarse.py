"""Segment-wise (coarse) gist layout ("A Silver Bullet or a Compromise for Full
Attention? A Comprehensive Study of Gist Token-based Context Compression",
sections 2 and 6; appendix E for the 16K / ratio 4 / 1K-segment case): the
builder's permutation, gist bits, tile lists and far-key arrays bit-exact
against the oracle; forward and backward against the oracle on small cases,
on both implementations; sampled rows and the dV identity on the appendix-E
sizes."""
import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import attention as A
from oracle import gist as Gi
from oracle import gzip_mask as G

from _cases import check_close, sample_rows, to_dev, to_np

pytestmark = pytest.mark.gpu

IMPLS = {"cuda_cores": 1, "tensor_cores": 2}


def layout(N, sinks, L, r):
    g = Gi.coarse_gist_flags(N, sinks, L, r)
    seg = Gi.segment_ids(N, sinks, L, r)
    perm = Gi.shift_permutation(g, 128)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(N, dtype=perm.dtype)
    return g, seg, perm, inv


def _np(t, dt=None):
    a = t.cpu().numpy()
    return a.view(dt) if dt is not None else a


@pytest.mark.parametrize("N,sinks,L,r", [
    (20480, 0, 1024, 4), (3000, 128, 96, 4), (2500, 5, 200, 8), (1300, 300, 40, 2),
    (777, 0, 1024, 4), (4096 + 77, 130, 512, 4)])
def test_coarse_layout_lists(sa, N, sinks, L, r):
    md = sa.gist_mask(N, 8, sinks, r, 0, segment=L)
    lists = sa.build_block_mask(md, None)
    torch.cuda.synchronize()
    g, seg, perm, _ = layout(N, sinks, L, r)
    assert np.array_equal(_np(lists.perm), perm)
    words = _np(lists.gist_bits, np.uint32)
    bits = ((words[:, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(-1)[:N].astype(bool)
    assert np.array_equal(bits, g)
    T = (N + 127) // 128
    vis = lambda rows: Gi.coarse_visibility(g, seg, sinks, rows=perm[rows])[:, perm]
    otrp, otc, otk = Gi.tile_lists(vis, 128, 32, N=N)
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


def case(N, sinks, L, r, heads, kv_heads, d, index):
    return W.scaled("gist_coarse_20k", index=index, seq_len=N, sinks=sinks, gist_segment=L,
                    ratio=r, heads=heads, kv_heads=kv_heads, head_dim=d)


def run(sa, w, q, k, v, do=None, impl=0):
    md = sa.gist_mask(w["seq_len"], w["heads"], w["sinks"], w["ratio"], w["window"],
                      segment=w["gist_segment"])
    lists = sa.build_block_mask(md, None)
    tq, tk, tv = (to_dev(x, "bf16") for x in (q, k, v))
    o, lse = sa.forward(tq, tk, tv, md, lists, impl=impl)
    out = [to_np(o), to_np(lse)]
    if do is not None:
        dq, dk, dv = sa.backward(tq, tk, tv, o, lse, to_dev(do, "bf16"), md, lists, impl=impl)
        out += [to_np(dq), to_np(dk), to_np(dv)]
    torch.cuda.synchronize()
    return out


SMALL = [(1000, 16, 96, 4, 64), (2000, 130, 400, 4, 128), (700, 0, 64, 2, 128),
         (128 * 8, 128, 256, 4, 128), (900, 0, 2048, 4, 64)]


@pytest.mark.parametrize("N,sinks,L,r,d", SMALL)
@pytest.mark.parametrize("impl", list(IMPLS))
def test_coarse_forward_small(sa, N, sinks, L, r, d, impl):
    w = case(N, sinks, L, r, 4, 2, d, 600 + N + d)
    q, k, v = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v"))  # physical order
    o, lse = run(sa, w, q, k, v, impl=IMPLS[impl])
    g, seg, perm, inv = layout(N, sinks, L, r)
    vis = Gi.coarse_visibility(g, seg, sinks)
    for h in range(4):
        hk = h // 2
        ro, rl = A.forward(q[0, inv, h], k[0, inv, hk], v[0, inv, hk], vis)
        check_close(o[0, inv, h], ro, "bf16", f"O h{h}")
        check_close(lse[0, h, inv], rl, "bf16", f"LSE h{h}")


@pytest.mark.parametrize("N,sinks,L,r,d", SMALL[:4])
@pytest.mark.parametrize("impl", list(IMPLS))
def test_coarse_backward_small(sa, N, sinks, L, r, d, impl):
    heads, kv_heads = 4, 2
    w = case(N, sinks, L, r, heads, kv_heads, d, 700 + N + d)
    q, k, v, do = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v", "do"))
    _, _, dq, dk, dv = run(sa, w, q, k, v, do, impl=IMPLS[impl])
    g, seg, perm, inv = layout(N, sinks, L, r)
    vis = Gi.coarse_visibility(g, seg, sinks)
    rep = heads // kv_heads
    rk = np.zeros((N, kv_heads, d))
    rv = np.zeros((N, kv_heads, d))
    for h in range(heads):
        hk = h // rep
        rq, rk_h, rv_h, _, _ = A.backward(q[0, inv, h], k[0, inv, hk], v[0, inv, hk], do[0, inv, h], vis)
        check_close(dq[0, inv, h], rq, "bf16", f"dQ h{h}")
        rk[:, hk] += rk_h
        rv[:, hk] += rv_h
    for hk in range(kv_heads):
        check_close(dk[0, inv, hk], rk[:, hk], "bf16", f"dK kv{hk}")
        check_close(dv[0, inv, hk], rv[:, hk], "bf16", f"dV kv{hk}")


def test_coarse_full_size_sampled(sa):
    """16 segments of 1024 raw tokens and 256 gists (ratio 4), 32 query / 8 KV
    heads: sampled O / LSE / dQ rows, dK / dV of sampled raw keys (seen only
    inside their segment), and sum_j dV_j = sum over the group's rows of dO."""
    w = W.WORKLOADS["gist_coarse_20k"]
    q, k, v, do = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v", "do"))
    o, lse, dq, dk, dv = run(sa, w, q, k, v, do)
    assert all(np.isfinite(x).all() for x in (o, lse, dq, dk, dv))
    N, S, L, r = w["seq_len"], w["sinks"], w["gist_segment"], w["ratio"]
    rep = w["heads"] // w["kv_heads"]
    g, seg, perm, inv = layout(N, S, L, r)
    for hk in range(w["kv_heads"]):
        want = do[0, :, hk * rep:(hk + 1) * rep].astype(np.float64).sum((0, 1))
        np.testing.assert_allclose(dv[0, :, hk].sum(0), want, rtol=1e-3, atol=0.5)
    keys_of = lambda P: np.sort(inv[Gi.coarse_visible_keys(g, seg, S, int(perm[P]))])
    for h in (0, 13, w["heads"] - 1):
        rows = sample_rows(N, 8, seed=h)
        ro, rl = A.forward_rows(q[0, :, h], k[0, :, h // rep], v[0, :, h // rep], keys_of, rows)
        check_close(o[0, rows, h], ro, "bf16", f"O rows h{h}")
        check_close(lse[0, h, rows], rl, "bf16", f"LSE rows h{h}")
        rq = A.backward_rows(q[0, :, h], k[0, :, h // rep], v[0, :, h // rep], do[0, :, h], keys_of, rows)
        check_close(dq[0, rows, h], rq, "bf16", f"dQ rows h{h}")
    period = L + L // r
    # raw keys late in their segments: each is seen by the few hundred rows up to the segment's end
    raw = [j for j in (S + 1000, S + 5 * period + 1010, S + 12 * period + 900, N - 300) if not g[j]]
    assert len(raw) == 4
    cols = inv[np.array(raw)]
    seg_end = lambda j: S + (seg[j] + 1) * period
    rows_of = lambda P: inv[np.arange(int(perm[P]), min(N, seg_end(int(perm[P]))))]
    for hk in (0, w["kv_heads"] - 1):
        rk = np.zeros((len(cols), w["head_dim"]))
        rv = np.zeros_like(rk)
        for h in range(hk * rep, (hk + 1) * rep):
            a, b = A.backward_cols(q[0, :, h], k[0, :, hk], v[0, :, hk], do[0, :, h], keys_of, rows_of, cols)
            rk += a
            rv += b
        check_close(dk[0, cols, hk], rk, "bf16", f"dK raw cols kv{hk}")
        check_close(dv[0, cols, hk], rv, "bf16", f"dV raw cols kv{hk}")
