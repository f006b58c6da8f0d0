"""sa_backward vs the oracle: dQ, dK, dV element by element on small cases
and on whole heads whose lists are long (a 16K sequence with 60% literal
blocks); at the 64K workload sampled dQ rows, whole key blocks that every
later literal query block sees (the longest column lists) and keys seen only
nearby, and the identity sum_j dV_j = sum_p dO_p that holds at any size."""
import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import attention as A
from oracle import gist as Gi
from oracle import gzip_mask as G

from _cases import (check_close, gist_layout, gzip_flags_oracle, gzip_flags_product, gzip_inputs,
                    to_dev, to_np)

pytestmark = pytest.mark.gpu


IMPLS = {"cuda_cores": 1, "tensor_cores": 2}


def run(sa, w, q, k, v, do, flags, impl=0):
    dt = w["dtype"]
    md = sa.gzip_mask(w["batch"], w["seq_len"], w["block"], w["window"], w["heads"])
    lists = sa.build_block_mask(md, flags)
    tq, tk, tv, tdo = (to_dev(x, dt) for x in (q, k, v, do))
    o, lse = sa.forward(tq, tk, tv, md, lists)
    dq, dk, dv = sa.backward(tq, tk, tv, o, lse, tdo, md, lists, impl=impl)
    torch.cuda.synchronize()
    return to_np(o), to_np(dq), to_np(dk), to_np(dv)


@pytest.mark.parametrize("w", [
    W.scaled("gzip_8k", index=301, batch=2, seq_len=16 * 24, block=16, window=1, heads=4,
             kv_heads=4, head_dim=32, dtype="fp32"),
    W.scaled("gzip_8k", index=302, batch=1, seq_len=64 * 11, block=64, window=2, heads=4,
             kv_heads=4, head_dim=64, dtype="bf16"),
    W.scaled("gzip_8k", index=303, batch=1, seq_len=128 * 6, block=128, window=1, heads=4,
             kv_heads=4, head_dim=128, dtype="bf16", p_literal=0.5),
    W.scaled("gzip_8k", index=304, batch=2, seq_len=16 * 40, block=16, window=3, heads=4,
             kv_heads=4, head_dim=64, dtype="bf16", p_literal=0.4),
    W.scaled("gzip_8k", index=305, batch=1, seq_len=256 * 4, block=256, window=1, heads=6,
             kv_heads=6, head_dim=128, dtype="bf16", p_literal=0.5),
], ids=["b16_fp32", "b64_ragged_bf16", "b128_bf16", "b16_bf16", "b256_h6_bf16"])
@pytest.mark.parametrize("impl", list(IMPLS))
def test_backward_small(sa, w, impl):
    if w["dtype"] == "fp32" and impl == "tensor_cores":
        pytest.skip("tensor cores take bf16 only")
    q, k, v, do = gzip_inputs(w, with_do=True)
    fp, fo = gzip_flags_product(sa, w), gzip_flags_oracle(w)
    o, dq, dk, dv = run(sa, w, q, k, v, do, fp, IMPLS[impl])
    cls = G.head_classes(w["heads"])
    for bt in range(w["batch"]):
        masks = G.block_masks(fo[bt], w["window"])
        for h in range(w["heads"]):
            allowed = G.token_mask(masks[cls[h]], w["block"])
            # the oracle's upstream gradient is the one the kernel was given
            rq, rk, rv, _, _ = A.backward(q[bt, :, h], k[bt, :, h], v[bt, :, h], do[bt, :, h], allowed)
            check_close(dq[bt, :, h], rq, w["dtype"], f"dQ b{bt} h{h}")
            check_close(dk[bt, :, h], rk, w["dtype"], f"dK b{bt} h{h}")
            check_close(dv[bt, :, h], rv, w["dtype"], f"dV b{bt} h{h}")


def test_backward_full_size(sa):
    w = W.WORKLOADS["gzip_64k_fwdbwd"]
    q, k, v, do = gzip_inputs(w, with_do=True)
    fp, fo = gzip_flags_product(sa, w), gzip_flags_oracle(w)
    o, dq, dk, dv = run(sa, w, q, k, v, do, fp)
    assert all(np.isfinite(x).all() for x in (dq, dk, dv))
    b, B = w["block"], w["seq_len"] // w["block"]
    cls = G.head_classes(w["heads"])
    rng = np.random.default_rng(0)
    for bt in range(w["batch"]):
        masks = G.block_masks(fo[bt], w["window"])
        # identity over all keys of every head (any size): sum_j dV_j = sum_i dO_i,
        # since every row of P sums to one. (The companion identity sum_j dK_j = 0
        # is not checked here: it holds only up to the bf16 rounding of O inside
        # Delta = rowsum(dO * O) and of dS, which over 65536 rows grows to the
        # size of any fixed bound; the sampled rows and columns below are compared
        # with the oracle instead.)
        np.testing.assert_allclose(dv[bt].sum(0), do[bt].astype(np.float64).sum(0), rtol=1e-3, atol=0.5)
        for h in (0, w["heads"] // 2, w["heads"] - 1):
            bm = masks[cls[h]]
            keys_of = lambda p: np.nonzero(G.token_mask(bm, b, rows=[p])[0])[0]
            rows = np.unique(np.concatenate([[0, 127, 128, w["seq_len"] - 1], rng.choice(w["seq_len"], 6)]))
            rq = A.backward_rows(q[bt, :, h], k[bt, :, h], v[bt, :, h], do[bt, :, h], keys_of, rows)
            check_close(dq[bt, rows, h], rq, "bf16", f"dQ rows b{bt} h{h}")
            # keys whose block is seen only by nearby query blocks (cheap to sum)
            lit = fo[bt].astype(bool)
            cheap = [j for j in range(B) if not (lit[j] and cls[h] != G.LOCAL) or
                     lit[j] and not lit[j + 1:].any()]
            jb = [cheap[0], cheap[len(cheap) // 2], cheap[-1]]
            cols = np.array([x * b + o_ for x in jb for o_ in (0, 77)])
            rows_of = lambda j: np.nonzero(G.token_mask(bm, b, rows=np.arange(j, min(w["seq_len"], j + (w["window"] + 2) * b)))[:, j])[0] + j
            rk, rv = A.backward_cols(q[bt, :, h], k[bt, :, h], v[bt, :, h], do[bt, :, h], keys_of, rows_of, cols)
            check_close(dk[bt, cols, h], rk, "bf16", f"dK cols b{bt} h{h}")
            check_close(dv[bt, cols, h], rv, "bf16", f"dV cols b{bt} h{h}")
        # long column lists: the first and a middle literal key block of the
        # literal and hybrid heads, seen by every later literal query block
        # (the key-major pass walks about 200 query blocks for each)
        lit_blocks = np.nonzero(fo[bt])[0]
        for h in (w["heads"] // 2, w["heads"] - 1):
            bm = masks[cls[h]]
            jb = [int(lit_blocks[0]), int(lit_blocks[len(lit_blocks) // 2])]
            cols = np.concatenate([np.arange(j * b, (j + 1) * b) for j in jb])
            qblocks = np.nonzero(bm[:, jb].any(axis=1))[0]
            assert len(qblocks) >= 64, len(qblocks)
            rows = (qblocks[:, None] * b + np.arange(b)[None, :]).ravel()
            mask = lambda r: G.token_mask(bm, b, rows=r)
            rk, rv = A.backward_cols_chunked(q[bt, :, h], k[bt, :, h], v[bt, :, h], do[bt, :, h],
                                             mask, rows, cols)
            check_close(dk[bt, cols, h], rk, "bf16", f"dK literal blocks {jb} b{bt} h{h}")
            check_close(dv[bt, cols, h], rv, "bf16", f"dV literal blocks {jb} b{bt} h{h}")


def test_backward_long_lists_whole_heads(sa):
    """Whole literal and hybrid heads of a 16K sequence with 60% literal
    128-token blocks: row lists and column lists of 60 to 80 blocks, compared
    element by element (dQ, dK, dV) with the oracle, on both implementations."""
    w = W.scaled("gzip_8k", index=310, batch=1, seq_len=16384, block=128, window=2, heads=4,
                 kv_heads=4, head_dim=128, dtype="bf16", p_literal=0.6)
    q, k, v, do = gzip_inputs(w, with_do=True)
    flags = gzip_flags_oracle(w)
    assert np.array_equal(flags, gzip_flags_product(sa, w))
    masks = G.block_masks(flags[0], w["window"])
    cls = G.head_classes(w["heads"])
    got = {impl: run(sa, w, q, k, v, do, flags, IMPLS[impl]) for impl in IMPLS}
    for h in (2, 3):  # the literal head and the hybrid head
        bm = masks[cls[h]]
        assert bm.sum(axis=0).max() >= 60 and bm.sum(axis=1).max() >= 60
        allowed = G.token_mask(bm, w["block"])
        rq, rk, rv, _, _ = A.backward(q[0, :, h], k[0, :, h], v[0, :, h], do[0, :, h], allowed)
        for impl, (o, dq, dk, dv) in got.items():
            check_close(dq[0, :, h], rq, "bf16", f"{impl} dQ h{h}")
            check_close(dk[0, :, h], rk, "bf16", f"{impl} dK h{h}")
            check_close(dv[0, :, h], rv, "bf16", f"{impl} dV h{h}")


# ------------------------------------------------------------------ gist layout
def run_gist_backward(sa, w, q, k, v, do, impl):
    md = sa.gist_mask(w["seq_len"], w["heads"], w["sinks"], w["ratio"], w["window"],
                      gist_tail=w.get("gist_tail", 32))
    lists = sa.build_block_mask(md, None)
    tq, tk, tv, tdo = (to_dev(x, "bf16") for x in (q, k, v, do))
    o, lse = sa.forward(tq, tk, tv, md, lists)
    dq, dk, dv = sa.backward(tq, tk, tv, o, lse, tdo, md, lists, impl=impl)
    torch.cuda.synchronize()
    return to_np(dq), to_np(dk), to_np(dv)


@pytest.mark.parametrize("N,sinks,window,heads,kv_heads,d", [
    (1000, 16, 32, 4, 2, 64), (128 * 6, 128, 128, 4, 2, 128), (2000, 130, 200, 4, 1, 128),
    (700, 0, 300, 2, 2, 64)])
@pytest.mark.parametrize("impl", list(IMPLS))
def test_gist_backward_small(sa, N, sinks, window, heads, kv_heads, d, impl):
    """Gist layout (UniGist, Approach): dQ, dK, dV in physical order against the
    oracle in logical order; dK and dV of a KV head sum the group's query heads."""
    w = W.scaled("gist_prefill_32k", index=400 + N + d, seq_len=N, sinks=sinks, window=window,
                 heads=heads, kv_heads=kv_heads, head_dim=d)
    q, k, v, do = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v", "do"))  # physical order
    dq, dk, dv = run_gist_backward(sa, w, q, k, v, do, IMPLS[impl])
    g, perm, inv = gist_layout(N, sinks, w["ratio"])
    vis = Gi.visibility(g, sinks, window)
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


def test_gist_backward_full_size_sampled(sa):
    """The 32K gist workload (32 query / 8 KV heads): sampled dQ rows, dK/dV of
    sampled raw keys (seen only by the queries of their window), and the
    identity sum_j dV_j = sum over the group's rows of dO, which holds at any size."""
    from _cases import sample_rows
    w = W.WORKLOADS["gist_prefill_32k"]
    q, k, v, do = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v", "do"))
    dq, dk, dv = run_gist_backward(sa, w, q, k, v, do, 0)
    assert all(np.isfinite(x).all() for x in (dq, dk, dv))
    N, S, Wn = w["seq_len"], w["sinks"], w["window"]
    rep = w["heads"] // w["kv_heads"]
    g, perm, inv = gist_layout(N, S, w["ratio"])
    for hk in range(w["kv_heads"]):
        want = do[0, :, hk * rep:(hk + 1) * rep].astype(np.float64).sum((0, 1))
        np.testing.assert_allclose(dv[0, :, hk].sum(0), want, rtol=1e-3, atol=0.5)
    keys_of = lambda P: np.sort(inv[Gi.visible_keys(g, S, Wn, int(perm[P]))])  # ascending physical
    for h in (0, 13, w["heads"] - 1):
        rows = sample_rows(N, 8, seed=h)
        rq = A.backward_rows(q[0, :, h], k[0, :, h // rep], v[0, :, h // rep], do[0, :, h], keys_of, rows)
        check_close(dq[0, rows, h], rq, "bf16", f"dQ rows h{h}")
    raw = [j for j in (S + 1, 5000, 16001, N - 130) if not g[j]]
    cols = inv[np.array(raw)]
    rows_of = lambda P: inv[np.arange(int(perm[P]), min(N, int(perm[P]) + Wn))]
    for hk in (0, w["kv_heads"] - 1):
        rk = np.zeros((len(cols), w["head_dim"]))
        rv = np.zeros_like(rk)
        for h in range(hk * rep, (hk + 1) * rep):
            a, b = A.backward_cols(q[0, :, h], k[0, :, hk], v[0, :, hk], do[0, :, h], keys_of, rows_of, cols)
            rk += a
            rv += b
        check_close(dk[0, cols, hk], rk, "bf16", f"dK raw cols kv{hk}")
        check_close(dv[0, cols, hk], rv, "bf16", f"dV raw cols kv{hk}")
    # keys every later query sees (sinks and gists): their gradients come from the
    # far items of the dK/dV pass (about 256 query tiles each) and the far scatter
    gists = np.nonzero(g)[0]
    far = {0: [3, S - 1, int(gists[len(gists) // 2])], w["kv_heads"] - 1: [int(gists[-40])]}
    vis = lambda r: Gi.visibility(g, S, Wn, rows=r)
    for hk, logical in far.items():
        logical = np.array(logical)
        rows = np.arange(logical.min(), N)
        rk = np.zeros((len(logical), w["head_dim"]))
        rv = np.zeros_like(rk)
        for h in range(hk * rep, (hk + 1) * rep):
            a, b = A.backward_cols_chunked(q[0, inv, h], k[0, inv, hk], v[0, inv, hk], do[0, inv, h],
                                           vis, rows, logical)
            rk += a
            rv += b
        check_close(dk[0, inv[logical], hk], rk, "bf16", f"dK far keys {logical.tolist()} kv{hk}")
        check_close(dv[0, inv[logical], hk], rv, "bf16", f"dV far keys {logical.tolist()} kv{hk}")
