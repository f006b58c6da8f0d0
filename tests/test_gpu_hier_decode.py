"""sa_gist_hier_decode (gist of gists) vs the oracle: the kept groups and
chunks (exact, except across float32-level near ties of the summed logits,
see the flat decode's tests) and O / LSE over the selected key set, on shapes
of both implementations (the tensor-core kernel takes at least 128 level-2
gists and groups of 8 to 128 level-1 gists that divide 128; the CUDA-core
passes the rest)."""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import decode as D

from _cases import check_close, to_np

pytestmark = pytest.mark.gpu


def bound(q, gk, s, g, rep, d):
    qg = np.abs(q[s, g * rep:(g + 1) * rep].astype(np.float64))
    return lambda c: 2 * d * 2.0 ** -24 / np.sqrt(d) * (qg @ np.abs(gk[s, g, c])).sum()


def near_tie_ok(got, want, scores, eligible, b):
    """got and want pick equally many; every swapped pair is a near tie."""
    gs, ws_ = set(got[got >= 0].tolist()), set(want[want >= 0].tolist())
    assert len(gs) == len(ws_) and gs <= set(np.nonzero(eligible)[0].tolist())
    lo_in = min(gs - ws_, key=lambda c: scores[c], default=None)
    hi_out = max(ws_ - gs, key=lambda c: scores[c], default=None)
    if lo_in is not None:
        assert scores[hi_out] - scores[lo_in] <= b(lo_in) + b(hi_out)


def check(sa, w, seqs=None):
    n, Hkv, L, d = w["n_seq"], w["kv_heads"], w["cache_len"], w["head_dim"]
    chunk, fo, k2, k1, win = w["chunk"], w["fanout"], w["top_k2"], w["top_k"], w["window"]
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda", torch.bfloat16)
    q = W.decode_query(w)
    g2k = np.stack([W.decode_gists2(w, s, "k") for s in range(n)])
    g2v = np.stack([W.decode_gists2(w, s, "v") for s in range(n)])
    g1k = np.stack([W.decode_gists(w, s, "k") for s in range(n)])
    g1v = np.stack([W.decode_gists(w, s, "v") for s in range(n)])
    kc = torch.empty(n, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)

    def one(i):
        s_, g_ = divmod(i, Hkv)
        return s_, g_, W.decode_raw(w, s_, g_, "k"), W.decode_raw(w, s_, g_, "v")

    with ThreadPoolExecutor(8) as ex:
        for s_, g_, rk_, rv_ in ex.map(one, range(n * Hkv)):
            kc[s_, g_] = dev(rk_)
            vc[s_, g_] = dev(rv_)
    sel2, sel1, o, lse = sa.gist_hier_decode(dev(q), dev(g2k), dev(g2v), dev(g1k), dev(g1v), kc, vc,
                                             chunk, fo, k2, k1, win)
    torch.cuda.synchronize()
    st = sa.gist_hier_decode.last_workspace[:8].view(torch.int32).cpu().tolist()
    assert st[0] == 0, f"device status {st[0]} at {st[1]}"
    sel2, sel1, o, lse = sel2.cpu().numpy(), sel1.cpu().numpy(), to_np(o), to_np(lse)
    rep = w["heads"] // Hkv
    n2 = w["n_gists"] // fo
    for s in (range(n) if seqs is None else seqs):
        rk = [to_np(kc[s, g]) for g in range(Hkv)]
        rv = [to_np(vc[s, g]) for g in range(Hkv)]
        osel2, osel1, oo, ol = D.hier_decode_one(q[s], g2k[s], g2v[s], g1k[s], g1v[s], rk, rv, chunk,
                                                 fo, k2, k1, win)
        s2 = D.group_scores(q[s], g2k[s])
        s1 = D.group_scores(q[s], g1k[s])
        for g in range(Hkv):
            if np.array_equal(sel2[s, g], osel2[g]) and np.array_equal(sel1[s, g], osel1[g]):
                continue
            elig2 = (np.arange(n2) + 1) * fo * chunk <= L - win
            near_tie_ok(sel2[s, g], osel2[g], s2[g], elig2, bound(q, g2k, s, g, rep, d))
            # the chunks must be the best of the GPU's own groups
            groups = sel2[s, g][sel2[s, g] >= 0]
            cand = np.zeros(w["n_gists"], bool)
            for c in groups:
                cand[c * fo:(c + 1) * fo] = True
            want1 = D.select_top_k(s1[g], cand, k1)
            near_tie_ok(sel1[s, g], want1, s1[g], cand, bound(q, g1k, s, g, rep, d))
            # O on the GPU's own selection
            pos = D.raw_key_positions(sel1[s, g], chunk, L, win)
            lv1 = np.nonzero(cand)[0]
            keys = np.concatenate([g2k[s, g], g1k[s, g][lv1], rk[g][pos]])
            vals = np.concatenate([g2v[s, g], g1v[s, g][lv1], rv[g][pos]])
            for h in range(g * rep, (g + 1) * rep):
                oo[h], ol[h] = D.attend(q[s, h], keys, vals, 1 / np.sqrt(d))
        check_close(o[s], oo, "bf16", f"O seq {s}")
        check_close(lse[s], ol, "bf16", f"LSE seq {s}")


@pytest.mark.parametrize("chunk,n_gists,fanout,k2,k1,window,heads", [
    (16, 64, 8, 3, 10, 64, 8),      # small, GQA 4
    (32, 128, 16, 2, 40, 0, 8),     # no window: every group eligible; k1 > one group
    (8, 300, 10, 40, 5, 100, 4),    # more groups asked than eligible
    (16, 96, 4, 4, 0, 32, 16),      # nothing unfolded to raw tokens (GQA 8)
    (16, 96, 4, 0, 6, 32, 2),       # no group kept: nothing to unfold
    (32, 4096, 32, 8, 64, 512, 8),  # the workload's level sizes, two sequences
    # shapes the tensor-core kernel takes (at least 128 level-2 gists, 8 <= fanout | 128)
    (16, 2048, 16, 3, 10, 64, 8),     # GQA 4, groups of 16 level-1 gists
    (8, 1024, 8, 200, 5, 1792, 4),    # 200 groups asked, 100 eligible
    (16, 2048, 16, 4, 0, 32, 16),     # nothing unfolded to raw tokens (GQA 8)
    (16, 2048, 16, 0, 6, 32, 2),      # no group kept (one query head per KV head)
    (32, 4096, 32, 8, 64, 0, 8),      # no window
    (8, 8192, 64, 5, 20, 300, 8),     # groups of 64 level-1 gists, a ragged window
])
def test_hier_decode_small(sa, chunk, n_gists, fanout, k2, k1, window, heads):
    w = W.scaled("gist_hier_decode_128k", index=700 + n_gists + k2, n_seq=2, cache_len=chunk * n_gists,
                 chunk=chunk, n_gists=n_gists, fanout=fanout, top_k2=k2, top_k=k1, window=window,
                 heads=heads, kv_heads=2)
    check(sa, w)


def test_hier_decode_full_size(sa):
    check(sa, W.WORKLOADS["gist_hier_decode_128k"], seqs=[0, 9, 15])
