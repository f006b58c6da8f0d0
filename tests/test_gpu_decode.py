"""sa_gist_decode vs the oracle: the selected chunks (exact, except where the
oracle's k-th and (k+1)-th scores are closer than float32 accumulation can
resolve), and O / LSE over the selected key set.

Near ties: the kernel accumulates each score in fp32 (tensor-core dot products
over d = 128, summed over the group's heads). Its error is bounded by
2 * d * 2^-24 * scale * sum_h sum_i |q_hi * k_ci| per chunk c; when the
oracle's boundary scores are closer than the sum of their two bounds, either
choice is correct and O is checked against the oracle on the kernel's set."""
import numpy as np
import pytest
import torch
from concurrent.futures import ThreadPoolExecutor

import sa_workloads as W
from oracle import decode as D

from _cases import check_close, to_np

pytestmark = pytest.mark.gpu


def upload_workload(w):
    """Device tensors [n_seq, Hkv, L, d] for raw K/V, [n_seq, Hkv, G, d] gists."""
    n, Hkv, L, d = w["n_seq"], w["kv_heads"], w["cache_len"], w["head_dim"]
    kc = torch.empty(n, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.empty_like(kc)

    def one(i):
        s, g = divmod(i, Hkv)
        return i, W.decode_raw(w, s, g, "k"), W.decode_raw(w, s, g, "v")

    with ThreadPoolExecutor(8) as ex:
        for i, rk, rv in ex.map(one, range(n * Hkv)):
            s, g = divmod(i, Hkv)
            kc[s, g] = torch.from_numpy(rk).to("cuda", torch.bfloat16)
            vc[s, g] = torch.from_numpy(rv).to("cuda", torch.bfloat16)
    gk = np.stack([W.decode_gists(w, s, "k") for s in range(n)])
    gv = np.stack([W.decode_gists(w, s, "v") for s in range(n)])
    q = W.decode_query(w)
    dev = lambda x: torch.from_numpy(x).to("cuda", torch.bfloat16)
    return q, gk, gv, dev(q), dev(gk), dev(gv), kc, vc


def logit_bound(q, gk, s, g, rep, d, heads=None):
    """Float32 accumulation bound of each chunk's summed logit (see above),
    over the group's heads or the given ones."""
    hs = range(g * rep, (g + 1) * rep) if heads is None else heads
    qg = np.abs(q[s, list(hs)].astype(np.float64))
    return lambda c: 2 * d * 2.0 ** -24 / np.sqrt(d) * (qg @ np.abs(gk[s, g, c])).sum()


def valid_alternative(w, rule, top_p, q, gk, s, x, got, want_scores):
    """Is the kernel's selection `got` (ascending, -1 padded) one the rule
    admits given float32 near ties? Sum of logits / of probabilities: a top-k
    set whose boundary scores are within their rounding bounds. Top-p: a
    score-ordered prefix (up to the same near ties) that reaches p and is
    shortest, each up to 1e-4 of probability."""
    d, rep = w["head_dim"], w["heads"] // w["kv_heads"]
    # x is the KV group, or the query head under the per-head rule
    g, heads = (x // rep, [x]) if rule == D.PER_HEAD else (x, None)
    elig = D.eligible_chunks(w["n_gists"], w["chunk"], w["cache_len"], w["window"])
    K = got[got >= 0]
    assert elig[K].all() and len(set(K.tolist())) == len(K)
    sc = np.where(elig, want_scores, -np.inf)
    if rule == D.SUM_PROBS:
        # a probability moves by about p * (its logit error + the normaliser's)
        b = logit_bound(q, gk, s, g, rep, d)
        bound = lambda c: want_scores[c] * (b(c) + 1e-5)
    else:
        bound = logit_bound(q, gk, s, g, rep, d, heads)
    rest = np.setdiff1d(np.nonzero(elig)[0], K)
    if len(K) and len(rest):
        c_in = K[np.argmin(sc[K])]
        c_out = rest[np.argmax(sc[rest])]
        assert sc[c_out] - sc[c_in] <= bound(c_in) + bound(c_out), (s, g, sc[c_in], sc[c_out])
    n_el = int(elig.sum())
    if rule != D.TOP_P:
        assert len(K) == min(w["top_k"], n_el)
        return
    if n_el == 0 or w["top_k"] == 0:
        assert len(K) == 0
        return
    e = np.exp(sc[elig] - sc[elig].max())
    prob = np.zeros(len(sc))
    prob[elig] = e / e.sum()
    assert 1 <= len(K) <= w["top_k"]
    if len(K) < min(w["top_k"], n_el):
        assert prob[K].sum() >= top_p - 1e-4
    shorter = np.delete(K, np.argmin(sc[K]))
    assert prob[shorter].sum() < top_p + 1e-4


def check(sa, w, seqs=None, rule=0, top_p=1.0, edit=None, exact=()):
    """edit(q, gk) may change the gist keys in place before the run; `exact`
    lists (sequence, group) pairs whose selection must equal the oracle's
    exactly (no near-tie allowance)."""
    q, gk, gv, tq, tgk, tgv, kc, vc = upload_workload(w)
    if edit is not None:
        edit(q, gk)
        tgk.copy_(torch.from_numpy(gk).to(torch.bfloat16))
        gk = tgk.float().cpu().numpy()  # the oracle sees the same bf16 gists
    sel, o, lse = sa.gist_decode(tq, tgk, tgv, kc, vc, w["chunk"], w["top_k"], w["window"],
                                 select_rule=rule, top_p=top_p)
    torch.cuda.synchronize()
    ws = sa.gist_decode.last_workspace
    st = ws[:8].view(torch.int32).cpu().tolist()
    assert st[0] == 0, f"device status {st[0]} at {st[1]}"
    sel, o, lse = sel.cpu().numpy(), to_np(o), to_np(lse)
    rep = w["heads"] // w["kv_heads"]
    for s in (range(w["n_seq"]) if seqs is None else seqs):
        raw_k = lambda g: to_np(kc[s, g])
        raw_v = lambda g: to_np(vc[s, g])
        osel, oo, ol, scores = D.decode_one(q[s], gk[s], gv[s], raw_k, raw_v, w["chunk"],
                                            w["window"], w["top_k"], rule=rule, top_p=top_p)
        per_head = rule == D.PER_HEAD
        for x in range(w["heads"] if per_head else w["kv_heads"]):
            if (s, x) in exact:
                np.testing.assert_array_equal(sel[s, x], osel[x], err_msg=f"seq {s} group {x}")
            if not np.array_equal(sel[s, x], osel[x]):
                # accept a different set only where float32 rounding can decide it
                valid_alternative(w, rule, top_p, q, gk, s, x, sel[s, x], scores[x])
                g = x // rep if per_head else x
                # O must then match the oracle evaluated on the GPU's own set
                pos = D.raw_key_positions(sel[s, x], w["chunk"], w["cache_len"], w["window"])
                keys = np.concatenate([gk[s, g], raw_k(g)[pos]])
                vals = np.concatenate([gv[s, g], raw_v(g)[pos]])
                for h in ([x] if per_head else range(g * rep, (g + 1) * rep)):
                    oo[h], ol[h] = D.attend(q[s, h], keys, vals, 1 / np.sqrt(w["head_dim"]))
        check_close(o[s], oo, "bf16", f"O seq {s}")
        check_close(lse[s], ol, "bf16", f"LSE seq {s}")


@pytest.mark.parametrize("top_k,window,chunk,G", [(8, 64, 16, 64), (0, 64, 16, 64), (60, 64, 16, 64),
                                                  (5, 0, 32, 40), (3, 100, 8, 300)])
def test_decode_small(sa, top_k, window, chunk, G):
    w = W.scaled("gist_decode_128k", index=400 + top_k + G, n_seq=3, cache_len=chunk * G,
                 chunk=chunk, n_gists=G, top_k=top_k, window=window, heads=8, kv_heads=2)
    check(sa, w)


@pytest.mark.parametrize("rep", [1, 8])
def test_decode_group_sizes(sa, rep):
    w = W.scaled("gist_decode_128k", index=450 + rep, n_seq=2, cache_len=32 * 128, chunk=32,
                 n_gists=128, top_k=16, window=128, heads=2 * rep, kv_heads=2)
    check(sa, w)


def test_decode_full_size(sa):
    check(sa, W.WORKLOADS["gist_decode_128k"], seqs=[0, 7, 15])


@pytest.mark.parametrize("top_k,window,chunk,G", [
    (0, 256, 16, 256),     # nothing unfolded
    (40, 0, 32, 256),      # no window: chunk blocks follow the gist blocks
    (256, 128, 8, 200),    # fewer eligible chunks than top_k: -1 padding
    (17, 1000, 128, 130),  # one chunk per block, ragged window and gist blocks
    (33, 300, 64, 777),    # two chunks per block, ragged everywhere
])
def test_decode_tensor_core_shapes(sa, top_k, window, chunk, G):
    """Shapes of the one-CTA-per-(sequence, KV head) tensor-core kernel
    (G >= 128, 8 <= chunk <= 128 dividing 128)."""
    w = W.scaled("gist_decode_128k", index=500 + top_k + G, n_seq=2, cache_len=chunk * G,
                 chunk=chunk, n_gists=G, top_k=top_k, window=window, heads=8, kv_heads=2)
    check(sa, w)


RULES = {"sum_probs": (1, 1.0), "top_p_0.3": (2, 0.3), "top_p_0.9": (2, 0.9), "top_p_1": (2, 1.0),
         "per_head": (3, 1.0)}


@pytest.mark.parametrize("rule", list(RULES))
@pytest.mark.parametrize("top_k,window,chunk,G", [(8, 64, 16, 64), (60, 64, 16, 64), (5, 0, 32, 40),
                                                  (40, 0, 32, 256), (256, 128, 8, 200),
                                                  (33, 300, 64, 777)])
def test_decode_select_rules(sa, rule, top_k, window, chunk, G):
    """Sum-of-probabilities and top-p selection on both kernels (G < 128 or a
    chunk of 16 with 64 gists takes the CUDA-core path, the rest the tensor cores)."""
    w = W.scaled("gist_decode_128k", index=600 + top_k + G, n_seq=2, cache_len=chunk * G,
                 chunk=chunk, n_gists=G, top_k=top_k, window=window, heads=8, kv_heads=2)
    r, p = RULES[rule]
    check(sa, w, rule=r, top_p=p)


@pytest.mark.parametrize("rep", [1, 8])
def test_decode_per_head_group_sizes(sa, rep):
    """Per-head selection with one and eight query heads per KV head; with
    eight, 8 * top_k = 256 unfolded slots is the tensor-core kernel's limit."""
    w = W.scaled("gist_decode_128k", index=650 + rep, n_seq=2, cache_len=32 * 256, chunk=32,
                 n_gists=256, top_k=32, window=128, heads=2 * rep, kv_heads=2)
    check(sa, w, rule=3)


def test_decode_per_head_past_the_union_limit(sa):
    """8 heads per group x top_k 40 > 256 slots: the CUDA-core kernels take it."""
    w = W.scaled("gist_decode_128k", index=660, n_seq=1, cache_len=16 * 512, chunk=16,
                 n_gists=512, top_k=40, window=64, heads=16, kv_heads=2)
    check(sa, w, rule=3)


@pytest.mark.parametrize("rule", ["sum_probs", "top_p_0.9", "per_head"])
def test_decode_select_rules_full_size(sa, rule):
    r, p = RULES[rule]
    check(sa, W.WORKLOADS["gist_decode_128k"], seqs=[0, 15], rule=r, top_p=p)


@pytest.mark.parametrize("top_k,G,chunk", [(64, 1024, 32), (1, 1500, 16), (128, 3000, 32), (129, 2000, 16)])
def test_decode_list_selection_shapes(sa, top_k, G, chunk):
    """8 to 32 candidates per thread: the selection ranks a short candidate list
    (ragged last thread at G = 1500 and 3000; k = 1 and k = 128, the list's
    limits); k = 129 takes the radix passes."""
    w = W.scaled("gist_decode_128k", index=700 + top_k + G, n_seq=2, cache_len=chunk * G,
                 chunk=chunk, n_gists=G, top_k=top_k, window=256, heads=8, kv_heads=2)
    check(sa, w)
    if top_k <= 128:
        check(sa, w, rule=3)  # per head: one list selection per query head


def _tie_edit(w, groups, rank, copies, seed):
    """Copy the gist of the eligible chunk ranked `rank` (sum of logits) into
    `copies` other eligible chunks of each listed (sequence, group): the
    selection boundary then falls inside a run of exactly equal scores, which
    both sides break toward the lower index."""
    def edit(q, gk):
        rng = np.random.default_rng(seed)
        rep = w["heads"] // w["kv_heads"]
        elig = np.nonzero(D.eligible_chunks(w["n_gists"], w["chunk"], w["cache_len"], w["window"]))[0]
        for s, g in groups:
            gb = gk[s, g].astype(np.float32)
            sc = (q[s, g * rep:(g + 1) * rep].astype(np.float64) @ gb.T.astype(np.float64)).sum(0)
            order = elig[np.argsort(-sc[elig], kind="stable")]
            src = order[rank]
            dst = rng.choice(np.setdiff1d(elig, [src]), copies, replace=False)
            gk[s, g, dst] = gk[s, g, src]
    return edit


def test_decode_exact_ties_inside_the_list(sa):
    """k = 64 with 40 copies of the 50th best gist: the list path takes the
    lowest-index copies that fit, as the oracle does."""
    w = W.scaled("gist_decode_128k", index=720, n_seq=1)
    groups = [(0, 0), (0, 5)]
    check(sa, w, edit=_tie_edit(w, groups, 50, 40, 1), exact=groups)


def test_decode_exact_ties_past_the_list(sa):
    """3000 copies of one gist: more than 128 keys reach the thread-maximum
    bound, so the radix passes decide, with the same ties to the lower index."""
    w = W.scaled("gist_decode_128k", index=721, n_seq=1)
    groups = [(0, 2)]
    check(sa, w, edit=_tie_edit(w, groups, 10, 3000, 2), exact=groups)
