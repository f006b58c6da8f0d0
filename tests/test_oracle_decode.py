"""Pins for the oracle's gist-scored top-k decode (CPU only)."""
import numpy as np
import torch

from oracle import decode as D


def _case(seed, Hq=8, Hkv=2, d=16, cache=512, chunk=16):
    rng = np.random.default_rng(seed)
    G = cache // chunk
    return (rng.standard_normal((Hq, d)), rng.standard_normal((Hkv, G, d)),
            rng.standard_normal((Hkv, G, d)), rng.standard_normal((Hkv, cache, d)),
            rng.standard_normal((Hkv, cache, d)))


def _softmax_attend(q, keys, vals):
    t = lambda x: torch.from_numpy(np.asarray(x, np.float64))
    s = t(keys) @ t(q) / np.sqrt(len(q))
    return (torch.softmax(s, 0) @ t(vals)).numpy(), torch.logsumexp(s, 0).item()


def test_group_scores_match_einsum():
    q, gk, *_ = _case(0)
    s = D.group_scores(q, gk)
    ref = torch.einsum("gcd,gjd->gc", torch.from_numpy(gk),
                       torch.from_numpy(q).reshape(2, 4, 16)).numpy() / 4.0
    np.testing.assert_allclose(s, ref, atol=1e-12)


def test_top_k_ties_go_to_lower_index():
    s = np.array([1.0, 3.0, 2.0, 3.0, 3.0, 0.5])
    elig = np.ones(6, bool)
    assert D.select_top_k(s, elig, 2).tolist() == [1, 3]
    assert D.select_top_k(s, elig, 4).tolist() == [1, 2, 3, 4]
    elig[3] = False
    assert D.select_top_k(s, elig, 2).tolist() == [1, 4]
    assert D.select_top_k(s, np.zeros(6, bool), 2).tolist() == [-1, -1]


def test_eligibility_excludes_window():
    e = D.eligible_chunks(4096, 32, 131072, 512)
    assert e.sum() == 4080 and e[:4080].all() and not e[4080:].any()


def test_all_chunks_selected_equals_dense_attention():
    q, gk, gv, rk, rv = _case(1)
    G = gk.shape[1]
    sel, o, lse, _ = D.decode_one(q, gk, gv, rk, rv, chunk=16, window=64, top_k=G)
    for h in range(8):
        g = h // 4
        keys = np.concatenate([gk[g], rk[g]])
        vals = np.concatenate([gv[g], rv[g]])
        ref_o, ref_l = _softmax_attend(q[h], keys, vals)
        np.testing.assert_allclose(o[h], ref_o, atol=1e-12)
        assert abs(lse[h] - ref_l) < 1e-12


def test_zero_k_is_gists_plus_window():
    q, gk, gv, rk, rv = _case(2)
    sel, o, lse, _ = D.decode_one(q, gk, gv, rk, rv, chunk=16, window=64, top_k=0)
    assert sel.shape == (2, 0)
    for h in range(8):
        g = h // 4
        ref_o, _ = _softmax_attend(q[h], np.concatenate([gk[g], rk[g][-64:]]),
                                   np.concatenate([gv[g], rv[g][-64:]]))
        np.testing.assert_allclose(o[h], ref_o, atol=1e-12)


def test_selection_is_the_best_eligible_set():
    q, gk, gv, rk, rv = _case(3)
    sel, o, lse, scores = D.decode_one(q, gk, gv, rk, rv, chunk=16, window=64, top_k=5)
    for g in range(2):
        elig = np.nonzero(D.eligible_chunks(32, 16, 512, 64))[0]
        best = elig[np.argsort(-scores[g][elig], kind="stable")[:5]]
        assert sel[g].tolist() == sorted(best.tolist())
        pos = D.raw_key_positions(sel[g], 16, 512, 64)
        assert len(np.unique(pos)) == len(pos) == 5 * 16 + 64


def test_gist_kv_is_one_chunk_th_of_raw():
    # one gist key/value per chunk: the scored set is cache_len / chunk rows
    assert D.eligible_chunks(4096, 32, 131072, 0).sum() * 32 == 131072


# ---------------------------------------------------------------- selection variants
def test_prob_scores_sum_to_group_size_and_match_torch_softmax():
    q, gk, *_ = _case(3)
    s = D.group_prob_scores(q, gk)
    np.testing.assert_allclose(s.sum(1), [4.0, 4.0], atol=1e-12)  # 4 heads, each sums to one
    logits = torch.einsum("gcd,ghd->ghc", torch.from_numpy(gk),
                          torch.from_numpy(q).reshape(2, 4, 16)) / 4.0
    np.testing.assert_allclose(s, torch.softmax(logits, -1).sum(1).numpy(), atol=1e-12)


def test_prob_scores_rank_like_logits_for_one_head_per_group():
    # one head per group: a softmax is monotone, so the two rules select the same chunks
    q, gk, *_ = _case(4, Hq=2, Hkv=2)
    elig = np.ones(gk.shape[1], bool)
    for g in range(2):
        assert np.array_equal(D.select_top_k(D.group_prob_scores(q, gk)[g], elig, 7),
                              D.select_top_k(D.group_scores(q, gk)[g], elig, 7))


def test_prob_scores_differ_from_logit_sums_across_heads():
    # head 0 is sharp on chunk 0, head 1 flat but slightly higher on chunk 1:
    # logit sums prefer chunk 1, probability sums chunk 0
    logits = np.array([[10.0, 0.0, 0.0], [0.0, 10.5, 10.4]])
    d = 2
    q = np.eye(d)
    gk = logits.T[None] * np.sqrt(d)  # gist c's key = column c, so q_h . k_c * scale = logits[h, c]
    sl = D.group_scores(q, gk)[0]
    sp = D.group_prob_scores(q, gk)[0]
    assert np.argmax(sl) == 1 and np.argmax(sp) == 0


def test_top_p_closed_form():
    probs = np.array([0.2, 0.5, 0.3])
    s = np.log(probs)
    elig = np.ones(3, bool)
    assert D.select_top_p(s, elig, 3, 0.45).tolist() == [1, -1, -1]
    assert D.select_top_p(s, elig, 3, 0.75).tolist() == [1, 2, -1]
    assert D.select_top_p(s, elig, 3, 0.85).tolist() == [0, 1, 2]
    assert D.select_top_p(s, elig, 2, 0.85).tolist() == [1, 2]  # capped at k
    assert D.select_top_p(s, elig, 3, 1e-9).tolist() == [1, -1, -1]  # never empty
    elig[1] = False  # renormalised over the eligible chunks: 0.2 / 0.5 and 0.3 / 0.5
    assert D.select_top_p(s, elig, 3, 0.55).tolist() == [2, -1, -1]
    assert D.select_top_p(s, elig, 3, 0.65).tolist() == [0, 2, -1]
    assert D.select_top_p(s, np.zeros(3, bool), 2, 0.5).tolist() == [-1, -1]


def test_top_p_is_the_smallest_set_reaching_p_by_brute_force():
    from itertools import combinations
    rng = np.random.default_rng(7)
    for trial in range(40):
        n = 7
        s = rng.standard_normal(n) * 2
        elig = rng.random(n) < 0.8
        p = rng.uniform(0.05, 0.99)
        ids = np.nonzero(elig)[0]
        if len(ids) == 0:
            continue
        prob = np.zeros(n)
        prob[ids] = np.exp(s[ids] - s[ids].max())
        prob /= prob.sum()
        best = None
        for m in range(1, len(ids) + 1):
            sets = [c for c in combinations(ids, m) if prob[list(c)].sum() >= p]
            if sets:
                best = max(sets, key=lambda c: prob[list(c)].sum())
                break
        got = D.select_top_p(s, elig, n, p)
        assert sorted(got[got >= 0].tolist()) == sorted(best), (trial, p)


def test_top_p_one_equals_top_k():
    q, gk, *_ = _case(5)
    s = D.group_scores(q, gk)[1]
    elig = D.eligible_chunks(len(s), 16, 512, 64)
    for k in (1, 5, 20):
        assert np.array_equal(D.select_top_p(s, elig, k, 1.0), D.select_top_k(s, elig, k))


def test_per_head_selection_reduces_to_group_rule_with_one_head_per_group():
    q, gk, gv, rk, rv = _case(6, Hq=2, Hkv=2)
    a = D.decode_one(q, gk, gv, rk, rv, 16, 64, 5, rule=D.PER_HEAD)
    b = D.decode_one(q, gk, gv, rk, rv, 16, 64, 5)
    assert np.array_equal(a[0], b[0])
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


def test_per_head_selection_is_each_heads_best_set_and_its_own_attention():
    q, gk, gv, rk, rv = _case(8)
    sel, o, lse, scores = D.decode_one(q, gk, gv, rk, rv, 16, 64, 6, rule=D.PER_HEAD)
    elig = D.eligible_chunks(32, 16, 512, 64)
    for h in range(8):
        g = h // 4
        s_h = gk[g] @ q[h] / 4.0
        best = np.argsort(-np.where(elig, s_h, -np.inf), kind="stable")[:6]
        assert sorted(best.tolist()) == sel[h].tolist()
        pos = np.concatenate([np.arange(c * 16, c * 16 + 16) for c in sel[h]] + [np.arange(448, 512)])
        ref_o, ref_l = _softmax_attend(q[h], np.concatenate([gk[g], rk[g][pos]]),
                                       np.concatenate([gv[g], rv[g][pos]]))
        np.testing.assert_allclose(o[h], ref_o, atol=1e-12)
        assert abs(lse[h] - ref_l) < 1e-12
    # heads of one group generally pick different chunks
    assert any(not np.array_equal(sel[0], sel[h]) for h in range(1, 4))


# ---------------------------------------------------------------- gist-of-gist
def _hier_case(seed, Hq=8, Hkv=2, d=16, chunk=8, fanout=4, n2=16):
    rng = np.random.default_rng(seed)
    n1 = n2 * fanout
    L = n1 * chunk
    r = lambda *s: rng.standard_normal(s)
    return r(Hq, d), r(Hkv, n2, d), r(Hkv, n2, d), r(Hkv, n1, d), r(Hkv, n1, d), r(Hkv, L, d), r(Hkv, L, d)


def test_hier_selection_with_every_group_unfolded_is_the_flat_selection():
    q, g2k, g2v, g1k, g1v, rk, rv = _hier_case(10)
    window = 64
    sel2, sel1, _, _ = D.hier_decode_one(q, g2k, g2v, g1k, g1v, rk, rv, 8, 4, 16, 9, window)
    flat_sel = D.decode_one(q, g1k, g1v, rk, rv, 8, window, 9)[0]
    assert np.array_equal(sel1, flat_sel)
    elig2 = (np.arange(16) + 1) * 32 <= 512 - window
    assert (sel2 >= 0).sum(1).tolist() == [int(elig2.sum())] * 2


def test_hier_attention_is_one_softmax_over_the_stated_keys():
    q, g2k, g2v, g1k, g1v, rk, rv = _hier_case(11)
    chunk, fanout, k2, k1, window = 8, 4, 3, 5, 40
    sel2, sel1, o, lse = D.hier_decode_one(q, g2k, g2v, g1k, g1v, rk, rv, chunk, fanout, k2, k1, window)
    for g in range(2):
        # the unfolded chunks lie inside the kept groups and are the best of them
        groups = sel2[g][sel2[g] >= 0]
        assert len(groups) == k2 and set(sel1[g] // fanout) <= set(groups)
        cand = np.concatenate([np.arange(c * fanout, (c + 1) * fanout) for c in groups])
        s1 = (g1k[g] @ q[g * 4:(g + 1) * 4].T).sum(1) / 4.0
        assert sorted(cand[np.argsort(-s1[cand], kind="stable")][:k1].tolist()) == sel1[g].tolist()
        raw = np.concatenate([np.arange(c * chunk, (c + 1) * chunk) for c in sel1[g]] +
                             [np.arange(512 - window, 512)])
        keys = np.concatenate([g2k[g], g1k[g][cand], rk[g][raw]])
        vals = np.concatenate([g2v[g], g1v[g][cand], rv[g][raw]])
        assert len(keys) == D.hier_key_counts(16, fanout, chunk, k2, k1, window)
        for h in range(g * 4, (g + 1) * 4):
            ref_o, ref_l = _softmax_attend(q[h], keys, vals)
            np.testing.assert_allclose(o[h], ref_o, atol=1e-12)
            assert abs(lse[h] - ref_l) < 1e-12


def test_hier_key_count_is_logarithmic_against_flat():
    # 128K cache, 32-token chunks, 32 chunk gists per group: 128 level-2 gists
    assert D.hier_key_counts(128, 32, 32, 8, 64, 512) == 128 + 256 + 2048 + 512
    assert 4096 + 64 * 32 + 512 == 6656  # the flat selection over the same cache
