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
