"""Gist-scored selective unfolding at decode (oracle; test infrastructure only).

Source: "Simplified Sparse Attention via Gist Tokens" (abstract: chunks are
scored by attention between the current query and the gist tokens only, the
top-k chunks are unfolded by bringing back their raw tokens) and "Forget, Then
Recall: Learnable Compression and Selective Unfolding via Gist Sparse
Attention" (abstract: compress into gists, select the most relevant gists,
restore the corresponding raw chunks for detailed attention). The record of
the first page also names a per-group selection routine.

Readings taken where the pages are silent:
* one gist key/value per chunk of ``chunk`` raw tokens; selection is shared by
  the query heads of one KV group and scores a chunk by the SUM over the
  group's heads of q_h . k_gist / sqrt(d);
* chunks that lie entirely before the local window are eligible; the others
  are covered by the window;
* top-k keeps the k highest scores, ties going to the lower chunk index; the
  result is reported as the ascending set of chunk indices (-1 padded when
  fewer than k chunks are eligible);
* every head attends over all gists of its group, the raw tokens of the
  selected chunks and the last ``window`` raw tokens, with one softmax.

Selection variants (the first page's record names a top-p routine next to the
top-k one; the pages give nothing more):
* sum of probabilities: each query head's softmax over all gists of its
  group (the attention it would pay to the gists alone), summed over the
  group's heads, ranks the chunks; top-k as above;
* per query head: every query head ranks the chunks by its own q_h . k_gist
  * scale and unfolds its own top-k; it attends over the gists, its own
  chunks and the window (the selection is reported per query head);
* top-p: the group scores (sum of logits) are turned into probabilities by a
  softmax over the eligible chunks; taking chunks in score order (ties to the
  lower index), the smallest prefix whose probability reaches p is kept, at
  most k chunks.
"""
from __future__ import annotations

import numpy as np


def group_scores(q, gist_k, scale=None) -> np.ndarray:
    """s[g, c] = sum over q heads h of group g of q_h . gist_k[g, c] * scale.

    q [Hq, d]; gist_k [Hkv, G, d]; q head h belongs to group h // (Hq/Hkv).
    """
    q = np.asarray(q, np.float64)
    gk = np.asarray(gist_k, np.float64)
    Hq, d = q.shape
    Hkv = gk.shape[0]
    rep = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.zeros((Hkv, gk.shape[1]))
    for h in range(Hq):
        out[h // rep] += (gk[h // rep] @ q[h]) * scale
    return out


def group_prob_scores(q, gist_k, scale=None) -> np.ndarray:
    """s[g, c] = sum over q heads h of group g of softmax_c(q_h . gist_k[g, c] * scale),
    each head's softmax taken over all the group's gists."""
    q = np.asarray(q, np.float64)
    gk = np.asarray(gist_k, np.float64)
    Hq, d = q.shape
    Hkv = gk.shape[0]
    rep = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.zeros((Hkv, gk.shape[1]))
    for h in range(Hq):
        logits = (gk[h // rep] @ q[h]) * scale
        e = np.exp(logits - logits.max())
        out[h // rep] += e / e.sum()
    return out


def eligible_chunks(n_gists: int, chunk: int, cache_len: int, window: int) -> np.ndarray:
    """Chunks whose raw tokens all lie before the last ``window`` positions."""
    c = np.arange(n_gists)
    return (c + 1) * chunk <= cache_len - window


def select_top_k(scores, eligible, k: int) -> np.ndarray:
    """Ascending indices of the k best eligible chunks (score descending,
    ties to the lower index), padded with -1 to length k."""
    idx = [c for c in range(len(scores)) if eligible[c]]
    idx.sort(key=lambda c: (-float(scores[c]), c))
    chosen = sorted(idx[:k])
    return np.asarray(chosen + [-1] * (k - len(chosen)), dtype=np.int32)


def select_top_p(scores, eligible, k: int, p: float) -> np.ndarray:
    """Ascending indices of the smallest score-ordered prefix of the eligible
    chunks whose softmax probability (over the eligible chunks) reaches p, at
    most k of them; padded with -1 to length k."""
    idx = [c for c in range(len(scores)) if eligible[c]]
    idx.sort(key=lambda c: (-float(scores[c]), c))
    chosen = []
    if idx:
        s = np.asarray([scores[c] for c in idx], np.float64)
        prob = np.exp(s - s.max())
        prob /= prob.sum()
        cum = 0.0
        for c, pc in zip(idx[:k], prob[:k]):
            if chosen and cum >= p:
                break
            chosen.append(c)
            cum += pc
    chosen = sorted(chosen)
    return np.asarray(chosen + [-1] * (k - len(chosen)), dtype=np.int32)


def raw_key_positions(sel, chunk: int, cache_len: int, window: int) -> np.ndarray:
    """Raw cache positions attended: the selected chunks, then the window."""
    pos = [np.arange(c * chunk, (c + 1) * chunk) for c in sel if c >= 0]
    pos.append(np.arange(max(0, cache_len - window), cache_len))
    return np.concatenate(pos)


def attend(qh, keys, values, scale):
    s = (np.asarray(keys, np.float64) @ np.asarray(qh, np.float64)) * scale
    m = s.max()
    lse = m + np.log(np.exp(s - m).sum())
    return np.exp(s - lse) @ np.asarray(values, np.float64), lse


SUM_LOGITS, SUM_PROBS, TOP_P, PER_HEAD = 0, 1, 2, 3


def decode_one(q, gist_k, gist_v, raw_k, raw_v, chunk, window, top_k, scale=None,
               rule=SUM_LOGITS, top_p=1.0):
    """One sequence. ``rule``: SUM_LOGITS (top-k of the summed logits),
    SUM_PROBS (top-k of the summed per-head probabilities), TOP_P (top-p of
    the summed logits, at most top_k chunks) or PER_HEAD (each query head's
    own top-k; then sel is [Hq, top_k] and scores [Hq, G]).

    q [Hq, d]; gist_k/gist_v [Hkv, G, d]; raw_k/raw_v: callables
    (kv_head) -> [cache_len, d] (or arrays [Hkv, cache_len, d]).
    Returns (sel [Hkv, top_k] int32, o [Hq, d], lse [Hq]).
    """
    q = np.asarray(q, np.float64)
    Hq, d = q.shape
    Hkv, G, _ = np.shape(gist_k)
    rep = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    get_k = raw_k if callable(raw_k) else (lambda g: raw_k[g])
    get_v = raw_v if callable(raw_v) else (lambda g: raw_v[g])
    scores = group_prob_scores(q, gist_k, scale) if rule == SUM_PROBS else group_scores(q, gist_k, scale)
    sel = np.empty((Hkv, top_k), np.int32)
    o = np.empty((Hq, d))
    lse = np.empty(Hq)
    if rule == PER_HEAD:
        # one selection per query head, from that head's own logits
        scores = np.stack([(np.asarray(gist_k[h // rep], np.float64) @ q[h]) * scale
                           for h in range(Hq)])
        sel = np.empty((Hq, top_k), np.int32)
        for h in range(Hq):
            rk, rv = get_k(h // rep), get_v(h // rep)
            cache_len = rk.shape[0]
            sel[h] = select_top_k(scores[h], eligible_chunks(G, chunk, cache_len, window), top_k)
            pos = raw_key_positions(sel[h], chunk, cache_len, window)
            keys = np.concatenate([np.asarray(gist_k[h // rep], np.float64),
                                   np.asarray(rk[pos], np.float64)])
            vals = np.concatenate([np.asarray(gist_v[h // rep], np.float64),
                                   np.asarray(rv[pos], np.float64)])
            o[h], lse[h] = attend(q[h], keys, vals, scale)
        return sel, o, lse, scores
    for g in range(Hkv):
        rk, rv = get_k(g), get_v(g)
        cache_len = rk.shape[0]
        elig = eligible_chunks(G, chunk, cache_len, window)
        sel[g] = (select_top_p(scores[g], elig, top_k, top_p) if rule == TOP_P
                  else select_top_k(scores[g], elig, top_k))
        pos = raw_key_positions(sel[g], chunk, cache_len, window)
        keys = np.concatenate([np.asarray(gist_k[g], np.float64), np.asarray(rk[pos], np.float64)])
        vals = np.concatenate([np.asarray(gist_v[g], np.float64), np.asarray(rv[pos], np.float64)])
        for h in range(g * rep, (g + 1) * rep):
            o[h], lse[h] = attend(q[h], keys, vals, scale)
    return sel, o, lse, scores


# ---------------------------------------------------------------- gist-of-gist
# "Forget, Then Recall: ... Gist Sparse Attention" (abstract) and "Simplified
# Sparse Attention via Gist Tokens" (abstract) extend the selection
# hierarchically: gists of gists give multi-resolution access with a
# logarithmic per-step cost. The pages give no more; the readings taken:
# * level 1 is the chunk gists above (one per `chunk` raw tokens); level 2 has
#   one gist per `fanout` consecutive level-1 gists (a "group");
# * a group is eligible iff all of its raw tokens lie before the window;
# * step 1 scores every level-2 gist with the group's summed logits and keeps
#   the top k2 eligible groups; step 2 scores the level-1 gists of those groups
#   the same way and keeps the top k1 of them; ties go to the lower index;
# * every head attends, in one softmax, over all level-2 gists, the level-1
#   gists of the kept groups, the raw tokens of the kept chunks and the last
#   `window` raw tokens. Deeper hierarchies repeat step 1 per level.
def hier_key_counts(n2: int, fanout: int, chunk: int, k2: int, k1: int, window: int) -> int:
    """Keys one head attends when every selection is full."""
    return n2 + k2 * fanout + k1 * chunk + window


def hier_decode_one(q, g2k, g2v, g1k, g1v, raw_k, raw_v, chunk, fanout, k2, k1, window,
                    scale=None):
    """One sequence. q [Hq, d]; g2k/g2v [Hkv, n2, d]; g1k/g1v [Hkv, n1, d]
    (n1 = n2 * fanout); raw_k/raw_v callables (kv head) -> [cache_len, d] or
    arrays. Returns (sel2 [Hkv, k2], sel1 [Hkv, k1] chunk indices, o, lse)."""
    q = np.asarray(q, np.float64)
    Hq, d = q.shape
    Hkv, n2, _ = np.shape(g2k)
    n1 = np.shape(g1k)[1]
    assert n1 == n2 * fanout
    rep = Hq // Hkv
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    get_k = raw_k if callable(raw_k) else (lambda g: raw_k[g])
    get_v = raw_v if callable(raw_v) else (lambda g: raw_v[g])
    s2 = group_scores(q, g2k, scale)
    s1 = group_scores(q, g1k, scale)
    sel2 = np.empty((Hkv, k2), np.int32)
    sel1 = np.empty((Hkv, k1), np.int32)
    o = np.empty((Hq, d))
    lse = np.empty(Hq)
    for g in range(Hkv):
        rk, rv = get_k(g), get_v(g)
        cache_len = rk.shape[0]
        elig2 = (np.arange(n2) + 1) * fanout * chunk <= cache_len - window
        sel2[g] = select_top_k(s2[g], elig2, k2)
        groups = [c for c in sel2[g] if c >= 0]
        cand = np.zeros(n1, bool)
        for c in groups:
            cand[c * fanout:(c + 1) * fanout] = True
        sel1[g] = select_top_k(s1[g], cand, k1)
        pos = raw_key_positions(sel1[g], chunk, cache_len, window)
        lvl1 = np.nonzero(cand)[0]
        keys = np.concatenate([np.asarray(g2k[g], np.float64), np.asarray(g1k[g], np.float64)[lvl1],
                               np.asarray(rk[pos], np.float64)])
        vals = np.concatenate([np.asarray(g2v[g], np.float64), np.asarray(g1v[g], np.float64)[lvl1],
                               np.asarray(rv[pos], np.float64)])
        for h in range(g * rep, (g + 1) * rep):
            o[h], lse[h] = attend(q[h], keys, vals, scale)
    return sel2, sel1, o, lse
