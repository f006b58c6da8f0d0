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
