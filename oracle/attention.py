"""Masked softmax attention and its gradients in float64 (oracle; test
infrastructure only).

The computation is the plain definition of attention restricted to a mask:
"Gzip-guided sparse attention: Selecting long-range content by
compressibility" (Core equations: the mask M selects which key blocks a query
block attends; Scope: the reproduction computes dense scores and then masks),
with FlashAttention named as the building block on the UniGist summary page
("UniGist: ...", Builds on). Readings (not printed on the pages): scores are
q.k / sqrt(d); LSE is the natural-log log-sum-exp of the masked scores.

For one head: s = (q k^T) * scale with disallowed pairs removed,
LSE_p = log sum_q exp(s_pq), P = exp(s - LSE), O = P V.
Gradients for a loss with upstream dO:
dV = P^T dO, dP = dO V^T, D_p = sum_c dO_pc O_pc, dS = P * (dP - D),
dQ = dS K * scale, dK = dS^T Q * scale.

Long inputs are processed in chunks of query rows; every query row is
independent, so chunking only changes the order in which dK and dV sum over
rows.
"""
from __future__ import annotations

import numpy as np


def _mask_rows(mask, r0, r1):
    if callable(mask):
        return np.asarray(mask(np.arange(r0, r1)), dtype=bool)
    return np.asarray(mask[r0:r1], dtype=bool)


def _scores(q, k, allowed, scale):
    s = (q @ k.T) * scale
    if not allowed.any(axis=1).all():
        raise ValueError("a query row has no allowed key")
    return np.where(allowed, s, -np.inf)


def forward(q, k, v, mask, scale=None, row_chunk=2048):
    """O [Nq, dv] and LSE [Nq] for one head.

    q [Nq, d], k [Nk, d], v [Nk, dv]; ``mask`` is a bool [Nq, Nk] array or a
    callable rows -> bool [len(rows), Nk].
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    Nq = q.shape[0]
    o = np.empty((Nq, v.shape[1]), np.float64)
    lse = np.empty(Nq, np.float64)
    for r0 in range(0, Nq, row_chunk):
        r1 = min(Nq, r0 + row_chunk)
        s = _scores(q[r0:r1], k, _mask_rows(mask, r0, r1), scale)
        m = s.max(axis=1, keepdims=True)
        lse_c = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
        p = np.exp(s - lse_c[:, None])
        o[r0:r1] = p @ v
        lse[r0:r1] = lse_c
    return o, lse


def probabilities(q, k, mask, scale=None):
    """The full softmax matrix P [Nq, Nk] (small inputs only)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    s = _scores(q, k, _mask_rows(mask, 0, q.shape[0]), scale)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)


def backward(q, k, v, do, mask, scale=None, row_chunk=2048):
    """(dQ, dK, dV, O, LSE) for one head, float64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    Nq = q.shape[0]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.empty((Nq, v.shape[1]), np.float64)
    lse = np.empty(Nq, np.float64)
    for r0 in range(0, Nq, row_chunk):
        r1 = min(Nq, r0 + row_chunk)
        s = _scores(q[r0:r1], k, _mask_rows(mask, r0, r1), scale)
        m = s.max(axis=1, keepdims=True)
        lse_c = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
        p = np.exp(s - lse_c[:, None])
        o_c = p @ v
        do_c = do[r0:r1]
        dv += p.T @ do_c
        dp = do_c @ v.T
        D = (do_c * o_c).sum(axis=1)
        ds = p * (dp - D[:, None])
        dq[r0:r1] = (ds @ k) * scale
        dk += (ds.T @ q[r0:r1]) * scale
        o[r0:r1] = o_c
        lse[r0:r1] = lse_c
    return dq, dk, dv, o, lse


def forward_rows(q, k, v, keys_of_row, rows, scale=None):
    """O and LSE for selected query rows only, each row over its own key set.

    ``keys_of_row(p)`` returns the indices of the keys row p may attend; this
    is the same definition evaluated one row at a time, for spot checks of
    inputs too large to materialise.
    """
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    o = np.empty((len(rows), v.shape[1]), np.float64)
    lse = np.empty(len(rows), np.float64)
    for n, p in enumerate(rows):
        keys = np.asarray(keys_of_row(int(p)))
        if keys.size == 0:
            raise ValueError("a query row has no allowed key")
        s = (np.asarray(k[keys], np.float64) @ np.asarray(q[p], np.float64)) * scale
        m = s.max()
        l = np.log(np.exp(s - m).sum()) + m
        o[n] = np.exp(s - l) @ np.asarray(v[keys], np.float64)
        lse[n] = l
    return o, lse


def _row_terms(q, k, v, do, keys, p, scale):
    """Softmax row p over `keys`: (P, O_p, D_p) in float64."""
    kk = np.asarray(k[keys], np.float64)
    s = (kk @ np.asarray(q[p], np.float64)) * scale
    m = s.max()
    P = np.exp(s - (m + np.log(np.exp(s - m).sum())))
    o = P @ np.asarray(v[keys], np.float64)
    return P, o, float(np.asarray(do[p], np.float64) @ o)


def backward_rows(q, k, v, do, keys_of_row, rows, scale=None):
    """dQ for selected query rows only: dQ_p = sum_j dS_pj k_j * scale with
    dS_pj = P_pj (dO_p . v_j - D_p) over the keys row p may attend."""
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    out = np.empty((len(rows), k.shape[1]), np.float64)
    for n, p in enumerate(rows):
        keys = np.asarray(keys_of_row(int(p)))
        P, _, D = _row_terms(q, k, v, do, keys, p, scale)
        dP = np.asarray(v[keys], np.float64) @ np.asarray(do[p], np.float64)
        out[n] = ((P * (dP - D)) @ np.asarray(k[keys], np.float64)) * scale
    return out


def backward_cols(q, k, v, do, keys_of_row, rows_of_key, cols, scale=None):
    """dK and dV for selected keys only: sums over the query rows that attend
    key j of dS_pj q_p * scale and P_pj dO_p."""
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    dk = np.zeros((len(cols), k.shape[1]))
    dv = np.zeros((len(cols), v.shape[1]))
    vj_all = np.asarray(v, np.float64)
    for n, j in enumerate(cols):
        for p in rows_of_key(int(j)):
            keys = np.asarray(keys_of_row(int(p)))
            P, _, D = _row_terms(q, k, v, do, keys, p, scale)
            pj = P[np.searchsorted(keys, j)]
            dop = np.asarray(do[p], np.float64)
            ds = pj * (dop @ vj_all[j] - D)
            dk[n] += ds * np.asarray(q[p], np.float64) * scale
            dv[n] += pj * dop
    return dk, dv


def backward_cols_chunked(q, k, v, do, mask, rows, cols, scale=None, row_chunk=256):
    """dK and dV for selected keys only, by whole chunks of query rows.

    The same sums as ``backward_cols`` (over the query rows p that attend key
    j: dS_pj q_p * scale and P_pj dO_p), evaluated a chunk of rows at a time:
    each row's softmax is taken over its own allowed keys, restricted to the
    union of the chunk's keys (a key no row of the chunk may attend adds
    nothing). ``rows`` must hold every query row that attends any of ``cols``
    (extra rows add zero); ``mask`` is a callable rows -> bool [len(rows), Nk].
    """
    q = np.asarray(q, np.float64)
    scale = 1.0 / np.sqrt(q.shape[1]) if scale is None else float(scale)
    cols = np.asarray(cols)
    rows = np.asarray(rows)
    vc = np.asarray(v[cols], np.float64)
    dk = np.zeros((len(cols), k.shape[1]))
    dv = np.zeros((len(cols), v.shape[1]))
    for r0 in range(0, len(rows), row_chunk):
        rr = rows[r0:r0 + row_chunk]
        allowed = np.asarray(mask(rr), dtype=bool)
        keys = np.nonzero(allowed.any(axis=0))[0]
        qc = q[rr]
        doc = np.asarray(do[rr], np.float64)
        s = _scores(qc, np.asarray(k[keys], np.float64), allowed[:, keys], scale)
        m = s.max(axis=1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
        p = np.exp(s - lse[:, None])
        D = (doc * (p @ np.asarray(v[keys], np.float64))).sum(axis=1)
        at = np.searchsorted(keys, cols)
        seen = (at < len(keys)) & (keys[np.minimum(at, len(keys) - 1)] == cols)
        pc = np.where(seen[None, :], p[:, np.minimum(at, len(keys) - 1)], 0.0)
        ds = pc * (doc @ vc.T - D[:, None])
        dk += (ds.T @ qc) * scale
        dv += pc.T @ doc
    return dk, dv
