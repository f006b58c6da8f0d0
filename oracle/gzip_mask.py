"""Gzip-guided block masks (oracle; test infrastructure only).

Source: "Gzip-guided sparse attention: Selecting long-range content by
compressibility" (reproduction write-up), sections "Background and main
changes" (head split), the flowchart, and "Core equations" (the ratio/flag
equation, the mask equation and the O(L^2 + Nw) edge count).
"""
from __future__ import annotations

import zlib

import numpy as np

LOCAL, LITERAL, HYBRID = 0, 1, 2
CLASS_NAMES = ("local", "literal", "hybrid")


def block_compressed_sizes(x: bytes, b: int, compress=None) -> list[int]:
    """|gzip(x_{ib:(i+1)b})| for every block i (Core equations, ratio r_i).

    The bytes are cut into B = N/b fixed blocks and each block is compressed
    on its own at level 1 (flowchart: "fixed-size blocks" -> "gzip level-1
    per block"). Reading: zlib level 1 is the deflate implementation; the
    container (zlib, gzip or raw deflate) adds the same number of bytes to
    every block, which cannot change a comparison against the mean (pinned by
    a test). ``compress`` lets a test swap in another container.
    """
    if len(x) % b:
        raise ValueError("byte length must be a multiple of the block size")
    comp = compress or (lambda blk: zlib.compress(blk, 1))
    return [len(comp(bytes(x[i:i + b]))) for i in range(0, len(x), b)]


def literal_flags_from_sizes(sizes) -> np.ndarray:
    """l_i = 1[r_i > mean(r)] with r_i = c_i / b (Core equations).

    Since r_i = c_i/b and mean(r) = (1/B) sum_j c_j / b, the test r_i > mean(r)
    is exactly c_i * B > sum_j c_j; it is evaluated in Python integers so no
    rounding can move a block across the mean. Strict '>' as printed, so a
    block exactly at the mean is not literal and equal sizes give no literals.
    """
    c = [int(v) for v in sizes]
    B, total = len(c), sum(c)
    return np.array([1 if ci * B > total else 0 for ci in c], dtype=np.uint8)


def literal_flags(x: bytes, b: int) -> np.ndarray:
    return literal_flags_from_sizes(block_compressed_sizes(x, b))


def head_classes(H: int) -> list[int]:
    """Per-head mask class (Background and main changes: 50% local only, 25%
    literal-long-range only, 25% both).

    Reading for H not divisible by 4: floor(H/2) local heads first, then
    floor(H/4) literal heads, the rest hybrid.
    """
    n_loc, n_lit = H // 2, H // 4
    return [LOCAL] * n_loc + [LITERAL] * n_lit + [HYBRID] * (H - n_loc - n_lit)


def block_masks(flags, w: int) -> dict[int, np.ndarray]:
    """The three block masks over B blocks (Core equations, mask equation).

    M = M^lit U M^local U I, intersected with the causal mask, where
    M^lit_ij = 1[l_i = l_j = 1] and M^local_ij = 1[|i - j| <= w]; i, j and w
    are in block units. The local-only heads use M^local (which holds I), the
    literal-long-range-only heads use M^lit U I (self kept so every query
    block has a key), the hybrid heads use all three. Causal at block level is
    j <= i; the token-level causal cut inside the diagonal block is applied by
    ``token_mask``.
    """
    l = np.asarray(flags, dtype=bool)
    B = len(l)
    i = np.arange(B)[:, None]
    j = np.arange(B)[None, :]
    causal = j <= i
    ident = i == j
    local = np.abs(i - j) <= w
    lit = l[:, None] & l[None, :]
    return {
        LOCAL: causal & (local | ident),
        LITERAL: causal & (lit | ident),
        HYBRID: causal & (lit | local | ident),
    }


def token_mask(block_mask: np.ndarray, b: int, rows=None) -> np.ndarray:
    """allowed(p, q) = M[p // b, q // b] and q <= p, as a dense bool matrix.

    "intersects with the causal mask" is read at token level: off-diagonal
    visited blocks are fully visible, the diagonal block is lower-triangular.
    ``rows`` restricts the result to some query positions.
    """
    B = block_mask.shape[0]
    N = B * b
    p = np.arange(N) if rows is None else np.asarray(rows)
    q = np.arange(N)
    return block_mask[p[:, None] // b, q[None, :] // b] & (q[None, :] <= p[:, None])


def csr(mask: np.ndarray):
    """Row-major lists: for every query block i the ascending key blocks j
    with mask[i, j]; returned as (row_ptr [B+1], col_idx [nnz]) int32."""
    rows, cols = np.nonzero(mask)
    counts = np.bincount(rows, minlength=mask.shape[0])
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return row_ptr, cols.astype(np.int32)


def csc(mask: np.ndarray):
    """Column-major lists: for every key block j the ascending query blocks i
    with mask[i, j]; returned as (col_ptr [B+1], row_idx [nnz]) int32."""
    ptr, idx = csr(mask.T.copy())
    return ptr, idx


def bitmask(mask: np.ndarray) -> np.ndarray:
    """Packed rows: word w of row i holds bit (j - 32 w) for key block j."""
    B = mask.shape[0]
    nw = (B + 31) // 32
    out = np.zeros((B, nw), dtype=np.uint32)
    for i in range(B):
        for j in np.nonzero(mask[i])[0]:
            out[i, j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return out


def tile_lists(block_mask: np.ndarray, b: int, tile: int = 128):
    """Tile-level lists of the token mask: for every query tile I (rows
    [tile*I, tile*I + tile)), the key tiles J holding at least one allowed
    pair, ascending, with kind 0 (every pair of the tile block allowed) or
    1 (some pair not allowed). Returned as (row_ptr [T+1], key_tile [nnz],
    kind [nnz]) int32 and computed from the dense token mask one query tile
    at a time."""
    N = block_mask.shape[0] * b
    T = (N + tile - 1) // tile
    row_ptr, keys, kinds = [0], [], []
    for I in range(T):
        tm = token_mask(block_mask, b, rows=np.arange(I * tile, min(N, I * tile + tile)))
        for J in range(T):
            blk = tm[:, J * tile:min(N, J * tile + tile)]
            if blk.any():
                keys.append(J)
                kinds.append(0 if blk.all() else 1)
        row_ptr.append(len(keys))
    return (np.asarray(row_ptr, np.int32), np.asarray(keys, np.int32),
            np.asarray(kinds, np.int32))


def transpose_lists(row_ptr, cols, kinds, n_cols):
    """CSR (row -> ascending cols, kind) to CSC (col -> ascending rows, kind)."""
    ent = []
    for r in range(len(row_ptr) - 1):
        for e in range(row_ptr[r], row_ptr[r + 1]):
            ent.append((int(cols[e]), r, int(kinds[e])))
    ent.sort()
    counts = np.bincount([c for c, _, _ in ent], minlength=n_cols)
    ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return (ptr, np.asarray([r for _, r, _ in ent], np.int32),
            np.asarray([k for _, _, k in ent], np.int32))
