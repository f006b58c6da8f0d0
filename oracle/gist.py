"""UniGist prefill layout (oracle; test infrastructure only).

Source: "UniGist: Towards General and Hardware-aligned Sequence-level Long
Context Compression" (AI summary page): Approach (one-pass training with a
unified sparse pattern of sink tokens, gist tokens and a local window; the gist
shift trick that moves gists to the right so kernels skip non-visible blocks),
Measured effects table (128 sink tokens; local window 128). Interleaved
fine-grained gists and the compression ratio come from "A Silver Bullet or a
Compromise for Full Attention? A Comprehensive Study of Gist Token-based
Context Compression" (section 2, Preliminaries).

Readings taken where the pages are silent:
* positions 0..sinks-1 are raw sink tokens with no gists among them;
* after the sinks a gist follows every ``ratio`` raw tokens (R..RG repeated),
  so position p >= sinks is a gist iff (p - sinks) mod (ratio + 1) == ratio;
* the window is a distance in logical positions: i - j < window (self
  included); gist queries use the same rule as raw queries;
* the gist shift acts inside each tile of ``tile`` positions: the tile's raw
  tokens keep their order and come first, its gists follow in order.

Segment-wise (coarse) layout, from the same study (section 2: coarse gists
follow all raw tokens of a segment; section 6: gist compression as
segment-wise sparse attention with full attention inside each segment;
appendix E: 16K input, ratio 4, 1K segments give at most 4.75K positions for
a block to model). Readings:
* after the sinks the sequence is a run of segments, each ``seg_len`` raw
  tokens followed by ``seg_len / ratio`` gists (one period of
  ``seg_len + seg_len / ratio`` positions); a ragged last segment keeps the
  same positions;
* a segment's own gists belong to it, so a gist sees its whole segment;
* query i sees the sinks, every gist that is not in its future and every
  position of its own segment up to itself: the window rule with "i - j <
  window" replaced by "same segment".
"""
from __future__ import annotations

import numpy as np

FULL, MASKED, TAIL = 0, 1, 2


def gist_flags(N: int, sinks: int, ratio: int) -> np.ndarray:
    p = np.arange(N)
    return (p >= sinks) & ((p - sinks) % (ratio + 1) == ratio)


def visibility(is_gist, sinks: int, window: int, rows=None) -> np.ndarray:
    """vis[i, j] = j <= i and (j < sinks or gist(j) or i - j < window), in
    logical positions (dense bool, optionally for some query rows only)."""
    g = np.asarray(is_gist, bool)
    N = len(g)
    i = (np.arange(N) if rows is None else np.asarray(rows))[:, None]
    j = np.arange(N)[None, :]
    return (j <= i) & ((j < sinks) | g[None, :] | (i - j < window))


def visible_keys(is_gist, sinks: int, window: int, i: int) -> np.ndarray:
    """Logical key positions visible from query i (one row of visibility)."""
    g = np.asarray(is_gist, bool)
    j = np.arange(i + 1)
    return j[(j < sinks) | g[: i + 1] | (i - j < window)]


def shift_permutation(is_gist, tile: int) -> np.ndarray:
    """perm[physical index] = logical position stored there."""
    g = np.asarray(is_gist, bool)
    N = len(g)
    perm = []
    for t0 in range(0, N, tile):
        idx = np.arange(t0, min(N, t0 + tile))
        perm.extend(idx[~g[idx]].tolist())
        perm.extend(idx[g[idx]].tolist())
    return np.asarray(perm, dtype=np.int32)


def tile_lists(vis_phys, tile: int, tail: int, N: int | None = None, query_tiles=None):
    """Per query tile, the key tiles that hold at least one visible pair.

    ``vis_phys`` is the visibility matrix in physical (shifted) order. Each
    entry is (key tile, kind): FULL if every pair of the tile block is
    visible, TAIL if every visible column lies in the last ``tail`` of the
    tile's ``tile`` nominal columns (where the shift puts a full tile's
    gists), MASKED otherwise. Returned as
    (row_ptr [T+1], key_tile [nnz], kind [nnz]) int32 with key tiles ascending.
    ``vis_phys`` may also be a callable rows -> bool [len(rows), N] (then N
    must be given), evaluated one query tile at a time. ``query_tiles``
    restricts the lists to some query tiles (row_ptr then has one entry per
    listed tile, plus one).
    """
    N = vis_phys.shape[0] if N is None else N
    T = (N + tile - 1) // tile
    row_ptr, keys, kinds = [0], [], []
    for I in (range(T) if query_tiles is None else query_tiles):
        rows = np.arange(I * tile, min(N, (I + 1) * tile))
        vrows = vis_phys(rows) if callable(vis_phys) else vis_phys[rows]
        for J in range(T):
            c0, c1 = J * tile, min(N, (J + 1) * tile)
            blk = vrows[:, c0:c1]
            if not blk.any():
                continue
            cols = np.nonzero(blk.any(axis=0))[0]
            if blk.all():
                kind = FULL
            elif cols.min() >= tile - tail:
                kind = TAIL
            else:
                kind = MASKED
            keys.append(J)
            kinds.append(kind)
        row_ptr.append(len(keys))
    return (np.asarray(row_ptr, np.int32), np.asarray(keys, np.int32),
            np.asarray(kinds, np.int32))


def always_visible_keys(is_gist, sinks: int, perm, tile: int):
    """Keys every later query sees whatever its window: sinks and gists.

    Returns (far_idx, far_ptr): far_idx[f] is the PHYSICAL index of the f-th
    such key in logical order, far_ptr[J] the number of them at logical
    positions below tile * J (J = 0..T). A query tile I whose window cannot
    reach below key tile J sees, among keys below tile * J, exactly
    far_idx[:far_ptr[J]].
    """
    g = np.asarray(is_gist, bool)
    N = len(g)
    inv = np.empty(N, np.int64)
    inv[np.asarray(perm)] = np.arange(N)
    pos = np.nonzero((np.arange(N) < sinks) | g)[0]
    T = (N + tile - 1) // tile
    far_ptr = np.array([np.count_nonzero(pos < tile * J) for J in range(T + 1)], np.int32)
    return inv[pos].astype(np.int32), far_ptr


def near_tile_start(I: int, window: int, tile: int) -> int:
    """First key tile that query tile I must visit with the element rule: for
    every key below tile * Jlo and query at or above tile * I, i - j >= window."""
    return max(0, I - (window - 1 + tile - 1) // tile)


# ---------------------------------------------------------------- coarse layout
def coarse_gist_flags(N: int, sinks: int, seg_len: int, ratio: int) -> np.ndarray:
    """Gist bit of each position: the last seg_len / ratio positions of every
    period of seg_len + seg_len / ratio positions after the sinks."""
    assert seg_len % ratio == 0
    period = seg_len + seg_len // ratio
    p = np.arange(N)
    return (p >= sinks) & ((p - sinks) % period >= seg_len)


def segment_ids(N: int, sinks: int, seg_len: int, ratio: int) -> np.ndarray:
    """Segment of each position (-1 for the sinks)."""
    period = seg_len + seg_len // ratio
    p = np.arange(N)
    return np.where(p < sinks, -1, (p - sinks) // period)


def coarse_visibility(is_gist, seg, sinks: int, rows=None) -> np.ndarray:
    """vis[i, j] = j <= i and (j < sinks or gist(j) or seg(i) == seg(j))."""
    g = np.asarray(is_gist, bool)
    sg = np.asarray(seg)
    N = len(g)
    i = (np.arange(N) if rows is None else np.asarray(rows))[:, None]
    j = np.arange(N)[None, :]
    return (j <= i) & ((j < sinks) | g[None, :] | (sg[i] == sg[None, :]))


def coarse_visible_keys(is_gist, seg, sinks: int, i: int) -> np.ndarray:
    """Logical key positions visible from query i under the coarse rule."""
    return np.nonzero(coarse_visibility(is_gist, seg, sinks, rows=[i])[0])[0]


def coarse_near_tile_start(I: int, sinks: int, seg_len: int, ratio: int, tile: int) -> int:
    """First key tile query tile I visits with the element rule: the tile that
    holds the start of the segment of the tile's first row (I itself while that
    row is a sink: everything below it is a sink). Keys below it are sinks or
    earlier segments' positions, seen by the whole query tile exactly when they
    are sinks or gists."""
    p = I * tile
    if p < sinks:
        return I
    period = seg_len + seg_len // ratio
    return (sinks + (p - sinks) // period * period) // tile
