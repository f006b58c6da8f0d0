"""Pins for the oracle's UniGist layout (CPU only): gist counts in closed
form, the page's compression ratio and 75% memory figure, visible-key counts,
reductions to dense causal and self-only attention, the shift permutation
against NumPy's stable sort, and the tile lists' closed-form structure."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import gist as Gi

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_values.json")))


def test_gist_count_and_ratio():
    g = Gi.gist_flags(32768, 128, 4)
    assert g.sum() == 6528 and (~g).sum() == 26240
    assert not g[:128].any()
    gold = GOLD["kv_reduction_at_ratio_4"]
    body = Gi.gist_flags(4000, 0, gold["ratio"])
    raw_per_gist = (~body).sum() / body.sum()
    assert raw_per_gist == gold["ratio"]
    assert 1 - 1 / raw_per_gist == gold["reduction"]


def test_visible_key_count_closed_form():
    S, W, N = GOLD["unigist_sinks_and_window"]["sinks"], GOLD["unigist_sinks_and_window"]["window"], 3000
    g = Gi.gist_flags(N, S, 4)
    for i in (255, 256, 700, 1234, 2999):
        n_gist = (i - 128 - 128 + 1) // 5
        assert len(Gi.visible_keys(g, S, W, i)) == S + n_gist + W
    vis = Gi.visibility(g, S, W, rows=[300, 2999])
    assert vis.sum(1).tolist() == [len(Gi.visible_keys(g, S, W, i)) for i in (300, 2999)]


def test_wide_window_is_dense_causal_and_unit_window_is_self():
    N = 200
    g = Gi.gist_flags(N, 16, 4)
    assert np.array_equal(Gi.visibility(g, 16, N), np.tril(np.ones((N, N), bool)))
    g0 = Gi.gist_flags(N, 0, N)  # no gists at all
    assert not g0.any()
    vis = Gi.visibility(g0, 0, 1)
    assert np.array_equal(vis, np.eye(N, dtype=bool))
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((3, N, 8))
    assert np.array_equal(A.forward(q, k, v, vis)[0], v)


def test_gist_attention_matches_torch_sdpa():
    N, d = 300, 16
    g = Gi.gist_flags(N, 8, 4)
    vis = Gi.visibility(g, 8, 16)
    rng = np.random.default_rng(1)
    q, k, v = rng.standard_normal((3, N, d))
    o, _ = A.forward(q, k, v, vis)
    t = lambda x: torch.from_numpy(x)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v),
                                                           attn_mask=torch.from_numpy(vis)[None, None])
    np.testing.assert_allclose(o, ref[0, 0].numpy(), atol=1e-12)


@pytest.mark.parametrize("N,tile", [(32768, 128), (1000, 128), (77, 16)])
def test_shift_permutation_is_stable_partition_per_tile(N, tile):
    g = Gi.gist_flags(N, 128 if N > 1000 else 5, 4)
    perm = Gi.shift_permutation(g, tile)
    assert sorted(perm.tolist()) == list(range(N))
    for t0 in range(0, N, tile):
        idx = np.arange(t0, min(N, t0 + tile))
        want = idx[np.argsort(g[idx].astype(np.int8), kind="stable")]
        assert np.array_equal(perm[idx], want)


def test_tile_lists_structure():
    # tiles of 128 positions, 128 sinks, ratio 4, window 128, 32-wide tail
    N, tile = 128 * 12 + 77, 128
    g = Gi.gist_flags(N, 128, 4)
    perm = Gi.shift_permutation(g, tile)
    vis = Gi.visibility(g, 128, 128)[np.ix_(perm, perm)]
    rp, kt, kd = Gi.tile_lists(vis, tile, 32)
    T = (N + tile - 1) // tile
    for I in range(T):
        got = list(zip(kt[rp[I]:rp[I + 1]].tolist(), kd[rp[I]:rp[I + 1]].tolist()))
        if I == 0:
            want = [(0, Gi.MASKED)]
        elif I == 1:
            want = [(0, Gi.FULL), (1, Gi.MASKED)]
        else:
            want = [(0, Gi.FULL)] + [(J, Gi.TAIL) for J in range(1, I - 1)] + \
                   [(I - 1, Gi.MASKED), (I, Gi.MASKED)]
        assert got == want, I
    # every gist of a full tile sits in its last 32 columns after the shift
    for t0 in range(tile, N - tile, tile):
        gp = g[perm[t0:t0 + tile]]
        assert gp[-32:].sum() == gp.sum() and gp.sum() in (25, 26)


def test_tile_lists_row_callable_matches_dense():
    N = 600
    g = Gi.gist_flags(N, 16, 4)
    perm = Gi.shift_permutation(g, 128)
    dense = Gi.visibility(g, 16, 40)[np.ix_(perm, perm)]
    fn = lambda rows: Gi.visibility(g, 16, 40, rows=perm[rows])[:, perm]
    for a, b in zip(Gi.tile_lists(dense, 128, 32), Gi.tile_lists(fn, 128, 32, N=N)):
        assert np.array_equal(a, b)
    # the lists of some query tiles are those tiles' rows of the full lists
    rp, kt, kd = Gi.tile_lists(dense, 128, 32)
    rp2, kt2, kd2 = Gi.tile_lists(fn, 128, 32, N=N, query_tiles=[1, 4])
    want = np.r_[rp[1]:rp[2], rp[4]:rp[5]]
    assert np.array_equal(kt2, kt[want]) and np.array_equal(kd2, kd[want])
    assert np.array_equal(np.diff(rp2), [rp[2] - rp[1], rp[5] - rp[4]])


@pytest.mark.parametrize("N,sinks,window", [(2000, 128, 128), (1500, 5, 300), (777, 0, 1)])
def test_far_prefix_covers_exactly_the_visible_keys_outside_the_near_tiles(N, sinks, window):
    g = Gi.gist_flags(N, sinks, 4)
    perm = Gi.shift_permutation(g, 128)
    far_idx, far_ptr = Gi.always_visible_keys(g, sinks, perm, 128)
    T = (N + 127) // 128
    for I in range(T):
        Jlo = Gi.near_tile_start(I, window, 128)
        rows = np.arange(I * 128, min(N, I * 128 + 128))
        vis = Gi.visibility(g, sinks, window, rows=rows)[:, : 128 * Jlo]
        # every key below the near tiles is visible to all rows of the tile or to none
        cols = np.nonzero(vis.any(axis=0))[0]
        assert vis[:, cols].all()
        assert np.array_equal(np.sort(perm[far_idx[: far_ptr[Jlo]]]), cols)
    assert far_ptr[-1] == len(far_idx) == sinks + g[sinks:].sum()


# ---------------------------------------------------------------- coarse layout
def _coarse_vis_by_scanning(g, sinks):
    """Visibility from the gist flags alone: a segment starts at the first raw
    token after the sinks or after a run of gists; query i sees the sinks, the
    gists before it, and every position from its segment's start to itself."""
    N = len(g)
    vis = np.zeros((N, N), bool)
    for i in range(N):
        if i < sinks:
            vis[i, : i + 1] = True
            continue
        s = i  # back to the segment's start: a raw token after a gist, or the sinks' end
        while s > sinks and not (g[s - 1] and not g[s]):
            s -= 1
        for j in range(i + 1):
            vis[i, j] = j < sinks or g[j] or j >= s
    return vis


def test_coarse_flags_closed_form():
    g = Gi.coarse_gist_flags(20480, 0, 1024, 4)
    assert g.sum() == 16 * 256
    for s in range(16):
        assert not g[s * 1280: s * 1280 + 1024].any() and g[s * 1280 + 1024:(s + 1) * 1280].all()
    seg = Gi.segment_ids(20480, 0, 1024, 4)
    assert np.array_equal(np.bincount(seg), np.full(16, 1280))
    # sinks are not part of any segment
    assert (Gi.segment_ids(300, 7, 40, 4)[:7] == -1).all()


def test_coarse_max_block_length_matches_page():
    gold = GOLD["segment_wise_max_length"]
    L, r, n_in = gold["segment"], gold["ratio"], gold["input_tokens"]
    nseg = n_in // L
    N = nseg * (L + L // r)
    g = Gi.coarse_gist_flags(N, 0, L, r)
    seg = Gi.segment_ids(N, 0, L, r)
    raw = np.nonzero(~g)[0]
    counts = Gi.coarse_visibility(g, seg, 0, rows=raw[-L:]).sum(1)  # last segment's raw tokens
    assert counts.max() == gold["max_positions"] == (n_in - L) // r + L
    # every raw query: earlier segments' gists plus its segment's raw tokens up to itself
    rows = raw[:: 97]
    want = seg[rows] * (L // r) + (rows - seg[rows] * (L + L // r)) + 1
    assert np.array_equal(Gi.coarse_visibility(g, seg, 0, rows=rows).sum(1), want)


@pytest.mark.parametrize("N,sinks,L,r", [(300, 7, 40, 4), (257, 0, 16, 8), (190, 33, 20, 2)])
def test_coarse_visibility_matches_scan_from_flags(N, sinks, L, r):
    g = Gi.coarse_gist_flags(N, sinks, L, r)
    seg = Gi.segment_ids(N, sinks, L, r)
    assert np.array_equal(Gi.coarse_visibility(g, seg, sinks), _coarse_vis_by_scanning(g, sinks))


def test_coarse_single_segment_is_dense_causal():
    N = 180
    g = Gi.coarse_gist_flags(N, 5, 160, 4)  # 5 sinks, one segment of 200 positions
    seg = Gi.segment_ids(N, 5, 160, 4)
    assert np.array_equal(Gi.coarse_visibility(g, seg, 5), np.tril(np.ones((N, N), bool)))


@pytest.mark.parametrize("N,sinks,L,r", [(3000, 128, 1024, 4), (2500, 5, 96, 4), (1300, 300, 200, 8),
                                         (900, 0, 64, 2)])
def test_coarse_far_prefix_covers_exactly_the_visible_keys_outside_the_near_tiles(N, sinks, L, r):
    g = Gi.coarse_gist_flags(N, sinks, L, r)
    seg = Gi.segment_ids(N, sinks, L, r)
    perm = Gi.shift_permutation(g, 128)
    far_idx, far_ptr = Gi.always_visible_keys(g, sinks, perm, 128)
    period = L + L // r
    for I in range((N + 127) // 128):
        Jlo = Gi.coarse_near_tile_start(I, sinks, L, r, 128)
        assert 0 <= I - Jlo <= (period + 126) // 128
        rows = np.arange(I * 128, min(N, I * 128 + 128))
        vis = Gi.coarse_visibility(g, seg, sinks, rows=rows)[:, : 128 * Jlo]
        cols = np.nonzero(vis.any(axis=0))[0]
        assert vis[:, cols].all()
        assert np.array_equal(np.sort(perm[far_idx[: far_ptr[Jlo]]]), cols)


def test_coarse_attention_matches_torch_sdpa():
    N, d = 260, 16
    g = Gi.coarse_gist_flags(N, 6, 48, 4)
    vis = Gi.coarse_visibility(g, Gi.segment_ids(N, 6, 48, 4), 6)
    rng = np.random.default_rng(2)
    q, k, v = rng.standard_normal((3, N, d))
    o, _ = A.forward(q, k, v, vis)
    t = lambda x: torch.from_numpy(x)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v),
                                                           attn_mask=torch.from_numpy(vis)[None, None])
    np.testing.assert_allclose(o, ref[0, 0].numpy(), atol=1e-12)
