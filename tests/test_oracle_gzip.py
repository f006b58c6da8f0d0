"""Pins for the oracle's gzip flags and block masks (CPU only).

Each check is independent of the oracle's own formulas: closed-form edge
counts, the container invariance of the mean comparison, exact rationals,
special cases that reduce to dense causal or self-only masks, and brute force
over every flag vector of tiny inputs.
"""
import gzip
import itertools
import json
import os
import zlib
from fractions import Fraction

import numpy as np
import pytest

import sa_workloads as W
from oracle import gzip_mask as G

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_values.json")))


def test_tiny_workload_flags_mark_random_runs_literal():
    # Even 32-byte runs repeat an 8-byte pattern (compressible), odd runs are
    # random bytes; with b=16 each run is two blocks. Literal = above-mean
    # compressed size, so only the random runs are literal.
    x = W.workload_bytes("gzip_tiny_fp32", 0)
    assert G.literal_flags(x, 16).tolist() == [0, 0, 1, 1] * 4


@pytest.mark.parametrize("name,b", [("gzip_tiny_fp32", 16), ("gzip_64k_fwdbwd", 128)])
def test_flags_do_not_depend_on_container(name, b):
    x = W.workload_bytes(name, 0)
    raw = lambda blk: (lambda c: c.compress(blk) + c.flush())(zlib.compressobj(1, zlib.DEFLATED, -15))
    gz = lambda blk: gzip.compress(blk, compresslevel=1, mtime=0)
    ref = G.literal_flags(x, b)
    assert np.array_equal(G.literal_flags_from_sizes(G.block_compressed_sizes(x, b, raw)), ref)
    assert np.array_equal(G.literal_flags_from_sizes(G.block_compressed_sizes(x, b, gz)), ref)


def test_flags_equal_exact_rational_ratio_test():
    x = W.workload_bytes("gzip_64k_fwdbwd", 1)
    b = 128
    sizes = G.block_compressed_sizes(x, b)
    r = [Fraction(c, b) for c in sizes]
    rbar = sum(r) / len(r)
    assert G.literal_flags(x, b).tolist() == [int(ri > rbar) for ri in r]
    # the synthetic mix gives a sensible literal fraction (~40% random segments)
    assert 0.2 < np.mean(G.literal_flags(x, b)) < 0.6


def test_mean_tie_is_not_literal():
    assert G.literal_flags_from_sizes([7] * 9).tolist() == [0] * 9
    assert G.literal_flags_from_sizes([1, 2, 3]).tolist() == [0, 0, 1]


def test_head_split_matches_page():
    gold = GOLD["head_split"]
    for H in (4, 8, 16, 32):
        cls = G.head_classes(H)
        assert cls == sorted(cls)  # local, then literal, then hybrid
        assert cls.count(G.LOCAL) == gold["local"] * H
        assert cls.count(G.LITERAL) == gold["literal"] * H
        assert cls.count(G.HYBRID) == gold["hybrid"] * H
    assert G.head_classes(6) == [0, 0, 0, 1, 2, 2]


def _closed_form_counts(flags, w):
    B, L = len(flags), int(np.sum(flags))
    local = (w + 1) * B - w * (w + 1) // 2 if B > w else B * (B + 1) // 2
    literal = L * (L + 1) // 2 + (B - L)
    overlap = sum(1 for d in range(min(w, B - 1) + 1) for i in range(d, B)
                  if flags[i] and flags[i - d])
    hybrid = L * (L + 1) // 2 + local - overlap
    return local, literal, hybrid


@pytest.mark.parametrize("B,w,p,seed", [(16, 1, 0.5, 0), (128, 2, 0.3, 1), (512, 2, 0.4, 2),
                                        (37, 5, 0.2, 3), (64, 0, 0.9, 4), (9, 20, 0.5, 5)])
def test_block_mask_edge_counts_closed_form(B, w, p, seed):
    flags = (np.random.default_rng(seed).random(B) < p).astype(np.uint8)
    m = G.block_masks(flags, w)
    assert (int(m[G.LOCAL].sum()), int(m[G.LITERAL].sum()), int(m[G.HYBRID].sum())) == \
        _closed_form_counts(flags, w)


def test_tiny_workload_counts():
    m = G.block_masks([0, 0, 1, 1] * 4, 1)
    assert [int(m[c].sum()) for c in (0, 1, 2)] == [31, 44, 55]


def test_special_cases_reduce_to_dense_causal_or_self():
    B = 24
    causal = np.tril(np.ones((B, B), bool))
    m = G.block_masks(np.ones(B, np.uint8), 1)
    assert np.array_equal(m[G.LITERAL], causal) and np.array_equal(m[G.HYBRID], causal)
    m = G.block_masks((np.arange(B) % 3 == 0).astype(np.uint8), B - 1)
    assert np.array_equal(m[G.LOCAL], causal) and np.array_equal(m[G.HYBRID], causal)
    m = G.block_masks(np.zeros(B, np.uint8), 0)
    for c in (0, 1, 2):
        assert np.array_equal(m[c], np.eye(B, dtype=bool))


def test_brute_force_all_flag_vectors():
    for B in range(1, 7):
        for bits in itertools.product([0, 1], repeat=B):
            for w in (0, 1, 2, 8):
                lit = {(i, j) for i in range(B) for j in range(B) if bits[i] and bits[j]}
                loc = {(i, j) for i in range(B) for j in range(B) if abs(i - j) <= w}
                ident = {(i, i) for i in range(B)}
                causal = {(i, j) for i in range(B) for j in range(i + 1)}
                want = {G.LOCAL: loc & causal, G.LITERAL: (lit | ident) & causal,
                        G.HYBRID: (lit | loc | ident) & causal}
                got = G.block_masks(bits, w)
                for c, s in want.items():
                    assert set(zip(*np.nonzero(got[c]))) == s


def test_token_mask_edge_count_and_diagonal():
    flags = (np.random.default_rng(7).random(20) < 0.4).astype(np.uint8)
    b = 8
    for c, m in G.block_masks(flags, 2).items():
        tm = G.token_mask(m, b)
        B = m.shape[0]
        assert tm.sum() == b * b * (m.sum() - B) + B * b * (b + 1) // 2
        assert np.array_equal(tm, tm & np.tril(np.ones_like(tm)))
        assert tm.diagonal().all()
        rows = [0, 13, 100, 159]
        assert np.array_equal(G.token_mask(m, b, rows=rows), tm[rows])


def test_edges_grow_linearly_when_literals_grow_like_sqrt_n():
    # Core equations: O(L^2 + N w), roughly linear in N when L = O(sqrt N).
    w, edges = 2, []
    for B in (256, 1024, 4096):
        L = int(np.sqrt(B))
        flags = np.zeros(B, np.uint8)
        flags[np.linspace(0, B - 1, L).astype(int)] = 1
        edges.append(_closed_form_counts(flags, w)[2])
        assert edges[-1] == int(G.block_masks(flags, w)[G.HYBRID].sum()) if B <= 1024 else True
    assert 3.0 < edges[1] / edges[0] < 5.0 and 3.0 < edges[2] / edges[1] < 5.0


def test_lists_and_bits():
    flags = (np.random.default_rng(11).random(70) < 0.3).astype(np.uint8)
    m = G.block_masks(flags, 2)[G.HYBRID]
    rp, ci = G.csr(m)
    cp, ri = G.csc(m)
    bits = G.bitmask(m)
    for i in range(70):
        assert ci[rp[i]:rp[i + 1]].tolist() == [j for j in range(70) if m[i, j]]
        assert ri[cp[i]:cp[i + 1]].tolist() == [r for r in range(70) if m[r, i]]
        for j in range(70):
            assert bool((int(bits[i, j // 32]) >> (j % 32)) & 1) == bool(m[i, j])


def test_tile_lists_closed_forms():
    # b = 128: tile lists equal block lists, diagonal masked, others full
    flags = (np.random.default_rng(12).random(20) < 0.3).astype(np.uint8)
    m = G.block_masks(flags, 2)[G.HYBRID]
    rp, kt, kd = G.tile_lists(m, 128)
    brp, bci = G.csr(m)
    assert np.array_equal(rp, brp) and np.array_equal(kt, bci)
    assert all(kd[e] == (1 if kt[e] == i else 0) for i in range(20) for e in range(rp[i], rp[i + 1]))
    # b = 64, local class, w = 2: query tile I covers blocks 2I, 2I+1 whose union
    # reaches back to block 2I-2 -> key tiles I-1 (not all pairs) and I (diag)
    m = G.block_masks(np.zeros(16, np.uint8), 2)[G.LOCAL]
    rp, kt, kd = G.tile_lists(m, 64)
    for I in range(8):
        got = list(zip(kt[rp[I]:rp[I + 1]].tolist(), kd[rp[I]:rp[I + 1]].tolist()))
        assert got == ([(I - 1, 1)] if I else []) + [(I, 1)]
    # b = 256: two tiles per block; all-literal -> dense causal at tile level
    m = G.block_masks(np.ones(4, np.uint8), 0)[G.LITERAL]
    rp, kt, kd = G.tile_lists(m, 256)
    for I in range(8):
        assert kt[rp[I]:rp[I + 1]].tolist() == list(range(I + 1))
        assert kd[rp[I]:rp[I + 1]].tolist() == [0] * I + [1]
    cp, ri, rk = G.transpose_lists(rp, kt, kd, 8)
    for J in range(8):
        assert ri[cp[J]:cp[J + 1]].tolist() == list(range(J, 8))
