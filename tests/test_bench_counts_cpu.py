"""The work counts bench.py reports, checked on CPU against the oracle's
masks: exact visible pairs of the gist layouts (fine and coarse) and the
exact token edges of a gzip mask from its visited block pairs."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import sa_workloads as W  # noqa: E402
from oracle import gist as Gi  # noqa: E402
from oracle import gzip_mask as G  # noqa: E402


@pytest.mark.parametrize("N,S,Wn", [(1000, 16, 32), (777, 0, 1), (2000, 128, 128), (300, 300, 5),
                                    (640, 3, 1000)])
def test_gist_visible_pairs_fine_layout(N, S, Wn):
    w = W.scaled("gist_prefill_32k", seq_len=N, sinks=S, window=Wn)
    assert bench.gist_visible_pairs(w) == int(Gi.visibility(Gi.gist_flags(N, S, 4), S, Wn).sum())


@pytest.mark.parametrize("N,S,L", [(1300, 0, 64), (1000, 7, 32), (2560, 128, 1024)])
def test_gist_visible_pairs_coarse_layout(N, S, L):
    w = W.scaled("gist_coarse_20k", seq_len=N, sinks=S, gist_segment=L)
    g = Gi.coarse_gist_flags(N, S, L, 4)
    seg = Gi.segment_ids(N, S, L, 4)
    assert bench.gist_visible_pairs(w) == int(Gi.coarse_visibility(g, seg, S).sum())


def test_gzip_exact_edges_from_block_pairs():
    """b^2 (pairs - B) + B b(b+1)/2 per list: the count the bench derives from
    the lists, against the dense token mask."""
    b, B = 16, 12
    flags = (np.random.default_rng(3).random(B) < 0.4).astype(np.uint8)
    for c, m in G.block_masks(flags, 2).items():
        pairs = int(m.sum())
        assert b * b * (pairs - B) + B * b * (b + 1) // 2 == int(G.token_mask(m, b).sum()), c
