"""Visited and skipped tiles, counted on the device.

The instrumented variant of the library (libsa_count.so, built with
-DSA_COUNT_TILES) adds, per work item, the tiles each attention kernel loads
and multiplies to counters in the workspace's status header. These tests run
it on the full-size workloads and compare the counts with what the oracle's
masks fix: the forward visits exactly the mask's blocks (gzip, b = 128: one
128 x 128 tile per block pair of the lists; pair mode, b = 64: every block
pair of the mask once, inside visits of two 64-key blocks), the gist layout
exactly the compacted sink/gist tiles below each query tile's near tiles plus
the near tiles, and both backward passes the same tiles as the forward. The
dense causal count of the same items gives the skipped tiles (dense - visited).
The inputs are zeros: the counts do not depend on values.
"""
import os

import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import gist as Gi
from oracle import gzip_mask as G

pytestmark = pytest.mark.gpu

FWD_VISITS, FWD_DENSE, PAIR_BLOCKS, PAIR_DENSE, DQ_VISITS, DKDV_VISITS = range(6)
COUNTER_BYTE = 8 + 4 * 8  # aux[8] of the status header


@pytest.fixture(scope="module")
def csa(sa):
    """The binding with the instrumented library in place of libsa.so."""
    from content_adaptive_block_sa_b200 import build
    assert os.path.exists(build.LIB_COUNT), "libsa_count.so is built by __graft_entry__.build()"
    saved = sa._lib
    sa._lib = sa._abi.load(build.LIB_COUNT)
    yield sa
    sa._lib = saved


def counters(ws):
    torch.cuda.synchronize()
    c = ws[COUNTER_BYTE:COUNTER_BYTE + 8 * 6].view(torch.int64).cpu().tolist()
    assert ws[:4].view(torch.int32).item() == 0, "device status set"
    return c


def run(sa, w, md, lists, backward):
    Bt, N, H, Hkv, d = w.get("batch", 1), w["seq_len"], w["heads"], w["kv_heads"], w["head_dim"]
    q = torch.zeros(Bt, N, H, d, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(Bt, N, Hkv, d, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    o = torch.empty_like(q)
    lse = torch.empty(Bt, H, N, dtype=torch.float32, device="cuda")
    ad = sa.attn_desc(q, k, v, o)
    fws = sa.forward_workspace(ad, md)
    sa.sa_forward(ad, md, q, k, v, lists, o, lse, fws)
    fwd = counters(fws)
    if not backward:
        return fwd, None
    do = torch.zeros_like(q)
    dq = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    dk = torch.empty(k.shape, dtype=torch.float32, device="cuda")
    dv = torch.empty_like(dk)
    bws = sa.backward_workspace(ad, md)
    sa.sa_backward(ad, md, q, k, v, o, lse, do, lists, dq, dk, dv, bws)
    return fwd, counters(bws)


def gzip_block_pairs(w, flags):
    cls = G.head_classes(w["heads"])
    return sum(int(G.block_masks(flags[bt], w["window"])[cls[h]].sum())
               for bt in range(w["batch"]) for h in range(w["heads"]))


def test_gzip_8k_pair_mode_visits_every_mask_block_once(csa):
    w = W.WORKLOADS["gzip_8k"]
    flags = W.bernoulli_flags(w)
    md = csa.gzip_mask(w["batch"], w["seq_len"], w["block"], w["window"], w["heads"])
    lists = csa.build_block_mask(md, flags)
    fwd, _ = run(csa, w, md, lists, backward=False)
    B = w["seq_len"] // w["block"]
    dense = w["batch"] * w["heads"] * B * (B + 1) // 2
    assert fwd[PAIR_BLOCKS] == gzip_block_pairs(w, flags)
    assert fwd[PAIR_DENSE] == dense
    # a visit multiplies four 64 x 64 block pairs, some outside the mask
    assert 4 * fwd[FWD_VISITS] >= fwd[PAIR_BLOCKS]
    print(f"gzip 8K: {fwd[PAIR_BLOCKS]} block pairs visited, {dense - fwd[PAIR_BLOCKS]} skipped "
          f"of {dense}; {fwd[FWD_VISITS]} tiles, {4 * fwd[FWD_VISITS] / fwd[PAIR_BLOCKS]:.3f}x executed")


def test_gzip_64k_forward_and_backward_visit_exactly_the_lists(csa):
    w = W.WORKLOADS["gzip_64k_fwdbwd"]
    flags = np.stack([G.literal_flags(W.workload_bytes(w, b), w["block"]) for b in range(w["batch"])])
    md = csa.gzip_mask(w["batch"], w["seq_len"], w["block"], w["window"], w["heads"])
    lists = csa.build_block_mask(md, flags)
    fwd, bwd = run(csa, w, md, lists, backward=True)
    B = w["seq_len"] // w["block"]
    pairs = gzip_block_pairs(w, flags)
    dense = w["batch"] * w["heads"] * B * (B + 1) // 2
    assert fwd[FWD_VISITS] == pairs
    assert fwd[FWD_DENSE] == dense
    assert bwd[DQ_VISITS] == pairs and bwd[DKDV_VISITS] == pairs
    print(f"gzip 64K: {pairs} tiles visited, {dense - pairs} skipped of {dense} "
          f"({100 * pairs / dense:.2f}% of dense causal)")


def gist_kernel_tiles(w):
    """Per query head: compacted sink/gist tiles below the near tiles, plus the
    near tiles, summed over the query tiles (the oracle's prefix rule)."""
    N, S, Wn = w["seq_len"], w["sinks"], w["window"]
    g = Gi.gist_flags(N, S, w["ratio"])
    perm = Gi.shift_permutation(g, 128)
    _, far_ptr = Gi.always_visible_keys(g, S, perm, 128)
    T = (N + 127) // 128
    total = 0
    for I in range(T):
        jlo = Gi.near_tile_start(I, Wn, 128)
        total += -(-int(far_ptr[jlo]) // 128) + (I - jlo + 1)
    return total, T * (T + 1) // 2


def test_gist_32k_forward_and_backward_visit_the_compacted_layout(csa):
    w = W.WORKLOADS["gist_prefill_32k"]
    md = csa.gist_mask(w["seq_len"], w["heads"], w["sinks"], w["ratio"], w["window"],
                       gist_tail=w["gist_tail"])
    lists = csa.build_block_mask(md, None)
    fwd, bwd = run(csa, w, md, lists, backward=True)
    per_head, dense = gist_kernel_tiles(w)
    H = w["heads"]
    assert fwd[FWD_VISITS] == H * per_head
    assert fwd[FWD_DENSE] == H * dense
    assert bwd[DQ_VISITS] == H * per_head and bwd[DKDV_VISITS] == H * per_head
    print(f"gist 32K: {H * per_head} tiles visited, {H * (dense - per_head)} skipped of "
          f"{H * dense} ({dense / per_head:.2f}x fewer than dense causal)")
