"""Pins for the oracle's attention forward/backward (CPU only).

The oracle (NumPy fp64) is checked against PyTorch's scaled_dot_product_attention
and autograd in float64 (an independent library), against closed-form special
cases (self-only attention gives O = V), against central finite differences,
and against invariants every softmax attention satisfies.
"""
import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import gzip_mask as G


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, allowed):
    t = lambda x: torch.from_numpy(np.asarray(x, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=torch.from_numpy(allowed)[None, None])[0, 0].numpy()


@pytest.mark.parametrize("seed,N,b,d,w", [(0, 64, 8, 16, 1), (1, 96, 16, 32, 2), (2, 40, 4, 8, 0)])
def test_forward_matches_torch_sdpa(seed, N, b, d, w):
    flags = (np.random.default_rng(seed).random(N // b) < 0.4).astype(np.uint8)
    for c, bm in G.block_masks(flags, w).items():
        allowed = G.token_mask(bm, b)
        q, k, v = _rand(seed, N, d), _rand(seed + 10, N, d), _rand(seed + 20, N, d)
        o, lse = A.forward(q, k, v, allowed, row_chunk=17)
        np.testing.assert_allclose(o, _sdpa(q, k, v, allowed), rtol=0, atol=1e-12)
        s = np.where(allowed, q @ k.T / np.sqrt(d), -np.inf)
        np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(s), 1).numpy(), atol=1e-12)


def test_dense_causal_special_case():
    # all blocks literal -> the literal and hybrid classes are dense causal
    N, b, d = 128, 16, 32
    q, k, v = _rand(3, N, d), _rand(4, N, d), _rand(5, N, d)
    bm = G.block_masks(np.ones(N // b, np.uint8), 1)[G.LITERAL]
    o, _ = A.forward(q, k, v, G.token_mask(bm, b))
    t = lambda x: torch.from_numpy(x)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
    np.testing.assert_allclose(o, ref[0, 0].numpy(), atol=1e-12)


def test_self_only_gives_v_exactly():
    # no literal blocks, w = 0, b = 1: every token attends only to itself
    N, d = 50, 8
    q, k, v = _rand(6, N, d), _rand(7, N, d), _rand(8, N, d)
    allowed = G.token_mask(G.block_masks(np.zeros(N, np.uint8), 0)[G.HYBRID], 1)
    o, lse = A.forward(q, k, v, allowed)
    assert np.array_equal(o, v)
    np.testing.assert_allclose(lse, (q * k).sum(1) / np.sqrt(d), atol=1e-14)


def test_rows_sum_to_one_and_row_form_agrees():
    N, b, d = 80, 8, 16
    flags = (np.random.default_rng(9).random(N // b) < 0.5).astype(np.uint8)
    allowed = G.token_mask(G.block_masks(flags, 1)[G.HYBRID], b)
    q, k, v = _rand(10, N, d), _rand(11, N, d), _rand(12, N, d)
    P = A.probabilities(q, k, allowed)
    assert np.abs(P.sum(1) - 1).max() < 1e-12
    assert (P[~allowed] == 0).all()
    o, lse = A.forward(q, k, v, allowed)
    rows = [0, 7, 33, 79]
    o2, lse2 = A.forward_rows(q, k, v, lambda p: np.nonzero(allowed[p])[0], rows)
    np.testing.assert_allclose(o2, o[rows], atol=1e-13)
    np.testing.assert_allclose(lse2, lse[rows], atol=1e-13)


def _loss(q, k, v, do, allowed):
    return float((A.forward(q, k, v, allowed)[0] * do).sum())


def test_backward_matches_finite_differences():
    N, b, d = 32, 4, 8
    flags = np.array([1, 0, 1, 1, 0, 0, 1, 0], np.uint8)
    allowed = G.token_mask(G.block_masks(flags, 1)[G.HYBRID], b)
    q, k, v, do = (_rand(s, N, d) for s in (13, 14, 15, 16))
    dq, dk, dv, _, _ = A.backward(q, k, v, do, allowed)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            i, j = rng.integers(N), rng.integers(d)
            xp, xm = x.copy(), x.copy()
            xp[i, j] += eps
            xm[i, j] -= eps
            args = {"q": q, "k": k, "v": v}
            fp = _loss(**{**args, name: xp}, do=do, allowed=allowed)
            fm = _loss(**{**args, name: xm}, do=do, allowed=allowed)
            fd = (fp - fm) / (2 * eps)
            assert abs(fd - g[i, j]) <= 1e-6 * max(1.0, abs(g[i, j])), (name, i, j, fd, g[i, j])


def test_backward_matches_torch_autograd_and_invariants():
    N, b, d = 96, 16, 32
    flags = (np.random.default_rng(17).random(N // b) < 0.5).astype(np.uint8)
    allowed = G.token_mask(G.block_masks(flags, 2)[G.HYBRID], b)
    q, k, v, do = (_rand(s, N, d) for s in (18, 19, 20, 21))
    dq, dk, dv, o, lse = A.backward(q, k, v, do, allowed, row_chunk=40)
    tq, tk, tv = (torch.from_numpy(x)[None, None].requires_grad_() for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=torch.from_numpy(allowed)[None, None])
    out.backward(torch.from_numpy(do)[None, None])
    for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, ref.grad[0, 0].numpy(), atol=1e-11)
    # sum over keys of dS is zero per row -> dK sums to zero; rows of P sum to 1
    np.testing.assert_allclose(dk.sum(0), 0, atol=1e-10)
    np.testing.assert_allclose(dv.sum(0), do.sum(0), atol=1e-10)
    P = A.probabilities(q, k, allowed)
    dP = do @ v.T
    np.testing.assert_allclose((P * dP).sum(1), (do * o).sum(1), atol=1e-12)


def test_row_and_column_forms_of_backward_agree_with_dense():
    N, b, d = 64, 8, 16
    flags = (np.random.default_rng(22).random(N // b) < 0.5).astype(np.uint8)
    allowed = G.token_mask(G.block_masks(flags, 1)[G.HYBRID], b)
    q, k, v, do = (_rand(s, N, d) for s in (23, 24, 25, 26))
    dq, dk, dv, _, _ = A.backward(q, k, v, do, allowed)
    keys_of = lambda p: np.nonzero(allowed[p])[0]
    rows_of = lambda j: np.nonzero(allowed[:, j])[0]
    sel = [0, 9, 40, 63]
    np.testing.assert_allclose(A.backward_rows(q, k, v, do, keys_of, sel), dq[sel], atol=1e-12)
    dk2, dv2 = A.backward_cols(q, k, v, do, keys_of, rows_of, sel)
    np.testing.assert_allclose(dk2, dk[sel], atol=1e-12)
    np.testing.assert_allclose(dv2, dv[sel], atol=1e-12)
    # chunked column form: every row, or only the rows that attend the keys,
    # in chunks that split query blocks
    mask = lambda r: allowed[r]
    for rows in (np.arange(N), np.unique(np.concatenate([rows_of(j) for j in sel]))):
        dk3, dv3 = A.backward_cols_chunked(q, k, v, do, mask, rows, sel, row_chunk=7)
        np.testing.assert_allclose(dk3, dk[sel], atol=1e-12)
        np.testing.assert_allclose(dv3, dv[sel], atol=1e-12)
    # rows that do not attend a key add nothing to its gradients
    others = np.setdiff1d(np.arange(N), rows_of(sel[1]))
    z = A.backward_cols_chunked(q, k, v, do, mask, others, sel[1:2])
    assert others.size and not z[0].any() and not z[1].any()
