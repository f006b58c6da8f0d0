"""Shared helpers of the GPU parity tests: seeded inputs, uploads and the
element-wise comparison against the oracle."""
from __future__ import annotations

import numpy as np
import torch

import sa_workloads as W
from oracle import gist as Gi
from oracle import gzip_mask as G

# max-abs and relative-L2 bounds for outputs, LSE and gradients
TOL = {"bf16": (2e-2, 5e-3), "fp32": (1e-5, 1e-5)}


def check_close(got, want, dtype: str, what: str):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    ma, rl2 = TOL[dtype]
    err = np.abs(got - want).max() if got.size else 0.0
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert err <= ma and rel <= rl2, f"{what}: max-abs {err:.3g} (<= {ma}), rel-L2 {rel:.3g} (<= {rl2})"
    return err, rel


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


# ------------------------------------------------------------------ gzip
def gzip_inputs(w: dict, with_do: bool = False):
    """Stacked [Bt, N, H, d] inputs of a gzip workload (float32 values)."""
    qs = np.stack([W.qkv(w, "q", b) for b in range(w["batch"])])
    ks = np.stack([W.qkv(w, "k", b) for b in range(w["batch"])])
    vs = np.stack([W.qkv(w, "v", b) for b in range(w["batch"])])
    dos = np.stack([W.qkv(w, "do", b) for b in range(w["batch"])]) if with_do else None
    return qs, ks, vs, dos


def gzip_flags_product(sa, w: dict) -> np.ndarray:
    """Literal flags as the library's host path computes them."""
    if w.get("flags_from") == "bernoulli":
        return W.bernoulli_flags(w)
    return np.stack([sa.literal_flags(W.workload_bytes(w, b), w["block"]) for b in range(w["batch"])])


def gzip_flags_oracle(w: dict) -> np.ndarray:
    if w.get("flags_from") == "bernoulli":
        return W.bernoulli_flags(w)
    return np.stack([G.literal_flags(W.workload_bytes(w, b), w["block"]) for b in range(w["batch"])])


def sample_rows(N: int, n: int, seed: int, tile: int = 128) -> np.ndarray:
    rng = np.random.default_rng(seed)
    fixed = [0, 1, N - 1] + [t * tile - 1 for t in (1, 2) if t * tile - 1 < N] + \
            [t * tile for t in (1, 2) if t * tile < N]
    return np.unique(np.concatenate([fixed, rng.choice(N, size=min(n, N), replace=False)]))


# ------------------------------------------------------------------ gist
def gist_layout(N, sinks, ratio, flags=None, tile=128):
    g = Gi.gist_flags(N, sinks, ratio) if flags is None else np.asarray(flags, bool)
    perm = Gi.shift_permutation(g, tile)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm), dtype=perm.dtype)
    return g, perm, inv
