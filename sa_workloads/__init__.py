"""Seeded synthetic inputs for the five workloads of this library.

This module is shared by the CUDA path's tests/bench and by the CPU oracle.
It holds no arithmetic of the attention method itself: it only draws random
bytes, Bernoulli flags and N(0,1) tensors, and rounds floats to bfloat16.

Every tensor is drawn from its own NumPy ``SeedSequence`` keyed by
``(1000 + workload index, stream id, *slice indices)``, so any slice (one
batch row, one decode sequence/head) can be regenerated alone and both sides
see the same values without materialising the whole workload.

Workloads (sizes and value distributions follow the method's published
settings; no real corpus is used anywhere):

1. ``gzip_tiny_fp32`` - 256 bytes, block 16, window 1, 4 heads, d=32, fp32.
2. ``gzip_8k``        - batch 8, N=8192, block 64, window 2, 8 heads, d=64,
                        bf16, Bernoulli(0.3) literal flags with block 0 literal.
3. ``gist_prefill_32k`` - batch 1, 32768 positions, 128 sinks, ratio 4,
                        window 128, 32 q / 8 kv heads, d=128, bf16.
4. ``gist_decode_128k`` - 16 sequences, 131072-token cache, 32-token chunks,
                        4096 gists, top-64, window 512, 32 q / 8 kv heads.
5. ``gzip_64k_fwdbwd`` - batch 2, N=65536, block 128, window 2, 16 heads,
                        d=128, bf16, flags from synthetic mixed text/random bytes.
8. ``gzip_flags_128m``  - on-device literal flags: the 64K workload's two byte
                        rows repeated to 2048 rows of 64 KiB (128 MiB), b=128.
7. ``gist_hier_decode_128k`` - gist-of-gist decode over the decode workload's
                        cache shape: 32 chunk gists per level-2 gist (128 of
                        them), top-8 groups, then top-64 chunks, window 512.
6. ``gist_coarse_20k`` - segment-wise coarse gist layout: 16 segments of 1024
                        raw tokens, each followed by 256 gists (ratio 4), no
                        sinks (20480 positions), 32 q / 8 kv heads, d=128, bf16.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

# stream ids: one per independently drawn tensor
S_BYTES, S_FLAGS, S_Q, S_K, S_V, S_DO, S_GK, S_GV, S_RK, S_RV, S_VOCAB, S_G2K, S_G2V = range(13)

WORKLOADS = {
    "gzip_tiny_fp32": dict(index=1, kind="gzip", batch=1, seq_len=256, block=16,
                           window=1, heads=4, kv_heads=4, head_dim=32,
                           dtype="fp32", flags_from="bytes_pattern"),
    "gzip_8k": dict(index=2, kind="gzip", batch=8, seq_len=8192, block=64,
                    window=2, heads=8, kv_heads=8, head_dim=64, dtype="bf16",
                    flags_from="bernoulli", p_literal=0.3),
    "gist_prefill_32k": dict(index=3, kind="gist", batch=1, seq_len=32768,
                             sinks=128, ratio=4, window=128, heads=32,
                             kv_heads=8, head_dim=128, dtype="bf16", tile=128,
                             gist_tail=32),
    "gist_decode_128k": dict(index=4, kind="decode", n_seq=16, cache_len=131072,
                             chunk=32, n_gists=4096, top_k=64, window=512,
                             heads=32, kv_heads=8, head_dim=128, dtype="bf16"),
    "gist_coarse_20k": dict(index=6, kind="gist", batch=1, seq_len=20480,
                            sinks=0, ratio=4, window=0, gist_segment=1024, heads=32,
                            kv_heads=8, head_dim=128, dtype="bf16", tile=128, gist_tail=32),
    "gist_hier_decode_128k": dict(index=7, kind="hier", n_seq=16, cache_len=131072,
                                  chunk=32, n_gists=4096, fanout=32, top_k2=8, top_k=64,
                                  window=512, heads=32, kv_heads=8, head_dim=128, dtype="bf16"),
    "gzip_flags_128m": dict(index=8, kind="flags", rows_from="gzip_64k_fwdbwd", batch=2048,
                            n_bytes=65536, block=128),
    "gzip_64k_fwdbwd": dict(index=5, kind="gzip", batch=2, seq_len=65536,
                            block=128, window=2, heads=16, kv_heads=16,
                            head_dim=128, dtype="bf16", flags_from="bytes_mixed",
                            segment=4096, p_random=0.4, vocab_words=16),
}


def rng(index: int, stream: int, *idx: int) -> np.random.Generator:
    """Independent generator for one tensor (or one slice of it)."""
    return np.random.default_rng([1000 + int(index), int(stream), *map(int, idx)])


# ----------------------------------------------------------------- bf16 helpers
def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); fp32 out."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def normal(index: int, stream: int, shape, bf16: bool, *idx: int) -> np.ndarray:
    x = rng(index, stream, *idx).standard_normal(size=shape, dtype=np.float32)
    return round_to_bf16(x) if bf16 else x


# ------------------------------------------------------------- byte sequences
def bytes_pattern(index: int, n_bytes: int = 256, run: int = 32) -> bytes:
    """Alternating runs: even runs repeat a seeded 8-byte pattern, odd runs are
    uniform random bytes (the tiny workload's byte stream)."""
    g = rng(index, S_BYTES, 0)
    pat = g.integers(0, 256, size=8, dtype=np.uint8)
    out = []
    for r in range(n_bytes // run):
        if r % 2 == 0:
            out.append(np.tile(pat, run // 8))
        else:
            out.append(g.integers(0, 256, size=run, dtype=np.uint8))
    return bytes(np.concatenate(out).tobytes())


def vocabulary(index: int, n_words: int) -> list[bytes]:
    g = rng(index, S_VOCAB)
    words = []
    for _ in range(n_words):
        n = int(g.integers(3, 9))
        words.append(bytes((g.integers(0, 26, size=n) + ord("a")).astype(np.uint8).tobytes()))
    return words


def bytes_mixed(index: int, batch_row: int, n_bytes: int, segment: int,
                p_random: float, n_words: int) -> bytes:
    """Segments of ``segment`` bytes; each is uniform random bytes with
    probability ``p_random``, else space-separated words drawn uniformly from a
    small seeded vocabulary (low-entropy text)."""
    words = vocabulary(index, n_words)
    g = rng(index, S_BYTES, batch_row)
    out = bytearray()
    for _ in range(n_bytes // segment):
        if g.random() < p_random:
            out += g.integers(0, 256, size=segment, dtype=np.uint8).tobytes()
        else:
            seg = bytearray()
            while len(seg) < segment:
                seg += words[int(g.integers(0, n_words))] + b" "
            out += seg[:segment]
    return bytes(out)


def _w(w) -> dict:
    return WORKLOADS[w] if isinstance(w, str) else w


def workload_bytes(w, batch_row: int) -> bytes:
    w = _w(w)
    if w.get("flags_from") == "bytes_pattern":
        return bytes_pattern(w["index"], w["seq_len"])
    if w.get("flags_from") == "bytes_mixed":
        return bytes_mixed(w["index"], batch_row, w["seq_len"], w["segment"],
                           w["p_random"], w["vocab_words"])
    raise ValueError("workload has no byte stream")


def bernoulli_flags(w) -> np.ndarray:
    """uint8 [batch, B] literal flags drawn Bernoulli(p), block 0 forced to 1."""
    w = _w(w)
    B = w["seq_len"] // w["block"]
    g = rng(w["index"], S_FLAGS)
    f = (g.random((w["batch"], B)) < w["p_literal"]).astype(np.uint8)
    f[:, 0] = 1
    return f


# ------------------------------------------------------------ tensor draws
def qkv(w, which: str, batch_row: int, head: int | None = None) -> np.ndarray:
    """Q, K, V or dO of one batch row. Each (batch row, head) slice [N, d] is
    its own stream; with ``head=None`` all heads are drawn (in threads) and
    stacked to the [N, heads, d] layout (one BSHD batch slice)."""
    w = _w(w)
    stream = {"q": S_Q, "k": S_K, "v": S_V, "do": S_DO}[which]
    bf16 = w["dtype"] == "bf16"
    shape = (w["seq_len"], w["head_dim"])
    if head is not None:
        return normal(w["index"], stream, shape, bf16, batch_row, head)
    h = w["heads"] if which in ("q", "do") else w["kv_heads"]
    out = np.empty((w["seq_len"], h, w["head_dim"]), np.float32)

    def one(hh):
        out[:, hh, :] = normal(w["index"], stream, shape, bf16, batch_row, hh)

    with ThreadPoolExecutor(max_workers=min(h, 16)) as ex:
        list(ex.map(one, range(h)))
    return out


def decode_query(w) -> np.ndarray:
    """[n_seq, heads, d] - one new query token per sequence."""
    w = _w(w)
    return normal(w["index"], S_Q, (w["n_seq"], w["heads"], w["head_dim"]), True)


def decode_gists(w, seq: int, which: str) -> np.ndarray:
    """Gist K or V of one sequence: [kv_heads, n_gists, d]."""
    w = _w(w)
    stream = S_GK if which == "k" else S_GV
    return normal(w["index"], stream, (w["kv_heads"], w["n_gists"], w["head_dim"]), True, seq)


def decode_gists2(w, seq: int, which: str) -> np.ndarray:
    """Level-2 gist K or V of one sequence (gist of gists): [kv_heads, n_gists / fanout, d]."""
    w = _w(w)
    stream = S_G2K if which == "k" else S_G2V
    return normal(w["index"], stream, (w["kv_heads"], w["n_gists"] // w["fanout"], w["head_dim"]),
                  True, seq)


def decode_raw(w, seq: int, kv_head: int, which: str) -> np.ndarray:
    """Raw K or V cache of one (sequence, kv head): [cache_len, d]."""
    w = _w(w)
    stream = S_RK if which == "k" else S_RV
    return normal(w["index"], stream, (w["cache_len"], w["head_dim"]), True, seq, kv_head)


def scaled(name: str, **overrides) -> dict:
    """A copy of a workload's parameters with some sizes overridden (used for
    the smaller parity cases that keep the same structure). ``index`` may be
    overridden too, to draw different values for the same shapes."""
    w = dict(WORKLOADS[name])
    w.update(overrides)
    return w
