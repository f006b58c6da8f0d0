"""Per-block compressed size by a fixed-Huffman DEFLATE coder (oracle; test
infrastructure only).

The method's pages rank blocks by their gzip level-1 size ("Gzip-guided
sparse attention: Selecting long-range content by compressibility", Core
equations: r_i = |gzip(block_i)| / b and the flag rule). Computing that size
on the GPU means running a deflate encoder there. zlib's own level-1 encoder
is not restated here; this module defines a plain DEFLATE encoder from the
format's specification ("RFC 1951: DEFLATE Compressed Data Format
Specification version 1.3"), and its sizes are an ESTIMATE of zlib's, not
equal to them. The definition, which the device kernel follows exactly:

* every block is compressed on its own into one final block with the fixed
  Huffman codes (RFC 1951 section 3.2.6): 3 header bits, the symbols, and
  the end-of-block symbol 256;
* greedy LZ77 parse from the block's first byte: at position p the match
  candidate is the nearest earlier position q with x[q:q+3] == x[p:p+3] and
  p - q <= 32768; the match length is the common prefix of x[q:] and x[p:],
  at most 258 and within the block; a match of 3 or more bytes is emitted
  and the parse moves past it, otherwise the byte is a literal;
* code lengths (section 3.2.6): literals 0..143 take 8 bits, 144..255 take
  9; length symbols 256..279 take 7 bits and 280..287 take 8; a distance
  code takes 5 bits; plus the extra bits of section 3.2.5's length and
  distance tables;
* the size in bytes is ceil(bits / 8). A container (zlib or gzip header and
  trailer) would add the same bytes to every block, which a comparison with
  the mean ignores.
"""
from __future__ import annotations

import numpy as np

# RFC 1951 section 3.2.5: length symbols 257..285 and distance codes 0..29
LEN_BASE = [3, 4, 5, 6, 7, 8, 9, 10, 11, 13, 15, 17, 19, 23, 27, 31, 35, 43, 51, 59,
            67, 83, 99, 115, 131, 163, 195, 227, 258]
LEN_EXTRA = [0] * 8 + [1] * 4 + [2] * 4 + [3] * 4 + [4] * 4 + [5] * 4 + [0]
DIST_BASE = [1, 2, 3, 4, 5, 7, 9, 13, 17, 25, 33, 49, 65, 97, 129, 193, 257, 385, 513, 769,
             1025, 1537, 2049, 3073, 4097, 6145, 8193, 12289, 16385, 24577]
DIST_EXTRA = [0, 0, 0, 0, 1, 1, 2, 2, 3, 3, 4, 4, 5, 5, 6, 6, 7, 7, 8, 8, 9, 9, 10, 10,
              11, 11, 12, 12, 13, 13]


def length_symbol(n: int) -> tuple[int, int]:
    """(symbol 257..285, extra-bit value) for a match length 3..258."""
    for i in range(len(LEN_BASE) - 1, -1, -1):
        if n >= LEN_BASE[i]:
            return 257 + i, n - LEN_BASE[i]
    raise ValueError(n)


def distance_code(dist: int) -> tuple[int, int]:
    """(code 0..29, extra-bit value) for a distance 1..32768."""
    for i in range(len(DIST_BASE) - 1, -1, -1):
        if dist >= DIST_BASE[i]:
            return i, dist - DIST_BASE[i]
    raise ValueError(dist)


def literal_bits(v: int) -> int:
    return 8 if v <= 143 else 9


def symbol_bits(sym: int) -> int:
    """Fixed code length of a length symbol (256..287)."""
    return 7 if sym <= 279 else 8


def parse(block: bytes) -> list[tuple]:
    """Greedy parse: ('lit', byte) and ('match', length, distance) tokens."""
    x = bytes(block)
    n = len(x)
    last: dict[bytes, int] = {}
    cand = [-1] * n  # nearest earlier position with the same three bytes
    for p in range(n - 2):
        key = x[p:p + 3]
        q = last.get(key, -1)
        cand[p] = q if q >= 0 and p - q <= 32768 else -1
        last[key] = p
    out, p = [], 0
    while p < n:
        q = cand[p]
        m = 0
        if q >= 0:
            while p + m < n and m < 258 and x[q + m] == x[p + m]:
                m += 1
        if m >= 3:
            out.append(("match", m, p - q))
            p += m
        else:
            out.append(("lit", x[p]))
            p += 1
    return out


def token_bits(tok) -> int:
    if tok[0] == "lit":
        return literal_bits(tok[1])
    sym, _ = length_symbol(tok[1])
    dc, _ = distance_code(tok[2])
    return symbol_bits(sym) + LEN_EXTRA[sym - 257] + 5 + DIST_EXTRA[dc]


def block_bits(block: bytes) -> int:
    """Bits of the one fixed-Huffman final block: header, symbols, end of block."""
    return 3 + sum(token_bits(t) for t in parse(block)) + symbol_bits(256)


def block_size(block: bytes) -> int:
    return (block_bits(block) + 7) // 8


def block_sizes(x: bytes, b: int) -> np.ndarray:
    if len(x) % b:
        raise ValueError("byte length must be a multiple of the block size")
    return np.array([block_size(x[i:i + b]) for i in range(0, len(x), b)], dtype=np.int64)


def literal_flags(x: bytes, b: int) -> np.ndarray:
    """l_i = 1[c_i * B > sum_j c_j] on these sizes (integer comparison)."""
    c = block_sizes(x, b)
    return (c * len(c) > c.sum()).astype(np.uint8)
