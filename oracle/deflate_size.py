"""Per-block compressed size by a plain DEFLATE coder (oracle; test
infrastructure only).

The method's pages rank blocks by their gzip level-1 size ("Gzip-guided
sparse attention: Selecting long-range content by compressibility", Core
equations: r_i = |gzip(block_i)| / b and the flag rule). Computing that size
on the GPU means running a deflate encoder there. zlib's own level-1 encoder
is not restated here; this module defines a plain DEFLATE encoder from the
format's specification ("RFC 1951: DEFLATE Compressed Data Format
Specification version 1.3"), and its sizes are an ESTIMATE of zlib's, not
equal to them. The definition, which the device kernel follows exactly:

* every block is compressed on its own into one final block, whichever of
  the three block types of the specification is smallest;
* greedy LZ77 parse from the block's first byte, with the candidate table of
  the specification's section 4 in its fast form (new strings are entered
  only where no match was found or the match was short): at position p the
  match candidate is the most recent ENTERED position q with x[q:q+3] ==
  x[p:p+3] and p - q <= 32768; the match length is the common prefix of
  x[q:] and x[p:], at most 258 and within the block; a match of 3 or more
  bytes is emitted and the parse moves past it, otherwise the byte is a
  literal. Every position the parse stops at is entered after its lookup,
  and so is every position inside a match of at most MAX_INSERT (4) bytes;
  the inside of a longer match is not;
* fixed Huffman codes (section 3.2.6): literals 0..143 take 8 bits, 144..255
  take 9; length symbols 256..279 take 7 bits and 280..287 take 8; a distance
  code takes 5 bits; plus the extra bits of section 3.2.5's length and
  distance tables; 3 header bits and the end-of-block symbol 256;
* dynamic Huffman codes (section 3.2.7): code lengths for the symbols the
  parse uses (end of block included) by Huffman's construction (the optimal
  prefix code; at most 15 bits, else the optimal length-limited code), sent
  as run-length coded code lengths (`length_runs`) under a third code of at
  most 7 bits; header fields HLIT, HDIST, HCLEN as the specification lays
  them out;
* stored (section 3.2.4): 3 header bits, padding to the byte, LEN and NLEN,
  the bytes;
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


MAX_INSERT = 4  # longest match whose inside positions are entered


def parse(block: bytes) -> list[tuple]:
    """Greedy parse: ('lit', byte) and ('match', length, distance) tokens."""
    x = bytes(block)
    n = len(x)
    last: dict[bytes, int] = {}  # three bytes -> most recent entered position

    def enter(i):
        if i + 3 <= n:
            last[x[i:i + 3]] = i

    out, p = [], 0
    while p < n:
        q = last.get(x[p:p + 3], -1) if p + 3 <= n else -1
        m = 0
        if q >= 0 and p - q <= 32768:
            while p + m < n and m < 258 and x[q + m] == x[p + m]:
                m += 1
        if m >= 3:
            out.append(("match", m, p - q))
            for i in range(p, p + (m if m <= MAX_INSERT else 1)):
                enter(i)
            p += m
        else:
            out.append(("lit", x[p]))
            enter(p)
            p += 1
    return out


def token_bits(tok) -> int:
    if tok[0] == "lit":
        return literal_bits(tok[1])
    sym, _ = length_symbol(tok[1])
    dc, _ = distance_code(tok[2])
    return symbol_bits(sym) + LEN_EXTRA[sym - 257] + 5 + DIST_EXTRA[dc]


def fixed_block_bits(block: bytes) -> int:
    """Bits of the one fixed-Huffman final block: header, symbols, end of block."""
    return 3 + sum(token_bits(t) for t in parse(block)) + symbol_bits(256)


def stored_block_bits(block: bytes) -> int:
    """Bits of one stored final block starting a stream: 3 header bits, 5 bits
    of padding to the byte boundary, LEN and NLEN, then the bytes."""
    return 3 + 5 + 32 + 8 * len(block)


# RFC 1951 section 3.2.7: order in which the code-length code lengths are sent
CL_ORDER = [16, 17, 18, 0, 8, 7, 9, 6, 10, 5, 11, 4, 12, 3, 13, 2, 14, 1, 15]


def huffman_lengths(freq, limit: int) -> list[int]:
    """Code lengths of a prefix code for the symbols with freq > 0.

    Huffman's construction with two queues: the leaves in ascending (frequency,
    symbol) order, the merged nodes in the order they are made; every step joins
    the two lightest queue fronts, taking a leaf before a merged node of equal
    weight. A symbol's length is its leaf's depth. One used symbol gets length 1
    (the specification's rule for a single distance code). When the longest
    code exceeds `limit`, the package-merge construction (Larmore and
    Hirschberg, 1990: the optimal lengths within a limit) replaces it, its
    lists ordered by weight with leaves before packages of equal weight.
    """
    n = len(freq)
    L = [0] * n
    leaves = sorted((f, s) for s, f in enumerate(freq) if f > 0)
    if not leaves:
        return L
    if len(leaves) == 1:
        L[leaves[0][1]] = 1
        return L
    # nodes: leaves 0..m-1, merged nodes m.. with parent links
    m = len(leaves)
    weight = [f for f, _ in leaves]
    parent = [-1] * m
    internal = []  # indices of merged nodes, in creation order
    li = ii = 0

    def take():
        nonlocal li, ii
        if li < m and (ii >= len(internal) or weight[li] <= weight[internal[ii]]):
            li += 1
            return li - 1
        ii += 1
        return internal[ii - 1]

    for _ in range(m - 1):
        a = take()
        b = take()
        node = len(weight)
        weight.append(weight[a] + weight[b])
        parent.append(-1)
        parent[a] = parent[b] = node
        internal.append(node)
    depth = [0] * len(weight)
    for node in reversed(range(len(weight) - 1)):  # parents come after children
        depth[node] = depth[parent[node]] + 1
    for k, (_, sym) in enumerate(leaves):
        L[sym] = depth[k]
    if max(L) <= limit:
        return L
    # package-merge
    items = [(f, 0, [sym]) for f, sym in leaves]  # (weight, kind: 0 leaf 1 package, symbols)
    cur = list(items)
    for _ in range(limit - 1):
        pk = [(cur[i][0] + cur[i + 1][0], 1, cur[i][2] + cur[i + 1][2])
              for i in range(0, len(cur) - 1, 2)]
        cur = sorted(items + pk, key=lambda t: (t[0], t[1]))
    L = [0] * n
    for _, _, syms in cur[:2 * m - 2]:
        for sym in syms:
            L[sym] += 1
    return L


def length_runs(lengths) -> list[tuple[int, int, int]]:
    """Run-length coding of a code-length sequence (section 3.2.7 symbols):
    (symbol, extra-bit value, extra-bit count). A run of zeros is sent as
    symbol 18 (11..138 zeros) while at least 11 remain, then 17 (3..10), then
    single 0s; a run of a non-zero length sends the length once, then 16
    (3..6 repeats) while at least 3 repeats remain, then the length again."""
    out, i, n = [], 0, len(lengths)
    while i < n:
        v = lengths[i]
        j = i
        while j < n and lengths[j] == v:
            j += 1
        run = j - i
        if v == 0:
            while run >= 11:
                t = min(run, 138)
                out.append((18, t - 11, 7))
                run -= t
            if run >= 3:
                out.append((17, run - 3, 3))
                run = 0
            out += [(0, 0, 0)] * run
        else:
            out.append((v, 0, 0))
            run -= 1
            while run >= 3:
                t = min(run, 6)
                out.append((16, t - 3, 2))
                run -= t
            out += [(v, 0, 0)] * run
        i = j
    return out


def dynamic_code(block: bytes):
    """The dynamic block's parse and codes: (tokens, literal/length lengths,
    distance lengths, HLIT, HDIST, run-length symbols, code-length lengths,
    HCLEN)."""
    toks = parse(block)
    ll, dd = [0] * 286, [0] * 30
    for t in toks:
        if t[0] == "lit":
            ll[t[1]] += 1
        else:
            ll[length_symbol(t[1])[0]] += 1
            dd[distance_code(t[2])[0]] += 1
    ll[256] += 1
    Lll, Ldd = huffman_lengths(ll, 15), huffman_lengths(dd, 15)
    hlit = max(257, max(i for i, v in enumerate(Lll) if v) + 1)
    used_d = [i for i, v in enumerate(Ldd) if v]
    hdist = max(1, used_d[-1] + 1) if used_d else 1
    runs = length_runs(Lll[:hlit] + Ldd[:hdist])
    cf = [0] * 19
    for sym, _, _ in runs:
        cf[sym] += 1
    Lcl = huffman_lengths(cf, 7)
    hclen = max(4, max(k for k, sym in enumerate(CL_ORDER) if Lcl[sym]) + 1)
    return toks, Lll, Ldd, hlit, hdist, runs, Lcl, hclen


def dynamic_block_bits(block: bytes) -> int:
    """Bits of one dynamic-Huffman final block: header fields, the code-length
    code, the run-length coded lengths, the symbols with their extra bits and
    the end of block."""
    toks, Lll, Ldd, hlit, hdist, runs, Lcl, hclen = dynamic_code(block)
    bits = 3 + 5 + 5 + 4 + 3 * hclen + sum(Lcl[s] + nb for s, _, nb in runs)
    for t in toks:
        if t[0] == "lit":
            bits += Lll[t[1]]
        else:
            s, _ = length_symbol(t[1])
            c, _ = distance_code(t[2])
            bits += Lll[s] + LEN_EXTRA[s - 257] + Ldd[c] + DIST_EXTRA[c]
    return bits + Lll[256]


def block_bits(block: bytes) -> int:
    """Bits of the smallest of the three final blocks."""
    return min(fixed_block_bits(block), dynamic_block_bits(block), stored_block_bits(block))


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
