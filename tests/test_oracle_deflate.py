"""Pins for the oracle's DEFLATE block sizes (CPU only): the specification's
length and distance tables, closed forms, real bitstreams of all three block
types written from the oracle's parse and codes that zlib's decoder must
inflate back to the block with exactly the oracle's bit count, and the
optimality of the Huffman and length-limited code lengths (against an
independent heap construction and brute force)."""
import heapq
import itertools
import zlib

import numpy as np
import pytest

import sa_workloads as W
from oracle import deflate_size as F
from oracle import gzip_mask as G


def test_spec_tables():
    # RFC 1951 section 3.2.5
    assert F.length_symbol(3) == (257, 0) and F.length_symbol(10) == (264, 0)
    assert F.length_symbol(11) == (265, 0) and F.length_symbol(12) == (265, 1)
    assert F.length_symbol(115) == (280, 0) and F.length_symbol(130) == (280, 15)
    assert F.length_symbol(257) == (284, 30) and F.length_symbol(258) == (285, 0)
    assert F.distance_code(1) == (0, 0) and F.distance_code(4) == (3, 0)
    assert F.distance_code(5) == (4, 0) and F.distance_code(6) == (4, 1)
    assert F.distance_code(32768) == (29, 8191)
    # every length and distance has exactly one code
    for n in range(3, 259):
        s, e = F.length_symbol(n)
        assert 0 <= e < 2 ** F.LEN_EXTRA[s - 257] or (e == 0 and F.LEN_EXTRA[s - 257] == 0)
    for dist in range(1, 32769, 7):
        c, e = F.distance_code(dist)
        assert 0 <= e < max(1, 2 ** F.DIST_EXTRA[c])


def test_zero_block_closed_form():
    # one literal (8 bits), one match of 127 at distance 1 (symbol 280: 8 + 4
    # extra bits; distance code 0: 5 bits), 3 header bits, 7 for end of block
    assert F.fixed_block_bits(bytes(128)) == 3 + 8 + 12 + 5 + 7
    assert F.block_bits(bytes(128)) == 35  # the fixed block is the smallest
    assert F.block_size(bytes(128)) == 5
    # a stored block: 3 header bits, 5 of padding, LEN and NLEN, the bytes
    assert F.stored_block_bits(bytes(7)) == 40 + 56


class BitWriter:
    def __init__(self):
        self.bits = []

    def lsb(self, v, n):  # extra bits and header fields: least significant first
        self.bits += [(v >> i) & 1 for i in range(n)]

    def huff(self, code, n):  # Huffman codes: most significant first
        self.bits += [(code >> (n - 1 - i)) & 1 for i in range(n)]

    def data(self):
        b = self.bits + [0] * (-len(self.bits) % 8)
        return bytes(sum(b[i + j] << j for j in range(8)) for i in range(0, len(b), 8))


def fixed_code(sym):
    """RFC 1951 section 3.2.6 fixed literal/length code of a symbol."""
    if sym <= 143:
        return 0x30 + sym, 8
    if sym <= 255:
        return 0x190 + sym - 144, 9
    if sym <= 279:
        return sym - 256, 7
    return 0xC0 + sym - 280, 8


def canonical_codes(lengths):
    """RFC 1951 section 3.2.2: codes from code lengths."""
    mx = max(lengths)
    bl = [0] * (mx + 1)
    for L in lengths:
        if L:
            bl[L] += 1
    code, nxt = 0, [0] * (mx + 2)
    for bits in range(1, mx + 1):
        code = (code + bl[bits - 1]) << 1
        nxt[bits] = code
    out = [None] * len(lengths)
    for sym, L in enumerate(lengths):
        if L:
            out[sym] = (nxt[L], L)
            nxt[L] += 1
    return out


def encode_dynamic(block):
    toks, Lll, Ldd, hlit, hdist, runs, Lcl, hclen = F.dynamic_code(block)
    cll, cdd, ccl = canonical_codes(Lll), canonical_codes(Ldd), canonical_codes(Lcl)
    w = BitWriter()
    w.lsb(1, 1)  # final block
    w.lsb(2, 2)  # dynamic Huffman codes
    w.lsb(hlit - 257, 5)
    w.lsb(hdist - 1, 5)
    w.lsb(hclen - 4, 4)
    for sym in F.CL_ORDER[:hclen]:
        w.lsb(Lcl[sym], 3)
    for sym, extra, nb in runs:
        w.huff(*ccl[sym])
        w.lsb(extra, nb)
    for t in toks:
        if t[0] == "lit":
            w.huff(*cll[t[1]])
        else:
            s, e = F.length_symbol(t[1])
            w.huff(*cll[s])
            w.lsb(e, F.LEN_EXTRA[s - 257])
            c, e = F.distance_code(t[2])
            w.huff(*cdd[c])
            w.lsb(e, F.DIST_EXTRA[c])
    w.huff(*cll[256])
    return w


def encode_stored(block):
    w = BitWriter()
    w.lsb(1, 1)  # final block
    w.lsb(0, 2)  # stored
    w.lsb(0, 5)  # to the byte boundary
    w.lsb(len(block), 16)
    w.lsb(len(block) ^ 0xFFFF, 16)
    for byte in block:
        w.lsb(byte, 8)
    return w


def encode(block):
    w = BitWriter()
    w.lsb(1, 1)  # final block
    w.lsb(1, 2)  # fixed Huffman codes
    for t in F.parse(block):
        if t[0] == "lit":
            w.huff(*fixed_code(t[1]))
        else:
            s, e = F.length_symbol(t[1])
            w.huff(*fixed_code(s))
            w.lsb(e, F.LEN_EXTRA[s - 257])
            c, e = F.distance_code(t[2])
            w.huff(c, 5)
            w.lsb(e, F.DIST_EXTRA[c])
    w.huff(*fixed_code(256))
    return w


@pytest.mark.parametrize("kind", ["random", "text", "zeros", "mixed", "periodic"])
def test_bitstream_inflates_to_the_block_with_the_oracles_bit_count(kind):
    rng = np.random.default_rng(3)
    if kind == "random":
        blocks = [rng.integers(0, 256, 200, dtype=np.uint8).tobytes() for _ in range(5)]
    elif kind == "text":
        blocks = [W.workload_bytes(W.WORKLOADS["gzip_64k_fwdbwd"], 0)[i * 128:(i + 1) * 128] for i in range(0, 512, 37)]
    elif kind == "zeros":
        blocks = [bytes(n) for n in (1, 2, 3, 4, 259, 300, 40000)]
    elif kind == "periodic":
        blocks = [(b"abcabcabd" * 5000)[:n] for n in (9, 100, 33000)]
    else:
        blocks = [bytes(rng.integers(0, 4, 3000, dtype=np.uint8)) + b"hello world " * 30]
    for blk in blocks:
        for w, bits in ((encode(blk), F.fixed_block_bits(blk)),
                        (encode_dynamic(blk), F.dynamic_block_bits(blk))):
            assert len(w.bits) == bits
            assert zlib.decompress(w.data(), -15) == blk
        if len(blk) < 65536:
            w = encode_stored(blk)
            assert len(w.bits) == F.stored_block_bits(blk)
            assert zlib.decompress(w.data(), -15) == blk


def heap_huffman_cost(freq):
    """Total weighted length of an optimal prefix code, by an independent heap
    construction of Huffman's algorithm (sum of the merged weights)."""
    h = [f for f in freq if f > 0]
    if len(h) == 1:
        return h[0]
    heapq.heapify(h)
    cost = 0
    while len(h) > 1:
        a, b = heapq.heappop(h), heapq.heappop(h)
        cost += a + b
        heapq.heappush(h, a + b)
    return cost


@pytest.mark.parametrize("seed", range(6))
def test_huffman_lengths_are_optimal_and_complete(seed):
    rng = np.random.default_rng(seed)
    freq = [int(x) for x in rng.integers(0, 40, 60) * (rng.random(60) < 0.6)]
    L = F.huffman_lengths(freq, 15)
    used = [i for i, f in enumerate(freq) if f]
    assert all((L[i] > 0) == (freq[i] > 0) for i in range(len(freq)))
    assert sum(2.0 ** -L[i] for i in used) == 1.0  # a complete code (Kraft equality)
    assert sum(f * l for f, l in zip(freq, L)) == heap_huffman_cost(freq)


def test_length_limited_code_is_optimal_by_brute_force():
    # Fibonacci weights force depth len - 1 without a limit; with a limit of 4
    # the package-merge lengths must reach the least cost of every length
    # assignment that satisfies Kraft's inequality within the limit
    freq = [1, 1, 2, 3, 5, 8, 13, 21]
    L = F.huffman_lengths(freq, 4)
    assert max(L) <= 4 and sum(2.0 ** -l for l in L) <= 1.0
    best = min(sum(f * l for f, l in zip(freq, ls))
               for ls in itertools.product(range(1, 5), repeat=len(freq))
               if sum(2.0 ** -l for l in ls) <= 1.0)
    assert sum(f * l for f, l in zip(freq, L)) == best
    assert max(F.huffman_lengths(freq, 15)) == len(freq) - 1


def test_single_and_missing_distance_codes():
    # one used symbol gets a 1-bit code; all literals: one zero-length distance code
    assert F.huffman_lengths([0, 5, 0], 15) == [0, 1, 0]
    _, _, Ldd, _, hdist, _, _, _ = F.dynamic_code(bytes(range(50)))
    assert hdist == 1 and Ldd[0] == 0


def test_length_runs_follow_the_specification():
    runs = F.length_runs([0] * 150 + [5] * 8 + [0, 0] + [3])
    # 150 zeros: 138 (the longest run of code 18) then 12; eight 5s: one
    # literal length, a repeat of 6 (code 16, the longest) and one more; runs
    # shorter than 3 are sent as literal lengths
    assert runs == [(18, 127, 7), (18, 1, 7), (5, 0, 0), (16, 3, 2), (5, 0, 0),
                    (0, 0, 0), (0, 0, 0), (3, 0, 0)]
    out = []
    for sym, extra, nb in runs:
        assert 0 <= extra < (1 << nb) if nb else extra == 0
        if sym == 18:
            out += [0] * (11 + extra)
        elif sym == 17:
            out += [0] * (3 + extra)
        elif sym == 16:
            out += [out[-1]] * (3 + extra)
        else:
            out.append(sym)
    assert out == [0] * 150 + [5] * 8 + [0, 0] + [3]


def test_long_match_inside_is_not_entered():
    # "abcdefgh" twice: the second copy is one match of 8 (distance 8) whose
    # inside positions 9..15 are not entered; "cdefgh" at 16 must then take
    # the literal-visited position 2 (distance 14), not 10 (distance 6)
    toks = F.parse(b"abcdefgh" * 2 + b"cdefgh")
    assert toks == [("lit", c) for c in b"abcdefgh"] + [("match", 8, 8), ("match", 6, 14)]
    # a short match (4 bytes) enters its inside: "bcd" at 9 finds position 5
    toks = F.parse(b"abcdxabcdybcd")
    assert toks[-1] == ("match", 3, 4)
    assert toks == [("lit", c) for c in b"abcdx"] + [("match", 4, 5), ("lit", ord("y")), ("match", 3, 4)]


def test_flags_track_zlib_on_the_workload_bytes():
    """An estimate, not zlib: on the tiny workload's bytes and on the
    text/random mix of the 64K workload the block sizes correlate with zlib
    level 1's (r >= 0.99) and the flags agree on every block."""
    for name in ("gzip_tiny_fp32", "gzip_64k_fwdbwd"):
        w = W.WORKLOADS[name]
        for bt in range(w["batch"]):
            x = W.workload_bytes(w, bt)
            ours, ref = F.block_sizes(x, w["block"]), np.array(G.block_compressed_sizes(x, w["block"]))
            assert np.corrcoef(ours, ref)[0, 1] >= 0.99
            agree = (F.literal_flags(x, w["block"]) == G.literal_flags(x, w["block"])).mean()
            assert agree == 1.0, (name, bt, agree)
