"""Pins for the oracle's fixed-Huffman DEFLATE block sizes (CPU only): the
specification's length and distance tables, a closed form, and a real
bitstream written from the oracle's parse that zlib's decoder must inflate
back to the block, with exactly the oracle's bit count."""
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
    assert F.block_bits(bytes(128)) == 3 + 8 + 12 + 5 + 7
    assert F.block_size(bytes(128)) == 5


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
        w = encode(blk)
        assert len(w.bits) == F.block_bits(blk)
        assert zlib.decompress(w.data(), -15) == blk


def test_flags_track_zlib_on_the_mixed_workload_bytes():
    """An estimate, not zlib: on the text/random mix of the 64K workload the
    block sizes correlate with zlib level 1's (r >= 0.98) and the flags agree
    on at least 90% of the blocks; the disagreements are text blocks within a
    few bytes of the mean."""
    w = W.WORKLOADS["gzip_64k_fwdbwd"]
    for bt in range(w["batch"]):
        x = W.workload_bytes(w, bt)
        ours, ref = F.block_sizes(x, w["block"]), np.array(G.block_compressed_sizes(x, w["block"]))
        assert np.corrcoef(ours, ref)[0, 1] >= 0.98
        agree = (F.literal_flags(x, w["block"]) == G.literal_flags(x, w["block"])).mean()
        assert agree >= 0.9, (bt, agree)
