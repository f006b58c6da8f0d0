"""The device compressor reaches the oracle's DEFLATE definition by other
steps than the oracle takes; these CPU tests check, block by block, that those
steps give the same result (a restatement of the steps here, not the kernel):

* the parse: every position's nearest earlier position with the same three
  bytes (what the kernel's sorted (key, position) pairs give), a walk that
  treats a position without one as a literal, and, where that nearest position
  lies inside a match longer than 4 bytes, the chain of same-key positions
  followed back to an entered one - against the oracle's table of entered
  positions (RFC 1951 section 4, fast form);
* the run-length coding of the code lengths counted in closed form per run of
  equal lengths - against the oracle's symbol-by-symbol coding (section 3.2.7).
"""
import numpy as np
import pytest

import sa_workloads as W
from oracle import deflate_size as F


def nearest_same_key(x):
    """(common prefix, distance) to the nearest earlier position with the same
    three bytes, 0 where there is none."""
    b = len(x)
    mlen, mdist = [0] * b, [0] * b
    last = {}
    for p in range(b - 2):
        key = x[p:p + 3]
        q = last.get(key)
        if q is not None:
            m = 3
            while p + m < b and m < 258 and x[q + m] == x[p + m]:
                m += 1
            mlen[p], mdist[p] = m, p - q
        last[key] = p
    return mlen, mdist


def walk(x):
    b = len(x)
    mlen, mdist = nearest_same_key(x)
    inside_long = [False] * b
    toks, p = [], 0
    while p < b:
        m = mlen[p]
        if m >= 3:
            q = p - mdist[p]
            if inside_long[q]:
                while q >= 0 and inside_long[q]:
                    q = q - mdist[q] if mlen[q] >= 3 else -1
                if q < 0:
                    m = 0
                else:
                    m = 3
                    while p + m < b and m < 258 and x[q + m] == x[p + m]:
                        m += 1
                    mlen[p], mdist[p] = m, p - q
        if m >= 3:
            toks.append(("match", m, mdist[p]))
            if m > F.MAX_INSERT:
                for i in range(p + 1, p + m):
                    inside_long[i] = True
            p += m
        else:
            toks.append(("lit", x[p]))
            p += 1
    return toks


def runs_closed_form(lengths):
    cf, extra, i, n = [0] * 19, 0, 0, len(lengths)
    while i < n:
        j = i
        while j < n and lengths[j] == lengths[i]:
            j += 1
        R, v = j - i, lengths[i]
        if v == 0:
            n18, rem = divmod(R, 138)
            if rem >= 11:
                n18, rem = n18 + 1, 0
            n17 = 1 if rem >= 3 else 0
            rem = 0 if n17 else rem
            cf[18] += n18
            cf[17] += n17
            cf[0] += rem
            extra += 7 * n18 + 3 * n17
        else:
            n16, rem = divmod(R - 1, 6)
            if rem >= 3:
                n16, rem = n16 + 1, 0
            cf[v] += 1 + rem
            cf[16] += n16
            extra += 2 * n16
        i = j
    return cf, extra


def blocks():
    rng = np.random.default_rng(7)
    out = []
    w = W.WORKLOADS["gzip_64k_fwdbwd"]
    for bt in range(w["batch"]):
        x = W.workload_bytes(w, bt)
        out += [x[i:i + 128] for i in range(0, 16384, 128)]
        out += [x[i:i + 1024] for i in range(0, 16384, 1024)]
    for b in (1, 3, 16, 100, 1000):
        out += [rng.integers(0, 256, b, dtype=np.uint8).tobytes(), bytes(b),
                (b"the cat sat on the mat. " * (b // 24 + 1))[:b],
                rng.integers(0, 3, b, dtype=np.uint8).tobytes()]
    return out


BLOCKS = blocks()


@pytest.mark.parametrize("part", range(4))
def test_walk_equals_the_table_parse(part):
    for blk in BLOCKS[part::4]:
        assert walk(blk) == F.parse(blk)


def test_the_table_rule_changes_some_parses():
    # the walk's chain step matters: on the workload's text some parses differ
    # from the plain nearest-position parse
    def plain(x):
        mlen, mdist = nearest_same_key(x)
        toks, p = [], 0
        while p < len(x):
            if mlen[p] >= 3:
                toks.append(("match", mlen[p], mdist[p]))
                p += mlen[p]
            else:
                toks.append(("lit", x[p]))
                p += 1
        return toks
    assert any(plain(blk) != F.parse(blk) for blk in BLOCKS)


def test_run_counts_in_closed_form():
    for blk in BLOCKS:
        _, Lll, Ldd, hlit, hdist, runs, _, _ = F.dynamic_code(blk)
        cf, extra = [0] * 19, 0
        for sym, _, nb in runs:
            cf[sym] += 1
            extra += nb
        assert runs_closed_form(Lll[:hlit] + Ldd[:hdist]) == (cf, extra)
