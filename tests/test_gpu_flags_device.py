"""sa_literal_flags_device vs the oracle's DEFLATE sizes: every block size
and every flag bit-exact, on the workloads' byte generators, random and
degenerate blocks, and ragged block sizes; and the device flags against
zlib level 1's on the workloads' bytes."""
import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import deflate_size as F
from oracle import gzip_mask as G

pytestmark = pytest.mark.gpu


def run(sa, rows, b):
    x = torch.from_numpy(np.stack([np.frombuffer(r, np.uint8) for r in rows])).cuda()
    sizes, flags = sa.literal_flags_device(x, b)
    torch.cuda.synchronize()
    return sizes.cpu().numpy().view(np.uint32), flags.cpu().numpy()


def check(sa, rows, b):
    sizes, flags = run(sa, rows, b)
    for i, r in enumerate(rows):
        want = F.block_sizes(r, b)
        np.testing.assert_array_equal(sizes[i], want)
        np.testing.assert_array_equal(flags[i], F.literal_flags(r, b))


def test_workload_bytes_64k(sa):
    w = W.WORKLOADS["gzip_64k_fwdbwd"]
    check(sa, [W.workload_bytes(w, bt) for bt in range(w["batch"])], w["block"])


def test_tiny_pattern_bytes(sa):
    w = W.WORKLOADS["gzip_tiny_fp32"]
    check(sa, [W.workload_bytes(w, 0)], w["block"])


@pytest.mark.parametrize("name", ["gzip_tiny_fp32", "gzip_64k_fwdbwd"])
def test_device_flags_equal_zlib_flags(sa, name):
    # the method's flags come from gzip level 1: on these workloads' bytes
    # the device estimate gives the same flag on every block
    w = W.WORKLOADS[name]
    rows = [W.workload_bytes(w, bt) for bt in range(w["batch"])]
    _, flags = run(sa, rows, w["block"])
    for i, r in enumerate(rows):
        np.testing.assert_array_equal(flags[i], G.literal_flags(r, w["block"]))


@pytest.mark.parametrize("b", [1, 3, 16, 100, 128, 1000, 1024])
def test_random_text_and_degenerate_blocks(sa, b):
    rng = np.random.default_rng(b)
    n = b * 12
    rows = [rng.integers(0, 256, n, dtype=np.uint8).tobytes(),       # incompressible
            bytes(n),                                                  # all zeros
            (b"the cat sat on the mat. " * (n // 24 + 1))[:n],         # periodic text
            rng.integers(0, 3, n, dtype=np.uint8).tobytes()]           # three symbols
    check(sa, rows, b)


def _zipf_rows(b, n_rows=2, seed=0):
    """Bytes drawn from a Zipf law over a shuffled alphabet: few matches and a
    wide spread of literal counts, so the code-length code of some blocks is
    deeper than 7 bits and needs package-merge."""
    rng = np.random.default_rng(seed)
    rows = []
    for a in np.linspace(0.75, 1.6, n_rows):
        p = 1.0 / np.arange(1, 257) ** a
        perm = rng.permutation(256)
        rows.append(perm[rng.choice(256, b * 24, p=p / p.sum())].astype(np.uint8).tobytes())
    return rows


def _code_length_code_depth(block):
    # the unlimited Huffman depth of the block's code-length code
    _, _, _, _, _, runs, _, _ = F.dynamic_code(block)
    cf = [0] * 19
    for sym, _, _ in runs:
        cf[sym] += 1
    return max(F.huffman_lengths(cf, 99))


@pytest.mark.parametrize("b", [256, 1000, 1024])
def test_zipf_bytes_package_merge(sa, b):
    rows = _zipf_rows(b, seed=b)
    depths = [_code_length_code_depth(r[i:i + b]) for r in rows for i in range(0, len(r), b)]
    if b >= 1000:
        assert max(depths) > 7  # the limited code-length code is reached
    check(sa, rows, b)
