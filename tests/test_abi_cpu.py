"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/sa.h declares, its struct layouts match the ctypes mirror, host-side
validation rejects bad arguments before any launch, and the host flag helper
follows the integer form of the mean test."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import sa_workloads as W
from oracle import gzip_mask as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sa.h")


@pytest.fixture(scope="module")
def sa():
    from content_adaptive_block_sa_b200 import build
    build.build()
    import content_adaptive_block_sa_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(sa_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(sa):
    names = declared_functions()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", sa._abi.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert n in sa._abi.PROTOTYPES, f"binding lacks {n}"
        getattr(sa.lib(), n)


def test_struct_layouts_match_c(sa, tmp_path):
    structs = {"sa_mask_desc": sa._abi.sa_mask_desc, "sa_block_lists": sa._abi.sa_block_lists,
               "sa_block_lists_sizes": sa._abi.sa_block_lists_sizes,
               "sa_attn_desc": sa._abi.sa_attn_desc, "sa_decode_desc": sa._abi.sa_decode_desc}
    src = ['#include <stdio.h>', '#include <stddef.h>', '#include "sa.h"', "int main(void){"]
    for name, cls in structs.items():
        src.append(f'printf("{name} %zu\\n", sizeof({name}));')
        for f, _ in cls._fields_:
            src.append(f'printf("{name}.{f} %zu\\n", offsetof({name}, {f}));')
    src.append("return 0;}")
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    for name, cls in structs.items():
        assert int(got[name]) == C.sizeof(cls), name
        for f, _ in cls._fields_:
            assert int(got[f"{name}.{f}"]) == getattr(cls, f).offset, (name, f)


def test_version_and_status_strings(sa):
    assert "sm_100a" in sa.version()
    assert sa.lib().sa_status_string(3).decode() == "SA_ERR_WORKSPACE"


@pytest.mark.parametrize("name,b", [("gzip_tiny_fp32", 16), ("gzip_64k_fwdbwd", 128)])
def test_host_flag_helper_matches_oracle(sa, name, b):
    x = W.workload_bytes(name, 0)
    assert np.array_equal(sa.literal_flags(x, b), G.literal_flags(x, b))
    assert sa.sa_literal_flags_from_sizes(np.array([5, 5, 5])).tolist() == [0, 0, 0]


def _caps(sa, desc):
    caps = sa._abi.sa_block_lists_sizes()
    return sa.lib().sa_block_lists_capacity(C.byref(desc), C.byref(caps)), caps


def test_capacity_and_validation(sa):
    st, caps = _caps(sa, sa.gzip_mask(2, 65536, 128, 2, 16))
    assert st == 0
    assert caps.row_ptr == 6 * 513 and caps.nnz == 6 * 512 * 513 // 2
    assert caps.tile_nnz == 6 * 512 * 513 // 2 and caps.bits == 6 * 512 * 16
    st, caps = _caps(sa, sa.gist_mask(32768, 32, 128, 4, 128))
    assert st == 0 and caps.perm == 32768 and caps.gist_bits == 1024 and caps.tile_row_ptr == 257
    assert caps.far_idx == 32768 and caps.far_ptr == 257
    bad = [sa.gzip_mask(1, 1000, 64, 1, 4),      # N % b != 0
           sa.gzip_mask(1, 960, 96, 1, 4),       # b neither divides nor is a multiple of 128
           sa.gzip_mask(1, 1024, 64, -1, 4),     # negative window
           sa.gzip_mask(0, 1024, 64, 1, 4),      # no batch
           sa.gist_mask(4096, 8, 128, 0, 128),   # ratio 0
           sa.gist_mask(4096, 8, 128, 4, 0),     # empty window
           sa.gist_mask(4096, 8, 128, 4, 128, gist_tail=40),
           sa.gist_mask(4096, 8, 0, 4, 0, segment=1022),   # segment not a multiple of the ratio
           sa.gist_mask(4096, 8, 0, 4, 0, segment=-4)]     # negative segment
    codes = [_caps(sa, d)[0] for d in bad]
    assert all(c in (1, 2) for c in codes), codes
    d = sa.gzip_mask(1, 1024, 64, 1, 4, head_class=[0, 1, 2, 3])
    assert _caps(sa, d)[0] == 1
    # the coarse layout ignores the window
    assert _caps(sa, sa.gist_mask(20480, 32, 0, 4, 0, segment=1024))[0] == 0


def test_coarse_layout_rejects_explicit_flags_without_a_device(sa):
    md = sa.gist_mask(4096, 8, 0, 4, 0, segment=1024)
    caps = sa._abi.sa_block_lists_sizes()
    assert sa.lib().sa_block_lists_capacity(C.byref(md), C.byref(caps)) == 0
    lists = sa._abi.sa_block_lists()
    flags = C.c_void_p(16)  # never dereferenced: the descriptor check comes first
    assert sa.lib().sa_build_block_mask(C.byref(md), flags, C.byref(lists), None, 0, None) == 1


def test_calls_reject_null_and_small_workspace_without_a_device(sa):
    L = sa._abi
    md = sa.gzip_mask(1, 1024, 64, 1, 4)
    lists = L.sa_block_lists()
    assert sa.lib().sa_build_block_mask(C.byref(md), None, C.byref(lists), None, 0, None) == 1
    ad = L.sa_attn_desc(dtype=0, batch=1, seq_len=1024, num_q_heads=4, num_kv_heads=4, head_dim=64,
                        q_strides=(C.c_int64 * 3)(0, 256, 64), k_strides=(C.c_int64 * 3)(0, 256, 64),
                        v_strides=(C.c_int64 * 3)(0, 256, 64), o_strides=(C.c_int64 * 3)(0, 256, 64))
    n = C.c_size_t()
    assert sa.lib().sa_forward_workspace_size(C.byref(ad), C.byref(md), C.byref(n)) == 0
    assert sa.lib().sa_backward_workspace_size(C.byref(ad), C.byref(md), C.byref(n)) == 0
    assert n.value >= 256 + 4 * 1024 * 4
    assert sa.lib().sa_forward(C.byref(ad), C.byref(md), None, None, None, C.byref(lists),
                               None, None, None, 0, None) == 1
    ad.num_kv_heads = 3
    assert sa.lib().sa_forward_workspace_size(C.byref(ad), C.byref(md), C.byref(n)) == 1
    ad.num_kv_heads, ad.head_dim = 4, 80
    assert sa.lib().sa_forward_workspace_size(C.byref(ad), C.byref(md), C.byref(n)) == 2
    dd = L.sa_decode_desc(n_seq=16, cache_len=131072, chunk=32, n_gists=4096, top_k=64, window=512,
                          num_q_heads=32, num_kv_heads=8, head_dim=128,
                          gist_strides=(C.c_int64 * 3)(8 * 4096 * 128, 4096 * 128, 128),
                          cache_strides=(C.c_int64 * 3)(8 * 131072 * 128, 131072 * 128, 128))
    assert sa.lib().sa_gist_decode_workspace_size(C.byref(dd), C.byref(n)) == 0
    assert n.value > 16 * 8 * 4096 * 4
    dd.top_k = 300
    assert sa.lib().sa_gist_decode_workspace_size(C.byref(dd), C.byref(n)) == 2
    dd.top_k, dd.n_gists = 64, 4095
    assert sa.lib().sa_gist_decode_workspace_size(C.byref(dd), C.byref(n)) == 1


def test_tensor_core_request_on_fp32_is_unsupported_before_any_launch(sa):
    L = sa._abi
    md = sa.gzip_mask(1, 1024, 128, 1, 4)
    fake = C.c_void_p(1 << 20)  # never dereferenced: validation fails first
    caps = L.sa_block_lists_sizes()
    sa.lib().sa_block_lists_capacity(C.byref(md), C.byref(caps))
    lists = L.sa_block_lists(*([fake.value] * 15), caps.nnz, caps.tile_nnz)
    st = (C.c_int64 * 3)(1024 * 4 * 64, 4 * 64, 64)
    ad = L.sa_attn_desc(dtype=L.SA_DTYPE_FP32, batch=1, seq_len=1024, num_q_heads=4, num_kv_heads=4,
                        head_dim=64, q_strides=st, k_strides=st, v_strides=st, o_strides=st,
                        impl=L.SA_IMPL_TENSOR_CORES)
    assert sa.lib().sa_forward(C.byref(ad), C.byref(md), fake, fake, fake, C.byref(lists), fake,
                               fake, fake, 4096, None) == L.SA_ERR_UNSUPPORTED
    ad.impl = 7
    assert sa.lib().sa_forward(C.byref(ad), C.byref(md), fake, fake, fake, C.byref(lists), fake,
                               fake, fake, 4096, None) == L.SA_ERR_INVALID_ARG


def test_selftest_rejects_bad_arguments_without_a_device(sa):
    f = sa.lib().sa_selftest_wait_timeout
    fake = C.c_void_p(256)  # never dereferenced: every check comes before a launch
    assert f(fake, 256, 0, None) == 1      # no CTA
    assert f(fake, 256, 2000, None) == 1   # too many CTAs
    assert f(fake, 16, 4, None) == 3       # workspace shorter than the status word


def _decode_desc(sa, **kw):
    L = sa._abi
    d = dict(n_seq=16, cache_len=131072, chunk=32, n_gists=4096, top_k=64, window=512,
             num_q_heads=32, num_kv_heads=8, head_dim=128, select_rule=0, softmax_scale=0.0,
             q_strides=(C.c_int64 * 2)(4096, 128), gist_strides=(C.c_int64 * 3)(4096 * 1024, 4096 * 128, 128),
             cache_strides=(C.c_int64 * 3)(131072 * 1024, 131072 * 128, 128),
             o_strides=(C.c_int64 * 2)(4096, 128), top_p=1.0)
    d.update(kw)
    return L.sa_decode_desc(**d)


def test_decode_select_rules_validated_without_a_device(sa):
    n = C.c_size_t()
    f = lambda d: sa.lib().sa_gist_decode_workspace_size(C.byref(d), C.byref(n))
    for rule in range(4):
        assert f(_decode_desc(sa, select_rule=rule, top_p=0.5)) == 0
    assert f(_decode_desc(sa)) == 0
    base = n.value
    assert f(_decode_desc(sa, select_rule=1)) == 0 and n.value > base  # per-head logits kept
    assert f(_decode_desc(sa, select_rule=4)) == 1                     # no such rule
    assert f(_decode_desc(sa, select_rule=2, top_p=0.0)) == 1          # empty nucleus
    assert f(_decode_desc(sa, select_rule=2, top_p=1.5)) == 1


def _hier_desc(sa, **kw):
    d = dict(n_seq=16, cache_len=131072, chunk=32, n_gists=4096, fanout=32, top_k2=8, top_k=64,
             window=512, num_q_heads=32, num_kv_heads=8, head_dim=128, softmax_scale=0.0,
             q_strides=(C.c_int64 * 2)(4096, 128), gist_strides=(C.c_int64 * 3)(4096 * 1024, 4096 * 128, 128),
             gist2_strides=(C.c_int64 * 3)(128 * 1024, 128 * 128, 128),
             cache_strides=(C.c_int64 * 3)(131072 * 1024, 131072 * 128, 128),
             o_strides=(C.c_int64 * 2)(4096, 128))
    d.update(kw)
    return sa._abi.sa_hier_decode_desc(**d)


def test_hier_decode_validated_without_a_device(sa):
    n = C.c_size_t()
    f = lambda d: sa.lib().sa_gist_hier_decode_workspace_size(C.byref(d), C.byref(n))
    assert f(_hier_desc(sa)) == 0 and n.value >= 256
    assert f(_hier_desc(sa, fanout=3)) == 1          # n_gists % fanout != 0
    assert f(_hier_desc(sa, cache_len=1000)) == 1    # n_gists * chunk != cache_len
    assert f(_hier_desc(sa, top_k2=300)) == 2        # above 256
    assert f(_hier_desc(sa, head_dim=64)) == 2
    assert f(_hier_desc(sa, num_kv_heads=3)) == 1
    # null outputs are refused before any launch
    d = _hier_desc(sa)
    fake = C.c_void_p(4096)
    assert sa.lib().sa_gist_hier_decode(C.byref(d), fake, fake, fake, fake, fake, fake, fake, None, fake,
                                        fake, fake, fake, 1 << 30, None) == 1


def test_device_flags_validated_without_a_device(sa):
    f = sa.lib().sa_literal_flags_device
    fake = C.c_void_p(4096)
    assert f(None, 1, 1024, 128, fake, fake, None) == 1      # no bytes
    assert f(fake, 1, 1000, 128, fake, fake, None) == 1      # n_bytes % b != 0
    assert f(fake, 1, 4096, 2048, fake, fake, None) == 2     # b above 1024
    assert f(fake, 0, 1024, 128, fake, fake, None) == 1      # no sequence
