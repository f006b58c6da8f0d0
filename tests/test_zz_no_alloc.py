"""The allocation-free decode entry point against the regular one.

sa_gist_decode_noalloc exists for callers that may not allocate device memory
(for example a serving engine that has reserved all free memory for its KV
cache, or a plugin that is only handed raw pointers); it keeps its scratch in a
fixed array inside the library instead of a caller-provided workspace. This
test calls both entry points through the C ABI on the same inputs, twice in a
row with different inputs (the shared scratch keeps the previous call's
contents), and requires the same selection and outputs within the tolerance of
the other decode tests. It runs last so that a failure here cannot stop the
rest of the suite, and it passes alone in a fresh process as well.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import sa_workloads as W

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


def _inputs(index):
    w = W.scaled("gist_decode_128k", index=index, n_seq=4, cache_len=32 * 256, chunk=32,
                 n_gists=256, top_k=16, window=256, heads=16, kv_heads=4)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16)
    q = bf(W.decode_query(w))
    gk = bf(np.stack([W.decode_gists(w, s, "k") for s in range(4)]))
    gv = bf(np.stack([W.decode_gists(w, s, "v") for s in range(4)]))
    kc = bf(np.stack([[W.decode_raw(w, s, g, "k") for g in range(4)] for s in range(4)]))
    vc = bf(np.stack([[W.decode_raw(w, s, g, "v") for g in range(4)] for s in range(4)]))
    return w, q, gk, gv, kc, vc


def _close(a, b, what):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {err:.3g}, rel-L2 {rel:.3g}"


def test_noalloc_decode_matches_workspace_decode_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import content_adaptive_block_sa_b200 as sa
    lib = sa.lib()
    stream = torch.cuda.current_stream()
    for index in (901, 902):  # two calls in a row, different inputs
        w, q, gk, gv, kc, vc = _inputs(index)
        sel_ref, o_ref, lse_ref = sa.gist_decode(q, gk, gv, kc, vc, w["chunk"], w["top_k"], w["window"])
        o = torch.empty_like(q)
        lse = torch.empty(4, 16, dtype=torch.float32, device="cuda")
        sel = torch.full((4, 4, w["top_k"]), -7, dtype=torch.int32, device="cuda")
        dd = sa.decode_desc(q, gk, kc, o, w["chunk"], w["top_k"], w["window"])
        st = lib.sa_gist_decode_noalloc(C.byref(dd), q.data_ptr(), gk.data_ptr(), gv.data_ptr(),
                                        kc.data_ptr(), vc.data_ptr(), sel.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), C.c_void_p(stream.cuda_stream))
        assert st == sa.SA_OK, lib.sa_status_string(st).decode()
        torch.cuda.synchronize()
        assert torch.equal(sel, sel_ref)
        _close(o, o_ref, f"O (call {index})")
        _close(lse, lse_ref, f"LSE (call {index})")
    # a size whose scratch exceeds the fixed array is refused before any launch
    big = sa._abi.sa_decode_desc(n_seq=64, cache_len=32 * 8192, chunk=32, n_gists=8192, top_k=64,
                                 window=512, num_q_heads=64, num_kv_heads=8, head_dim=128,
                                 gist_strides=(C.c_int64 * 3)(8 * 8192 * 128, 8192 * 128, 128),
                                 cache_strides=(C.c_int64 * 3)(8 * 262144 * 128, 262144 * 128, 128),
                                 q_strides=(C.c_int64 * 2)(64 * 128, 128),
                                 o_strides=(C.c_int64 * 2)(64 * 128, 128))
    p = q.data_ptr()
    st = lib.sa_gist_decode_noalloc(C.byref(big), p, p, p, p, p, p, p, p, None)
    assert st == sa.SA_ERR_WORKSPACE
