"""The allocation-free decode entry point against the regular one and the
oracle.

sa_gist_decode_noalloc exists for callers that may not allocate device memory
(for example a serving engine that has reserved all free memory for its KV
cache, or a plugin that is only handed raw pointers); it keeps its scratch in a
fixed array inside the library instead of a caller-provided workspace. This
test calls both entry points through the C ABI on the same inputs, twice in a
row with different inputs (the shared scratch keeps the previous call's
contents), on a shape the tensor-core kernel takes (only the status word lives
in the array) and on one that runs the CUDA-core passes (per-group scores and
split-K partials live in the array too). It requires the same selection and
outputs as sa_gist_decode within the tolerance of the other decode tests, the
oracle's selection (or a float32 near tie) and outputs, and a clear status
word read back through sa_get_device_status(NULL, ...). It runs last so that a
failure here cannot stop the rest of the suite, and it passes alone in a
fresh process as well.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import decode as D

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3

# (chunk, gists, top_k, window): the first shape runs the tensor-core decode,
# the second (fewer than 128 gists) the CUDA-core passes
SHAPES = {"tensor_cores": (32, 256, 16, 256), "cuda_cores": (16, 64, 8, 64)}


def _inputs(index, chunk, G, top_k, window):
    w = W.scaled("gist_decode_128k", index=index, n_seq=4, cache_len=chunk * G, chunk=chunk,
                 n_gists=G, top_k=top_k, window=window, heads=16, kv_heads=4)
    host = dict(q=W.decode_query(w),
                gk=np.stack([W.decode_gists(w, s, "k") for s in range(4)]),
                gv=np.stack([W.decode_gists(w, s, "v") for s in range(4)]),
                kc=np.stack([[W.decode_raw(w, s, g, "k") for g in range(4)] for s in range(4)]),
                vc=np.stack([[W.decode_raw(w, s, g, "v") for g in range(4)] for s in range(4)]))
    dev = {n: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.bfloat16)
           for n, a in host.items()}
    return w, host, dev


def _close(a, b, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.abs(a - b).max()
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {err:.3g}, rel-L2 {rel:.3g}"


def _np(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("path", list(SHAPES))
def test_noalloc_decode_matches_workspace_decode_and_oracle_on_two_calls(path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import content_adaptive_block_sa_b200 as sa
    from test_gpu_decode import valid_alternative
    lib = sa.lib()
    stream = torch.cuda.current_stream()
    chunk, G, top_k, window = SHAPES[path]
    for index in (901, 902):  # two calls in a row, different inputs
        w, host, t = _inputs(index, chunk, G, top_k, window)
        q, gk, gv, kc, vc = t["q"], t["gk"], t["gv"], t["kc"], t["vc"]
        sel_ref, o_ref, lse_ref = sa.gist_decode(q, gk, gv, kc, vc, chunk, top_k, window)
        o = torch.empty_like(q)
        lse = torch.empty(4, 16, dtype=torch.float32, device="cuda")
        sel = torch.full((4, 4, top_k), -7, dtype=torch.int32, device="cuda")
        dd = sa.decode_desc(q, gk, kc, o, chunk, top_k, window)
        st = lib.sa_gist_decode_noalloc(C.byref(dd), q.data_ptr(), gk.data_ptr(), gv.data_ptr(),
                                        kc.data_ptr(), vc.data_ptr(), sel.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), C.c_void_p(stream.cuda_stream))
        assert st == sa.SA_OK, lib.sa_status_string(st).decode()
        torch.cuda.synchronize()
        assert sa.device_status(None) == sa.SA_OK  # the fixed array's status word
        assert torch.equal(sel, sel_ref)
        _close(_np(o), _np(o_ref), f"O vs sa_gist_decode (call {index})")
        _close(_np(lse), _np(lse_ref), f"LSE vs sa_gist_decode (call {index})")
        # against the oracle on the bf16-rounded inputs
        sel_h, o_h, lse_h = sel.cpu().numpy(), _np(o), _np(lse)
        rep = w["heads"] // w["kv_heads"]
        for s in range(4):
            rk = lambda g: host["kc"][s, g]
            rv = lambda g: host["vc"][s, g]
            osel, oo, ol, scores = D.decode_one(host["q"][s], host["gk"][s], host["gv"][s], rk, rv,
                                                chunk, window, top_k)
            for g in range(w["kv_heads"]):
                if not np.array_equal(sel_h[s, g], osel[g]):
                    valid_alternative(w, 0, 1.0, host["q"], host["gk"], s, g, sel_h[s, g], scores[g])
                    pos = D.raw_key_positions(sel_h[s, g], chunk, w["cache_len"], window)
                    keys = np.concatenate([host["gk"][s, g], rk(g)[pos]])
                    vals = np.concatenate([host["gv"][s, g], rv(g)[pos]])
                    for h in range(g * rep, (g + 1) * rep):
                        oo[h], ol[h] = D.attend(host["q"][s, h], keys, vals, 1 / np.sqrt(w["head_dim"]))
            _close(o_h[s], oo, f"O vs oracle seq {s} (call {index})")
            _close(lse_h[s], ol, f"LSE vs oracle seq {s} (call {index})")


def test_noalloc_decode_refuses_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import content_adaptive_block_sa_b200 as sa
    lib = sa.lib()
    # a size whose scratch exceeds the fixed array is refused before any launch
    big = sa._abi.sa_decode_desc(n_seq=64, cache_len=32 * 8192, chunk=32, n_gists=8192, top_k=64,
                                 window=512, num_q_heads=64, num_kv_heads=8, head_dim=128,
                                 gist_strides=(C.c_int64 * 3)(8 * 8192 * 128, 8192 * 128, 128),
                                 cache_strides=(C.c_int64 * 3)(8 * 262144 * 128, 262144 * 128, 128),
                                 q_strides=(C.c_int64 * 2)(64 * 128, 128),
                                 o_strides=(C.c_int64 * 2)(64 * 128, 128))
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    p = x.data_ptr()
    st = lib.sa_gist_decode_noalloc(C.byref(big), p, p, p, p, p, p, p, p, None)
    assert st == sa.SA_ERR_WORKSPACE
