"""Device failure path without a fault: the library's bounded wait (4 s), given
a flag nothing sets, records SA_ERR_TIMEOUT with its location in the status
word, every CTA leaves, and the context keeps working."""
import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import decode as D

from _cases import check_close, to_np

pytestmark = pytest.mark.gpu

SA_ERR_TIMEOUT = 5


@pytest.mark.parametrize("n_ctas", [1, 148])
def test_bounded_wait_reports_timeout(sa, n_ctas):
    code, where = sa.selftest_wait_timeout(n_ctas=n_ctas)
    assert (code, where) == (SA_ERR_TIMEOUT, 900)


def test_context_still_works_after_a_timeout(sa):
    assert sa.selftest_wait_timeout(n_ctas=4)[0] == SA_ERR_TIMEOUT
    w = W.scaled("gist_decode_128k", index=990, n_seq=1, cache_len=16 * 64, chunk=16, n_gists=64,
                 top_k=4, window=32, heads=4, kv_heads=2)
    q = W.decode_query(w)
    gk, gv = W.decode_gists(w, 0, "k")[None], W.decode_gists(w, 0, "v")[None]
    rk = np.stack([W.decode_raw(w, 0, g, "k") for g in range(2)])[None]
    rv = np.stack([W.decode_raw(w, 0, g, "v") for g in range(2)])[None]
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to("cuda", torch.bfloat16)
    sel, o, lse = sa.gist_decode(dev(q), dev(gk), dev(gv), dev(rk), dev(rv), 16, 4, 32)
    torch.cuda.synchronize()
    assert sa.gist_decode.last_workspace[:4].view(torch.int32).item() == 0
    osel, oo, ol, _ = D.decode_one(q[0], gk[0], gv[0], rk[0], rv[0], 16, 32, 4)
    assert np.array_equal(sel[0].cpu().numpy(), osel)
    check_close(to_np(o)[0], oo, "bf16", "O after a timeout")
