"""sa_forward vs the oracle: O and LSE element by element on small cases,
and on sampled rows at the workloads' full sizes."""
import numpy as np
import pytest
import torch

import sa_workloads as W
from oracle import attention as A
from oracle import gist as Gi
from oracle import gzip_mask as G

from _cases import (check_close, gist_layout, gzip_flags_oracle, gzip_flags_product, gzip_inputs,
                    sample_rows, to_dev, to_np)

pytestmark = pytest.mark.gpu


IMPLS = {"cuda_cores": 1, "tensor_cores": 2}


def run_gzip(sa, w, q, k, v, flags, impl=0):
    md = sa.gzip_mask(w["batch"], w["seq_len"], w["block"], w["window"], w["heads"])
    lists = sa.build_block_mask(md, flags)
    o, lse = sa.forward(to_dev(q, w["dtype"]), to_dev(k, w["dtype"]), to_dev(v, w["dtype"]), md, lists,
                        impl=impl)
    torch.cuda.synchronize()
    return to_np(o), to_np(lse)


def gzip_case(index, batch, N, b, w, H, d, dtype, p=0.3):
    return W.scaled("gzip_8k", index=index, batch=batch, seq_len=N, block=b, window=w, heads=H,
                    kv_heads=H, head_dim=d, dtype=dtype, p_literal=p)


@pytest.mark.parametrize("w", [
    W.WORKLOADS["gzip_tiny_fp32"],
    gzip_case(101, 2, 64 * 19, 64, 2, 4, 64, "bf16"),
    gzip_case(102, 1, 128 * 5, 128, 1, 6, 128, "bf16"),
    gzip_case(103, 2, 16 * 50, 16, 3, 4, 32, "fp32"),
    gzip_case(104, 1, 256 * 3, 256, 0, 4, 128, "bf16", p=0.6),
    gzip_case(105, 1, 64 * 12, 64, 20, 4, 64, "fp32"),
    gzip_case(106, 2, 32 * 40, 32, 1, 8, 128, "bf16", p=0.5),
    gzip_case(107, 1, 16 * 72, 16, 4, 4, 64, "bf16", p=0.4),
    gzip_case(108, 2, 64 * 33, 64, 1, 8, 128, "bf16", p=0.5),
    gzip_case(109, 1, 64 * 40, 64, 3, 4, 64, "bf16", p=1.0),
    gzip_case(110, 3, 64 * 8, 64, 0, 4, 64, "bf16", p=0.0),
], ids=["tiny_fp32", "b64_ragged_bf16", "b128_h6_bf16", "b16_fp32", "b256_bf16", "wide_w_fp32",
        "b32_d128_bf16", "b16_d64_bf16", "b64_d128_odd_bf16", "b64_all_literal_bf16",
        "b64_no_literal_w0_bf16"])
@pytest.mark.parametrize("impl", list(IMPLS))
def test_gzip_forward_small(sa, w, impl):
    if w["dtype"] == "fp32" and impl == "tensor_cores":
        pytest.skip("tensor cores take bf16 only")
    q, k, v, _ = gzip_inputs(w)
    fp, fo = gzip_flags_product(sa, w), gzip_flags_oracle(w)
    o, lse = run_gzip(sa, w, q, k, v, fp, IMPLS[impl])
    cls = G.head_classes(w["heads"])
    for bt in range(w["batch"]):
        masks = G.block_masks(fo[bt], w["window"])
        for h in range(w["heads"]):
            allowed = G.token_mask(masks[cls[h]], w["block"])
            ro, rl = A.forward(q[bt, :, h], k[bt, :, h], v[bt, :, h], allowed)
            check_close(o[bt, :, h], ro, w["dtype"], f"O b{bt} h{h}")
            check_close(lse[bt, h], rl, w["dtype"], f"LSE b{bt} h{h}")


@pytest.mark.parametrize("name", ["gzip_8k", "gzip_64k_fwdbwd"])
def test_gzip_forward_full_size_sampled(sa, name):
    w = W.WORKLOADS[name]
    q, k, v, _ = gzip_inputs(w)
    fp, fo = gzip_flags_product(sa, w), gzip_flags_oracle(w)
    o, lse = run_gzip(sa, w, q, k, v, fp)
    cls = G.head_classes(w["heads"])
    b = w["block"]
    for bt in range(w["batch"]):
        masks = G.block_masks(fo[bt], w["window"])
        for h in range(w["heads"]):
            rows = sample_rows(w["seq_len"], 24, seed=bt * 100 + h)
            keys = lambda p: np.nonzero(G.token_mask(masks[cls[h]], b, rows=[p])[0])[0]
            ro, rl = A.forward_rows(q[bt, :, h], k[bt, :, h], v[bt, :, h], keys, rows)
            check_close(o[bt, rows, h], ro, w["dtype"], f"O b{bt} h{h}")
            check_close(lse[bt, h, rows], rl, w["dtype"], f"LSE b{bt} h{h}")
    assert np.isfinite(o).all() and np.isfinite(lse).all()


def run_gist(sa, w, q, k, v, impl=0):
    md = sa.gist_mask(w["seq_len"], w["heads"], w["sinks"], w["ratio"], w["window"],
                      gist_tail=w.get("gist_tail", 32))
    lists = sa.build_block_mask(md, None)
    o, lse = sa.forward(to_dev(q, "bf16"), to_dev(k, "bf16"), to_dev(v, "bf16"), md, lists,
                        impl=impl)
    torch.cuda.synchronize()
    return to_np(o), to_np(lse)


@pytest.mark.parametrize("N,sinks,window", [(1000, 16, 32), (128 * 6, 128, 128), (2000, 130, 200)])
@pytest.mark.parametrize("impl", list(IMPLS))
def test_gist_forward_small(sa, N, sinks, window, impl):
    w = W.scaled("gist_prefill_32k", index=200 + N, seq_len=N, sinks=sinks, window=window,
                 heads=4, kv_heads=2)
    q, k, v = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v"))  # physical order
    o, lse = run_gist(sa, w, q, k, v, IMPLS[impl])
    g, perm, inv = gist_layout(N, sinks, w["ratio"])
    vis = Gi.visibility(g, sinks, window)
    for h in range(4):
        hk = h // 2
        # the oracle works in logical order: logical position i sits at physical inv[i]
        ro, rl = A.forward(q[0, inv, h], k[0, inv, hk], v[0, inv, hk], vis)
        check_close(o[0, inv, h], ro, "bf16", f"O h{h}")
        check_close(lse[0, h, inv], rl, "bf16", f"LSE h{h}")


def test_gist_forward_full_size_sampled(sa):
    w = W.WORKLOADS["gist_prefill_32k"]
    q, k, v = (W.qkv(w, t, 0)[None] for t in ("q", "k", "v"))
    o, lse = run_gist(sa, w, q, k, v)
    N = w["seq_len"]
    g, perm, inv = gist_layout(N, w["sinks"], w["ratio"])
    rep = w["heads"] // w["kv_heads"]
    for h in range(0, w["heads"], 3):
        rows = sample_rows(N, 16, seed=h)  # physical rows
        keys = lambda P: inv[Gi.visible_keys(g, w["sinks"], w["window"], int(perm[P]))]
        ro, rl = A.forward_rows(q[0, :, h], k[0, :, h // rep], v[0, :, h // rep], keys, rows)
        check_close(o[0, rows, h], ro, "bf16", f"O h{h}")
        check_close(lse[0, h, rows], rl, "bf16", f"LSE h{h}")
    assert np.isfinite(o).all() and np.isfinite(lse).all()


def test_tensor_cores_agree_with_cuda_cores_on_strided_inputs(sa):
    # q/k/v as slices of one packed [Bt, N, 3, H, d] buffer (non-contiguous heads)
    w = gzip_case(108, 2, 128 * 4, 128, 1, 4, 64, "bf16")
    q, k, v, _ = gzip_inputs(w)
    packed = torch.from_numpy(np.stack([q, k, v], axis=2)).to("cuda", torch.bfloat16)
    tq, tk, tv = packed[:, :, 0], packed[:, :, 1], packed[:, :, 2]
    fp = gzip_flags_product(sa, w)
    md = sa.gzip_mask(2, w["seq_len"], 128, 1, 4)
    lists = sa.build_block_mask(md, fp)
    o1, l1 = sa.forward(tq, tk, tv, md, lists, impl=1)
    o2, l2 = sa.forward(tq, tk, tv, md, lists, impl=2)
    torch.cuda.synchronize()
    check_close(to_np(o2), to_np(o1), "bf16", "O tc vs cuda cores")
    check_close(to_np(l2), to_np(l1), "bf16", "LSE tc vs cuda cores")
