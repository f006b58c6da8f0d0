"""Content-adaptive block-sparse attention on B200 (sm_100a).

A thin binding over the C ABI of ``libsa.so`` (include/sa.h). The functions
named ``sa_*`` have the C entry points' names and only marshal arguments
(tensor pointers, strides and the current CUDA stream); every step of the
computation runs in the library's CUDA kernels. The helpers below them
(``BlockLists``, ``forward``, ``backward``, ``gist_decode``) allocate outputs
and workspaces with PyTorch, which this package uses for device memory and
streams only.
"""
from __future__ import annotations

import ctypes as C
import zlib

import numpy as np
import torch

from . import _abi
from ._abi import *  # noqa: F401,F403  (enums and structs)

_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        _lib = _abi.load()
    return _lib


class SAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib().sa_status_string(status).decode()}")


def _check(status: int, where: str) -> None:
    if status != _abi.SA_OK:
        raise SAError(status, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def version() -> str:
    return lib().sa_version().decode()


# ------------------------------------------------------------------ a1 flags
def block_compressed_sizes(x: bytes, b: int) -> np.ndarray:
    """Level-1 zlib size of every b-byte block (host input preparation)."""
    if len(x) % b:
        raise ValueError("byte length must be a multiple of the block size")
    return np.array([len(zlib.compress(x[i:i + b], 1)) for i in range(0, len(x), b)],
                    dtype=np.uint32)


def sa_literal_flags_from_sizes(sizes: np.ndarray) -> np.ndarray:
    sizes = np.ascontiguousarray(sizes, dtype=np.uint32)
    flags = np.zeros(len(sizes), np.uint8)
    _check(lib().sa_literal_flags_from_sizes(
        sizes.ctypes.data_as(C.POINTER(C.c_uint32)), len(sizes),
        flags.ctypes.data_as(C.POINTER(C.c_uint8))), "sa_literal_flags_from_sizes")
    return flags


def literal_flags(x: bytes, b: int) -> np.ndarray:
    return sa_literal_flags_from_sizes(block_compressed_sizes(x, b))


def literal_flags_device(x: torch.Tensor, b: int, stream=None, sizes=None, flags=None):
    """Flags from device bytes x (uint8 [batch, n_bytes]) by the library's
    DEFLATE size estimate (greedy fast-table parse, the smallest of the fixed,
    dynamic and stored block): (sizes uint32 as int32 [batch, B], flags uint8
    [batch, B]), written into `sizes`/`flags` when given."""
    if x.dtype != torch.uint8 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous uint8 [batch, n_bytes] tensor")
    batch, n = x.shape
    B = n // b
    if sizes is None:
        sizes = torch.empty(batch, B, dtype=torch.int32, device=x.device)
    if flags is None:
        flags = torch.empty(batch, B, dtype=torch.uint8, device=x.device)
    for t, dt in ((sizes, torch.int32), (flags, torch.uint8)):
        if t.dtype != dt or t.shape != (batch, B) or not t.is_contiguous() or t.device != x.device:
            raise ValueError("sizes/flags must be contiguous [batch, n_bytes // b] int32/uint8 "
                             "tensors on x's device")
    _check(lib().sa_literal_flags_device(_ptr(x), batch, n, b, _ptr(sizes), _ptr(flags),
                                         _stream(stream)), "sa_literal_flags_device")
    return sizes, flags


# ---------------------------------------------------------------- mask desc
def mask_desc(kind: int, seq_len: int, num_heads: int, batch: int = 1, block_size: int = 0,
              window: int = 0, sinks: int = 0, gist_ratio: int = 0, gist_tail: int = 0,
              head_class=None) -> _abi.sa_mask_desc:
    d = _abi.sa_mask_desc(kind=kind, batch=batch, seq_len=seq_len, block_size=block_size,
                          window=window, num_heads=num_heads, sinks=sinks,
                          gist_ratio=gist_ratio, gist_tail=gist_tail, head_class=None)
    if head_class is not None:
        buf = (C.c_int8 * num_heads)(*[int(c) for c in head_class])
        d._head_class_buf = buf  # keep alive
        d.head_class = C.cast(buf, C.c_void_p)
    return d


def gzip_mask(batch, seq_len, block_size, window, num_heads, head_class=None):
    return mask_desc(_abi.SA_MASK_GZIP, seq_len, num_heads, batch=batch, block_size=block_size,
                     window=window, head_class=head_class)


def gist_mask(seq_len, num_heads, sinks, gist_ratio, window, gist_tail=32, segment=0):
    """Gist layout. segment = 0: interleaved gists and a local window of
    `window` positions; segment = L > 0: the coarse layout, L raw tokens then
    L / gist_ratio gists per segment, full attention inside a segment (window
    ignored)."""
    return mask_desc(_abi.SA_MASK_GIST, seq_len, num_heads, sinks=sinks, gist_ratio=gist_ratio,
                     window=window, gist_tail=gist_tail, block_size=segment)


class BlockLists:
    """Device buffers of sa_block_lists, sized by sa_block_lists_capacity."""

    def __init__(self, desc: _abi.sa_mask_desc, device="cuda"):
        caps = _abi.sa_block_lists_sizes()
        _check(lib().sa_block_lists_capacity(C.byref(desc), C.byref(caps)),
               "sa_block_lists_capacity")
        self.desc = desc
        self.caps = caps
        mk = lambda n, dt: torch.zeros(max(int(n), 1), dtype=dt, device=device) if n else None
        self.row_ptr = mk(caps.row_ptr, torch.int32)
        self.col_idx = mk(caps.nnz, torch.int32)
        self.col_ptr = mk(caps.row_ptr, torch.int32)
        self.row_idx = mk(caps.nnz, torch.int32)
        self.bits = mk(caps.bits, torch.int32)
        self.tile_row_ptr = mk(caps.tile_row_ptr, torch.int32)
        self.tile_col = mk(caps.tile_nnz, torch.int32)
        self.tile_kind = mk(caps.tile_nnz, torch.int8)
        self.tile_col_ptr = mk(caps.tile_row_ptr, torch.int32)
        self.tile_row = mk(caps.tile_nnz, torch.int32)
        self.tile_kind_t = mk(caps.tile_nnz, torch.int8)
        self.perm = mk(caps.perm, torch.int32)
        self.gist_bits = mk(caps.gist_bits, torch.int32)
        self.far_idx = mk(caps.far_idx, torch.int32)
        self.far_ptr = mk(caps.far_ptr, torch.int32)
        self.struct = _abi.sa_block_lists(
            *[_ptr(getattr(self, n)) for n in ("row_ptr", "col_idx", "col_ptr", "row_idx", "bits",
                                                "tile_row_ptr", "tile_col", "tile_kind",
                                                "tile_col_ptr", "tile_row", "tile_kind_t",
                                                "perm", "gist_bits", "far_idx", "far_ptr")],
            int(caps.nnz), int(caps.tile_nnz))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def sa_build_block_mask(desc, flags, lists: BlockLists, ws: torch.Tensor, stream=None) -> None:
    _check(lib().sa_build_block_mask(C.byref(desc), _ptr(flags), C.byref(lists.struct),
                                     _ptr(ws), ws.numel(), _stream(stream)),
           "sa_build_block_mask")


def build_block_mask(desc, flags=None, device="cuda", stream=None) -> BlockLists:
    """Allocates lists + workspace and runs sa_build_block_mask.

    flags: gzip - uint8 [batch, B] literal flags (host numpy or device tensor);
    gist - None (regular pattern) or uint8 [N] gist flags per logical position."""
    lists = BlockLists(desc, device)
    if flags is not None and not torch.is_tensor(flags):
        flags = torch.from_numpy(np.ascontiguousarray(flags, dtype=np.uint8)).to(device)
    n = C.c_size_t()
    _check(lib().sa_build_block_mask_workspace_size(C.byref(desc), C.byref(n)),
           "sa_build_block_mask_workspace_size")
    ws = _workspace(n.value, device)
    sa_build_block_mask(desc, flags, lists, ws, stream)
    lists._flags = flags
    lists._ws = ws
    return lists


# ---------------------------------------------------------------- attention
def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _abi.SA_DTYPE_BF16
    if t.dtype == torch.float32:
        return _abi.SA_DTYPE_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def attn_desc(q, k, v, o, softmax_scale: float = 0.0, impl: int = 0) -> _abi.sa_attn_desc:
    """Descriptor from [Bt, N, H, d] tensors (any strides, last dim contiguous)."""
    Bt, N, Hq, d = q.shape
    st = lambda t: (i64 * 3)(t.stride(0), t.stride(1), t.stride(2))
    for t in (q, k, v, o):
        if t.stride(3) != 1:
            raise ValueError("head_dim must be contiguous")
    return _abi.sa_attn_desc(dtype=_dtype_code(q), batch=Bt, seq_len=N, num_q_heads=Hq,
                             num_kv_heads=k.shape[2], head_dim=d, softmax_scale=softmax_scale,
                             q_strides=st(q), k_strides=st(k), v_strides=st(v), o_strides=st(o),
                             impl=impl)


i64 = C.c_int64


def sa_forward(adesc, mdesc, q, k, v, lists: BlockLists, o, lse, ws, stream=None) -> None:
    _check(lib().sa_forward(C.byref(adesc), C.byref(mdesc), _ptr(q), _ptr(k), _ptr(v),
                            C.byref(lists.struct), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                            _stream(stream)), "sa_forward")


def forward_workspace(adesc, mdesc, device="cuda") -> torch.Tensor:
    n = C.c_size_t()
    _check(lib().sa_forward_workspace_size(C.byref(adesc), C.byref(mdesc), C.byref(n)),
           "sa_forward_workspace_size")
    return _workspace(n.value, device)


def forward(q, k, v, mdesc, lists: BlockLists, softmax_scale: float = 0.0, stream=None,
            impl: int = 0):
    """O [Bt, N, Hq, d] (dtype of q) and LSE fp32 [Bt, Hq, N]."""
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[2], q.shape[1], dtype=torch.float32, device=q.device)
    ad = attn_desc(q, k, v, o, softmax_scale, impl)
    ws = forward_workspace(ad, mdesc, q.device)
    sa_forward(ad, mdesc, q, k, v, lists, o, lse, ws, stream)
    return o, lse


def sa_backward(adesc, mdesc, q, k, v, o, lse, dout, lists, dq, dk, dv, ws, stream=None) -> None:
    _check(lib().sa_backward(C.byref(adesc), C.byref(mdesc), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                             _ptr(lse), _ptr(dout), C.byref(lists.struct), _ptr(dq), _ptr(dk),
                             _ptr(dv), _ptr(ws), ws.numel(), _stream(stream)), "sa_backward")


def backward_workspace(adesc, mdesc, device="cuda") -> torch.Tensor:
    n = C.c_size_t()
    _check(lib().sa_backward_workspace_size(C.byref(adesc), C.byref(mdesc), C.byref(n)),
           "sa_backward_workspace_size")
    return _workspace(n.value, device)


def backward(q, k, v, o, lse, dout, mdesc, lists, softmax_scale: float = 0.0, stream=None,
             impl: int = 0):
    """fp32 dQ [Bt, N, Hq, d], dK and dV [Bt, N, Hkv, d]. dout has o's strides."""
    if dout.stride() != o.stride():
        raise ValueError("dout must have the same strides as o")
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    ad = attn_desc(q, k, v, o, softmax_scale, impl)
    ws = backward_workspace(ad, mdesc, q.device)
    sa_backward(ad, mdesc, q, k, v, o, lse, dout, lists, dq, dk, dv, ws, stream)
    return dq, dk, dv


# ------------------------------------------------------------------- decode
def decode_desc(q, gist_k, k_cache, o, chunk: int, top_k: int, window: int,
                softmax_scale: float = 0.0, select_rule: int = 0,
                top_p: float = 1.0) -> _abi.sa_decode_desc:
    n_seq, Hq, d = q.shape
    _, Hkv, G, _ = gist_k.shape
    L = k_cache.shape[2]
    return _abi.sa_decode_desc(
        n_seq=n_seq, cache_len=L, chunk=chunk, n_gists=G, top_k=top_k, window=window,
        num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d,
        select_rule=select_rule, softmax_scale=softmax_scale, top_p=top_p,
        q_strides=(i64 * 2)(q.stride(0), q.stride(1)),
        gist_strides=(i64 * 3)(gist_k.stride(0), gist_k.stride(1), gist_k.stride(2)),
        cache_strides=(i64 * 3)(k_cache.stride(0), k_cache.stride(1), k_cache.stride(2)),
        o_strides=(i64 * 2)(o.stride(0), o.stride(1)))


def decode_workspace(ddesc, device="cuda") -> torch.Tensor:
    n = C.c_size_t()
    _check(lib().sa_gist_decode_workspace_size(C.byref(ddesc), C.byref(n)),
           "sa_gist_decode_workspace_size")
    return _workspace(n.value, device)


def sa_gist_decode(ddesc, q, gist_k, gist_v, k_cache, v_cache, sel, o, lse, ws, stream=None):
    _check(lib().sa_gist_decode(C.byref(ddesc), _ptr(q), _ptr(gist_k), _ptr(gist_v),
                                _ptr(k_cache), _ptr(v_cache), _ptr(sel), _ptr(o), _ptr(lse),
                                _ptr(ws), ws.numel(), _stream(stream)), "sa_gist_decode")


def gist_decode(q, gist_k, gist_v, k_cache, v_cache, chunk: int, top_k: int, window: int,
                softmax_scale: float = 0.0, stream=None, select_rule: int = 0, top_p: float = 1.0):
    """(sel int32 [n_seq, Hkv, top_k], o bf16 [n_seq, Hq, d], lse fp32 [n_seq, Hq]).
    select_rule: 0 top-k of summed logits, 1 top-k of summed per-head
    probabilities, 2 top-p (at most top_k chunks) of the summed logits, 3 each
    query head's own top-k (sel is then [n_seq, Hq, top_k])."""
    if gist_v.stride() != gist_k.stride() or v_cache.stride() != k_cache.stride():
        raise ValueError("K and V must share strides")
    n_seq, Hq, d = q.shape
    Hkv = gist_k.shape[1]
    o = torch.empty_like(q)
    lse = torch.empty(n_seq, Hq, dtype=torch.float32, device=q.device)
    rows = Hq if select_rule == _abi.SA_SELECT_TOP_K_PER_HEAD else Hkv
    sel = torch.empty(n_seq, rows, max(top_k, 1), dtype=torch.int32, device=q.device)
    dd = decode_desc(q, gist_k, k_cache, o, chunk, top_k, window, softmax_scale, select_rule, top_p)
    ws = decode_workspace(dd, q.device)
    sa_gist_decode(dd, q, gist_k, gist_v, k_cache, v_cache, sel, o, lse, ws, stream)
    gist_decode.last_workspace = ws
    return sel[:, :, :top_k], o, lse


def hier_decode_desc(q, gist2_k, gist_k, k_cache, o, chunk: int, fanout: int, top_k2: int,
                     top_k: int, window: int, softmax_scale: float = 0.0) -> _abi.sa_hier_decode_desc:
    n_seq, Hq, d = q.shape
    _, Hkv, G, _ = gist_k.shape
    return _abi.sa_hier_decode_desc(
        n_seq=n_seq, cache_len=k_cache.shape[2], chunk=chunk, n_gists=G, fanout=fanout,
        top_k2=top_k2, top_k=top_k, window=window, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d,
        softmax_scale=softmax_scale, q_strides=(i64 * 2)(q.stride(0), q.stride(1)),
        gist_strides=(i64 * 3)(*gist_k.stride()[:3]), gist2_strides=(i64 * 3)(*gist2_k.stride()[:3]),
        cache_strides=(i64 * 3)(*k_cache.stride()[:3]), o_strides=(i64 * 2)(o.stride(0), o.stride(1)))


def hier_decode_workspace(hdesc, device="cuda") -> torch.Tensor:
    n = C.c_size_t()
    _check(lib().sa_gist_hier_decode_workspace_size(C.byref(hdesc), C.byref(n)),
           "sa_gist_hier_decode_workspace_size")
    return _workspace(n.value, device)


def sa_gist_hier_decode(hdesc, q, gist2_k, gist2_v, gist_k, gist_v, k_cache, v_cache, sel2, sel1,
                        o, lse, ws, stream=None):
    _check(lib().sa_gist_hier_decode(C.byref(hdesc), _ptr(q), _ptr(gist2_k), _ptr(gist2_v),
                                     _ptr(gist_k), _ptr(gist_v), _ptr(k_cache), _ptr(v_cache),
                                     _ptr(sel2), _ptr(sel1), _ptr(o), _ptr(lse), _ptr(ws),
                                     ws.numel(), _stream(stream)), "sa_gist_hier_decode")


def gist_hier_decode(q, gist2_k, gist2_v, gist_k, gist_v, k_cache, v_cache, chunk: int, fanout: int,
                     top_k2: int, top_k: int, window: int, softmax_scale: float = 0.0, stream=None):
    """Gist-of-gist decode: (sel2 int32 [n_seq, Hkv, top_k2], sel1 int32
    [n_seq, Hkv, top_k], o bf16 [n_seq, Hq, d], lse fp32 [n_seq, Hq])."""
    for a, b in ((gist2_k, gist2_v), (gist_k, gist_v), (k_cache, v_cache)):
        if a.stride() != b.stride():
            raise ValueError("K and V must share strides")
    n_seq, Hq, d = q.shape
    Hkv = gist_k.shape[1]
    o = torch.empty_like(q)
    lse = torch.empty(n_seq, Hq, dtype=torch.float32, device=q.device)
    sel2 = torch.empty(n_seq, Hkv, max(top_k2, 1), dtype=torch.int32, device=q.device)
    sel1 = torch.empty(n_seq, Hkv, max(top_k, 1), dtype=torch.int32, device=q.device)
    hd = hier_decode_desc(q, gist2_k, gist_k, k_cache, o, chunk, fanout, top_k2, top_k, window,
                          softmax_scale)
    ws = hier_decode_workspace(hd, q.device)
    sa_gist_hier_decode(hd, q, gist2_k, gist2_v, gist_k, gist_v, k_cache, v_cache, sel2, sel1, o, lse,
                        ws, stream)
    gist_hier_decode.last_workspace = ws
    return sel2[:, :, :top_k2], sel1[:, :, :top_k], o, lse


def selftest_wait_timeout(n_ctas: int = 8, device="cuda", stream=None):
    """Runs the device failure-path self-test (about 4 s; a test-only export of
    the library, declared outside the public header); returns (status code,
    location) read from the status word after the stream synchronises."""
    ws = _workspace(256, device)
    _check(lib().sa_selftest_wait_timeout(_ptr(ws), ws.numel(), n_ctas, _stream(stream)),
           "sa_selftest_wait_timeout")
    torch.cuda.synchronize(ws.device)
    code, where = ws[:8].view(torch.int32).cpu().tolist()
    return code, where


def device_status(ws: torch.Tensor | None, stream=None) -> int:
    """The device status word of a workspace an earlier call used (None: the
    fixed scratch array of the allocation-free decode on the current device).
    Synchronises the stream."""
    st = C.c_int()
    _check(lib().sa_get_device_status(_ptr(ws), _stream(stream), C.byref(st)),
           "sa_get_device_status")
    return st.value
