"""ctypes mirror of include/sa.h (structs, enums and prototypes).

Loading fails loudly when libsa.so is missing: there is no other compute path.
"""
from __future__ import annotations

import ctypes as C
import os

from .build import LIB

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA, \
    SA_ERR_TIMEOUT, SA_ERR_DEVICE = range(7)
SA_MASK_GZIP, SA_MASK_GIST = 0, 1
SA_CLASS_LOCAL, SA_CLASS_LITERAL, SA_CLASS_HYBRID = 0, 1, 2
SA_DTYPE_BF16, SA_DTYPE_FP32 = 0, 1
SA_TILE_FULL, SA_TILE_MASKED, SA_TILE_TAIL = 0, 1, 2
SA_SELECT_SUM_LOGITS_PER_GROUP = 0
SA_SELECT_SUM_PROBS_PER_GROUP = 1
SA_SELECT_TOP_P_PER_GROUP = 2
SA_SELECT_TOP_K_PER_HEAD = 3
SA_IMPL_AUTO, SA_IMPL_CUDA_CORES, SA_IMPL_TENSOR_CORES = 0, 1, 2
SA_TILE = 128

i32, i64, f32, vp = C.c_int32, C.c_int64, C.c_float, C.c_void_p


class sa_mask_desc(C.Structure):
    _fields_ = [("kind", i32), ("batch", i32), ("seq_len", i64), ("block_size", i32),
                ("window", i32), ("num_heads", i32), ("sinks", i32), ("gist_ratio", i32),
                ("gist_tail", i32), ("head_class", vp)]


class sa_block_lists(C.Structure):
    _fields_ = [(n, vp) for n in ("row_ptr", "col_idx", "col_ptr", "row_idx", "bits",
                                  "tile_row_ptr", "tile_col", "tile_kind", "tile_col_ptr",
                                  "tile_row", "tile_kind_t", "perm", "gist_bits", "far_idx",
                                  "far_ptr")] + \
               [("cap_nnz", i64), ("cap_tile_nnz", i64)]


class sa_block_lists_sizes(C.Structure):
    _fields_ = [(n, i64) for n in ("row_ptr", "nnz", "bits", "tile_row_ptr", "tile_nnz",
                                   "perm", "gist_bits", "far_idx", "far_ptr")]


class sa_attn_desc(C.Structure):
    _fields_ = [("dtype", i32), ("batch", i32), ("seq_len", i64), ("num_q_heads", i32),
                ("num_kv_heads", i32), ("head_dim", i32), ("softmax_scale", f32),
                ("q_strides", i64 * 3), ("k_strides", i64 * 3), ("v_strides", i64 * 3),
                ("o_strides", i64 * 3), ("impl", i32)]


class sa_decode_desc(C.Structure):
    _fields_ = [("n_seq", i32), ("cache_len", i32), ("chunk", i32), ("n_gists", i32),
                ("top_k", i32), ("window", i32), ("num_q_heads", i32), ("num_kv_heads", i32),
                ("head_dim", i32), ("select_rule", i32), ("softmax_scale", f32),
                ("q_strides", i64 * 2), ("gist_strides", i64 * 3), ("cache_strides", i64 * 3),
                ("o_strides", i64 * 2), ("top_p", f32)]


class sa_hier_decode_desc(C.Structure):
    _fields_ = [("n_seq", i32), ("cache_len", i32), ("chunk", i32), ("n_gists", i32),
                ("fanout", i32), ("top_k2", i32), ("top_k", i32), ("window", i32),
                ("num_q_heads", i32), ("num_kv_heads", i32), ("head_dim", i32),
                ("softmax_scale", f32), ("q_strides", i64 * 2), ("gist_strides", i64 * 3),
                ("gist2_strides", i64 * 3), ("cache_strides", i64 * 3), ("o_strides", i64 * 2)]


P = C.POINTER
PROTOTYPES = {
    "sa_version": (C.c_char_p, []),
    "sa_status_string": (C.c_char_p, [C.c_int]),
    "sa_get_device_status": (C.c_int, [vp, vp, P(C.c_int)]),
    "sa_literal_flags_from_sizes": (C.c_int, [P(C.c_uint32), i32, P(C.c_uint8)]),
    "sa_literal_flags_device": (C.c_int, [vp, i32, i64, i32, vp, vp, vp]),
    "sa_selftest_wait_timeout": (C.c_int, [vp, C.c_size_t, i32, vp]),
    "sa_block_lists_capacity": (C.c_int, [P(sa_mask_desc), P(sa_block_lists_sizes)]),
    "sa_build_block_mask_workspace_size": (C.c_int, [P(sa_mask_desc), P(C.c_size_t)]),
    "sa_build_block_mask": (C.c_int, [P(sa_mask_desc), vp, P(sa_block_lists), vp, C.c_size_t, vp]),
    "sa_forward_workspace_size": (C.c_int, [P(sa_attn_desc), P(sa_mask_desc), P(C.c_size_t)]),
    "sa_forward": (C.c_int, [P(sa_attn_desc), P(sa_mask_desc), vp, vp, vp, P(sa_block_lists),
                             vp, vp, vp, C.c_size_t, vp]),
    "sa_backward_workspace_size": (C.c_int, [P(sa_attn_desc), P(sa_mask_desc), P(C.c_size_t)]),
    "sa_backward": (C.c_int, [P(sa_attn_desc), P(sa_mask_desc), vp, vp, vp, vp, vp, vp,
                              P(sa_block_lists), vp, vp, vp, vp, C.c_size_t, vp]),
    "sa_gist_decode_workspace_size": (C.c_int, [P(sa_decode_desc), P(C.c_size_t)]),
    "sa_gist_decode": (C.c_int, [P(sa_decode_desc), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                 C.c_size_t, vp]),
    "sa_gist_decode_noalloc": (C.c_int, [P(sa_decode_desc), vp, vp, vp, vp, vp, vp, vp, vp, vp]),
    "sa_gist_hier_decode_workspace_size": (C.c_int, [P(sa_hier_decode_desc), P(C.c_size_t)]),
    "sa_gist_hier_decode": (C.c_int, [P(sa_hier_decode_desc), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      vp, vp, vp, C.c_size_t, vp]),
}


def load(path: str = LIB) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"libsa.so not found at {path}; build it with "
                          "`python -m content_adaptive_block_sa_b200.build`")
    lib = C.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
