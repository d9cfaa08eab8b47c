"""ctypes declarations of libdsa.so (the C ABI in include/dsa.h)."""

from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")

_i, _f, _p, _sz, _u64, _i64 = C.c_int, C.c_float, C.c_void_p, C.c_size_t, C.c_uint64, C.c_int64

# name -> (restype, argtypes)
SIGNATURES = {
    "dsa_version": (C.c_char_p, []),
    "dsa_last_error": (C.c_char_p, []),
    "dsa_status_string": (C.c_char_p, [_i]),
    "dsa_set_wait_timeout_ns": (None, [_u64]),
    "dsa_get_wait_timeout_ns": (_u64, []),
    "dsa_workspace_init": (_i, [_p, _sz, _p]),
    "dsa_read_device_status": (_i, [_p, _p, C.POINTER(C.c_uint32)]),
    "dsa_indexer_topk_prefill_workspace": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "dsa_indexer_topk_prefill_workspace_full": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "dsa_indexer_topk_prefill": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dsa_sparse_attn_workspace": (_sz, []),
    "dsa_sparse_attn_prefill": (_i, [_i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dsa_indexer_topk_decode_workspace": (_sz, [_i, _i, _i, _i, _i, _i64, _i]),
    "dsa_indexer_topk_decode": (_i, [_i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _i64, _i, _p, _p, _p, _sz, _p]),
    "dsa_indexer_topk_decode_noalloc": (_i, [_i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _i64, _i, _p, _p, _p, _p]),
    "dsa_sparse_attn_decode": (_i, [_i, _i, _i, _i, _i, _f, _p, _p, _p, _i64, _p, _p, _p, _p, _sz, _p]),
    "dsa_small_workspace": (_sz, []),
    "dsa_indexer_scores": (_i, [_i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dsa_topk_rows": (_i, [_i, _i, _i64, _p, _p, _i, _p, _p, _p, _sz, _p]),
    "dsa_selftest_bounded_wait": (_i, [_u64, _p, _sz, _p]),
    "dsa_selection_overlap": (_i, [_i, _i, _i, _p, _p, _p, _p, _p]),
    "dsa_indexer_kl_workspace": (_sz, []),
    "dsa_attn_dense_prefill_workspace": (_sz, [_i, _i, _i, _i]),
    "dsa_attn_dense_prefill": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dsa_mass_coverage": (_i, [_i, _i, _p, _p, _p, _p, _p, _p]),
    "dsa_prefill_attention_path": (_i, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "dsa_attn_prefill_workspace": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "dsa_attn_prefill": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dsa_attn_teacher_prefill": (_i, [_i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dsa_indexer_kl_sparse": (_i, [_i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _f, _p, _p, _p, _p, _p, _p, _sz, _p]),
}

_lib = None


def load() -> C.CDLL:
    """Load libdsa.so from the package directory (fails loudly if missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m learned_token_indexer_b200.build`")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
