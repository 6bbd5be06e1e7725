"""ctypes loader for libcpattn.so (the C ABI in include/cpattn.h).

There is no fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcpattn.so")

c_int, c_uint, c_size_t, c_void_p, c_char_p = ctypes.c_int, ctypes.c_uint, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_char_p
P_INT = ctypes.POINTER(ctypes.c_int)
P_UINT = ctypes.POINTER(ctypes.c_uint)

# name -> (restype, argtypes); mirrors include/cpattn.h
SIGNATURES = {
    "cpattn_status_string": (c_char_p, [c_int]),
    "cpattn_last_cuda_error": (c_int, []),
    "cpattn_last_cuda_error_string": (c_char_p, []),
    "cpattn_version": (c_int, []),
    "cpattn_ring_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_int, c_int, c_int, c_int, c_int, P_INT, c_void_p]),
    "cpattn_ring_step": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_int, c_int, c_int, c_int, c_int, P_INT, c_int, c_void_p]),
    "cpattn_lse_merge": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                 c_void_p, c_void_p, c_void_p, c_void_p]),
    "cpattn_kv_gather_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_int, c_int, c_int, c_int, c_int, P_INT, c_void_p]),
    "cpattn_ulysses_permute": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                       P_INT, P_INT, c_void_p]),
    "cpattn_ulysses_permute_qkv": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_int, c_int, c_int, c_int, c_int, c_int, P_INT, P_INT, c_void_p]),
    "cpattn_ulysses_unpermute": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                         P_INT, P_INT, c_void_p]),
    "cpattn_ulysses_qkv_projection": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                              c_int, c_int, c_int, c_int, c_int, c_int, P_INT, P_INT, c_void_p]),
    "cpattn_ulysses_output_projection": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                                 c_int, P_INT, P_INT, c_void_p]),
    "cpattn_head_sharded_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                              c_int, c_int, c_int, c_int, c_int, P_INT, c_void_p]),
    "cpattn_ulysses_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "cpattn_ulysses_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_int, c_int, c_int, c_int, c_int, P_INT, P_INT,
                                         c_void_p, c_size_t, c_void_p]),
    "cpattn_unified_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "cpattn_unified_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_int, c_int, c_int, c_int, c_int, c_int, P_INT, P_INT,
                                         c_void_p, c_size_t, c_void_p]),
    "cpattn_causal_ring_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_int, c_int, c_int, c_int, c_int, P_INT, c_void_p]),
    "cpattn_causal_ring_step": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_int, c_int, c_int, c_int, c_int, P_INT, c_int, c_void_p]),
    "cpattn_causal_head_sharded_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                     c_int, c_int, c_int, c_int, c_int, P_INT, c_void_p]),
    "cpattn_causal_ulysses_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                c_int, c_int, c_int, c_int, c_int, P_INT, P_INT,
                                                c_void_p, c_size_t, c_void_p]),
    "cpattn_causal_unified_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                c_int, c_int, c_int, c_int, c_int, c_int, P_INT, P_INT,
                                                c_void_p, c_size_t, c_void_p]),
    "cpattn_attention_backward_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "cpattn_attention_backward_ds_bytes": (c_size_t, [c_int, c_int, c_int]),
    "cpattn_attention_backward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                          c_void_p, c_size_t, c_void_p]),
    "cpattn_ulysses_attention_backward_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "cpattn_ulysses_attention_backward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                  c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
                                                  P_INT, P_INT, c_int, c_void_p, c_size_t, c_void_p]),
    "cpattn_ulysses_attention_noalloc": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                 c_int, c_int, c_int, c_int, c_int, P_INT, P_INT, c_void_p]),
    "cpattn_ring_chunk_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                            c_void_p]),
    "cpattn_gathered_kv_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_int, c_int, c_int, c_int, P_INT, c_int, c_int, c_int, c_void_p]),
    "cpattn_rank_buffer_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                             c_int, c_int, c_int, c_int, c_int, P_INT, c_int, c_void_p]),
    "cpattn_front_loaded_splits": (c_int, [c_int, c_int, P_INT]),
    "cpattn_exchange_bytes": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_int, P_INT, P_INT,
                                      ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_ulonglong)]),
    "cpattn_plan_exchange": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, P_INT, P_INT,
                                     ctypes.c_void_p, ctypes.c_void_p]),
    "cpattn_device_status": (c_int, [c_void_p, P_UINT]),
    "cpattn_debug_wait_timeout": (c_int, [c_uint, c_void_p]),
}

_LIB = None


def load() -> ctypes.CDLL:
    """Load libcpattn.so and declare every C ABI signature; raise if missing."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m context_attention_long_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def int_array(values):
    """Host int[] for a split/length argument, or None for NULL."""
    if values is None:
        return None
    vals = [int(x) for x in values]
    return (ctypes.c_int * len(vals))(*vals)
