"""ctypes declarations of the C ABI in include/msa.h (loaded from the in-tree libmsa.so)."""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

P = C.c_void_p
I32 = C.c_int32
I64 = C.c_int64
F32 = C.c_float
SZ = C.c_size_t

# name -> (restype, argtypes), in the order of include/msa.h
SIGNATURES = {
    "msa_status_string": (C.c_char_p, [C.c_int]),
    "msa_version": (C.c_char_p, []),
    "msa_kernel_launch_count": (C.c_uint64, []),
    "msa_testing_set_wait_polls": (None, [I64]),
    "msa_rope_table_host": (C.c_int, [C.c_double, C.c_int, C.c_int, P]),
    "msa_chunk_offsets_host": (C.c_int, [P, I64, C.c_int, P]),
    "msa_pool": (C.c_int, [C.c_int, P, P, P, P, P, I64, I64, I64, C.c_int, C.c_int, C.c_int, C.c_int,
                           C.c_int, P, C.c_int, P, P, P, P, P, P]),
    "msa_bank_rnorm": (C.c_int, [C.c_int, P, I64, C.c_int, C.c_int, P, P]),
    "msa_route_topk_workspace_size": (SZ, [I64, C.c_int, C.c_int, I64, I64, C.c_int]),
    "msa_route_topk": (C.c_int, [C.c_int, P, I64, C.c_int, C.c_int, C.c_int, P, P, P, I64, I64, C.c_int,
                                 P, P, P, P, SZ, P, P]),
    "msa_route_topk_noalloc": (C.c_int, [C.c_int, P, I64, C.c_int, C.c_int, C.c_int, P, P, P, I64, I64,
                                         C.c_int, P, P, P, P, P]),
    "msa_gather": (C.c_int, [C.c_int, P, I64, C.c_int, P, I64, I64, P, P, C.c_int, C.c_int, C.c_int,
                             P, P, P, P, P]),
    "msa_sparse_attn_workspace_size": (SZ, [I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int]),
    "msa_sparse_attn": (C.c_int, [C.c_int, P, P, P, I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                  P, P, P, C.c_int, F32, P, P, P, SZ, P, P]),
    "msa_sparse_attn_indexed_workspace_size": (SZ, [I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                                    C.c_int]),
    "msa_sparse_attn_indexed": (C.c_int, [C.c_int, P, P, P, I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                          P, C.c_int, P, I64, I64, P, P, C.c_int, F32, P, P, P, SZ, P, P]),
    "msa_sparse_attn_backward_workspace_size": (SZ, [I64, C.c_int, C.c_int]),
    "msa_sparse_attn_backward": (C.c_int, [C.c_int, P, P, P, I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                           P, P, P, C.c_int, F32, P, P, P, P, P, P, P, P, P, SZ, P, P]),
    "msa_gather_backward": (C.c_int, [P, I64, C.c_int, P, I64, I64, P, P, P, C.c_int, C.c_int, C.c_int,
                                      P, P, P, P]),
    "msa_route_backward_workspace_size": (SZ, [I64, C.c_int, C.c_int]),
    "msa_route_backward": (C.c_int, [C.c_int, P, I64, C.c_int, C.c_int, C.c_int, P, P, P, I64, I64, C.c_int,
                                     P, P, P, P, P, SZ, P, P]),
    "msa_layer_forward_workspace_size": (SZ, [I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                              I64, I64, C.c_int, C.c_int]),
    "msa_layer_forward": (C.c_int, [C.c_int, P, C.c_int, C.c_int, P, P, P, I64, I64, C.c_int,
                                    P, P, P, I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                    P, P, C.c_int, F32, P, P, P, P, P, P, SZ, P, P]),
    "msa_interleave_workspace_size": (SZ, [I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                           I64, I64, C.c_int, C.c_int, C.c_int]),
    "msa_interleave_forward": (C.c_int, [C.c_int, P, C.c_int, C.c_int, P, P, P, I64, I64, C.c_int, C.c_int, P,
                                         P, P, P, I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                         P, P, C.c_int, F32, P, P, P, P, P, P, P, SZ, P, P]),
    "msa_state_gather_sum": (C.c_int, [C.c_int, P, I64, I64, P, I64, C.c_int, P, P, P]),
    "msa_gated_delta_rule": (C.c_int, [C.c_int, P, P, P, P, P, I64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                       P, F32, P, P, P]),
}

_lib = None


def load() -> C.CDLL:
    """The loaded library; raises if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m routed_sparse_attention_chunk_b200.build`")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
