"""ctypes declarations of the C ABI in include/dllm.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libdllm.so")

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t
_st = ctypes.c_int32

# name -> (restype, argtypes); every symbol declared in include/dllm.h
PROTOTYPES = {
    "dllm_version": (_i32, []),
    "dllm_status_string": (ctypes.c_char_p, [_st]),
    "dllm_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "dllm_workspace_bytes_rows": (_sz, [_i32, _i32, _i32, _i32, ctypes.c_int64]),
    "dllm_workspace_rows": (ctypes.c_int64, [_i32, _i32, _i32, _i32, _sz]),
    "dllm_arena_create": (_st, [_sz, _sz, ctypes.POINTER(_p)]),
    "dllm_arena_map": (_st, [_p, _sz]),
    "dllm_arena_ptr": (_p, [_p]),
    "dllm_arena_reserved": (_sz, [_p]),
    "dllm_arena_mapped": (_sz, [_p]),
    "dllm_arena_chunk": (_sz, [_p]),
    "dllm_arena_destroy": (_st, [_p]),
    "dllm_mask_compact": (_st, [_p, _i32, _i32, _p, _p, _p, _p, _sz, _p]),
    "dllm_mask_compact_window": (_st, [_p, _i32, _i32, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dllm_mask_compact_noalloc": (_st, [_p, _i32, _i32, _p, _p, _p, _p]),
    "dllm_masked_logits": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p,
                                 _p, _sz, _p]),
    "dllm_masked_logits_ex": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, ctypes.c_uint32, _p, _p,
                                    _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dllm_masked_logits_window": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, _p, _p,
                                        ctypes.c_uint32, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz,
                                        _p]),
    "dllm_prepare_rows": (_st, [_p, _p, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dllm_masked_logits_prepared": (_st, [_p, _i32, _i32, _i32, _i32, ctypes.c_uint32, _p, _p, _p,
                                          _p, _p, _p, _p, _sz, _p]),
    "dllm_masked_partials": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p,
                                   ctypes.c_uint32, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dllm_lse_merge": (_st, [_p, _p, _p, _p, _p, ctypes.c_int64, _i32, _p, _i32, ctypes.c_uint32,
                             _p, _p, _p, _p, _p, _p]),
    "dllm_select_unmask": (_st, [_p, _p, _p, _i32, _i32, _i32, _p, _p, _p, _p, _p, _p, _p, _p]),
    "dllm_select_unmask_ex": (_st, [_p, _p, _p, _i32, _i32, _i32, ctypes.c_float, _i32, _i32, _p,
                                    _p, _p, _p, _p, _p, _p, _p]),
    "dllm_decode_step": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p,
                               _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dllm_decode_block_step": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _p,
                                     _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "dllm_get_status": (_st, [_p]),
    "dllm_debug_lmhead_logits": (_st, [_p, _p, _p, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p,
                                       _sz, _p]),
    "dllm_debug_lse_merge": (_st, [_p, _p, _p, _i32, _i32, _p, _p, _p, _p]),
    "dllm_debug_set_gemm_variant": (_st, [_i32]),
    "dllm_prof_begin": (_st, []),
    "dllm_prof_end": (_st, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i32),
                            ctypes.POINTER(_i32)]),
}

_lib = None


def load_from(path: str) -> ctypes.CDLL:
    """Load another build of the library (e.g. a test variant) with the same prototypes."""
    lib = ctypes.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load() -> ctypes.CDLL:
    """Load libdllm.so from the package directory; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mask_only_logits_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
