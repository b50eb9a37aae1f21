"""ctypes loader for libfa_sm100.so and the raw C entry points of include/fa.h.

Loading fails loudly: there is no fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libfa_sm100.so")
# The same entry points built with index checks (FA_DEBUG); loaded only when asked for by path.
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libfa_sm100_debug.so")

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _I, _I]),
    "fa_fwd_prefix": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _I, _I]),
    "fa_decode_workspace_bytes": (_Z, [_I, _I, _I, _I]),
    "fa_bwd_workspace_bytes": (_Z, [_I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _Z, _P, _I, _I]),
    "fa_bwd_masked": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _I, _P, _P, _Z, _P, _I,
                           _I]),
    "fa_decode_splitkv": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _Z, _P, _I, _I]),
    "fa_decode_splitkv_gqa": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _Z, _P, _I, _I]),
    "fa_decode_splitkv_paged": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _Z, _P,
                                     _I, _I]),
    "fa_decode_splitkv_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _I, _I]),
    "fa_decode_part_bytes": (_Z, [_I, _I, _I]),
    "fa_decode_splitkv_shard": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _P, _Z, _P, _I]),
    "fa_decode_merge": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _I]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_device_status": (_I, [ctypes.POINTER(_I), _I]),
    "fa_abi_version": (_I, []),
    "fa_build_flags": (_I, []),
    "fa_selftest_wait_timeout": (_I, [ctypes.POINTER(_I), _P]),
}

_lock = threading.Lock()
_lib = None


class LibraryMissing(RuntimeError):
    pass


def load(path: str | None = None):
    """Load (once) and return the ctypes handle; raises LibraryMissing if the library is not built."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise LibraryMissing(
                f"{p} is missing: build it with `python -m exact_tiled_attention_47_b200.build` "
                "(there is no CPU or fallback implementation)")
        lib = ctypes.CDLL(p)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        if path is None:
            _lib = lib
        return lib
