"""ctypes binding of libfa.so: the C entry points of include/fa.h, same names.

Argument marshalling only.  The shared library must have been built in-tree
(``python -m exact_attention_121_b200.build``); there is no fallback path.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_BOUNDS = range(6)
FA_FP16, FA_BF16 = 0, 1
FA_MAX_SPLITS = 64

# Every symbol include/fa.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t
SIGNATURES = {
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F, _P]),
    "fa_bwd_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "fa_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                    _F, _I, _P, _Z, _P]),
    "fa_fwd_strided": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F, _P, _P]),
    "fa_bwd_strided": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                            _F, _I, _P, _Z, _P, _P]),
    "fa_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _F, _I, _I, _I, _F, _P]),
    "fa_fwd_alibi": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _F, _P, _P, _I, _P]),
    "fa_bwd_alibi": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                          _F, _I, _P, _Z, _P, _P, _I, _P]),
    "fa_fwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I,
                           _F, _P]),
    "fa_bwd_varlen_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "fa_bwd_varlen": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                           _F, _I, _I, _I, _F, _I, _P, _Z, _P]),
    "fa_kvcache_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "fa_fwd_kvcache": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                            _I, _F, _I, _I, _I, _F, _I, _P, _Z, _P]),
    "fa_kvcache_rotary_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "fa_fwd_kvcache_rotary": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                                   _I, _F, _I, _I, _I, _F, _P, _P, _I, _I, _I, _I, _P, _Z, _P]),
    "fa_fwd_kvcache_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                                    _I, _F, _I, _I, _I, _F, _I, _P]),
    "fa_last_device_status": (_I, [_P]),
    "fa_set_fwd_kernel": (None, [_I]),
    "fa_set_bwd_kernel": (None, [_I]),
    "fa_selftest_bounded_wait": (_I, [_P, _I, ctypes.c_longlong, _P]),
    "fa_selftest_exp2_poly": (_I, [_P, _P, _I, _P]),
    "fa_last_launch_count": (_I, []),
    "fa_build_flags": (_I, []),
    "fa_set_trace_events": (None, [_P, _P]),
}

_lib = None


def load():
    """Load libfa.so once and attach the signatures; raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfa.so not built at {LIB_PATH}; run python -m exact_attention_121_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class FaError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        name = load().fa_status_string(code).decode()
        super().__init__(f"{where} returned {name} ({code})")


def check(code, where):
    if code != FA_OK:
        raise FaError(code, where)
