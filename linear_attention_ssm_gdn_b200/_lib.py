"""ctypes loader for libgdn.so (the in-tree C-ABI library, include/gdn.h).

There is no fallback: if the library is missing or was built for another
architecture, loading raises.  Build it with
``python -m linear_attention_ssm_gdn_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK = 0
GDN_ERR_NULL = 1
GDN_ERR_SHAPE = 2
GDN_ERR_STRIDE = 3
GDN_ERR_WORKSPACE = 4
GDN_ERR_CUDA = 5
GDN_ERR_ALIGN = 6
GDN_FLAG_ENGAGED = 1
GDN_FLAG_ERROR = 2
GDN_FLAG_STASH_BAD = 4

ERROR_NAMES = {1: "GDN_ERR_NULL", 2: "GDN_ERR_SHAPE", 3: "GDN_ERR_STRIDE",
               4: "GDN_ERR_WORKSPACE", 5: "GDN_ERR_CUDA", 6: "GDN_ERR_ALIGN"}

# Every symbol include/gdn.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t
SIGNATURES = {
    "gdn_last_error": (ctypes.c_char_p, []),
    "gdn_version": (ctypes.c_char_p, []),
    "gdn_ba_gates": (_I, [_P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "gdn_chunk_prefill_workspace_bytes": (_S, [_I, _I, _I, _I, _I, _I]),
    "gdn_chunk_prefill": (_I, [_P, _P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _P, _P, _P, _I, _I,
                               _I, _I, _F, _P, _S, _P]),
    "gdn_chunk_prefill_x2": (_I, [_P, _P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _P, _P, _P, _I, _I,
                                  _I, _I, _F, _P, _S, _P]),
    "gdn_chunk_prefill_segmented_workspace_bytes": (_S, [_I, _I, _I, _I, _I, _I, _I]),
    "gdn_chunk_prefill_segmented": (_I, [_P, _P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _P, _P, _P,
                                         _I, _I, _I, _I, _F, _I, _I, _P, _S, _P]),
    "gdn_stash_seq_floats": (_I, [_I, _I, _I]),
    "gdn_verify_woa": (_I, [_P, _P, _P, _I, _P, _I, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I,
                            _F, _P, _P]),
    "gdn_verify_woa_static": (_I, [_P, _P, _P, _I, _P, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                                   _F, _P, _P, _P]),
    "gdn_verify_parent": (_I, [_P, _P, _P, _I, _P, _I, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I,
                               _I, _F, _P]),
    "gdn_fold": (_I, [_P, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "gdn_flag_clear": (_I, [_P, _P]),
    "gdn_debug_device_errors": (_I, [_P]),
    "gdn_debug_set_spin_limit": (_I, [ctypes.c_longlong]),
}

_lock = threading.Lock()
_lib = None


class GdnError(RuntimeError):
    """A libgdn entry point refused the call (named guard in the message)."""

    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} -> {ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libgdn.so and bind every declared symbol (raises if absent)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise ImportError(
                f"{p} is missing: build it with `python -m linear_attention_ssm_gdn_b200.build`")
        lib = ctypes.CDLL(p)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)  # AttributeError if a declared symbol is not exported
            f.restype = res
            f.argtypes = args
        if path is None:
            _lib = lib
        return lib


def check(fn: str, rc: int) -> None:
    if rc != GDN_OK:
        raise GdnError(fn, rc, load().gdn_last_error().decode())
