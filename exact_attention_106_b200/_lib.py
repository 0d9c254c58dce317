"""ctypes binding to the C ABI of ``libexattn.so`` (declared in include/exattn.h).

Argument marshalling only.  Loading fails loudly if the library has not been
built: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libexattn.so")

ATTN_OK = 0
ATTN_ERR_INVALID = 1
ATTN_ERR_UNSUPPORTED_DEVICE = 2
ATTN_ERR_LAUNCH = 3
ATTN_ERR_TIMEOUT = 4

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

# name -> (restype, argtypes); one entry per function of include/exattn.h
SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_bwd_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "attn_bwd_preprocess": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "attn_bwd_dkdv": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "attn_bwd_dq_convert": (_i, [_vp, _i, _i, _i, _i, _f, _vp, _sz, _vp]),
    "attn_fwd_fp8": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _f, _f, _f, _vp]),
    "attn_fwd_kvsplit": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _sz, _vp]),
    "attn_fwd_kvsplit_fp16": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _sz, _vp]),
    "attn_fwd_kvsplit_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "attn_fwd_kvsplit_count": (_i, [_i, _i, _i, _i, _i, _i, _i]),
    "attn_fwd_fp16": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_bwd_fp16": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]),
    "attn_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_fwd_bwd_host": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _sz, _i,
                               _vp]),
    "attn_fwd_bwd_host_buffer_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "attn_set_wait_timeout_ns": (None, [ctypes.c_ulonglong]),
    "attn_debug_inject_stall": (None, [_i]),
    "attn_get_device_status": (_i, [_vp]),
    "attn_status_string": (ctypes.c_char_p, [_i]),
}

_lib = None


class ExattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(
                f"exattn CUDA library not built ({path} missing); run "
                "`python -m exact_attention_106_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        env = os.environ.get("EXATTN_WAIT_TIMEOUT_NS")
        if env:  # the limit of every device-side wait, in ns (a malformed value raises ValueError)
            ns = int(env)
            if ns < 0:
                raise ValueError("EXATTN_WAIT_TIMEOUT_NS must be >= 0")
            lib.attn_set_wait_timeout_ns(ns)
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().attn_status_string(status).decode()


def check(fn: str, status: int) -> None:
    if status != ATTN_OK:
        raise ExattnError(fn, status)
