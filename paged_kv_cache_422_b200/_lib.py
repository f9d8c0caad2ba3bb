"""ctypes view of libnvpa.so: the C ABI declared in include/nvpa.h, with the same names.

Loading fails loudly when the library has not been built; there is no other
implementation to fall back to.
"""

from __future__ import annotations

import ctypes
import os

# NVPA_LIB names another build of the same library (a variant built with
# `python -m paged_kv_cache_422_b200.build --out PATH`).
LIB_PATH = os.environ.get("NVPA_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                       "libnvpa.so")

NVPA_OK = 0
NVPA_ERR_INVALID_ARG = 1
NVPA_ERR_UNSUPPORTED = 2
NVPA_ERR_CUDA = 3
NVPA_ERR_WORKSPACE_TOO_SMALL = 4

NVPA_FLAG_BAD_SLOT = 1
NVPA_FLAG_BAD_BLOCK_ID = 2
NVPA_FLAG_BAD_LENGTH = 4
NVPA_FLAG_TIMEOUT = 8

# Every function the header declares, with (restype, argtypes).
_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_sz = ctypes.c_size_t
SIGNATURES = {
    "nvpa_version": (_i, []),
    "nvpa_status_string": (ctypes.c_char_p, [_i]),
    "nvpa_last_error": (ctypes.c_char_p, []),
    "nvpa_kernel_launch_count": (ctypes.c_uint64, []),
    "nvpa_store_kvcache": (_i, [_p, _p, _i64, _i64, _p, _p, _p, _i, _i, _i, _i, _i, _p, _p]),
    "nvpa_paged_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "nvpa_paged_decode_attention": (_i, [_p, _p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i,
                                         _i, _f, _i, _p, _sz, _p, _p]),
    "nvpa_decode_step": (_i, [_p, _p, _p, _p, _p, _i64, _i64, _p, _p, _p, _p, _i, _p, _i, _i, _i,
                              _i, _i, _i, _i, _f, _i, _p, _sz, _p, _p]),
    "nvpa_decode_shared_prefix_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "nvpa_decode_step_shared_prefix": (_i, [_p, _p, _p, _p, _p, _i64, _i64, _p, _p, _p, _p, _i, _p,
                                            _i, _i, _i, _i, _i, _i, _i, _f, _i, _i, _p, _sz, _p,
                                            _p]),
    "nvpa_paged_decode_attention_static_scratch": (_i, [_p, _p, _p, _p, _p, _p, _i, _p, _i, _i,
                                                        _i, _i, _i, _i, _i, _f, _i, _p, _p]),
    "nvpa_paged_decode_partial": (_i, [_p, _p, _p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i,
                                       _f, _i, _p, _sz, _p, _p]),
    "nvpa_lse_combine": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _p]),
    "nvpa_varlen_prefill_workspace_size": (_sz, [_i, _i]),
    "nvpa_varlen_prefill_attention": (_i, [_p, _p, _p, _p, _p, _p, _i, _p, _p, _i, _i, _i, _i,
                                           _i, _i, _i, _i, _i, _f, _i, _p, _sz, _p, _p]),
    "nvpa_gather_kv": (_i, [_p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _p, _p]),
    "nvpa_check_bounded_wait": (_i, [_p, _p]),
}


class NvpaError(RuntimeError):
    def __init__(self, status: int, func: str, detail: str):
        self.status = status
        super().__init__(f"{func} failed with status {status}: {detail}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is not built; run `python -m paged_kv_cache_422_b200.build` "
                "(nvcc, sm_100a)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status: int, func: str) -> None:
    if status != NVPA_OK:
        detail = lib().nvpa_last_error().decode(errors="replace")
        raise NvpaError(status, func, detail)
