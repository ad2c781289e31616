"""ctypes binding of libmoe.so (the C ABI declared in include/moe.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  If libmoe.so is missing this module raises; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe.so")

# moe_status_t / moe_dtype_t values (include/moe.h)
MOE_OK = 0
MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = 1, 2, 3, 4
MOE_F32, MOE_F16, MOE_BF16, MOE_FP8_E4M3 = 0, 1, 2, 3
MOE_I32, MOE_I64 = 0, 1
MAX_EXPERTS = 1024
FUSED_MAX_SLOTS = 4096
EP_MAX_GROUPS = 8192

# every symbol include/moe.h declares
EXPORTED = (
    "moe_status_string",
    "moe_version",
    "moe_last_cuda_error",
    "moe_prepare_workspace_bytes",
    "moe_prepare",
    "moe_dispatch_rows",
    "moe_dispatch_error",
    "moe_set_wait_limits",
    "moe_dispatch_rows_fp8",
    "moe_dispatch_rows_nvfp4",
    "moe_combine",
    "moe_prepare_dispatch",
    "moe_prepare_no_alloc",
    "moe_problem_sizes",
    "moe_tile_layout",
    "moe_prepare_local",
    "moe_output_memset",
    "moe_ep_recv_layout",
    "moe_ep_peer_layout",
    "moe_ep_dispatch_peer",
    "moe_ep_combine_peer",
)

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_int = ctypes.c_int

_SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_int]),
    "moe_version": (_i32, []),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_prepare_workspace_bytes": (ctypes.c_size_t, [_i64, _i32, _i32]),
    "moe_prepare": (_int, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp,
                           ctypes.c_size_t, _vp]),
    "moe_dispatch_rows": (_int, [_vp, _int, _i64, _i64, _i32, _vp, _vp, _vp, _vp]),
    "moe_dispatch_error": (_int, [_vp, _vp]),
    "moe_set_wait_limits": (_int, [_i64, _i64]),
    "moe_dispatch_rows_fp8": (_int, [_vp, _int, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp,
                                     _vp, _vp]),
    "moe_dispatch_rows_nvfp4": (_int, [_vp, _int, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp,
                                       _vp, _vp]),
    "moe_combine": (_int, [_vp, _int, _i64, _i64, _i32, _vp, _vp, _vp, _int, _vp]),
    "moe_prepare_dispatch": (_int, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp,
                                    _vp, _int, _i64, _vp, _vp]),
    "moe_prepare_no_alloc": (_int, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp,
                                    _vp]),
    "moe_problem_sizes": (_int, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_tile_layout": (_int, [_i64, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp,
                               _vp, _vp, _vp, _vp, _vp]),
    "moe_prepare_local": (_int, [_vp, _int, _i64, _i32, _i64, _i32, _vp, _vp, _vp, _i32, _vp,
                                 _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "moe_output_memset": (_int, [_vp, _int, _i64, _i64, _i32, _vp, _vp]),
    "moe_ep_recv_layout": (_int, [_vp, _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_ep_peer_layout": (_int, [_vp, _i32, _i32, _i32, _vp, _i64, _i32, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _vp]),
    "moe_ep_dispatch_peer": (_int, [_vp, _int, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _i32, _vp]),
    "moe_ep_combine_peer": (_int, [_vp, _vp, _i32, _int, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _int,
                                   _vp]),
}

_lib = None


class MoeError(RuntimeError):
    """A libmoe call returned a status other than MOE_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn}: {status_string(status)}"
        if status == MOE_ERR_CUDA:
            msg += f" ({load().moe_last_cuda_error().decode()})"
        super().__init__(msg)


def load():
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build the CUDA library first "
            "(python -m combine_permute_b200.build); there is no non-CUDA fallback")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def check(fn: str, status: int):
    if status != MOE_OK:
        raise MoeError(fn, status)
