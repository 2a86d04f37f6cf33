"""ctypes declarations of the C ABI in include/sfn.h (libsfn.so, built in-tree).

There is no fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsfn.so")

SFN_OK = 0
SFN_ERR_INVALID_VALUE = 1
SFN_ERR_MISALIGNED = 2
SFN_ERR_UNSUPPORTED = 3
SFN_ERR_WORKSPACE = 4
SFN_ERR_CUDA = 5

SFN_PATH_AUTO = 0
SFN_PATH_CUDA_CORE = 1
SFN_PATH_TENSOR = 2

SFN_DTYPE_BF16 = 0
SFN_DTYPE_F32 = 1

# Every function declared in include/sfn.h, with (restype, argtypes).
_vp, _i64, _ci, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_FWD = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _ci, _ci, _ci, _ci, _ci]
SIGNATURES = {
    "sfn_status_string": (ctypes.c_char_p, [_ci]),
    "sfn_abi_version": (_ci, []),
    "sfn_last_error_string": (ctypes.c_char_p, []),
    "sfn_kernel_launch_count": (ctypes.c_uint64, []),
    "sfn_predict": (_ci, [_vp, _vp, _vp, _vp, _i64, _ci, _ci, _ci, _vp]),
    "sfn_predict_f32": (_ci, [_vp, _vp, _vp, _vp, _i64, _ci, _ci, _ci, _vp]),
    "sfn_bank_topk": (_ci, [_vp, _vp, _i64, _ci, _ci, _ci, _vp]),
    "sfn_workspace_bytes": (_sz, [_i64, _ci, _ci, _ci, _ci, _ci, _ci]),
    "sfn_sparse_ffn_forward": (_ci, _FWD + [_vp]),
    "sfn_sparse_ffn_forward_ws": (_ci, _FWD + [_vp, _sz, _vp]),
    "sfn_sparse_ffn_forward_static": (_ci, _FWD + [_vp]),
    "sfn_sparse_ffn_forward_path": (_ci, _FWD + [_ci, _vp, _sz, _vp]),
    "sfn_sparse_ffn_forward_partial": (_ci, _FWD + [_ci, _vp, _sz, _vp]),
    "sfn_sparse_ffn_forward_f32": (_ci, _FWD + [_vp]),
    "sfn_sparse_ffn_forward_f32_ws": (_ci, _FWD + [_vp, _sz, _vp]),
    "sfn_dense4x_workspace_bytes": (_sz, [_i64, _ci, _ci, _ci, _ci]),
    "sfn_dense4x_forward": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _ci, _ci, _ci, _ci, _vp,
                                  _sz, _vp]),
    "sfn_backward_workspace_bytes": (_sz, [_i64, _ci, _ci, _ci, _ci, _ci]),
    "sfn_sparse_ffn_backward": (_ci, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp,
                                      _vp, _vp, _vp, _vp, _vp, _i64, _ci, _ci, _ci, _ci, _ci,
                                      _vp, _sz, _vp]),
    "sfn_timing_begin": (_ci, []),
    "sfn_device_errors": (_ci, [_vp, _ci]),
    "sfn_debug_wait_timeout": (_ci, [ctypes.c_longlong, _vp, _vp]),
    "sfn_timing_end": (_ci, [_vp, _vp, _ci]),
    "sfn_stage_name": (ctypes.c_char_p, [_ci]),
}
SFN_STAGE_COUNT = 16
SFN_STATIC_SCRATCH_BYTES = 16 << 20

_lib = None
_lock = threading.Lock()


class SfnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status in (SFN_ERR_CUDA, SFN_ERR_UNSUPPORTED):
            msg += f" ({lib().sfn_last_error_string().decode()})"
        super().__init__(msg)


def lib():
    """The loaded libsfn.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libsfn.so not found at {LIB_PATH}; build it with "
                    "`python -m predictor_gated_channel_b200.build` (there is no fallback)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
        return _lib


def status_string(status: int) -> str:
    return lib().sfn_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != SFN_OK:
        raise SfnError(status, where)
