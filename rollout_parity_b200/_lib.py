"""ctypes view of librn's C ABI (include/rn.h).  Loading fails loudly if the
library has not been built: there is no other implementation to fall back to."""
from __future__ import annotations

import ctypes
import enum
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librn.so")

c_i64, c_i32, c_f32, c_sz, c_vp = (ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                   ctypes.c_size_t, ctypes.c_void_p)


class Status(enum.IntEnum):
    OK = 0
    E_ARG = 1
    E_DTYPE = 2
    E_WIDTH = 3
    E_ALIGN = 4
    E_WORKSPACE = 5
    E_CUDA = 6


class DType(enum.IntEnum):
    F32 = 0
    BF16 = 1
    F16 = 2


class Act(enum.IntEnum):
    NONE = 0
    SILU = 1
    SIGMOID = 2


class RNError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str, cuda_err: int = 0):
        self.status = Status(status)
        self.cuda_error = cuda_err
        super().__init__(f"{fn}: {self.status.name} ({msg})"
                         + (f", cudaError {cuda_err}" if cuda_err else ""))


# name -> (restype, argtypes); the same set include/rn.h declares
SIGNATURES = {
    "rmsnorm_fwd": (c_i32, [c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp,
                            c_vp, c_vp]),
    "rmsnorm_bwd": (c_i32, [c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp,
                            c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "rmsnorm_add_fwd": (c_i32, [c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp,
                                c_vp, c_vp, c_vp, c_vp]),
    "rmsnorm_add_bwd": (c_i32, [c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp,
                                c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "norm_fwd": (c_i32, [c_i64, c_i32, c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "gated_norm_fwd": (c_i32, [c_i64, c_i32, c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "norm_bwd_workspace_bytes": (c_sz, [c_i64, c_i32]),
    "norm_bwd": (c_i32, [c_i64, c_i32, c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                         c_vp, c_sz, c_vp]),
    "gated_norm_bwd": (c_i32, [c_i64, c_i32, c_f32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                               c_vp, c_vp, c_vp, c_sz, c_vp]),
    "gated_norm_bwd_static_ws": (c_i32, [c_i64, c_i32, c_f32, c_i32, c_vp, c_vp, c_vp, c_vp,
                                         c_vp, c_vp, c_vp, c_vp, c_vp]),
    "rmsnorm_bwd_chunk_count": (c_i64, [c_i64]),
    "rmsnorm_bwd_chunks": (c_i32, [c_i64, c_i32, c_f32, c_f32, c_i32, c_i32, c_vp, c_vp, c_vp,
                                   c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "rn_fold_tree_workspace_bytes": (c_sz, [c_i64, c_i32]),
    "rn_fold_tree": (c_i32, [c_i64, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "rn_fold_rows": (c_i32, [c_i64, c_i32, c_vp, c_vp, c_vp]),
    "rn_describe": (ctypes.c_char_p, [c_i32, c_i32]),
    "rn_bwd_launches": (c_i32, [c_i64, c_i32, c_i32]),
    "rn_status_string": (ctypes.c_char_p, [c_i32]),
    "rn_last_cuda_error": (ctypes.c_int, []),
    "rn_last_launches": (c_i32, []),
    "rn_test_set_geometry": (c_i32, [c_i32, c_i32, c_i32]),
    "rn_test_set_validate_only": (None, [c_i32]),
    "rn_test_rcp_1to2": (c_i32, [c_i64, c_vp, c_vp, c_i32, c_vp]),
    "rn_test_sigmoid": (c_i32, [c_i64, c_vp, c_vp, c_vp]),
}

_lib = None
_lock = threading.Lock()


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librn.so once (thread-safe) and attach the signatures."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"librn.so not found at {path}; build it with `python -m rollout_parity_b200.build` "
                "(there is no CPU or Python fallback)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def check(fn: str, status: int) -> None:
    if status != Status.OK:
        lib = load()
        msg = lib.rn_status_string(status).decode()
        raise RNError(fn, status, msg, lib.rn_last_cuda_error() if status == Status.E_CUDA else 0)
