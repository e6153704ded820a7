"""ctypes loader for libkda_b200.so: argument types and status handling only."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda_b200.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(5)
KDA_F32, KDA_BF16 = 0, 1

# every symbol include/kda.h declares
EXPORTED = ("kda_chunk_fwd", "kda_chunk_fwd_workspace_size", "kda_chunk_fwd_static_ws", "kda_recurrent_fwd",
            "kda_decode_step", "gdn_chunk_fwd", "gdn_recurrent_fwd", "gdn_decode_step", "kda_chunk_fwd_fused",
            "kda_decode_step_fused", "kda_status_string", "kda_get_last_device_error", "kda_version",
            "kda_testing_set_chunk_fault", "kda_chunk_bwd", "kda_chunk_bwd_workspace_size")

_lib = None


class KdaError(RuntimeError):
    """A kda_* call returned a non-OK status."""

    def __init__(self, status: int, call: str):
        self.status = status
        name = status_string(status) if _lib is not None else str(status)
        super().__init__(f"{call} failed: {name}")


def load() -> ctypes.CDLL:
    """Load the in-tree library.  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with gated_delta_rule_86_b200.build.build_library()"
                          " (or __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32p = ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p
    prefill_args = [vp, vp, vp, vp, vp, f32p, vp, i32, i32, i32, i32, i32, i32]
    for name in ("kda_chunk_fwd", "gdn_chunk_fwd", "kda_chunk_fwd_fused"):
        fn = getattr(lib, name)
        fn.argtypes = prefill_args + [i32, ctypes.c_int, ctypes.c_int, vp, f32p, vp, ctypes.c_size_t, vp]
        fn.restype = ctypes.c_int
    lib.kda_chunk_fwd_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_chunk_fwd_workspace_size.restype = ctypes.c_int
    for name in ("kda_recurrent_fwd", "gdn_recurrent_fwd"):
        fn = getattr(lib, name)
        fn.argtypes = prefill_args + [ctypes.c_int, ctypes.c_int, vp, f32p, vp]
        fn.restype = ctypes.c_int
    for name in ("kda_decode_step", "gdn_decode_step", "kda_decode_step_fused"):
        fn = getattr(lib, name)
        fn.argtypes = [vp, vp, vp, vp, vp, f32p, vp, i32, i32, i32, i32, ctypes.c_int, ctypes.c_int, vp]
        fn.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_get_last_device_error.argtypes = [vp]
    lib.kda_get_last_device_error.restype = ctypes.c_int
    lib.kda_version.argtypes = []
    lib.kda_version.restype = ctypes.c_char_p
    lib.kda_testing_set_chunk_fault.argtypes = [i32, ctypes.c_uint32]
    lib.kda_testing_set_chunk_fault.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = prefill_args + [i32, ctypes.c_int, vp, ctypes.c_int, f32p] + [f32p] * 6 + \
        [vp, ctypes.c_size_t, vp]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_chunk_bwd_workspace_size.argtypes = [i32, i32, ctypes.c_int64, i32, i32, i32,
                                                 ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_chunk_bwd_workspace_size.restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def check(status: int, call: str) -> None:
    if status != KDA_OK:
        raise KdaError(status, call)
